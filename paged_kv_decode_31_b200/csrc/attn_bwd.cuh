// attn_bwd.cuh -- deterministic backward of paged prefill attention, sm_100a.
//
// The training-side backward over the same forward graph (RL-Kernel PR #284
// "feat(attention): add CP backward drift validation", Changes: a backward
// reference over the saved forward, dq / dk / dv, fixed merge order, fp32
// accumulation).  With p_ij = 2^(s_ij * c - lse2_i) (c = scale * log2 e,
// lse2 = lse * log2 e from the forward), D_i = dout_i . out_i:
//   ds_ij = p_ij (dout_i . v_j - D_i)
//   dq_i = scale * sum_j ds_ij k_j,  dk_j = scale * sum_i ds_ij q_i,
//   dv_j = sum_i p_ij dout_i
// where i runs over the query rows r = i * G + g of the KV head.  No atomics:
//   bwd_kv_kernel   one CTA per (sequence, KV head, 128-key tile): S^T = K Q^T
//                   and dP^T = V dO^T on the tensor cores (keys on M), P^T and
//                   dS^T to shared memory as bf16, dV += P^T dO and dK += dS^T Q
//                   accumulated in TMEM over the 128-row tiles in ascending
//                   order, then written once;
//   bwd_q_kernel    one CTA per (sequence, KV head, 128-row tile): S = Q K^T,
//                   dP = dO V^T (rows on M), dS to shared memory, dQ += dS K
//                   accumulated over the key tiles in ascending order.
// Every sum therefore has one fixed order and the result is bitwise
// reproducible and independent of the batch around a sequence.
//
// 544 threads: warps 0-15 stage operands and do the elementwise work -- warps
// w, w + 4, w + 8, w + 12 share TMEM lanes 32 (w % 4) .. + 31 (thread t = lane
// t of the 128) and split the columns in quarters -- and warp 16 owns TMEM,
// its lane 0 issuing the MMAs.  Phases are separated by __syncthreads and
// MMA-completion mbarriers (bounded waits).
#pragma once

#include <cuda_bf16.h>

#include "attn_split.cuh"
#include "ptx.cuh"

namespace pkv {

constexpr int kBwdCompute = 512;               // staging / elementwise threads
constexpr int kBwdGroups = kBwdCompute / 128;  // column groups per TMEM lane
constexpr int kBwdThreads = kBwdCompute + 32;
constexpr int kBwdMmaWarp = kBwdCompute / 32;
constexpr int kBwdTile = 128;  // keys per key tile and rows per row tile

struct BwdParams {
  const __nv_bfloat16 *q, *dout;
  int64_t q_sb, q_ss, q_sh, g_sb, g_ss, g_sh;  // element strides (batch, token, head)
  const __nv_bfloat16 *k_cache, *v_cache;
  int64_t k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
  __nv_bfloat16 *dk_cache, *dv_cache;          // gradients, laid out like the caches
  int64_t dk_sb, dk_ss, dk_sh, dv_sb, dv_ss, dv_sh;
  __nv_bfloat16 *dq;
  int64_t dq_sb, dq_ss, dq_sh;
  const int32_t *block_table;
  int64_t bt_stride;
  int max_blocks_per_seq;
  int64_t num_blocks;
  const int32_t *seqlens;
  int batch, seqlen_q, Hq, Hkv, G, block_shift, causal;
  int n_key_tiles, n_row_tiles;
  float cscale, scale;
  const float *row_d;     // [rows] dout . out
  const float *row_lse2;  // [rows] lse * log2 e
  int32_t *err;
};

// Per-row statistics: D = dout . out (fp32, fixed lane order and shuffle
// tree) and lse in base-2 units.  One warp per row (b, i, h).
struct BwdPrepParams {
  const __nv_bfloat16 *dout, *out;
  int64_t g_sb, g_ss, g_sh, o_sb, o_ss, o_sh;
  const float *lse;  // [batch, Hq, seqlen_q]
  int batch, seqlen_q, Hq, D;
  float *row_d, *row_lse2;
  // a context longer than max_seqlen_k (the host bound that sized the key
  // tiles; keys past it are not read) is flagged once per sequence
  const int32_t *seqlens;
  int max_seqlen_k;
  int32_t *err;
};

__global__ void __launch_bounds__(256) bwd_prep_kernel(const __grid_constant__ BwdPrepParams p) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(p.batch) * p.seqlen_q * p.Hq;
  if (row >= rows) return;
  const int h = static_cast<int>(row % p.Hq);
  const int64_t bi = row / p.Hq;
  const int i = static_cast<int>(bi % p.seqlen_q);
  const int b = static_cast<int>(bi / p.seqlen_q);
  const __nv_bfloat16 *g = p.dout + b * p.g_sb + i * p.g_ss + h * p.g_sh;
  const __nv_bfloat16 *o = p.out + b * p.o_sb + i * p.o_ss + h * p.o_sh;
  // lane l: elements [l V, l V + V), V = D / 32, summed in order, then a
  // fixed xor tree over the lanes
  float acc = 0.f;
  if (p.D == 128) {  // 8-byte loads: 4 elements per lane
    const uint2 gv = *reinterpret_cast<const uint2 *>(g + lane * 4);
    const uint2 ov = *reinterpret_cast<const uint2 *>(o + lane * 4);
    const __nv_bfloat162 *g2 = reinterpret_cast<const __nv_bfloat162 *>(&gv);
    const __nv_bfloat162 *o2 = reinterpret_cast<const __nv_bfloat162 *>(&ov);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      acc = __fmaf_rn(__low2float(g2[e]), __low2float(o2[e]), acc);
      acc = __fmaf_rn(__high2float(g2[e]), __high2float(o2[e]), acc);
    }
  } else {  // D = 64: 4-byte loads, 2 elements per lane
    const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162 *>(g + lane * 2);
    const __nv_bfloat162 o2 = *reinterpret_cast<const __nv_bfloat162 *>(o + lane * 2);
    acc = __fmaf_rn(__low2float(g2), __low2float(o2), acc);
    acc = __fmaf_rn(__high2float(g2), __high2float(o2), acc);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
  if (lane == 0) {
    if (h == 0 && i == 0 && p.err && __ldg(p.seqlens + b) > p.max_seqlen_k)
      atomicOr(p.err, kErrSeqLen);
    p.row_d[row] = acc;
    const float l = p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.seqlen_q + i];
    p.row_lse2[row] = __fmul_rn(l, 1.4426950408889634f);
  }
}

template <int D>
struct BwdCfg {
  static constexpr int kHalf = kBwdTile * 128;          // 128 rows x 64 elements x bf16
  static constexpr int kTile = (D / 64) * kHalf;        // a [128][D] operand
  static constexpr int kSq = 2 * kHalf;                 // a [128][128] operand
  struct Small {
    uint64_t mma_a, mma_b, drain;
    uint32_t tmem_base;
    int abort_any;
    int lim[kBwdTile];       // key limit of each row of the current row tile
    float lse2[kBwdTile];
    float dsum[kBwdTile];
  };
};

// Stage [128][D] bf16 tiles, rows given by `src_row(c)` (nullptr: zeros),
// 128-byte swizzled K-major (row c at c * 128 bytes of its 64-element half).
// Every load of a thread is issued before its first store, so the tile costs
// about one memory round trip.
template <int D, class F>
__device__ __forceinline__ void stage_rows(uint8_t *dst, int t, F src_row) {
  constexpr int kPer = kBwdTile * (D / 8) / kBwdCompute;  // 16-byte chunks per thread
  uint4 v[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int idx = t + k * kBwdCompute;
    const int c = idx / (D / 8), ch = idx % (D / 8);
    const __nv_bfloat16 *s = src_row(c);
    v[k] = s ? __ldg(reinterpret_cast<const uint4 *>(s) + ch) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int idx = t + k * kBwdCompute;
    const int c = idx / (D / 8), ch = idx % (D / 8);
    const int h = ch >> 3, cc = ch & 7;
    *reinterpret_cast<uint4 *>(dst + h * BwdCfg<D>::kHalf + c * 128 + ((cc ^ (c & 7)) << 4)) = v[k];
  }
}

// Eight bf16 (one 16-byte chunk) into row `row` of a [128][128] K-major
// swizzled operand, columns [col8 * 8, col8 * 8 + 8).
__device__ __forceinline__ void put8(uint8_t *dst, int row, int col8, uint4 v) {
  const int h = col8 >> 3, cc = col8 & 7;
  *reinterpret_cast<uint4 *>(dst + h * (kBwdTile * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = v;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h2);
}

// Key limit of row r of row tile rt (0 for padded rows).
__device__ __forceinline__ int bwd_row_lim(const BwdParams &p, int seqlen, int r) {
  if (r >= p.G * p.seqlen_q) return 0;
  const int i = r / p.G;
  int lim = seqlen;
  if (p.causal) lim = min(lim, seqlen - p.seqlen_q + i + 1);
  return lim > 0 ? lim : 0;
}

// Cache row of token `tok` of sequence b (nullptr past the table or the
// cache, with the error bits set as in the forward).
__device__ __forceinline__ int64_t bwd_block(const BwdParams &p, int b, int tok) {
  const int col = tok >> p.block_shift;
  if (col >= p.max_blocks_per_seq) {
    if (p.err) atomicOr(p.err, kErrTableWidth);
    return -1;
  }
  const int blk = __ldg(p.block_table + b * p.bt_stride + col);
  if (blk < 0 || static_cast<int64_t>(blk) >= p.num_blocks) {
    if (p.err) atomicOr(p.err, kErrBadBlock);
    return -1;
  }
  return blk;
}

// Issue D[tmem] = A[128 x K] * B^T for two K-major [128][K] operands.
template <int K>
__device__ __forceinline__ void mma_kk(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < K / 16; ++kk) {
    const int h = kk >> 2, off = (kk & 3) * 32;
    umma_bf16(d, smem_desc(a + h * (kBwdTile * 128) + off, 16, 1024, kLayoutSw128),
              smem_desc(b + h * (kBwdTile * 128) + off, 16, 1024, kLayoutSw128), idesc,
              kk > 0 ? 1u : 0u);
  }
}

// Issue D[tmem] (+)= A[128 x 128] * B[128 x N], A K-major, B MN-major (a
// [128][N] tile read along its rows).
template <int N>
__device__ __forceinline__ void mma_kn(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc,
                                       bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < kBwdTile / 16; ++kk) {
    const int h = kk >> 2, off = (kk & 3) * 32;
    umma_bf16(d, smem_desc(a + h * (kBwdTile * 128) + off, 16, 1024, kLayoutSw128),
              smem_desc(b + kk * 2048, kBwdTile * 128, 1024, kLayoutSw128), idesc,
              (accumulate || kk > 0) ? 1u : 0u);
  }
}

// ---------------------------------------------------------------------------
// dK / dV: one CTA per (b, kvh, key tile).
// smem: K, V, Q, dO tiles ([128][D]), P^T and dS^T ([128 keys][128 rows]).
// TMEM: S^T [0,128), dP^T [128,256), dV [256, 256 + D), dK [256 + D, 256 + 2D).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kv_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sK = smem, *sV = sK + C::kTile, *sQ = sV + C::kTile, *sG = sQ + C::kTile;
  uint8_t *sP = sG + C::kTile, *sS = sP + C::kSq;
  auto *sm = reinterpret_cast<typename C::Small *>(sS + C::kSq);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int t = tid & 127, hf = tid >> 7;  // TMEM lane / token, column group (compute threads)
  volatile int *abort_any = &sm->abort_any;

  int u = blockIdx.x;
  const int kt = u % p.n_key_tiles;
  u /= p.n_key_tiles;
  const int kvh = u % p.Hkv;
  const int b = u / p.Hkv;
  const int seqlen = max(__ldg(p.seqlens + b), 0);
  const int tok0 = kt * kBwdTile;
  if (tok0 >= seqlen) return;  // uniform: the whole CTA leaves before any barrier

  if (tid == 0) {
    mbar_init(&sm->mma_a, 1);
    mbar_init(&sm->mma_b, 1);
    mbar_init(&sm->drain, 1);
    sm->abort_any = 0;
    fence_barrier_init();
  }
  if (warp == kBwdMmaWarp) tmem_alloc(&sm->tmem_base, 512);
  // K and V of this key tile (tokens past the context are zeros)
  if (tid < kBwdCompute) {
    stage_rows<D>(sK, tid, [&](int c) -> const __nv_bfloat16 * {
      const int tok = tok0 + c;
      if (tok >= seqlen) return nullptr;
      const int64_t blk = bwd_block(p, b, tok);
      if (blk < 0) return nullptr;
      return p.k_cache + blk * p.k_sb + (tok & ((1 << p.block_shift) - 1)) * p.k_ss + kvh * p.k_sh;
    });
    stage_rows<D>(sV, tid, [&](int c) -> const __nv_bfloat16 * {
      const int tok = tok0 + c;
      if (tok >= seqlen) return nullptr;
      const int64_t blk = bwd_block(p, b, tok);
      if (blk < 0) return nullptr;
      return p.v_cache + blk * p.v_sb + (tok & ((1 << p.block_shift) - 1)) * p.v_ss + kvh * p.v_sh;
    });
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t aK = sbase, aV = aK + C::kTile, aQ = aV + C::kTile, aG = aQ + C::kTile;
  const uint32_t aP = aG + C::kTile, aS = aP + C::kSq;
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const float NEG_INF = neg_inf();
  const int R = p.G * p.seqlen_q;

  // first row tile with a row that sees key tok0: rows r with i >= tok0 - (seqlen - sq)
  int rt0 = 0;
  if (p.causal) {
    const int i_min = tok0 - (seqlen - p.seqlen_q);
    rt0 = i_min > 0 ? (i_min * p.G) / kBwdTile : 0;
  }
  int it = 0;
  for (int rt = rt0; rt * kBwdTile < R; ++rt, ++it) {
    const int row0 = rt * kBwdTile;
    if (tid < kBwdCompute) {
      auto rowptr = [&](const __nv_bfloat16 *base, int64_t sb, int64_t ss, int64_t sh, int c)
          -> const __nv_bfloat16 * {
        const int r = row0 + c;
        if (r >= R) return nullptr;
        const int i = r / p.G, g = r - i * p.G;
        return base + b * sb + static_cast<int64_t>(i) * ss + static_cast<int64_t>(kvh * p.G + g) * sh;
      };
      stage_rows<D>(sQ, tid, [&](int c) { return rowptr(p.q, p.q_sb, p.q_ss, p.q_sh, c); });
      stage_rows<D>(sG, tid, [&](int c) { return rowptr(p.dout, p.g_sb, p.g_ss, p.g_sh, c); });
      if (hf == 0) {
        const int r = row0 + t;
        sm->lim[t] = bwd_row_lim(p, seqlen, r);
        float l2 = 0.f, ds = 0.f;
        if (r < R) {
          const int i = r / p.G, g = r - i * p.G;
          const int64_t row_id = (static_cast<int64_t>(b) * p.seqlen_q + i) * p.Hq + kvh * p.G + g;
          l2 = p.row_lse2[row_id];
          ds = p.row_d[row_id];
        }
        sm->lse2[t] = l2;
        sm->dsum[t] = ds;
      }
      fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (*abort_any) break;
    if (warp == kBwdMmaWarp && lane == 0) {
      tc_fence_after_sync();
      constexpr uint32_t kId = idesc_bf16(128, 128, 0, 0);
      mma_kk<D>(tS, aK, aQ, kId);   // S^T = K Q^T
      mma_kk<D>(tdP, aV, aG, kId);  // dP^T = V dO^T
      umma_commit(&sm->mma_a);
    }
    if (tid < kBwdCompute) {
      mbar_wait(&sm->mma_a, it & 1, abort_any);
      __syncwarp();
      tc_fence_after_sync();
      const int tok = tok0 + t;
#pragma unroll 1
      for (int ch = hf * (8 / kBwdGroups); ch < (hf + 1) * (8 / kBwdGroups); ++ch) {  // its rows
        float sv[16], dp[16];
        tmem_ld16(tS + lane_off + ch * 16, sv);
        tmem_ld16(tdP + lane_off + ch * 16, dp);
        tmem_ld_wait_for(sv);
        tmem_ld_wait_for(dp);
        uint32_t pw[8], sw[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float pv[2], dv[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int c = ch * 16 + e + k;
            const bool vis = tok < sm->lim[c];
            const float pr = vis ? ex2(__fsub_rn(__fmul_rn(sv[e + k], p.cscale), sm->lse2[c])) : 0.f;
            pv[k] = pr;
            dv[k] = __fmul_rn(pr, __fsub_rn(dp[e + k], sm->dsum[c]));
          }
          pw[e / 2] = pack_bf16(pv[0], pv[1]);
          sw[e / 2] = pack_bf16(dv[0], dv[1]);
        }
        put8(sP, t, ch * 2, make_uint4(pw[0], pw[1], pw[2], pw[3]));
        put8(sP, t, ch * 2 + 1, make_uint4(pw[4], pw[5], pw[6], pw[7]));
        put8(sS, t, ch * 2, make_uint4(sw[0], sw[1], sw[2], sw[3]));
        put8(sS, t, ch * 2 + 1, make_uint4(sw[4], sw[5], sw[6], sw[7]));
      }
      fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (*abort_any) break;
    if (warp == kBwdMmaWarp && lane == 0) {
      tc_fence_after_sync();
      constexpr uint32_t kId = idesc_bf16(128, D, 0, 1);
      mma_kn<D>(tdV, aP, aG, kId, it > 0);  // dV += P^T dO
      mma_kn<D>(tdK, aS, aQ, kId, it > 0);  // dK += dS^T Q
      umma_commit(&sm->mma_b);
    }
    // operands are overwritten by the next row tile only after these MMAs
    mbar_wait(&sm->mma_b, it & 1, abort_any);
    __syncwarp();
  }
  tc_fence_before_sync();
  __syncthreads();
  const bool ok = !*abort_any;
  if (tid < kBwdCompute && ok) {
    tc_fence_after_sync();
    const int tok = tok0 + t;
    int64_t blk = -1;
    if (tok < seqlen) blk = bwd_block(p, b, tok);
    const int slot = tok & ((1 << p.block_shift) - 1);
#pragma unroll 1
    for (int ch = hf * (D / 16 / kBwdGroups); ch < (hf + 1) * (D / 16 / kBwdGroups); ++ch) {  // its part of D
      float vv[16], kv[16];
      tmem_ld16(tdV + lane_off + ch * 16, vv);
      tmem_ld16(tdK + lane_off + ch * 16, kv);
      tmem_ld_wait_for(vv);
      tmem_ld_wait_for(kv);
      if (blk >= 0) {
        uint32_t wv[8], wk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          // a tile no row reached leaves zeros (it = 0: accumulators unwritten)
          const float v0 = it > 0 ? vv[2 * e] : 0.f, v1 = it > 0 ? vv[2 * e + 1] : 0.f;
          const float k0 = it > 0 ? __fmul_rn(kv[2 * e], p.scale) : 0.f;
          const float k1 = it > 0 ? __fmul_rn(kv[2 * e + 1], p.scale) : 0.f;
          wv[e] = pack_bf16(v0, v1);
          wk[e] = pack_bf16(k0, k1);
        }
        uint4 *dv = reinterpret_cast<uint4 *>(p.dv_cache + blk * p.dv_sb + slot * p.dv_ss + kvh * p.dv_sh + ch * 16);
        uint4 *dk = reinterpret_cast<uint4 *>(p.dk_cache + blk * p.dk_sb + slot * p.dk_ss + kvh * p.dk_sh + ch * 16);
        dv[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        dv[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
        dk[0] = make_uint4(wk[0], wk[1], wk[2], wk[3]);
        dk[1] = make_uint4(wk[4], wk[5], wk[6], wk[7]);
      }
    }
  }
  if (!ok && warp == kBwdMmaWarp && lane == 0) {
    umma_commit(&sm->drain);
    volatile int no_abort = 0;
    mbar_wait(&sm->drain, 0, &no_abort);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
  if (tid == 0 && !ok && p.err) atomicOr(p.err, kErrTimeout);
}

// ---------------------------------------------------------------------------
// dQ: one CTA per (b, kvh, row tile).
// smem: Q, dO, K, V tiles ([128][D]), dS ([128 rows][128 keys]).
// TMEM: S [0,128), dP [128,256), dQ [256, 256 + D).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_q_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem, *sG = sQ + C::kTile, *sK = sG + C::kTile, *sV = sK + C::kTile;
  uint8_t *sS = sV + C::kTile;
  auto *sm = reinterpret_cast<typename C::Small *>(sS + C::kSq);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int t = tid & 127, hf = tid >> 7;  // TMEM lane / row, column group (compute threads)
  volatile int *abort_any = &sm->abort_any;

  int u = blockIdx.x;
  const int rt = u % p.n_row_tiles;
  u /= p.n_row_tiles;
  const int kvh = u % p.Hkv;
  const int b = u / p.Hkv;
  const int seqlen = max(__ldg(p.seqlens + b), 0);
  const int R = p.G * p.seqlen_q;
  const int row0 = rt * kBwdTile;
  // keys [0, lim_max) cover every row of the tile
  const int lim_max = bwd_row_lim(p, seqlen, min(row0 + kBwdTile, R) - 1);

  if (tid == 0) {
    mbar_init(&sm->mma_a, 1);
    mbar_init(&sm->mma_b, 1);
    mbar_init(&sm->drain, 1);
    sm->abort_any = 0;
    fence_barrier_init();
  }
  if (warp == kBwdMmaWarp) tmem_alloc(&sm->tmem_base, 512);
  const int r_t = row0 + t;
  int my_lim = 0;
  float my_l2 = 0.f, my_d = 0.f;
  int64_t my_row = -1;
  if (tid < kBwdCompute) {
    auto rowptr = [&](const __nv_bfloat16 *base, int64_t sb, int64_t ss, int64_t sh, int c)
        -> const __nv_bfloat16 * {
      const int r = row0 + c;
      if (r >= R) return nullptr;
      const int i = r / p.G, g = r - i * p.G;
      return base + b * sb + static_cast<int64_t>(i) * ss + static_cast<int64_t>(kvh * p.G + g) * sh;
    };
    stage_rows<D>(sQ, tid, [&](int c) { return rowptr(p.q, p.q_sb, p.q_ss, p.q_sh, c); });
    stage_rows<D>(sG, tid, [&](int c) { return rowptr(p.dout, p.g_sb, p.g_ss, p.g_sh, c); });
    my_lim = bwd_row_lim(p, seqlen, r_t);
    if (r_t < R) {
      const int i = r_t / p.G, g = r_t - i * p.G;
      my_row = (static_cast<int64_t>(b) * p.seqlen_q + i) * p.Hq + kvh * p.G + g;
      my_l2 = p.row_lse2[my_row];
      my_d = p.row_d[my_row];
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t aQ = sbase, aG = aQ + C::kTile, aK = aG + C::kTile, aV = aK + C::kTile;
  const uint32_t aS = aV + C::kTile;
  const uint32_t tS = tmem, tdP = tmem + 128, tdQ = tmem + 256;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;

  const int n_kt = (lim_max + kBwdTile - 1) / kBwdTile;
  int it = 0;
  for (int kt = 0; kt < n_kt; ++kt, ++it) {
    const int tok0 = kt * kBwdTile;
    if (tid < kBwdCompute) {
      stage_rows<D>(sK, tid, [&](int c) -> const __nv_bfloat16 * {
        const int tok = tok0 + c;
        if (tok >= seqlen) return nullptr;
        const int64_t blk = bwd_block(p, b, tok);
        if (blk < 0) return nullptr;
        return p.k_cache + blk * p.k_sb + (tok & ((1 << p.block_shift) - 1)) * p.k_ss + kvh * p.k_sh;
      });
      stage_rows<D>(sV, tid, [&](int c) -> const __nv_bfloat16 * {
        const int tok = tok0 + c;
        if (tok >= seqlen) return nullptr;
        const int64_t blk = bwd_block(p, b, tok);
        if (blk < 0) return nullptr;
        return p.v_cache + blk * p.v_sb + (tok & ((1 << p.block_shift) - 1)) * p.v_ss + kvh * p.v_sh;
      });
      fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (*abort_any) break;
    if (warp == kBwdMmaWarp && lane == 0) {
      tc_fence_after_sync();
      constexpr uint32_t kId = idesc_bf16(128, 128, 0, 0);
      mma_kk<D>(tS, aQ, aK, kId);   // S = Q K^T
      mma_kk<D>(tdP, aG, aV, kId);  // dP = dO V^T
      umma_commit(&sm->mma_a);
    }
    if (tid < kBwdCompute) {
      mbar_wait(&sm->mma_a, it & 1, abort_any);
      __syncwarp();
      tc_fence_after_sync();
#pragma unroll 1
      for (int ch = hf * (8 / kBwdGroups); ch < (hf + 1) * (8 / kBwdGroups); ++ch) {  // its keys
        float sv[16], dp[16];
        tmem_ld16(tS + lane_off + ch * 16, sv);
        tmem_ld16(tdP + lane_off + ch * 16, dp);
        tmem_ld_wait_for(sv);
        tmem_ld_wait_for(dp);
        uint32_t sw[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float dv[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int tok = tok0 + ch * 16 + e + k;
            const float pr = tok < my_lim ? ex2(__fsub_rn(__fmul_rn(sv[e + k], p.cscale), my_l2)) : 0.f;
            dv[k] = __fmul_rn(pr, __fsub_rn(dp[e + k], my_d));
          }
          sw[e / 2] = pack_bf16(dv[0], dv[1]);
        }
        put8(sS, t, ch * 2, make_uint4(sw[0], sw[1], sw[2], sw[3]));
        put8(sS, t, ch * 2 + 1, make_uint4(sw[4], sw[5], sw[6], sw[7]));
      }
      fence_proxy_async_smem();
    }
    tc_fence_before_sync();
    __syncthreads();
    if (*abort_any) break;
    if (warp == kBwdMmaWarp && lane == 0) {
      tc_fence_after_sync();
      mma_kn<D>(tdQ, aS, aK, idesc_bf16(128, D, 0, 1), it > 0);  // dQ += dS K
      umma_commit(&sm->mma_b);
    }
    mbar_wait(&sm->mma_b, it & 1, abort_any);
    __syncwarp();
  }
  tc_fence_before_sync();
  __syncthreads();
  const bool ok = !*abort_any;
  if (tid < kBwdCompute && ok) {
    tc_fence_after_sync();
#pragma unroll 1
    for (int ch = hf * (D / 16 / kBwdGroups); ch < (hf + 1) * (D / 16 / kBwdGroups); ++ch) {  // its part of D
      float qv[16];
      tmem_ld16(tdQ + lane_off + ch * 16, qv);
      tmem_ld_wait_for(qv);
      if (my_row >= 0) {
        const int i = r_t / p.G, g = r_t - i * p.G;
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          w[e] = pack_bf16(it > 0 ? __fmul_rn(qv[2 * e], p.scale) : 0.f,
                           it > 0 ? __fmul_rn(qv[2 * e + 1], p.scale) : 0.f);
        uint4 *dst = reinterpret_cast<uint4 *>(p.dq + b * p.dq_sb + static_cast<int64_t>(i) * p.dq_ss +
                                               static_cast<int64_t>(kvh * p.G + g) * p.dq_sh + ch * 16);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  }
  if (!ok && warp == kBwdMmaWarp && lane == 0) {
    umma_commit(&sm->drain);
    volatile int no_abort = 0;
    mbar_wait(&sm->drain, 0, &no_abort);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
  if (tid == 0 && !ok && p.err) atomicOr(p.err, kErrTimeout);
}

}  // namespace pkv
