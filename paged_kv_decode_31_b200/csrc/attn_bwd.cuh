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
//                   dS^T packed as bf16 into TMEM, dV += P^T dO and
//                   dK += dS^T Q accumulated in TMEM over the 128-row tiles in
//                   ascending order, then written once;
//   bwd_q_kernel    one CTA per (sequence, KV head, 128-row tile): S = Q K^T,
//                   dP = dO V^T (rows on M), dS packed into TMEM, dQ += dS K
//                   accumulated over the key tiles in ascending order.
// Every sum therefore has one fixed order and the result is bitwise
// reproducible and independent of the batch around a sequence.
//
// Warps 0-15 do the elementwise work -- warps w, w + 4, w + 8, w + 12 share
// TMEM lanes 32 (w % 4) .. + 31 (thread t = lane t of the 128) and split the
// columns in quarters --, warp 16 owns TMEM, its lane 0 issuing the MMAs, and
// the warps after it load every operand tile with TMA (the cache's K / V rows
// in boxes addressed through the block table, as the forward does; Q and dO
// in boxes of 128 / G tokens x G heads): one load warp for dK/dV (576
// threads), one per cache for dQ (608 threads).  The second operand of each
// accumulating product (P^T and dS^T, or dS) never touches shared memory:
// the elementwise pass packs it as bf16 into the TMEM columns its S / dP
// values came from and the next MMAs read it from there as their A operand.
// The shared memory this frees holds deeper rings of the streamed tiles (Q
// and dO, or K and V).  The elementwise warps and the MMA warp hand off
// through mbarriers (no block-wide barrier per tile).  Where a row tile
// cannot be one Q box (G not dividing 128, or fewer than 128 / G query
// tokens), the compute threads stage the Q / dO tiles with cp.async instead.
#pragma once

#include <cuda_bf16.h>

#include "attn_split.cuh"
#include "ptx.cuh"

namespace pkv {

constexpr int kBwdCompute = 512;               // elementwise threads
constexpr int kBwdGroups = kBwdCompute / 128;  // column groups per TMEM lane
constexpr int kBwdMmaWarp = kBwdCompute / 32;
constexpr int kBwdLoadWarp = kBwdMmaWarp + 1;
constexpr int kBwdThreads = kBwdCompute + 64;
constexpr int kBwdQThreads = kBwdCompute + 96;  // dQ: a second load warp (K and V boxes in parallel)
constexpr int kBwdTile = 128;  // keys per key tile and rows per row tile
constexpr uint32_t kBwdBar = 1;                   // named barrier of compute + MMA warps
constexpr uint32_t kBwdBarThreads = kBwdCompute + 32;
constexpr uint32_t kBwdComputeBar = 2;            // named barrier of the elementwise warps

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
  int box_slots;       // cache rows per K / V box = min(block_size, 128)
  int map_head_first;  // K / V map dimension order (D, Hkv, slot, block) vs (D, slot, Hkv, block)
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
  static constexpr int kHalf = kBwdTile * 128;    // 128 rows x 64 elements x bf16
  static constexpr int kTile = (D / 64) * kHalf;  // a [128][D] operand
  static constexpr int kTiles = 6;                // two fixed + two double-buffered
  struct Small {
    uint64_t full[2], empty[2];  // streamed tile buffers: loaded / free again
    uint64_t fixed;              // the fixed tiles loaded
    uint64_t mma_a, mma_b, mma_bv, drain;
    uint64_t ds_ready, fin;  // elementwise pass -> MMA warp; last accumulation done
    uint32_t tmem_base;
    alignas(16) int lim[2][kBwdTile];  // key limit of each row of the row tile in buffer j
    alignas(16) float lse2[2][kBwdTile];
    alignas(16) float dsum[2][kBwdTile];
  };
  static constexpr int kSmem = kTiles * kTile + static_cast<int>(sizeof(Small)) + 1024;
};

// dQ: Q and dO, then three K buffers and two V buffers (V is free again once
// a tile's S / dP products are done, K only after its dQ product).
template <int D>
struct BwdQCfg {
  static constexpr int kTile = BwdCfg<D>::kTile;
  static constexpr int kKBufs = 3, kVBufs = 2;
  static constexpr int kTiles = 2 + kKBufs + kVBufs;
  struct Small {
    uint64_t kfull[kKBufs], kempty[kKBufs], vfull[kVBufs], vempty[kVBufs];
    uint64_t fixed;  // Q and dO loaded
    uint64_t mma_a, mma_b, drain;
    uint64_t dp_free, ds_ready, fin;  // elementwise pass <-> MMA warp hand-offs
    uint32_t tmem_base;
  };
  static constexpr int kSmem = kTiles * kTile + static_cast<int>(sizeof(Small)) + 1024;
};

// cp.async a [128][D] bf16 tile, rows given by `src_row(c)` (nullptr: zeros),
// into the 128-byte swizzled K-major layout of the MMA operands (row c at
// c * 128 bytes of its 64-element half, 16-byte chunk cc at (cc ^ (c % 8)) * 16,
// the layout a 128-byte-swizzled TMA box writes).  `any` is a valid global
// address for the zero-filled chunks, of which nothing is read.  The caller
// commits the group.
template <int D, class F>
__device__ __forceinline__ void async_rows(uint8_t *dst, int t, const void *any, F src_row) {
  constexpr int kPer = kBwdTile * (D / 8) / kBwdCompute;  // 16-byte chunks per thread
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int idx = t + k * kBwdCompute;
    const int c = idx / (D / 8), ch = idx % (D / 8);
    const __nv_bfloat16 *s = src_row(c);
    const int h = ch >> 3, cc = ch & 7;
    cp_async16(dst + h * BwdCfg<D>::kHalf + c * 128 + ((cc ^ (c & 7)) << 4),
               s ? static_cast<const void *>(s + ch * 8) : any, s ? 16u : 0u);
  }
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

// Cache row of token `tok` of sequence b (-1 past the table or the cache,
// with the error bits set as in the forward).
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

// Row r = i G + g of the row tiles of (b, kvh) in a [batch][seqlen_q][Hq][D]
// tensor (nullptr for padded rows).
__device__ __forceinline__ const __nv_bfloat16 *bwd_query_row(const BwdParams &p, const __nv_bfloat16 *base,
                                                              int64_t sb, int64_t ss, int64_t sh, int b,
                                                              int kvh, int r) {
  if (r >= p.G * p.seqlen_q) return nullptr;
  const int i = r / p.G, g = r - i * p.G;
  return base + b * sb + static_cast<int64_t>(i) * ss + static_cast<int64_t>(kvh * p.G + g) * sh;
}

// Load warp: the K and V rows of tokens [tok0, tok0 + 128) of sequence b,
// KV head kvh, as TMA boxes of box_slots cache rows (lane l: box l) into
// dk / dv, completing on `bar` (count 1: lane 0 arrives after every lane has
// announced its bytes).  Boxes of tokens past the context, past the table or
// of an invalid block read a block coordinate outside the map and land as
// zeros (the latter two set the error bits as in the forward); rows past the
// context inside a loaded block keep the cache's bytes and are zeroed by the
// consumer.
template <int D>
__device__ __forceinline__ void load_kv_tile(const BwdParams &p, const CUtensorMap *mk, const CUtensorMap *mv,
                                             uint8_t *dk, uint8_t *dv, uint64_t *bar, int b, int kvh,
                                             int seqlen, int tok0, int lane) {
  const int nbox = kBwdTile / p.box_slots;
  int errs = 0;
  if (lane < nbox) {
    const int r = lane * p.box_slots;
    const int tok = tok0 + r;
    int blk = static_cast<int>(p.num_blocks);
    if (tok < seqlen) {
      const int col = tok >> p.block_shift;
      if (col >= p.max_blocks_per_seq) {
        errs = kErrTableWidth;
      } else {
        const int id = __ldg(p.block_table + b * p.bt_stride + col);
        if (id < 0 || static_cast<int64_t>(id) >= p.num_blocks)
          errs = kErrBadBlock;
        else
          blk = id;
      }
    }
    const int slot = tok & ((1 << p.block_shift) - 1);
    const int c1 = p.map_head_first ? kvh : slot;
    const int c2 = p.map_head_first ? slot : kvh;
    mbar_expect_tx(bar, static_cast<uint32_t>(2 * (D / 64) * p.box_slots * 128));
#pragma unroll
    for (int h = 0; h < D / 64; ++h) {
      tma_load_4d(dk + h * BwdCfg<D>::kHalf + r * 128, mk, bar, h * 64, c1, c2, blk);
      tma_load_4d(dv + h * BwdCfg<D>::kHalf + r * 128, mv, bar, h * 64, c1, c2, blk);
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  if (errs && p.err) atomicOr(p.err, errs);
}

// Load warp: lane l's box of the cache rows of tokens [tok0, tok0 + 128) of
// sequence b (box l covers rows [l box_slots, (l + 1) box_slots)), resolved
// once per tile for both caches: the block coordinate (outside the map, so
// the box lands as zeros, past the context, the table or the cache -- the
// latter two flagged as in the forward) and the slot / head coordinates.
struct CacheBox {
  int r, c1, c2, blk;
  bool on;
};
__device__ __forceinline__ CacheBox cache_box(const BwdParams &p, int b, int kvh, int seqlen, int tok0,
                                              int lane) {
  CacheBox x{0, 0, 0, static_cast<int>(p.num_blocks), lane < kBwdTile / p.box_slots};
  if (!x.on) return x;
  x.r = lane * p.box_slots;
  const int tok = tok0 + x.r;
  int errs = 0;
  if (tok < seqlen) {
    const int col = tok >> p.block_shift;
    if (col >= p.max_blocks_per_seq) {
      errs = kErrTableWidth;
    } else {
      const int id = __ldg(p.block_table + b * p.bt_stride + col);
      if (id < 0 || static_cast<int64_t>(id) >= p.num_blocks)
        errs = kErrBadBlock;
      else
        x.blk = id;
    }
  }
  const int slot = tok & ((1 << p.block_shift) - 1);
  x.c1 = p.map_head_first ? kvh : slot;
  x.c2 = p.map_head_first ? slot : kvh;
  if (errs && p.err) atomicOr(p.err, errs);
  return x;
}
// Issue one cache's boxes of a tile (every lane with a box), completing on
// `bar` (count 1: lane 0 arrives after every lane has announced its bytes).
template <int D>
__device__ __forceinline__ void issue_cache_boxes(const BwdParams &p, const CUtensorMap *map, uint8_t *dst,
                                                  uint64_t *bar, const CacheBox &x, int lane) {
  if (x.on) {
    mbar_expect_tx(bar, static_cast<uint32_t>((D / 64) * p.box_slots * 128));
#pragma unroll
    for (int h = 0; h < D / 64; ++h)
      tma_load_4d(dst + h * BwdCfg<D>::kHalf + x.r * 128, map, bar, h * 64, x.c1, x.c2, x.blk);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// Load warp, lane 0: the Q and dO rows of row tile rt of (b, kvh) -- one box
// of 128 / G tokens x G heads per 64-element half -- into dq / dg.
template <int D>
__device__ __forceinline__ void load_row_tile(const BwdParams &p, const CUtensorMap *mq, const CUtensorMap *mg,
                                              uint8_t *dq, uint8_t *dg, uint64_t *bar, int b, int kvh, int rt) {
  mbar_expect_tx(bar, static_cast<uint32_t>(2 * BwdCfg<D>::kTile));
  const int i0 = rt * (kBwdTile / p.G);
#pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    tma_load_4d(dq + h * BwdCfg<D>::kHalf, mq, bar, h * 64, kvh * p.G, i0, b);
    tma_load_4d(dg + h * BwdCfg<D>::kHalf, mg, bar, h * 64, kvh * p.G, i0, b);
  }
  mbar_arrive(bar);
}

// Zero rows [from, 128) of a K tile and of a V tile (compute threads; thread
// (t, hf) takes row t of tensor hf % 2, half hf / 2).
template <int D>
__device__ __forceinline__ void zero_rows_from(uint8_t *dk, uint8_t *dv, int from, int t, int hf) {
  if (t < from || hf / 2 >= D / 64) return;
  uint8_t *row = ((hf & 1) ? dv : dk) + (hf / 2) * BwdCfg<D>::kHalf + t * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(row + c * 16) = make_uint4(0u, 0u, 0u, 0u);
}

// Issue D[tmem] = A[128 x K] * B^T for two K-major [128][K] operands in
// shared memory.
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

// Issue D[tmem] (+)= A[128 x 128] * B[128 x N]: A packed bf16 in TMEM, its
// K steps of 16 at columns a + 16 kk .. + 8 (where the elementwise pass wrote
// them over the 16 fp32 columns they came from); B a [128][N] tile in shared
// memory read along its rows (MN-major).
__device__ __forceinline__ void mma_tn(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < kBwdTile / 16; ++kk)
    umma_bf16_ts(d, a + kk * 16, smem_desc(b + kk * 2048, kBwdTile * 128, 1024, kLayoutSw128), idesc,
                 (accumulate || kk > 0) ? 1u : 0u);
}

__device__ __forceinline__ uint8_t *bwd_smem_base(uint8_t *raw) {
  return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                     ~static_cast<uintptr_t>(1023));
}

template <class Small>
__device__ __forceinline__ void bwd_init_barriers(Small *sm) {
  for (int j = 0; j < 2; ++j) {
    mbar_init(&sm->full[j], 1);
    mbar_init(&sm->empty[j], 1);
  }
  mbar_init(&sm->fixed, 1);
  mbar_init(&sm->mma_a, 1);
  mbar_init(&sm->mma_b, 1);
  mbar_init(&sm->mma_bv, 1);
  mbar_init(&sm->drain, 1);
  mbar_init(&sm->ds_ready, kBwdCompute / 32);  // one arrival per elementwise warp
  mbar_init(&sm->fin, 1);
  fence_barrier_init();
}

// ---------------------------------------------------------------------------
// dK / dV: one CTA per (b, kvh, key tile).
// smem: K, V, then Q and dO of row tile j (j = it % 2) at (2 + 2 j) and
// (3 + 2 j) tiles.
// TMEM: S^T [0,128) (P^T packed over it), dP^T [128,256) (dS^T packed over
// it), dV [256, 256 + D), dK [256 + D, 256 + 2D).
// Row tile it: MMA warp: once P^T / dS^T(it - 1) are in TMEM (ds_ready),
// dV += P^T(it - 1) dO, dK += dS^T(it - 1) Q, then S^T = K Q(it)^T,
// dP^T = V dO(it)^T; elementwise warps: once the second pair is done (mma_a),
// P^T / dS^T of it into TMEM, then ds_ready; load warp: row tile it + 2 into
// buffer j once the first pair of it is done.  MMAs into different
// accumulators carry no ordering guarantee among themselves, so S^T(it),
// which overwrites the P^T that dV(it - 1) reads, is issued once dV(it - 1)
// has completed (its own commit, `mma_bv`, landing while dK(it - 1) runs),
// and dP^T(it) once dK(it - 1) has (`mma_b`, landing while S^T(it) runs).
// The elementwise warps meet at a barrier of their own at the start of each
// tile (the row statistics they share); the MMA warp takes no part in it.
// kRowsTma false: the compute threads stage the row tiles with cp.async.
// ---------------------------------------------------------------------------
template <int D, bool kRowsTma>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_kv_kernel(const __grid_constant__ BwdParams p, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_q,
                  const __grid_constant__ CUtensorMap map_g) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = bwd_smem_base(smem_raw);
  auto *sm = reinterpret_cast<typename C::Small *>(smem + C::kTiles * C::kTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int t = tid & 127, hf = tid >> 7;  // TMEM lane / key, column group (compute threads)
  const bool compute = tid < kBwdCompute;
  const bool issuer = warp == kBwdMmaWarp && lane == 0;
  int abort_flag = 0;  // the waits' abort word; agreement goes through the barriers
  volatile int *abort_any = &abort_flag;

  // key tiles in ascending order across the grid: under causal masking the
  // first ones meet the most row tiles, and CTAs start roughly in index
  // order, so the longest run first and the short ones fill the tail
  int u = blockIdx.x;
  const int kt = u / (p.batch * p.Hkv);
  u -= kt * (p.batch * p.Hkv);
  const int kvh = u % p.Hkv;
  const int b = u / p.Hkv;
  const int seqlen = max(__ldg(p.seqlens + b), 0);
  const int tok0 = kt * kBwdTile;
  if (tok0 >= seqlen) return;  // uniform: the whole CTA leaves before any barrier
  const int R = p.G * p.seqlen_q;
  // first row tile with a row that sees key tok0: rows r with i >= tok0 - (seqlen - sq)
  int rt0 = 0;
  if (p.causal) {
    const int i_min = tok0 - (seqlen - p.seqlen_q);
    rt0 = i_min > 0 ? (i_min * p.G) / kBwdTile : 0;
  }
  const int n = (R + kBwdTile - 1) / kBwdTile - rt0;  // row tiles, >= 1
  uint8_t *sK = smem, *sV = smem + C::kTile;
  auto sQ = [&](int j) { return smem + (2 + 2 * j) * C::kTile; };
  auto sG = [&](int j) { return smem + (3 + 2 * j) * C::kTile; };

  if (tid == 0) bwd_init_barriers(sm);
  if (warp == kBwdMmaWarp) tmem_alloc(&sm->tmem_base, 512);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  if (warp == kBwdLoadWarp) {
    // ---------------- load warp ----------------
    if (lane == 0) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      if (kRowsTma) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_g);
      }
    }
    load_kv_tile<D>(p, &map_k, &map_v, sK, sV, &sm->fixed, b, kvh, seqlen, tok0, lane);
    if constexpr (kRowsTma) {
      bool okl = true;
      for (int it = 0; it < n && okl; ++it) {
        const int j = it & 1;
        if (lane == 0) {
          if (it >= 2) okl = mbar_wait(&sm->empty[j], ((it >> 1) - 1) & 1, abort_any);
          if (okl) load_row_tile<D>(p, &map_q, &map_g, sQ(j), sG(j), &sm->full[j], b, kvh, rt0 + it);
        }
        okl = __shfl_sync(0xffffffffu, okl ? 1 : 0, 0) != 0;
      }
      // nothing of ours may still be landing when the CTA exits
      if (lane == 0) {
        for (int it = max(n - 2, 0); it < n; ++it) {
          int no_abort = 0;
          mbar_wait(&sm->full[it & 1], (it >> 1) & 1, &no_abort);
        }
      }
    }
    if (lane == 0) {
      int no_abort = 0;
      mbar_wait(&sm->fixed, 0, &no_abort);
    }
    __syncwarp();
    __syncthreads();  // the final barrier below
    return;
  }

  // ---------------- compute + MMA warps ----------------
  int n_lim = 0;
  float n_l2 = 0.f, n_ds = 0.f;
  auto row_stats = [&](int rt) {  // statistics of row t of row tile rt (registers)
    if (hf != 0) return;
    const int r = rt * kBwdTile + t;
    n_lim = bwd_row_lim(p, seqlen, r);
    n_l2 = 0.f;
    n_ds = 0.f;
    if (r < R) {
      const int i = r / p.G, g = r - i * p.G;
      const int64_t row_id = (static_cast<int64_t>(b) * p.seqlen_q + i) * p.Hq + kvh * p.G + g;
      n_l2 = p.row_lse2[row_id];
      n_ds = p.row_d[row_id];
    }
  };
  auto store_stats = [&](int j) {
    if (hf == 0) {
      sm->lim[j][t] = n_lim;
      sm->lse2[j][t] = n_l2;
      sm->dsum[j][t] = n_ds;
    }
  };
  auto async_row_tile = [&](int rt, int j) {  // cp.async staging (kRowsTma false)
    const int row0 = rt * kBwdTile;
    async_rows<D>(sQ(j), tid, p.q, [&](int c) {
      return bwd_query_row(p, p.q, p.q_sb, p.q_ss, p.q_sh, b, kvh, row0 + c);
    });
    async_rows<D>(sG(j), tid, p.q, [&](int c) {
      return bwd_query_row(p, p.dout, p.g_sb, p.g_ss, p.g_sh, b, kvh, row0 + c);
    });
    cp_async_commit();
  };

  bool ok = true, failed = false;
  if (compute) {
    if constexpr (!kRowsTma) async_row_tile(rt0, 0);
    row_stats(rt0);
    store_stats(0);
    // key rows past the context: zeros (their cache bytes may be anything)
    if (tok0 + kBwdTile > seqlen) {
      ok = mbar_wait(&sm->fixed, 0, abort_any);
      if (ok) zero_rows_from<D>(sK, sV, seqlen - tok0, t, hf);
    }
    if constexpr (!kRowsTma) cp_async_wait<0>();
    fence_proxy_async_smem();
  }
  tc_fence_before_sync();
  failed = named_bar_or(kBwdBar, kBwdBarThreads, !ok);
  tc_fence_after_sync();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const int tok = tok0 + t;
  constexpr uint32_t kIdA = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t kIdB = idesc_bf16(128, D, 0, 1);

  if (!failed && issuer) {
    // ---------------- MMA warp ----------------
    tc_fence_after_sync();
    ok = mbar_wait(&sm->fixed, 0, abort_any);
    for (int it = 0; it < n && ok; ++it) {
      const int j = it & 1;
      if (it > 0) {
        // P^T / dS^T of tile it - 1 are in TMEM
        ok = mbar_wait(&sm->ds_ready, (it - 1) & 1, abort_any);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t aQ = smem_u32(sQ(j ^ 1)), aG = smem_u32(sG(j ^ 1));
        mma_tn(tdV, tS, aG, kIdB, it > 1);   // dV += P^T dO
        umma_commit(&sm->mma_bv);
        mma_tn(tdK, tdP, aQ, kIdB, it > 1);  // dK += dS^T Q
        umma_commit(&sm->mma_b);
        if (kRowsTma) umma_commit(&sm->empty[j ^ 1]);
      }
      if (kRowsTma && ok) ok = mbar_wait(&sm->full[j], (it >> 1) & 1, abort_any);
      const uint32_t aQ = smem_u32(sQ(j)), aG = smem_u32(sG(j));
      if (ok && it > 0) ok = mbar_wait(&sm->mma_bv, (it - 1) & 1, abort_any);
      if (ok) {
        tc_fence_after_sync();
        mma_kk<D>(tS, sbase, aQ, kIdA);  // S^T = K Q^T
      }
      if (ok && it > 0) ok = mbar_wait(&sm->mma_b, (it - 1) & 1, abort_any);
      if (ok) {
        tc_fence_after_sync();
        mma_kk<D>(tdP, sbase + C::kTile, aG, kIdA);  // dP^T = V dO^T
        umma_commit(&sm->mma_a);
      }
    }
    if (ok) {
      ok = mbar_wait(&sm->ds_ready, (n - 1) & 1, abort_any);
      if (ok) {
        tc_fence_after_sync();
        const uint32_t aQ = smem_u32(sQ((n - 1) & 1)), aG = smem_u32(sG((n - 1) & 1));
        mma_tn(tdV, tS, aG, kIdB, n > 1);
        mma_tn(tdK, tdP, aQ, kIdB, n > 1);
        umma_commit(&sm->fin);
      }
    }
  } else if (!failed && compute) {
    // ---------------- elementwise warps ----------------
    for (int it = 0; it < n && ok; ++it) {
      const int j = it & 1;
      const bool next = it + 1 < n;
      if constexpr (!kRowsTma) {
        // buffer j ^ 1 is free once the accumulation of tile it - 1 is done
        if (it > 0) ok = ok && mbar_wait(&sm->mma_b, (it - 1) & 1, abort_any);
        if (ok && next) async_row_tile(rt0 + it + 1, j ^ 1);
      }
      if (next) row_stats(rt0 + it + 1);
      ok = ok && mbar_wait(&sm->mma_a, it & 1, abort_any);
      // the row statistics of tile it (written during tile it - 1) are
      // visible to every elementwise thread past this barrier, and nobody
      // reads the other buffer's any more
      if (named_bar_or(kBwdComputeBar, kBwdCompute, !ok)) {
        ok = false;
        break;
      }
      __syncwarp();
      tc_fence_after_sync();
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
            const bool vis = tok < sm->lim[j][c];
            const float pr =
                vis ? ex2(__fsub_rn(__fmul_rn(sv[e + k], p.cscale), sm->lse2[j][c])) : 0.f;
            pv[k] = pr;
            dv[k] = __fmul_rn(pr, __fsub_rn(dp[e + k], sm->dsum[j][c]));
          }
          pw[e / 2] = pack_bf16(pv[0], pv[1]);
          sw[e / 2] = pack_bf16(dv[0], dv[1]);
        }
        tmem_st8(tS + lane_off + ch * 16, pw);
        tmem_st8(tdP + lane_off + ch * 16, sw);
      }
      tmem_st_wait();
      if (next) store_stats(j ^ 1);
      if constexpr (!kRowsTma) {
        cp_async_wait<0>();
        fence_proxy_async_smem();
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm->ds_ready);
    }
    // the last accumulation (and every MMA before it) has completed
    if (ok) ok = mbar_wait(&sm->fin, 0, abort_any);
  }
  tc_fence_before_sync();
  failed = named_bar_or(kBwdBar, kBwdBarThreads, failed || !ok);
  if (compute && !failed) {
    tc_fence_after_sync();
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
          wv[e] = pack_bf16(vv[2 * e], vv[2 * e + 1]);
          wk[e] = pack_bf16(__fmul_rn(kv[2 * e], p.scale), __fmul_rn(kv[2 * e + 1], p.scale));
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
  if (failed && issuer) {
    umma_commit(&sm->drain);
    int no_abort = 0;
    mbar_wait(&sm->drain, 0, &no_abort);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
  if (tid == 0 && failed && p.err) atomicOr(p.err, kErrTimeout);
}

// ---------------------------------------------------------------------------
// dQ: one CTA per (b, kvh, row tile).
// smem: Q, dO, K buffers k % 3 at 2 + k % 3, V buffers at 5 + k % 2 (tiles).
// TMEM: S of key tile it (dS packed over it) at [0,128) for even it and
// [384,512) for odd it, dP [128,256), dQ [256, 256 + D).
// No per-tile barrier: the elementwise warps and the MMA warp hand off
// through mbarriers, so the MMAs of the next key tile run while the
// elementwise pass of this one computes.  Per key tile it:
//   elementwise warps: wait for S / dP(it) (mma_a), load their dP columns
//   (and the first S chunk) into registers, arrive dp_free; compute dS(it)
//   into the S columns; arrive ds_ready.
//   MMA warp: once K / V(it) have landed, dP(it - 1) has been read
//   (dp_free) and dQ += dS(it - 2) K has completed (S(it) reuses those
//   columns; MMAs into different accumulators are not ordered among
//   themselves), S(it) = Q K(it)^T and dP(it) = dO V(it)^T, which frees
//   V(it)'s buffer; then, once dS(it - 1) is written (ds_ready),
//   dQ += dS(it - 1) K(it - 1), which frees K(it - 1)'s buffer.
// With K three deep and V two deep the load warp's TMA latency stays behind
// the pipeline.  Rows past the context in the next key tile are zeroed
// before dp_free.
// kRowsTma false: the compute threads stage Q and dO with cp.async.
// ---------------------------------------------------------------------------
template <int D, bool kRowsTma>
__global__ void __launch_bounds__(kBwdQThreads, 1)
    bwd_q_kernel(const __grid_constant__ BwdParams p, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_q,
                 const __grid_constant__ CUtensorMap map_g) {
  using C = BwdQCfg<D>;
  constexpr int KB = C::kKBufs, VB = C::kVBufs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = bwd_smem_base(smem_raw);
  auto *sm = reinterpret_cast<typename C::Small *>(smem + C::kTiles * C::kTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int t = tid & 127, hf = tid >> 7;  // TMEM lane / row, column group (compute threads)
  const bool compute = tid < kBwdCompute;
  const bool issuer = warp == kBwdMmaWarp && lane == 0;
  int abort_flag = 0;
  volatile int *abort_any = &abort_flag;

  // row tiles in descending order across the grid (the last rows see the
  // most keys under causal masking): longest runs first
  int u = blockIdx.x;
  const int rt = p.n_row_tiles - 1 - u / (p.batch * p.Hkv);
  u %= p.batch * p.Hkv;
  const int kvh = u % p.Hkv;
  const int b = u / p.Hkv;
  const int seqlen = max(__ldg(p.seqlens + b), 0);
  const int R = p.G * p.seqlen_q;
  const int row0 = rt * kBwdTile;
  // keys [0, lim_max) cover every row of the tile
  const int lim_max = bwd_row_lim(p, seqlen, min(row0 + kBwdTile, R) - 1);
  const int n = (lim_max + kBwdTile - 1) / kBwdTile;
  uint8_t *sQ = smem, *sG = smem + C::kTile;
  auto sK = [&](int k) { return smem + (2 + k % KB) * C::kTile; };
  auto sV = [&](int k) { return smem + (2 + KB + k % VB) * C::kTile; };

  if (tid == 0) {
    for (int i = 0; i < KB; ++i) {
      mbar_init(&sm->kfull[i], 1);
      mbar_init(&sm->kempty[i], 1);
    }
    for (int i = 0; i < VB; ++i) {
      mbar_init(&sm->vfull[i], 1);
      mbar_init(&sm->vempty[i], 1);
    }
    mbar_init(&sm->fixed, 1);
    mbar_init(&sm->mma_a, 1);
    mbar_init(&sm->mma_b, 1);
    mbar_init(&sm->drain, 1);
    mbar_init(&sm->dp_free, kBwdCompute / 32);  // one arrival per elementwise warp
    mbar_init(&sm->ds_ready, kBwdCompute / 32);
    mbar_init(&sm->fin, 1);
    fence_barrier_init();
  }
  if (warp == kBwdMmaWarp) tmem_alloc(&sm->tmem_base, 512);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  if (warp >= kBwdLoadWarp) {
    // ---------------- load warps: K (and Q / dO), V ----------------
    // A TMA box of a block-size-16 cache costs the issuing warp ~90 cycles,
    // so K and V each have a warp.  Per key tile: the block coordinates
    // first (nothing to wait for), then the boxes once the buffer is free
    // (V: after S / dP of tile it - 2; K: after dQ of tile it - 3).
    const bool is_v = warp == kBwdLoadWarp + 1;
    if (lane == 0) {
      tma_prefetch_desc(is_v ? &map_v : &map_k);
      if (kRowsTma && !is_v) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_g);
        load_row_tile<D>(p, &map_q, &map_g, sQ, sG, &sm->fixed, b, kvh, rt);
      }
    }
    const int nbuf = is_v ? VB : KB;
    uint64_t *full = is_v ? sm->vfull : sm->kfull;
    uint64_t *empty = is_v ? sm->vempty : sm->kempty;
    bool okl = true;
    for (int it = 0; it < n && okl; ++it) {
      const CacheBox y = cache_box(p, b, kvh, seqlen, it * kBwdTile, lane);
      if (lane == 0 && it >= nbuf) okl = mbar_wait(&empty[it % nbuf], ((it / nbuf) - 1) & 1, abort_any);
      okl = __shfl_sync(0xffffffffu, okl ? 1 : 0, 0) != 0;
      if (!okl) break;
      issue_cache_boxes<D>(p, is_v ? &map_v : &map_k, is_v ? sV(it) : sK(it), &full[it % nbuf], y, lane);
    }
    // nothing of ours may still be landing when the CTA exits
    if (lane == 0) {
      int no_abort = 0;
      for (int it = max(n - nbuf, 0); it < n; ++it) mbar_wait(&full[it % nbuf], (it / nbuf) & 1, &no_abort);
      if (kRowsTma && !is_v) mbar_wait(&sm->fixed, 0, &no_abort);
    }
    __syncwarp();
    __syncthreads();  // the final barrier below
    return;
  }

  // ---------------- compute + MMA warps ----------------
  const int r_t = row0 + t;
  int my_lim = 0;
  float my_l2 = 0.f, my_d = 0.f;
  int64_t my_row = -1;
  bool ok = true, failed = false;
  if (compute) {
    if constexpr (!kRowsTma) {
      async_rows<D>(sQ, tid, p.q, [&](int c) {
        return bwd_query_row(p, p.q, p.q_sb, p.q_ss, p.q_sh, b, kvh, row0 + c);
      });
      async_rows<D>(sG, tid, p.q, [&](int c) {
        return bwd_query_row(p, p.dout, p.g_sb, p.g_ss, p.g_sh, b, kvh, row0 + c);
      });
      cp_async_commit();
    }
    my_lim = bwd_row_lim(p, seqlen, r_t);
    if (r_t < R) {
      const int i = r_t / p.G, g = r_t - i * p.G;
      my_row = (static_cast<int64_t>(b) * p.seqlen_q + i) * p.Hq + kvh * p.G + g;
      my_l2 = p.row_lse2[my_row];
      my_d = p.row_d[my_row];
    }
    // key rows past the context in the first key tile: zeros
    if (n > 0 && kBwdTile > seqlen) {
      ok = mbar_wait(&sm->kfull[0], 0, abort_any) && mbar_wait(&sm->vfull[0], 0, abort_any);
      if (ok) zero_rows_from<D>(sK(0), sV(0), seqlen, t, hf);
    }
    if constexpr (!kRowsTma) cp_async_wait<0>();
    fence_proxy_async_smem();
  }
  tc_fence_before_sync();
  failed = named_bar_or(kBwdBar, kBwdBarThreads, !ok);
  tc_fence_after_sync();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t tS0 = tmem, tdP = tmem + 128, tdQ = tmem + 256;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
  constexpr uint32_t kIdA = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t kIdB = idesc_bf16(128, D, 0, 1);
  static_assert(256 + D <= 384, "dQ below the second S range");

  if (!failed && issuer) {
    // ---------------- MMA warp ----------------
    tc_fence_after_sync();
    if (kRowsTma && n > 0) ok = mbar_wait(&sm->fixed, 0, abort_any);
    for (int it = 0; it < n && ok; ++it) {
      ok = mbar_wait(&sm->kfull[it % KB], (it / KB) & 1, abort_any) &&
           mbar_wait(&sm->vfull[it % VB], (it / VB) & 1, abort_any);
      if (ok && it >= 1) ok = mbar_wait(&sm->dp_free, (it - 1) & 1, abort_any);
      if (ok && it >= 2) ok = mbar_wait(&sm->mma_b, (it - 2) & 1, abort_any);
      if (!ok) break;
      tc_fence_after_sync();
      const uint32_t tS = tS0 + (it & 1) * 384;
      mma_kk<D>(tS, sbase, smem_u32(sK(it)), kIdA);              // S = Q K^T
      mma_kk<D>(tdP, sbase + C::kTile, smem_u32(sV(it)), kIdA);  // dP = dO V^T
      umma_commit(&sm->mma_a);
      umma_commit(&sm->vempty[it % VB]);
      if (it >= 1) {
        ok = mbar_wait(&sm->ds_ready, (it - 1) & 1, abort_any);
        if (!ok) break;
        tc_fence_after_sync();
        mma_tn(tdQ, tS0 + ((it - 1) & 1) * 384, smem_u32(sK(it - 1)), kIdB, it > 1);  // dQ += dS K
        umma_commit(&sm->mma_b);
        umma_commit(&sm->kempty[(it - 1) % KB]);
      }
    }
    if (ok && n > 0) {
      ok = mbar_wait(&sm->ds_ready, (n - 1) & 1, abort_any);
      if (ok) {
        tc_fence_after_sync();
        mma_tn(tdQ, tS0 + ((n - 1) & 1) * 384, smem_u32(sK(n - 1)), kIdB, n > 1);
        umma_commit(&sm->fin);
      }
    }
  } else if (!failed && compute) {
    // ---------------- elementwise warps ----------------
    const int ch0 = hf * (8 / kBwdGroups);  // its two 16-key chunks: ch0, ch0 + 1
    for (int it = 0; it < n && ok; ++it) {
      const int k0 = it * kBwdTile;
      const uint32_t tS = tS0 + (it & 1) * 384;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm->mma_a, it & 1, abort_any));  // warp-wide
      if (!ok) break;
      __syncwarp();
      tc_fence_after_sync();
      float sv[16], dp0[16], dp1[16];
      tmem_ld16(tdP + lane_off + ch0 * 16, dp0);
      tmem_ld16(tdP + lane_off + ch0 * 16 + 16, dp1);
      tmem_ld16(tS + lane_off + ch0 * 16, sv);
      tmem_ld_wait_for(dp0);
      tmem_ld_wait_for(dp1);
      tmem_ld_wait_for(sv);
      // key rows past the context in the next key tile: zeros, before its MMAs
      const int k1 = k0 + kBwdTile;
      if (it + 1 < n && k1 + kBwdTile > seqlen) {
        ok = mbar_wait(&sm->kfull[(it + 1) % KB], ((it + 1) / KB) & 1, abort_any) &&
             mbar_wait(&sm->vfull[(it + 1) % VB], ((it + 1) / VB) & 1, abort_any);
        if (ok) zero_rows_from<D>(sK(it + 1), sV(it + 1), seqlen - k1, t, hf);
        fence_proxy_async_smem();
      }
      // dP of this tile is in registers: the next tile's MMAs may overwrite it
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm->dp_free);
      auto ds_chunk = [&](int ch, const float (&s16)[16], const float (&d16)[16]) {
        uint32_t sw[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float dv[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int tok = k0 + ch * 16 + e + k;
            const float pr = tok < my_lim ? ex2(__fsub_rn(__fmul_rn(s16[e + k], p.cscale), my_l2)) : 0.f;
            dv[k] = __fmul_rn(pr, __fsub_rn(d16[e + k], my_d));
          }
          sw[e / 2] = pack_bf16(dv[0], dv[1]);
        }
        tmem_st8(tS + lane_off + ch * 16, sw);
      };
      ds_chunk(ch0, sv, dp0);
      tmem_ld16(tS + lane_off + ch0 * 16 + 16, sv);
      tmem_ld_wait_for(sv);
      ds_chunk(ch0 + 1, sv, dp1);
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm->ds_ready);
    }
    // the last accumulation (and every MMA before it) has completed
    if (ok && n > 0) ok = mbar_wait(&sm->fin, 0, abort_any);
  }
  tc_fence_before_sync();
  failed = named_bar_or(kBwdBar, kBwdBarThreads, failed || !ok);
  if (compute && !failed) {
    tc_fence_after_sync();
#pragma unroll 1
    for (int ch = hf * (D / 16 / kBwdGroups); ch < (hf + 1) * (D / 16 / kBwdGroups); ++ch) {  // its part of D
      float qv[16];
      tmem_ld16(tdQ + lane_off + ch * 16, qv);
      tmem_ld_wait_for(qv);
      if (my_row >= 0) {
        const int i = r_t / p.G, g = r_t - i * p.G;
        uint32_t w[8];
        // rows that see no key (n = 0) leave zeros: the accumulator is unwritten
#pragma unroll
        for (int e = 0; e < 8; ++e)
          w[e] = pack_bf16(n > 0 ? __fmul_rn(qv[2 * e], p.scale) : 0.f,
                           n > 0 ? __fmul_rn(qv[2 * e + 1], p.scale) : 0.f);
        uint4 *dst = reinterpret_cast<uint4 *>(p.dq + b * p.dq_sb + static_cast<int64_t>(i) * p.dq_ss +
                                               static_cast<int64_t>(kvh * p.G + g) * p.dq_sh + ch * 16);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  }
  if (failed && issuer) {
    umma_commit(&sm->drain);
    int no_abort = 0;
    mbar_wait(&sm->drain, 0, &no_abort);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
  if (tid == 0 && failed && p.err) atomicOr(p.err, kErrTimeout);
}

}  // namespace pkv
