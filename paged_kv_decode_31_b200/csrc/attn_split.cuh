// attn_split.cuh -- split-KV attention over a paged cache, sm_100a.
//
// One kernel serves decode (1..few query tokens) and prefill (many): the G
// query heads that share a KV head and the seqlen_q query tokens are packed
// into "rows" r = i * G + g, and a tile of N rows is attended against the KV
// context of one sequence.  Work unit = (sequence b, KV head, row tile, split
// s), where split s is the fixed token range [4096 s, 4096 (s + 1)) -- the
// "KV chunk" of RL-Kernel PR #284 "feat(attention): add CP backward drift
// validation" (Changes: fixed global_block_index merge order, fp32
// accumulation).  A unit produces an unnormalised partial (m, l, acc[D]) per
// row; merge.cuh folds the partials in ascending split order.
//
// The split is walked in 128-token tiles in ascending order.  Per tile:
//   gather   TMA copies K and V of the tile's blocks from the cache, each box
//            addressed by block_table[b][tok / block_size] and the cache's
//            REAL strides (the fix pinned by ROCm/aiter d293d61
//            "test(triton/decode): pin non-contiguous paged KV block stride"),
//            128-byte swizzled into shared memory;
//   S^T      = K_tile * Q^T on the tensor cores (tcgen05, M = 128 tokens,
//            N = rows, K = head_dim, fp32 accumulation in TMEM);
//   softmax  one thread per token: mask (key < row limit), scale to base 2,
//            column max over the 128 tokens (exact, order-free), running max,
//            p = 2^(s - m) stored as P^T in two bf16 parts, hi = bf16(p) and
//            lo = bf16(p - hi), so the tensor cores see p to ~16 bits;
//   O^T      = V^T * (P_hi + P_lo)^T and L = 1 * (P_hi + P_lo)^T on the tensor
//            cores (fresh accumulators each tile): the weighted values and the
//            row sums of the very weights used;
//   update   acc = fma(acc, alpha, O), l = fma(l, alpha, L), alpha = 2^(m_old - m_new),
//            skipped for rows the tile does not reach.
// Tiles start at absolute multiples of 128 and rows never influence each
// other, so a row's arithmetic depends only on its own query, its visible
// keys and the fixed constants: decode row t and prefill row t, batch 1 and
// batch N, contiguous and interleaved caches all give the same bits.
//
// Roles (192 threads): warps 0-3 softmax + correction + epilogue (thread t =
// TMEM lane t = token t of the tile = output column d), warp 4 TMA producer
// (+ Q staging), warp 5 MMA issuer (+ TMEM owner).  The kernel is persistent:
// CTA k takes units k, k + gridDim.x, ...; the producer and the MMA issuer
// run ahead across unit boundaries.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace pkv {

constexpr int kSplitTokens = 4096;
constexpr int kTileTokens = 128;
constexpr int kThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;

constexpr int kErrBadBlock = 1;
constexpr int kErrTableWidth = 2;
constexpr int kErrTimeout = 4;

struct AttnParams {
  const __nv_bfloat16 *q;
  int64_t q_sb, q_ss, q_sh;  // element strides of q (batch, token, head)
  const int32_t *block_table;
  int64_t bt_stride;
  int max_blocks_per_seq;
  int64_t num_blocks;
  const int32_t *seqlens;
  int batch, seqlen_q, Hq, Hkv, G;
  int block_shift;      // log2(block_size)
  int box_slots;        // cache rows per TMA box = min(block_size, 128)
  int map_head_first;   // tensor-map dim order (D, Hkv, slot, block) vs (D, slot, Hkv, block)
  int n_row_tiles, n_splits, n_units;
  float cscale;         // softmax scale * log2(e)
  int causal;
  float *ws_acc;        // [rows][n_splits][D]
  float *ws_ml;         // [rows][n_splits][2] (max in base-2 scaled units, sum)
  int32_t *err;
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// Named barrier over the 128 softmax threads that also ORs a predicate across
// them, so an abort decision is taken by all of them at the same barrier.
__device__ __forceinline__ bool softmax_bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred))
      : "memory");
  return r != 0;
}

// Shared-memory plan.  Every operand region is 1024-byte aligned (the 128-byte
// swizzle pattern repeats every 8 rows of 128 bytes).
template <int D, int N, int NS, int QB>
struct Cfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(N == 16 || N == 32 || N == 64, "rows per tile");
  static_assert(QB == 1 || QB == 2, "Q buffers");
  static constexpr int kHalfBytes = kTileTokens * 128;   // 128 tokens x 64 head_dim x bf16
  static constexpr int kKVBytes = (D / 64) * kHalfBytes;  // one K (or V) tile
  static constexpr int kStageBytes = 2 * kKVBytes;        // K tile then V tile
  static constexpr int kQHalfBytes = N * 128;
  static constexpr int kQBytes = (D / 64) * kQHalfBytes;
  static constexpr int kPBytes = kTileTokens * N * 2;     // one bf16 P^T (hi or lo part)
  static constexpr int kPKGroup = (N / 8) * 128;          // P^T stride between 8-token groups
  static constexpr int kOnesBytes = 4096;                 // 128 x 16 bf16 ones
  static constexpr int kOffStage = 0;
  static constexpr int kOffQ = NS * kStageBytes;
  static constexpr int kOffP = kOffQ + QB * kQBytes;      // 2 buffers x (hi, lo)
  static constexpr int kOffOnes = kOffP + 4 * kPBytes;
  static constexpr int kOffSmall = kOffOnes + kOnesBytes;
  struct Small {
    uint64_t full[NS], empty[NS];
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint64_t q_full[QB], q_empty[QB], drain;
    uint32_t tmem_base;
    int abort_any;
    float wmax[4][N];
    float mnew[2][N];
    float alpha[2][N];
    int skip[2][N];
    int lim[N];
  };
  static constexpr int kSmemBytes = kOffSmall + static_cast<int>(sizeof(Small)) + 1024;
  static constexpr int kTmemCols = (6 * N <= 128) ? 128 : (6 * N <= 256) ? 256 : 512;
};

struct Unit {
  int b, kvh, rt, s;
  int seqlen, row0, rows;
  int tok0;     // first token of the split
  int lim_max;  // keys [0, lim_max) cover every row of the tile
  int n_tiles;  // tiles of this split holding keys < lim_max
};

template <int N>
__device__ __forceinline__ Unit unit_at(const AttnParams &p, int u) {
  Unit x;
  x.rt = u % p.n_row_tiles;
  u /= p.n_row_tiles;
  x.kvh = u % p.Hkv;
  u /= p.Hkv;
  x.s = u % p.n_splits;
  x.b = u / p.n_splits;
  const int sl = __ldg(p.seqlens + x.b);
  x.seqlen = sl > 0 ? sl : 0;
  const int R = p.G * p.seqlen_q;
  x.row0 = x.rt * N;
  x.rows = min(N, R - x.row0);
  int lim = x.seqlen;
  if (p.causal) {
    const int i_last = (x.row0 + x.rows - 1) / p.G;
    lim = min(lim, x.seqlen - p.seqlen_q + i_last + 1);
  }
  x.lim_max = lim > 0 ? lim : 0;
  x.tok0 = x.s * kSplitTokens;
  const int ntok = min(kSplitTokens, x.lim_max - x.tok0);
  x.n_tiles = ntok > 0 ? (ntok + kTileTokens - 1) / kTileTokens : 0;
  return x;
}

template <int D, int N, int NS, int QB>
__global__ void __launch_bounds__(kThreads, 1)
    attn_split_kernel(const __grid_constant__ AttnParams p,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v) {
  using C = Cfg<D, N, NS, QB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  auto *sm = reinterpret_cast<typename C::Small *>(smem + C::kOffSmall);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int *abort_any = &sm->abort_any;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm->full[i], 1);
      mbar_init(&sm->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm->s_full[i], 1);
      mbar_init(&sm->p_full[i], 128);
      mbar_init(&sm->o_full[i], 1);
      mbar_init(&sm->o_free[i], 128);
    }
    for (int i = 0; i < QB; ++i) {
      mbar_init(&sm->q_full[i], 1);
      mbar_init(&sm->q_empty[i], 1);
    }
    mbar_init(&sm->drain, 1);
    sm->abort_any = 0;
    fence_barrier_init();
  }
  {  // the all-ones A operand that turns the row sum of P into an MMA
    uint4 ones = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    for (int i = threadIdx.x; i < C::kOnesBytes / 16; i += kThreads)
      reinterpret_cast<uint4 *>(smem + C::kOffOnes)[i] = ones;
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) tmem_alloc(&sm->tmem_base, C::kTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t sbase = smem_u32(smem);

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------
    // Producer: Q rows of each unit (all 32 lanes), K/V tiles via TMA (lane 0)
    // ------------------------------------------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
    }
    int gi = 0, ui = 0;
    bool failed = false;
    int last_gi[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) last_gi[i] = -1;
    const int R = p.G * p.seqlen_q;
    for (int u = blockIdx.x; u < p.n_units && !failed; u += gridDim.x) {
      const Unit x = unit_at<N>(p, u);
      if (x.n_tiles == 0) continue;
      const int qb = ui % QB;
      bool ok = mbar_wait(&sm->q_empty[qb], ((ui / QB) & 1) ^ 1, abort_any);
      if (__any_sync(0xffffffffu, !ok)) {
        failed = true;
        break;
      }
      uint8_t *qdst = smem + C::kOffQ + qb * C::kQBytes;
      for (int idx = lane; idx < N * (D / 8); idx += 32) {
        const int c = idx / (D / 8), ch = idx % (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c < x.rows) {
          const int r = x.row0 + c;
          const int i = r / p.G, g = r - i * p.G;
          const __nv_bfloat16 *src = p.q + x.b * p.q_sb + static_cast<int64_t>(i) * p.q_ss +
                                     static_cast<int64_t>(x.kvh * p.G + g) * p.q_sh + ch * 8;
          v = __ldg(reinterpret_cast<const uint4 *>(src));
        }
        const int h = ch >> 3, cc = ch & 7;
        *reinterpret_cast<uint4 *>(qdst + h * C::kQHalfBytes + c * 128 + ((cc ^ (c & 7)) << 4)) = v;
      }
      (void)R;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm->q_full[qb]);
        for (int j = 0; j < x.n_tiles; ++j, ++gi) {
          const int st = gi % NS;
          if (!mbar_wait(&sm->empty[st], ((gi / NS) & 1) ^ 1, abort_any)) {
            failed = true;
            break;
          }
          const int tok0 = x.tok0 + j * kTileTokens;
          const int nvalid = min(kTileTokens, x.lim_max - tok0);
          uint8_t *kdst = smem + C::kOffStage + st * C::kStageBytes;
          uint8_t *vdst = kdst + C::kKVBytes;
          int errs = 0;
          for (int k = 0; k * p.box_slots < nvalid; ++k) {
            const int tok = tok0 + k * p.box_slots;
            const int bi = tok >> p.block_shift;
            const int slot = tok & ((1 << p.block_shift) - 1);
            if (bi >= p.max_blocks_per_seq) {
              errs |= kErrTableWidth;
              continue;
            }
            const int blk = __ldg(p.block_table + x.b * p.bt_stride + bi);
            if (blk < 0 || static_cast<int64_t>(blk) >= p.num_blocks) {
              errs |= kErrBadBlock;
              continue;
            }
            mbar_expect_tx(&sm->full[st], 2u * (D / 64) * p.box_slots * 128u);
            const int c1 = p.map_head_first ? x.kvh : slot;
            const int c2 = p.map_head_first ? slot : x.kvh;
#pragma unroll
            for (int h = 0; h < D / 64; ++h) {
              const int off = h * C::kHalfBytes + k * p.box_slots * 128;
              tma_load_4d(kdst + off, &map_k, &sm->full[st], h * 64, c1, c2, blk);
              tma_load_4d(vdst + off, &map_v, &sm->full[st], h * 64, c1, c2, blk);
            }
          }
          mbar_arrive(&sm->full[st]);
          last_gi[st] = gi;
          if (errs && p.err) atomicOr(p.err, errs);
        }
      }
      failed = __any_sync(0xffffffffu, failed);
      ++ui;
    }
    if (failed && lane == 0) {
      // wait (bounded, ignoring the abort flag) for our own copies in flight
      volatile int no_abort = 0;
#pragma unroll
      for (int i = 0; i < NS; ++i)
        if (last_gi[i] >= 0) mbar_wait(&sm->full[i], (last_gi[i] / NS) & 1, &no_abort);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------
    // MMA issuer (one thread)
    // ------------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16(128, N, 0, 0);  // A = K tile, B = Q, both K-major
      constexpr uint32_t kIdescPV = idesc_bf16(128, N, 1, 1);  // A = V^T, B = P^T, both MN-major
      constexpr uint32_t kIdescL = idesc_bf16(128, N, 0, 1);   // A = ones, B = P^T
      const uint32_t tS = tmem, tO = tmem + 2 * N, tL = tmem + 4 * N;
      const uint64_t d_ones = smem_desc(sbase + C::kOffOnes, 128, 256, kLayoutInterleave);
      int gi = 0, ui = 0, prev = -1;
      bool failed = false;
      auto pv_step = [&](int g) -> bool {
        const int st = g % NS, bb = g & 1;
        if (!mbar_wait(&sm->p_full[bb], (g >> 1) & 1, abort_any)) return false;
        if (!mbar_wait(&sm->o_free[bb], ((g >> 1) & 1) ^ 1, abort_any)) return false;
        tc_fence_after_sync();
        const uint32_t vaddr = sbase + C::kOffStage + st * C::kStageBytes + C::kKVBytes;
        const uint32_t paddr = sbase + C::kOffP + bb * 2 * C::kPBytes;
        // P = P_hi + P_lo (two bf16 parts, ~16 significant bits): both the
        // weighted values and the row sums accumulate the hi part, then the lo
        // part, k-step by k-step, in one fixed order.
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          // V^T: MN-major, 128-byte swizzle; 64-wide d groups C::kHalfBytes apart
          // (D = 64: both M halves read the same 64 columns; lanes 64..127 are unused).
          const uint64_t a = smem_desc(vaddr + kk * 2048, D == 128 ? C::kHalfBytes : 0, 1024,
                                       kLayoutSw128);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            // P^T: MN-major, no swizzle; 8-row groups at 128 B (N), 8-token groups at kPKGroup (K).
            const uint64_t bd = smem_desc(paddr + part * C::kPBytes + kk * 2 * C::kPKGroup,
                                          C::kPKGroup, 128, kLayoutInterleave);
            const uint32_t acc = (kk > 0 || part > 0) ? 1u : 0u;
            umma_bf16(tO + bb * N, a, bd, kIdescPV, acc);
            umma_bf16(tL + bb * N, d_ones, bd, kIdescL, acc);
          }
        }
        umma_commit(&sm->o_full[bb]);
        umma_commit(&sm->empty[st]);
        return true;
      };
      for (int u = blockIdx.x; u < p.n_units && !failed; u += gridDim.x) {
        const Unit x = unit_at<N>(p, u);
        if (x.n_tiles == 0) continue;
        const int qb = ui % QB;
        if (!mbar_wait(&sm->q_full[qb], (ui / QB) & 1, abort_any)) {
          failed = true;
          break;
        }
        const uint32_t qaddr = sbase + C::kOffQ + qb * C::kQBytes;
        for (int j = 0; j < x.n_tiles; ++j, ++gi) {
          const int st = gi % NS, bb = gi & 1;
          if (!mbar_wait(&sm->full[st], (gi / NS) & 1, abort_any)) {
            failed = true;
            break;
          }
          tc_fence_after_sync();
          const uint32_t kaddr = sbase + C::kOffStage + st * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int h = kk >> 2, off = (kk & 3) * 32;
            const uint64_t a = smem_desc(kaddr + h * C::kHalfBytes + off, 16, 1024, kLayoutSw128);
            const uint64_t b = smem_desc(qaddr + h * C::kQHalfBytes + off, 16, 1024, kLayoutSw128);
            umma_bf16(tS + bb * N, a, b, kIdescQK, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm->s_full[bb]);
          if (j == x.n_tiles - 1) umma_commit(&sm->q_empty[qb]);
          if (prev >= 0 && !pv_step(prev)) {
            failed = true;
            break;
          }
          prev = gi;
        }
        ++ui;
      }
      if (!failed && prev >= 0) failed = !pv_step(prev);
      if (failed) {
        umma_commit(&sm->drain);
        volatile int no_abort = 0;
        mbar_wait(&sm->drain, 0, &no_abort);
      }
    }
  } else {
    // ------------------------------------------------------------------
    // Softmax + correction + epilogue: 128 threads, thread t <-> TMEM lane t
    // ------------------------------------------------------------------
    const int t = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float NEG_INF = neg_inf();
    float acc[N];
    float m_run = NEG_INF, l_run = 0.f;
    int gi = 0;
    bool stop = false;

    for (int u = blockIdx.x; u < p.n_units && !stop; u += gridDim.x) {
      const Unit x = unit_at<N>(p, u);
      if (x.n_tiles == 0) continue;
      if (t < N) {
        int lim = 0;
        if (t < x.rows) {
          const int i = (x.row0 + t) / p.G;
          lim = x.seqlen;
          if (p.causal) lim = min(lim, x.seqlen - p.seqlen_q + i + 1);
          lim = lim > 0 ? lim : 0;
        }
        sm->lim[t] = lim;
      }
#pragma unroll
      for (int c = 0; c < N; ++c) acc[c] = 0.f;
      m_run = NEG_INF;
      l_run = 0.f;
      if (softmax_bar_or(false)) {
        stop = true;
        break;
      }

      // correction of tile g: fold O_g, L_g into acc, l
      auto correction = [&](int g) -> bool {
        const int bb = g & 1;
        const bool ok = mbar_wait(&sm->o_full[bb], (g >> 1) & 1, abort_any);
        tc_fence_after_sync();
#pragma unroll
        for (int ch = 0; ch < N / 16; ++ch) {
          float o16[16], l16[16];
          tmem_ld16(tmem + lane_off + 2 * N + bb * N + ch * 16, o16);
          tmem_ld16(tmem + lane_off + 4 * N + bb * N + ch * 16, l16);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = ch * 16 + e;
            if (!sm->skip[bb][c]) acc[c] = __fmaf_rn(acc[c], sm->alpha[bb][c], o16[e]);
            if (c == t && !sm->skip[bb][c]) l_run = __fmaf_rn(l_run, sm->alpha[bb][c], l16[e]);
          }
        }
        tc_fence_before_sync();
        mbar_arrive(&sm->o_free[bb]);
        return ok;
      };

      bool fail = false;
      for (int j = 0; j < x.n_tiles; ++j, ++gi) {
        const int bb = gi & 1;
        const bool ok = mbar_wait(&sm->s_full[bb], (gi >> 1) & 1, abort_any);
        tc_fence_after_sync();
        float sv[N];
#pragma unroll
        for (int ch = 0; ch < N / 16; ++ch)
          tmem_ld16(tmem + lane_off + bb * N + ch * 16, *reinterpret_cast<float(*)[16]>(&sv[ch * 16]));
        tmem_ld_wait();
        const int tok = x.tok0 + j * kTileTokens + t;
#pragma unroll
        for (int c = 0; c < N; ++c) sv[c] = (tok < sm->lim[c]) ? __fmul_rn(sv[c], p.cscale) : NEG_INF;
        if (tok >= x.lim_max) {
          // keys past the loaded range: their V rows hold stale bytes (or the
          // cache's NaN tails); zero them so 0 * V stays 0 in P.V.
          uint8_t *vrow = smem + C::kOffStage + (gi % NS) * C::kStageBytes + C::kKVBytes + t * 128;
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              *reinterpret_cast<uint4 *>(vrow + h * C::kHalfBytes + k * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int c = 0; c < N; ++c) {
          const float wm = warp_max(sv[c]);
          if (lane == 0) sm->wmax[warp][c] = wm;
        }
        if (softmax_bar_or(!ok)) {
          fail = true;
          break;
        }
        if (t < N) {
          const float tmax = fmaxf(fmaxf(sm->wmax[0][t], sm->wmax[1][t]),
                                   fmaxf(sm->wmax[2][t], sm->wmax[3][t]));
          const int skip = (tmax == NEG_INF) ? 1 : 0;
          const float mnew = skip ? m_run : fmaxf(m_run, tmax);
          const float alpha = skip ? 1.f : ex2(__fsub_rn(m_run, mnew));
          m_run = mnew;
          sm->mnew[bb][t] = mnew;
          sm->alpha[bb][t] = alpha;
          sm->skip[bb][t] = skip;
        }
        softmax_bar_or(false);
        // P^T row t (MN-major, no swizzle: one 16-byte chunk per 8 rows), as a
        // bf16 hi part and the bf16 rounding of the remainder (lo part).
        uint8_t *prow = smem + C::kOffP + bb * 2 * C::kPBytes + (t >> 3) * C::kPKGroup + (t & 7) * 16;
#pragma unroll
        for (int grp = 0; grp < N / 8; ++grp) {
          uint32_t whi[4], wlo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c0 = grp * 8 + 2 * e;
            const float p0 = (sv[c0] == NEG_INF) ? 0.f : ex2(__fsub_rn(sv[c0], sm->mnew[bb][c0]));
            const float p1 =
                (sv[c0 + 1] == NEG_INF) ? 0.f : ex2(__fsub_rn(sv[c0 + 1], sm->mnew[bb][c0 + 1]));
            __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
            __nv_bfloat162 lo = __floats2bfloat162_rn(__fsub_rn(p0, __low2float(hi)),
                                                      __fsub_rn(p1, __high2float(hi)));
            whi[e] = *reinterpret_cast<uint32_t *>(&hi);
            wlo[e] = *reinterpret_cast<uint32_t *>(&lo);
          }
          *reinterpret_cast<uint4 *>(prow + grp * 128) = make_uint4(whi[0], whi[1], whi[2], whi[3]);
          *reinterpret_cast<uint4 *>(prow + C::kPBytes + grp * 128) =
              make_uint4(wlo[0], wlo[1], wlo[2], wlo[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        mbar_arrive(&sm->p_full[bb]);
        if (j > 0) correction(gi - 1);
      }
      if (fail) {
        stop = true;
        break;
      }
      correction(gi - 1);
      if (softmax_bar_or(false)) {
        stop = true;
        break;
      }
      // epilogue: unnormalised split partial of every real row
      const int64_t S = p.n_splits;
#pragma unroll
      for (int c = 0; c < N; ++c) {
        if (c < x.rows && t < D) {
          const int r = x.row0 + c;
          const int i = r / p.G, g = r - i * p.G;
          const int64_t row_id =
              (static_cast<int64_t>(x.b) * p.seqlen_q + i) * p.Hq + x.kvh * p.G + g;
          p.ws_acc[(row_id * S + x.s) * D + t] = acc[c];
        }
      }
      if (t < x.rows) {
        const int r = x.row0 + t;
        const int i = r / p.G, g = r - i * p.G;
        const int64_t row_id = (static_cast<int64_t>(x.b) * p.seqlen_q + i) * p.Hq + x.kvh * p.G + g;
        p.ws_ml[(row_id * S + x.s) * 2 + 0] = m_run;
        p.ws_ml[(row_id * S + x.s) * 2 + 1] = l_run;
      }
    }
    (void)stop;
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::kTmemCols);
  }
  if (threadIdx.x == 0 && sm->abort_any && p.err) atomicOr(p.err, kErrTimeout);
}

}  // namespace pkv
