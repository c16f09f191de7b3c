// merge.cuh -- deterministic merge of split partials and final write.
//
// For one output row (batch b, query token i, query head h) the partials
// (m_s, l_s, acc_s[D]) of splits s = 0, 1, ... are folded in ascending split
// order -- the fixed global_block_index merge order, fp32 accumulation and
// final-write downcast named in RL-Kernel PR #284 "feat(attention): add CP
// backward drift validation", Changes:
//
//   M' = max(M, m_s), a = 2^(M - M'), c = 2^(m_s - M')
//   L  = fma(l_s, c, L * a),  A = fma(acc_s, c, A * a),  M = M'
//   out = bf16_rn(A / L),     lse = (M + log2 L) * ln 2   (L = 0: out 0, lse -inf)
//
// m_s is in base-2 scaled units (scale * log2(e) * q.k), so lse comes out in
// the natural-log, scale * q.k domain.  The same code merges every row of
// every entry point, and a single split goes through it too.
#pragma once

#include <cuda_bf16.h>

#include "contract.cuh"
#include "packed.cuh"
#include "ptx.cuh"

namespace pkv {

struct MergeParams {
  const int32_t *seqlens;
  int seqlen_q, Hq, n_splits, causal;
  const float *ws_acc;
  const float *ws_ml;
  __nv_bfloat16 *out;
  int64_t o_sb, o_ss, o_sh;
  float *lse;
  // packed queries (as AttnParams): rows are token-major over the packed
  // tokens, lse [Hq, total_q]; the last query row of each sequence is also
  // written to fin_out / fin_lse when they are given
  const int32_t *cu_q;
  int batch, total_q;
  __nv_bfloat16 *fin_out;
  int64_t fo_sb, fo_sh;
  float *fin_lse;
  int64_t rows;     // output rows (tokens x Hq)
  int skip_single;  // rows of at most one split were finished by the split kernel ...
  int skip_min_nq;  // ... for sequences with at least this many queries
  // Partials of global split s live in block r = s / n_local (local split
  // s % n_local) -- one block per context-parallel rank, gathered side by
  // side rank_floats floats apart; a single call has one block (n_local =
  // n_splits).  Within a block: acc [rows][n_local][D], ml [rows][n_local][2].
  int n_local;
  int64_t rank_floats;
};

constexpr int kMergeRowsPerBlock = 8;  // one warp per row

// One step of the ascending fold: partial (m_s, l_s, x_s) into (M, L, X).
struct FoldCoef {
  float Mn, a, c;
};
__device__ __forceinline__ FoldCoef fold_coef(float M, float m_s) {
  const float Mn = fmaxf(M, m_s);
  return FoldCoef{Mn, ex2(__fsub_rn(M, Mn)), ex2(__fsub_rn(m_s, Mn))};
}
__device__ __forceinline__ float fold_val(float X, float x_s, const FoldCoef &k) {
  return __fmaf_rn(x_s, k.c, __fmul_rn(X, k.a));
}
// Final write of a folded row: out element and lse.  out = A / L rounded to
// nearest (the IEEE quotient), from the row's reciprocal rL = final_rcp(L),
// taken once per row, by two residual corrections:
//   q0 = A rL,  q1 = q0 + (A - L q0) rL,  out = q1 + (A - L q1) rL
// (each step one rounding; the residuals by FMA).  rL is the correctly
// rounded 1 / L and q1 lies within one ulp of A / L, so the residual A - L q1
// is exact and the last step rounds to the correctly rounded quotient
// (Markstein's theorem: P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; J.-M.
// Muller et al., Handbook of Floating-Point Arithmetic, division with an
// FMA).  The theorem needs every intermediate in the normal range:
// final_fast_ok holds for |A| in [2^-90, 2^96] and L in [2^-20, 2^40] (a row
// that saw a key has L >= 1), and for A = +-0, whose quotient is A rL itself;
// other operands (subnormal, infinite or NaN A) take the IEEE division.
// Either way the bits are __fdiv_rn(A, L)'s.
__device__ __forceinline__ float final_rcp(float L) { return L > 0.f ? __frcp_rn(L) : 0.f; }
__device__ __forceinline__ bool final_fast_ok(float A, float L) {
  const float aa = fabsf(A);
  return (aa == 0.f || (aa >= 0x1p-90f && aa <= 0x1p96f)) && L >= 0x1p-20f && L <= 0x1p40f;
}
__device__ __forceinline__ float final_out_fast(float A, float L, float rL) {
  const float q0 = __fmul_rn(A, rL);
  const float q1 = __fmaf_rn(__fmaf_rn(-L, q0, A), rL, q0);
  const float q2 = __fmaf_rn(__fmaf_rn(-L, q1, A), rL, q1);
  return A == 0.f ? q0 : q2;
}
__device__ __forceinline__ float final_out(float A, float L, float rL) {
  if (!(L > 0.f)) return 0.f;
  return final_fast_ok(A, L) ? final_out_fast(A, L, rL) : __fdiv_rn(A, L);
}
__device__ __forceinline__ float final_lse(float M, float L) {
  return L > 0.f ? __fmul_rn(__fadd_rn(M, log2f(L)), 0.69314718055994531f)
                 : __int_as_float(0xff800000);
}

// Two launch shapes, the same per-element arithmetic (every element runs the
// fold above in ascending split order):
//   WIDE = false: one warp per output row, 8 rows per block; lane l owns
//                 head_dim elements [l V, l V + V), V = D / 32 (many rows);
//   WIDE = true:  one block of D threads per row, V = 1 (few rows, many
//                 splits: more SMs share the partial reads).
// One output row (row = token * Hq + h; token = b * seqlen_q + i, or packed)
// by one block (WIDE) or one warp; `lane` is the thread's index in it.
template <int D, bool WIDE>
__device__ __forceinline__ void merge_row(const MergeParams &p, int64_t row, int lane) {
  constexpr int V = WIDE ? 1 : D / 32;
  const int h = static_cast<int>(row % p.Hq);
  const int64_t tok = row / p.Hq;
  int b, i, nq;
  if (p.cu_q) {
    b = seq_of_token(p.cu_q, p.batch, tok);
    const int a = __ldg(p.cu_q + b);
    i = static_cast<int>(tok - a);
    nq = __ldg(p.cu_q + b + 1) - a;
    if (i >= p.seqlen_q) return;  // past the host bound: flagged by the split kernel
  } else {
    i = static_cast<int>(tok % p.seqlen_q);
    b = static_cast<int>(tok / p.seqlen_q);
    nq = p.seqlen_q;
  }
  const int n = max(__ldg(p.seqlens + b), 0);
  int lim = n;
  if (p.causal) lim = min(lim, n - nq + i + 1);
  lim = max(lim, 0);
  const int n_s = min(splits_for(lim), p.n_splits);
  if (p.skip_single && nq >= p.skip_min_nq && n_s <= 1) return;
  const int d0 = lane * V;
  const float NEG_INF = __int_as_float(0xff800000);
  float M = NEG_INF, L = 0.f, A[V];
#pragma unroll
  for (int j = 0; j < V; ++j) A[j] = 0.f;
  // Partials are fetched kBatch splits at a time (independent loads in
  // flight together) and folded strictly in ascending split order.
  constexpr int kBatch = 16;
  for (int s0 = 0; s0 < n_s; s0 += kBatch) {
    float ms[kBatch], ls[kBatch], as[kBatch][V];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int s = s0 + k;
      ms[k] = NEG_INF;
      ls[k] = 0.f;
#pragma unroll
      for (int j = 0; j < V; ++j) as[k][j] = 0.f;
      if (s < n_s) {
        const int r = p.rank_floats == 0 ? 0 : s / p.n_local;  // one block: no division
        const int64_t e = r * p.rank_floats;  // this rank's block, in floats
        const int64_t slot = row * p.n_local + (s - r * p.n_local);
        ms[k] = p.ws_ml[e + slot * 2];
        ls[k] = p.ws_ml[e + slot * 2 + 1];
        const float *ap = p.ws_acc + e + slot * D + d0;
        if constexpr (V == 4) {
          const float4 v = *reinterpret_cast<const float4 *>(ap);
          as[k][0] = v.x; as[k][1] = v.y; as[k][2] = v.z; as[k][3] = v.w;
        } else if constexpr (V == 2) {
          const float2 v = *reinterpret_cast<const float2 *>(ap);
          as[k][0] = v.x; as[k][1] = v.y;
        } else {
          as[k][0] = *ap;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (ms[k] == NEG_INF) continue;  // the row sees no key of this split
      const FoldCoef kc = fold_coef(M, ms[k]);
      L = fold_val(L, ls[k], kc);
#pragma unroll
      for (int j = 0; j < V; ++j) A[j] = fold_val(A[j], as[k][j], kc);
      M = kc.Mn;
    }
  }
  const float ls = final_lse(M, L);
  const float rL = final_rcp(L);
  __nv_bfloat16 *o = p.cu_q ? p.out + tok * p.o_ss + h * p.o_sh
                            : p.out + b * p.o_sb + i * p.o_ss + h * p.o_sh;
  const bool fin = p.fin_out != nullptr && i == nq - 1;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const __nv_bfloat16 ob = __float2bfloat16_rn(final_out(A[j], L, rL));
    o[d0 + j] = ob;
    if (fin) p.fin_out[b * p.fo_sb + h * p.fo_sh + d0 + j] = ob;
  }
  if (lane == 0) {
    if (p.cu_q)
      p.lse[static_cast<int64_t>(h) * p.total_q + tok] = ls;
    else
      p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.seqlen_q + i] = ls;
    if (fin) p.fin_lse[static_cast<int64_t>(b) * p.Hq + h] = ls;
  }
}

// WIDE: one block per row.  Otherwise one warp per row, the warps of the grid
// striding over the rows (a few blocks per SM: most rows of a packed call may
// only need the check that the row-major kernel finished them).
template <int D, bool WIDE>
__global__ void __launch_bounds__(WIDE ? D : 32 * kMergeRowsPerBlock)
    merge_kernel(const __grid_constant__ MergeParams p) {
  if constexpr (WIDE) {
    if (static_cast<int64_t>(blockIdx.x) < p.rows) merge_row<D, true>(p, blockIdx.x, threadIdx.x);
  } else {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kMergeRowsPerBlock;
    for (int64_t row = static_cast<int64_t>(blockIdx.x) * kMergeRowsPerBlock + (threadIdx.x >> 5);
         row < p.rows; row += stride)
      merge_row<D, false>(p, row, threadIdx.x & 31);
  }
}

}  // namespace pkv
