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
};

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
// Final write of a folded row: out element and lse.
__device__ __forceinline__ float final_out(float A, float L) {
  return L > 0.f ? __fdiv_rn(A, L) : 0.f;
}
__device__ __forceinline__ float final_lse(float M, float L) {
  return L > 0.f ? __fmul_rn(__fadd_rn(M, log2f(L)), 0.69314718055994531f)
                 : __int_as_float(0xff800000);
}

template <int D>
__global__ void __launch_bounds__(D) merge_kernel(const __grid_constant__ MergeParams p) {
  const int64_t row = blockIdx.x;  // (b * seqlen_q + i) * Hq + h
  const int h = static_cast<int>(row % p.Hq);
  const int64_t bi = row / p.Hq;
  const int i = static_cast<int>(bi % p.seqlen_q);
  const int b = static_cast<int>(bi / p.seqlen_q);
  const int n = max(__ldg(p.seqlens + b), 0);
  int lim = n;
  if (p.causal) lim = min(lim, n - p.seqlen_q + i + 1);
  lim = max(lim, 0);
  const int n_s = min((lim + 4095) / 4096, p.n_splits);
  const int d = threadIdx.x;
  const float NEG_INF = __int_as_float(0xff800000);
  const float *ml = p.ws_ml + row * p.n_splits * 2;
  const float *ap = p.ws_acc + row * p.n_splits * D + d;
  float M = NEG_INF, L = 0.f, A = 0.f;
  // Partials are fetched kBatch splits at a time (independent loads in
  // flight together) and folded strictly in ascending split order.
  constexpr int kBatch = 16;
  for (int s0 = 0; s0 < n_s; s0 += kBatch) {
    float ms[kBatch], ls[kBatch], as[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int s = s0 + k;
      ms[k] = s < n_s ? ml[2 * s] : NEG_INF;
      ls[k] = s < n_s ? ml[2 * s + 1] : 0.f;
      as[k] = s < n_s ? ap[static_cast<int64_t>(s) * D] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (ms[k] == NEG_INF) continue;  // the row sees no key of this split
      const FoldCoef kc = fold_coef(M, ms[k]);
      L = fold_val(L, ls[k], kc);
      A = fold_val(A, as[k], kc);
      M = kc.Mn;
    }
  }
  p.out[b * p.o_sb + i * p.o_ss + h * p.o_sh + d] = __float2bfloat16_rn(final_out(A, L));
  if (d == 0) p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.seqlen_q + i] = final_lse(M, L);
}

}  // namespace pkv
