// attn_rows.cuh -- split-KV attention with the query rows on the MMA's M axis,
// for calls with many rows per KV head (prefill chunks, multi-token decode).
//
// Same units, tiles and per-row arithmetic as attn_split.cuh -- the reduction
// contract of RL-Kernel PR #284 "feat(attention): add CP backward drift
// validation" (fixed KV chunk merge order, fp32 accumulation), restated so a
// row's bits do not depend on which kernel ran it -- but the tile is laid out
// the other way round: 128 rows r = i * G + g of one KV head against 128 keys,
//   S      = Q * K_tile^T on the tensor cores (M = 128 rows, N = 128 keys),
//   softmax one thread per ROW: all of a row's reductions are in-thread
//           (the row sum replays the 32-key shuffle-down trees and the
//           four-warp combine of attn_split.cuh element for element),
//   P      = [bf16(p) | bf16(p - bf16(p))] written back over S in TMEM,
//   O      = P_hi * V and P_lo * V into two accumulators, with P read from
//           TMEM (A operand) and V from shared memory (MN-major),
//   update acc = fma(O_hi + O_lo, b, acc * a) per row in the correction warpgroup,
//           which owns the row's (m, l, acc[D]) in registers.
// The tensor cores give every output element the same bits whichever operand
// is A and whichever is B (the per-element dot products do not depend on the
// orientation or on N), so S, O_hi and O_lo here equal the transposed
// kernel's S^T, O_hi^T and O_lo^T bit for bit, and so does every row's result.
//
// Roles (512 threads): warps 0-3 / 4-7 softmax warpgroups (even / odd tiles;
// thread t = TMEM lane t = row t of the tile), 8-11 correction + epilogue,
// 12 K producer (+ Q by TMA), 13 V producer, 14 MMA issuer + TMEM owner,
// 15 idle.  Registers are rebalanced per warpgroup (setmaxnreg): the
// correction warpgroup holds a row's D fp32 accumulators.
//
// TMEM (512 columns): kSB S/P buffers of 128 columns (tile gi uses buffer
// gi % kSB, so the QK of tile gi waits only for the P.V of tile gi - kSB; P
// of keys [32 g, 32 g + 32) goes over those keys' own S columns: hi in the
// first 16, lo in the next 16), then O_hi and O_lo (D columns each).  kSB = 2
// at head_dim 128, 3 at 64.
#pragma once

#include <cuda_bf16.h>

#include "attn_split.cuh"
#include "merge.cuh"
#include "ptx.cuh"

namespace pkv {

constexpr int kRowThreads = 512;
constexpr int kRowsPerTile = 128;
constexpr int kRowsSoftmaxRegs = 104;
constexpr int kRowsCorrRegs = 216;
constexpr int kRowsAuxRegs = 88;
constexpr int kRowsLaunchRegs = 128;  // registers per thread the kernel must be built with
static_assert(2 * 128 * kRowsSoftmaxRegs + 128 * kRowsCorrRegs + 128 * kRowsAuxRegs ==
                  kRowThreads * kRowsLaunchRegs,
              "warpgroup register shares must add up to the launch allocation");

template <int D, int NS>
struct RowCfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int kD = D, kN = kRowsPerTile, kNS = NS, kQB = 2;
  static constexpr bool kQTma = true;  // Q rows arrive by TMA
  // a unit's Q buffer is released by its last QK^T alone, so the next unit's
  // Q may be loaded before the current unit's last tile is issued
  static constexpr bool kEarlyQ = true;
  static constexpr int kHalfBytes = kTileTokens * 128;  // 128 keys x 64 head_dim x bf16
  static constexpr int kKVBytes = (D / 64) * kHalfBytes;
  static constexpr int kQHalfBytes = kRowsPerTile * 128;
  static constexpr int kQBytes = (D / 64) * kQHalfBytes;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = NS * kKVBytes;
  static constexpr int kOffQ = 2 * NS * kKVBytes;
  static constexpr int kOffSmall = kOffQ + kQB * kQBytes;
  static constexpr int kSchedScratch = kQB * kQBytes;  // bytes free at kernel start
  struct Small {
    uint64_t full_k[NS], empty_k[NS], full_v[NS], empty_v[NS];
    uint64_t s_full[3], p_full[3], s_free[3], stat_free[3], o_full, o_free;
    uint64_t q_full[2], q_empty[2], drain;
    uint32_t tmem_base;
    int abort_any;
    float tmax[3][kRowsPerTile];  // [buffer][row]: the tile's max (base-2 units)
    float lsum[3][kRowsPerTile];  // [buffer][row]: the tile's sum of p
    int tab[2][2][kSplitTokens / 16];
    int sched_list[kSchedMaxMine];     // this CTA's units (balanced schedule)
    int sched_meta[kSchedMaxMine][3];  // their sequence length and query range
    int sched_hist[kSchedHist], sched_start[kSchedBuckets];
    int sched_count;
  };
  static constexpr int kSmemBytes = kOffSmall + static_cast<int>(sizeof(Small)) + 1024;
  static constexpr int kTmemCols = 512;
  static constexpr int kSB = (512 - 2 * D) / 128;  // S/P buffers next to O_hi and O_lo
  static_assert(kSB == 2 || kSB == 3, "S/P buffers");
  static constexpr uint32_t kColOhi = kSB * 128, kColOlo = kSB * 128 + D;
};

// Row t of a 128-row tile: out / lse through the merge's fold of one split.
template <int D>
__device__ __forceinline__ void write_final_row(const AttnParams &p, const Unit &x, int t,
                                                float m, float l, const float (&acc)[D]) {
  const int r = x.row0 + t;
  const int i = r / p.G, g = r - i * p.G;
  const int h = x.kvh * p.G + g;
  const float NEG_INF = neg_inf();
  float M = NEG_INF, L = 0.f;
  float k_a = 0.f, k_c = 0.f;
  if (m != NEG_INF) {
    const FoldCoef kc = fold_coef(M, m);
    L = fold_val(L, l, kc);
    M = kc.Mn;
    k_a = kc.a;
    k_c = kc.c;
  }
  const bool seen = m != NEG_INF;
  __nv_bfloat16 *o = p.out + o_tok_off(p, x, i) + h * p.o_sh;
  const bool fin = p.fin_out != nullptr && i == x.nq - 1;  // the sequence's last query row
  __nv_bfloat16 *fo = fin ? p.fin_out + x.b * p.fo_sb + h * p.fo_sh : nullptr;
  const float rL = final_rcp(L);
  auto emit = [&](auto div) {
#pragma unroll
    for (int c8 = 0; c8 < D / 8; ++c8) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        v[e] = div(seen ? fold_val(0.f, acc[c8 * 8 + e], FoldCoef{M, k_a, k_c}) : 0.f);
      if (p.out_vec) {
        __nv_bfloat162 h2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) h2[e] = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        *reinterpret_cast<uint4 *>(o + c8 * 8) = *reinterpret_cast<uint4 *>(h2);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) o[c8 * 8 + e] = __float2bfloat16_rn(v[e]);
      }
      if (fin) {
#pragma unroll
        for (int e = 0; e < 8; ++e) fo[c8 * 8 + e] = __float2bfloat16_rn(v[e]);
      }
    }
  };
  // one check of the whole row, then a loop without any IEEE division in it
  // (the quotients are the same either way; see final_out).  The fold of one
  // split multiplies by ex2(0) = 1 and adds 0 * 0, so |A| = |acc|.
  bool fast = seen && L > 0.f;
#pragma unroll
  for (int c = 0; c < D; ++c) fast = fast && final_fast_ok(acc[c], L);
  if (fast)
    emit([&](float A) { return final_out_fast(A, L, rL); });
  else
    emit([&](float A) { return final_out(A, L, rL); });
  const float ls = final_lse(M, L);
  p.lse[lse_index(p, x, i, h)] = ls;
  if (fin) p.fin_lse[static_cast<int64_t>(x.b) * p.Hq + h] = ls;
}

template <int D, int NS>
__global__ void __launch_bounds__(kRowThreads, 1)
    attn_rows_kernel(const __grid_constant__ AttnParams p,
                     const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v,
                     const __grid_constant__ CUtensorMap map_q) {
  using C = RowCfg<D, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  auto *sm = reinterpret_cast<typename C::Small *>(smem + C::kOffSmall);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int *abort_any = &sm->abort_any;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sm->full_k[i], 1);
      mbar_init(&sm->empty_k[i], 1);
      mbar_init(&sm->full_v[i], 1);
      mbar_init(&sm->empty_v[i], 1);
    }
    for (int i = 0; i < C::kSB; ++i) {
      mbar_init(&sm->s_full[i], 1);
      mbar_init(&sm->p_full[i], 4);     // one arrival per softmax warp
      mbar_init(&sm->s_free[i], 1);
      mbar_init(&sm->stat_free[i], 4);  // one arrival per correction warp
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm->q_full[i], 1);
      mbar_init(&sm->q_empty[i], 1);
    }
    mbar_init(&sm->o_full, 1);
    mbar_init(&sm->o_free, 4);
    mbar_init(&sm->drain, 1);
    sm->abort_any = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(&sm->tmem_base, C::kTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sm->tmem_base;
  const uint32_t sbase = smem_u32(smem);
  const float NEG_INF = neg_inf();
  // the Q buffers are not in use yet: the schedule's scratch
  Sched sc = strided_sched(p);
  if (p.sched) {
    build_schedule<kRowsPerTile>(p, smem + C::kOffQ, C::kSchedScratch, sm->sched_hist,
                                 sm->sched_start, sm->sched_list, sm->sched_meta, &sm->sched_count);
    if (sm->sched_count >= 0) sc = Sched{sm->sched_list, sm->sched_meta, sm->sched_count};
  }

  if (warp >= kKWarp) {
    regs_dec<kRowsAuxRegs>();
    if (warp == kKWarp) {
      produce<C>(p, &map_k, &map_q, smem, sm, sm->full_k, sm->empty_k, sm->tab[0], C::kOffK, true,
                 lane, abort_any, sc);
    } else if (warp == kVWarp) {
      produce<C>(p, &map_v, nullptr, smem, sm, sm->full_v, sm->empty_v, sm->tab[1], C::kOffV,
                 false, lane, abort_any, sc);
    } else if (warp == kMmaWarp && lane == 0) {
      // ----------------------------------------------------------------
      // MMA issuer.  Per tile gi: S[gi % kSB] = Q K^T once the K stage has
      // landed and P.V of tile gi - kSB (which read P from the same columns)
      // is done; then P.V of tile gi - (kSB - 1), so that the softmax of
      // kSB - 1 tiles can run while the tensor cores work.
      // ----------------------------------------------------------------
      constexpr uint32_t kIdescQK = idesc_bf16(128, 128, 0, 0);  // A = Q, B = K (K-major)
      constexpr uint32_t kIdescPV = idesc_bf16(128, D, 0, 1);    // A = P (TMEM), B = V (MN-major)
      // (phase parity of the k-th use of buffer gi % kSB is k & 1, k = gi / kSB)
      constexpr int SB = C::kSB;
      int gi = 0, ui = 0, pend0 = -1, pend1 = -1;  // tiles whose P.V is not issued yet
      bool failed = false;
      auto pv_step = [&](int g) -> bool {
        const int st = g % NS, bb = g % SB;
        if (!mbar_wait(&sm->p_full[bb], (g / SB) & 1, abort_any, p.wait_ns)) return false;
        if (!mbar_wait(&sm->o_free, (g & 1) ^ 1, abort_any, p.wait_ns)) return false;
        if (!mbar_wait(&sm->full_v[st], (g / NS) & 1, abort_any, p.wait_ns)) return false;
        tc_fence_after_sync();
        const uint32_t vaddr = sbase + C::kOffV + st * C::kKVBytes;
        const uint32_t pcol = tmem + bb * 128;
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          // V: MN-major (N = head_dim), 128-byte swizzle; 64-wide d groups
          // kHalfBytes apart, 8-key groups 1024 bytes apart.  P_hi of keys
          // [16 kk, 16 kk + 16): TMEM columns 32 (kk / 2) + 8 (kk % 2) + [0, 8),
          // P_lo 16 columns further.
          const uint64_t b = smem_desc(vaddr + kk * 2048, C::kHalfBytes, 1024, kLayoutSw128);
          const uint32_t a = pcol + (kk >> 1) * 32 + (kk & 1) * 8;
          umma_bf16_ts(tmem + C::kColOhi, a, b, kIdescPV, kk > 0 ? 1u : 0u);
          umma_bf16_ts(tmem + C::kColOlo, a + 16, b, kIdescPV, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm->o_full);
        umma_commit(&sm->empty_v[st]);
        umma_commit(&sm->s_free[bb]);
        return true;
      };
      for (int k = 0; k < sc.count && !failed; ++k) {
        const Unit x = sc.get<kRowsPerTile>(p, k);
        if (x.n_tiles == 0) continue;
        const int qb = ui & 1;
        if (!mbar_wait(&sm->q_full[qb], (ui >> 1) & 1, abort_any, p.wait_ns)) {
          failed = true;
          break;
        }
        const uint32_t qaddr = sbase + C::kOffQ + qb * C::kQBytes;
        for (int j = 0; j < x.n_tiles; ++j, ++gi) {
          const int st = gi % NS, bb = gi % SB;
          if (!mbar_wait(&sm->full_k[st], (gi / NS) & 1, abort_any, p.wait_ns) ||
              !mbar_wait(&sm->s_free[bb], ((gi / SB) & 1) ^ 1, abort_any, p.wait_ns)) {
            failed = true;
            break;
          }
          tc_fence_after_sync();
          const uint32_t kaddr = sbase + C::kOffK + st * C::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int h = kk >> 2, off = (kk & 3) * 32;
            const uint64_t a = smem_desc(qaddr + h * C::kQHalfBytes + off, 16, 1024, kLayoutSw128);
            const uint64_t b = smem_desc(kaddr + h * C::kHalfBytes + off, 16, 1024, kLayoutSw128);
            umma_bf16(tmem + bb * 128, a, b, kIdescQK, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm->s_full[bb]);
          umma_commit(&sm->empty_k[st]);
          if (j == x.n_tiles - 1) umma_commit(&sm->q_empty[qb]);
          // keep at most kSB - 1 tiles whose P.V is not issued yet
          if (SB == 2 && pend0 >= 0) {
            if (!pv_step(pend0)) {
              failed = true;
              break;
            }
            pend0 = gi;
          } else if (SB == 3 && pend1 >= 0) {
            if (!pv_step(pend0)) {
              failed = true;
              break;
            }
            pend0 = pend1;
            pend1 = gi;
          } else if (pend0 >= 0) {
            pend1 = gi;
          } else {
            pend0 = gi;
          }
        }
        ++ui;
      }
      if (!failed && pend0 >= 0) failed = !pv_step(pend0);
      if (!failed && pend1 >= 0) failed = !pv_step(pend1);
      // every MMA this thread issued completes before TMEM is released, also
      // when the consumers gave up (bounded wait, default limit)
      (void)failed;
      umma_commit(&sm->drain);
      volatile int no_abort = 0;
      mbar_wait(&sm->drain, 0, &no_abort);
    }
  } else if (warp < kCorrWarp0) {
    // ------------------------------------------------------------------
    // Softmax warpgroups: warpgroup wg takes the tiles with gi % 2 == wg;
    // thread t owns row t.  tmax = exact max of the row's masked scores,
    // p = 2^(s - tmax), P = [bf16(p) | bf16(p - bf16(p))] over S in TMEM,
    // L = the row's sum of the fp32 p in the contract's fixed tree.
    // ------------------------------------------------------------------
    regs_dec<kRowsSoftmaxRegs>();
    const int wg = warp >> 2, wq = warp & 3, t = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t bar_id = 1 + wg;
    int gbase = 0;
    bool stop = false;
    for (int k = 0; k < sc.count && !stop; ++k) {
      const Unit x = sc.get<kRowsPerTile>(p, k);
      if (x.n_tiles == 0) continue;
      int nlim = 0;  // keys [0, nlim) are visible to row t
      if (t < x.rows) {
        const int i = (x.row0 + t) / p.G;
        int lim = x.seqlen;
        if (p.causal) lim = min(lim, x.seqlen - x.nq + i + 1);
        nlim = lim > 0 ? lim : 0;
      }
      for (int j = 0; j < x.n_tiles; ++j) {
        const int gi = gbase + j;
        if ((gi & 1) != wg) continue;
        const int bb = gi % C::kSB, st = gi % NS, par = (gi / C::kSB) & 1;
        bool ok = mbar_wait(&sm->s_full[bb], par, abort_any, p.wait_ns);
        ok = mbar_wait(&sm->stat_free[bb], par ^ 1, abort_any, p.wait_ns) && ok;
        tc_fence_after_sync();
        const int tok0 = x.tok0 + j * kTileTokens;
        const int nvis = min(max(nlim - tok0, 0), kTileTokens);
        const uint32_t srow = tmem + lane_off + bb * 128;  // S of this tile, then its P
        // pass 1: the row's max.  Scaling by cscale > 0 rounds monotonically,
        // so on a fully visible tile max(s) * cscale is the max of the scaled
        // scores exactly.  The branch is taken per WARP (tcgen05.ld is
        // .sync.aligned: all 32 lanes must issue the same load together).
        __syncwarp();
        const bool full = __all_sync(0xffffffffu, nvis == kTileTokens);  // warp-uniform
        float mx = NEG_INF;
        if (full) {
          float raw = NEG_INF;
#pragma unroll 1
          for (int ch = 0; ch < 8; ch += 2) {
            float v0[16], v1[16];
            tmem_ld16(srow + ch * 16, v0);
            tmem_ld16(srow + ch * 16 + 16, v1);
            tmem_ld_wait_for(v0);
            tmem_ld_wait_for(v1);
#pragma unroll
            for (int e = 0; e < 16; ++e) raw = fmaxf(raw, fmaxf(v0[e], v1[e]));
          }
          mx = __fmul_rn(raw, p.cscale);
        } else {
#pragma unroll 1
          for (int ch = 0; ch < 8; ch += 2) {
            float v0[16], v1[16];
            tmem_ld16(srow + ch * 16, v0);
            tmem_ld16(srow + ch * 16 + 16, v1);
            tmem_ld_wait_for(v0);
            tmem_ld_wait_for(v1);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float s0 = (ch * 16 + e < nvis) ? __fmul_rn(v0[e], p.cscale) : NEG_INF;
              const float s1 = (ch * 16 + 16 + e < nvis) ? __fmul_rn(v1[e], p.cscale) : NEG_INF;
              mx = fmaxf(mx, fmaxf(s0, s1));
            }
          }
        }
        // pass 2: p, P_hi / P_lo back into TMEM, and the row sum, 32 keys at
        // a time (one warp's keys in the transposed kernel); the four 32-key
        // sums combine as (w0 + w1) + (w2 + w3)
        float w_even = 0.f, s01 = 0.f, s23 = 0.f;
#pragma unroll 1
        for (int grp = 0; grp < 4; ++grp) {
          float va[16], vb[16];  // keys 32 grp + [0, 16) and + [16, 32)
          tmem_ld16(srow + grp * 32, va);
          tmem_ld16(srow + grp * 32 + 16, vb);
          tmem_ld_wait_for(va);
          tmem_ld_wait_for(vb);
          if (full) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float sa = __fmul_rn(va[e], p.cscale);
              const float sb = __fmul_rn(vb[e], p.cscale);
              va[e] = (sa == NEG_INF) ? 0.f : ex2(__fsub_rn(sa, mx));
              vb[e] = (sb == NEG_INF) ? 0.f : ex2(__fsub_rn(sb, mx));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float sa = (grp * 32 + e < nvis) ? __fmul_rn(va[e], p.cscale) : NEG_INF;
              const float sb = (grp * 32 + 16 + e < nvis) ? __fmul_rn(vb[e], p.cscale) : NEG_INF;
              va[e] = (sa == NEG_INF) ? 0.f : ex2(__fsub_rn(sa, mx));
              vb[e] = (sb == NEG_INF) ? 0.f : ex2(__fsub_rn(sb, mx));
            }
          }
          uint32_t whi[16], wlo[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float x0 = k < 8 ? va[2 * k] : vb[2 * k - 16];
            const float x1 = k < 8 ? va[2 * k + 1] : vb[2 * k - 15];
            __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
            __nv_bfloat162 l2 = __floats2bfloat162_rn(__fsub_rn(x0, __low2float(h2)),
                                                      __fsub_rn(x1, __high2float(h2)));
            whi[k] = *reinterpret_cast<uint32_t *>(&h2);
            wlo[k] = *reinterpret_cast<uint32_t *>(&l2);
          }
          tmem_st16(srow + grp * 32, whi);
          tmem_st16(srow + grp * 32 + 16, wlo);
          // the shuffle-down tree of one warp's 32 keys: offsets 16, 8, 4, 2, 1
#pragma unroll
          for (int e = 0; e < 16; ++e) va[e] = __fadd_rn(va[e], vb[e]);
#pragma unroll
          for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
            for (int e = 0; e < off; ++e) va[e] = __fadd_rn(va[e], va[e + off]);
          if (grp & 1) {
            const float pair = __fadd_rn(w_even, va[0]);
            s01 = grp == 1 ? pair : s01;
            s23 = grp == 3 ? pair : s23;
          } else {
            w_even = va[0];
          }
        }
        if (tok0 + kTileTokens > x.lim_max) {
          // The last tile: keys past the loaded range hold stale bytes or the
          // cache's NaN tails; once V has landed, zero those V rows so that
          // 0 * V stays 0 in P.V.
          ok = mbar_wait(&sm->full_v[st], (gi / NS) & 1, abort_any, p.wait_ns) && ok;
          if (ok && tok0 + t >= x.lim_max) {
            uint8_t *vrow = smem + C::kOffV + st * C::kKVBytes + t * 128;
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
#pragma unroll
              for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4 *>(vrow + h * C::kHalfBytes + k * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        sm->tmax[bb][t] = mx;
        sm->lsum[bb][t] = __fadd_rn(s01, s23);
        if (wg_bar_or(bar_id, !ok)) {
          stop = true;
          break;
        }
        fence_proxy_async_smem();
        __syncwarp();
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->p_full[bb]);
      }
      gbase += x.n_tiles;
    }
    (void)stop;
  } else {
    // ------------------------------------------------------------------
    // Correction + epilogue warpgroup: thread t owns row t's running
    // (m, l, acc[D]).  Per tile, in order: m' = max(m, tmax), a = 2^(m - m'),
    // b = 2^(tmax - m'), acc = fma(O_hi + O_lo, b, acc * a), l = fma(L, b,
    // l * a); a tile the row does not reach (tmax = -inf) leaves it untouched.
    // ------------------------------------------------------------------
    regs_inc<kRowsCorrRegs>();
    const int wq = warp & 3, t = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    constexpr uint32_t bar_id = 3;
    float acc[D];
    int gbase = 0;
    bool stop = false;
    for (int k = 0; k < sc.count && !stop; ++k) {
      const Unit x = sc.get<kRowsPerTile>(p, k);
      if (t == 0) check_sequence(p, x);
      if (x.n_tiles == 0) {
        // rows that see no key: out = 0, lse = -inf (written by the unit of
        // split 0; the merge skips rows of at most one split)
        if (!p.part_only && x.s == 0 && t < x.rows) {
#pragma unroll
          for (int c = 0; c < D; ++c) acc[c] = 0.f;
          write_final_row<D>(p, x, t, NEG_INF, 0.f, acc);
        }
        continue;
      }
#pragma unroll
      for (int c = 0; c < D; ++c) acc[c] = 0.f;
      float m_run = NEG_INF, l_run = 0.f;
      for (int j = 0; j < x.n_tiles; ++j) {
        const int gi = gbase + j, bb = gi % C::kSB, par = (gi / C::kSB) & 1;
        bool ok = mbar_wait(&sm->p_full[bb], par, abort_any, p.wait_ns);  // the tile's row statistics
        ok = mbar_wait(&sm->o_full, gi & 1, abort_any, p.wait_ns) && ok;    // its P.V
        tc_fence_after_sync();
        __syncwarp();  // the waits above spin per thread; the TMEM loads below are warp-wide
        const float tm = sm->tmax[bb][t];
        const float lt = sm->lsum[bb][t];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->stat_free[bb]);
        if (wg_bar_or(bar_id, !ok)) {
          stop = true;
          break;
        }
        const bool skip = !(t < x.rows) || tm == NEG_INF;
        float a = 1.f, b = 0.f;
        if (!skip) {
          const float mn = fmaxf(m_run, tm);
          a = ex2(__fsub_rn(m_run, mn));
          b = ex2(__fsub_rn(tm, mn));
          l_run = __fmaf_rn(lt, b, __fmul_rn(l_run, a));
          m_run = mn;
        }
        const uint32_t orow = tmem + lane_off;
        __syncwarp();
        // two 16-column chunks of O_hi and O_lo per wait (tcgen05.wait::ld
        // waits for every load in flight, so loads are batched, not pipelined)
#pragma unroll
        for (int ch = 0; ch < D / 16; ch += 2) {
          float hi0[16], lo0[16], hi1[16], lo1[16];
          tmem_ld16(orow + C::kColOhi + ch * 16, hi0);
          tmem_ld16(orow + C::kColOlo + ch * 16, lo0);
          tmem_ld16(orow + C::kColOhi + ch * 16 + 16, hi1);
          tmem_ld16(orow + C::kColOlo + ch * 16 + 16, lo1);
          tmem_ld_wait_for(hi0);
          tmem_ld_wait_for(lo0);
          tmem_ld_wait_for(hi1);
          tmem_ld_wait_for(lo1);
          if (ch + 2 == D / 16) {
            // all of O is in registers: the next P.V may overwrite it while
            // the last chunks are folded in
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->o_free);
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {  // branch-free: the loop's TMEM loads are warp-wide
            const float nv0 = __fmaf_rn(__fadd_rn(hi0[e], lo0[e]), b, __fmul_rn(acc[ch * 16 + e], a));
            acc[ch * 16 + e] = skip ? acc[ch * 16 + e] : nv0;
            const float nv1 =
                __fmaf_rn(__fadd_rn(hi1[e], lo1[e]), b, __fmul_rn(acc[ch * 16 + 16 + e], a));
            acc[ch * 16 + 16 + e] = skip ? acc[ch * 16 + 16 + e] : nv1;
          }
        }
      }
      if (stop) break;
      if (t < x.rows) {
        // A row whose visible keys all lie in split 0 is finished here, with
        // the merge's fold of one split; other rows leave a partial.
        const int i = (x.row0 + t) / p.G;
        int lim = x.seqlen;
        if (p.causal) lim = min(lim, x.seqlen - x.nq + i + 1);
        const bool single = !p.part_only && lim <= kSplitTokens;
        if (single) {
          if (x.s == 0) write_final_row<D>(p, x, t, m_run, l_run, acc);
        } else {
          // unnormalised split partial of the row
          const int g = x.row0 + t - i * p.G;
          const int64_t S = p.n_splits;
          const int64_t row_id = (x.q0 + i) * p.Hq + x.kvh * p.G + g;
          float4 *dst = reinterpret_cast<float4 *>(p.ws_acc + (row_id * S + x.s) * D);
#pragma unroll
          for (int c4 = 0; c4 < D / 4; ++c4)
            dst[c4] = make_float4(acc[4 * c4], acc[4 * c4 + 1], acc[4 * c4 + 2], acc[4 * c4 + 3]);
          p.ws_ml[(row_id * S + x.s) * 2 + 0] = m_run;
          p.ws_ml[(row_id * S + x.s) * 2 + 1] = l_run;
        }
      }
      gbase += x.n_tiles;
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
