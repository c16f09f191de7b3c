// attn_rows.cuh -- split-KV attention with the query rows on the MMA's M axis,
// for calls with many rows per KV head (prefill chunks, multi-token decode).
//
// Same units, tiles and per-row arithmetic as attn_split.cuh -- the reduction
// contract of RL-Kernel PR #284 "feat(attention): add CP backward drift
// validation" (fixed KV chunk merge order, fp32 accumulation), restated so a
// row's bits do not depend on which kernel ran it -- but the tile is laid out
// the other way round: 128 rows r = i * G + g of one KV head against 128 keys,
//   S      = Q * K_tile^T on the tensor cores (M = 128 rows, N = 128 keys),
//   softmax one thread per ROW, two warpgroups on every tile (keys
//           [0, 64) and [64, 128)): the halves' maxima meet in shared
//           memory, the running max, the O rescale and l follow
//           attn_split.cuh's rule, and the row sum replays its 32-key
//           shuffle-down trees and four-warp combine element for element,
//   P      = [bf16(p) | bf16(p - bf16(p))] written back over S in TMEM,
//   O      += P_hi * V and P_lo * V into two accumulators that stay in TMEM
//           over the split's tiles, with P read from TMEM (A operand) and V
//           from shared memory (MN-major); acc = O_hi + O_lo at the split's
//           end.
// The tensor cores give every output element the same bits whichever operand
// is A and whichever is B (the per-element dot products do not depend on the
// orientation or on N), so S, O_hi and O_lo here equal the transposed
// kernel's S^T, O_hi^T and O_lo^T bit for bit, and so does every row's result.
//
// Roles (512 threads): warps 0-3 / 4-7 softmax warpgroups (thread t = TMEM
// lane t = row t of the tile; warpgroup 0 keeps the rows' l and rescales
// O_hi, warpgroup 1 rescales O_lo), 8-11 epilogue (a unit's O out of TMEM
// once its last P.V is done, then its out / lse or partials, while the next
// unit's tiles run), 12 K producer (+ Q by TMA), 13 V producer, 14 MMA issuer
// + TMEM owner, 15 idle.  Registers are rebalanced per warpgroup
// (setmaxnreg): the epilogue warpgroup holds a row's D fp32 accumulators.
//
// TMEM (512 columns): kSB S/P buffers of 128 columns (tile gi uses buffer
// gi % kSB, so the QK of tile gi waits only for the P.V of tile gi - kSB; P
// of keys [32 g, 32 g + 32) goes over those keys' own S columns: hi in the
// first 16, lo in the next 16), then O_hi and O_lo (D columns each, one
// unit at a time: the next unit's first P.V waits until the epilogue has read
// O out).  kSB = 2 at head_dim 128, 3 at 64.
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
    uint64_t s_full[3], p_full[3], s_free[3];
    uint64_t ml_full[2];  // [unit parity]: the unit's (m, l) rows are published
    uint64_t ml_free[2];  // [unit parity]: the epilogue has read them
    uint64_t unit_done;   // a unit's last P.V completed (one phase per unit)
    uint64_t o_free;      // O is read out: the next unit's P.V may start it afresh
    uint64_t q_full[2], q_empty[2], drain;
    uint32_t tmem_base;
    int abort_any;
    float xmax[2][2][kRowsPerTile];  // [tile parity][half][row]: the halves' maxima
    float xsum[2][kRowsPerTile];     // [tile parity][row]: the second half's sum of p
    float ml[2][2][kRowsPerTile];    // [unit parity][m, l][row]: the unit's final (m, l)
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
      mbar_init(&sm->p_full[i], 8);  // one arrival per softmax warp
      mbar_init(&sm->s_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm->q_full[i], 1);
      mbar_init(&sm->q_empty[i], 1);
      mbar_init(&sm->ml_full[i], 4);  // one arrival per warp of softmax warpgroup 0
      mbar_init(&sm->ml_free[i], 4);  // one arrival per epilogue warp
    }
    mbar_init(&sm->unit_done, 1);
    mbar_init(&sm->o_free, 4);  // one arrival per correction warp
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
      // a tile whose P.V is not issued yet: its index, whether it opens its
      // unit (P.V starts O afresh) and the unit's ordinal among units with tiles
      struct Pend {
        int g, first, last, uo;
      };
      int gi = 0, ui = 0, npend = 0;
      Pend pend[2] = {{-1, 0, 0, 0}, {-1, 0, 0, 0}};
      bool failed = false;
      auto pv_step = [&](const Pend &pd) -> bool {
        const int g = pd.g, st = g % NS, bb = g % SB;
        if (!mbar_wait(&sm->p_full[bb], (g / SB) & 1, abort_any, p.wait_ns)) return false;
        if (pd.first && !mbar_wait(&sm->o_free, (pd.uo & 1) ^ 1, abort_any, p.wait_ns)) return false;
        if (!mbar_wait(&sm->full_v[st], (g / NS) & 1, abort_any, p.wait_ns)) return false;
        tc_fence_after_sync();
        const uint32_t vaddr = sbase + C::kOffV + st * C::kKVBytes;
        const uint32_t pcol = tmem + bb * 128;
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          // V: MN-major (N = head_dim), 128-byte swizzle; 64-wide d groups
          // kHalfBytes apart, 8-key groups 1024 bytes apart.  P_hi of keys
          // [16 kk, 16 kk + 16): TMEM columns 32 (kk / 2) + 8 (kk % 2) + [0, 8),
          // P_lo 16 columns further.  O accumulates over the unit's tiles.
          const uint64_t b = smem_desc(vaddr + kk * 2048, C::kHalfBytes, 1024, kLayoutSw128);
          const uint32_t a = pcol + (kk >> 1) * 32 + (kk & 1) * 8;
          const uint32_t acc = (pd.first && kk == 0) ? 0u : 1u;
          umma_bf16_ts(tmem + C::kColOhi, a, b, kIdescPV, acc);
          umma_bf16_ts(tmem + C::kColOlo, a + 16, b, kIdescPV, acc);
        }
        umma_commit(&sm->empty_v[st]);
        umma_commit(&sm->s_free[bb]);
        if (pd.last) umma_commit(&sm->unit_done);
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
          if (npend == SB - 1) {
            if (!pv_step(pend[0])) {
              failed = true;
              break;
            }
            pend[0] = pend[1];
            --npend;
          }
          pend[npend++] = Pend{gi, j == 0 ? 1 : 0, j == x.n_tiles - 1 ? 1 : 0, ui};
        }
        ++ui;
      }
      for (int i = 0; i < npend && !failed; ++i) failed = !pv_step(pend[i]);
      // every MMA this thread issued completes before TMEM is released, also
      // when the consumers gave up (bounded wait, default limit)
      (void)failed;
      umma_commit(&sm->drain);
      volatile int no_abort = 0;
      mbar_wait(&sm->drain, 0, &no_abort);
    }
  } else if (warp < kCorrWarp0) {
    // ------------------------------------------------------------------
    // Softmax warpgroups: both take every tile, warpgroup wg its keys
    // [64 wg, 64 wg + 64); thread t owns row t.  tmax = exact max of the
    // row's masked scores (the two halves' maxima exchanged through shared
    // memory); the running max m rises to tmax only when tmax > m + kMaxSlack
    // (a unit starts from -inf), and then O (warpgroup 0: O_hi, 1: O_lo) and
    // l take the factor a = 2^(m - m') before this tile's P.V adds to O;
    // p = 2^(raw * scale - m), P = [bf16(p) | bf16(p - bf16(p))] over S in TMEM; the
    // row's sum of the fp32 p in the contract's fixed tree (each warpgroup's
    // two 32-key sums, then the halves), l = fma(l, a, sum).  Both
    // warpgroups keep m in registers, warpgroup 0 keeps l and publishes the
    // unit's (m, l) for the epilogue.
    // ------------------------------------------------------------------
    regs_dec<kRowsSoftmaxRegs>();
    const int wg = warp >> 2, wq = warp & 3, t = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t ocol = tmem + lane_off + (wg == 0 ? C::kColOhi : C::kColOlo);
    constexpr uint32_t kXchgBar = 1, kDoneBar = 2;  // named barriers over both warpgroups
    int gbase = 0, uo = 0;
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
      float m_run = NEG_INF, l_run = 0.f;
      // warpgroup 0 folds a tile's row sum into l one tile late (it needs
      // warpgroup 1's half, published before the next exchange): the factor
      // and its own half of the tile before
      float a_prev = 1.f, half_prev = 0.f;
      for (int j = 0; j < x.n_tiles; ++j) {
        const int gi = gbase + j;
        const int bb = gi % C::kSB, st = gi % NS, par = (gi / C::kSB) & 1;
        bool ok = mbar_wait(&sm->s_full[bb], par, abort_any, p.wait_ns);
        tc_fence_after_sync();
        const int tok0 = x.tok0 + j * kTileTokens;
        const int nvis = min(max(nlim - tok0, 0), kTileTokens);
        const uint32_t srow = tmem + lane_off + bb * 128;  // S of this tile, then its P
        // pass 1: this half's max over the visible keys, scaled once:
        // scaling by cscale > 0 rounds monotonically, so max(s) * cscale is
        // the max of the scaled scores exactly.  The branch is taken per WARP
        // (tcgen05.ld is .sync.aligned: all 32 lanes issue the same load).
        __syncwarp();
        const bool full = __all_sync(0xffffffffu, nvis == kTileTokens);  // warp-uniform
        float hm = NEG_INF;
        if (full) {
          float raw = NEG_INF;
#pragma unroll 1
          for (int ch = 4 * wg; ch < 4 * wg + 4; ch += 2) {
            float v0[16], v1[16];
            tmem_ld16(srow + ch * 16, v0);
            tmem_ld16(srow + ch * 16 + 16, v1);
            tmem_ld_wait_for(v0);
            tmem_ld_wait_for(v1);
#pragma unroll
            for (int e = 0; e < 16; ++e) raw = fmaxf(raw, fmaxf(v0[e], v1[e]));
          }
          hm = __fmul_rn(raw, p.cscale);
        } else {
          float raw = NEG_INF;
#pragma unroll 1
          for (int ch = 4 * wg; ch < 4 * wg + 4; ch += 2) {
            float v0[16], v1[16];
            tmem_ld16(srow + ch * 16, v0);
            tmem_ld16(srow + ch * 16 + 16, v1);
            tmem_ld_wait_for(v0);
            tmem_ld_wait_for(v1);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float s0 = (ch * 16 + e < nvis) ? v0[e] : NEG_INF;
              const float s1 = (ch * 16 + 16 + e < nvis) ? v1[e] : NEG_INF;
              raw = fmaxf(raw, fmaxf(s0, s1));
            }
          }
          hm = __fmul_rn(raw, p.cscale);
        }
        sm->xmax[gi & 1][wg][t] = hm;
        // both halves' maxima are published (and a failed wait is known to
        // both warpgroups, which then stop together)
        if (named_bar_or(kXchgBar, 256, !ok)) {
          stop = true;
          break;
        }
        if (wg == 0 && j > 0)
          l_run = __fmaf_rn(l_run, a_prev, __fadd_rn(half_prev, sm->xsum[(gi - 1) & 1][t]));
        const float mx = fmaxf(hm, sm->xmax[gi & 1][wg ^ 1][t]);
        const float m_prev = m_run;
        const float m_new = (mx > __fadd_rn(m_prev, kMaxSlack)) ? mx : m_prev;
        m_run = m_new;
        const float a = (m_prev == NEG_INF || m_new == m_prev) ? 1.f : ex2(__fsub_rn(m_prev, m_new));
        if (__any_sync(0xffffffffu, a != 1.f)) {
          // a != 1 only past the unit's first tile: O holds its tiles < gi.
          // P.V(gi - 1) completes on s_free[(gi - 1) % kSB]; that barrier's
          // previous phase (tile gi - 1 - kSB) completed before S(gi) could be
          // written, so this parity wait cannot alias an older phase.
          ok = mbar_wait(&sm->s_free[(gi - 1) % C::kSB], ((gi - 1) / C::kSB) & 1, abort_any,
                         p.wait_ns) && ok;
          if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after_sync();
#pragma unroll 1
            for (int ch = 0; ch < D / 16; ch += 2) {
              float o0[16], o1[16];
              tmem_ld16(ocol + ch * 16, o0);
              tmem_ld16(ocol + ch * 16 + 16, o1);
              tmem_ld_wait_for(o0);
              tmem_ld_wait_for(o1);
              uint32_t w0[16], w1[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                w0[e] = __float_as_uint(__fmul_rn(o0[e], a));
                w1[e] = __float_as_uint(__fmul_rn(o1[e], a));
              }
              tmem_st16(ocol + ch * 16, w0);
              tmem_st16(ocol + ch * 16 + 16, w1);
            }
          }
        }
        // pass 2: p, P_hi / P_lo back into TMEM, and this half's sum, 32 keys
        // at a time (one warp's keys in the transposed kernel); the four
        // 32-key sums combine as (w0 + w1) + (w2 + w3)
        float w_even = 0.f, half = 0.f;
#pragma unroll 1
        for (int grp = 2 * wg; grp < 2 * wg + 2; ++grp) {
          float va[16], vb[16];  // keys 32 grp + [0, 16) and + [16, 32)
          tmem_ld16(srow + grp * 32, va);
          tmem_ld16(srow + grp * 32 + 16, vb);
          tmem_ld_wait_for(va);
          tmem_ld_wait_for(vb);
          // p = 2^(raw * cscale - m), one rounding before ex2; masked keys 0
          const float nm = -m_new;
          if (full) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              va[e] = ex2(__fmaf_rn(va[e], p.cscale, nm));
              vb[e] = ex2(__fmaf_rn(vb[e], p.cscale, nm));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              va[e] = (grp * 32 + e < nvis) ? ex2(__fmaf_rn(va[e], p.cscale, nm)) : 0.f;
              vb[e] = (grp * 32 + 16 + e < nvis) ? ex2(__fmaf_rn(vb[e], p.cscale, nm)) : 0.f;
            }
          }
          uint32_t whi[16], wlo[16];
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            const float x0 = k2 < 8 ? va[2 * k2] : vb[2 * k2 - 16];
            const float x1 = k2 < 8 ? va[2 * k2 + 1] : vb[2 * k2 - 15];
            __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
            __nv_bfloat162 l2 = __floats2bfloat162_rn(__fsub_rn(x0, __low2float(h2)),
                                                      __fsub_rn(x1, __high2float(h2)));
            whi[k2] = *reinterpret_cast<uint32_t *>(&h2);
            wlo[k2] = *reinterpret_cast<uint32_t *>(&l2);
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
          if (grp & 1)
            half = __fadd_rn(w_even, va[0]);
          else
            w_even = va[0];
        }
        if (wg == 1) sm->xsum[gi & 1][t] = half;
        const bool last = j == x.n_tiles - 1;
        if (wg == 0 && tok0 + kTileTokens > x.lim_max) {  // (only a unit's last tile)
          // The last tile: keys past the loaded range hold stale bytes or the
          // cache's NaN tails; once V has landed, zero those V rows so that
          // 0 * V stays 0 in P.V.
          ok = mbar_wait(&sm->full_v[st], (gi / NS) & 1, abort_any, p.wait_ns) && ok;
          if (ok && tok0 + t >= x.lim_max) {
            uint8_t *vrow = smem + C::kOffV + st * C::kKVBytes + t * 128;
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
#pragma unroll
              for (int k2 = 0; k2 < 8; ++k2)
                *reinterpret_cast<uint4 *>(vrow + h * C::kHalfBytes + k2 * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        if (last) {
          // the unit's last tile: both halves' sums and any failed wait are
          // known to both warpgroups
          if (named_bar_or(kDoneBar, 256, !ok)) {
            stop = true;
            break;
          }
          if (wg == 0) {
            l_run = __fmaf_rn(l_run, a, __fadd_rn(half, sm->xsum[gi & 1][t]));
            // the slot of unit uo - 2 has been read by the epilogue (this wait
            // also keeps ml_full at most one phase ahead of its waiter)
            ok = mbar_wait(&sm->ml_free[uo & 1], ((uo >> 1) & 1) ^ 1, abort_any, p.wait_ns) && ok;
            sm->ml[uo & 1][0][t] = m_run;
            sm->ml[uo & 1][1][t] = l_run;
          }
        } else {
          a_prev = a;
          half_prev = half;
        }
        fence_proxy_async_smem();
        __syncwarp();
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm->p_full[bb]);
          if (wg == 0 && last) mbar_arrive(&sm->ml_full[uo & 1]);
        }
      }
      gbase += x.n_tiles;
      ++uo;
    }
    (void)stop;
  } else {
    // ------------------------------------------------------------------
    // Epilogue warpgroup: thread t takes row t of each unit once its last
    // P.V is done: (m, l) from the softmax warpgroups, acc = O_hi + O_lo out
    // of TMEM (O is then free for the next unit), and the row's out / lse or
    // split partial -- while the next unit's tiles already run.
    // ------------------------------------------------------------------
    regs_inc<kRowsCorrRegs>();
    const int wq = warp & 3, t = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t orow = tmem + lane_off;
    constexpr uint32_t bar_id = 3;
    float acc[D];
    int gbase = 0, uo = 0;
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
      // the unit's (m, l), then its last P.V (one unit_done phase per unit)
      bool ok = mbar_wait(&sm->ml_full[uo & 1], (uo >> 1) & 1, abort_any, p.wait_ns);
      const float m_run = sm->ml[uo & 1][0][t];
      const float l_run = sm->ml[uo & 1][1][t];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm->ml_free[uo & 1]);
      ok = mbar_wait(&sm->unit_done, uo & 1, abort_any, p.wait_ns) && ok;
      if (wg_bar_or(bar_id, !ok)) {
        stop = true;
        break;
      }
      tc_fence_after_sync();
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
          // all of O is in registers: the next unit's P.V may overwrite it
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm->o_free);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          acc[ch * 16 + e] = __fadd_rn(hi0[e], lo0[e]);
          acc[ch * 16 + 16 + e] = __fadd_rn(hi1[e], lo1[e]);
        }
      }
      ++uo;
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
