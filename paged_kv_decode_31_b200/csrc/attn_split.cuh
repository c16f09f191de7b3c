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
//            the tile's column max tmax over its 128 tokens (exact,
//            order-free); the row's running max m (-inf at the split's
//            start) rises to tmax only when tmax > m + kMaxSlack, and then
//            the row's O^T column takes the factor a = 2^(m - m') in TMEM
//            (an fp32 multiply) before this tile's P.V adds to it;
//            p = 2^(raw * scale - m) (one fused multiply-add); P^T holds p
//            as two bf16 parts side by side,
//            hi = bf16(p) and lo = bf16(p - hi), so the tensor cores see p to
//            ~16 bits; the fp32 p of each row are summed in one fixed
//            shuffle tree (the row sum never sees P's rounding), and
//            l = fma(l, a, sum);
//   O^T      += V^T * [P_hi | P_lo]^T on the tensor cores: O_hi and O_lo
//            accumulate in TMEM over the split's tiles (the first tile
//            starts them afresh), and acc = O_hi + O_lo in fp32 once, at the
//            split's end.
// Tiles start at absolute multiples of 128 and rows never influence each
// other, so a row's arithmetic depends only on its own query, its visible
// keys and the fixed constants: decode row t and prefill row t, batch 1 and
// batch N, contiguous and interleaved caches all give the same bits.
//
// Roles (480 threads): warps 0-3 / 4-7 softmax warpgroups on alternating
// tiles (thread t = TMEM lane t = token t of the tile; each passes its
// tile's running maxima to the other), warps 8-11 correction + epilogue (the
// rows' l per tile; at a unit's end thread t = output column d), warp 12 K
// producer (+ Q staging), warp 13 V producer, warp 14 MMA issuer (+ TMEM
// owner).  K and V have their own stage rings, so a K stage is refilled as
// soon as its S^T is computed; O^T has a buffer per unit parity, so a unit's
// read-out overlaps the next unit's tiles.  The kernel is persistent, with
// its units dealt by a balanced schedule; producers and the MMA issuer run
// ahead across unit boundaries.
#pragma once

#include <cuda_bf16.h>

#include "contract.cuh"
#include "merge.cuh"
#include "ptx.cuh"

namespace pkv {

constexpr int kThreads = 480;  // 15 warps
// warps 0-3 and 4-7: softmax warpgroups (even / odd tiles of the CTA's sequence)
constexpr int kCorrWarp0 = 8;  // warps 8-11: correction + epilogue warpgroup
constexpr int kKWarp = 12;     // K producer (+ Q staging)
constexpr int kVWarp = 13;     // V producer
constexpr int kMmaWarp = 14;   // MMA issuer + TMEM owner

// Balanced schedule limits (see build_schedule): units with work per CTA,
// and the tile-count buckets of the sort.  The units per call are bounded by
// each kernel's scratch (one byte per unit).
constexpr int kSchedMaxMine = 128;
constexpr int kSchedBuckets = kSplitTokens / kTileTokens + 1;  // tile counts 0 .. 32
constexpr int kSchedHist = kSchedBuckets + 3;                  // + min, max, units kept

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
  int max_seqlen_k;     // host bound on seqlens (n_splits = ceil(max_seqlen_k / 4096))
  uint64_t wait_ns;     // limit of every pipeline wait (kWaitTimeoutNs unless a debug call lowers it)
  float cscale;         // softmax scale * log2(e)
  int causal;
  float *ws_acc;        // [rows][n_splits][D]
  float *ws_ml;         // [rows][n_splits][2] (max in base-2 scaled units, sum)
  int32_t *err;
  // Fused append (n_new > 0): token t of k_new/v_new [batch, n_new, Hkv, D] is
  // written to position seqlens[b] - n_new + t before it is read.
  int n_new;
  const uint16_t *k_new, *v_new;
  int64_t kn_sb, kn_st, kn_sh, vn_sb, vn_st, vn_sh;
  uint16_t *k_cache, *v_cache;
  int64_t k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
  // Final write by the row-major kernel (rows of at most one split): out /
  // lse written with the merge's arithmetic.  direct: every row of the call
  // has at most one split (host side: no merge launch).
  int direct, out_vec;
  // sched: the kernel builds the balanced unit order (host: at most one unit
  // per byte of the kernel's schedule scratch); otherwise units are dealt
  // with stride gridDim.x
  int sched;
  __nv_bfloat16 *out;
  int64_t o_sb, o_ss, o_sh;
  float *lse;
  // Packed (varlen) queries, cu_q != null: sequence b's query tokens are the
  // tokens cu_q[b] .. cu_q[b+1] - 1 of q and out (token stride q_ss / o_ss),
  // lse is [Hq, total_q], and seqlen_q is the host bound on every sequence's
  // query count.  Dense (cu_q == null): q / out are [batch, seqlen_q, ...],
  // lse [batch, Hq, seqlen_q].
  const int32_t *cu_q;
  int total_q;
  // Optional copy of each sequence's last query row (its "final" row):
  // fin_out [batch, Hq, D] (strides fo_sb, fo_sh), fin_lse [batch, Hq].
  __nv_bfloat16 *fin_out;
  int64_t fo_sb, fo_sh;
  float *fin_lse;
  // Split range: the units cover absolute splits split_base .. split_base +
  // n_splits - 1 (one rank's share under context parallelism; 0 otherwise);
  // partials are stored by local split.  part_only: every row leaves
  // partials, none is finished in the split kernel.
  int split_base, part_only;
  // Packed calls may be served by two launches: this launch handles the
  // sequences with nq_lo <= query count <= nq_hi (dense: all).
  int nq_lo, nq_hi;
};

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// Named barrier `id` over one warpgroup (128 threads) that also ORs a
// predicate across it, so an abort decision is taken by the whole warpgroup
// at the same barrier.
__device__ __forceinline__ bool wg_bar_or(uint32_t id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id)
      : "memory");
  return r != 0;
}

// Cross-lane reductions over the 32 tokens of a warp, four columns at a time
// so the shuffles of the four columns overlap.  Each column's tree is fixed.
// Maximum: xor butterfly (max is exact, every lane ends with the same value).
__device__ __forceinline__ void warp_max4(float (&v)[4]) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __shfl_xor_sync(0xffffffffu, v[i], off);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = fmaxf(v[i], o[i]);
  }
}

// Sum: shift-down tree; lane 0 holds the result.
__device__ __forceinline__ void warp_sum4_lane0(float (&v)[4]) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    float o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __shfl_down_sync(0xffffffffu, v[i], off);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __fadd_rn(v[i], o[i]);
  }
}

// Shared-memory plan.  Every operand region is 1024-byte aligned (the 128-byte
// swizzle pattern repeats every 8 rows of 128 bytes).
template <int D, int N, int NS, int QB>
struct Cfg {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static_assert(N == 16 || N == 32 || N == 64, "rows per tile");
  static_assert(QB == 1 || QB == 2, "Q buffers");
  static constexpr int kD = D, kN = N, kNS = NS, kQB = QB;
  static constexpr bool kQTma = false;  // Q rows staged with plain loads
  // Two Q buffers: the epilogue of a unit is staged in its Q buffer, so the
  // next unit's Q is loaded only after the current unit's last tile is issued
  // (see produce()).
  static constexpr bool kEarlyQ = false;
  static constexpr int kHalfBytes = kTileTokens * 128;   // 128 tokens x 64 head_dim x bf16
  static constexpr int kKVBytes = (D / 64) * kHalfBytes;  // one K (or V) tile
  static constexpr int kQHalfBytes = N * 128;
  static constexpr int kQBytes = (D / 64) * kQHalfBytes;
  static constexpr int kPCols = 2 * N;                    // P^T columns: N hi, then N lo
  static constexpr int kPBytes = kTileTokens * kPCols * 2;
  static constexpr int kPKGroup = (kPCols / 8) * 128;     // P^T stride between 8-token groups
  static constexpr int kOffK = 0;
  static constexpr int kOffV = NS * kKVBytes;
  static constexpr int kOffQ = 2 * NS * kKVBytes;
  static constexpr int kOffP = kOffQ + QB * kQBytes;
  static constexpr int kOffSmall = kOffP + 2 * kPBytes;
  static constexpr int kSchedScratch = 2 * kPBytes;  // bytes free at kernel start
  struct Small {
    uint64_t full_k[NS], empty_k[NS], full_v[NS], empty_v[NS];
    uint64_t s_full[2], p_full[2], o_full[2], stat_free[2];
    uint64_t m_full[2];     // [tile parity]: the tile's running maxima are published
    uint64_t unit_done[2];  // [O buffer]: a unit's last P.V completed
    uint64_t o_free[2];     // [O buffer]: the unit's O is read out
    uint64_t q_full[QB], q_empty[QB], drain;
    uint32_t tmem_base;
    int abort_any;
    __align__(16) float wmax[2][2][4][N];  // [softmax warpgroup][tile parity][warp][row]
    __align__(16) float wsum[2][4][N];     // [buffer][warp][row]: per-warp sums of p
    float mnew[2][N];                      // [buffer][row]: the running max after the tile
    float scl[2][N];                       // [buffer][row]: factor O and l take before it
    float mrun[2][N];                      // [tile parity][row]: mnew for the next tile
    float fin_m[N], fin_l[N];              // each row's (m, l) for the direct final write
    int sched_list[kSchedMaxMine];         // this CTA's units (balanced schedule)
    int sched_meta[kSchedMaxMine][3];      // their sequence length and query range
    int sched_hist[kSchedHist], sched_start[kSchedBuckets];
    int sched_count;
    int lim[2][N];                         // [softmax warpgroup][row]: key limit
    int tab[2][2][kSplitTokens / 16];      // [producer][unit parity]: block-table entries
  };
  static constexpr int kSmemBytes = kOffSmall + static_cast<int>(sizeof(Small)) + 1024;
  // TMEM: S^T (N columns) x 2 buffers, then O^T (hi and lo, 2N columns) x 2
  // buffers (alternate units)
  static constexpr int kTmemCols = (6 * N <= 128) ? 128 : (6 * N <= 256) ? 256 : 512;
};

struct Unit {
  int b, kvh, rt, s;
  int nq;       // query tokens of sequence b
  int64_t q0;   // flat index of its first query token (row id = (q0 + i) * Hq + h)
  int seqlen, row0, rows;
  int tok0;     // first token of the split
  int lim_max;  // keys [0, lim_max) cover every row of the tile
  int n_tiles;  // tiles of this split holding keys < lim_max
};

// Unit u = kvh + Hkv * (s + n_splits * (b + batch * (n_row_tiles - 1 - rt))):
// the row tile varies slowest, so each row tile of every sequence (the only
// one of a decode step in a packed batch) spreads over all CTAs of the
// strided assignment, and the last row tiles -- the heaviest under causal
// masking, and those of the longest requests -- come first.
// Sequence of unit u.
__device__ __forceinline__ int unit_seq(const AttnParams &p, int u) {
  return (u / p.Hkv / p.n_splits) % p.batch;
}

// Unit u given its sequence's length sl and (packed calls) query range
// [a, e) -- arithmetic only.
template <int N>
__device__ __forceinline__ Unit unit_make(const AttnParams &p, int u, int sl, int a, int e) {
  Unit x;
  x.kvh = u % p.Hkv;
  u /= p.Hkv;
  x.s = u % p.n_splits;
  u /= p.n_splits;
  x.b = u % p.batch;
  x.rt = p.n_row_tiles - 1 - u / p.batch;
  x.seqlen = sl > 0 ? sl : 0;
  if (p.cu_q) {
    x.q0 = a;
    x.nq = min(max(e - a, 0), p.seqlen_q);  // more than the bound: flagged, rows past it unwritten
  } else {
    x.q0 = static_cast<int64_t>(x.b) * p.seqlen_q;
    x.nq = p.seqlen_q;
  }
  const bool mine = x.nq >= p.nq_lo && x.nq <= p.nq_hi;  // another launch serves the rest
  const int R = mine ? p.G * x.nq : 0;
  x.row0 = x.rt * N;
  x.rows = max(min(N, R - x.row0), 0);
  int lim = x.rows > 0 ? x.seqlen : 0;
  if (p.causal && x.rows > 0) {
    const int i_last = (x.row0 + x.rows - 1) / p.G;
    lim = min(lim, x.seqlen - x.nq + i_last + 1);
  }
  x.lim_max = lim > 0 ? lim : 0;
  x.tok0 = (p.split_base + x.s) * kSplitTokens;
  const int ntok = min(kSplitTokens, x.lim_max - x.tok0);
  x.n_tiles = ntok > 0 ? (ntok + kTileTokens - 1) / kTileTokens : 0;
  return x;
}

template <int N>
__device__ __forceinline__ Unit unit_at(const AttnParams &p, int u) {
  const int b = unit_seq(p, u);
  const int sl = __ldg(p.seqlens + b);
  const int a = p.cu_q ? __ldg(p.cu_q + b) : 0, e = p.cu_q ? __ldg(p.cu_q + b + 1) : 0;
  return unit_make<N>(p, u, sl, a, e);
}

constexpr int kPastWidth = static_cast<int>(0x80000000u);

// Element offsets of query token i of unit x's sequence in q and out, and the
// lse index of (token i, head h).
__device__ __forceinline__ int64_t q_tok_off(const AttnParams &p, const Unit &x, int i) {
  return p.cu_q ? (x.q0 + i) * p.q_ss : x.b * p.q_sb + static_cast<int64_t>(i) * p.q_ss;
}
__device__ __forceinline__ int64_t o_tok_off(const AttnParams &p, const Unit &x, int i) {
  return p.cu_q ? (x.q0 + i) * p.o_ss : x.b * p.o_sb + static_cast<int64_t>(i) * p.o_ss;
}
__device__ __forceinline__ int64_t lse_index(const AttnParams &p, const Unit &x, int i, int h) {
  return p.cu_q ? static_cast<int64_t>(h) * p.total_q + x.q0 + i
                : (static_cast<int64_t>(x.b) * p.Hq + h) * p.seqlen_q + i;
}

// Caller errors the host cannot see, flagged once per sequence (by the unit
// of its first row tile, KV head 0, split 0): a packed sequence with more
// queries than the host bound, and a context longer than max_seqlen_k (the
// host bound that sized the split grid; keys past the grid's last split are
// not read).
__device__ __forceinline__ void check_sequence(const AttnParams &p, const Unit &x) {
  if (x.rt == 0 && x.kvh == 0 && x.s == 0 && p.err) {
    if (p.cu_q) {
      const int n = __ldg(p.cu_q + x.b + 1) - __ldg(p.cu_q + x.b);
      if (n < 0 || n > p.seqlen_q) atomicOr(p.err, kErrQueryLen);
    }
    if (!p.part_only && x.seqlen > p.max_seqlen_k) atomicOr(p.err, kErrSeqLen);
  }
}

// The units this CTA runs, in order: the k-th is list[k] (a balanced order
// built at kernel start, see build_schedule) or, without a list, unit
// blockIdx.x + k gridDim.x.  Which CTA runs a unit never changes its
// arithmetic, so the order only moves the makespan.
// With a list, each entry's sequence length and packed query range were
// loaded into shared memory with the list (meta[k] = {seqlen, a, e}), so no
// role reads global memory to learn its next unit -- under a saturated memory
// system such a read costs microseconds at every unit boundary.
struct Sched {
  const int *list;
  const int (*meta)[3];
  int count;
  __device__ __forceinline__ int unit(int k) const {
    return list ? list[k] : static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
  }
  template <int N>
  __device__ __forceinline__ Unit get(const AttnParams &p, int k) const {
    if (list) return unit_make<N>(p, list[k], meta[k][0], meta[k][1], meta[k][2]);
    return unit_at<N>(p, unit(k));
  }
};

__device__ __forceinline__ Sched strided_sched(const AttnParams &p) {
  const int g = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
  return Sched{nullptr, nullptr, p.n_units > b ? (p.n_units - b + g - 1) / g : 0};
}

// First schedule slot at or after `from` whose unit has work, or -1.
template <int N>
__device__ __forceinline__ int next_unit(const AttnParams &p, const Sched &sc, int from,
                                         Unit &out) {
  for (int k = from; k < sc.count; ++k) {
    out = sc.get<N>(p, k);
    if (out.n_tiles > 0) return k;
  }
  return -1;
}

// Balanced schedule: every CTA sorts the units that have work by tile count,
// largest first -- a stable counting sort, so every CTA computes the same
// order -- and takes the positions of a snake deal over the grid: round r
// hands positions r G .. r G + G - 1 to CTAs 0 .. G - 1 when r is even and to
// CTAs G - 1 .. 0 when r is odd.  The CTA's k-th unit is the one at its
// position of round k.  With contexts of mixed lengths this evens out the
// tiles per CTA (a stride-G deal leaves some CTAs with far more).  A unit has
// work when it has a tile, or when it is split 0 of real rows (the rows that
// see no key get their zero output there); the others -- splits past a short
// context, row tiles past a short query range, sequences another launch
// serves -- are left out, so no role walks over them.  When every unit has
// work and all have the same tile count there is nothing to balance, and when
// a CTA's share would overflow its list, *count is set to -1 and the caller
// keeps the stride-G deal.  All threads of the CTA take part; `scratch`
// (free shared memory at kernel start, `scratch_bytes` >= n_units) holds one
// byte per unit and, when it fits behind them, each sequence's length and
// query range; hist has kSchedHist entries.

template <int N>
__device__ __forceinline__ void build_schedule(const AttnParams &p, uint8_t *scratch, int scratch_bytes,
                                               int *hist, int *start, int *list, int (*meta)[3],
                                               int *count) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  int *nt_min = hist + kSchedBuckets, *nt_max = hist + kSchedBuckets + 1;
  int *n_kept = hist + kSchedBuckets + 2;
  constexpr uint8_t kSkip = 0xFF;
  // per-sequence (length, query start, query end), cached behind the unit bytes
  const int seq_off = (p.n_units + 15) & ~15;
  int *seq = (seq_off + 12 * p.batch <= scratch_bytes) ? reinterpret_cast<int *>(scratch + seq_off) : nullptr;
  for (int i = tid; i < kSchedBuckets; i += nthr) hist[i] = 0;
  if (tid == 0) {
    *nt_min = kSchedBuckets;
    *nt_max = 0;
    *n_kept = 0;
  }
  if (seq) {
    for (int b = tid; b < p.batch; b += nthr) {
      seq[3 * b] = __ldg(p.seqlens + b);
      seq[3 * b + 1] = p.cu_q ? __ldg(p.cu_q + b) : 0;
      seq[3 * b + 2] = p.cu_q ? __ldg(p.cu_q + b + 1) : 0;
    }
  }
  __syncthreads();
  auto unit_of = [&](int u) {
    if (!seq) return unit_at<N>(p, u);
    const int b = unit_seq(p, u);
    return unit_make<N>(p, u, seq[3 * b], seq[3 * b + 1], seq[3 * b + 2]);
  };
  int lo = kSchedBuckets, hi = 0, kept = 0;
  for (int u = tid; u < p.n_units; u += nthr) {
    const Unit x = unit_of(u);
    const bool keep = x.n_tiles > 0 || (x.rows > 0 && x.s == 0);
    scratch[u] = keep ? static_cast<uint8_t>(x.n_tiles) : kSkip;
    if (keep) {
      atomicAdd(&hist[x.n_tiles], 1);
      ++kept;
      if (x.n_tiles > 0) {
        lo = min(lo, x.n_tiles);
        hi = max(hi, x.n_tiles);
      }
    }
  }
  // one lane per warp updates the shared counters
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  kept = __reduce_add_sync(0xffffffffu, kept);
  if ((tid & 31) == 0) {
    if (lo <= hi) {
      atomicMin(nt_min, lo);
      atomicMax(nt_max, hi);
    }
    if (kept) atomicAdd(n_kept, kept);
  }
  __syncthreads();
  const int G = static_cast<int>(gridDim.x), me = static_cast<int>(blockIdx.x);
  const int total = *n_kept;
  if ((total == p.n_units && *nt_min >= *nt_max) || (total + G - 1) / G > kSchedMaxMine) {
    __syncthreads();  // every thread has read the counters
    if (tid == 0) *count = -1;
    __syncthreads();
    return;
  }
  if (tid == 0) {  // bucket starts, largest tile count first
    int acc = 0;
    for (int nt = kSchedBuckets - 1; nt >= 0; --nt) {
      start[nt] = acc;
      acc += hist[nt];
      hist[nt] = 0;  // from here on: units of the bucket placed so far
    }
  }
  __syncthreads();
  if (tid < 32) {
    const int lane = tid;
    for (int base = 0; base < p.n_units; base += 32) {
      if constexpr (N >= 128) {
        // (row-major tiles: a call may have far more unit slots than units
        // with work) skip a run of 128 slots none of which is kept, four
        // unit bytes per lane
        if ((base & 127) == 0) {
          const int w0 = base + 4 * lane;
          bool any = false;
          if (w0 + 3 < p.n_units) {
            any = *reinterpret_cast<const uint32_t *>(scratch + w0) != 0xFFFFFFFFu;
          } else {
            for (int k = 0; k < 4; ++k) any = any || (w0 + k < p.n_units && scratch[w0 + k] != kSkip);
          }
          if (__ballot_sync(0xffffffffu, any) == 0u) {
            base += 96;  // with the loop's 32: the next run of 128
            continue;
          }
        }
      }
      const int u = base + lane;
      const int nt = (u < p.n_units && scratch[u] != kSkip) ? scratch[u] : -1;
      const unsigned same = __match_any_sync(0xffffffffu, nt);
      const int rank = __popc(same & ((1u << lane) - 1u));
      const int placed = nt >= 0 ? hist[nt] : 0;
      __syncwarp();
      if (nt >= 0) {
        if (rank == 0) hist[nt] = placed + __popc(same);
        const int pos = start[nt] + placed + rank;
        const int r = pos / G, i = pos - r * G;
        if (((r & 1) ? G - 1 - i : i) == me) list[r] = u;
      }
      __syncwarp();
    }
    if (lane == 0) {
      // rounds in which this CTA has a position below the kept units
      const int full_rounds = total / G, rem = total - full_rounds * G;
      const int pos_last = (full_rounds & 1) ? G - 1 - me : me;  // its position in the partial round
      *count = full_rounds + (pos_last < rem ? 1 : 0);
    }
  }
  __syncthreads();
  // the listed units' sequence lengths and query ranges
  for (int k = tid; k < *count; k += nthr) {
    const int b = unit_seq(p, list[k]);
    meta[k][0] = seq ? seq[3 * b] : __ldg(p.seqlens + b);
    meta[k][1] = seq ? seq[3 * b + 1] : (p.cu_q ? __ldg(p.cu_q + b) : 0);
    meta[k][2] = seq ? seq[3 * b + 2] : (p.cu_q ? __ldg(p.cu_q + b + 1) : 0);
  }
  __syncthreads();
}

// Stage the Q rows of unit x (the B operand of S^T = K Q^T, 128-byte
// swizzled); padded rows are zero.  Plain loads: cp.async here measurably
// slowed the TMA issue of the same warp.
template <int D, int N>
__device__ __forceinline__ void stage_q(const AttnParams &p, const Unit &x, uint8_t *qdst, int lane) {
  constexpr int kQHalf = N * 128;
  for (int idx = lane; idx < N * (D / 8); idx += 32) {
    const int c = idx / (D / 8), ch = idx % (D / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (c < x.rows) {
      const int r = x.row0 + c;
      const int i = r / p.G, g = r - i * p.G;
      v = __ldg(reinterpret_cast<const uint4 *>(p.q + q_tok_off(p, x, i) +
                                                static_cast<int64_t>(x.kvh * p.G + g) * p.q_sh +
                                                ch * 8));
    }
    const int h = ch >> 3, cc = ch & 7;
    *reinterpret_cast<uint4 *>(qdst + h * kQHalf + c * 128 + ((cc ^ (c & 7)) << 4)) = v;
  }
}

// Stage the block-table entries of unit x's split (columns past the table are
// marked kPastWidth).
__device__ __forceinline__ void stage_tab(const AttnParams &p, const Unit &x, int *tab, int lane) {
  const int ntok = min(kSplitTokens, x.lim_max - x.tok0);
  const int first = x.tok0 >> p.block_shift;
  const int nent = (ntok + (1 << p.block_shift) - 1) >> p.block_shift;
  for (int e = lane; e < nent; e += 32) {
    const int col = first + e;
    tab[e] = col < p.max_blocks_per_seq ? __ldg(p.block_table + x.b * p.bt_stride + col)
                                        : kPastWidth;
  }
}

// Fused append: write the new tokens that fall inside this unit's loaded key
// range [tok0, min(tok0 + 4096, lim_max)) for this unit's KV head -- K from the
// K producer, V from the V producer -- then order those generic writes before
// the warp's TMA reads of the same rows.  Every unit that loads a new position
// writes it itself (the same bits), so no unit depends on another.
template <int D>
__device__ __forceinline__ void append_new_tokens(const AttnParams &p, const Unit &x,
                                                  const int *tab, bool is_k, int lane) {
  const int first_new = x.seqlen - p.n_new;
  const int lo = max(first_new, x.tok0);
  const int hi = min(x.lim_max, x.tok0 + kSplitTokens);
  if (lo < hi) {
    const uint16_t *src = is_k ? p.k_new : p.v_new;
    uint16_t *cache = is_k ? p.k_cache : p.v_cache;
    const int64_t nb = is_k ? p.kn_sb : p.vn_sb, nt = is_k ? p.kn_st : p.vn_st,
                  nh = is_k ? p.kn_sh : p.vn_sh;
    const int64_t cb = is_k ? p.k_sb : p.v_sb, cs = is_k ? p.k_ss : p.v_ss,
                  ch_ = is_k ? p.k_sh : p.v_sh;
    const int bmask = (1 << p.block_shift) - 1;
    for (int idx = lane; idx < (hi - lo) * (D / 8); idx += 32) {
      const int tok = lo + idx / (D / 8), c = idx % (D / 8);
      const int blk = tab[(tok - x.tok0) >> p.block_shift];
      if (blk == kPastWidth || blk < 0 || static_cast<int64_t>(blk) >= p.num_blocks) continue;
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(
          src + x.b * nb + static_cast<int64_t>(tok - first_new) * nt + x.kvh * nh) + c);
      reinterpret_cast<uint4 *>(cache + blk * cb + static_cast<int64_t>(tok & bmask) * cs +
                                x.kvh * ch_)[c] = v;
    }
    fence_proxy_async_global();
  }
  __syncwarp();
}

// One producer warp.  The current unit's block-table entries (and, for the K
// warp, its Q rows) are already in shared memory when its first tile is
// issued: the warp stages the NEXT unit's entries at the start of every unit
// and (two Q buffers) the next unit's Q just before the current unit's last
// tile -- points where its stage ring is full and it would wait anyway.  Per tile, lane k issues the TMA boxes of the tile's k-th box of cache
// rows, all lanes in parallel; lane 0 arrives on `full`.
template <class C>
__device__ __forceinline__ void produce(const AttnParams &p, const CUtensorMap *map,
                                        const CUtensorMap *map_q, uint8_t *smem,
                                        typename C::Small *sm, uint64_t *full, uint64_t *empty,
                                        int (*tabs)[kSplitTokens / 16], uint32_t dst_off,
                                        bool with_q, int lane, volatile int *abort_any,
                                        const Sched &sc) {
  constexpr int D = C::kD, N = C::kN, NS = C::kNS, QB = C::kQB;
  // Q copies by TMA still to be accounted for at exit (lane 0): per buffer,
  // the ordinal of the last unit whose Q went there, and whether its q_full
  // arrival is still to come (the copy was issued, the unit boundary not yet
  // reached)
  int q_last[QB];
#pragma unroll
  for (int i = 0; i < QB; ++i) q_last[i] = -1;
  int q_pending = -1, q_pending_ord = -1;
  // Q of unit u (the warp's ord-th unit) into buffer qb: TMA (completing on
  // q_full[qb]) or plain loads
  auto put_q = [&](const Unit &u, int qb, int ord) {
    if constexpr (C::kQTma) {
      if (lane == 0) {
        q_pending = qb;
        q_pending_ord = ord;
        mbar_expect_tx(&sm->q_full[qb], static_cast<uint32_t>(C::kQBytes));
        const int i0 = u.row0 / p.G;
        // dense map (D, Hq, seqlen_q, batch); packed map (D, Hq, total_q, 1)
        const int c2 = p.cu_q ? static_cast<int>(u.q0) + i0 : i0;
        const int c3 = p.cu_q ? 0 : u.b;
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(smem + C::kOffQ + qb * C::kQBytes + h * C::kQHalfBytes, map_q,
                      &sm->q_full[qb], h * 64, u.kvh * p.G, c2, c3);
      }
    } else {
      stage_q<D, N>(p, u, smem + C::kOffQ + qb * C::kQBytes, lane);
    }
  };
  if (lane == 0) tma_prefetch_desc(map);
  if (C::kQTma && with_q && lane == 0) tma_prefetch_desc(map_q);
  int last_gi[NS];
#pragma unroll
  for (int i = 0; i < NS; ++i) last_gi[i] = -1;
  bool failed = false;
  Unit cur;
  int cu = next_unit<N>(p, sc, 0, cur);
  if (cu >= 0) {
    const int bmask = (1 << p.block_shift) - 1;
    int ui = 0, gi = 0;
    // the first unit (Q buffer 0 is free)
    stage_tab(p, cur, tabs[0], lane);
    if (with_q) put_q(cur, 0, 0);
    if (with_q) fence_proxy_async_smem();
    __syncwarp();
    if (with_q && lane == 0) {
      mbar_arrive(&sm->q_full[0]);
      if constexpr (C::kQTma) {
        q_last[0] = 0;
        q_pending = -1;
      }
    }
    while (true) {
      // stage the next unit while this one's tiles are issued
      Unit nxt;
      const int nu = next_unit<N>(p, sc, cu + 1, nxt);
      bool q_early = false;
      if (nu >= 0) stage_tab(p, nxt, tabs[(ui + 1) & 1], lane);
      const int *tab = tabs[ui & 1];
      if (p.n_new > 0) append_new_tokens<D>(p, cur, tab, with_q, lane);
      for (int j = 0; j < cur.n_tiles && !failed; ++j, ++gi) {
        if (C::kEarlyQ && with_q && QB == 2 && nu >= 0 && j == cur.n_tiles - 1) {
          // the next unit's Q goes to the buffer of the previous unit, whose
          // QKs are done by the time this unit's last tile is issued
          const int qb = (ui + 1) % QB;
          bool okq = true;
          if (lane == 0) okq = mbar_wait(&sm->q_empty[qb], (((ui + 1) / QB) & 1) ^ 1, abort_any, p.wait_ns);
          if (!__shfl_sync(0xffffffffu, okq ? 1 : 0, 0)) {
            failed = true;
            break;
          }
          put_q(nxt, qb, ui + 1);
          q_early = true;
        }
        const int st = gi % NS;
        bool okw = true;
        if (lane == 0) okw = mbar_wait(&empty[st], ((gi / NS) & 1) ^ 1, abort_any, p.wait_ns);
        if (!__shfl_sync(0xffffffffu, okw ? 1 : 0, 0)) {
          failed = true;
          break;
        }
        const int tok0 = cur.tok0 + j * kTileTokens;
        const int nvalid = min(kTileTokens, cur.lim_max - tok0);
        const int nbox = (nvalid + p.box_slots - 1) / p.box_slots;
        int errs = 0;
        if (lane < nbox) {
          const int tok = tok0 + lane * p.box_slots;
          const int blk = tab[(tok - cur.tok0) >> p.block_shift];
          if (blk == kPastWidth) {
            errs = kErrTableWidth;
          } else if (blk < 0 || static_cast<int64_t>(blk) >= p.num_blocks) {
            errs = kErrBadBlock;
          } else {
            uint8_t *d0 = smem + dst_off + st * C::kKVBytes + lane * p.box_slots * 128;
            const int slot = tok & bmask;
            const int c1 = p.map_head_first ? cur.kvh : slot;
            const int c2 = p.map_head_first ? slot : cur.kvh;
            mbar_expect_tx(&full[st], static_cast<uint32_t>((D / 64) * p.box_slots * 128));
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_load_4d(d0 + h * C::kHalfBytes, map, &full[st], h * 64, c1, c2, blk);
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full[st]);
          last_gi[st] = gi;
        }
        if (errs && p.err) atomicOr(p.err, errs);
      }
      if (failed || nu < 0) break;
      // unit boundary: the next unit's entries (and Q) are in shared memory
      // The next unit's Q goes into the buffer of the unit before this one,
      // once that unit has released it.  Without kEarlyQ the release also
      // waits for that unit's epilogue, which needs the P.V of its last
      // tile, which the MMA warp issues after the QK^T of this unit's first
      // tile: the wait then comes after every tile of this unit is issued
      // (waiting earlier would close a cycle when this unit has one tile).
      if (with_q && !q_early) {
        const int qb = (ui + 1) % QB;
        bool okq = true;
        if (lane == 0) okq = mbar_wait(&sm->q_empty[qb], (((ui + 1) / QB) & 1) ^ 1, abort_any, p.wait_ns);
        if (!__shfl_sync(0xffffffffu, okq ? 1 : 0, 0)) {
          failed = true;
          break;
        }
        put_q(nxt, qb, ui + 1);
      }
      if (with_q) fence_proxy_async_smem();
      __syncwarp();
      if (with_q && lane == 0) {
        mbar_arrive(&sm->q_full[(ui + 1) % QB]);
        if constexpr (C::kQTma) {
          q_last[(ui + 1) % QB] = ui + 1;
          q_pending = -1;
        }
      }
      ++ui;
      cur = nxt;
      cu = nu;
    }
  }
  if (lane == 0) {
    // Whatever ended the loop, wait (bounded, ignoring the abort flag) until
    // every copy this warp issued has landed, so that none is in flight when
    // the CTA exits even if its consumers gave up.  After a normal run these
    // phases have long completed and the waits return at once.  A Q copy whose
    // q_full arrival was still to come gets it now, so its phase can complete.
    volatile int no_abort = 0;
#pragma unroll
    for (int i = 0; i < NS; ++i)
      if (last_gi[i] >= 0) mbar_wait(&full[i], (last_gi[i] / NS) & 1, &no_abort);
    if constexpr (C::kQTma) {
      if (with_q && q_pending >= 0) {
        mbar_arrive(&sm->q_full[q_pending]);
        q_last[q_pending] = q_pending_ord;
      }
#pragma unroll
      for (int i = 0; i < QB; ++i)
        if (with_q && q_last[i] >= 0) mbar_wait(&sm->q_full[i], (q_last[i] / QB) & 1, &no_abort);
    }
  }
}

// Direct final write (calls whose every row has at most one split, no merge
// launch): row c of unit x gets out / lse through the merge's fold of that one
// partial, so the bits are those the merge would write.  Thread t < D writes
// column t of every row (acc[c] = the row's unnormalised column t); thread
// t < rows also writes row t's lse.  m / l of every row come from shared
// memory (fin_m / fin_l), published before the call.  With `stage` (shared
// memory, [rows][D] bf16) the out rows go there instead, for bulk stores.
template <int D, int N>
__device__ __forceinline__ void write_final_cols(const AttnParams &p, const Unit &x, int t,
                                                 const float (&acc)[N], const float *fin_m,
                                                 const float *fin_l,
                                                 __nv_bfloat16 *stage = nullptr) {
  const float NEG_INF = neg_inf();
#pragma unroll
  for (int c = 0; c < N; ++c) {
    if (c < x.rows && t < D) {
      const int r = x.row0 + c;
      const int i = r / p.G, g = r - i * p.G;
      const int h = x.kvh * p.G + g;
      const float m = fin_m[c];
      float L = 0.f, A = 0.f;
      if (m != NEG_INF) {
        const FoldCoef kc = fold_coef(NEG_INF, m);
        L = fold_val(0.f, fin_l[c], kc);
        A = fold_val(0.f, acc[c], kc);
      }
      // one quotient per (row, element) here: the IEEE division itself,
      // which final_out reproduces bit for bit elsewhere
      const __nv_bfloat16 ob = __float2bfloat16_rn(L > 0.f ? __fdiv_rn(A, L) : 0.f);
      if (stage)
        stage[c * D + t] = ob;
      else
        p.out[o_tok_off(p, x, i) + h * p.o_sh + t] = ob;
      if (p.fin_out != nullptr && i == x.nq - 1) p.fin_out[x.b * p.fo_sb + h * p.fo_sh + t] = ob;
    }
  }
  if (t < x.rows) {
    const int r = x.row0 + t;
    const int i = r / p.G, g = r - i * p.G;
    const int h = x.kvh * p.G + g;
    const float m = fin_m[t];
    float M = NEG_INF, L = 0.f;
    if (m != NEG_INF) {
      const FoldCoef kc = fold_coef(NEG_INF, m);
      L = fold_val(0.f, fin_l[t], kc);
      M = kc.Mn;
    }
    const float ls = final_lse(M, L);
    p.lse[lse_index(p, x, i, h)] = ls;
    if (p.fin_out != nullptr && i == x.nq - 1) p.fin_lse[static_cast<int64_t>(x.b) * p.Hq + h] = ls;
  }
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
      mbar_init(&sm->full_k[i], 1);
      mbar_init(&sm->empty_k[i], 1);
      mbar_init(&sm->full_v[i], 1);
      mbar_init(&sm->empty_v[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm->s_full[i], 1);
      mbar_init(&sm->p_full[i], 4);   // one arrival per warp of a softmax warpgroup
      mbar_init(&sm->o_full[i], 1);
      mbar_init(&sm->stat_free[i], 4);
      mbar_init(&sm->m_full[i], 1);
      mbar_init(&sm->unit_done[i], 1);
      mbar_init(&sm->o_free[i], 4);   // one arrival per correction warp
    }
    for (int i = 0; i < QB; ++i) {
      mbar_init(&sm->q_full[i], 1);
      // two Q buffers: the buffer is free once the unit's last QK^T is done
      // (MMA commit) and the correction warpgroup has staged that unit's
      // epilogue through it (one arrival)
      mbar_init(&sm->q_empty[i], QB == 2 ? 2 : 1);
    }
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
  // the P^T buffers are not in use yet: the schedule's scratch
  Sched sc = strided_sched(p);
  if (p.sched) {
    build_schedule<N>(p, smem + C::kOffP, C::kSchedScratch, sm->sched_hist, sm->sched_start,
                      sm->sched_list, sm->sched_meta, &sm->sched_count);
    if (sm->sched_count >= 0) sc = Sched{sm->sched_list, sm->sched_meta, sm->sched_count};
  }

  if (warp == kKWarp) {
    produce<C>(p, &map_k, nullptr, smem, sm, sm->full_k, sm->empty_k, sm->tab[0], C::kOffK, true,
               lane, abort_any, sc);
  } else if (warp == kVWarp) {
    produce<C>(p, &map_v, nullptr, smem, sm, sm->full_v, sm->empty_v, sm->tab[1], C::kOffV, false,
               lane, abort_any, sc);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------
    // MMA issuer (one thread)
    // ------------------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t kIdescQK = idesc_bf16(128, N, 0, 0);           // A = K tile, B = Q (K-major)
      constexpr uint32_t kIdescPV = idesc_bf16(128, C::kPCols, 1, 1);  // A = V^T, B = P^T (MN-major)
      const uint32_t tS = tmem, tO = tmem + 2 * N;
      // QK^T of tile gi, then P.V of tile gi - 1.  O^T accumulates over a
      // unit's tiles in the buffer of the unit's parity.
      struct Pend {
        int g, first, last, u;
      };
      int gi = 0, ui = 0;
      Pend prev{-1, 0, 0, 0};
      bool failed = false;
      auto pv_step = [&](const Pend &pd) -> bool {
        const int g = pd.g, st = g % NS, bb = g & 1, ob = pd.u & 1;
        if (!mbar_wait(&sm->p_full[bb], (g >> 1) & 1, abort_any, p.wait_ns)) return false;
        if (pd.first && !mbar_wait(&sm->o_free[ob], ((pd.u >> 1) & 1) ^ 1, abort_any, p.wait_ns))
          return false;
        if (!mbar_wait(&sm->full_v[st], (g / NS) & 1, abort_any, p.wait_ns)) return false;
        tc_fence_after_sync();
        const uint32_t vaddr = sbase + C::kOffV + st * C::kKVBytes;
        const uint32_t paddr = sbase + C::kOffP + bb * C::kPBytes;
#pragma unroll
        for (int kk = 0; kk < kTileTokens / 16; ++kk) {
          // V^T: MN-major, 128-byte swizzle, 64-wide d groups C::kHalfBytes apart
          // (D = 64: both M halves read the same 64 columns; lanes 64..127 are unused).
          const uint64_t a = smem_desc(vaddr + kk * 2048, D == 128 ? C::kHalfBytes : 0, 1024,
                                       kLayoutSw128);
          // P^T = [P_hi | P_lo]: MN-major, no swizzle; 8-column groups 128 B
          // apart, 8-token groups kPKGroup apart.  O_hi and O_lo side by side.
          const uint64_t b = smem_desc(paddr + kk * 2 * C::kPKGroup, C::kPKGroup, 128,
                                       kLayoutInterleave);
          umma_bf16(tO + ob * C::kPCols, a, b, kIdescPV, (pd.first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&sm->o_full[bb]);
        if (pd.last) umma_commit(&sm->unit_done[ob]);
        umma_commit(&sm->empty_v[st]);
        return true;
      };
      for (int k = 0; k < sc.count && !failed; ++k) {
        const Unit x = sc.get<N>(p, k);
        if (x.n_tiles == 0) continue;
        const int qb = ui % QB;
        if (!mbar_wait(&sm->q_full[qb], (ui / QB) & 1, abort_any, p.wait_ns)) {
          failed = true;
          break;
        }
        const uint32_t qaddr = sbase + C::kOffQ + qb * C::kQBytes;
        for (int j = 0; j < x.n_tiles; ++j, ++gi) {
          const int st = gi % NS, bb = gi & 1;
          if (!mbar_wait(&sm->full_k[st], (gi / NS) & 1, abort_any, p.wait_ns)) {
            failed = true;
            break;
          }
          tc_fence_after_sync();
          const uint32_t kaddr = sbase + C::kOffK + st * C::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int h = kk >> 2, off = (kk & 3) * 32;
            const uint64_t a = smem_desc(kaddr + h * C::kHalfBytes + off, 16, 1024, kLayoutSw128);
            const uint64_t b = smem_desc(qaddr + h * C::kQHalfBytes + off, 16, 1024, kLayoutSw128);
            umma_bf16(tS + bb * N, a, b, kIdescQK, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm->s_full[bb]);
          umma_commit(&sm->empty_k[st]);
          if (j == x.n_tiles - 1) umma_commit(&sm->q_empty[qb]);
          if (prev.g >= 0 && !pv_step(prev)) {
            failed = true;
            break;
          }
          prev = Pend{gi, j == 0 ? 1 : 0, j == x.n_tiles - 1 ? 1 : 0, ui};
        }
        ++ui;
      }
      if (!failed && prev.g >= 0) failed = !pv_step(prev);
      // every MMA this thread issued completes before TMEM is released, also
      // when the consumers gave up (bounded wait, default limit)
      (void)failed;
      umma_commit(&sm->drain);
      volatile int no_abort = 0;
      mbar_wait(&sm->drain, 0, &no_abort);
    }
  } else if (warp < kCorrWarp0) {
    // ------------------------------------------------------------------
    // Softmax warpgroups: warpgroup wg takes the tiles with gi % 2 == wg.
    // Thread t <-> TMEM lane t <-> token t of the tile.  Per tile and row:
    // tmax = exact max of the masked scores; the running max m (the
    // previous tile's, published by the other warpgroup; -inf at a unit's
    // start) rises to tmax only when tmax > m + kMaxSlack, and then the
    // row's column of O^T (hi and lo) takes the factor a = 2^(m - m') before
    // this tile's P.V adds to it; p = 2^(raw * scale - m) written as P^T = [bf16(p) |
    // bf16(p - bf16(p))]; per-warp sums of the fp32 p.
    // ------------------------------------------------------------------
    const int wg = warp >> 2, wq = warp & 3, t = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t bar_id = 1 + wg;
    const float NEG_INF = neg_inf();
    int gbase = 0, uo = 0;  // uo: ordinal of the unit among this CTA's units with work
    bool stop = false;
    for (int k = 0; k < sc.count && !stop; ++k) {
      const Unit x = sc.get<N>(p, k);
      if (x.n_tiles == 0) continue;
      const uint32_t ocol = tmem + lane_off + 2 * N + (uo & 1) * C::kPCols;  // this unit's O^T
      if (t < N) {
        int lim = 0;
        if (t < x.rows) {
          const int i = (x.row0 + t) / p.G;
          lim = x.seqlen;
          if (p.causal) lim = min(lim, x.seqlen - x.nq + i + 1);
          lim = lim > 0 ? lim : 0;
        }
        sm->lim[wg][t] = lim;
      }
      if (wg_bar_or(bar_id, false)) {
        stop = true;
        break;
      }
      for (int j = 0; j < x.n_tiles; ++j) {
        const int gi = gbase + j;
        if ((gi & 1) != wg) continue;
        const int bb = wg, st = gi % NS, par = (gi >> 1) & 1;
        bool ok = mbar_wait(&sm->s_full[bb], par, abort_any, p.wait_ns);
        // P^T[bb] is free once P.V of tile gi - 2 is done, the row statistics
        // once the correction of tile gi - 2 has read them
        ok = mbar_wait(&sm->o_full[bb], par ^ 1, abort_any, p.wait_ns) && ok;
        ok = mbar_wait(&sm->stat_free[bb], par ^ 1, abort_any, p.wait_ns) && ok;
        tc_fence_after_sync();
        float sv[N];
#pragma unroll
        for (int ch = 0; ch < N / 16; ++ch)
          if (ch * 16 < x.rows)
            tmem_ld16(tmem + lane_off + bb * N + ch * 16, *reinterpret_cast<float(*)[16]>(&sv[ch * 16]));
        tmem_ld_wait();
        const int tok0 = x.tok0 + j * kTileTokens;
        const int tok = tok0 + t;
        // raw scores of the visible keys (masked: -inf); the row's max over
        // them is scaled once (cscale > 0 rounds monotonically, so that is
        // the max of the scaled scores exactly), p = 2^(raw * cscale - m)
#pragma unroll
        for (int c = 0; c < N; ++c) sv[c] = (c < x.rows && tok < sm->lim[wg][c]) ? sv[c] : NEG_INF;
        if (tok0 + kTileTokens > x.lim_max) {
          // The last tile: keys past the loaded range hold stale bytes or the
          // cache's NaN tails; once V has landed, zero those V rows so that
          // 0 * V stays 0 in P.V.
          ok = mbar_wait(&sm->full_v[st], (gi / NS) & 1, abort_any, p.wait_ns) && ok;
          if (ok && tok >= x.lim_max) {
            uint8_t *vrow = smem + C::kOffV + st * C::kKVBytes + t * 128;
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
#pragma unroll
              for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4 *>(vrow + h * C::kHalfBytes + k * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        float(*wmax)[N] = sm->wmax[wg][par];
#pragma unroll
        for (int q4 = 0; q4 < N / 4; ++q4) {
          if (q4 * 4 < x.rows) {  // warp-uniform: padded rows need no reduction
            float v[4] = {sv[4 * q4], sv[4 * q4 + 1], sv[4 * q4 + 2], sv[4 * q4 + 3]};
            warp_max4(v);
            if (lane == 0)
              *reinterpret_cast<float4 *>(&wmax[wq][4 * q4]) = make_float4(v[0], v[1], v[2], v[3]);
          }
        }
        if (wg_bar_or(bar_id, !ok)) {
          stop = true;
          break;
        }
        // the running maxima: the previous tile's (its phase is awaited for
        // every tile, so the parity waits stay in step), this tile's
        if (gi > 0)
          ok = mbar_wait(&sm->m_full[(gi - 1) & 1], ((gi - 1) >> 1) & 1, abort_any, p.wait_ns) && ok;
        if (t < N) {
          float m_new = NEG_INF, a = 1.f;
          if (t < x.rows) {
            const float tmax = __fmul_rn(
                fmaxf(fmaxf(wmax[0][t], wmax[1][t]), fmaxf(wmax[2][t], wmax[3][t])), p.cscale);
            const float m_prev = j > 0 ? sm->mrun[(gi - 1) & 1][t] : NEG_INF;
            m_new = (tmax > __fadd_rn(m_prev, kMaxSlack)) ? tmax : m_prev;
            a = (m_prev == NEG_INF || m_new == m_prev) ? 1.f : ex2(__fsub_rn(m_prev, m_new));
          }
          sm->mnew[bb][t] = m_new;
          sm->scl[bb][t] = a;
          sm->mrun[gi & 1][t] = m_new;
        }
        if (wg_bar_or(bar_id, !ok)) {
          stop = true;
          break;
        }
        if (t == 0) mbar_arrive(&sm->m_full[gi & 1]);
        bool resc = false;
        for (int c = 0; c < x.rows; ++c) resc = resc || sm->scl[bb][c] != 1.f;
        if (resc) {
          // O^T holds the unit's tiles < gi once P.V(gi - 1) is done (o_full
          // of its parity; that barrier's previous phase, tile gi - 3, is done,
          // since this warpgroup waited for tile gi - 2's P.V above)
          ok = mbar_wait(&sm->o_full[(gi - 1) & 1], ((gi - 1) >> 1) & 1, abort_any, p.wait_ns) && ok;
          if (__all_sync(0xffffffffu, ok)) {
            tc_fence_after_sync();
#pragma unroll
            for (int ch = 0; ch < N / 16; ++ch) {
              if (ch * 16 < x.rows) {  // warp-uniform
                float hi[16], lo[16];
                tmem_ld16(ocol + ch * 16, hi);
                tmem_ld16(ocol + N + ch * 16, lo);
                tmem_ld_wait_for(hi);
                tmem_ld_wait_for(lo);
                uint32_t wh[16], wl[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const float a = sm->scl[bb][ch * 16 + e];
                  wh[e] = __float_as_uint(__fmul_rn(hi[e], a));
                  wl[e] = __float_as_uint(__fmul_rn(lo[e], a));
                }
                tmem_st16(ocol + ch * 16, wh);
                tmem_st16(ocol + N + ch * 16, wl);
              }
            }
            tmem_st_wait();
          }
        }
        // P^T row t (MN-major, no swizzle: one 16-byte chunk per 8 columns).
        uint8_t *prow = smem + C::kOffP + bb * C::kPBytes + (t >> 3) * C::kPKGroup + (t & 7) * 16;
#pragma unroll
        for (int grp = 0; grp < N / 8; ++grp) {
          uint32_t whi[4] = {0u, 0u, 0u, 0u}, wlo[4] = {0u, 0u, 0u, 0u};
          if (grp * 8 < x.rows) {  // groups of padded rows keep p = 0
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c0 = grp * 8 + 2 * e;
              const float m0 = sm->mnew[bb][c0];
              const float m1 = sm->mnew[bb][c0 + 1];
              const float p0 = (sv[c0] == NEG_INF) ? 0.f : ex2(__fmaf_rn(sv[c0], p.cscale, -m0));
              const float p1 =
                  (sv[c0 + 1] == NEG_INF) ? 0.f : ex2(__fmaf_rn(sv[c0 + 1], p.cscale, -m1));
              sv[c0] = p0;
              sv[c0 + 1] = p1;
              __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
              __nv_bfloat162 l2 = __floats2bfloat162_rn(__fsub_rn(p0, __low2float(h2)),
                                                        __fsub_rn(p1, __high2float(h2)));
              whi[e] = *reinterpret_cast<uint32_t *>(&h2);
              wlo[e] = *reinterpret_cast<uint32_t *>(&l2);
            }
          }
          *reinterpret_cast<uint4 *>(prow + grp * 128) = make_uint4(whi[0], whi[1], whi[2], whi[3]);
          *reinterpret_cast<uint4 *>(prow + (N / 8 + grp) * 128) =
              make_uint4(wlo[0], wlo[1], wlo[2], wlo[3]);
        }
#pragma unroll
        for (int q4 = 0; q4 < N / 4; ++q4) {
          if (q4 * 4 < x.rows) {
            float v[4] = {sv[4 * q4], sv[4 * q4 + 1], sv[4 * q4 + 2], sv[4 * q4 + 3]};
            warp_sum4_lane0(v);
            if (lane == 0)
              *reinterpret_cast<float4 *>(&sm->wsum[bb][wq][4 * q4]) = make_float4(v[0], v[1], v[2], v[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->p_full[bb]);
      }
      gbase += x.n_tiles;
      ++uo;
    }
    (void)stop;
  } else if (warp < kCorrWarp0 + 4) {
    // ------------------------------------------------------------------
    // Correction + epilogue warpgroup: thread r (< rows) owns row r's
    // running l; per tile, in order, l = fma(l, a, sum p) with the factor a
    // the softmax chose (1 unless the row's max rose).  At the unit's end,
    // once its last P.V is done, thread t <-> TMEM lane t <-> column d of
    // O^T: acc = O_hi + O_lo, then the partials or the final rows.
    // ------------------------------------------------------------------
    const int wq = warp & 3, t = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    constexpr uint32_t bar_id = 3;
    const float NEG_INF = neg_inf();
    float acc[N];
    float m_run = NEG_INF, l_run = 0.f;
    int gbase = 0, cui = 0;  // cui: ordinal of the unit among this CTA's units with work
    bool bulk_out = false;   // thread 0 has bulk stores to complete before exit
    bool stop = false;
    for (int k = 0; k < sc.count && !stop; ++k) {
      const Unit x = sc.get<N>(p, k);
      if (t == 0) check_sequence(p, x);
      if (x.n_tiles == 0) {
        // direct write: rows of this unit see no key (out = 0, lse = -inf)
        if (p.direct && x.rows > 0) {
#pragma unroll
          for (int c = 0; c < N; ++c) acc[c] = 0.f;
          float none[N];
#pragma unroll
          for (int c = 0; c < N; ++c) none[c] = NEG_INF;
          write_final_cols<D, N>(p, x, t, acc, none, none);
        }
        continue;
      }
#pragma unroll
      for (int c = 0; c < N; ++c) acc[c] = 0.f;
      m_run = NEG_INF;
      l_run = 0.f;
      for (int j = 0; j < x.n_tiles; ++j) {
        const int gi = gbase + j, bb = gi & 1, par = (gi >> 1) & 1;
        const bool ok = mbar_wait(&sm->p_full[bb], par, abort_any, p.wait_ns);  // the tile's row statistics
        if (t < x.rows) {
          const float lt = __fadd_rn(__fadd_rn(sm->wsum[bb][0][t], sm->wsum[bb][1][t]),
                                     __fadd_rn(sm->wsum[bb][2][t], sm->wsum[bb][3][t]));
          l_run = __fmaf_rn(l_run, sm->scl[bb][t], lt);
          m_run = sm->mnew[bb][t];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->stat_free[bb]);  // the tile's statistics are read
        if (wg_bar_or(bar_id, !ok)) {
          stop = true;
          break;
        }
      }
      if (stop) break;
      {
        // the unit's last P.V, then O^T out of TMEM (one unit_done phase per
        // unit of this buffer's parity)
        const int ob = cui & 1;
        const bool ok = mbar_wait(&sm->unit_done[ob], (cui >> 1) & 1, abort_any, p.wait_ns);
        if (wg_bar_or(bar_id, !ok)) {
          stop = true;
          break;
        }
        tc_fence_after_sync();
#pragma unroll
        for (int ch = 0; ch < N / 16; ++ch) {
          if (ch * 16 < x.rows) {  // warp-uniform
            float hi[16], lo[16];
            tmem_ld16(tmem + lane_off + 2 * N + ob * C::kPCols + ch * 16, hi);
            tmem_ld16(tmem + lane_off + 2 * N + ob * C::kPCols + N + ch * 16, lo);
            tmem_ld_wait_for(hi);
            tmem_ld_wait_for(lo);
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[ch * 16 + e] = __fadd_rn(hi[e], lo[e]);
          }
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->o_free[ob]);
      }
      if (stop) break;
      if (p.direct) {
        // every row of the call has at most one split: out / lse here
        if (t < x.rows) {
          sm->fin_m[t] = m_run;
          sm->fin_l[t] = l_run;
        }
        wg_bar_or(bar_id, false);
        if constexpr (QB == 2) {
          if (p.out_vec) {
            // the out rows go through this unit's Q buffer and bulk stores
            // (at most N rows of D bf16: the buffer's size)
            __nv_bfloat16 *stage =
                reinterpret_cast<__nv_bfloat16 *>(smem + C::kOffQ + (cui % QB) * C::kQBytes);
            write_final_cols<D, N>(p, x, t, acc, sm->fin_m, sm->fin_l, stage);
            fence_proxy_async_smem();
            wg_bar_or(bar_id, false);
            if (t == 0) {
              for (int c = 0; c < x.rows; ++c) {
                const int r = x.row0 + c;
                const int i = r / p.G, g = r - i * p.G;
                bulk_store(p.out + o_tok_off(p, x, i) + (x.kvh * p.G + g) * p.o_sh, stage + c * D,
                           D * 2);
              }
              bulk_commit();
              bulk_out = true;
            }
          } else {
            write_final_cols<D, N>(p, x, t, acc, sm->fin_m, sm->fin_l);
          }
        } else {
          write_final_cols<D, N>(p, x, t, acc, sm->fin_m, sm->fin_l);
        }
      } else {
        // epilogue: unnormalised split partial of every real row.  With two Q
        // buffers, this unit's (its QK^T are done) stages the rows and the
        // TMA engine stores them, so no thread waits on global stores while
        // the SM streams the cache.
        const int64_t S = p.n_splits;
        if constexpr (QB == 2) {
          float *stage = reinterpret_cast<float *>(smem + C::kOffQ + (cui % QB) * C::kQBytes);
          constexpr int kRowsStaged = C::kQBytes / (D * 4);
          for (int c0 = 0; c0 < x.rows; c0 += kRowsStaged) {
            if (c0 > 0 && t == 0) bulk_wait_read<0>();  // the previous round has read the stage
            if (c0 > 0) wg_bar_or(bar_id, false);
#pragma unroll
            for (int c = 0; c < N; ++c)
              if (c >= c0 && c < min(x.rows, c0 + kRowsStaged) && t < D)
                stage[(c - c0) * D + t] = acc[c];
            fence_proxy_async_smem();
            wg_bar_or(bar_id, false);
            if (t == 0) {
              for (int c = c0; c < min(x.rows, c0 + kRowsStaged); ++c) {
                const int r = x.row0 + c;
                const int i = r / p.G, g = r - i * p.G;
                const int64_t row_id = (x.q0 + i) * p.Hq + x.kvh * p.G + g;
                bulk_store(p.ws_acc + (row_id * S + x.s) * D, stage + (c - c0) * D, D * 4);
              }
              bulk_commit();
              bulk_out = true;
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < N; ++c) {
            if (c < x.rows && t < D) {
              const int r = x.row0 + c;
              const int i = r / p.G, g = r - i * p.G;
              const int64_t row_id = (x.q0 + i) * p.Hq + x.kvh * p.G + g;
              p.ws_acc[(row_id * S + x.s) * D + t] = acc[c];
            }
          }
        }
        if (t < x.rows) {
          const int r = x.row0 + t;
          const int i = r / p.G, g = r - i * p.G;
          const int64_t row_id = (x.q0 + i) * p.Hq + x.kvh * p.G + g;
          *reinterpret_cast<float2 *>(p.ws_ml + (row_id * S + x.s) * 2) = make_float2(m_run, l_run);
        }
      }
      if constexpr (QB == 2) {
        // the stage has been read: the producer may load a later unit's Q here
        if (t == 0) {
          if (bulk_out) bulk_wait_read<0>();
          mbar_arrive(&sm->q_empty[cui % QB]);
        }
      }
      ++cui;
      gbase += x.n_tiles;
    }
    // the partials are complete in global memory before the CTA leaves
    if (bulk_out) bulk_wait<0>();
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
