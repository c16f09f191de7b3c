// pagedkv.cu -- C ABI of libpagedkv.so (declarations and contract in
// include/pagedkv.h): argument validation, TMA tensor maps over the caller's
// cache views, and the kernel launches.  No allocation, no synchronisation.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "pagedkv.h"
#include "attn_bwd.cuh"
#include "attn_rows.cuh"
#include "attn_split.cuh"
#include "kv_append.cuh"
#include "merge.cuh"

static_assert(PKV_SPLIT_TOKENS == pkv::kSplitTokens, "split size");
static_assert(PKV_TILE_TOKENS == pkv::kTileTokens, "tile size");
static_assert(PKV_DEVERR_BAD_BLOCK == pkv::kErrBadBlock, "error bits");
static_assert(PKV_DEVERR_TABLE_WIDTH == pkv::kErrTableWidth, "error bits");
static_assert(PKV_DEVERR_TIMEOUT == pkv::kErrTimeout, "error bits");
static_assert(PKV_DEVERR_QUERY_LEN == pkv::kErrQueryLen, "error bits");
static_assert(PKV_DEVERR_SEQ_LEN == pkv::kErrSeqLen, "error bits");

namespace {

constexpr int kMaxDevices = 64;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

int sm_count(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    v = 148;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

int log2i(int v) {
  int s = 0;
  while ((1 << s) < v) ++s;
  return s;
}

// Element strides usable for 128-bit access: positive multiples of 8.
bool strides_ok(const int64_t *st) {
  if (!st) return false;
  for (int i = 0; i < 3; ++i)
    if (st[i] <= 0 || st[i] % 8 != 0) return false;
  return true;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t ws_acc_bytes(int64_t rows, int64_t splits, int D) {
  const size_t b = static_cast<size_t>(rows) * splits * D * sizeof(float);
  return (b + 255) & ~static_cast<size_t>(255);
}

size_t ws_bytes(int batch, int seqlen_q, int Hq, int D, int max_seqlen_k) {
  const int64_t rows = static_cast<int64_t>(batch) * seqlen_q * Hq;
  const int64_t splits = max_seqlen_k > 0 ? ceil_div(max_seqlen_k, pkv::kSplitTokens) : 1;
  return ws_acc_bytes(rows, splits, D) + static_cast<size_t>(rows) * splits * 2 * sizeof(float);
}

// TMA map over one cache view [num_blocks, block_size, Hkv, D] with the given
// element strides (block, slot, head).  Dimension 0 is head_dim; the head and
// slot dimensions are ordered by stride; the last is the block.  The box is
// 64 head_dim elements x box_slots slots of one head of one block, 128-byte
// swizzled, so every box lands as box_slots rows of 128 bytes.
int make_kv_map(CUtensorMap *map, const void *base, const int64_t st[3], int64_t num_blocks,
                int block_size, int Hkv, int D, int box_slots, int *head_first) {
  auto enc = encode_fn();
  if (!enc) return PKV_ERR_CUDA;
  const bool hf = st[2] <= st[1];
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], estr[4] = {1, 1, 1, 1};
  dims[0] = static_cast<cuuint64_t>(D);
  box[0] = 64;
  if (hf) {
    dims[1] = Hkv;
    dims[2] = block_size;
    strides[0] = st[2] * 2;
    strides[1] = st[1] * 2;
    box[1] = 1;
    box[2] = box_slots;
  } else {
    dims[1] = block_size;
    dims[2] = Hkv;
    strides[0] = st[1] * 2;
    strides[1] = st[2] * 2;
    box[1] = box_slots;
    box[2] = 1;
  }
  dims[3] = static_cast<cuuint64_t>(num_blocks);
  strides[2] = st[0] * 2;
  box[3] = 1;
  std::memset(map, 0, sizeof(*map));
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return PKV_ERR_LAYOUT;
  *head_first = hf ? 1 : 0;
  return PKV_OK;
}

// TMA map over q [batch, seqlen_q, Hq, D] with element strides (b, s, h).
// The box is 64 head_dim x G heads x 128 / G tokens of one sequence: it lands
// as the 128 rows r = i * G + g of one row tile (row r at r * 128 bytes,
// 128-byte swizzled); tokens past seqlen_q read as zeros.
// Packed queries use the same box over dims (D, Hq, total_q, 1).
int make_q_map(CUtensorMap *map, const void *q, const int64_t st[3], int batch, int seqlen_q,
               int Hq, int D, int G) {
  auto enc = encode_fn();
  if (!enc) return PKV_ERR_CUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hq),
                        static_cast<cuuint64_t>(seqlen_q), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(st[2] * 2), static_cast<cuuint64_t>(st[1] * 2),
                           static_cast<cuuint64_t>(st[0] * 2)};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(G),
                       static_cast<cuuint32_t>(pkv::kRowsPerTile / G), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  std::memset(map, 0, sizeof(*map));
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(q), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_LAYOUT;
}

// Pipeline depth (K/V stages) and Q buffers per instance, sized to the
// 227 KB of shared memory one CTA may use.
template <int D, int N>
constexpr int stages() {
  return D == 128 ? (N == 16 ? 3 : 2) : (N == 16 ? 6 : 4);
}
template <int D, int N>
constexpr int q_buffers() {
  return (D == 128 && N == 64) ? 1 : 2;
}

template <int D, int N>
int launch_split(const pkv::AttnParams &p, const CUtensorMap &mk, const CUtensorMap &mv,
                 cudaStream_t s, int dev) {
  constexpr int NS = stages<D, N>();
  constexpr int QB = q_buffers<D, N>();
  using C = pkv::Cfg<D, N, NS, QB>;
  static_assert(C::kSmemBytes <= 232448, "shared memory budget");
  static std::atomic<bool> attr_set[kMaxDevices];
  auto kern = pkv::attn_split_kernel<D, N, NS, QB>;
  if (dev < 0 || dev >= kMaxDevices || !attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return PKV_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices) attr_set[dev].store(true, std::memory_order_release);
  }
  const int grid = p.n_units < sm_count(dev) ? p.n_units : sm_count(dev);
  // balanced unit order when the units fit the kernel's schedule scratch
  // (the kernel itself falls back to the stride-grid deal when its share of
  // the units with work overflows its list)
  pkv::AttnParams pp = p;
  pp.sched = p.n_units <= C::kSchedScratch ? 1 : 0;
  kern<<<grid, pkv::kThreads, C::kSmemBytes, s>>>(pp, mk, mv);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// The row-major kernel rebalances registers between warpgroups; the shares
// add up to exactly the allocation of a launch built with kRowsLaunchRegs
// registers per thread, so the launch is refused if the build differs.
template <int D>
int launch_rows(const pkv::AttnParams &p, const CUtensorMap &mk, const CUtensorMap &mv,
                const CUtensorMap &mq, cudaStream_t s, int dev) {
  constexpr int NS = D == 128 ? 2 : 4;
  using C = pkv::RowCfg<D, NS>;
  static_assert(C::kSmemBytes <= 232448, "shared memory budget");
  static std::atomic<bool> attr_set[kMaxDevices];
  auto kern = pkv::attn_rows_kernel<D, NS>;
  if (dev < 0 || dev >= kMaxDevices || !attr_set[dev].load(std::memory_order_acquire)) {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return PKV_ERR_CUDA;
    if (fa.numRegs != pkv::kRowsLaunchRegs) return PKV_ERR_CUDA;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return PKV_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices) attr_set[dev].store(true, std::memory_order_release);
  }
  const int grid = p.n_units < sm_count(dev) ? p.n_units : sm_count(dev);
  pkv::AttnParams pp = p;
  pp.sched = p.n_units <= C::kSchedScratch ? 1 : 0;
  kern<<<grid, pkv::kRowThreads, C::kSmemBytes, s>>>(pp, mk, mv, mq);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// Backward kernels: one CTA per key tile (dK, dV) and per row tile (dQ).
// Both hold 512 TMEM columns; shared memory is requested at >= 120 KB so that
// only one CTA of either kernel sits on an SM.
template <int D, bool kRowsTma>
int launch_bwd(const pkv::BwdParams &p, int64_t kv_ctas, int64_t q_ctas, const CUtensorMap &mk,
               const CUtensorMap &mv, const CUtensorMap &mq, const CUtensorMap &mg, cudaStream_t s) {
  constexpr int kKvSmem = pkv::BwdCfg<D>::kSmem > 120 * 1024 ? pkv::BwdCfg<D>::kSmem : 120 * 1024;
  constexpr int kQSmem = pkv::BwdQCfg<D>::kSmem > 120 * 1024 ? pkv::BwdQCfg<D>::kSmem : 120 * 1024;
  static_assert(kKvSmem <= 232448 && kQSmem <= 232448, "shared memory budget");
  auto kv = pkv::bwd_kv_kernel<D, kRowsTma>;
  auto qk = pkv::bwd_q_kernel<D, kRowsTma>;
  if (cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem) != cudaSuccess ||
      cudaFuncSetAttribute(qk, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem) != cudaSuccess)
    return PKV_ERR_CUDA;
  kv<<<static_cast<unsigned>(kv_ctas), pkv::kBwdThreads, kKvSmem, s>>>(p, mk, mv, mq, mg);
  if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
  qk<<<static_cast<unsigned>(q_ctas), pkv::kBwdQThreads, kQSmem, s>>>(p, mk, mv, mq, mg);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// Few rows (decode: rows x splits partials spread over one block per row)
// or many (prefill, packed batches: one warp per row).
// Few rows (decode: rows x splits partials spread over one block per row)
// or many (prefill, packed batches: one warp per row).
template <int D>
int launch_merge(const pkv::MergeParams &m, int64_t rows, cudaStream_t s) {
  if (rows <= 4096) {
    pkv::merge_kernel<D, true><<<static_cast<unsigned>(rows), D, 0, s>>>(m);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
  }
  // the warps stride over the rows: at most 8 blocks of 8 warps per SM
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  const int64_t need = ceil_div(rows, pkv::kMergeRowsPerBlock);
  const int64_t cap = static_cast<int64_t>(sm_count(dev)) * 8;
  const int64_t blocks = need < cap ? need : cap;
  pkv::merge_kernel<D, false><<<static_cast<unsigned>(blocks), 32 * pkv::kMergeRowsPerBlock, 0, s>>>(m);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// Rows of query heads x tokens per tile: 16 when a KV head's whole query
// group fits (decode), 64 up to 64 rows, else 128 rows in the row-major
// kernel -- when G divides 128 (a Q box is whole tokens) and the box's
// 128 / G tokens fit inside seqlen_q (no TMA box is ever larger than the
// tensor it reads); otherwise 64.  Every size runs the same arithmetic per row.
int rows_per_tile(int64_t rows, int G, int seqlen_q) {
  if (rows <= 16) return 16;
  if (rows <= 64 || pkv::kRowsPerTile % G != 0 || pkv::kRowsPerTile / G > seqlen_q) return 64;
  return pkv::kRowsPerTile;
}

// The append kernel: token t of sequence b to position seqlens[b] - seq_bias + t.
int launch_append(const void *k_new, const int64_t kn_strides[3], const void *v_new,
                  const int64_t vn_strides[3], void *k_cache, const int64_t k_strides[3],
                  void *v_cache, const int64_t v_strides[3], int64_t num_blocks,
                  const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                  const int32_t *seqlens, int batch, int n_new, int Hkv, int D, int block_size,
                  int seq_bias, int32_t *err, cudaStream_t stream,
                  const int32_t *cu_new = nullptr, int total_new = 0) {
  pkv::AppendParams p{};
  p.k_new = static_cast<const uint16_t *>(k_new);
  p.v_new = static_cast<const uint16_t *>(v_new);
  p.kn_sb = kn_strides[0];
  p.kn_st = kn_strides[1];
  p.kn_sh = kn_strides[2];
  p.vn_sb = vn_strides[0];
  p.vn_st = vn_strides[1];
  p.vn_sh = vn_strides[2];
  p.k_cache = static_cast<uint16_t *>(k_cache);
  p.v_cache = static_cast<uint16_t *>(v_cache);
  p.k_sb = k_strides[0];
  p.k_ss = k_strides[1];
  p.k_sh = k_strides[2];
  p.v_sb = v_strides[0];
  p.v_ss = v_strides[1];
  p.v_sh = v_strides[2];
  p.num_blocks = num_blocks;
  p.block_table = block_table;
  p.bt_stride = bt_stride;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.seqlens = seqlens;
  p.batch = batch;
  p.n_new = n_new;
  p.Hkv = Hkv;
  p.chunks = D / 8;
  p.block_shift = log2i(block_size);
  p.seq_bias = seq_bias;
  p.cu_new = cu_new;
  p.total_new = total_new;
  p.err = err;
  // one block per new token, a thread per 16-byte piece of its Hkv heads (up
  // to 256, looping beyond)
  const int64_t tokens = cu_new ? static_cast<int64_t>(total_new) : static_cast<int64_t>(batch) * n_new;
  if (tokens <= 0) return PKV_OK;
  if (tokens > INT32_MAX) return PKV_ERR_ARG;
  const int pieces = Hkv * (D / 8);
  const int threads = pieces < 256 ? ((pieces + 31) / 32) * 32 : 256;
  pkv::kv_append_kernel<<<static_cast<unsigned>(tokens), threads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// New tokens written into the cache by the attention call itself.  The
// producers write them just before loading the tiles that hold them when
// there are few (decode steps) and one row tile reads them.
constexpr int kFuseMaxNew = 16;
struct FusedAppend {
  const void *k_new, *v_new;
  const int64_t *kn_strides, *vn_strides;
  int n_new;
};

// Packed (varlen) queries: cu_q [batch + 1] on the device, total_q tokens;
// optional copies of each sequence's last query row.
struct PackedQ {
  const int32_t *cu_q;
  int total_q;
  void *fin_out;
  const int64_t *fin_strides;  // (batch, head)
  float *fin_lse;
};

// Context-parallel share: partials of absolute splits [split_begin,
// split_begin + n_local) into `partials` (acc then ml, local split order);
// nothing is merged or written to out / lse.
struct SplitShare {
  int split_begin, n_local;
};

int attn_entry(const void *q, const int64_t q_strides[3], const void *k_cache,
               const int64_t k_strides[3], const void *v_cache, const int64_t v_strides[3],
               int64_t num_blocks, const int32_t *block_table, int64_t bt_stride,
               int max_blocks_per_seq, const int32_t *seqlens, int max_seqlen_k, int batch,
               int seqlen_q, int Hq, int Hkv, int D, int block_size, float scale, int causal,
               void *out, const int64_t out_strides[3], float *lse, void *workspace,
               size_t workspace_bytes, int32_t *err, void *stream,
               const FusedAppend *app = nullptr, const PackedQ *pq = nullptr,
               const SplitShare *share = nullptr, uint64_t wait_ns = pkv::kWaitTimeoutNs) {
  if (!q || !k_cache || !v_cache || !block_table || !seqlens) return PKV_ERR_ARG;
  if (!share && (!out || !lse)) return PKV_ERR_ARG;
  if (share && (pq || app || share->split_begin < 0 || share->n_local <= 0)) return PKV_ERR_ARG;
  if (batch <= 0 || seqlen_q <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return PKV_ERR_ARG;
  if (D != 64 && D != 128) return PKV_ERR_ARG;
  if (!pow2_in(block_size, 16, 256)) return PKV_ERR_ARG;
  if (num_blocks <= 0 || num_blocks > INT32_MAX || max_blocks_per_seq <= 0 || bt_stride < max_blocks_per_seq)
    return PKV_ERR_ARG;
  if (max_seqlen_k < 0) return PKV_ERR_ARG;
  if (!strides_ok(q_strides) || !strides_ok(k_strides) || !strides_ok(v_strides)) return PKV_ERR_ARG;
  if (!share && (!out_strides || out_strides[0] <= 0 || out_strides[1] <= 0 || out_strides[2] <= 0))
    return PKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PKV_ERR_ARG;
  if (!(scale > 0.f) || !(scale < 3.0e38f)) return PKV_ERR_ARG;
  const int G = Hq / Hkv;
  const int64_t R = static_cast<int64_t>(G) * seqlen_q;
  if (pq && (!pq->cu_q || pq->total_q <= 0 || (app && app->n_new > 0))) return PKV_ERR_ARG;
  if (pq && pq->fin_out && (!pq->fin_lse || !pq->fin_strides || pq->fin_strides[0] <= 0 ||
                            pq->fin_strides[1] <= 0))
    return PKV_ERR_ARG;
  const int64_t tokens = pq ? static_cast<int64_t>(pq->total_q) : static_cast<int64_t>(batch) * seqlen_q;
  const int64_t rows = tokens * Hq;
  if (R > INT32_MAX / 2 || rows > INT32_MAX) return PKV_ERR_ARG;
  alignas(64) CUtensorMap mq;
  // (a Q box spans 128 / G tokens: of one sequence when dense, of the packed
  // token axis otherwise)
  int N = rows_per_tile(R, G, pq ? pq->total_q : seqlen_q);
  if (N == pkv::kRowsPerTile &&
      (pq ? make_q_map(&mq, q, q_strides, 1, pq->total_q, Hq, D, G)
          : make_q_map(&mq, q, q_strides, batch, seqlen_q, Hq, D, G)) != PKV_OK)
    N = 64;  // q's strides cannot be described to the TMA unit: transposed kernel
  const int64_t S = share ? share->n_local
                          : (max_seqlen_k > 0 ? ceil_div(max_seqlen_k, pkv::kSplitTokens) : 1);
  const int64_t RT = ceil_div(R, N);
  const int64_t units = static_cast<int64_t>(batch) * S * Hkv * RT;
  if (units > INT32_MAX) return PKV_ERR_ARG;
  const size_t need = share ? ws_bytes(batch, seqlen_q, Hq, D, static_cast<int>(S) * pkv::kSplitTokens)
                     : pq ? ws_bytes(1, pq->total_q, Hq, D, max_seqlen_k)
                          : ws_bytes(batch, seqlen_q, Hq, D, max_seqlen_k);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PKV_ERR_WORKSPACE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  const int box_slots = block_size < pkv::kTileTokens ? block_size : pkv::kTileTokens;
  alignas(64) CUtensorMap mk, mv;
  int hf_k = 0, hf_v = 0;
  int rc = make_kv_map(&mk, k_cache, k_strides, num_blocks, block_size, Hkv, D, box_slots, &hf_k);
  if (rc != PKV_OK) return rc;
  rc = make_kv_map(&mv, v_cache, v_strides, num_blocks, block_size, Hkv, D, box_slots, &hf_v);
  if (rc != PKV_OK) return rc;
  if (hf_k != hf_v) return PKV_ERR_LAYOUT;  // K and V must order head/slot alike

  float *ws_acc = static_cast<float *>(workspace);
  float *ws_ml = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                           ws_acc_bytes(rows, S, D));
  pkv::AttnParams p{};
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.q_sb = q_strides[0];
  p.q_ss = q_strides[1];
  p.q_sh = q_strides[2];
  p.block_table = block_table;
  p.bt_stride = bt_stride;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.seqlens = seqlens;
  p.batch = batch;
  p.seqlen_q = seqlen_q;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.block_shift = log2i(block_size);
  p.box_slots = box_slots;
  p.map_head_first = hf_k;
  p.n_row_tiles = static_cast<int>(RT);
  p.n_splits = static_cast<int>(S);
  p.n_units = static_cast<int>(units);
  p.max_seqlen_k = max_seqlen_k;
  p.wait_ns = wait_ns;
  p.cscale = scale * 1.4426950408889634f;  // host IEEE multiply, one rounding
  p.causal = causal ? 1 : 0;
  p.ws_acc = ws_acc;
  p.ws_ml = ws_ml;
  p.err = err;
  p.nq_lo = 0;
  p.nq_hi = INT_MAX;
  if (share) {
    p.split_base = share->split_begin;
    p.part_only = 1;
  }
  if (pq) {
    p.cu_q = pq->cu_q;
    p.total_q = pq->total_q;
    if (pq->fin_out) {
      p.fin_out = static_cast<__nv_bfloat16 *>(pq->fin_out);
      p.fo_sb = pq->fin_strides[0];
      p.fo_sh = pq->fin_strides[1];
      p.fin_lse = pq->fin_lse;
    }
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (app && app->n_new > 0) {
    if (!app->k_new || !app->v_new || !strides_ok(app->kn_strides) ||
        !strides_ok(app->vn_strides) || !aligned16(app->k_new) || !aligned16(app->v_new) ||
        app->n_new > pkv::kSplitTokens)
      return PKV_ERR_ARG;
  }
  if (app && app->n_new > 0 && (app->n_new > kFuseMaxNew || RT > 1)) {
    // Many new tokens, or several row tiles that would each write them: one
    // append launch first (the same bits in the cache), then plain attention.
    rc = launch_append(app->k_new, app->kn_strides, app->v_new, app->vn_strides,
                       const_cast<void *>(k_cache), k_strides, const_cast<void *>(v_cache),
                       v_strides, num_blocks, block_table, bt_stride, max_blocks_per_seq, seqlens,
                       batch, app->n_new, Hkv, D, block_size, app->n_new, err, s);
    if (rc != PKV_OK) return rc;
  } else if (app && app->n_new > 0) {
    p.n_new = app->n_new;
    p.k_new = static_cast<const uint16_t *>(app->k_new);
    p.v_new = static_cast<const uint16_t *>(app->v_new);
    p.kn_sb = app->kn_strides[0];
    p.kn_st = app->kn_strides[1];
    p.kn_sh = app->kn_strides[2];
    p.vn_sb = app->vn_strides[0];
    p.vn_st = app->vn_strides[1];
    p.vn_sh = app->vn_strides[2];
    p.k_cache = static_cast<uint16_t *>(const_cast<void *>(k_cache));
    p.v_cache = static_cast<uint16_t *>(const_cast<void *>(v_cache));
    p.k_sb = k_strides[0];
    p.k_ss = k_strides[1];
    p.k_sh = k_strides[2];
    p.v_sb = v_strides[0];
    p.v_ss = v_strides[1];
    p.v_sh = v_strides[2];
  }

  // Every row of a call with one split is finished by the kernel that computed
  // it, with the merge's fold of one partial (the same bits): no merge launch.
  // With more splits the row-major kernel still finishes rows of at most one
  // split and the merge skips them.
  p.direct = (S == 1 && !share) ? 1 : 0;
  if (!share) {
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.o_sb = out_strides[0];
    p.o_ss = out_strides[1];
    p.o_sh = out_strides[2];
    p.lse = lse;
    p.out_vec = (aligned16(out) && out_strides[0] % 8 == 0 && out_strides[1] % 8 == 0 &&
                 out_strides[2] % 8 == 0)
                    ? 1
                    : 0;
  }
  // A packed call whose longest request needs the row-major kernel also
  // serves its short requests (at most 16 / G queries: one 16-row tile) with
  // the transposed kernel, which keeps decode steps at memory speed; each
  // launch skips the other's sequences.
  const int small_nq = G <= 16 ? 16 / G : 0;
  const bool split_by_size = pq && N == pkv::kRowsPerTile && small_nq > 0;
  if (split_by_size) {
    pkv::AttnParams ps = p;
    ps.nq_lo = 1;
    ps.nq_hi = small_nq;
    ps.n_row_tiles = 1;
    ps.n_units = static_cast<int>(static_cast<int64_t>(batch) * S * Hkv);
    rc = D == 128 ? launch_split<128, 16>(ps, mk, mv, s, dev) : launch_split<64, 16>(ps, mk, mv, s, dev);
    if (rc != PKV_OK) return rc;
    p.nq_lo = small_nq + 1;
  }
  if (N == pkv::kRowsPerTile) {
    rc = D == 128 ? launch_rows<128>(p, mk, mv, mq, s, dev) : launch_rows<64>(p, mk, mv, mq, s, dev);
  } else if (D == 128) {
    rc = N == 16 ? launch_split<128, 16>(p, mk, mv, s, dev) : launch_split<128, 64>(p, mk, mv, s, dev);
  } else {
    rc = N == 16 ? launch_split<64, 16>(p, mk, mv, s, dev) : launch_split<64, 64>(p, mk, mv, s, dev);
  }
  if (rc != PKV_OK || share || p.direct) return rc;

  pkv::MergeParams m{};
  m.seqlens = seqlens;
  m.seqlen_q = seqlen_q;
  m.Hq = Hq;
  m.n_splits = static_cast<int>(S);
  m.causal = p.causal;
  m.ws_acc = ws_acc;
  m.ws_ml = ws_ml;
  m.out = static_cast<__nv_bfloat16 *>(out);
  m.o_sb = out_strides[0];
  m.o_ss = out_strides[1];
  m.o_sh = out_strides[2];
  m.lse = lse;
  m.cu_q = p.cu_q;
  m.batch = batch;
  m.total_q = p.total_q;
  m.fin_out = p.fin_out;
  m.fo_sb = p.fo_sb;
  m.fo_sh = p.fo_sh;
  m.fin_lse = p.fin_lse;
  m.rows = rows;
  m.skip_single = N == pkv::kRowsPerTile ? 1 : 0;
  m.skip_min_nq = split_by_size ? small_nq + 1 : 0;
  m.n_local = static_cast<int>(S);
  m.rank_floats = 0;
  return D == 128 ? launch_merge<128>(m, rows, s) : launch_merge<64>(m, rows, s);
}

}  // namespace

extern "C" {

int pkv_kv_append(const void *k_new, const int64_t kn_strides[3], const void *v_new,
                  const int64_t vn_strides[3], void *k_cache, const int64_t k_strides[3],
                  void *v_cache, const int64_t v_strides[3], int64_t num_blocks,
                  const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                  const int32_t *seqlens, int batch, int n_new, int Hkv, int D, int block_size,
                  int32_t *err, void *stream) {
  if (!k_new || !v_new || !k_cache || !v_cache || !block_table || !seqlens) return PKV_ERR_ARG;
  if (batch <= 0 || n_new < 0 || Hkv <= 0 || (D != 64 && D != 128)) return PKV_ERR_ARG;
  if (!pow2_in(block_size, 16, 256)) return PKV_ERR_ARG;
  if (num_blocks <= 0 || num_blocks > INT32_MAX || max_blocks_per_seq <= 0 || bt_stride < max_blocks_per_seq)
    return PKV_ERR_ARG;
  if (!strides_ok(kn_strides) || !strides_ok(vn_strides) || !strides_ok(k_strides) ||
      !strides_ok(v_strides))
    return PKV_ERR_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_ARG;
  if (n_new == 0) return PKV_OK;
  return launch_append(k_new, kn_strides, v_new, vn_strides, k_cache, k_strides, v_cache,
                       v_strides, num_blocks, block_table, bt_stride, max_blocks_per_seq, seqlens,
                       batch, n_new, Hkv, D, block_size, 0, err, static_cast<cudaStream_t>(stream));
}

int pkv_paged_decode_attn(const void *q, const int64_t q_strides[3], const void *k_cache,
                          const int64_t k_strides[3], const void *v_cache,
                          const int64_t v_strides[3], int64_t num_blocks,
                          const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                          const int32_t *seqlens, int max_seqlen_k, int batch, int seqlen_q,
                          int Hq, int Hkv, int D, int block_size, float scale, int causal,
                          void *out, const int64_t out_strides[3], float *lse, void *workspace,
                          size_t workspace_bytes, int32_t *err, void *stream) {
  return attn_entry(q, q_strides, k_cache, k_strides, v_cache, v_strides, num_blocks, block_table,
                    bt_stride, max_blocks_per_seq, seqlens, max_seqlen_k, batch, seqlen_q, Hq, Hkv,
                    D, block_size, scale, causal, out, out_strides, lse, workspace,
                    workspace_bytes, err, stream);
}

int pkv_paged_prefill_attn(const void *q, const int64_t q_strides[3], const void *k_cache,
                           const int64_t k_strides[3], const void *v_cache,
                           const int64_t v_strides[3], int64_t num_blocks,
                           const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                           const int32_t *seqlens, int max_seqlen_k, int batch, int seqlen_q,
                           int Hq, int Hkv, int D, int block_size, float scale, int causal,
                           void *out, const int64_t out_strides[3], float *lse, void *workspace,
                           size_t workspace_bytes, int32_t *err, void *stream) {
  return attn_entry(q, q_strides, k_cache, k_strides, v_cache, v_strides, num_blocks, block_table,
                    bt_stride, max_blocks_per_seq, seqlens, max_seqlen_k, batch, seqlen_q, Hq, Hkv,
                    D, block_size, scale, causal, out, out_strides, lse, workspace,
                    workspace_bytes, err, stream);
}

int pkv_debug_paged_decode_attn(const void *q, const int64_t q_strides[3], const void *k_cache,
                                const int64_t k_strides[3], const void *v_cache,
                                const int64_t v_strides[3], int64_t num_blocks,
                                const int32_t *block_table, int64_t bt_stride,
                                int max_blocks_per_seq, const int32_t *seqlens, int max_seqlen_k,
                                int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                                float scale, int causal, void *out, const int64_t out_strides[3],
                                float *lse, void *workspace, size_t workspace_bytes, int32_t *err,
                                void *stream, uint64_t wait_limit_ns) {
  if (wait_limit_ns > pkv::kWaitTimeoutNs) return PKV_ERR_ARG;
  return attn_entry(q, q_strides, k_cache, k_strides, v_cache, v_strides, num_blocks, block_table,
                    bt_stride, max_blocks_per_seq, seqlens, max_seqlen_k, batch, seqlen_q, Hq, Hkv,
                    D, block_size, scale, causal, out, out_strides, lse, workspace,
                    workspace_bytes, err, stream, nullptr, nullptr, nullptr, wait_limit_ns);
}

namespace {
__global__ void final_out_kernel(const float *A, const float *L, float *out, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = pkv::final_out(A[i], L[i], pkv::final_rcp(L[i]));
}
}  // namespace

int pkv_debug_final_out(const float *A, const float *L, float *out, int64_t n, void *stream) {
  if (n < 0 || (n > 0 && (!A || !L || !out))) return PKV_ERR_ARG;
  if (n == 0) return PKV_OK;
  if (ceil_div(n, 256) > INT32_MAX) return PKV_ERR_ARG;
  final_out_kernel<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      A, L, out, n);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_paged_decode_attn_append(const void *q, const int64_t q_strides[3], const void *k_new,
                                 const int64_t kn_strides[3], const void *v_new,
                                 const int64_t vn_strides[3], int n_new, void *k_cache,
                                 const int64_t k_strides[3], void *v_cache,
                                 const int64_t v_strides[3], int64_t num_blocks,
                                 const int32_t *block_table, int64_t bt_stride,
                                 int max_blocks_per_seq, const int32_t *seqlens, int max_seqlen_k,
                                 int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                                 float scale, int causal, void *out, const int64_t out_strides[3],
                                 float *lse, void *workspace, size_t workspace_bytes, int32_t *err,
                                 void *stream) {
  if (n_new < 1) return PKV_ERR_ARG;
  const FusedAppend app{k_new, v_new, kn_strides, vn_strides, n_new};
  return attn_entry(q, q_strides, k_cache, k_strides, v_cache, v_strides, num_blocks, block_table,
                    bt_stride, max_blocks_per_seq, seqlens, max_seqlen_k, batch, seqlen_q, Hq, Hkv,
                    D, block_size, scale, causal, out, out_strides, lse, workspace,
                    workspace_bytes, err, stream, &app);
}

int pkv_paged_varlen_attn(const void *q, const int64_t q_strides[2], const int32_t *cu_seqlens_q,
                          int total_q, int max_seqlen_q, const void *k_cache,
                          const int64_t k_strides[3], const void *v_cache,
                          const int64_t v_strides[3], int64_t num_blocks,
                          const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                          const int32_t *seqlens, int max_seqlen_k, int batch, int Hq, int Hkv,
                          int D, int block_size, float scale, int causal, void *out,
                          const int64_t out_strides[2], float *lse, void *final_out,
                          const int64_t final_strides[2], float *final_lse, void *workspace,
                          size_t workspace_bytes, int32_t *err, void *stream) {
  if (!q_strides || !out_strides || !cu_seqlens_q || total_q <= 0 || max_seqlen_q <= 0)
    return PKV_ERR_ARG;
  // the batch stride of the packed views is never used; repeat the token stride
  const int64_t qs[3] = {q_strides[0], q_strides[0], q_strides[1]};
  const int64_t os[3] = {out_strides[0], out_strides[0], out_strides[1]};
  const PackedQ pq{cu_seqlens_q, total_q, final_out, final_strides, final_lse};
  return attn_entry(q, qs, k_cache, k_strides, v_cache, v_strides, num_blocks, block_table,
                    bt_stride, max_blocks_per_seq, seqlens, max_seqlen_k, batch, max_seqlen_q, Hq,
                    Hkv, D, block_size, scale, causal, out, os, lse, workspace, workspace_bytes,
                    err, stream, nullptr, &pq);
}

size_t pkv_varlen_workspace_size(int total_q, int Hq, int D, int max_seqlen_k) {
  if (total_q <= 0 || Hq <= 0 || D <= 0 || max_seqlen_k < 0) return 0;
  return ws_bytes(1, total_q, Hq, D, max_seqlen_k);
}

int pkv_kv_append_varlen(const void *k_new, const int64_t kn_strides[2], const void *v_new,
                         const int64_t vn_strides[2], const int32_t *cu_seqlens_new, int total_new,
                         void *k_cache, const int64_t k_strides[3], void *v_cache,
                         const int64_t v_strides[3], int64_t num_blocks,
                         const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                         const int32_t *seqlens, int batch, int Hkv, int D, int block_size,
                         int32_t *err, void *stream) {
  if (!k_new || !v_new || !k_cache || !v_cache || !block_table || !seqlens || !cu_seqlens_new ||
      !kn_strides || !vn_strides)
    return PKV_ERR_ARG;
  if (batch <= 0 || total_new < 0 || Hkv <= 0 || (D != 64 && D != 128)) return PKV_ERR_ARG;
  if (!pow2_in(block_size, 16, 256)) return PKV_ERR_ARG;
  if (num_blocks <= 0 || num_blocks > INT32_MAX || max_blocks_per_seq <= 0 || bt_stride < max_blocks_per_seq)
    return PKV_ERR_ARG;
  const int64_t kn[3] = {kn_strides[0], kn_strides[0], kn_strides[1]};
  const int64_t vn[3] = {vn_strides[0], vn_strides[0], vn_strides[1]};
  if (!strides_ok(kn) || !strides_ok(vn) || !strides_ok(k_strides) || !strides_ok(v_strides))
    return PKV_ERR_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
    return PKV_ERR_ARG;
  if (total_new == 0) return PKV_OK;
  return launch_append(k_new, kn, v_new, vn, k_cache, k_strides, v_cache, v_strides, num_blocks,
                       block_table, bt_stride, max_blocks_per_seq, seqlens, batch, 0, Hkv, D,
                       block_size, 0, err, static_cast<cudaStream_t>(stream), cu_seqlens_new,
                       total_new);
}

int pkv_paged_attn_partials(const void *q, const int64_t q_strides[3], const void *k_cache,
                            const int64_t k_strides[3], const void *v_cache,
                            const int64_t v_strides[3], int64_t num_blocks,
                            const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                            const int32_t *seqlens, int batch, int seqlen_q, int Hq, int Hkv,
                            int D, int block_size, float scale, int causal, int split_begin,
                            int n_splits_local, void *partials, size_t partials_bytes,
                            int32_t *err, void *stream) {
  const SplitShare share{split_begin, n_splits_local};
  return attn_entry(q, q_strides, k_cache, k_strides, v_cache, v_strides, num_blocks, block_table,
                    bt_stride, max_blocks_per_seq, seqlens,
                    (split_begin + n_splits_local) * pkv::kSplitTokens, batch, seqlen_q, Hq, Hkv,
                    D, block_size, scale, causal, nullptr, nullptr, nullptr, partials,
                    partials_bytes, err, stream, nullptr, nullptr, &share);
}

size_t pkv_partials_size(int batch, int seqlen_q, int Hq, int D, int n_splits_local) {
  if (batch <= 0 || seqlen_q <= 0 || Hq <= 0 || D <= 0 || n_splits_local <= 0) return 0;
  return ws_bytes(batch, seqlen_q, Hq, D, n_splits_local * pkv::kSplitTokens);
}

int pkv_merge_partials(const void *partials, int world, int n_splits_local, size_t rank_bytes,
                       const int32_t *seqlens, int batch, int seqlen_q, int Hq, int D, int causal,
                       void *out, const int64_t out_strides[3], float *lse, void *stream) {
  if (!partials || !seqlens || !out || !lse || !out_strides) return PKV_ERR_ARG;
  if (world <= 0 || n_splits_local <= 0 || batch <= 0 || seqlen_q <= 0 || Hq <= 0 ||
      (D != 64 && D != 128))
    return PKV_ERR_ARG;
  if (out_strides[0] <= 0 || out_strides[1] <= 0 || out_strides[2] <= 0) return PKV_ERR_ARG;
  const int64_t rows = static_cast<int64_t>(batch) * seqlen_q * Hq;
  if (rows > INT32_MAX) return PKV_ERR_ARG;
  const size_t acc_bytes = ws_acc_bytes(rows, n_splits_local, D);
  if (rank_bytes < acc_bytes + static_cast<size_t>(rows) * n_splits_local * 2 * sizeof(float) ||
      rank_bytes % 16 != 0 || !aligned16(partials))
    return PKV_ERR_WORKSPACE;
  pkv::MergeParams m{};
  m.seqlens = seqlens;
  m.seqlen_q = seqlen_q;
  m.Hq = Hq;
  m.n_splits = world * n_splits_local;
  m.causal = causal ? 1 : 0;
  m.ws_acc = static_cast<const float *>(partials);
  m.ws_ml = reinterpret_cast<const float *>(static_cast<const uint8_t *>(partials) + acc_bytes);
  m.out = static_cast<__nv_bfloat16 *>(out);
  m.o_sb = out_strides[0];
  m.o_ss = out_strides[1];
  m.o_sh = out_strides[2];
  m.lse = lse;
  m.batch = batch;
  m.rows = rows;
  m.skip_single = 0;
  m.n_local = n_splits_local;
  m.rank_floats = static_cast<int64_t>(rank_bytes / sizeof(float));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch_merge<128>(m, rows, s) : launch_merge<64>(m, rows, s);
}

size_t pkv_bwd_workspace_size(int batch, int seqlen_q, int Hq) {
  if (batch <= 0 || seqlen_q <= 0 || Hq <= 0) return 0;
  const size_t rows = static_cast<size_t>(batch) * seqlen_q * Hq;
  return 2 * ((rows * sizeof(float) + 255) & ~static_cast<size_t>(255));
}

int pkv_paged_prefill_attn_bwd(const void *q, const int64_t q_strides[3], const void *k_cache,
                               const int64_t k_strides[3], const void *v_cache,
                               const int64_t v_strides[3], int64_t num_blocks,
                               const int32_t *block_table, int64_t bt_stride,
                               int max_blocks_per_seq, const int32_t *seqlens, int max_seqlen_k,
                               int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                               float scale, int causal, const void *out,
                               const int64_t out_strides[3], const float *lse, const void *dout,
                               const int64_t dout_strides[3], void *dq,
                               const int64_t dq_strides[3], void *dk_cache,
                               const int64_t dk_strides[3], void *dv_cache,
                               const int64_t dv_strides[3], void *workspace,
                               size_t workspace_bytes, int32_t *err, void *stream) {
  if (!q || !k_cache || !v_cache || !block_table || !seqlens || !out || !lse || !dout || !dq ||
      !dk_cache || !dv_cache)
    return PKV_ERR_ARG;
  if (batch <= 0 || seqlen_q <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return PKV_ERR_ARG;
  if (D != 64 && D != 128) return PKV_ERR_ARG;
  if (!pow2_in(block_size, 16, 256)) return PKV_ERR_ARG;
  if (num_blocks <= 0 || num_blocks > INT32_MAX || max_blocks_per_seq <= 0 ||
      bt_stride < max_blocks_per_seq || max_seqlen_k < 0)
    return PKV_ERR_ARG;
  if (!strides_ok(q_strides) || !strides_ok(k_strides) || !strides_ok(v_strides) ||
      !strides_ok(dout_strides) || !strides_ok(dq_strides) || !strides_ok(dk_strides) ||
      !strides_ok(dv_strides))
    return PKV_ERR_ARG;
  if (!strides_ok(out_strides)) return PKV_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(dout) ||
      !aligned16(out) ||
      !aligned16(dq) || !aligned16(dk_cache) || !aligned16(dv_cache))
    return PKV_ERR_ARG;
  if (!(scale > 0.f) || !(scale < 3.0e38f)) return PKV_ERR_ARG;
  const int G = Hq / Hkv;
  const int64_t rows = static_cast<int64_t>(batch) * seqlen_q * Hq;
  const int64_t R = static_cast<int64_t>(G) * seqlen_q;
  if (rows > INT32_MAX || R > INT32_MAX / 2) return PKV_ERR_ARG;
  const size_t need = pkv_bwd_workspace_size(batch, seqlen_q, Hq);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return PKV_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float *row_d = static_cast<float *>(workspace);
  float *row_lse2 = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + need / 2);

  pkv::BwdPrepParams pp{};
  pp.dout = static_cast<const __nv_bfloat16 *>(dout);
  pp.out = static_cast<const __nv_bfloat16 *>(out);
  pp.g_sb = dout_strides[0];
  pp.g_ss = dout_strides[1];
  pp.g_sh = dout_strides[2];
  pp.o_sb = out_strides[0];
  pp.o_ss = out_strides[1];
  pp.o_sh = out_strides[2];
  pp.lse = lse;
  pp.batch = batch;
  pp.seqlen_q = seqlen_q;
  pp.Hq = Hq;
  pp.D = D;
  pp.row_d = row_d;
  pp.row_lse2 = row_lse2;
  pp.seqlens = seqlens;
  pp.max_seqlen_k = max_seqlen_k;
  pp.err = err;
  pkv::bwd_prep_kernel<<<static_cast<unsigned>(ceil_div(rows, 8)), 256, 0, s>>>(pp);
  if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;

  pkv::BwdParams p{};
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.dout = static_cast<const __nv_bfloat16 *>(dout);
  p.q_sb = q_strides[0];
  p.q_ss = q_strides[1];
  p.q_sh = q_strides[2];
  p.g_sb = dout_strides[0];
  p.g_ss = dout_strides[1];
  p.g_sh = dout_strides[2];
  p.k_cache = static_cast<const __nv_bfloat16 *>(k_cache);
  p.v_cache = static_cast<const __nv_bfloat16 *>(v_cache);
  p.k_sb = k_strides[0];
  p.k_ss = k_strides[1];
  p.k_sh = k_strides[2];
  p.v_sb = v_strides[0];
  p.v_ss = v_strides[1];
  p.v_sh = v_strides[2];
  p.dk_cache = static_cast<__nv_bfloat16 *>(dk_cache);
  p.dv_cache = static_cast<__nv_bfloat16 *>(dv_cache);
  p.dk_sb = dk_strides[0];
  p.dk_ss = dk_strides[1];
  p.dk_sh = dk_strides[2];
  p.dv_sb = dv_strides[0];
  p.dv_ss = dv_strides[1];
  p.dv_sh = dv_strides[2];
  p.dq = static_cast<__nv_bfloat16 *>(dq);
  p.dq_sb = dq_strides[0];
  p.dq_ss = dq_strides[1];
  p.dq_sh = dq_strides[2];
  p.block_table = block_table;
  p.bt_stride = bt_stride;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_blocks = num_blocks;
  p.seqlens = seqlens;
  p.batch = batch;
  p.seqlen_q = seqlen_q;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.block_shift = log2i(block_size);
  p.causal = causal ? 1 : 0;
  p.n_key_tiles = static_cast<int>(ceil_div(max_seqlen_k > 0 ? max_seqlen_k : 1, pkv::kBwdTile));
  p.n_row_tiles = static_cast<int>(ceil_div(R, pkv::kBwdTile));
  p.cscale = scale * 1.4426950408889634f;
  p.scale = scale;
  p.row_d = row_d;
  p.row_lse2 = row_lse2;
  p.err = err;
  const int64_t kv_ctas = static_cast<int64_t>(batch) * Hkv * p.n_key_tiles;
  const int64_t q_ctas = static_cast<int64_t>(batch) * Hkv * p.n_row_tiles;
  if (kv_ctas > INT32_MAX || q_ctas > INT32_MAX) return PKV_ERR_ARG;
  // K / V tiles through the same TMA boxes as the forward; Q / dO row tiles
  // as one box of 128 / G tokens x G heads where that covers the tile.
  const int box_slots = block_size < pkv::kBwdTile ? block_size : pkv::kBwdTile;
  alignas(64) CUtensorMap mk, mv, mq, mg;
  int hf_k = 0, hf_v = 0;
  int rc = make_kv_map(&mk, k_cache, k_strides, num_blocks, block_size, Hkv, D, box_slots, &hf_k);
  if (rc != PKV_OK) return rc;
  rc = make_kv_map(&mv, v_cache, v_strides, num_blocks, block_size, Hkv, D, box_slots, &hf_v);
  if (rc != PKV_OK) return rc;
  if (hf_k != hf_v) return PKV_ERR_LAYOUT;
  p.box_slots = box_slots;
  p.map_head_first = hf_k;
  std::memset(&mq, 0, sizeof(mq));
  std::memset(&mg, 0, sizeof(mg));
  const bool rows_tma = G <= pkv::kBwdTile && pkv::kBwdTile % G == 0 && pkv::kBwdTile / G <= seqlen_q &&
                        make_q_map(&mq, q, q_strides, batch, seqlen_q, Hq, D, G) == PKV_OK &&
                        make_q_map(&mg, dout, dout_strides, batch, seqlen_q, Hq, D, G) == PKV_OK;
  if (D == 128)
    return rows_tma ? launch_bwd<128, true>(p, kv_ctas, q_ctas, mk, mv, mq, mg, s)
                    : launch_bwd<128, false>(p, kv_ctas, q_ctas, mk, mv, mq, mg, s);
  return rows_tma ? launch_bwd<64, true>(p, kv_ctas, q_ctas, mk, mv, mq, mg, s)
                  : launch_bwd<64, false>(p, kv_ctas, q_ctas, mk, mv, mq, mg, s);
}

size_t pkv_workspace_size(int batch, int seqlen_q, int Hq, int D, int max_seqlen_k) {
  if (batch <= 0 || seqlen_q <= 0 || Hq <= 0 || D <= 0 || max_seqlen_k < 0) return 0;
  return ws_bytes(batch, seqlen_q, Hq, D, max_seqlen_k);
}

const char *pkv_strerror(int code) {
  switch (code) {
    case PKV_OK: return "ok";
    case PKV_ERR_ARG: return "invalid argument (size, stride, alignment or pointer)";
    case PKV_ERR_WORKSPACE: return "workspace missing, misaligned or smaller than pkv_workspace_size()";
    case PKV_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
    case PKV_ERR_LAYOUT: return "cache strides cannot be described to the TMA unit";
    default: return "unknown pagedkv status";
  }
}

int pkv_split_tokens(void) { return PKV_SPLIT_TOKENS; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode: scratch in a library-owned device array.
// ---------------------------------------------------------------------------
// For callers that may not allocate device memory at call time (see
// pkv_paged_decode_attn_static_ws in pagedkv.h).  In host code
// g_static_workspace is only a host-side stand-in for the device array: its
// device address comes from cudaGetSymbolAddress, once per device, and only
// that address is handed to the kernels.
static __device__ __align__(256) unsigned char g_static_workspace[PKV_STATIC_WORKSPACE_BYTES];

namespace {

void *static_workspace_address(int dev) {
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" {

int pkv_paged_decode_attn_static_ws(const void *q, const int64_t q_strides[3],
                                    const void *k_cache, const int64_t k_strides[3],
                                    const void *v_cache, const int64_t v_strides[3],
                                    int64_t num_blocks, const int32_t *block_table,
                                    int64_t bt_stride, int max_blocks_per_seq,
                                    const int32_t *seqlens, int max_seqlen_k, int batch,
                                    int seqlen_q, int Hq, int Hkv, int D, int block_size,
                                    float scale, int causal, void *out,
                                    const int64_t out_strides[3], float *lse, int32_t *err,
                                    void *stream) {
  if (batch <= 0 || seqlen_q <= 0 || Hq <= 0 || (D != 64 && D != 128) || max_seqlen_k < 0)
    return PKV_ERR_ARG;
  if (ws_bytes(batch, seqlen_q, Hq, D, max_seqlen_k) > PKV_STATIC_WORKSPACE_BYTES)
    return PKV_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  void *ws = static_workspace_address(dev);
  if (!ws) return PKV_ERR_CUDA;
  return attn_entry(q, q_strides, k_cache, k_strides, v_cache, v_strides, num_blocks, block_table,
                    bt_stride, max_blocks_per_seq, seqlens, max_seqlen_k, batch, seqlen_q, Hq, Hkv,
                    D, block_size, scale, causal, out, out_strides, lse, ws,
                    PKV_STATIC_WORKSPACE_BYTES, err, stream);
}

}  // extern "C"
