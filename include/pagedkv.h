/*
 * pagedkv.h -- C ABI of the B200 (sm_100a) paged-KV attention library
 * (libpagedkv.so).
 *
 * Three operations, all enqueued on the caller's CUDA stream:
 *
 *   pkv_kv_append          write new K/V tokens into cache blocks;
 *   pkv_paged_decode_attn  attention of one or a few query tokens against a
 *                          paged KV cache (split-K / flash-decoding over a
 *                          block table), returning out and lse;
 *   pkv_paged_prefill_attn causal or chunked prefill over the same cache,
 *                          under the same reduction contract.
 *
 * The call shape follows flash_attn_with_kvcache(q, k_cache, v_cache,
 * cache_seqlens=, page_table=, causal=) as exercised by ROCm/aiter commit
 * d293d61 "test(triton/decode): pin non-contiguous paged KV block stride"
 * (test_flash_attn_kvcache_noncontiguous_paged), extended with lse, an
 * explicit softmax scale, the real per-component cache strides and kv_append.
 *
 * Reduction contract (shared by decode and prefill).  The KV context of every
 * query row is cut into fixed chunks ("splits") of PKV_SPLIT_TOKENS tokens
 * starting at absolute position 0, each split into tiles of PKV_TILE_TOKENS
 * tokens.  Within a split, tiles are folded in ascending order with an online
 * softmax in fp32: scores and P.V on the tensor cores with fp32 accumulation
 * (each probability entering P.V as a bf16 part and a bf16 remainder, ~16
 * significant bits, into two accumulators kept over the split's tiles and
 * added in fp32 at its end), each tile's max and row sums of the fp32
 * probabilities on the CUDA cores in fixed reduction trees, and a running max
 * that rises only when a tile's max exceeds it by more than 2^8 (the
 * accumulators and the row sum are then rescaled in fp32).  Split
 * partials are merged in ascending split index (= global block index) order
 * in fp32, and out is rounded to bf16 once, at the final write.  Source:
 * RL-Kernel PR #284
 * "feat(attention): add CP backward drift validation", Changes ("fixed
 * global_block_index merge order, fp32 accumulation, final-write downcast"),
 * and the [WS1] "KV-cache path consistency (prefill & decode)" issue, Notes
 * ("share one reduction-order contract across prefill and decode").  None of
 * the constants depends on the batch, the SM count or the block size, so a
 * row's result is bitwise independent of batch composition, padding, cache
 * layout and of which entry point computed it.
 *
 * Conventions shared by all calls
 * -------------------------------
 * - All pointers except the stride arrays are DEVICE pointers on the current
 *   device.  Stride arrays are HOST arrays of element (not byte) strides.
 * - q, K, V, k_new, v_new and out are bf16 (IEEE bfloat16 bits); lse is fp32;
 *   block_table and seqlens are int32.
 * - The last axis (head_dim D) of every bf16 tensor has unit stride.  Every
 *   other stride of q, K, V, k_new and v_new must be a multiple of 8 elements
 *   (16 bytes) and their base pointers 16-byte aligned (128-bit loads, TMA).
 * - Cache views are [num_blocks, block_size, Hkv, D] with element strides
 *   (block, slot, head) given per component, so the non-contiguous K = kv[:,0]
 *   and V = kv[:,1] views of an interleaved [num_blocks, 2, block_size, Hkv, D]
 *   buffer work as is (block stride 2*block_size*Hkv*D).
 * - block_table row b lists the cache block of tokens
 *   [j*block_size, (j+1)*block_size) of sequence b at column j; the row stride
 *   is bt_stride elements and at most max_blocks_per_seq columns are read.
 * - seqlens[b] (device) is the context length of sequence b INCLUDING the
 *   query tokens: the caller appends the queries' K/V with pkv_kv_append
 *   first.  Query row i of seqlen_q sits at absolute position
 *   seqlens[b] - seqlen_q + i (bottom-right alignment); under causal it sees
 *   keys 0..position, otherwise keys 0..seqlens[b]-1.  A row that sees no key
 *   gets out = 0 and lse = -inf.
 * - GQA: query head h reads KV head h / (Hq / Hkv).
 * - The library allocates nothing, never synchronises the device and only
 *   enqueues work on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   The caller owns every buffer, including the workspace.
 * - err (optional, may be NULL) is a device int32 the kernels OR error bits
 *   into (PKV_DEVERR_*).  It is never read or cleared by the library, so the
 *   hot path never synchronises; the caller zeroes it and reads it when it
 *   wants to check.  Out-of-range table entries are skipped, never read.
 * - Every call returns PKV_OK or a PKV_ERR_* code and launches nothing when
 *   it returns an error.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Fixed constants of the reduction contract. */
#define PKV_SPLIT_TOKENS 4096
#define PKV_TILE_TOKENS 128

/* Return codes. */
#define PKV_OK 0
#define PKV_ERR_ARG 1        /* a size, stride, alignment or pointer is invalid */
#define PKV_ERR_WORKSPACE 2  /* workspace NULL or smaller than pkv_workspace_size() */
#define PKV_ERR_CUDA 3       /* a CUDA runtime call or kernel launch failed */
#define PKV_ERR_LAYOUT 4     /* the cache strides cannot be described to the TMA unit */

/* Device error bits OR-ed into *err by the kernels. */
#define PKV_DEVERR_BAD_BLOCK 1   /* block_table entry outside [0, num_blocks) */
#define PKV_DEVERR_TABLE_WIDTH 2 /* a position needs a column >= max_blocks_per_seq */
#define PKV_DEVERR_TIMEOUT 4     /* an internal pipeline wait gave up (no result) */
#define PKV_DEVERR_QUERY_LEN 8   /* packed call: a sequence has more than max_seqlen_q
                                    queries (or cu_seqlens_q decreases); rows past the
                                    bound are not written */
#define PKV_DEVERR_SEQ_LEN 16    /* a sequence's seqlens[b] exceeds max_seqlen_k: the
                                    split grid (or the backward's key tiles) was sized
                                    from max_seqlen_k, so keys past its last split (key
                                    tile) are not read and the result is not that
                                    context's attention */

/*
 * pkv_kv_append: for every sequence b and new token t < n_new, copy the bf16
 * bits of k_new[b, t, :, :] and v_new[b, t, :, :] (shape [batch, n_new, Hkv, D],
 * element strides kn_strides / vn_strides = (batch, token, head)) to cache
 * position p = seqlens[b] + t: block block_table[b][p / block_size], slot
 * p % block_size.  The bits are stored unchanged, so the reader sees exactly
 * what the writer produced ([WS1] KV-cache path consistency, Scope: stored-KV
 * dtype/layout must add no drift).  seqlens are NOT modified: the caller
 * advances them (put-then-advance, as jouleclaw's in-place KV cache does).
 * block_size: a power of two in [16, 256]; D: 64 or 128.
 */
int pkv_kv_append(const void *k_new, const int64_t kn_strides[3],
                  const void *v_new, const int64_t vn_strides[3],
                  void *k_cache, const int64_t k_strides[3],
                  void *v_cache, const int64_t v_strides[3],
                  int64_t num_blocks,
                  const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                  const int32_t *seqlens, int batch, int n_new, int Hkv, int D,
                  int block_size, int32_t *err, void *stream);

/*
 * pkv_paged_decode_attn: out[b, i, h, :] = softmax(scale * q K^T) V over the
 * keys visible to query row i (see Conventions), lse[b, h, i] = natural-log
 * log-sum-exp of scale * q.k over those keys.
 *
 *   q            [batch, seqlen_q, Hq, D] bf16, element strides q_strides = (b, s, h)
 *   k_cache/v_cache  cache views, element strides (block, slot, head)
 *   num_blocks   number of blocks in the cache (table entries are checked against it)
 *   seqlens      [batch] int32 device, context lengths incl. the query tokens
 *   max_seqlen_k host upper bound of seqlens (sizes the split grid); a sequence
 *                longer than it is an error of the caller: it sets
 *                PKV_DEVERR_SEQ_LEN in *err, and keys past the grid's last split
 *                (ceil(max_seqlen_k / PKV_SPLIT_TOKENS) splits) are not read
 *   scale        softmax scale applied to q.k (e.g. 1/sqrt(D))
 *   causal       0 or 1 (bottom-right aligned)
 *   out          [batch, seqlen_q, Hq, D] bf16, element strides out_strides = (b, s, h)
 *   lse          [batch, Hq, seqlen_q] fp32, contiguous
 *   workspace    >= pkv_workspace_size(batch, seqlen_q, Hq, D, max_seqlen_k) bytes,
 *                16-byte aligned, no initialisation needed
 * D: 64 or 128; Hq % Hkv == 0; block_size: power of two in [16, 256].
 * Split-K decode over the block table (aiter d293d61 commit message), honouring
 * the real k/v_cache.stride(0) instead of assuming block_size * slot_stride.
 */
int pkv_paged_decode_attn(const void *q, const int64_t q_strides[3],
                          const void *k_cache, const int64_t k_strides[3],
                          const void *v_cache, const int64_t v_strides[3],
                          int64_t num_blocks,
                          const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                          const int32_t *seqlens, int max_seqlen_k,
                          int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                          float scale, int causal,
                          void *out, const int64_t out_strides[3], float *lse,
                          void *workspace, size_t workspace_bytes,
                          int32_t *err, void *stream);

/*
 * pkv_paged_prefill_attn: same arguments and semantics as
 * pkv_paged_decode_attn, for many query rows per sequence (a causal prefill,
 * or one chunk of a chunked prefill: append the chunk's K/V, then call with
 * seqlen_q = chunk length and seqlens = tokens cached so far).  Every row is
 * reduced under the same contract as a decode row at the same position, so
 * decode row t equals prefill row t bit for bit ([WS1] KV-cache path
 * consistency, Acceptance criteria).
 */
int pkv_paged_prefill_attn(const void *q, const int64_t q_strides[3],
                           const void *k_cache, const int64_t k_strides[3],
                           const void *v_cache, const int64_t v_strides[3],
                           int64_t num_blocks,
                           const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                           const int32_t *seqlens, int max_seqlen_k,
                           int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                           float scale, int causal,
                           void *out, const int64_t out_strides[3], float *lse,
                           void *workspace, size_t workspace_bytes,
                           int32_t *err, void *stream);

/*
 * pkv_debug_paged_decode_attn: pkv_paged_decode_attn (same arguments, same
 * results) with every internal pipeline wait limited to wait_limit_ns instead
 * of the 2 s every other call uses.  It has no counterpart on the pages: it
 * exists to exercise the library's own failure handling (every pipeline wait
 * is bounded and a stuck pipeline ends the call with an error bit instead of a
 * hung GPU).  A wait that runs out makes the
 * kernel give up: each CTA waits (with the full 2 s limit) for its own copies
 * and tensor-core operations in flight, releases its tensor memory, sets
 * PKV_DEVERR_TIMEOUT in *err and returns; out / lse then hold no result, and
 * the device stays usable for the next call.  wait_limit_ns may be 0 (any wait
 * not satisfied at once gives up); more than 2e9 is PKV_ERR_ARG.
 */
int pkv_debug_paged_decode_attn(const void *q, const int64_t q_strides[3],
                                const void *k_cache, const int64_t k_strides[3],
                                const void *v_cache, const int64_t v_strides[3],
                                int64_t num_blocks,
                                const int32_t *block_table, int64_t bt_stride,
                                int max_blocks_per_seq, const int32_t *seqlens, int max_seqlen_k,
                                int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                                float scale, int causal,
                                void *out, const int64_t out_strides[3], float *lse,
                                void *workspace, size_t workspace_bytes,
                                int32_t *err, void *stream, uint64_t wait_limit_ns);

/*
 * pkv_debug_final_out: out[i] = the library's final division of a folded
 * row, A[i] / L[i] (0 where L[i] <= 0), computed on the device exactly as the
 * attention calls compute every out element (the row's reciprocal once, then
 * residual corrections; see the kernels).  It has no counterpart on the
 * pages: it exists so that a test can hold that arithmetic to the IEEE
 * quotient bit for bit.  A, L, out: device arrays of n floats (caller-owned;
 * out may not alias A or L).  Returns PKV_ERR_ARG for n < 0 or a null
 * pointer with n > 0, PKV_ERR_CUDA when the launch fails; n = 0 does nothing.
 */
int pkv_debug_final_out(const float *A, const float *L, float *out, int64_t n, void *stream);

/*
 * pkv_paged_decode_attn_append: kv_append fused into the attention call --
 * the "new_kv" form of flash_attn_with_kvcache in the aiter test grid.  The
 * n_new tokens of k_new/v_new ([batch, n_new, Hkv, D] bf16, element strides
 * kn_strides / vn_strides = (batch, token, head)) are written to cache
 * positions seqlens[b] - n_new + t (seqlens count them: the context length
 * AFTER the append, as in pkv_paged_decode_attn), and the attention then reads
 * them.  On return the cache holds exactly the bits pkv_kv_append would have
 * written (with seqlens - n_new), and out / lse are bitwise those of
 * pkv_kv_append followed by pkv_paged_decode_attn.  With at most 16 new
 * tokens and at most one tile of query rows per KV head (decode steps) the
 * attention kernel writes them itself, one launch fewer per step; otherwise
 * (prefill chunks) an append launch precedes the attention on the same
 * stream.  Requires 1 <= n_new <= PKV_SPLIT_TOKENS and n_new <= seqlens[b]
 * (positions below 0 are not written).  Other arguments as for
 * pkv_paged_decode_attn; the cache views must be writable.
 */
int pkv_paged_decode_attn_append(const void *q, const int64_t q_strides[3],
                                 const void *k_new, const int64_t kn_strides[3],
                                 const void *v_new, const int64_t vn_strides[3], int n_new,
                                 void *k_cache, const int64_t k_strides[3],
                                 void *v_cache, const int64_t v_strides[3],
                                 int64_t num_blocks,
                                 const int32_t *block_table, int64_t bt_stride,
                                 int max_blocks_per_seq,
                                 const int32_t *seqlens, int max_seqlen_k,
                                 int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                                 float scale, int causal,
                                 void *out, const int64_t out_strides[3], float *lse,
                                 void *workspace, size_t workspace_bytes,
                                 int32_t *err, void *stream);

/*
 * pkv_paged_varlen_attn: packed multi-request attention -- the "cumulative
 * query lengths" form of a packed forward (AstrAI commit search page: "Pack
 * prompts ... into one forward", "Select per-request final logits from
 * cumulative query lengths").  Request b owns the packed query tokens
 * cu_seqlens_q[b] .. cu_seqlens_q[b+1] - 1 (device int32 [batch + 1],
 * non-decreasing, cu_seqlens_q[0] = 0, cu_seqlens_q[batch] = total_q; empty
 * requests allowed); its n_b queries are the last n_b positions of its
 * context, exactly as seqlen_q = n_b in pkv_paged_decode_attn (bottom-right,
 * causal or not, seqlens[b] counts them).  Every row is bitwise the row the
 * dense call on that request alone returns.
 *   q        [total_q, Hq, D] bf16, element strides q_strides = (token, head)
 *   out      [total_q, Hq, D] bf16, strides out_strides = (token, head)
 *   lse      [Hq, total_q] fp32, contiguous
 *   max_seqlen_q  host bound on every n_b (sizes the grid; a larger n_b sets
 *                 PKV_DEVERR_QUERY_LEN and its rows past the bound stay unwritten)
 *   final_out / final_lse  optional (both null, or both given): each
 *                 request's last query row (token cu_seqlens_q[b+1] - 1) is also
 *                 written to final_out [batch, Hq, D] (strides final_strides =
 *                 (batch, head)) and final_lse [batch, Hq]; requests with no
 *                 query leave their final row untouched
 *   workspace     >= pkv_varlen_workspace_size(total_q, Hq, D, max_seqlen_k)
 * Other arguments and all error codes as for pkv_paged_decode_attn.
 */
int pkv_paged_varlen_attn(const void *q, const int64_t q_strides[2], const int32_t *cu_seqlens_q,
                          int total_q, int max_seqlen_q,
                          const void *k_cache, const int64_t k_strides[3],
                          const void *v_cache, const int64_t v_strides[3],
                          int64_t num_blocks,
                          const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                          const int32_t *seqlens, int max_seqlen_k,
                          int batch, int Hq, int Hkv, int D, int block_size,
                          float scale, int causal,
                          void *out, const int64_t out_strides[2], float *lse,
                          void *final_out, const int64_t final_strides[2], float *final_lse,
                          void *workspace, size_t workspace_bytes,
                          int32_t *err, void *stream);

/* Workspace bytes pkv_paged_varlen_attn needs (0 on invalid arguments). */
size_t pkv_varlen_workspace_size(int total_q, int Hq, int D, int max_seqlen_k);

/*
 * pkv_kv_append_varlen: pkv_kv_append for packed new tokens.  Sequence b's
 * new tokens are rows cu_seqlens_new[b] .. cu_seqlens_new[b+1] - 1 of k_new /
 * v_new ([total_new, Hkv, D] bf16, element strides (token, head)); token t of
 * sequence b goes to position seqlens[b] + t (seqlens BEFORE the append).
 * Bits, errors and device error bits as for pkv_kv_append.
 */
int pkv_kv_append_varlen(const void *k_new, const int64_t kn_strides[2],
                         const void *v_new, const int64_t vn_strides[2],
                         const int32_t *cu_seqlens_new, int total_new,
                         void *k_cache, const int64_t k_strides[3],
                         void *v_cache, const int64_t v_strides[3],
                         int64_t num_blocks,
                         const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                         const int32_t *seqlens, int batch, int Hkv, int D, int block_size,
                         int32_t *err, void *stream);

/*
 * Context parallelism (CP) over the KV context -- the CP forward of RL-Kernel
 * PR #284 "feat(attention): add CP backward drift validation" (Changes: CP
 * world size, KV chunk size, fixed global_block_index merge order, fp32
 * accumulation, final-write downcast).  Rank r of W owns the contiguous
 * splits [split_begin, split_begin + n_splits_local) of every sequence (its
 * slice of the context; its cache and block table need only hold those
 * tokens), computes their partials with pkv_paged_attn_partials, the ranks
 * all-gather the partial buffers (any transport; each rank's buffer is one
 * block of pkv_partials_size bytes), and every rank calls pkv_merge_partials
 * on the gathered blocks.  A split's partial does not depend on which rank or
 * call computed it and the merge folds splits in ascending global index, so
 * out / lse are bitwise those of one pkv_paged_decode_attn /
 * pkv_paged_prefill_attn call over the whole context.
 *
 * pkv_paged_attn_partials: arguments as pkv_paged_decode_attn (dense q,
 * seqlens = the FULL context lengths) without out / lse / max_seqlen_k; writes
 * into `partials` (>= pkv_partials_size(batch, seqlen_q, Hq, D,
 * n_splits_local) bytes, 16-byte aligned) the fp32 partials (m, l, acc[D]) of
 * every (row, local split): acc [rows][n_local][D] (256-byte padded), then
 * (m, l) [rows][n_local][2], rows = batch * seqlen_q * Hq in (b, i, h) order;
 * m is the split's max score in base-2 units (scale * log2(e) * q.k), l the
 * sum of 2^(s - m) and acc the sum of 2^(s - m) v over the split's visible
 * keys (s in the same units).  Partials of
 * (row, split) pairs the row does not reach are left unwritten (the merge
 * never reads them).  Errors as pkv_paged_decode_attn (PKV_ERR_WORKSPACE if
 * partials is too small).
 */
int pkv_paged_attn_partials(const void *q, const int64_t q_strides[3],
                            const void *k_cache, const int64_t k_strides[3],
                            const void *v_cache, const int64_t v_strides[3],
                            int64_t num_blocks,
                            const int32_t *block_table, int64_t bt_stride, int max_blocks_per_seq,
                            const int32_t *seqlens,
                            int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                            float scale, int causal,
                            int split_begin, int n_splits_local,
                            void *partials, size_t partials_bytes,
                            int32_t *err, void *stream);

/* Bytes of one rank's partial buffer (0 on invalid arguments). */
size_t pkv_partials_size(int batch, int seqlen_q, int Hq, int D, int n_splits_local);

/*
 * pkv_merge_partials: the ascending-split merge and final write over
 * `world` partial buffers laid side by side (block r, rank_bytes bytes from
 * block r - 1, holds global splits [r * n_splits_local, (r + 1) *
 * n_splits_local)).  rank_bytes >= pkv_partials_size(...) and a multiple of
 * 16; seqlens are the full context lengths; out [batch, seqlen_q, Hq, D]
 * bf16 (strides as pkv_paged_decode_attn), lse [batch, Hq, seqlen_q] fp32.
 */
int pkv_merge_partials(const void *partials, int world, int n_splits_local, size_t rank_bytes,
                       const int32_t *seqlens, int batch, int seqlen_q, int Hq, int D,
                       int causal, void *out, const int64_t out_strides[3], float *lse,
                       void *stream);

/*
 * pkv_paged_prefill_attn_bwd: deterministic backward of causal / chunked
 * prefill (or any seqlen_q) over the paged cache -- the training-side
 * backward over the same forward graph (RL-Kernel PR #284 "feat(attention):
 * add CP backward drift validation", Changes: backward reference, dq / dk /
 * dv, fixed order, fp32 accumulation; decode backward stays unsupported
 * there, and this call is the prefill form).  Inputs as pkv_paged_prefill_attn
 * plus the forward's out / lse and dout ([batch, seqlen_q, Hq, D] bf16,
 * strides dout_strides).  Outputs:
 *   dq        [batch, seqlen_q, Hq, D] bf16 (strides dq_strides)
 *   dk_cache / dv_cache  gradient buffers laid out like the caches (views
 *             [num_blocks, block_size, Hkv, D], strides dk/dv_strides): the
 *             row of every position < seqlens[b] of every sequence is
 *             written (a context position with no query row that sees it
 *             gets zeros); other rows are left untouched.
 * Every sum (over query rows for dk / dv, over keys for dq) runs in one
 * fixed ascending order on fp32 accumulators, P and dS enter the tensor
 * cores as bf16: the result is bitwise reproducible and independent of the
 * rest of the batch.  Two sequences must not share a cache block.
 *   workspace >= pkv_bwd_workspace_size(batch, seqlen_q, Hq) bytes.
 * Errors and device error bits as pkv_paged_prefill_attn (strides of out,
 * dq, dout, dk_cache, dv_cache: multiples of 8 elements, bases 16-byte
 * aligned).
 */
int pkv_paged_prefill_attn_bwd(const void *q, const int64_t q_strides[3],
                               const void *k_cache, const int64_t k_strides[3],
                               const void *v_cache, const int64_t v_strides[3],
                               int64_t num_blocks,
                               const int32_t *block_table, int64_t bt_stride,
                               int max_blocks_per_seq,
                               const int32_t *seqlens, int max_seqlen_k,
                               int batch, int seqlen_q, int Hq, int Hkv, int D, int block_size,
                               float scale, int causal,
                               const void *out, const int64_t out_strides[3], const float *lse,
                               const void *dout, const int64_t dout_strides[3],
                               void *dq, const int64_t dq_strides[3],
                               void *dk_cache, const int64_t dk_strides[3],
                               void *dv_cache, const int64_t dv_strides[3],
                               void *workspace, size_t workspace_bytes,
                               int32_t *err, void *stream);

/* Workspace bytes pkv_paged_prefill_attn_bwd needs (0 on invalid arguments). */
size_t pkv_bwd_workspace_size(int batch, int seqlen_q, int Hq);

/* Workspace bytes the attention calls need: fp32 split partials
 * (m, l, acc[D]) for every (batch, query row, query head, split). */
size_t pkv_workspace_size(int batch, int seqlen_q, int Hq, int D, int max_seqlen_k);

/* Static description of a return code (never NULL). */
const char *pkv_strerror(int code);

/* PKV_SPLIT_TOKENS, for bindings that cannot read the macro. */
int pkv_split_tokens(void);

/*
 * pkv_paged_decode_attn_static_ws: pkv_paged_decode_attn for callers that
 * cannot allocate device memory when they call, and have no buffer to lend as
 * workspace -- for example a host framework that owns the whole device-memory
 * budget and forbids cudaMalloc after start-up, or a latency-bound serving
 * loop that cannot afford cudaMalloc's implicit device synchronisation.  The
 * pages have no counterpart of this call; it exists only for such callers.
 *
 * Same arguments and results as pkv_paged_decode_attn, minus the workspace:
 * the split partials go to a scratch array of PKV_STATIC_WORKSPACE_BYTES that
 * the library keeps in device memory (a file-scope __device__ array, so every
 * GPU that loads the library holds it until the process exits).  The call
 * itself allocates nothing.
 *
 * - Limit: returns PKV_ERR_WORKSPACE, launching nothing, when
 *   pkv_workspace_size(batch, seqlen_q, Hq, D, max_seqlen_k) exceeds
 *   PKV_STATIC_WORKSPACE_BYTES.
 * - Set-up: the first call on each device (with that device current) looks up
 *   the array's device address once; make that first call before any stream
 *   capture begins.  A failed look-up returns PKV_ERR_CUDA.
 * - Sharing: every call on a device uses the same array and leaves its
 *   partials there.  Nothing in it needs to start at zero (each call writes
 *   every partial it reads), but two calls whose kernels overlap on the GPU --
 *   on different streams, or from different host threads -- race on it and
 *   give undefined results.  Serialise them (one stream) or use
 *   pkv_paged_decode_attn with a workspace per stream.
 */
#define PKV_STATIC_WORKSPACE_BYTES (8u << 20)

int pkv_paged_decode_attn_static_ws(const void *q, const int64_t q_strides[3],
                                    const void *k_cache, const int64_t k_strides[3],
                                    const void *v_cache, const int64_t v_strides[3],
                                    int64_t num_blocks,
                                    const int32_t *block_table, int64_t bt_stride,
                                    int max_blocks_per_seq,
                                    const int32_t *seqlens, int max_seqlen_k,
                                    int batch, int seqlen_q, int Hq, int Hkv, int D,
                                    int block_size, float scale, int causal,
                                    void *out, const int64_t out_strides[3], float *lse,
                                    int32_t *err, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
