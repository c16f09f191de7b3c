/*
 * pkv_oracle.c -- CPU fp64 oracle for paged-KV attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load this library.  The product path
 * (the CUDA library under paged_kv_decode_31_b200/) never calls it and shares
 * no code with it.
 *
 * What it computes, and where each step comes from:
 *
 *   1. Dense gather from the paged buffer.  Token j of sequence b lives in
 *      block block_table[b][j / block_size], slot j % block_size, addressed
 *      with the cache's REAL element strides (block, slot, head), so the
 *      K/V-interleaved [num_blocks, 2, block_size, Hkv, D] views work like
 *      contiguous ones.  Source: ROCm/aiter commit d293d61 "test(triton/decode):
 *      pin non-contiguous paged KV block stride", helper
 *      _generate_interleaved_block_kvcache (gather k_cache_paged[block_table]
 *      and rearrange to (b, nblocks*block_size)) and the commit message
 *      ("honor the real k/v_cache.stride(0)").
 *   2. GQA: query head h reads KV head h / (Hq/Hkv).  Source: same test,
 *      repeat(k_cache, "b s h d -> b s (h g) d") -- the (h g) grouping puts
 *      the G query heads of one KV head next to each other.
 *   3. Padding mask: key j is visible only if j < cache_seqlens[b].  Source:
 *      same test, key_padding_mask = arange(seqlen_k) < cache_seqlens.
 *   4. Causal mask, bottom-right aligned: query row i of seqlen_q sits at
 *      absolute position pos_i = seqlens[b] - seqlen_q + i and sees keys
 *      j <= pos_i.  The pages never print attention_ref's alignment; this is
 *      the only reading under which "one query against N cached KV reduces
 *      like the equivalent prefill" ([WS1] KV-cache path consistency, Scope)
 *      can hold for the last prefill row.
 *   5. Softmax attention in fp64: s_j = scale * q.k_j, m = max s_j,
 *      l = sum exp(s_j - m), out = sum exp(s_j - m) v_j / l, and the
 *      attention-domain log-sum-exp lse = m + ln l (natural log of the sum of
 *      exp(scale*q.k)), the "attention-domain lse" named in RL-Kernel PR #284
 *      "feat(attention): add CP backward drift validation", Changes.
 *   6. A row with no visible key (causal with seqlen_q > seqlens[b]) returns
 *      out = 0 and lse = -inf.  The pages are silent; this is the reading
 *      taken.
 *
 * kv_append writes token t of sequence b at position p = seqlens[b] + t, in
 * block block_table[b][p / block_size], slot p % block_size, copying the bf16
 * bits unchanged (the [WS1] issue's Scope: stored-KV dtype/layout must add no
 * drift between writer and reader).  The caller advances seqlens afterwards,
 * like the in-place cache's put + advance in jouleclaw's kv_cache_inplace.rs.
 *
 * Numbers: bf16 inputs are widened exactly to fp64; all arithmetic is fp64.
 * Parallelism: OpenMP over query rows (sequence, query head, query token);
 * each row reads its keys and values through the table itself, so results do
 * not depend on the thread count, and one sequence can use every host core.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_BLOCK 2
#define ORACLE_ERR_NOMEM 3

/* bf16 -> fp64, exact: a bf16 is the top half of an IEEE binary32. */
static double bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Step 1, the dense gather, one token at a time: the row of token j of one
 * sequence at KV head kvh in a cache view with element strides st = (block,
 * slot, head).  Token j lives in block table_row[j / block_size], slot
 * j % block_size.  Returns NULL when the table has no column for j (column
 * >= max_blocks_per_seq) or names a block outside [0, num_blocks). */
static const uint16_t *token_row(const uint16_t *cache, const int64_t st[3],
                                 const int32_t *table_row, int max_blocks_per_seq,
                                 int64_t num_blocks, int block_size, int kvh, int j)
{
    const int col = j / block_size;
    if (col >= max_blocks_per_seq)
        return NULL;
    const int32_t blk = table_row[col];
    if (blk < 0 || (int64_t)blk >= num_blocks)
        return NULL;
    return cache + (int64_t)blk * st[0] + (int64_t)(j % block_size) * st[1]
                 + (int64_t)kvh * st[2];
}

/*
 * oracle_paged_attn: steps 1-6 above for sequences b in [b_begin, b_end) and
 * KV heads in [kvh_begin, kvh_end) (all query heads of those KV heads).
 *
 *   q        bf16 bits, element strides q_st = (batch, token, head), d-stride 1
 *   k_cache  bf16 bits, element strides k_st = (block, slot, head), d-stride 1
 *   v_cache  same with v_st
 *   block_table int32 [batch][bt_stride]; only the first max_blocks_per_seq
 *            columns of a row describe that sequence's blocks
 *   seqlens  int32 [batch] (context length including the query tokens)
 *   out      fp64 [batch][seqlen_q][Hq][D] (only the selected rows written)
 *   lse      fp64 [batch][Hq][seqlen_q]
 *
 * Returns ORACLE_ERR_BLOCK, with nothing written, if a selected sequence has
 * a token whose table column is at or past max_blocks_per_seq or whose block
 * lies outside [0, num_blocks): the table does not describe that context.
 * Each query row (b, h, i) is an independent task; the work is spread over
 * the threads by row, and a row's arithmetic does not depend on the thread
 * count.
 */
int oracle_paged_attn(const uint16_t *q, const int64_t q_st[3],
                      const uint16_t *k_cache, const int64_t k_st[3],
                      const uint16_t *v_cache, const int64_t v_st[3],
                      int64_t num_blocks, const int32_t *block_table,
                      int64_t bt_stride, int max_blocks_per_seq,
                      const int32_t *seqlens,
                      int batch, int seqlen_q, int Hq, int Hkv, int D,
                      int block_size, double scale, int causal,
                      int b_begin, int b_end, int kvh_begin, int kvh_end,
                      double *out, double *lse)
{
    if (batch <= 0 || seqlen_q <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 ||
        block_size <= 0 || max_blocks_per_seq <= 0 || bt_stride < max_blocks_per_seq ||
        Hq % Hkv != 0 || b_begin < 0 || b_end > batch ||
        kvh_begin < 0 || kvh_end > Hkv)
        return ORACLE_ERR_ARG;
    const int G = Hq / Hkv;
    const int nb = b_end - b_begin, nh = kvh_end - kvh_begin;

    /* step 1's bounds: every token of every selected sequence has a block */
    for (int b = b_begin; b < b_end; ++b) {
        const int n = seqlens[b] > 0 ? seqlens[b] : 0;
        const int32_t *row = block_table + (int64_t)b * bt_stride;
        for (int j = 0; j < n; j += block_size)
            if (!token_row(k_cache, k_st, row, max_blocks_per_seq, num_blocks,
                           block_size, 0, j))
                return ORACLE_ERR_BLOCK;
    }

    const int64_t ntask = (int64_t)nb * nh * G * seqlen_q;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t task = 0; task < ntask; ++task) {
        const int i = (int)(task % seqlen_q);
        const int g = (int)((task / seqlen_q) % G);
        const int kvh = kvh_begin + (int)((task / ((int64_t)seqlen_q * G)) % nh);
        const int b = b_begin + (int)(task / ((int64_t)seqlen_q * G * nh));
        const int h = kvh * G + g;                             /* step 2 */
        const int n = seqlens[b] > 0 ? seqlens[b] : 0;
        const int32_t *row = block_table + (int64_t)b * bt_stride;
        double *o = out + (((int64_t)b * seqlen_q + i) * Hq + h) * D;
        double *ls = lse + ((int64_t)b * Hq + h) * seqlen_q + i;
        const int pos = n - seqlen_q + i;                      /* step 4 */
        int nvis = n;                                          /* step 3 */
        if (causal && pos + 1 < nvis)
            nvis = pos + 1;
        if (nvis <= 0) {                                       /* step 6 */
            for (int d = 0; d < D; ++d)
                o[d] = 0.0;
            *ls = -INFINITY;
            continue;
        }
        double *s = (double *)malloc(sizeof(double) * (size_t)nvis);
        if (!s) {
#pragma omp critical
            status = ORACLE_ERR_NOMEM;
            continue;
        }
        const uint16_t *qr = q + (int64_t)b * q_st[0] + (int64_t)i * q_st[1]
                               + (int64_t)h * q_st[2];
        double m = -INFINITY;                                  /* step 5 */
        for (int j = 0; j < nvis; ++j) {
            const uint16_t *kr = token_row(k_cache, k_st, row, max_blocks_per_seq,
                                           num_blocks, block_size, kvh, j);
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += bf16_to_f64(qr[d]) * bf16_to_f64(kr[d]);
            s[j] = scale * acc;
            if (s[j] > m)
                m = s[j];
        }
        double l = 0.0;
        for (int d = 0; d < D; ++d)
            o[d] = 0.0;
        for (int j = 0; j < nvis; ++j) {
            const uint16_t *vr = token_row(v_cache, v_st, row, max_blocks_per_seq,
                                           num_blocks, block_size, kvh, j);
            const double p = exp(s[j] - m);
            l += p;
            for (int d = 0; d < D; ++d)
                o[d] += p * bf16_to_f64(vr[d]);
        }
        for (int d = 0; d < D; ++d)
            o[d] /= l;
        *ls = m + log(l);
        free(s);
    }
    return status;
}

/*
 * oracle_kv_append: host-side reference of kv_append.  Copies the bf16 bits
 * of k_new/v_new [batch][n_new][Hkv][D] (element strides kn_st / vn_st =
 * (batch, token, head)) into the caches at positions seqlens[b] + t.
 * Returns ORACLE_ERR_BLOCK if a position falls outside the table row or the
 * table names a block outside [0, num_blocks).
 */
int oracle_kv_append(const uint16_t *k_new, const int64_t kn_st[3],
                     const uint16_t *v_new, const int64_t vn_st[3],
                     uint16_t *k_cache, const int64_t k_st[3],
                     uint16_t *v_cache, const int64_t v_st[3],
                     int64_t num_blocks, const int32_t *block_table,
                     int64_t bt_stride, int max_blocks_per_seq,
                     const int32_t *seqlens, int batch, int n_new, int Hkv,
                     int D, int block_size)
{
    if (batch <= 0 || n_new < 0 || Hkv <= 0 || D <= 0 || block_size <= 0)
        return ORACLE_ERR_ARG;
    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < n_new; ++t) {
            const int64_t p = (int64_t)seqlens[b] + t;
            if (p < 0 || p / block_size >= max_blocks_per_seq)
                return ORACLE_ERR_BLOCK;
            const int32_t blk = block_table[(int64_t)b * bt_stride + p / block_size];
            if (blk < 0 || (int64_t)blk >= num_blocks)
                return ORACLE_ERR_BLOCK;
            const int64_t slot = p % block_size;
            for (int h = 0; h < Hkv; ++h) {
                const uint16_t *ks = k_new + b * kn_st[0] + t * kn_st[1] + h * kn_st[2];
                const uint16_t *vs = v_new + b * vn_st[0] + t * vn_st[1] + h * vn_st[2];
                uint16_t *kd = k_cache + blk * k_st[0] + slot * k_st[1] + h * k_st[2];
                uint16_t *vd = v_cache + blk * v_st[0] + slot * v_st[1] + h * v_st[2];
                memcpy(kd, ks, sizeof(uint16_t) * (size_t)D);
                memcpy(vd, vs, sizeof(uint16_t) * (size_t)D);
            }
        }
    }
    return ORACLE_OK;
}

/* Cap the number of OpenMP threads the oracle runs on (n <= 0: no change). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Number of OpenMP threads the oracle runs on (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
