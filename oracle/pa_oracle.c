/*
 * Paged-KV oracle: a plain, slow, obviously correct CPU implementation of the
 * three device operations of the paged decode path, in double precision.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header or constant with the CUDA library; the two meet only through the
 * seeded inputs both are given.
 *
 * Storage conventions (the plainest reading of the pages, stated once):
 *   - bf16 values travel as their 16-bit patterns (uint16_t).
 *   - A KV cache is block-major: [num_blocks][block_size][num_kv_heads][head_dim],
 *     one tensor for K and one for V.  Block i owns the contiguous range
 *     [i*page, (i+1)*page) ("PagedAttention: fragmentation, blocks, block
 *     tables", section 3 "The slot mapping"), and a flat row index
 *     block*block_size + offset is a "slot": row `slot` of the cache viewed as
 *     [num_blocks*block_size][num_kv_heads*head_dim] (same page, walkthrough
 *     step 9: the new token is stored "at flat row 30,608").
 *   - Query head j reads KV head j / (num_q_heads/num_kv_heads) (contiguous
 *     grouped-query heads; the pages are silent, this is the standard reading).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double, exact: the bf16 pattern is the top half of a float32. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Write: token i's K row (num_kv_heads*head_dim values) is stored at flat
 * row slot_mapping[i] of k_cache, and its V row at the same row of v_cache.
 * A negative slot is padding and is skipped.  ("PagedAttention: fragmentation,
 * blocks, block tables", section 3 "The slot mapping": the kernel writes new
 * K/V at slot_mapping[i]; padded positions carry PAD_ID.)
 * Returns 0, or -1 if a slot is >= num_slots (nothing is written then).
 */
int oracle_write_kv(const uint16_t *k, const uint16_t *v, const int64_t *slot_mapping,
                    int64_t num_tokens, int64_t row_elems, int64_t num_slots,
                    uint16_t *k_cache, uint16_t *v_cache)
{
    for (int64_t i = 0; i < num_tokens; ++i)
        if (slot_mapping[i] >= num_slots)
            return -1;
    for (int64_t i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        for (int64_t e = 0; e < row_elems; ++e) {
            k_cache[slot * row_elems + e] = k[i * row_elems + e];
            v_cache[slot * row_elems + e] = v[i * row_elems + e];
        }
    }
    return 0;
}

/*
 * Copy-on-write block copy: for every (src, dst) pair, the whole block dst of
 * K and of V becomes a copy of block src, all block_elems values of it,
 * including slots no token has written.  All sources are read before any
 * destination is written, which is what one fancy-index assignment
 * blocks[dst] = blocks[src] does ("PagedAttention: fragmentation, blocks,
 * block tables", copy-on-write for partial prefix hits).
 * Returns 0, or -1 if an id is outside [0, num_blocks) (nothing is written).
 */
int oracle_copy_blocks(const int64_t *pairs, int64_t num_pairs, int64_t block_elems,
                       int64_t num_blocks, uint16_t *k_cache, uint16_t *v_cache)
{
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t s = pairs[2 * p], d = pairs[2 * p + 1];
        if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks)
            return -1;
    }
    if (num_pairs == 0)
        return 0;
    uint16_t *tmp = (uint16_t *)malloc((size_t)(2 * num_pairs * block_elems) * sizeof(uint16_t));
    if (!tmp)
        return -2;
    /* gather */
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t s = pairs[2 * p];
        for (int64_t e = 0; e < block_elems; ++e) {
            tmp[(2 * p) * block_elems + e] = k_cache[s * block_elems + e];
            tmp[(2 * p + 1) * block_elems + e] = v_cache[s * block_elems + e];
        }
    }
    /* scatter */
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t d = pairs[2 * p + 1];
        for (int64_t e = 0; e < block_elems; ++e) {
            k_cache[d * block_elems + e] = tmp[(2 * p) * block_elems + e];
            v_cache[d * block_elems + e] = tmp[(2 * p + 1) * block_elems + e];
        }
    }
    free(tmp);
    return 0;
}

/*
 * Decode attention over a paged cache, for the (sequence, query head) pairs
 * selected by `which` (num_which pairs of int32 (s, j); NULL = all pairs).
 *
 * For sequence s with n = seq_lens[s] tokens and query head j, with
 * h = j / (num_q_heads / num_kv_heads):
 *   1. rebuild the contiguous K and V of (s, h): token t lives in physical
 *      block block_tables[s][t / B] at offset t % B ("PagedAttention:
 *      fragmentation, blocks, block tables", section 2 "The block table":
 *      position p lives in block table[p // block_size] at offset
 *      p % block_size; the kernel walks ceil(seq_len / block_size) entries);
 *   2. z_t = scale * sum_d q[s][j][d] * K_t[d]            (all in double);
 *   3. p_t = exp(z_t - max z) / sum_u exp(z_u - max z);
 *   4. out[s][j][d] = sum_t p_t * V_t[d].
 * n == 0 gives a zero output row (the pages are silent; the plainest reading).
 * `out` is double [num_seqs][num_q_heads][head_dim]; rows not selected are
 * left untouched.  Returns 0, -1 for a block id outside [0, num_blocks) or a
 * length needing more than max_blocks_per_seq table entries, -2 on OOM.
 */
int oracle_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                  const int32_t *seq_lens, int32_t num_seqs, int32_t num_q_heads,
                  int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                  int64_t num_blocks, double scale, const int32_t *which, int64_t num_which,
                  double *out)
{
    const int32_t group = num_q_heads / num_kv_heads;
    int64_t max_n = 0;
    for (int32_t s = 0; s < num_seqs; ++s)
        if (seq_lens[s] > max_n)
            max_n = seq_lens[s];
    double *kk = (double *)malloc((size_t)(max_n + 1) * head_dim * sizeof(double));
    double *vv = (double *)malloc((size_t)(max_n + 1) * head_dim * sizeof(double));
    double *z = (double *)malloc((size_t)(max_n + 1) * sizeof(double));
    if (!kk || !vv || !z) {
        free(kk); free(vv); free(z);
        return -2;
    }
    int64_t total = which ? num_which : (int64_t)num_seqs * num_q_heads;
    int rc = 0;
    for (int64_t w = 0; w < total && rc == 0; ++w) {
        int32_t s = which ? which[2 * w] : (int32_t)(w / num_q_heads);
        int32_t j = which ? which[2 * w + 1] : (int32_t)(w % num_q_heads);
        int32_t h = j / group;
        int64_t n = seq_lens[s];
        double *o = out + ((int64_t)s * num_q_heads + j) * head_dim;
        if (n == 0) {
            for (int32_t d = 0; d < head_dim; ++d)
                o[d] = 0.0;
            continue;
        }
        if ((n + block_size - 1) / block_size > max_blocks_per_seq) {
            rc = -1;
            break;
        }
        /* 1. rebuild contiguous K, V from the block table */
        for (int64_t t = 0; t < n; ++t) {
            int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + t / block_size];
            if (blk < 0 || blk >= num_blocks) {
                rc = -1;
                break;
            }
            int64_t row = (blk * block_size + t % block_size) * num_kv_heads + h;
            for (int32_t d = 0; d < head_dim; ++d) {
                kk[t * head_dim + d] = bf16_to_double(k_cache[row * head_dim + d]);
                vv[t * head_dim + d] = bf16_to_double(v_cache[row * head_dim + d]);
            }
        }
        if (rc)
            break;
        /* 2. scores */
        const uint16_t *qr = q + ((int64_t)s * num_q_heads + j) * head_dim;
        double zmax = -INFINITY;
        for (int64_t t = 0; t < n; ++t) {
            double acc = 0.0;
            for (int32_t d = 0; d < head_dim; ++d)
                acc += bf16_to_double(qr[d]) * kk[t * head_dim + d];
            z[t] = scale * acc;
            if (z[t] > zmax)
                zmax = z[t];
        }
        /* 3. softmax weights (unnormalised) and their sum */
        double denom = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            z[t] = exp(z[t] - zmax);
            denom += z[t];
        }
        /* 4. weighted sum of V */
        for (int32_t d = 0; d < head_dim; ++d) {
            double acc = 0.0;
            for (int64_t t = 0; t < n; ++t)
                acc += z[t] * vv[t * head_dim + d];
            o[d] = acc / denom;
        }
    }
    free(kk);
    free(vv);
    free(z);
    return rc;
}
