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
 *     step 9: the new token lands at row 30,608 of the cache so viewed).
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
 * blocks, block tables", section 3 "The slot mapping": each new token's K/V
 * go to the slot slot_mapping[i] names; padding entries hold a sentinel.)
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
 *      token p is reached through table entry p / block_size, at offset
 *      p % block_size, and n tokens use ceil(n / block_size) entries);
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

/*
 * Attention for several query tokens per request over the paged cache
 * ("PagedAttention: fragmentation, blocks, block tables", the attention
 * metadata passage: query_start_loc is [num_reqs + 1], the start of each
 * request's rows in the query tensor; seq_lens is [num_reqs], the computed
 * tokens of each request; max_query_len is the longest query).
 *
 * Reading (the pages name the fields but do not spell the masking out): the
 * q_len = query_start_loc[r+1] - query_start_loc[r] query rows of request r
 * are its last q_len tokens, whose K/V are already in the cache and counted
 * in n = seq_lens[r].  Query row i (0-based within the request) is the token
 * at position n - q_len + i and attends to positions 0 .. n - q_len + i
 * (causal).  q_len = 1 is one decode step; q_len = n is a whole prefill.
 *
 * For each request r, query row i and query head j (KV head h = j / group):
 *   1. rebuild the contiguous K and V of (r, h) through the block table;
 *   2. z_t = scale * q[row][j] . K_t for t = 0 .. n - q_len + i;
 *   3. p_t = exp(z_t - max z) / sum exp(z - max z);
 *   4. out[row][j] = sum_t p_t V_t.
 * `out` is double [num_tokens][num_q_heads][head_dim] with num_tokens =
 * query_start_loc[num_reqs].  Returns 0; -1 for a block id out of range or a
 * table too narrow; -2 on OOM; -3 for q_len < 0 or q_len > n.
 */
int oracle_attention(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                     const int32_t *block_tables, int32_t max_blocks_per_seq,
                     const int32_t *query_start_loc, const int32_t *seq_lens, int32_t num_reqs,
                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                     int32_t block_size, int64_t num_blocks, double scale, double *out)
{
    const int32_t group = num_q_heads / num_kv_heads;
    int64_t max_n = 0;
    for (int32_t r = 0; r < num_reqs; ++r) {
        int64_t q_len = (int64_t)query_start_loc[r + 1] - query_start_loc[r];
        if (q_len < 0 || q_len > seq_lens[r])
            return -3;
        if (seq_lens[r] > max_n)
            max_n = seq_lens[r];
    }
    double *kk = (double *)malloc((size_t)(max_n + 1) * head_dim * sizeof(double));
    double *vv = (double *)malloc((size_t)(max_n + 1) * head_dim * sizeof(double));
    double *z = (double *)malloc((size_t)(max_n + 1) * sizeof(double));
    if (!kk || !vv || !z) {
        free(kk); free(vv); free(z);
        return -2;
    }
    int rc = 0;
    for (int32_t r = 0; r < num_reqs && rc == 0; ++r) {
        const int64_t n = seq_lens[r];
        const int64_t row0 = query_start_loc[r];
        const int64_t q_len = query_start_loc[r + 1] - row0;
        if (q_len == 0)
            continue;
        if ((n + block_size - 1) / block_size > max_blocks_per_seq) {
            rc = -1;
            break;
        }
        for (int32_t h = 0; h < num_kv_heads && rc == 0; ++h) {
            /* 1. contiguous K, V of (r, h) */
            for (int64_t t = 0; t < n; ++t) {
                int64_t blk = block_tables[(int64_t)r * max_blocks_per_seq + t / block_size];
                if (blk < 0 || blk >= num_blocks) {
                    rc = -1;
                    break;
                }
                int64_t slot_row = (blk * block_size + t % block_size) * num_kv_heads + h;
                for (int32_t d = 0; d < head_dim; ++d) {
                    kk[t * head_dim + d] = bf16_to_double(k_cache[slot_row * head_dim + d]);
                    vv[t * head_dim + d] = bf16_to_double(v_cache[slot_row * head_dim + d]);
                }
            }
            if (rc)
                break;
            for (int64_t i = 0; i < q_len; ++i) {
                const int64_t visible = n - q_len + i + 1; /* positions 0 .. n - q_len + i */
                for (int32_t j = h * group; j < (h + 1) * group; ++j) {
                    const uint16_t *qr = q + ((row0 + i) * num_q_heads + j) * head_dim;
                    double *o = out + ((row0 + i) * num_q_heads + j) * head_dim;
                    /* 2. scores */
                    double zmax = -INFINITY;
                    for (int64_t t = 0; t < visible; ++t) {
                        double acc = 0.0;
                        for (int32_t d = 0; d < head_dim; ++d)
                            acc += bf16_to_double(qr[d]) * kk[t * head_dim + d];
                        z[t] = scale * acc;
                        if (z[t] > zmax)
                            zmax = z[t];
                    }
                    /* 3. softmax weights and their sum */
                    double denom = 0.0;
                    for (int64_t t = 0; t < visible; ++t) {
                        z[t] = exp(z[t] - zmax);
                        denom += z[t];
                    }
                    /* 4. weighted sum of V */
                    for (int32_t d = 0; d < head_dim; ++d) {
                        double acc = 0.0;
                        for (int64_t t = 0; t < visible; ++t)
                            acc += z[t] * vv[t * head_dim + d];
                        o[d] = acc / denom;
                    }
                }
            }
        }
    }
    free(kk);
    free(vv);
    free(z);
    return rc;
}

/* ------------------------------------------------------------------------
 * FP8 (e4m3) KV cache.  The pages list an FP8 KV cache as a knob that halves
 * the bytes per token ("The pantry of pigeonholes", "The 10 knobs", knob 4
 * kv_cache_dtype; "How it connects to the rest of the stack", KV
 * quantisation).  The format is OCP FP8 E4M3: 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN, largest
 * finite 448 = 1.75 * 2^8, subnormals m/8 * 2^-6 (smallest 2^-9).
 * A stored code c of a tensor with scale s stands for value(c) * s.
 * ------------------------------------------------------------------------ */

/* value of an e4m3 code, exact in double */
double oracle_e4m3_to_double(uint8_t c)
{
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* x rounded to the nearest integer, ties to even (x has few significant
 * bits here, so x + 0.5 is exact) */
static double round_half_even(double x)
{
    double r = floor(x + 0.5);
    if (r - x == 0.5 && fmod(r, 2.0) != 0.0)
        r -= 1.0;
    return r;
}

/* e4m3 code of a float: round to nearest even, magnitudes at or above 448
 * (infinities included) saturate to 448, NaN gives 0x7F. */
uint8_t oracle_e4m3_from_float(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    const uint8_t sign = (uint8_t)((u >> 31) << 7);
    if (f != f)
        return 0x7F;
    const double a = fabs((double)f);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {               /* subnormal range: k * 2^-9 */
        const double k = round_half_even(a / ldexp(1.0, -9));
        return (uint8_t)(sign | (uint8_t)k); /* k == 8 encodes 2^-6 (exponent 1) */
    }
    int e = (int)floor(log2(a));
    if (ldexp(1.0, e) > a)                  /* guard log2 rounding */
        e -= 1;
    if (ldexp(1.0, e + 1) <= a)
        e += 1;
    double q = round_half_even((a / ldexp(1.0, e) - 1.0) * 8.0);
    if (q == 8.0) {
        q = 0.0;
        e += 1;
    }
    if (e + 7 > 15 || (e + 7 == 15 && q > 6.0))
        return (uint8_t)(sign | 0x7E);
    return (uint8_t)(sign | ((e + 7) << 3) | (uint8_t)q);
}

/*
 * FP8 write: each bf16 value x of token i's K (V) row is stored as the code
 * of x / k_scale (x / v_scale), the quotient taken in float (IEEE division,
 * round to nearest), at flat row slot_mapping[i] (negative = padding).
 */
int oracle_write_kv_fp8(const uint16_t *k, const uint16_t *v, const int64_t *slot_mapping,
                        int64_t num_tokens, int64_t row_elems, int64_t num_slots, float k_scale,
                        float v_scale, uint8_t *k_cache, uint8_t *v_cache)
{
    for (int64_t i = 0; i < num_tokens; ++i)
        if (slot_mapping[i] >= num_slots)
            return -1;
    for (int64_t i = 0; i < num_tokens; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        for (int64_t e = 0; e < row_elems; ++e) {
            const float kx = (float)bf16_to_double(k[i * row_elems + e]);
            const float vx = (float)bf16_to_double(v[i * row_elems + e]);
            k_cache[slot * row_elems + e] = oracle_e4m3_from_float(kx / k_scale);
            v_cache[slot * row_elems + e] = oracle_e4m3_from_float(vx / v_scale);
        }
    }
    return 0;
}

/*
 * FP8 decode: as oracle_decode, with K_t[d] = value(code) * k_scale and
 * V_t[d] = value(code) * v_scale (in double).
 */
int oracle_decode_fp8(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                      const int32_t *block_tables, int32_t max_blocks_per_seq,
                      const int32_t *seq_lens, int32_t num_seqs, int32_t num_q_heads,
                      int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                      int64_t num_blocks, double scale, double k_scale, double v_scale,
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
    int rc = 0;
    for (int32_t s = 0; s < num_seqs && rc == 0; ++s) {
        for (int32_t j = 0; j < num_q_heads && rc == 0; ++j) {
            const int32_t h = j / group;
            const int64_t n = seq_lens[s];
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
            for (int64_t t = 0; t < n; ++t) {
                const int64_t blk = block_tables[(int64_t)s * max_blocks_per_seq + t / block_size];
                if (blk < 0 || blk >= num_blocks) {
                    rc = -1;
                    break;
                }
                const int64_t row = (blk * block_size + t % block_size) * num_kv_heads + h;
                for (int32_t d = 0; d < head_dim; ++d) {
                    kk[t * head_dim + d] = oracle_e4m3_to_double(k_cache[row * head_dim + d]) * k_scale;
                    vv[t * head_dim + d] = oracle_e4m3_to_double(v_cache[row * head_dim + d]) * v_scale;
                }
            }
            if (rc)
                break;
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
            double denom = 0.0;
            for (int64_t t = 0; t < n; ++t) {
                z[t] = exp(z[t] - zmax);
                denom += z[t];
            }
            for (int32_t d = 0; d < head_dim; ++d) {
                double acc = 0.0;
                for (int64_t t = 0; t < n; ++t)
                    acc += z[t] * vv[t * head_dim + d];
                o[d] = acc / denom;
            }
        }
    }
    free(kk);
    free(vv);
    free(z);
    return rc;
}
