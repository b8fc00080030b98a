// Paged decode attention for sm_100a: a split-K partition kernel and a
// log-sum-exp merge kernel.
//
// What is computed ("PagedAttention: fragmentation, blocks, block tables",
// attention-metadata passage and section 2 "The block table"; "The pantry of
// pigeonholes", "The mechanism: blocks, block table and the kernel gather"):
// for sequence s, query head j and KV head h = j / G, walk the first
// ceil(n / B) entries of block-table row s; token t is row t % B of block
// table[s][t / B]; out = softmax(scale * q K^T) V over the n tokens.
//
// Design (one CTA per (partition, KV head, sequence)):
//   * warp 4 is the producer.  It copies the partition's slice of the block
//     table into shared memory once, then streams 16-token K and V tiles of
//     the sequence's KV head into a kStages-deep shared-memory ring with 3-D
//     TMA loads (box = 128 dims x 1 head x min(B,16) tokens), one full/empty
//     mbarrier pair per stage.  For B < 16 a tile takes 16/B loads, one per
//     block, issued by separate lanes.
//   * warps 0-3 are consumers; warp w takes tiles w, w+4, ...  Each K/V tile
//     is loaded once and used by all G query heads of the KV head.  A lane
//     owns 8 of the 128 dims (its "chunk" c = lane % 16) for 8 of the tile's
//     16 tokens (half = lane / 16).  QK: each lane forms 8-dim partial dot
//     products for its 8 tokens x G heads, then a 4-step butterfly
//     reduce-scatter across the 16 lanes of its half leaves every lane with
//     complete scores for one token and G/2 heads.  The partial sums are
//     stored in a lane-dependent order (token index XOR lane bits, head index
//     XOR lane bit 0) so that every butterfly step is one shuffle and one add,
//     with no selects.  Online softmax runs in the log2 domain (q is
//     pre-scaled by scale*log2(e)); maxima are combined with warp shuffles.
//     PV: probabilities go through a 512-byte per-warp scratch, and each lane
//     accumulates G x 8 outputs (its dims) over its 8 tokens.
//   * at the end the four warps' (max, sum, acc) are merged through shared
//     memory.  With one partition the CTA writes bf16 `out`; otherwise it
//     writes its unnormalised partial (m, l, acc) and the merge kernel
//     combines the partitions: M = max m_p, out = sum e^(m_p-M) acc_p /
//     sum e^(m_p-M) l_p.
// Unused storage (slots past n in the tail block, free blocks, table entries
// past ceil(n/B)) is never read into a result: scores of slots past n are set
// to -inf and their V rows are skipped, not multiplied by zero.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kD = 128;            // head_dim
constexpr int kTile = 16;          // tokens per pipeline stage
constexpr int kStages = 8;         // pipeline depth (8 x 8 KiB of K+V)
constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxPartBlocks = 1024;  // block-table entries one CTA may cover
constexpr int kDecodeCtasPerSm = 3;
// A stage is always consumed by the same warp (tile t: stage t % kStages,
// warp t % 4), so no parity wait can run a full phase ahead.
static_assert(kStages % kConsumerWarps == 0, "stages must be a multiple of the consumer warps");

struct DecodeParams {
    const uint4 *q;  // [S][Hq][D] bf16, 8 values per uint4
    const void *k_cache;  // [NB][B][H_kv][D] bf16 (read directly by the cp.async path)
    const void *v_cache;
    const int32_t *block_tables;
    const int32_t *seq_lens;
    __nv_bfloat16 *out;  // [S][Hq][D]
    float2 *part_ml;     // [S][Hq][P] (m, l), log2 domain
    float *part_acc;     // [S][Hq][P][D]
    int64_t num_blocks;
    int32_t max_blocks_per_seq;
    int32_t num_seqs;
    int32_t max_seq_len;
    int32_t num_q_heads;
    int32_t block_size;
    int32_t part_tokens;
    int32_t num_parts;
    float scale_log2;
    float k_scale;  // FP8 caches: value = code * k_scale (1 otherwise)
    float v_scale;  // FP8 caches: value = code * v_scale (1 otherwise)
};

struct DecodeSmem {
    uint16_t k[kStages][kTile][kD];
    uint16_t v[kStages][kTile][kD];
    float p[kConsumerWarps][kTile][8];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    float wm[kConsumerWarps][8];
    float wl[kConsumerWarps][8];
    int32_t blocks[kMaxPartBlocks];
};
// The final cross-warp merge reuses the K ring for the warps' accumulators.
static_assert(sizeof(float) * kConsumerWarps * 8 * kD <= sizeof(uint16_t) * kStages * kTile * kD,
              "merge scratch must fit in the K ring");

constexpr size_t kDecodeSmemBytes = sizeof(DecodeSmem) + 1024;  // + alignment slack

__device__ __forceinline__ int clamp_seq_len(const DecodeParams &p, int s) {
    int n = p.seq_lens[s];
    const int64_t cap64 = static_cast<int64_t>(p.max_blocks_per_seq) * p.block_size;
    const int cap = static_cast<int>(cap64 < p.max_seq_len ? cap64 : p.max_seq_len);
    if (n < 0 || n > cap) {
        flag_error(PA_DEVERR_SEQ_LEN);
        n = n < 0 ? 0 : cap;
    }
    return n;
}

// One 16-token tile for one consumer warp.  MASKED handles a final tile with
// fewer than 16 valid tokens.
template <int G, bool MASKED>
__device__ __forceinline__ void consume_tile(const DecodeSmem &sm, float *prow_base, int slot,
                                             int ntok, int half, int c, int c0, int mt,
                                             const float (&qf)[G][8], float (&m_run)[G],
                                             float (&l_part)[(G >= 2 ? G / 2 : 1)],
                                             float (&acc)[G][8]) {
    constexpr int GH = G >= 2 ? G / 2 : 1;
    constexpr unsigned FULL = 0xffffffffu;

    // ---- QK: partial dot products over this lane's 8 dims ----------------
    float sc[8 * G];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int tok = half * 8 + (i ^ mt);
        const uint4 u = *reinterpret_cast<const uint4 *>(&sm.k[slot][tok][c * 8]);
        float kf[8];
        unpack8(u, kf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float a = qf[g][0] * kf[0];
#pragma unroll
            for (int e = 1; e < 8; ++e)
                a = fmaf(qf[g][e], kf[e], a);
            sc[i * G + g] = a;
        }
    }
    // ---- butterfly reduce-scatter over the 16 lanes of this half ----------
#pragma unroll
    for (int j = 0; j < 4 * G; ++j)
        sc[j] += __shfl_xor_sync(FULL, sc[4 * G + j], 8);
#pragma unroll
    for (int j = 0; j < 2 * G; ++j)
        sc[j] += __shfl_xor_sync(FULL, sc[2 * G + j], 4);
#pragma unroll
    for (int j = 0; j < G; ++j)
        sc[j] += __shfl_xor_sync(FULL, sc[G + j], 2);
    if constexpr (G >= 2) {
#pragma unroll
        for (int j = 0; j < GH; ++j)
            sc[j] += __shfl_xor_sync(FULL, sc[GH + j], 1);
    } else {
        sc[0] += __shfl_xor_sync(FULL, sc[0], 1);
    }
    // Lane now holds scores of token (half*8 + mt) for heads c0*GH + j.

    // ---- online softmax ---------------------------------------------------
    const int tok_l = half * 8 + mt;
    const bool valid = !MASKED || tok_l < ntok;
    float tmax[GH];
#pragma unroll
    for (int j = 0; j < GH; ++j) {
        sc[j] = valid ? sc[j] : -INFINITY;
        tmax[j] = sc[j];
    }
#pragma unroll
    for (int off = 2; off <= 16; off <<= 1)
#pragma unroll
        for (int j = 0; j < GH; ++j)
            tmax[j] = fmaxf(tmax[j], __shfl_xor_sync(FULL, tmax[j], off));
    float mx[G];
    if constexpr (G >= 2) {
        float other[GH];
#pragma unroll
        for (int j = 0; j < GH; ++j)
            other[j] = __shfl_xor_sync(FULL, tmax[j], 1);
#pragma unroll
        for (int g = 0; g < G; ++g)
            mx[g] = ((g / GH) == c0) ? tmax[g % GH] : other[g % GH];
    } else {
        mx[0] = tmax[0];
    }
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float mn = fmaxf(m_run[g], mx[g]);
        alpha[g] = exp2f(m_run[g] - mn);
        m_run[g] = mn;
    }
    float pv[GH];
#pragma unroll
    for (int j = 0; j < GH; ++j) {
        const float m_g = (G >= 2 && c0) ? m_run[(GH + j) % G] : m_run[j];
        const float a_g = (G >= 2 && c0) ? alpha[(GH + j) % G] : alpha[j];
        pv[j] = exp2f(sc[j] - m_g);  // 0 for masked slots
        l_part[j] = fmaf(l_part[j], a_g, pv[j]);
    }
    float *prow = prow_base + tok_l * 8;
    if constexpr (G >= 2) {
#pragma unroll
        for (int j = 0; j < GH; ++j)
            prow[c0 * GH + j] = pv[j];
    } else {
        if (c0 == 0)
            prow[0] = pv[0];
    }
    __syncwarp();

    // ---- PV ---------------------------------------------------------------
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            acc[g][e] *= alpha[g];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int tok = half * 8 + i;
        if (MASKED && tok >= ntok)
            break;
        float pw[G];
        const float *pr = prow_base + tok * 8;
        if constexpr (G >= 4) {
#pragma unroll
            for (int g4 = 0; g4 < G; g4 += 4) {
                const float4 t = *reinterpret_cast<const float4 *>(pr + g4);
                pw[g4] = t.x; pw[g4 + 1] = t.y; pw[g4 + 2] = t.z; pw[g4 + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int g = 0; g < G; ++g)
                pw[g] = pr[g];
        }
        const uint4 u = *reinterpret_cast<const uint4 *>(&sm.v[slot][tok][c * 8]);
        float vf[8];
        unpack8(u, vf);
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 8; ++e)
                acc[g][e] = fmaf(pw[g], vf[e], acc[g][e]);
    }
}

template <int G>
__global__ void __launch_bounds__(kDecodeThreads, (G >= 8 ? 2 : kDecodeCtasPerSm))
decode_partition_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
    constexpr int GH = G >= 2 ? G / 2 : 1;
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ uint8_t smem_raw[];
    DecodeSmem &sm = *reinterpret_cast<DecodeSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int part = blockIdx.x;
    const int h = blockIdx.y;
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    grid_dependency_wait();  // the preceding kernel's writes are visible after this
    const int n = clamp_seq_len(p, s);
    const int t_begin = part * p.part_tokens;
    if (part > 0 && t_begin >= n)
        return;  // past the end of this sequence: the merge ignores it
    const int t_end = min(n, t_begin + p.part_tokens);
    const int num_tiles = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        mbar_init_fence();
    }
    __syncthreads();

    // =================================================================== producer
    if (warp == kConsumerWarps) {
        if (num_tiles == 0)
            return;
        const int B = p.block_size;
        const int first_blk = t_begin / B;
        const int nblk = (t_end - 1) / B - first_blk + 1;
        const int32_t *row = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq + first_blk;
        for (int i = lane; i < nblk; i += 32) {
            int32_t b = __ldg(row + i);
            if (b < 0 || b >= p.num_blocks) {
                flag_error(PA_DEVERR_BLOCK_ID);
                b = 0;
            }
            sm.blocks[i] = b;
        }
        __syncwarp();
        if (lane == 0) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
        }
        const uint64_t pol = l2_evict_first_policy();
        int issued = 0;
        for (int it = 0; it < num_tiles; ++it) {
            const int slot = it % kStages;
            if (it >= kStages) {
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait(&sm.empty[slot], ((it / kStages) + 1) & 1);
                if (!__shfl_sync(FULL, ok, 0))
                    break;
            }
            const int t0 = t_begin + it * kTile;
            const int ntok = min(kTile, t_end - t0);
            if (B >= kTile) {
                if (lane == 0) {
                    const int32_t blk = sm.blocks[t0 / B - first_blk];
                    const int32_t r = blk * B + (t0 % B);
                    mbar_arrive_expect_tx(&sm.full[slot], 2u * kTile * kD * 2u);
                    tma_load_3d(&sm.k[slot][0][0], &tm_k, 0, h, r, &sm.full[slot], pol);
                    tma_load_3d(&sm.v[slot][0][0], &tm_v, 0, h, r, &sm.full[slot], pol);
                }
            } else {
                const int nb = (ntok + B - 1) / B;
                if (lane == 0)
                    mbar_arrive_expect_tx(&sm.full[slot], 2u * nb * B * kD * 2u);
                __syncwarp();
                const int j = lane & 15;
                if (j < nb) {
                    const int32_t blk = sm.blocks[t0 / B - first_blk + j];
                    if (lane < 16)
                        tma_load_3d(&sm.k[slot][j * B][0], &tm_k, 0, h, blk * B, &sm.full[slot], pol);
                    else
                        tma_load_3d(&sm.v[slot][j * B][0], &tm_v, 0, h, blk * B, &sm.full[slot], pol);
                }
            }
            issued = it + 1;
        }
        // Drain: do not leave the CTA while a load still targets its smem.
        if (lane == 0) {
            for (int slot = 0; slot < kStages && slot < issued; ++slot) {
                const int last = slot + ((issued - 1 - slot) / kStages) * kStages;
                mbar_wait(&sm.full[slot], (last / kStages) & 1);
            }
        }
        return;
    }

    // =================================================================== consumers
    const int half = lane >> 4;
    const int c = lane & 15;
    const int c0 = c & 1;
    const int mt = c >> 1;
    const int mg = (G >= 2) ? c0 * GH : 0;

    float qf[G][8];
    {
        const uint4 *qrow = p.q + (static_cast<int64_t>(s) * p.num_q_heads + h * G) * (kD / 8);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const uint4 u = __ldg(qrow + (g ^ mg) * (kD / 8) + c);
            float t[8];
            unpack8(u, t);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                qf[g][e] = t[e] * p.scale_log2;
        }
    }
    float m_run[G], l_part[GH], acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m_run[g] = -INFINITY;
#pragma unroll
        for (int e = 0; e < 8; ++e)
            acc[g][e] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < GH; ++j)
        l_part[j] = 0.f;

    float *prow_base = &sm.p[warp][0][0];
    for (int it = warp; it < num_tiles; it += kConsumerWarps) {
        const int slot = it % kStages;
        bool ok = true;
        if (lane == 0)
            ok = mbar_wait(&sm.full[slot], (it / kStages) & 1);
        if (!__shfl_sync(FULL, ok, 0))
            break;
        const int ntok = min(kTile, t_end - (t_begin + it * kTile));
        if (ntok == kTile)
            consume_tile<G, false>(sm, prow_base, slot, ntok, half, c, c0, mt, qf, m_run, l_part, acc);
        else
            consume_tile<G, true>(sm, prow_base, slot, ntok, half, c, c0, mt, qf, m_run, l_part, acc);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.empty[slot]);
    }

    // ---- warp totals --------------------------------------------------------
#pragma unroll
    for (int off = 2; off <= 16; off <<= 1)
#pragma unroll
        for (int j = 0; j < GH; ++j)
            l_part[j] += __shfl_xor_sync(FULL, l_part[j], off);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            acc[g][e] += __shfl_xor_sync(FULL, acc[g][e], 16);

    // The merge kernel (if any) may start launching: this CTA's reads of K/V
    // are done and only its epilogue is left.
    if (threadIdx.x == 0)
        grid_launch_dependents();

    // ---- cross-warp merge through shared memory ----------------------------
    // All consumer warps must be done with the K ring before it is reused.
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    float *wacc = reinterpret_cast<float *>(&sm.k[0][0][0]);  // [warp][G][D]
    if (half == 0) {
        float *dst = wacc + (warp * G) * kD + c * 8;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            reinterpret_cast<float4 *>(dst + g * kD)[0] =
                make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
            reinterpret_cast<float4 *>(dst + g * kD)[1] =
                make_float4(acc[g][4], acc[g][5], acc[g][6], acc[g][7]);
        }
    }
    if (lane < 2) {
        if constexpr (G >= 2) {
#pragma unroll
            for (int j = 0; j < GH; ++j)
                sm.wl[warp][lane * GH + j] = l_part[j];
        } else {
            if (lane == 0)
                sm.wl[warp][0] = l_part[0];
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
            sm.wm[warp][g] = m_run[g];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");

    const int d = threadIdx.x;  // 0..127
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w)
            M = fmaxf(M, sm.wm[w][g]);
        float L = 0.f, o = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float mw = sm.wm[w][g];
                if (mw == -INFINITY)
                    continue;
                const float sc = exp2f(mw - M);
                L = fmaf(sm.wl[w][g], sc, L);
                o = fmaf(wacc[(w * G + g) * kD + d], sc, o);
            }
        }
        const int j = h * G + g;
        if (p.num_parts == 1) {
            const float r = L > 0.f ? o / L : 0.f;
            p.out[(static_cast<int64_t>(s) * p.num_q_heads + j) * kD + d] = __float2bfloat16_rn(r);
        } else {
            const int64_t idx = (static_cast<int64_t>(s) * p.num_q_heads + j) * p.num_parts + part;
            p.part_acc[idx * kD + d] = o;
            if (d == 0)
                p.part_ml[idx] = make_float2(M, L);
        }
    }
}

// One CTA per (query head, group of rows); thread d owns output dim d.  The
// grid's y extent may be smaller than the row count (at most 65535), so each
// CTA strides over rows.  A row's partition count follows from its length
// (seq_lens[s]; for pa_attention the per-row visible length).
__global__ void __launch_bounds__(kD) decode_merge_kernel(const DecodeParams p) {
    grid_dependency_wait();  // partials of the partition kernel are visible after this
    grid_launch_dependents();
    const int j = blockIdx.x;
    const int d = threadIdx.x;
    for (int s = blockIdx.y; s < p.num_seqs; s += gridDim.y) {
        const int n = clamp_seq_len(p, s);
        const int parts = n > 0 ? (n + p.part_tokens - 1) / p.part_tokens : 0;
        const int64_t base = (static_cast<int64_t>(s) * p.num_q_heads + j) * p.num_parts;
        float M = -INFINITY;
        for (int i = 0; i < parts; ++i)
            M = fmaxf(M, p.part_ml[base + i].x);
        float L = 0.f, o = 0.f;
        if (M != -INFINITY) {
            for (int i = 0; i < parts; ++i) {
                const float2 ml = p.part_ml[base + i];
                if (ml.x == -INFINITY)
                    continue;
                const float w = exp2f(ml.x - M);
                L = fmaf(ml.y, w, L);
                o = fmaf(p.part_acc[(base + i) * kD + d], w, o);
            }
        }
        const float r = L > 0.f ? o / L : 0.f;
        p.out[(static_cast<int64_t>(s) * p.num_q_heads + j) * kD + d] = __float2bfloat16_rn(r);
    }
}

}  // namespace pa
