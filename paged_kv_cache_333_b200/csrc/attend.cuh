// Attention of several query tokens per request over the paged cache: the
// rows of a request are its last q_len tokens (query_start_loc gives each
// request's rows, seq_lens its computed tokens including those rows), and row
// i attends causally to positions 0 .. n - q_len + i ("PagedAttention:
// fragmentation, blocks, block tables", the attention-metadata passage:
// query_start_loc, seq_lens, max_query_len).  q_len = 1 is a decode step, a
// few rows are speculative tokens, hundreds a chunk of a prefill.
//
// Work decomposition.  A "column" is one (query row, query head of the KV
// group) pair of a request: column c = i * G + g.  One CTA handles one
// (split-K partition, KV head, request, chunk of 8W columns); each of its W
// consumer warps owns 8 consecutive columns, which are
// the N = 8 side of the same tensor-core tiles the decode kernel uses:
//   S^T(16 tokens x 8 columns) = K(16x128) Q^T, mma.m16n8k16 bf16;
//   O^T(128 x 8) += V^T(128x16) P^T, with P^T from movmatrix.trans.
// The chunk's columns form c = ceil(columns / 8) groups of 8 (c <= W).  With
// fewer groups than warps, the s = W / c' warps of a group (c' = c rounded up
// to a power of two, at most W) split its tiles round-robin, as the decode
// kernel's two consumer warps do, and their (max, sum, acc) are merged
// through shared memory at the end; with c' = W each warp owns one group and
// reads every tile.  Every tile of the CTA's token range is fetched from HBM once
// and read by one warp of each group, so the ring's "empty" barrier counts
// c' arrivals per phase (set once the request's row count is known).  Tile t
// is read by the warps with t % s == their split index and lives in stage
// t % kStagesA; kStagesA is a multiple of every s, so a stage is only ever
// read by the warps of one split index, each of which has read the stage's
// previous phase before it waits on the next.  The token range of a CTA ends
// at the last position its last row may see; a warp skips the math (still
// releasing the stage) for tiles past its own rows' range.
//
// Masking is per column: token t is seen by column c iff t <= n - q_len +
// c / G.  A column can see no token of a whole tile (or of a whole split-K
// partition); its running max then stays -inf and the online-softmax update
// uses 0 in place of the max so that no NaN arises (its weights are 0).
//
// Feeding.  For blocks of >= 8 tokens the producer warp loads each 16-token
// tile with TMA (the decode kernel's tensor maps and boxes).  For blocks of
// 1, 2 or 4 tokens the producer warp gathers the rows with 16-byte cp.async
// copies and each lane's copies complete on the stage's "full" barrier
// (cp.async.mbarrier.arrive.noinc; the barrier expects 32 arrivals).  In a
// partial tile the rows past the range hold data of other tokens (or
// anything); their scores are masked and their V^T fragments are zeroed in
// registers (0 * NaN would be NaN), without touching the shared stage that
// the other warps read.
//
// Split-K: with more than one partition each CTA writes (m, l, acc) per
// (row, query head, partition) like the decode kernel, and the partition-0
// CTAs of KV head 0 write each row's visible length n - q_len + i + 1, which
// the decode merge kernel then uses as that row's length.
#pragma once

#include "decode_mma.cuh"

namespace pa {

// Two shapes of CTA, chosen per call from the columns a request has
// (max_query_len * G): W = 2 consumer warps (16 columns, 96 threads, 4 CTAs
// per SM, as the decode kernel) for up to 16 columns, W = 4 (32 columns, 160
// threads, 2 CTAs per SM) above.  Four CTAs per SM keep a chat-sized batch
// (512 CTAs) in one wave: measured on B200 (64 requests of 512..612
// tokens, Llama-3-8B heads), 4 query rows per request took 32.6 us with
// W = 2 against 57 us with W = 4, while 8 rows took 57 us with W = 4 against
// 70 us with W = 2.  When each warp owns a whole group (no split) its
// columns are written from registers; a shared-memory round trip there cost
// 20-30% on B200.
template <int W>
struct AttendCfg;
template <>
struct AttendCfg<2> {
    static constexpr int kStages = 6, kCtasPerSm = 4;
};
template <>
struct AttendCfg<4> {
    static constexpr int kStages = 8, kCtasPerSm = 2;
};
template <int W>
constexpr int attend_threads() { return (W + 1) * 32; }
template <int W>
constexpr int attend_cols() { return 8 * W; }  // (row, head) columns per CTA

struct AttendParams {
    DecodeParams d;  // q / out rows are query rows; seq_lens, block_tables per request (num_seqs = requests)
    const int32_t *query_start_loc;  // [num_reqs + 1]
    int32_t *row_len;                // [num_tokens] visible length of each row (split-K only)
    int32_t num_tokens;
    int32_t max_query_len;
    int32_t chunks;                  // column chunks per request
    int32_t num_kv_heads;            // tcgen05 kernel: the KV heads (its grid is 1-D)
    int32_t head_groups;             // tcgen05 kernel: KV heads / heads per work unit
    int32_t num_units;               // tcgen05 kernel: partitions x head groups x requests x chunks
};

template <int W>
struct AttendSmem {
    static constexpr int kStages = AttendCfg<W>::kStages;
    static_assert(kStages % W == 0, "stages must be a multiple of every split");
    uint16_t kv[kStages][4][kHalfElems];  // [stage][K lo, K hi, V lo, V hi][16 x 64], 128B-swizzled rows
    uint64_t full[kStages];
    uint64_t empty[kStages];
    float wm[W][8];  // per warp and column: running max, sum (for the split merge)
    float wl[W][8];
    int32_t blocks[kMaxPartBlocksM];
};
template <int W>
constexpr size_t attend_smem_bytes() { return sizeof(AttendSmem<W>) + 1024; }

__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

template <int G, int W>
__global__ void __launch_bounds__(attend_threads<W>(), AttendCfg<W>::kCtasPerSm)
attend_partition_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const AttendParams ap) {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
    constexpr unsigned FULL = 0xffffffffu;
    constexpr int kAttendWarps = W;
    constexpr int kAttendCols = attend_cols<W>();
    constexpr int kStagesA = AttendCfg<W>::kStages;
    static_assert(sizeof(float) * W * 8 * kD <= sizeof(AttendSmem<W>::kv), "merge scratch must fit in the KV ring");
    const DecodeParams &p = ap.d;
    extern __shared__ uint8_t smem_raw[];
    AttendSmem<W> &sm = *reinterpret_cast<AttendSmem<W> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int part = blockIdx.x;
    const int h = blockIdx.y;
    const int r = blockIdx.z / ap.chunks;
    const int chunk = blockIdx.z % ap.chunks;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int B = p.block_size;
    const bool use_tma = B >= 8;

    if (use_tma && warp == kAttendWarps && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    grid_dependency_wait();

    // ---- the request's rows and this CTA's columns and token range ----------
    const int q0 = ap.query_start_loc[r];
    const int q1 = ap.query_start_loc[r + 1];
    const int n = clamp_seq_len(p, r);
    int q_len = q1 - q0;
    if (q_len < 0 || q_len > n || q_len > ap.max_query_len || q0 < 0 || q1 > ap.num_tokens ||
        (r == 0 && q0 != 0) || (r == p.num_seqs - 1 && q1 != ap.num_tokens)) {
        if (part == 0 && h == 0 && chunk == 0 && threadIdx.x == 0)
            flag_error(PA_DEVERR_QUERY_LOC);
        return;
    }
    const int cols = q_len * G;
    const int col0 = chunk * kAttendCols;
    if (col0 >= cols)
        return;
    const int last_col = min(cols, col0 + kAttendCols) - 1;
    const int first_visible = n - q_len;                      // row i sees positions <= first_visible + i
    const int lim_max = first_visible + last_col / G;         // >= 0: every row sees position 0
    const int t_begin = part * p.part_tokens;
    if (t_begin > lim_max)
        return;
    const int t_end = min(lim_max + 1, t_begin + p.part_tokens);
    const int num_tiles = (t_end - t_begin + kTile - 1) / kTile;
    const int Hkv = gridDim.y;
    // column groups (rounded up to a power of two) and the tile split
    const int groups_used = (last_col - col0) / 8 + 1;
    const int ngroups = groups_used == 1 ? 1 : groups_used == 2 ? 2 : kAttendWarps;
    const int split = kAttendWarps / ngroups;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStagesA; ++i) {
            mbar_init(&sm.full[i], use_tma ? 1 : 32);
            mbar_init(&sm.empty[i], ngroups);
        }
        mbar_init_fence();
    }

    if (p.num_parts > 1 && part == 0 && h == 0 && warp == 0) {
        for (int i = col0 / G + lane; i <= last_col / G; i += 32)
            ap.row_len[q0 + i] = first_visible + i + 1;
    }

    const int first_blk = t_begin / B;
    const int32_t *row = p.block_tables + static_cast<int64_t>(r) * p.max_blocks_per_seq + first_blk;
    if (warp == kAttendWarps) {
        const int nblk = (t_end - 1) / B - first_blk + 1;
        for (int i = lane; i < nblk; i += 32) {
            int32_t b = __ldg(row + i);
            if (b < 0 || b >= p.num_blocks) {
                flag_error(PA_DEVERR_BLOCK_ID);
                b = 0;
            }
            sm.blocks[i] = b;
        }
    }
    __syncthreads();

    // =================================================================== producer
    if (warp == kAttendWarps) {
        const uint64_t pol = l2_evict_first_policy();
        int issued = 0;
        for (int it = 0; it < num_tiles; ++it) {
            const int slot = it % kStagesA;
            if (it >= kStagesA) {
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait(&sm.empty[slot], ((it / kStagesA) + 1) & 1);
                if (!__shfl_sync(FULL, ok, 0))
                    break;
            }
            const int t0 = t_begin + it * kTile;
            const int ntok = min(kTile, t_end - t0);
            if (use_tma) {
                const int rows = B < kTile ? B : kTile;
                const int nb = B >= kTile ? 1 : (ntok + B - 1) / B;
                if (lane == 0)
                    mbar_arrive_expect_tx(&sm.full[slot], static_cast<uint32_t>(nb * rows * 128 * 4));
                __syncwarp();
                const int j = lane >> 2, q = lane & 3;  // box j of quarter q (K lo, K hi, V lo, V hi)
                if (j < nb) {
                    const int32_t blk = sm.blocks[(t0 + j * rows) / B - first_blk];
                    const int32_t rr = blk * B + ((t0 + j * rows) % B);
                    tma_load_3d(&sm.kv[slot][q][j * rows * 64], (q < 2) ? &tm_k : &tm_v, (q & 1) * 64, h, rr,
                                &sm.full[slot], pol);
                }
            } else {
                // lane = (tensor, 64-dim half, 16-byte chunk); token i's cache row
                // comes from lane i by shuffle
                const int tensor = lane >> 4, half = (lane >> 3) & 1, ch = lane & 7;
                const uint16_t *cache = static_cast<const uint16_t *>(tensor ? p.v_cache : p.k_cache);
                int64_t my_row = 0;
                if (lane < ntok) {
                    const int t = t0 + lane;
                    my_row = (static_cast<int64_t>(sm.blocks[t / B - first_blk]) * B + (t % B)) * Hkv + h;
                }
                const uint32_t base = smem_addr(&sm.kv[slot][tensor * 2 + half][0]);
                for (int i = 0; i < ntok; ++i) {
                    const int64_t rr = __shfl_sync(FULL, my_row, i);
                    cp_async16(base + swz(i, ch), cache + rr * kD + half * 64 + ch * 8);
                }
                cp_async_mbar_arrive_noinc(&sm.full[slot]);
            }
            issued = it + 1;
        }
        if (use_tma) {
            if (lane == 0) {
                for (int sl = 0; sl < kStagesA && sl < issued; ++sl) {
                    const int last = sl + ((issued - 1 - sl) / kStagesA) * kStagesA;
                    mbar_wait(&sm.full[sl], (last / kStagesA) & 1);
                }
            }
        } else {
            asm volatile("cp.async.wait_all;" ::: "memory");
        }
        return;
    }

    // =================================================================== consumers
    const int grp = warp % ngroups;            // this warp's column group
    const int sub = warp / ngroups;            // its split index: tiles t with t % split == sub
    const int wcol0 = col0 + 8 * grp;          // the group's first column
    const bool active = wcol0 <= last_col;
    // q as the B operand: column n = lane / 4 is row (wcol0 + n) / G, head
    // h*G + (wcol0 + n) % G; zero for columns past the chunk.
    const int qn = lane >> 2;
    const int qk = (lane & 3) * 2;
    uint32_t qb[8][2];
    {
        const int col = wcol0 + qn;
        const bool ok = active && col <= last_col;
        const int i = ok ? col / G : 0, g = ok ? col % G : 0;
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(p.q) +
                               ((static_cast<int64_t>(q0 + i) * p.num_q_heads + h * G + g) * kD) / 2;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qb[ks][0] = ok ? __ldg(qrow + (16 * ks + qk) / 2) : 0u;
            qb[ks][1] = ok ? __ldg(qrow + (16 * ks + 8 + qk) / 2) : 0u;
        }
    }
    // C-fragment columns of this lane: cA = wcol0 + 2(lane%4), cB = cA + 1
    const int cA = wcol0 + 2 * (lane & 3), cB = cA + 1;
    const int limA = (active && cA <= last_col) ? first_visible + cA / G : -1;
    const int limB = (active && cB <= last_col) ? first_visible + cB / G : -1;
    const int wlim = active ? first_visible + min(wcol0 + 7, last_col) / G : -1;
    const float sl2 = p.scale_log2;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
        acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    const int k_row = (lane & 7) + (((lane >> 3) & 1) << 3);
    const int k_chk = lane >> 4;
    const int v_row = (lane & 7) + ((lane >> 4) << 3);
    const int v_chk = (lane >> 3) & 1;
    const int tok0 = lane >> 2;  // C-fragment token rows tok0, tok0 + 8

    for (int it = sub; it < num_tiles; it += split) {
        const int slot = it % kStagesA;
        bool ok = true;
        if (lane == 0)
            ok = mbar_wait(&sm.full[slot], (it / kStagesA) & 1);
        if (!__shfl_sync(FULL, ok, 0))
            break;
        const int t0 = t_begin + it * kTile;
        const int ntok = min(kTile, t_end - t0);
        if (t0 > wlim) {  // no row of this warp sees this tile (or the warp has no rows)
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.empty[slot]);
            continue;
        }
        const uint32_t kb0 = smem_addr(&sm.kv[slot][0][0]);
        const uint32_t kb1 = smem_addr(&sm.kv[slot][1][0]);
        const uint32_t vb0 = smem_addr(&sm.kv[slot][2][0]);
        const uint32_t vb1 = smem_addr(&sm.kv[slot][3][0]);
        uint32_t ka[8][4], va[8][4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            ldmatrix_x4(ka[ks], ((ks < 4) ? kb0 : kb1) + swz(k_row, (ks & 3) * 2 + k_chk));
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int c = 2 * mt + v_chk;
            ldmatrix_x4_trans(va[mt], ((c < 8) ? vb0 : vb1) + swz(v_row, c & 7));
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sm.empty[slot]);
        if (ntok < kTile) {
            // V^T fragment registers 0,1 hold tokens 2(lane%4) + {0,1}; 2,3 the same + 8
            const int ta = 2 * (lane & 3);
            const uint32_t m01 = (ta < ntok ? 0x0000ffffu : 0u) | (ta + 1 < ntok ? 0xffff0000u : 0u);
            const uint32_t m23 = (ta + 8 < ntok ? 0x0000ffffu : 0u) | (ta + 9 < ntok ? 0xffff0000u : 0u);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                va[mt][0] &= m01;
                va[mt][1] &= m01;
                va[mt][2] &= m23;
                va[mt][3] &= m23;
            }
        }

        // ---- S^T = K Q^T ------------------------------------------------
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_16816(sc, ka[ks], qb[ks][0], qb[ks][1]);
        // ---- masks: past the range, or after the column's row ----------
        const int pos0 = t0 + tok0, pos1 = pos0 + 8;
        const bool in0 = tok0 < ntok, in1 = tok0 + 8 < ntok;
        const float x0 = (in0 && pos0 <= limA) ? sc[0] * sl2 : -INFINITY;
        const float x1 = (in0 && pos0 <= limB) ? sc[1] * sl2 : -INFINITY;
        const float x2 = (in1 && pos1 <= limA) ? sc[2] * sl2 : -INFINITY;
        const float x3 = (in1 && pos1 <= limB) ? sc[3] * sl2 : -INFINITY;
        float tA = fmaxf(x0, x2), tB = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1) {
            tA = fmaxf(tA, __shfl_xor_sync(FULL, tA, off));
            tB = fmaxf(tB, __shfl_xor_sync(FULL, tB, off));
        }
        const float nA = fmaxf(mA, tA), nB = fmaxf(mB, tB);
        const float sA = nA == -INFINITY ? 0.f : nA;  // a column that has seen nothing yet
        const float sB = nB == -INFINITY ? 0.f : nB;
        const float aA = exp2_approx(mA - sA), aB = exp2_approx(mB - sB);
        mA = nA;
        mB = nB;
        const float p0 = exp2_approx(x0 - sA), p1 = exp2_approx(x1 - sB);
        const float p2 = exp2_approx(x2 - sA), p3 = exp2_approx(x3 - sB);
        lA = fmaf(lA, aA, p0 + p2);
        lB = fmaf(lB, aB, p1 + p3);
        const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));  // tokens 0..7
        const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));  // tokens 8..15
        // ---- O^T = alpha O^T + V^T P^T ----------------------------------
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            acc[mt][0] *= aA;
            acc[mt][1] *= aB;
            acc[mt][2] *= aA;
            acc[mt][3] *= aB;
            mma_16816(acc[mt], va[mt], pb0, pb1);
        }
    }
    if (threadIdx.x == 0)
        grid_launch_dependents();
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) {
        lA += __shfl_xor_sync(FULL, lA, off);
        lB += __shfl_xor_sync(FULL, lB, off);
    }
    // ---- one warp per group: its lane's two columns go straight out ---------
    // (dims 16mt + tok0 in acc 0/1 and 16mt + tok0 + 8 in acc 2/3)
    if (split == 1) {
        if (!active)
            return;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int col = u ? cB : cA;
            if ((u ? limB : limA) < 0)
                continue;
            const float M = u ? mB : mA, L = u ? lB : lA;
            const int64_t qrow = q0 + col / G;
            const int j = h * G + col % G;
            if (p.num_parts == 1) {
                __nv_bfloat16 *o = p.out + (qrow * p.num_q_heads + j) * kD;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    o[16 * mt + tok0] = __float2bfloat16_rn(L > 0.f ? acc[mt][u] / L : 0.f);
                    o[16 * mt + tok0 + 8] = __float2bfloat16_rn(L > 0.f ? acc[mt][2 + u] / L : 0.f);
                }
            } else {
                const int64_t idx = (qrow * p.num_q_heads + j) * p.num_parts + part;
                float *o = p.part_acc + idx * kD;
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    o[16 * mt + tok0] = acc[mt][u];
                    o[16 * mt + tok0 + 8] = acc[mt][2 + u];
                }
                if (tok0 == 0)
                    p.part_ml[idx] = make_float2(M, L);
            }
        }
        return;
    }
    // ---- several warps per group: merge them through shared memory ---------
    // Every tile has been waited for by some consumer warp before this
    // barrier, so no copy into the ring is still in flight.
    asm volatile("bar.sync 1, %0;" ::"n"(kAttendWarps * 32) : "memory");
    float *wacc = reinterpret_cast<float *>(&sm.kv[0][0][0]);  // [warp][8 columns][D]
    {
        const int ca = 2 * (lane & 3);
        float *wa = wacc + (warp * 8 + ca) * kD;
        float *wb = wa + kD;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d = mt * 16 + tok0;
            wa[d] = acc[mt][0];
            wb[d] = acc[mt][1];
            wa[d + 8] = acc[mt][2];
            wb[d + 8] = acc[mt][3];
        }
        if (lane < 4) {
            sm.wm[warp][ca] = mA;
            sm.wm[warp][ca + 1] = mB;
            sm.wl[warp][ca] = lA;
            sm.wl[warp][ca + 1] = lB;
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kAttendWarps * 32) : "memory");
    // the W*32 consumer threads finish every column, thread t dims t, t + 32W, ...
    for (int gi = 0; gi < ngroups; ++gi) {
        for (int c = 0; c < 8; ++c) {
            const int col = col0 + 8 * gi + c;
            if (col > last_col)
                break;
            float M = -INFINITY;
            for (int si = 0; si < split; ++si)
                M = fmaxf(M, sm.wm[si * ngroups + gi][c]);
            float L = 0.f;
            for (int si = 0; si < split && M != -INFINITY; ++si) {
                const float mw = sm.wm[si * ngroups + gi][c];
                if (mw != -INFINITY)
                    L = fmaf(sm.wl[si * ngroups + gi][c], exp2f(mw - M), L);
            }
            const int64_t qrow = q0 + col / G;
            const int j = h * G + col % G;
            const int64_t idx = (qrow * p.num_q_heads + j) * p.num_parts + part;
            for (int d = threadIdx.x; d < kD; d += kAttendWarps * 32) {
                float o = 0.f;
                for (int si = 0; si < split && M != -INFINITY; ++si) {
                    const int w = si * ngroups + gi;
                    const float mw = sm.wm[w][c];
                    if (mw != -INFINITY)
                        o = fmaf(wacc[(w * 8 + c) * kD + d], exp2f(mw - M), o);
                }
                if (p.num_parts == 1)
                    p.out[(qrow * p.num_q_heads + j) * kD + d] = __float2bfloat16_rn(L > 0.f ? o / L : 0.f);
                else
                    p.part_acc[idx * kD + d] = o;
            }
            if (p.num_parts > 1 && threadIdx.x == 0)
                p.part_ml[idx] = make_float2(M, L);
        }
    }
}

}  // namespace pa
