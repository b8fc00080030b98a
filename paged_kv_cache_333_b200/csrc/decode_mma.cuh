// Paged decode attention, tensor-core variant (the default pa_decode path).
//
// Same contract and same CTA decomposition as decode.cuh (one CTA per
// (partition, KV head, sequence); a producer warp streams 16-token K/V tiles
// into a shared-memory ring; consumer warps take tiles round-robin; the
// partition's (max, sum, acc) go to `out` or to the split-K workspace).  What
// changes is the consumer: with G query heads sharing a KV head, one tile's
// QK^T is a 16 (tokens) x 8 (heads, G real) x 128 contraction and its PV a
// 128 x 8 x 16 one, small but dense, so each runs as eight
// mma.m16n8k16 (bf16 in, fp32 accumulate) instead of ~500 FMAs and a
// 30-shuffle reduce-scatter per lane.  Measured on B200 the CUDA-core
// consumer spent most of its time issuing those shuffles and FMAs; this one
// issues about 100 instructions per tile and leaves the kernel bound by HBM.
//
// Tile layout in shared memory: each 16-token tile holds K and V as two
// 64-dim halves each ([half][token][64] bf16, 2 KiB per half, 1 KiB aligned)
// in the 128-byte swizzle (16-byte chunk c of row r stored at chunk
// c ^ (r % 8)), which makes every ldmatrix below conflict-free.  For block
// sizes >= 8 the producer fills a tile with 3-D TMA loads whose box is
// (64 dims x 1 head x min(B,16) tokens) using the tensor map's 128B swizzle;
// for block sizes 1, 2 and 4 (boxes would land at offsets that are not
// multiples of the swizzle atom) each consumer warp gathers its own tiles'
// rows with 16-byte cp.async copies at the same swizzled positions, three
// tiles ahead of the one it computes on.
//
// Per tile and consumer warp:
//   S^T(16x8) = K(16x128) Q^T(128x8): A = K via ldmatrix.x4, B = q (kept in
//     registers for the whole kernel, rows >= G zero).  Lane holds scores of
//     tokens lane/4 and lane/4+8 for heads 2(lane%4), 2(lane%4)+1.
//   online softmax in the log2 domain (scores * scale*log2 e), per-head max
//     over the 16 tokens with 3 shuffles; p rounded to bf16 for the PV MMA,
//     the running sum l kept in fp32.
//   movmatrix.trans turns the two 8x8 bf16 blocks of P^T into the B operand
//     of the PV MMA without touching shared memory.
//   O^T(128x8) += V^T(128x16) P^T(16x8): A = V^T via ldmatrix.x4.trans.
// A consumer warp reads the whole tile into registers (K and V^T fragments)
// and releases the stage before any arithmetic; the CTA has two consumer
// warps and a six-stage ring, so each warp always has loads in flight for
// its next two tiles while it computes (up to 4 CTAs, ~190 KiB of loads in
// flight, per SM).
// Unused storage never reaches a result: scores of slots past the sequence
// end are set to -inf and, in a partial tile, the V rows of those slots are
// zeroed in shared memory before the MMA (0 * NaN would be NaN).
#pragma once

#include "decode.cuh"

namespace pa {

constexpr int kConsumerWarpsM = 2;
constexpr int kDecodeThreadsM = (kConsumerWarpsM + 1) * 32;
constexpr int kStagesM = 6;
constexpr int kMmaCtasPerSm = 4;
constexpr int kMaxPartBlocksM = 512;    // block-table entries one CTA may cover
constexpr int kHalfElems = kTile * 64;  // one 64-dim half of a 16-token tile
// Tile t lives in stage t % kStagesM and is consumed by warp t % kConsumerWarpsM.
// With a stage count that is a multiple of the consumer-warp count, a stage
// is only ever consumed by one warp, which has itself consumed the stage's
// previous phase before it waits on the next one; a parity wait can then
// never be a full phase early (a parity test cannot tell phase k+2 from k).
// Each consumer warp owns kStagesM / kConsumerWarpsM stages, so loads keep
// streaming into its other stages while it computes on one.
static_assert(kStagesM % kConsumerWarpsM == 0, "stages must be a multiple of the consumer warps");

// Multi-wave grids of ragged work (the host decides: more CTAs than 4 per SM
// and at most 16 partitions per sequence) run a variant with three consumer
// warps, so that each short CTA finishes sooner; it keeps within 128
// registers per thread (4 CTAs per SM) by loading the V^T fragments of a tile
// in two halves.  Other grids keep two consumer warps.
constexpr int kMaxConsumerWarpsM = 3;
static_assert(kStagesM % 3 == 0, "stages must be a multiple of every consumer-warp count");
template <int CW>
constexpr int mma_threads() { return (CW + 1) * 32; }

struct DecodeSmemM {
    uint16_t kv[kStagesM][4][kHalfElems];  // [stage][K lo, K hi, V lo, V hi][16 x 64]
    uint64_t full[kStagesM];
    uint64_t empty[kStagesM];
    float wm[kMaxConsumerWarpsM][8];
    float wl[kMaxConsumerWarpsM][8];
    int32_t blocks[kMaxPartBlocksM];
};
static_assert(sizeof(float) * kMaxConsumerWarpsM * 8 * kD <= sizeof(uint16_t) * kStagesM * 4 * kHalfElems,
              "merge scratch must fit in the KV ring");
constexpr size_t kDecodeSmemBytesM = sizeof(DecodeSmemM) + 1024;

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` in a swizzled
// [rows][64] bf16 half-tile.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int G, int CW>
__global__ void __launch_bounds__(mma_threads<CW>(), kMmaCtasPerSm)
decode_partition_mma_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
    static_assert(CW == 2 || CW == 3, "consumer warps");
    constexpr int kCW = CW;
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ uint8_t smem_raw[];
    DecodeSmemM &sm = *reinterpret_cast<DecodeSmemM *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int part = blockIdx.x;
    const int h = blockIdx.y;
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int B = p.block_size;
    const bool use_tma = B >= 8;

    // Set-up that touches no global memory runs before the wait on the
    // preceding kernel of the stream (programmatic dependent launch).
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStagesM; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        mbar_init_fence();
    }
    if (use_tma && warp == kCW && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    grid_dependency_wait();

    // The producer reads the first 32 table entries of its slice while every
    // thread reads the sequence length (two loads in flight, not one after
    // the other).  Entries past the row's end are never read.
    const int t_begin = part * p.part_tokens;
    const int first_blk = t_begin / B;
    const int32_t *row = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq + first_blk;
    int32_t first_ids = 0;
    if (warp == kCW && lane < p.max_blocks_per_seq - first_blk)
        first_ids = __ldg(row + lane);
    const int n = clamp_seq_len(p, s);
    if (part > 0 && t_begin >= n)
        return;
    const int t_end = min(n, t_begin + p.part_tokens);
    const int num_tiles = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
    const int Hkv = gridDim.y;
    // The producer warp copies the partition's slice of the block table into
    // shared memory (read once, bounds-checked) before the CTA barrier.
    if (warp == kCW && num_tiles > 0) {
        const int nblk = (t_end - 1) / B - first_blk + 1;
        for (int i = lane; i < nblk; i += 32) {
            int32_t b = i < 32 ? first_ids : __ldg(row + i);
            if (b < 0 || b >= p.num_blocks) {
                flag_error(PA_DEVERR_BLOCK_ID);
                b = 0;
            }
            sm.blocks[i] = b;
        }
    }
    __syncthreads();

    // =================================================================== producer
    if (warp == kCW) {
        if (num_tiles == 0 || !use_tma)
            return;  // with blocks < 8 tokens each consumer warp gathers its own tiles
        const uint64_t pol = l2_evict_first_policy();
        int issued = 0;
        for (int it = 0; it < num_tiles; ++it) {
            const int slot = it % kStagesM;
            if (it >= kStagesM) {
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait(&sm.empty[slot], ((it / kStagesM) + 1) & 1);
                if (!__shfl_sync(FULL, ok, 0))
                    break;
            }
            const int t0 = t_begin + it * kTile;
            const int ntok = min(kTile, t_end - t0);
            uint16_t(*dst)[kHalfElems] = sm.kv[slot];
            {
                const int rows = B < kTile ? B : kTile;
                const int nb = B >= kTile ? 1 : (ntok + B - 1) / B;
                if (lane == 0)
                    mbar_arrive_expect_tx(&sm.full[slot], static_cast<uint32_t>(nb * rows * 128 * 4));
                __syncwarp();
                // lane = (box j, part q): q 0..3 = K lo, K hi, V lo, V hi
                const int j = lane >> 2, q = lane & 3;
                if (j < nb) {
                    const int32_t blk = sm.blocks[(t0 + j * rows) / B - first_blk];
                    const int32_t r = blk * B + ((t0 + j * rows) % B);
                    tma_load_3d(&dst[q][j * rows * 64], (q < 2) ? &tm_k : &tm_v, (q & 1) * 64, h, r,
                                &sm.full[slot], pol);
                }
            }
            issued = it + 1;
        }
        if (lane == 0) {
            for (int sl = 0; sl < kStagesM && sl < issued; ++sl) {
                const int last = sl + ((issued - 1 - sl) / kStagesM) * kStagesM;
                mbar_wait(&sm.full[sl], (last / kStagesM) & 1);
            }
        }
        return;
    }

    // =================================================================== consumers
    // q as the B operand of S^T = K Q^T: for k-step ks, b0 holds q[n][16ks +
    // 2(lane%4) + {0,1}] and b1 the same 8 dims later, n = lane/4 (zero if
    // n >= G).  Kept in registers for the whole kernel.
    const int qn = lane >> 2;
    const int qk = (lane & 3) * 2;
    uint32_t qb[8][2];
    {
        const int qh = qn < G ? qn : G - 1;  // rows >= G are zero; never read past q
        const uint32_t *qrow = reinterpret_cast<const uint32_t *>(p.q) +
                               ((static_cast<int64_t>(s) * p.num_q_heads + h * G + qh) * kD) / 2;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qb[ks][0] = qn < G ? __ldg(qrow + (16 * ks + qk) / 2) : 0u;
            qb[ks][1] = qn < G ? __ldg(qrow + (16 * ks + 8 + qk) / 2) : 0u;
        }
    }
    const float sl2 = p.scale_log2;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
        acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    // per-lane ldmatrix row/chunk selectors
    const int k_row = (lane & 7) + (((lane >> 3) & 1) << 3);  // token row for K (A, non-trans)
    const int k_chk = lane >> 4;                               // +0 / +1 chunk
    const int v_row = (lane & 7) + ((lane >> 4) << 3);         // token row for V (A, trans)
    const int v_chk = (lane >> 3) & 1;
    const int tok0 = lane >> 2;                                // C-fragment rows: tok0, tok0 + 8

    // One tile: zero the V rows past the end (partial tile), pull K and V^T
    // fragments into registers, run `loaded()` (hand the stage back), then
    // QK^T, the online softmax and PV.
    auto consume = [&](int slot, int ntok, auto &&loaded) {
        const uint32_t kb0 = smem_addr(&sm.kv[slot][0][0]);
        const uint32_t kb1 = smem_addr(&sm.kv[slot][1][0]);
        const uint32_t vb0 = smem_addr(&sm.kv[slot][2][0]);
        const uint32_t vb1 = smem_addr(&sm.kv[slot][3][0]);
        if (ntok < kTile) {
            uint4 *v0 = reinterpret_cast<uint4 *>(&sm.kv[slot][2][0]);
            uint4 *v1 = reinterpret_cast<uint4 *>(&sm.kv[slot][3][0]);
            for (int idx = ntok * 8 + lane; idx < kTile * 8; idx += 32) {
                v0[idx] = make_uint4(0, 0, 0, 0);
                v1[idx] = make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
        }
        // two consumer warps: all V^T fragments now; three: the first half now
        constexpr int kVa = kCW == 2 ? 8 : 4;
        uint32_t ka[8][4], va[kVa][4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            ldmatrix_x4(ka[ks], ((ks < 4) ? kb0 : kb1) + swz(k_row, (ks & 3) * 2 + k_chk));
        auto load_va = [&](int mt0) {
#pragma unroll
            for (int i = 0; i < kVa; ++i) {
                const int chunk = 2 * (mt0 + i) + v_chk;  // 16-byte chunk of the 128-dim row
                ldmatrix_x4_trans(va[i], ((chunk < 8) ? vb0 : vb1) + swz(v_row, chunk & 7));
            }
        };
        load_va(0);
        if constexpr (kCW == 2)
            loaded();

        // ---- S^T = K Q^T ------------------------------------------------
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
            mma_16816(sc, ka[ks], qb[ks][0], qb[ks][1]);
        // ---- online softmax (log2 domain) -------------------------------
        float x0 = sc[0] * sl2, x1 = sc[1] * sl2, x2 = sc[2] * sl2, x3 = sc[3] * sl2;
        if (ntok < kTile) {
            if (tok0 >= ntok) x0 = x1 = -INFINITY;
            if (tok0 + 8 >= ntok) x2 = x3 = -INFINITY;
        }
        float tA = fmaxf(x0, x2), tB = fmaxf(x1, x3);
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1) {
            tA = fmaxf(tA, __shfl_xor_sync(FULL, tA, off));
            tB = fmaxf(tB, __shfl_xor_sync(FULL, tB, off));
        }
        const float nA = fmaxf(mA, tA), nB = fmaxf(mB, tB);
        const float aA = exp2_approx(mA - nA), aB = exp2_approx(mB - nB);
        mA = nA;
        mB = nB;
        const float p0 = exp2_approx(x0 - nA), p1 = exp2_approx(x1 - nB);
        const float p2 = exp2_approx(x2 - nA), p3 = exp2_approx(x3 - nB);
        lA = fmaf(lA, aA, p0 + p2);
        lB = fmaf(lB, aB, p1 + p3);
        const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));  // tokens 0..7
        const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));  // tokens 8..15
        // ---- O^T = alpha O^T + V^T P^T ----------------------------------
#pragma unroll
        for (int half = 0; half < 8 / kVa; ++half) {
            if (half == 1) {  // three consumer warps: second half of V^T, then hand the stage back
                load_va(kVa);
                loaded();
            }
#pragma unroll
            for (int i = 0; i < kVa; ++i) {
                const int mt = half * kVa + i;
                acc[mt][0] *= aA;
                acc[mt][1] *= aB;
                acc[mt][2] *= aA;
                acc[mt][3] *= aB;
                mma_16816(acc[mt], va[i], pb0, pb1);
            }
        }
    };
    auto tile_tokens = [&](int it) { return min(kTile, t_end - (t_begin + it * kTile)); };

    if (use_tma) {
        // Fed by the producer warp: wait for the stage, release it as soon as
        // the fragments are in registers.
        for (int it = warp; it < num_tiles; it += kCW) {
            const int slot = it % kStagesM;
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait(&sm.full[slot], (it / kStagesM) & 1);
            if (!__shfl_sync(FULL, ok, 0))
                break;
            const int ntok = tile_tokens(it);
            consume(slot, ntok, [&] {
                if (ntok < kTile)
                    fence_proxy_async_smem();  // order the zero-fill before the next async refill
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.empty[slot]);
            });
        }
    } else {
        // Blocks of 1, 2 or 4 tokens: every row of a tile may live in another
        // block, so each consumer warp gathers its own tiles with 16-byte
        // cp.async copies, kAhead tiles ahead, into the stages it owns (tile t
        // in stage t % kStagesM, always this warp's).  Lane i < 16 computes the
        // cache row of token i once; the row is broadcast by shuffle to the
        // lanes that copy its 16 chunks (lanes 0-15 K, 16-31 V).
        constexpr int kAhead = kStagesM / kCW;
        const int tensor = lane >> 4;
        const int ch = lane & 15;
        const uint16_t *cache = static_cast<const uint16_t *>(tensor ? p.v_cache : p.k_cache);
        auto gather = [&](int it) {
            if (it < num_tiles) {
                const int slot = it % kStagesM;
                const int t0 = t_begin + it * kTile;
                const int ntok = tile_tokens(it);
                int64_t my_row = 0;
                if (lane < ntok) {
                    const int t = t0 + lane;
                    my_row = (static_cast<int64_t>(sm.blocks[t / B - first_blk]) * B + (t % B)) * Hkv + h;
                }
                const uint32_t base = smem_addr(&sm.kv[slot][tensor * 2 + (ch >> 3)][0]);
                for (int i = 0; i < ntok; ++i) {
                    const int64_t r = __shfl_sync(FULL, my_row, i);
                    cp_async16(base + swz(i, ch & 7), cache + r * kD + ch * 8);
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
#pragma unroll
        for (int k = 0; k < kAhead; ++k)
            gather(warp + k * kCW);
        for (int it = warp; it < num_tiles; it += kCW) {
            asm volatile("cp.async.wait_group %0;" ::"n"(kAhead - 1) : "memory");
            __syncwarp();
            consume(it % kStagesM, tile_tokens(it), [] {});
            __syncwarp();  // every lane is done with this stage before it is refilled
            gather(it + kAhead * kCW);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    }

    // ---- warp totals (sum over the 8 lanes sharing lane % 4) ----------------
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) {
        lA += __shfl_xor_sync(FULL, lA, off);
        lB += __shfl_xor_sync(FULL, lB, off);
    }
    if (threadIdx.x == 0)
        grid_launch_dependents();

    asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
    float *wacc = reinterpret_cast<float *>(&sm.kv[0][0][0]);  // [warp][8 heads][D]
    {
        const int hA = (lane & 3) * 2;
        float *wa = wacc + (warp * 8 + hA) * kD;
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
            sm.wm[warp][hA] = mA;
            sm.wm[warp][hA + 1] = mB;
            sm.wl[warp][hA] = lA;
            sm.wl[warp][hA + 1] = lB;
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");

    // the consumer threads finish dims t, t + 32 * kCW, ... of every real head
    constexpr int kStride = kCW * 32;
    constexpr int kPer = (kD + kStride - 1) / kStride;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kCW; ++w)
            M = fmaxf(M, sm.wm[w][g]);
        float L = 0.f, o[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u)
            o[u] = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kCW; ++w) {
                const float mw = sm.wm[w][g];
                if (mw == -INFINITY)
                    continue;
                const float sc = exp2f(mw - M);
                L = fmaf(sm.wl[w][g], sc, L);
#pragma unroll
                for (int u = 0; u < kPer; ++u)
                    if (threadIdx.x + kStride * u < kD)
                        o[u] = fmaf(wacc[(w * 8 + g) * kD + threadIdx.x + kStride * u], sc, o[u]);
            }
        }
        const int j = h * G + g;
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int d = threadIdx.x + kStride * u;
            if (d >= kD)
                break;
            if (p.num_parts == 1) {
                const float r = L > 0.f ? o[u] / L : 0.f;
                p.out[(static_cast<int64_t>(s) * p.num_q_heads + j) * kD + d] = __float2bfloat16_rn(r);
            } else {
                const int64_t idx = (static_cast<int64_t>(s) * p.num_q_heads + j) * p.num_parts + part;
                p.part_acc[idx * kD + d] = o[u];
                if (d == 0)
                    p.part_ml[idx] = make_float2(M, L);
            }
        }
    }
}

}  // namespace pa
