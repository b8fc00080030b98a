// Paged decode attention over an FP8 (OCP E4M3) KV cache.
//
// An FP8 cache halves the bytes per token ("The pantry of pigeonholes", "The
// 10 knobs", knob 4 kv_cache_dtype; "How it connects to the rest of the
// stack": moving the KV to FP8 halves the bytes per token).  A stored code c
// of the K (V) tensor stands for value(c) * k_scale (v_scale).
//
// Same CTA decomposition, producer and split-K as decode_mma.cuh; a 16-token
// tile is now 2 KiB of K and 2 KiB of V (rows of 128 one-byte codes, 128-byte
// swizzle), so the ring has twice the stages for the same bytes in flight.
// The consumer feeds the codes straight into f16 tensor-core MMAs (every
// e4m3 value is exact in f16), without a staging pass through shared memory:
//   * K: ldmatrix (b16) on the code tile gives each lane four consecutive
//     codes of a row (dims 4(lane%4)..+3 of a 16-dim chunk); converted to two
//     f16 pairs they fill the A-operand slots of MMA k-indices 2q, 2q+1
//     (dims 4q, 4q+1) and 2q+8, 2q+9 (dims 4q+2, 4q+3), q = lane % 4.  The
//     reduction dimension is only reordered, so q's B operand is loaded with
//     the same order and S^T is unchanged.
//   * V: ldmatrix.trans (b16) on the code tile gives each lane codes of two
//     consecutive tokens for a pair of dims (2r, 2r+1), r = lane / 4; a byte
//     permute splits them into the (token, token+1) pairs of dim 2r and of dim
//     2r+1, which become A-operand rows r and r+8 of V^T.  Only the output rows
//     of O^T are reordered (row m <-> dim 2m, row m+8 <-> dim 2m+1), which the
//     epilogue undoes.
//   * scales: k_scale joins the softmax scale (scores * scale*k_scale*log2 e);
//     v_scale multiplies the partition's accumulator in the epilogue.
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "decode_mma.cuh"

namespace pa {

constexpr int kStagesF = 12;
constexpr int kTileBytesF = kTile * kD;  // 16 tokens x 128 one-byte codes
static_assert(kStagesF % kConsumerWarpsM == 0, "stages must be a multiple of the consumer warps");

struct DecodeSmemF {
    uint8_t kv[kStagesF][2][kTileBytesF];  // [stage][K, V][16 x 128], 128B-swizzled rows
    uint64_t full[kStagesF];
    uint64_t empty[kStagesF];
    float wm[kConsumerWarpsM][8];
    float wl[kConsumerWarpsM][8];
    int32_t blocks[kMaxPartBlocksM];
};
static_assert(sizeof(float) * kConsumerWarpsM * 8 * kD <= sizeof(uint8_t) * kStagesF * 2 * kTileBytesF,
              "merge scratch must fit in the KV ring");
constexpr size_t kDecodeSmemBytesF = sizeof(DecodeSmemF) + 1024;

__device__ __forceinline__ void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two e4m3 codes (low byte first) -> two f16 values (exact), low half first.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xffffu),
                                                     __NV_E4M3);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

template <int G>
__global__ void __launch_bounds__(kDecodeThreadsM, kMmaCtasPerSm)
decode_partition_fp8_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ uint8_t smem_raw[];
    DecodeSmemF &sm = *reinterpret_cast<DecodeSmemF *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int part = blockIdx.x;
    const int h = blockIdx.y;
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int B = p.block_size;
    const bool use_tma = B >= 8;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStagesF; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        mbar_init_fence();
    }
    if (use_tma && warp == kConsumerWarpsM && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    grid_dependency_wait();

    const int t_begin = part * p.part_tokens;
    const int first_blk = t_begin / B;
    const int32_t *row = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq + first_blk;
    int32_t first_ids = 0;
    if (warp == kConsumerWarpsM && lane < p.max_blocks_per_seq - first_blk)
        first_ids = __ldg(row + lane);
    const int n = clamp_seq_len(p, s);
    if (part > 0 && t_begin >= n)
        return;
    const int t_end = min(n, t_begin + p.part_tokens);
    const int num_tiles = t_end > t_begin ? (t_end - t_begin + kTile - 1) / kTile : 0;
    const int Hkv = gridDim.y;
    if (warp == kConsumerWarpsM && num_tiles > 0) {
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
    if (warp == kConsumerWarpsM) {
        if (num_tiles == 0 || !use_tma)
            return;
        const uint64_t pol = l2_evict_first_policy();
        int issued = 0;
        for (int it = 0; it < num_tiles; ++it) {
            const int slot = it % kStagesF;
            if (it >= kStagesF) {
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait(&sm.empty[slot], ((it / kStagesF) + 1) & 1);
                if (!__shfl_sync(FULL, ok, 0))
                    break;
            }
            const int t0 = t_begin + it * kTile;
            const int ntok = min(kTile, t_end - t0);
            const int rows = B < kTile ? B : kTile;
            const int nb = B >= kTile ? 1 : (ntok + B - 1) / B;
            if (lane == 0)
                mbar_arrive_expect_tx(&sm.full[slot], static_cast<uint32_t>(nb * rows * kD * 2));
            __syncwarp();
            const int j = lane >> 1, q = lane & 1;  // box j of tensor q (0 = K, 1 = V)
            if (j < nb) {
                const int32_t blk = sm.blocks[(t0 + j * rows) / B - first_blk];
                const int32_t r = blk * B + ((t0 + j * rows) % B);
                tma_load_3d(&sm.kv[slot][q][j * rows * kD], q ? &tm_v : &tm_k, 0, h, r, &sm.full[slot], pol);
            }
            issued = it + 1;
        }
        if (lane == 0) {
            for (int sl = 0; sl < kStagesF && sl < issued; ++sl) {
                const int last = sl + ((issued - 1 - sl) / kStagesF) * kStagesF;
                mbar_wait(&sm.full[sl], (last / kStagesF) & 1);
            }
        }
        return;
    }

    // =================================================================== consumers
    // q as the B operand, with the reduction order of the K fragments: for
    // k-step ks, b0 = q[n][16ks + 4(lane%4) + {0,1}], b1 = ... + {2,3}.
    const int qn = lane >> 2;
    const int q4 = (lane & 3) * 4;
    uint32_t qb[8][2];
    {
        const int qh = qn < G ? qn : G - 1;
        const __nv_bfloat16 *qrow = reinterpret_cast<const __nv_bfloat16 *>(p.q) +
                                    (static_cast<int64_t>(s) * p.num_q_heads + h * G + qh) * kD;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            const uint2 u = __ldg(reinterpret_cast<const uint2 *>(qrow + 16 * ks + q4));
            const float a0 = bf16lo(u.x), a1 = bf16hi(u.x), a2 = bf16lo(u.y), a3 = bf16hi(u.y);
            qb[ks][0] = qn < G ? pack_f16x2(a0, a1) : 0u;
            qb[ks][1] = qn < G ? pack_f16x2(a2, a3) : 0u;
        }
    }
    const float sl2 = p.scale_log2 * p.k_scale;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
        acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    const int mi = lane >> 3;                                  // which 8x8 matrix of an x4 load
    const int k_tok = (lane & 7) + ((mi & 1) << 3), k_chk = mi >> 1;
    const int v_tok = (lane & 7) + ((mi >> 1) << 3), v_chk = mi & 1;
    const int tok0 = lane >> 2;

    auto consume = [&](int slot, int ntok, auto &&loaded) {
        const uint32_t kb = smem_addr(&sm.kv[slot][0][0]);
        const uint32_t vb = smem_addr(&sm.kv[slot][1][0]);
        if (ntok < kTile) {
            uint4 *v = reinterpret_cast<uint4 *>(&sm.kv[slot][1][0]);
            for (int idx = ntok * 8 + lane; idx < kTile * 8; idx += 32)
                v[idx] = make_uint4(0, 0, 0, 0);
            __syncwarp();
        }
        uint32_t kr[4][4], vr[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            ldmatrix_x4(kr[j], kb + swz(k_tok, 2 * j + k_chk));
            ldmatrix_x4_trans(vr[j], vb + swz(v_tok, 2 * j + v_chk));
        }
        loaded();

        // ---- S^T = K Q^T: k-step 2j+hf uses registers 2hf (tokens 0-7) and 2hf+1 (8-15)
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t lo = kr[j][2 * hf], hi = kr[j][2 * hf + 1];
                const uint32_t a[4] = {e4m3x2_to_f16x2(lo), e4m3x2_to_f16x2(hi), e4m3x2_to_f16x2(lo >> 16),
                                       e4m3x2_to_f16x2(hi >> 16)};
                mma_16816_f16(sc, a, qb[2 * j + hf][0], qb[2 * j + hf][1]);
            }
        }
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
        const float aA = exp2f(mA - nA), aB = exp2f(mB - nB);
        mA = nA;
        mB = nB;
        const float p0 = exp2f(x0 - nA), p1 = exp2f(x1 - nB);
        const float p2 = exp2f(x2 - nA), p3 = exp2f(x3 - nB);
        lA = fmaf(lA, aA, p0 + p2);
        lB = fmaf(lB, aB, p1 + p3);
        const uint32_t pb0 = movmatrix_trans(pack_f16x2(p0, p1));  // tokens 0..7
        const uint32_t pb1 = movmatrix_trans(pack_f16x2(p2, p3));  // tokens 8..15
        // ---- O^T += V^T P^T: m-tile 2j+hh from matrices hh (tokens 0-7) and 2+hh (8-15)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int mt = 2 * j + hh;
                acc[mt][0] *= aA;
                acc[mt][1] *= aB;
                acc[mt][2] *= aA;
                acc[mt][3] *= aB;
                const uint32_t lo = vr[j][hh], hi = vr[j][2 + hh];
                const uint32_t a[4] = {e4m3x2_to_f16x2(__byte_perm(lo, 0, 0x4420)),   // dim 2r, tokens 0-7
                                       e4m3x2_to_f16x2(__byte_perm(lo, 0, 0x4431)),   // dim 2r+1
                                       e4m3x2_to_f16x2(__byte_perm(hi, 0, 0x4420)),   // dim 2r, tokens 8-15
                                       e4m3x2_to_f16x2(__byte_perm(hi, 0, 0x4431))};  // dim 2r+1
                mma_16816_f16(acc[mt], a, pb0, pb1);
            }
        }
    };
    auto tile_tokens = [&](int it) { return min(kTile, t_end - (t_begin + it * kTile)); };

    if (use_tma) {
        for (int it = warp; it < num_tiles; it += kConsumerWarpsM) {
            const int slot = it % kStagesF;
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait(&sm.full[slot], (it / kStagesF) & 1);
            if (!__shfl_sync(FULL, ok, 0))
                break;
            const int ntok = tile_tokens(it);
            consume(slot, ntok, [&] {
                if (ntok < kTile)
                    fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.empty[slot]);
            });
        }
    } else {
        // Blocks of 1, 2 or 4 tokens: each consumer warp gathers its own tiles
        // (lane = token parity, tensor, 16-byte chunk of the 128-byte row).
        constexpr int kAhead = kStagesF / kConsumerWarpsM;
        const int par = lane >> 4, tensor = (lane >> 3) & 1, ch = lane & 7;
        const uint8_t *cache = static_cast<const uint8_t *>(tensor ? p.v_cache : p.k_cache);
        auto gather = [&](int it) {
            if (it < num_tiles) {
                const int slot = it % kStagesF;
                const int t0 = t_begin + it * kTile;
                const int ntok = tile_tokens(it);
                int64_t my_row = 0;
                if (lane < ntok) {
                    const int t = t0 + lane;
                    my_row = (static_cast<int64_t>(sm.blocks[t / B - first_blk]) * B + (t % B)) * Hkv + h;
                }
                const uint32_t base = smem_addr(&sm.kv[slot][tensor][0]);
                for (int i = 0; i < ntok; i += 2) {
                    const int tk = i + par;
                    const int64_t r = __shfl_sync(FULL, my_row, tk < ntok ? tk : i);
                    if (tk < ntok)
                        cp_async16(base + swz(tk, ch), cache + r * kD + ch * 16);
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
#pragma unroll
        for (int k = 0; k < kAhead; ++k)
            gather(warp + k * kConsumerWarpsM);
        for (int it = warp; it < num_tiles; it += kConsumerWarpsM) {
            asm volatile("cp.async.wait_group %0;" ::"n"(kAhead - 1) : "memory");
            __syncwarp();
            consume(it % kStagesF, tile_tokens(it), [] {});
            __syncwarp();
            gather(it + kAhead * kConsumerWarpsM);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    }

    // ---- warp totals, cross-warp merge, output (dims un-permuted) ----------
#pragma unroll
    for (int off = 4; off <= 16; off <<= 1) {
        lA += __shfl_xor_sync(FULL, lA, off);
        lB += __shfl_xor_sync(FULL, lB, off);
    }
    if (threadIdx.x == 0)
        grid_launch_dependents();
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarpsM * 32) : "memory");
    float *wacc = reinterpret_cast<float *>(&sm.kv[0][0][0]);  // [warp][8 heads][D]
    {
        const int hA = (lane & 3) * 2;
        float *wa = wacc + (warp * 8 + hA) * kD;
        float *wb = wa + kD;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d = mt * 16 + 2 * tok0;  // O^T row m <-> dim 2m, row m+8 <-> dim 2m+1
            wa[d] = acc[mt][0];
            wb[d] = acc[mt][1];
            wa[d + 1] = acc[mt][2];
            wb[d + 1] = acc[mt][3];
        }
        if (lane < 4) {
            sm.wm[warp][hA] = mA;
            sm.wm[warp][hA + 1] = mB;
            sm.wl[warp][hA] = lA;
            sm.wl[warp][hA + 1] = lB;
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarpsM * 32) : "memory");
#pragma unroll
    for (int g = 0; g < G; ++g) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarpsM; ++w)
            M = fmaxf(M, sm.wm[w][g]);
        float L = 0.f, o[2] = {0.f, 0.f};
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarpsM; ++w) {
                const float mw = sm.wm[w][g];
                if (mw == -INFINITY)
                    continue;
                const float sc = exp2f(mw - M);
                L = fmaf(sm.wl[w][g], sc, L);
#pragma unroll
                for (int u = 0; u < 2; ++u)
                    o[u] = fmaf(wacc[(w * 8 + g) * kD + threadIdx.x + 64 * u], sc, o[u]);
            }
        }
        const int jq = h * G + g;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int d = threadIdx.x + 64 * u;
            const float ov = o[u] * p.v_scale;
            if (p.num_parts == 1) {
                const float r = L > 0.f ? ov / L : 0.f;
                p.out[(static_cast<int64_t>(s) * p.num_q_heads + jq) * kD + d] = __float2bfloat16_rn(r);
            } else {
                const int64_t idx = (static_cast<int64_t>(s) * p.num_q_heads + jq) * p.num_parts + part;
                p.part_acc[idx * kD + d] = ov;
                if (d == 0)
                    p.part_ml[idx] = make_float2(M, L);
            }
        }
    }
}

}  // namespace pa
