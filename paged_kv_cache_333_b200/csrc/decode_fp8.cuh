// Paged decode attention over an FP8 (OCP E4M3) KV cache.
//
// An FP8 cache stores one byte per value where bf16 takes two ("The pantry
// of pigeonholes", "The 10 knobs", knob 4 kv_cache_dtype, and "How it
// connects to the rest of the stack", on quantising the cache).  A stored code c
// of the K (V) tensor stands for value(c) * k_scale (v_scale).
//
// Same CTA decomposition, producer and split-K as decode_mma.cuh.  With half
// the bytes per token the consumer, not HBM, would set the pace if every code
// were first converted to f16 (one conversion per two codes, about 2x the
// instructions of the bf16 consumer per byte).  Here the codes go into the
// FP8 tensor-core MMA as they are (mma.m16n8k32, e4m3 x e4m3, fp32
// accumulate), and the two operands that are not codes are written as sums of
// two e4m3 numbers:
//   * q: each query head is scaled by a power of two 2^s_j that brings its
//     largest |element| into [128, 256), then split as q' = hi + lo with
//     hi = e4m3(q'), lo = e4m3(q' - hi).  For a bf16 q this is exact (the
//     residual of rounding 8 significant bits to 4 has at most 4) except for
//     elements below 2^-10 of the head's largest, whose error is under 2^-17
//     of it.  S = K.hi + K.lo (two MMAs), and 2^-s_j joins the score scale.
//   * P: probabilities are formed as 256 * 2^(x - m) (the factor cancels in
//     acc / l and in the split-K merge), rounded to f16 for the movmatrix
//     transpose, then split the same way; hi + lo keeps 8 significant bits,
//     the precision bf16 P has in the bf16 kernel.
// A tile is 32 tokens (4 KiB of K codes + 4 KiB of V codes, 128-byte
// swizzled rows of 128 codes), which gives four independent MMA chains for
// S^T and spreads the per-tile softmax reductions over twice the tokens.
//
// Operand layouts (lane = 4g + t):
//   * K (A of S^T = K Q^T, m16 tokens x k32 dims): ldmatrix.x4 (b16) on the
//     code tile gives exactly the e4m3 A fragment (row g / g+8, codes
//     4t..4t+3 and 16+4t..16+4t+3 of the 32-dim step): no rearrangement.
//   * P^T (B of O^T = V^T P^T, k32 tokens x n8 heads): movmatrix.trans of the
//     f16 pairs leaves lane (g, t) with head g at tokens {2t, 2t+1} of each
//     8-token group; the B fragment's k index 4t + i (+16) is assigned the
//     tokens {2t, 2t+1, 8+2t, 9+2t} (+16): a permutation of the reduction.
//   * V^T (A of the same MMA, m16 dims x k32 tokens): ldmatrix.x4.trans (b16)
//     gives lane (g, t) the codes of dims 16c+2g, 16c+2g+1 for tokens 2t, 2t+1
//     of each 8-token group; one byte permute per register builds the A
//     fragment with the same token permutation, A row g <-> dim 16c + 2g and
//     row g+8 <-> dim 16c + 2g + 1 (undone in the epilogue).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <type_traits>

#include "decode_mma.cuh"

namespace pa {

constexpr int kTileF = 32;
constexpr int kStagesF = 6;
// Consumer warps per CTA, CW = 2 or 3, chosen per call: the FP8 consumer
// does twice the tensor and byte-permute work per byte of the bf16 one.
// When the grid fits in one wave (at most 4 CTAs per SM) every CTA is
// resident from the start and two consumer warps at up to 168 registers do
// best (chat on B200: 21.2 us against 22.8 us with three); when it takes
// several waves, CTAs finish faster with three consumer warps at 128
// registers (B=16 and B=1 sweeps on B200: 15% and 21% more bandwidth).
template <int CW>
constexpr int fp8_threads() { return (CW + 1) * 32; }
constexpr int kFp8CtasPerSm = 4;
constexpr int kMaxConsumerWarpsF = 3;
constexpr int kTileBytesF = kTileF * kD;  // 32 tokens x 128 one-byte codes
static_assert(kStagesF % 2 == 0 && kStagesF % 3 == 0, "stages must be a multiple of the consumer warps");

struct DecodeSmemF {
    uint8_t kv[kStagesF][2][kTileBytesF];  // [stage][K, V][32 x 128], 128B-swizzled rows
    uint64_t full[kStagesF];
    uint64_t empty[kStagesF];
    float wm[kMaxConsumerWarpsF][8];
    float wl[kMaxConsumerWarpsF][8];
    int32_t blocks[kMaxPartBlocksM];
};
static_assert(sizeof(float) * kMaxConsumerWarpsF * 8 * kD <= sizeof(uint8_t) * kStagesF * 2 * kTileBytesF,
              "merge scratch must fit in the KV ring");
constexpr size_t kDecodeSmemBytesF = sizeof(DecodeSmemF) + 1024;

// D = A(16x32 e4m3, row) * B(32x8 e4m3, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_16832_e4m3(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}

// Two f16 (low half first) -> two e4m3 codes (low byte first), nearest even,
// saturating: one cvt.rn.satfinite.e4m3x2.f16x2.
__device__ __forceinline__ uint32_t f16x2_to_e4m3x2(uint32_t h2) {
    uint16_t c;
    asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(c) : "r"(h2));
    return c;
}

// Two e4m3 codes (low byte first) -> two f16 values (exact), low half first:
// one cvt.rn.f16x2.e4m3x2.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(two_codes & 0xffffu)));
    return h2;
}

// f16x2 value v -> (hi, lo) e4m3x2 code pairs with v ~ hi + lo (hi nearest to
// v, lo nearest to the residual v - hi, which f16 holds exactly).
__device__ __forceinline__ void split_f16x2(uint32_t v, uint32_t &hi, uint32_t &lo) {
    hi = f16x2_to_e4m3x2(v);
    const uint32_t back = e4m3x2_to_f16x2(hi);
    const __half2 r = __hsub2(*reinterpret_cast<const __half2 *>(&v), *reinterpret_cast<const __half2 *>(&back));
    lo = f16x2_to_e4m3x2(*reinterpret_cast<const uint32_t *>(&r));
}

// Four floats -> (hi, lo) codes, byte i from x[i].
__device__ __forceinline__ void split_f32x4(const float (&x)[4], uint32_t &hi, uint32_t &lo) {
    uint32_t hc[2], lc[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const __nv_fp8x2_storage_t c =
            __nv_cvt_float2_to_fp8x2(make_float2(x[2 * k], x[2 * k + 1]), __NV_SATFINITE, __NV_E4M3);
        const __half2_raw b = __nv_cvt_fp8x2_to_halfraw2(c, __NV_E4M3);
        const float r0 = x[2 * k] - __half2float(__ushort_as_half(b.x));  // raw bits, not a numeric cast
        const float r1 = x[2 * k + 1] - __half2float(__ushort_as_half(b.y));
        hc[k] = c;
        lc[k] = __nv_cvt_float2_to_fp8x2(make_float2(r0, r1), __NV_SATFINITE, __NV_E4M3);
    }
    hi = hc[0] | (hc[1] << 16);
    lo = lc[0] | (lc[1] << 16);
}

template <int G, int CW>
__global__ void __launch_bounds__(fp8_threads<CW>(), kFp8CtasPerSm)
decode_partition_fp8_kernel(const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
    static_assert(CW == 2 || CW == 3, "consumer warps");
    constexpr int kConsumerWarpsF = CW;
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
            mbar_init(&sm.empty[i], 32);  // every lane of the consuming warp releases the stage
        }
        mbar_init_fence();
    }
    if (use_tma && warp == kConsumerWarpsF && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    grid_dependency_wait();

    const int t_begin = part * p.part_tokens;
    const int first_blk = t_begin / B;
    const int32_t *row = p.block_tables + static_cast<int64_t>(s) * p.max_blocks_per_seq + first_blk;
    int32_t first_ids = 0;
    if (warp == kConsumerWarpsF && lane < p.max_blocks_per_seq - first_blk)
        first_ids = __ldg(row + lane);
    const int n = clamp_seq_len(p, s);
    if (part > 0 && t_begin >= n)
        return;
    const int t_end = min(n, t_begin + p.part_tokens);
    const int num_tiles = t_end > t_begin ? (t_end - t_begin + kTileF - 1) / kTileF : 0;
    const int Hkv = gridDim.y;
    if (warp == kConsumerWarpsF && num_tiles > 0) {
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
    if (warp == kConsumerWarpsF) {
        if (num_tiles == 0 || !use_tma)
            return;
        const uint64_t pol = l2_evict_first_policy();
        const int rows = B < kTileF ? B : kTileF;  // tokens per box (the tensor map's box height)
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
            const int t0 = t_begin + it * kTileF;
            const int ntok = min(kTileF, t_end - t0);
            const int nb = (ntok + rows - 1) / rows;  // boxes per tensor (blocks of B < 32 tokens)
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
    const int g = lane >> 2;  // MMA group: S^T token row / B column (head)
    const int t4 = lane & 3;  // thread in group
    // Packed columns (group sizes up to 4).  The MMAs' N = 8 columns hold 8
    // heads; with G <= 4 half of them would be empty.  There column n < 4
    // carries the hi part of head n and column n + 4 its lo part, for q
    // (S^T) and for P (O^T alike): one MMA where two would run.  The lane of
    // a hi column and the lane of its lo column (t4 and t4 ^ 2 in the C
    // fragments) then hold the same two heads: their partial scores are
    // summed by one shuffle, and the two halves of O are summed at the end.
    constexpr bool kPack = G <= 4;
    // q as the B operand of S^T, split into e4m3 hi + lo after a per-head
    // power-of-two scale.  Lane (g, t) holds head g (packed: head g % 4, hi
    // part for g < 4, lo part above), dims 32kk + 4t + i (register 0) and
    // 32kk + 16 + 4t + i (register 1) of k-step kk.
    uint32_t qh[4][2], ql[4][2];
    float sl2A, sl2B;  // score scale (log2 domain) of the lane's two C-fragment heads
    {
        const int qhead = kPack ? (g & 3) : g;
        const bool qreal = qhead < G;
        const int qr = qreal ? qhead : G - 1;
        const __nv_bfloat16 *qrow = reinterpret_cast<const __nv_bfloat16 *>(p.q) +
                                    (static_cast<int64_t>(s) * p.num_q_heads + h * G + qr) * kD;
        float qv[4][2][4];
        float amax = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint2 u = __ldg(reinterpret_cast<const uint2 *>(qrow + 32 * kk + 16 * r + 4 * t4));
                qv[kk][r][0] = qreal ? bf16lo(u.x) : 0.f;
                qv[kk][r][1] = qreal ? bf16hi(u.x) : 0.f;
                qv[kk][r][2] = qreal ? bf16lo(u.y) : 0.f;
                qv[kk][r][3] = qreal ? bf16hi(u.y) : 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    amax = fmaxf(amax, fabsf(qv[kk][r][i]));
            }
        }
        amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
        // 2^sh brings amax into [128, 256): amax in [2^(e-1), 2^e) -> sh = 8 - e.
        int sh = 0;
        if (amax > 0.f && amax <= 3.0e38f) {
            int e;
            frexpf(amax, &e);
            sh = max(-120, min(126, 8 - e));
        }
        const float up = __int_as_float((127 + sh) << 23);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float x[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    x[i] = qv[kk][r][i] * up;
                split_f32x4(x, qh[kk][r], ql[kk][r]);
                if constexpr (kPack)
                    qh[kk][r] = g < 4 ? qh[kk][r] : ql[kk][r];  // lo columns carry the lo part
            }
        }
        const float base = p.scale_log2 * p.k_scale;
        // the lane's C-fragment columns 2t, 2t+1 are heads 2hs, 2hs+1 (packed:
        // column c is head c % 4), whose shifts live in groups 2hs and 2hs+1
        const int hs = kPack ? (t4 & 1) : t4;
        const int shA = __shfl_sync(FULL, sh, 8 * hs);
        const int shB = __shfl_sync(FULL, sh, 8 * hs + 4);
        sl2A = base * __int_as_float((127 - shA) << 23);
        sl2B = base * __int_as_float((127 - shB) << 23);
    }
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    float acc[8][4];
#pragma unroll
    for (int c = 0; c < 8; ++c)
        acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;

    const int mi = lane >> 3;  // which 8x8 matrix of an x4 load this lane addresses
    const int k_tok = (lane & 7) + ((mi & 1) << 3), k_chk = mi >> 1;

    // One tile.  kFull (compile time): all 32 tokens are in range, which is
    // every tile but the last of a partition; the masked body is only
    // instantiated for that last one.
    auto consume = [&](auto full, int slot, int ntok, auto &&loaded) {
        constexpr bool kFull = decltype(full)::value;
        const uint32_t kb = smem_addr(&sm.kv[slot][0][0]);
        const uint32_t vb = smem_addr(&sm.kv[slot][1][0]);
        if constexpr (!kFull) {
            uint4 *v = reinterpret_cast<uint4 *>(&sm.kv[slot][1][0]);
            for (int idx = ntok * 8 + lane; idx < kTileF * 8; idx += 32)
                v[idx] = make_uint4(0, 0, 0, 0);
            __syncwarp();
        }
        // ---- S^T = K Q^T for tokens 16mt + {g, g+8}, heads 2t, 2t+1
        float shi[2][4], slo[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                shi[mt][i] = slo[mt][i] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                uint32_t kf[4];
                ldmatrix_x4(kf, kb + swz(16 * mt + k_tok, 2 * kk + k_chk));
                mma_16832_e4m3(shi[mt], kf, qh[kk][0], qh[kk][1]);
                if constexpr (!kPack)
                    mma_16832_e4m3(slo[mt], kf, ql[kk][0], ql[kk][1]);
            }
        }
        if constexpr (kPack) {
            // the other part of the same heads' scores, from the lane two over
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    slo[mt][i] = __shfl_xor_sync(FULL, shi[mt][i], 2);
        }
        // V^T fragments, in two halves of four 16-dim tiles (fewer live
        // registers): matrix i of load c = tokens 8i..8i+7, dims 16c..16c+15.
        // The first half is loaded now, the second after the first half's
        // MMAs; the stage is released once both are in registers.
        uint32_t vf[4][4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
            ldmatrix_x4_trans(vf[c], vb + swz(lane, c));
        // ---- online softmax (log2 domain) -------------------------------
        float x[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            x[mt][0] = (shi[mt][0] + slo[mt][0]) * sl2A;
            x[mt][1] = (shi[mt][1] + slo[mt][1]) * sl2B;
            x[mt][2] = (shi[mt][2] + slo[mt][2]) * sl2A;
            x[mt][3] = (shi[mt][3] + slo[mt][3]) * sl2B;
            if constexpr (!kFull) {
                if (16 * mt + g >= ntok) x[mt][0] = x[mt][1] = -INFINITY;
                if (16 * mt + g + 8 >= ntok) x[mt][2] = x[mt][3] = -INFINITY;
            }
        }
        float tA = fmaxf(fmaxf(x[0][0], x[0][2]), fmaxf(x[1][0], x[1][2]));
        float tB = fmaxf(fmaxf(x[0][1], x[0][3]), fmaxf(x[1][1], x[1][3]));
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1) {
            tA = fmaxf(tA, __shfl_xor_sync(FULL, tA, off));
            tB = fmaxf(tB, __shfl_xor_sync(FULL, tB, off));
        }
        const float nA = fmaxf(mA, tA), nB = fmaxf(mB, tB);
        const float aA = exp2_approx(mA - nA), aB = exp2_approx(mB - nB);
        mA = nA;
        mB = nB;
        // 256 * 2^(x - m): p in [0, 256], clear of the e4m3 subnormals
        const float oA = nA - 8.f, oB = nB - 8.f;
        float pr[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            pr[mt][0] = exp2_approx(x[mt][0] - oA);
            pr[mt][1] = exp2_approx(x[mt][1] - oB);
            pr[mt][2] = exp2_approx(x[mt][2] - oA);
            pr[mt][3] = exp2_approx(x[mt][3] - oB);
        }
        lA = fmaf(lA, aA, (pr[0][0] + pr[0][2]) + (pr[1][0] + pr[1][2]));
        lB = fmaf(lB, aB, (pr[0][1] + pr[0][3]) + (pr[1][1] + pr[1][3]));
        // P^T as the B operand: movmatrix k gives head g, tokens 8k + 2t, 8k + 2t + 1
        uint32_t ph[4];
        [[maybe_unused]] uint32_t pl[4];  // unpacked path only
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                if constexpr (kPack) {
                    // lanes of lo columns (t >= 2) hand over the f16 residual
                    // P - hi(P); after the transpose every lane encodes what it
                    // holds: hi(P) in columns 0-3, lo(P) in columns 4-7, exactly
                    // the split_f16x2 pair of the unpacked path
                    const uint32_t v = pack_f16x2(pr[mt][2 * hf], pr[mt][2 * hf + 1]);
                    const uint32_t back = e4m3x2_to_f16x2(f16x2_to_e4m3x2(v));
                    const __half2 r = __hsub2(*reinterpret_cast<const __half2 *>(&v),
                                              *reinterpret_cast<const __half2 *>(&back));
                    const uint32_t w = t4 >= 2 ? *reinterpret_cast<const uint32_t *>(&r) : v;
                    ph[2 * mt + hf] = f16x2_to_e4m3x2(movmatrix_trans(w));
                } else {
                    const uint32_t u = movmatrix_trans(pack_f16x2(pr[mt][2 * hf], pr[mt][2 * hf + 1]));
                    split_f16x2(u, ph[2 * mt + hf], pl[2 * mt + hf]);
                }
            }
        }
        const uint32_t pbh0 = __byte_perm(ph[0], ph[1], 0x5410), pbh1 = __byte_perm(ph[2], ph[3], 0x5410);
        [[maybe_unused]] uint32_t pbl0 = 0, pbl1 = 0;
        if constexpr (!kPack) {
            pbl0 = __byte_perm(pl[0], pl[1], 0x5410);
            pbl1 = __byte_perm(pl[2], pl[3], 0x5410);
        }
        // ---- O^T = alpha O^T + V^T P^T: d-tile c, A row g <-> dim 16c+2g, row
        // g+8 <-> 16c+2g+1.  The tile's product starts from zero and joins the
        // running sum in fp32 outside the MMA, so the sum over thousands of
        // tiles does not depend on how the FP8 MMA rounds its accumulator.
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            if (half == 1) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    ldmatrix_x4_trans(vf[c], vb + swz(lane, 4 + c));
                loaded();
            }
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const int c = 4 * half + c4;
                const uint32_t a[4] = {__byte_perm(vf[c4][0], vf[c4][1], 0x6420),   // dim 2g, tokens 2t,2t+1,8+2t,9+2t
                                       __byte_perm(vf[c4][0], vf[c4][1], 0x7531),   // dim 2g+1
                                       __byte_perm(vf[c4][2], vf[c4][3], 0x6420),   // dim 2g, tokens +16
                                       __byte_perm(vf[c4][2], vf[c4][3], 0x7531)};  // dim 2g+1, tokens +16
                float o[4] = {0.f, 0.f, 0.f, 0.f};
                mma_16832_e4m3(o, a, pbh0, pbh1);
                if constexpr (!kPack)
                    mma_16832_e4m3(o, a, pbl0, pbl1);
                acc[c][0] = fmaf(acc[c][0], aA, o[0]);
                acc[c][1] = fmaf(acc[c][1], aB, o[1]);
                acc[c][2] = fmaf(acc[c][2], aA, o[2]);
                acc[c][3] = fmaf(acc[c][3], aB, o[3]);
            }
        }
    };
    auto tile_tokens = [&](int it) { return min(kTileF, t_end - (t_begin + it * kTileF)); };

    if (use_tma) {
        // Every lane polls the stage's barrier (no divergent branch around a
        // single waiter) and, once its own fragment loads are done, arrives
        // on the stage's release barrier (count 32).
        for (int it = warp; it < num_tiles; it += kConsumerWarpsF) {
            const int slot = it % kStagesF;
            if (!__all_sync(FULL, mbar_wait(&sm.full[slot], (it / kStagesF) & 1)))
                break;
            const int ntok = tile_tokens(it);
            if (ntok == kTileF) {
                consume(std::true_type{}, slot, ntok, [&] { mbar_arrive(&sm.empty[slot]); });
            } else {
                consume(std::false_type{}, slot, ntok, [&] {
                    fence_proxy_async_smem();  // the V rows this warp zeroed, before the next async refill
                    mbar_arrive(&sm.empty[slot]);
                });
            }
        }
    } else {
        // Blocks of 1, 2 or 4 tokens: each consumer warp gathers its own tiles
        // (lane = token parity, tensor, 16-byte chunk of the 128-byte row).
        constexpr int kAhead = kStagesF / kConsumerWarpsF;
        const int par = lane >> 4, tensor = (lane >> 3) & 1, ch = lane & 7;
        const uint8_t *cache = static_cast<const uint8_t *>(tensor ? p.v_cache : p.k_cache);
        auto gather = [&](int it) {
            if (it < num_tiles) {
                const int slot = it % kStagesF;
                const int t0 = t_begin + it * kTileF;
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
            gather(warp + k * kConsumerWarpsF);
        for (int it = warp; it < num_tiles; it += kConsumerWarpsF) {
            asm volatile("cp.async.wait_group %0;" ::"n"(kAhead - 1) : "memory");
            __syncwarp();
            const int ntok = tile_tokens(it);
            if (ntok == kTileF)
                consume(std::true_type{}, it % kStagesF, ntok, [] {});
            else
                consume(std::false_type{}, it % kStagesF, ntok, [] {});
            __syncwarp();
            gather(it + kAhead * kConsumerWarpsF);
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
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarpsF * 32) : "memory");
    float *wacc = reinterpret_cast<float *>(&sm.kv[0][0][0]);  // [warp][8 heads][D]
    {
        const int hA = t4 * 2;
        float *wa = wacc + (warp * 8 + hA) * kD;
        float *wb = wa + kD;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int d = c * 16 + 2 * g;  // O^T row g <-> dim 16c+2g, row g+8 <-> dim 16c+2g+1
            wa[d] = acc[c][0];
            wb[d] = acc[c][1];
            wa[d + 1] = acc[c][2];
            wb[d + 1] = acc[c][3];
        }
        if (lane < 4) {
            sm.wm[warp][hA] = mA;
            sm.wm[warp][hA + 1] = mB;
            sm.wl[warp][hA] = lA;
            sm.wl[warp][hA + 1] = lB;
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarpsF * 32) : "memory");
#pragma unroll
    for (int gq = 0; gq < G; ++gq) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarpsF; ++w)
            M = fmaxf(M, sm.wm[w][gq]);
        // the consumer threads finish dims t, t + 32 * kConsumerWarpsF, ...
        constexpr int kStride = kConsumerWarpsF * 32;
        constexpr int kPer = (kD + kStride - 1) / kStride;
        float L = 0.f, o[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u)
            o[u] = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarpsF; ++w) {
                const float mw = sm.wm[w][gq];
                if (mw == -INFINITY)
                    continue;
                const float sc = exp2f(mw - M);
                L = fmaf(sm.wl[w][gq], sc, L);
#pragma unroll
                for (int u = 0; u < kPer; ++u)
                    if (threadIdx.x + kStride * u < kD) {
                        const int d = threadIdx.x + kStride * u;
                        float part = wacc[(w * 8 + gq) * kD + d];
                        if constexpr (kPack)
                            part += wacc[(w * 8 + gq + 4) * kD + d];  // the lo columns' share
                        o[u] = fmaf(part, sc, o[u]);
                    }
            }
        }
        const int jq = h * G + gq;
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int d = threadIdx.x + kStride * u;
            if (d >= kD)
                break;
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
