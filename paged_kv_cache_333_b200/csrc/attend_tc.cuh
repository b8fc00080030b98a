// Attention of several query tokens per request over the paged cache on the
// fifth-generation tensor cores (tcgen05): the same operation as
// attend_partition_kernel ("PagedAttention: fragmentation, blocks, block
// tables", the attention-metadata passage: query_start_loc, seq_lens,
// max_query_len; row i of a request with q_len rows and n tokens attends to
// positions 0 .. n - q_len + i), for requests with many rows: chunks of a
// prefill, long speculative runs.
//
// Work decomposition.  A column is one (query row, query head of the KV group)
// pair, c = i * G + g, as in attend.cuh.  A work unit is one (split-K
// partition, KV head, request, chunk of 128 columns), or, when every request
// has at most 64 columns and the KV head count is even, one (partition, pair
// of KV heads, request) with each head's columns in 64 of the 128 MMA rows
// (HP = 2, described at the kernel).  Its token range is streamed in tiles
// of 64 rows (64 tokens of the head, or 32 tokens of each of the two):
//   S = Q K^T    M = 128 columns, N = 64 rows, K = 128 dims: 8 MMAs of K = 16
//   O += P V     M = 128 columns, N = 128 dims, K = 64 rows: 4 MMAs of K = 16
// (tcgen05.mma.cta_group::1.kind::f16, bf16 operands, fp32 accumulators in
// tensor memory).  Q and K are K-major and V is MN-major in shared memory, in
// the 128-byte swizzled layout the TMA loads write: rows of 128 bytes, 16-byte
// chunk j of row r at position j ^ (r % 8), 8-row groups 1024 bytes apart.
// P is the A operand of the P V product straight from tensor memory.
//
// Persistent grid.  One CTA per SM (shared memory) walks the units
// blockIdx.x, blockIdx.x + gridDim.x, ...; every role derives the same unit
// fields from global memory (loaded one unit ahead) and skips the same empty
// units.  Tiles, S buffers and P buffers are counted across units, so the
// producer streams the next unit's q tile and K/V tiles while the current
// unit's softmax and epilogue finish; a CTA per unit left its SM without
// loads in flight for about a third of its life (set-up, first load,
// epilogue).
//
// Roles (352 threads):
//   warps 0-3  softmax: thread t owns column t of the unit, which is tensor-
//              memory lane t (a warp may only read lanes 32 * (warp % 4) ..
//              + 31).  Per tile: read its S row (64 fp32), mask, online
//              softmax with a lazily moved reference max, write its P row
//              (bf16 pairs) to tensor memory; per unit: leave (m_ref, l) in
//              tensor memory for the epilogue warps and go on to the next;
//   warps 4, 10 producers: per unit, the block-table slice into shared memory
//              (each its own copy), the q tile by TMA (two buffers; warp 4),
//              and the K/V tiles into a 5-stage ring (warp 4 the even slots,
//              warp 10 the odd ones), by TMA for whole tiles of blocks >= 8
//              tokens, else by a cp.async gather that zero-fills the rows past
//              the range;
//   warp 5     allocates tensor memory; one thread issues the MMAs;
//   warps 6-9  epilogue: warp w reads lane quarter w % 4 of a finished
//              unit's O buffer and (m_ref, l), and writes the output rows (or
//              the split-K partials), while the softmax warps already work on
//              the next unit.
// Tensor memory (512 columns): S double-buffered in [0, 64) and [64, 128),
// O double-buffered by unit in [128, 256) and [256, 384), P double-buffered
// in [384, 416) and [416, 448), (m_ref, l) of unit k at 448 + 2 (k % 2).
//
// Lazy rescaling.  A column keeps a reference max m_ref (log2 domain) and
// moves it only when a tile's max exceeds it by more than 8; the weights
// 2^(x - m_ref) then stay <= 256, exact enough in bf16 for P and far from
// fp32 overflow in O and l.  Moving m_ref multiplies that column's O row in
// tensor memory by 2^(old - new), after the previous tile's P V has
// completed.  (m_ref, l, O) is a consistent triple at any reference, which is
// all the final division and the split-K merge need.
//
// Synchronisation (all mbarriers, every wait bounded; t counts tiles and k
// units with work, both across the CTA's units):
//   full[s]     producer -> MMA       stage s holds tile t (TMA bytes or cp.async)
//   empty[s]    MMA commit -> producer  P V of tile t done: stage s reusable
//   q_full[b]   producer (TMA) -> MMA  q tile of unit k in buffer b = k % 2
//   q_empty[b]  MMA commit -> producer  unit k's last S read buffer b
//   s_full[b]   MMA commit -> softmax  S of tile t in buffer b = t % 2
//   s_free[b]   softmax (4 warps) -> MMA  S buffer b read
//   p_full[b]   softmax (4 warps) -> MMA  P buffer b written, O rescaled
//   pv_done[b]  MMA commit -> softmax  P V of tile t done: P buffer b free, O current
//   o_full[b]   MMA commit -> epilogue  unit k's last P V done: O buffer b = k % 2 final
//   ml_full[b]  softmax (4 warps) -> epilogue  unit k's (m_ref, l) in tensor memory
//   o_free[b]   epilogue (4 warps) -> MMA, softmax  unit k's O and (m_ref, l) read:
//               unit k + 2 may overwrite them
// The MMA thread issues S(t + 1) before P V(t), so the tensor pipe computes
// the next scores while the softmax warps work on the current tile.  No
// waiter can fall two phases behind a barrier: each phase it waits for is
// the latest one that the other side can have completed.
#pragma once

#include "attend.cuh"

namespace pa {

constexpr int kTokTc = 64;      // tokens per tile
constexpr int kStagesTc = 5;    // K/V ring depth
constexpr int kMaxPartBlocksTc = 192;  // block-table entries one work unit may cover
constexpr int kColsTc = 128;    // columns per CTA (= MMA M = tensor-memory lanes)
constexpr int kTmemColsTc = 512;  // S 2x64, O 2x128, P 2x32 (bf16 pairs), (m_ref, l) 2x2
constexpr int kTmemOTc = 2 * kTokTc;             // O of unit k in [128 + 128 (k % 2), ...)
constexpr int kTmemPTc = kTmemOTc + 2 * kD;      // P of tile t in [384 + 32 (t % 2), ...)
constexpr int kTmemMlTc = kTmemPTc + 2 * 32;     // (m_ref, l) of unit k at 448 + 2 (k % 2)
static_assert(kTmemMlTc + 4 <= kTmemColsTc, "tensor memory columns");
constexpr int kTcThreads = 352;
constexpr int kTcProducerWarp = 4;
constexpr int kTcMmaWarp = 5;
constexpr int kTcEpilogueWarp0 = 6;  // warps 6-9: lane quarters 2, 3, 0, 1
constexpr int kTcProducer2Warp = 10;  // the second producer
constexpr float kLazyRescaleLog2 = 8.f;

// ---------------------------------------------------------------- descriptors
// Instruction descriptor of tcgen05.mma.kind::f16 with bf16 A and B and an
// fp32 accumulator (PTX ISA, "Instruction descriptor"): bits 4-5 D format
// (1 = f32), 7-9 A format (1 = bf16), 10-12 B format (1 = bf16), 15 A
// major-ness, 16 B major-ness (0 = K-major, 1 = MN-major), 17-22 N / 8,
// 24-28 M / 16.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int m, int n, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn_major) << 15) |
           (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}
// Shared-memory matrix descriptor (PTX ISA, "Shared memory descriptor"):
// bits 0-13 start address / 16, 16-29 leading-dimension byte offset / 16,
// 32-45 stride-dimension byte offset / 16, 46-47 version (1), 49-51 base
// offset (0: every swizzle atom here starts on a 1024-byte boundary), 61-63
// layout (2 = 128-byte swizzle).
__host__ __device__ constexpr uint64_t umma_sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// The two MMA shapes of this kernel, written out bit by bit.
static_assert(umma_idesc_bf16(128, 64, false, false) == 0x08100490u, "S = Q K^T descriptor");
static_assert(umma_idesc_bf16(128, 128, false, true) == 0x08210490u, "O += P V descriptor");
static_assert(umma_sdesc_sw128(0x1000u, 16u, 1024u) == 0x4000404000010100ull, "K-major operand descriptor");
static_assert(umma_sdesc_sw128(0x2000u, 8192u, 1024u) == 0x4000404002000200ull, "MN-major operand descriptor");

constexpr uint32_t kIdescS = umma_idesc_bf16(kColsTc, kTokTc, false, false);
constexpr uint32_t kIdescPV = umma_idesc_bf16(kColsTc, kD, false, true);

// ---------------------------------------------------------------- operand views
// Byte offsets (from 1024-aligned tile bases) and strides of the four MMA
// operands, k-step kk covering 16 values of the reduction dimension.
constexpr uint32_t kQHalfBytes = kColsTc * 128;  // Q: [dims 0-63 | 64-127][128 columns x 128 B]
constexpr uint32_t kKvQuarterBytes = kTokTc * 128;  // K lo, K hi, V lo, V hi: [64 tokens x 128 B]
constexpr uint32_t kSbo = 1024;                  // 8 rows of 128 B
constexpr uint32_t kLboK = 16;                   // unused by swizzled K-major operands
__host__ __device__ constexpr uint32_t q_step(int kk) { return (kk >> 2) * kQHalfBytes + (kk & 3) * 32; }
__host__ __device__ constexpr uint32_t k_step(int kk) { return (kk >> 2) * kKvQuarterBytes + (kk & 3) * 32; }
__host__ __device__ constexpr uint32_t p_step(int kk) { return kk * 32; }
__host__ __device__ constexpr uint32_t v_step(int kk) { return kk * 16 * 128; }
constexpr uint32_t kLboV = kKvQuarterBytes;      // V's dims 64-127 (V hi) after dims 0-63 (V lo)

// Where the tensor cores read element (mn, k) of a bf16 operand given by a
// 128-byte-swizzle descriptor, in the canonical layouts of the tcgen05
// matrix descriptors (T = 8 bf16 = 16 bytes; CUTLASS cute/atom/
// mma_traits_sm100.hpp, make_umma_desc):
//   K-major  ((8, m), (T, 2)) : ((8T, SBO), (1, T))
//   MN-major ((T, 8, m), (8, k)) : ((1, T, LBO), (8T, SBO))
// followed by the 128-byte swizzle of the address (bits 4-6 ^= bits 7-9).
__host__ __device__ constexpr uint32_t sw128_read(uint32_t start, uint32_t lbo, uint32_t sbo, bool mn_major,
                                                  int mn, int k) {
    const uint32_t off = mn_major ? 2u * (mn % 64) + (mn / 64) * lbo + (k % 8) * 128u + (k / 8) * sbo
                                  : (mn % 8) * 128u + (mn / 8) * sbo + 2u * k;
    const uint32_t a = start + off;
    return a ^ (((a >> 7) & 7u) << 4);
}
// Where the TMA boxes (128-byte swizzle) and swz() put element (row, col) of
// a tile stored as [col / 64][rows x 128 B], `half` bytes apart.
__host__ __device__ constexpr uint32_t sw128_written(uint32_t half, int row, int col) {
    return (col / 64) * half + static_cast<uint32_t>(row * 128 + ((((col % 64) / 8) ^ (row & 7)) << 4)) +
           2u * (col % 8);
}
// Every element each k-step of the four operands reads is the element the
// kernel wrote there: Q[column][dim], K[token][dim], P[column][token],
// V[token][dim] (V read MN-major: mn = dim, k = token).
__host__ __device__ constexpr bool operand_views_agree() {
    for (int kk = 0; kk < kD / 16; ++kk)
        for (int mn = 0; mn < kColsTc; ++mn)
            for (int kl = 0; kl < 16; ++kl) {
                if (sw128_read(q_step(kk), kLboK, kSbo, false, mn, kl) != sw128_written(kQHalfBytes, mn, 16 * kk + kl))
                    return false;
                if (mn < kTokTc &&
                    sw128_read(k_step(kk), kLboK, kSbo, false, mn, kl) != sw128_written(kKvQuarterBytes, mn, 16 * kk + kl))
                    return false;
            }
    for (int kk = 0; kk < kTokTc / 16; ++kk)
        for (int mn = 0; mn < kColsTc; ++mn)
            for (int kl = 0; kl < 16; ++kl) {
                if (sw128_read(p_step(kk), kLboK, kSbo, false, mn, kl) != sw128_written(0, mn, 16 * kk + kl))
                    return false;
                if (sw128_read(v_step(kk), kLboV, kSbo, true, mn, kl) != sw128_written(kKvQuarterBytes, 16 * kk + kl, mn))
                    return false;
            }
    return true;
}
static_assert(operand_views_agree(), "MMA operand descriptors must read what the tiles hold");

// ---------------------------------------------------------------- tcgen05 PTX
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D (tensor memory) = A B (+ D when accumulate != 0); A and B in shared memory.
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D (tensor memory) = A B (+ D); A in tensor memory (K-major: lane = row m,
// 32-bit column j = elements 2j, 2j+1 of the k-step), B in shared memory.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on `bar` when every tcgen05.mma this thread issued so far is complete.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}
// 32 consecutive fp32 columns of this thread's tensor-memory lane, waited for
// in the same statement (so no use of r can be scheduled before the wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st2(uint32_t taddr, uint32_t a, uint32_t b) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void tmem_ld2(uint32_t taddr, uint32_t &a, uint32_t &b) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(a), "=r"(b)
        : "r"(taddr)
        : "memory");
}
// 64 consecutive fp32 columns of this thread's lane, one load and one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

// mbar_wait for warps off the critical path: sleeps between polls so that
// its spinning takes few issue slots from the warps it shares a scheduler
// with; the same time limit.
__device__ __forceinline__ bool mbar_wait_idle(uint64_t *bar, uint32_t parity) {
    const uint32_t addr = smem_addr(bar);
    if (mbar_try_wait(addr, parity))
        return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        __nanosleep(200);
        if (mbar_try_wait(addr, parity))
            return true;
        if (global_ns() - t0 > kWaitLimitNs) {
            flag_error(PA_DEVERR_TIMEOUT);
            return false;
        }
    }
}

// max(a, b, c) in one instruction (the three-input form of max.f32, sm_100).
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// Largest of 8 consecutive values.
__device__ __forceinline__ float max8(const float *x) {
    return fmax3f(fmax3f(x[0], x[1], x[2]), fmax3f(x[3], x[4], x[5]), fmaxf(x[6], x[7]));
}

// 16-byte cp.async that writes zeros when src_bytes is 0.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
// Arrive on `bar` when this thread's cp.async copies so far have landed; the
// pending count is raised first, so the arrival does not count toward the
// barrier's expected count.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

struct AttendTcSmem {
    uint16_t kv[kStagesTc][4][kTokTc * 64];  // [stage][K lo, K hi, V lo, V hi][64 tokens x 64 dims], swizzled
    uint16_t q[2][2][kColsTc * 64];          // [buffer][dims lo, dims hi][128 columns x 64 dims], swizzled
    uint64_t full[kStagesTc];
    uint64_t empty[kStagesTc];
    uint64_t s_full[2];
    uint64_t s_free[2];
    uint64_t p_full[2];
    uint64_t pv_done[2];
    uint64_t q_full[2];
    uint64_t q_empty[2];
    uint64_t o_full[2];
    uint64_t o_free[2];
    uint64_t ml_full[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int32_t blocks[2][kMaxPartBlocksTc];  // each producer's copy of the unit's table slice
};
constexpr size_t kAttendTcSmemBytes = sizeof(AttendTcSmem) + 1024;
static_assert(kAttendTcSmemBytes <= 227 * 1024, "shared memory per CTA");
static_assert(offsetof(AttendTcSmem, q) % 1024 == 0, "swizzle atoms start on 1024-byte boundaries");

// One work unit: (split-K partition, group of HP KV heads, request, chunk of
// 128 / HP columns), numbered as part + P * (group + (Hkv / HP) * (request *
// chunks + chunk)).  Every role derives the same fields from global memory,
// so all agree on which units have work and on their tile counts.
struct TcUnit {
    int part, h, r, chunk;  // h: the head group (KV heads h * HP .. h * HP + HP - 1)
    int q0, n, col0, last_col, first_visible, t_begin, t_end, num_tiles;
    bool bad;   // query_start_loc / seq_lens inconsistent for this request
    bool work;  // at least one tile
};

// n / d for 0 <= n < 2^31 by a multiply-high, an add and a shift, the
// divisor's constants set on the host (the round-up method of Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994):
// with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1, which fits in
// 32 bits, n / d = (umulhi(m, n) + n) >> s.  Every role decodes each work
// unit at its start; the GPU has no integer divide instruction, and the
// emulated division by a runtime divisor is a long dependent chain on the
// path from one unit's last tile to the next unit's first.
struct FastDiv {
    uint32_t d, m, s;
};
inline FastDiv make_fast_div(uint32_t d) {
    uint32_t s = 0;
    while ((uint64_t(1) << s) < d)
        ++s;
    const uint64_t m = ((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1;
    return FastDiv{d, static_cast<uint32_t>(m), s};
}
__device__ __forceinline__ int fast_div(int n, const FastDiv &f) {
    return static_cast<int>((__umulhi(static_cast<uint32_t>(n), f.m) + static_cast<uint32_t>(n)) >> f.s);
}
// The divisors of the unit number: partitions, head groups, column chunks.
struct TcDivs {
    FastDiv parts, groups, chunks;
};

// The unit's raw metadata, loaded one unit ahead so that its latency
// overlaps the current unit's tiles; tc_unit() derives the rest.
struct TcRaw {
    int u, q0, q1, n;
};
__device__ __forceinline__ TcRaw tc_raw(const AttendParams &ap, const TcDivs &dv, int u) {
    TcRaw raw{u, 0, 0, 0};
    if (u < ap.num_units) {
        const int r = fast_div(fast_div(fast_div(u, dv.parts), dv.groups), dv.chunks);
        raw.q0 = ap.query_start_loc[r];
        raw.q1 = ap.query_start_loc[r + 1];
        raw.n = ap.d.seq_lens[r];
    }
    return raw;
}

template <int G, int HP>
__device__ __forceinline__ TcUnit tc_unit(const AttendParams &ap, const TcDivs &dv, const TcRaw &raw) {
    const DecodeParams &p = ap.d;
    TcUnit w{};
    const int u = raw.u;
    int rest = fast_div(u, dv.parts);
    w.part = u - rest * p.num_parts;
    int next = fast_div(rest, dv.groups);
    w.h = rest - next * ap.head_groups;
    w.r = fast_div(next, dv.chunks);
    w.chunk = next - w.r * ap.chunks;
    int n = raw.n;  // clamped as clamp_seq_len does
    {
        const int64_t cap64 = static_cast<int64_t>(p.max_blocks_per_seq) * p.block_size;
        const int cap = static_cast<int>(cap64 < p.max_seq_len ? cap64 : p.max_seq_len);
        if (n < 0 || n > cap) {
            flag_error(PA_DEVERR_SEQ_LEN);
            n = n < 0 ? 0 : cap;
        }
    }
    const int q0 = raw.q0, q1 = raw.q1;
    const int q_len = q1 - q0;
    w.q0 = q0;
    w.n = n;
    w.bad = q_len < 0 || q_len > n || q_len > ap.max_query_len || q0 < 0 || q1 > ap.num_tokens ||
            (w.r == 0 && q0 != 0) || (w.r == p.num_seqs - 1 && q1 != ap.num_tokens);
    if (w.bad)
        return w;
    const int cols = q_len * G;
    w.col0 = w.chunk * (kColsTc / HP);
    if (w.col0 >= cols)
        return w;
    w.last_col = min(cols, w.col0 + kColsTc / HP) - 1;
    w.first_visible = n - q_len;  // row i sees positions <= first_visible + i
    const int lim_max = w.first_visible + w.last_col / G;
    w.t_begin = w.part * p.part_tokens;
    if (w.t_begin > lim_max)
        return w;
    w.t_end = min(lim_max + 1, w.t_begin + p.part_tokens);
    w.num_tiles = (w.t_end - w.t_begin + kTokTc / HP - 1) / (kTokTc / HP);
    w.work = true;
    return w;
}

// Persistent: one CTA per SM walks the work units blockIdx.x, blockIdx.x +
// gridDim.x, ...  Tiles, S buffers and P buffers are counted across units
// (T), so the producer streams the next unit's q tile and K/V tiles while
// the current unit's softmax and epilogue finish.
//
// kZeroScale: the caller's scale is 0, so every visible token weighs 1 and a
// masked one 0; the scaled-score form below would give 0 * inf there.
//
// HP (1 or 2): KV heads per work unit.  With HP = 2 (at most 64 columns per
// head) a tile is 32 tokens of both heads: stage rows 0-31 hold head 2g's K
// (V) rows, rows 32-63 head 2g + 1's, and the q tile holds head 2g's columns
// in MMA rows 0-63 and head 2g + 1's in rows 64-127.  The MMAs are those of
// HP = 1; S's two off-diagonal 64 x 32 blocks (one head's q against the
// other's K) are not read, and each softmax warp writes zeros into the P
// columns of the other head's tokens, so P V adds only a head's own tokens
// into its O rows.  All four softmax warps then have live columns, and a
// 32 KiB stage still feeds one tile, so the ring keeps its depth.
template <int G, bool kZeroScale, int HP>
__global__ void __launch_bounds__(kTcThreads, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const __grid_constant__ CUtensorMap tm_q, const AttendParams ap, const TcDivs dv) {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
    static_assert(HP == 1 || HP == 2, "heads per work unit");
    constexpr int kTokH = kTokTc / HP;   // tokens of one head per tile
    constexpr int kColsH = kColsTc / HP;  // columns of one head per unit
    constexpr unsigned FULL = 0xffffffffu;
    const DecodeParams &p = ap.d;
    extern __shared__ uint8_t smem_raw[];
    AttendTcSmem &sm = *reinterpret_cast<AttendTcSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int B = p.block_size;
    const int Hkv = ap.num_kv_heads;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStagesTc; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.s_free[b], 4);
            mbar_init(&sm.p_full[b], 4);
            mbar_init(&sm.pv_done[b], 1);
            mbar_init(&sm.q_full[b], 1);
            mbar_init(&sm.q_empty[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.o_full[b], 1);
            mbar_init(&sm.o_free[b], 4);
            mbar_init(&sm.ml_full[b], 4);
        }
        mbar_init(&sm.mma_done, 1);
        mbar_init_fence();
    }
    if (warp == kTcProducerWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        if (B >= 8) {
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
        }
    }
    if (warp == kTcMmaWarp) {
        tmem_alloc(&sm.tmem_base, kTmemColsTc);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tmem_o = tmem + kTmemOTc;
    const uint32_t tmem_p = tmem + kTmemPTc;
    grid_dependency_wait();

    if (warp == kTcProducerWarp || warp == kTcProducer2Warp) {
        // ============================================================ producers
        // Producer p fills the ring slots s with s % 2 == p, so each slot has
        // one owner that waits for every phase of it; producer 0 also loads
        // the q tiles.  One warp issuing all 16 boxes of every tile could not
        // keep the stream at the rate two-head tiles are consumed.
        const int pidx = warp == kTcProducer2Warp;
        int32_t *const blocks = sm.blocks[pidx];
        const uint64_t pol = l2_evict_first_policy();
        int T = 0, k = 0;
        bool dead = false;
        TcRaw raw = tc_raw(ap, dv, blockIdx.x);
        for (int u = blockIdx.x; u < ap.num_units && !dead; u += gridDim.x) {
            const TcUnit w = tc_unit<G, HP>(ap, dv, raw);
            raw = tc_raw(ap, dv, u + gridDim.x);
            if (w.bad && w.part == 0 && w.h == 0 && w.chunk == 0 && lane == 0)
                flag_error(PA_DEVERR_QUERY_LOC);
            if (!w.work)
                continue;
            // the unit's slice of the block table (only this warp reads it)
            const int first_blk = w.t_begin / B;
            __syncwarp();
            {
                const int32_t *row = p.block_tables + static_cast<int64_t>(w.r) * p.max_blocks_per_seq + first_blk;
                const int nblk = (w.t_end - 1) / B - first_blk + 1;
                for (int i = lane; i < nblk; i += 32) {
                    int32_t b = __ldg(row + i);
                    if (b < 0 || b >= p.num_blocks) {
                        flag_error(PA_DEVERR_BLOCK_ID);
                        b = 0;
                    }
                    blocks[i] = b;
                }
            }
            __syncwarp();
            // the unit's q tile, both 64-dim halves, as two boxes of 64 columns
            // each: MMA rows 0-63 and 64-127 are columns col0 .. and col0 + 64 ..
            // of the unit's head (HP = 1) or columns col0 .. of its first and
            // second head (HP = 2); column c of head h is q row q0 + c / G, head
            // h G + c % G.  Rows past the request hold other rows or zeros
            // (their columns are masked).
            const int qb = k & 1;
            if (pidx == 0 && k >= 2) {
                bool ok = true;
                if (lane == 0)
                    ok = mbar_wait(&sm.q_empty[qb], ((k >> 1) - 1) & 1);
                if (!__shfl_sync(FULL, ok, 0)) {
                    dead = true;
                    break;
                }
            }
            if (pidx == 0 && lane == 0) {
                mbar_arrive_expect_tx(&sm.q_full[qb], static_cast<uint32_t>(2 * kColsTc * 128));
#pragma unroll
                for (int d = 0; d < 2; ++d)
#pragma unroll
                    for (int rb = 0; rb < 2; ++rb) {
                        const int head = w.h * HP + (HP == 2 ? rb : 0);
                        const int qrow = w.q0 + (w.col0 + (HP == 1 ? rb * 64 : 0)) / G;
                        tma_load_3d(&sm.q[qb][d][rb * 64 * 64], &tm_q, d * 64, head * G, qrow, &sm.q_full[qb], pol);
                    }
            }
            for (int it = 0; it < w.num_tiles; ++it, ++T) {
                const int slot = T % kStagesTc;
                if ((slot & 1) != pidx)
                    continue;
                if (T >= kStagesTc) {
                    bool ok = true;
                    if (lane == 0)
                        ok = mbar_wait(&sm.empty[slot], ((T / kStagesTc) + 1) & 1);
                    if (!__shfl_sync(FULL, ok, 0)) {
                        dead = true;
                        break;
                    }
                }
                // stage row hh * kTokH + i holds token t0 + i of head w.h * HP + hh
                const int t0 = w.t_begin + it * kTokH;
                const int ntok = min(kTokH, w.t_end - t0);
                if (B >= 8 && ntok == kTokH) {
                    // whole tile by TMA: boxes of min(B, 16) rows, 4 quarters each,
                    // per head
                    const int rows = B < kTile ? B : kTile;
                    const int nbox = kTokH / rows;  // HP * nbox * 4 <= 32 lanes
                    if (lane == 0)
                        mbar_arrive_expect_tx(&sm.full[slot], static_cast<uint32_t>(kTokTc * 128 * 4));
                    __syncwarp();
                    // box j of head hh of quarter qd (K lo, K hi, V lo, V hi)
                    const int qd = lane & 3, j = (lane >> 2) % nbox, hh = (lane >> 2) / nbox;
                    if (hh < HP) {
                        const int t = t0 + j * rows;
                        const int32_t rr = blocks[t / B - first_blk] * B + (t % B);
                        tma_load_3d(&sm.kv[slot][qd][(hh * kTokH + j * rows) * 64], (qd < 2) ? &tm_k : &tm_v,
                                    (qd & 1) * 64, w.h * HP + hh, rr, &sm.full[slot], pol);
                    }
                } else {
                    // gather: lane = (quarter, 16-byte chunk); rows past the range
                    // are zero-filled so that 0-weight V rows stay finite
                    const int qd = lane >> 3, ch = lane & 7;
                    const uint16_t *cache = static_cast<const uint16_t *>(qd < 2 ? p.k_cache : p.v_cache);
                    int64_t slot_lo = 0, slot_hi = 0;  // cache slots of tokens t0 + lane, t0 + lane + 32
                    if (lane < ntok) {
                        const int t = t0 + lane;
                        slot_lo = static_cast<int64_t>(blocks[t / B - first_blk]) * B + (t % B);
                    }
                    if (lane + 32 < ntok) {
                        const int t = t0 + lane + 32;
                        slot_hi = static_cast<int64_t>(blocks[t / B - first_blk]) * B + (t % B);
                    }
                    const uint32_t base = smem_addr(&sm.kv[slot][qd][0]);
                    for (int i = 0; i < kTokTc; ++i) {
                        const int hh = i / kTokH, tt = i % kTokH;
                        const int64_t sl = __shfl_sync(FULL, tt < 32 ? slot_lo : slot_hi, tt & 31);
                        const bool in = tt < ntok;
                        const int64_t rr = sl * Hkv + w.h * HP + hh;
                        cp_async16_zfill(base + swz(i, ch), cache + (in ? rr * kD + (qd & 1) * 64 + ch * 8 : 0),
                                         in ? 16u : 0u);
                    }
                    cp_async_mbar_arrive(&sm.full[slot]);
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&sm.full[slot]);
                }
            }
            ++k;
        }
        // nothing may still be copying into shared memory when the CTA ends
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0) {
            for (int sl = pidx; sl < kStagesTc && sl < T; sl += 2) {
                const int last = sl + ((T - 1 - sl) / kStagesTc) * kStagesTc;
                mbar_wait(&sm.full[sl], (last / kStagesTc) & 1);
            }
            for (int b = 0; b < 2 && b < k && pidx == 0; ++b) {
                const int last = b + ((k - 1 - b) / 2) * 2;
                mbar_wait(&sm.q_full[b], (last >> 1) & 1);
            }
        }
    } else if (warp == kTcMmaWarp) {
        // ============================================================ MMA issue
        if (lane == 0) {
            // P V of tile pt (the first / last of its unit when first / last;
            // unit index pk) into the O buffer of its unit: the first one
            // overwrites it, after the epilogue warps have read unit pk - 2's O
            // from it; the last one's completion hands it to the epilogue warps
            auto pv = [&](int pt, bool first, bool last, int pk) -> bool {
                const int ob = pk & 1;
                if (!mbar_wait(&sm.p_full[pt & 1], (pt >> 1) & 1))
                    return false;
                if (first && pk >= 2 && !mbar_wait(&sm.o_free[ob], ((pk >> 1) - 1) & 1))
                    return false;
                tc_fence_after();
                const uint32_t v_base = smem_addr(&sm.kv[pt % kStagesTc][2][0]);
#pragma unroll
                for (int kk = 0; kk < kTokTc / 16; ++kk)
                    umma_bf16_ts(tmem_o + ob * kD, tmem_p + (pt & 1) * 32 + kk * 8,
                                 umma_sdesc_sw128(v_base + v_step(kk), kLboV, kSbo), kIdescPV,
                                 (!first || kk > 0) ? 1u : 0u);
                umma_commit(&sm.pv_done[pt & 1]);
                umma_commit(&sm.empty[pt % kStagesTc]);
                if (last)
                    umma_commit(&sm.o_full[ob]);
                return true;
            };
            bool ok = true;
            int T = 0, k = 0;
            int prev_t = -1, prev_k = 0;
            bool prev_first = false, prev_last = false;
            TcRaw raw = tc_raw(ap, dv, blockIdx.x);
            for (int u = blockIdx.x; u < ap.num_units && ok; u += gridDim.x) {
                const TcUnit w = tc_unit<G, HP>(ap, dv, raw);
                raw = tc_raw(ap, dv, u + gridDim.x);
                if (!w.work)
                    continue;
                const int qb = k & 1;
                ok = mbar_wait(&sm.q_full[qb], (k >> 1) & 1);
                const uint32_t q_base = smem_addr(&sm.q[qb][0][0]);
                for (int t = 0; t < w.num_tiles && ok; ++t, ++T) {
                    const int slot = T % kStagesTc;
                    ok = mbar_wait(&sm.full[slot], (T / kStagesTc) & 1);
                    if (ok && T >= 2)
                        ok = mbar_wait(&sm.s_free[T & 1], ((T >> 1) - 1) & 1);
                    if (!ok)
                        break;
                    // a gathered stage was written by cp.async (generic proxy);
                    // the tensor cores read it through the async proxy
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t k_base = smem_addr(&sm.kv[slot][0][0]);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk)
                        umma_bf16_ss(tmem + (T & 1) * kTokTc, umma_sdesc_sw128(q_base + q_step(kk), kLboK, kSbo),
                                     umma_sdesc_sw128(k_base + k_step(kk), kLboK, kSbo), kIdescS, kk > 0 ? 1u : 0u);
                    umma_commit(&sm.s_full[T & 1]);
                    if (t == w.num_tiles - 1)
                        umma_commit(&sm.q_empty[qb]);  // the unit's last S read of this q buffer
                    if (prev_t >= 0)
                        ok = pv(prev_t, prev_first, prev_last, prev_k);
                    prev_t = T;
                    prev_first = t == 0;
                    prev_last = t == w.num_tiles - 1;
                    prev_k = k;
                }
                ++k;
            }
            if (ok && prev_t >= 0)
                pv(prev_t, prev_first, prev_last, prev_k);
            // everything issued above has completed before the allocation is freed
            umma_commit(&sm.mma_done);
            mbar_wait(&sm.mma_done, 0);
        }
        __syncwarp();
    } else if (warp >= kTcEpilogueWarp0 && warp < kTcEpilogueWarp0 + 4) {
        // ============================================================ epilogue
        // Warp 6 + i reads lane quarter (6 + i) % 4 of unit k's O buffer once
        // the unit's last P V has completed and the softmax warps have left
        // (m_ref, l), writes the output rows (or the split-K partials), and
        // frees the buffer; the softmax warps meanwhile work on unit k + 1.
        const int quarter = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        bool ok = true;
        int k = 0;
        TcRaw raw = tc_raw(ap, dv, blockIdx.x);
        for (int u = blockIdx.x; u < ap.num_units && ok; u += gridDim.x) {
            const TcUnit w = tc_unit<G, HP>(ap, dv, raw);
            raw = tc_raw(ap, dv, u + gridDim.x);
            if (!w.work)
                continue;
            const int ob = k & 1;
            if (lane == 0) {
                ok = mbar_wait_idle(&sm.o_full[ob], (k >> 1) & 1);
                if (ok)
                    ok = mbar_wait_idle(&sm.ml_full[ob], (k >> 1) & 1);
            }
            ok = __shfl_sync(FULL, ok, 0);
            if (!ok)
                break;
            tc_fence_after();
            const int hh = (quarter * 32) / kColsH;  // the unit's head of these rows
            const int c = w.col0 + (quarter * 32 + lane) % kColsH;
            const int lim = c <= w.last_col ? w.first_visible + c / G : -1;
            const bool warp_live = __any_sync(FULL, lim >= w.t_begin);
            if (warp_live) {
                uint32_t mr, lr;
                tmem_ld2(tmem + kTmemMlTc + 2 * ob + lane_base, mr, lr);
                const float m_ref = __uint_as_float(mr), l = __uint_as_float(lr);
                const bool valid = c <= w.last_col;
                const int64_t qrow = valid ? w.q0 + c / G : 0;
                const int j = (w.h * HP + hh) * G + c % G;
#pragma unroll 1
                for (int cc = 0; cc < kD / 32; ++cc) {
                    uint32_t o[32];
                    __syncwarp();  // the load is warp-collective
                    tmem_ld32(tmem_o + ob * kD + lane_base + cc * 32, o);
                    if (!valid) {
                    } else if (p.num_parts == 1) {
                        const float inv = l > 0.f ? 1.f / l : 0.f;
                        uint4 *dst = reinterpret_cast<uint4 *>(p.out + (qrow * p.num_q_heads + j) * kD + cc * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(o[8 * q4 + 0]) * inv, __uint_as_float(o[8 * q4 + 1]) * inv);
                            v.y = pack_bf16x2(__uint_as_float(o[8 * q4 + 2]) * inv, __uint_as_float(o[8 * q4 + 3]) * inv);
                            v.z = pack_bf16x2(__uint_as_float(o[8 * q4 + 4]) * inv, __uint_as_float(o[8 * q4 + 5]) * inv);
                            v.w = pack_bf16x2(__uint_as_float(o[8 * q4 + 6]) * inv, __uint_as_float(o[8 * q4 + 7]) * inv);
                            dst[q4] = v;
                        }
                    } else {
                        const int64_t idx = (qrow * p.num_q_heads + j) * p.num_parts + w.part;
                        float4 *dst = reinterpret_cast<float4 *>(p.part_acc + idx * kD + cc * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            dst[q4] = make_float4(__uint_as_float(o[4 * q4]), __uint_as_float(o[4 * q4 + 1]),
                                                  __uint_as_float(o[4 * q4 + 2]), __uint_as_float(o[4 * q4 + 3]));
                        if (cc == 0)
                            p.part_ml[idx] = make_float2(m_ref, l);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.o_free[ob]);
            ++k;
        }
    } else {
        // ============================================================ softmax
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const int hh = (warp * 32) / kColsH;  // the unit's head of this warp's columns
        if constexpr (HP == 2) {
            // the P columns of the other head's tokens stay zero in these lanes
            uint32_t z[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                z[j] = 0u;
            tmem_st16(tmem_p + lane_base + (1 - hh) * 16, z);
            tmem_st16(tmem_p + lane_base + 32 + (1 - hh) * 16, z);
            tmem_st_wait();
        }
        // score multiplier (log2 domain) with the scale's sign; masked tokens
        // are set to the value that the multiplier sends to -inf
        const float sl2 = p.scale_log2;
        const bool pos = sl2 >= 0.f;
        const float masked = pos ? -INFINITY : INFINITY;
        bool ok = true;
        int T = 0, k = 0;
        TcRaw raw = tc_raw(ap, dv, blockIdx.x);
        for (int u = blockIdx.x; u < ap.num_units && ok; u += gridDim.x) {
            const TcUnit w = tc_unit<G, HP>(ap, dv, raw);
            raw = tc_raw(ap, dv, u + gridDim.x);
            if (!w.work)
                continue;
            const int c = w.col0 + threadIdx.x % kColsH;
            const int lim = c <= w.last_col ? w.first_visible + c / G : -1;  // last position column c sees
            const bool warp_live = __any_sync(FULL, lim >= w.t_begin);
            if (p.num_parts > 1 && w.part == 0 && w.h == 0 && warp == 0) {
                for (int i = w.col0 / G + lane; i <= w.last_col / G; i += 32)
                    ap.row_len[w.q0 + i] = w.first_visible + i + 1;
            }
            float m_ref = -INFINITY, l = 0.f;
            for (int t = 0; t < w.num_tiles; ++t, ++T) {
                if (lane == 0)
                    ok = mbar_wait(&sm.s_full[T & 1], (T >> 1) & 1);
                if (!__shfl_sync(FULL, ok, 0))
                    break;
                tc_fence_after();
                const int t0 = w.t_begin + t * kTokH;
                const int ntok = min(kTokH, w.t_end - t0);
                const int jcount = max(0, min(ntok, lim - t0 + 1));  // tokens of this tile column c sees
                // raw scores of this head's tokens (S columns hh * kTokH ..);
                // tokens column c does not see get `masked`
                float x[kTokH];
                if (warp_live) {
                    uint32_t s[kTokH];
                    if constexpr (HP == 1)
                        tmem_ld64(tmem + lane_base + (T & 1) * kTokTc, s);
                    else
                        tmem_ld32(tmem + lane_base + (T & 1) * kTokTc + hh * kTokH, s);
                    if (jcount == kTokH) {
#pragma unroll
                        for (int j = 0; j < kTokH; ++j)
                            x[j] = __uint_as_float(s[j]);
                    } else {
#pragma unroll
                        for (int j = 0; j < kTokH; ++j)
                            x[j] = j < jcount ? __uint_as_float(s[j]) : masked;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.s_free[T & 1]);
                // the P buffer of this tile was last read by P V of tile T - 2
                if (T >= 2) {
                    if (lane == 0)
                        ok = mbar_wait(&sm.pv_done[T & 1], ((T >> 1) - 1) & 1);
                    if (!__shfl_sync(FULL, ok, 0))
                        break;
                }
                if (warp_live) {
                    // the tile's max of sl2 * x in the log2 domain: the max of x
                    // scaled, or with a negative scale the min of x
                    constexpr int NG = kTokH / 8;
                    float m8[NG];
                    float mt;
                    if (kZeroScale) {
                        mt = jcount > 0 ? 0.f : -INFINITY;
                    } else if (pos) {
#pragma unroll
                        for (int i = 0; i < NG; ++i)
                            m8[i] = max8(&x[8 * i]);
                        if constexpr (NG == 8)
                            mt = sl2 * fmax3f(fmax3f(m8[0], m8[1], m8[2]), fmax3f(m8[3], m8[4], m8[5]),
                                              fmaxf(m8[6], m8[7]));
                        else
                            mt = sl2 * fmax3f(m8[0], m8[1], fmaxf(m8[2], m8[3]));
                    } else {
#pragma unroll
                        for (int i = 0; i < NG; ++i) {
                            float v = x[8 * i];
#pragma unroll
                            for (int j = 1; j < 8; ++j)
                                v = fminf(v, x[8 * i + j]);
                            m8[i] = v;
                        }
                        float v = m8[0];
#pragma unroll
                        for (int i = 1; i < NG; ++i)
                            v = fminf(v, m8[i]);
                        mt = sl2 * v;
                    }
                    float alpha = 1.f;
                    bool rescale = false;
                    if (mt > m_ref + kLazyRescaleLog2) {  // false while the column has seen nothing
                        if (m_ref != -INFINITY) {
                            alpha = exp2_approx(m_ref - mt);
                            rescale = true;
                        }
                        m_ref = mt;
                    }
                    l *= alpha;
                    if (__any_sync(FULL, rescale)) {
                        // O must hold P V of tile T - 1 (of this unit: t >= 1) before it is scaled
                        if (lane == 0)
                            ok = mbar_wait(&sm.pv_done[(T - 1) & 1], ((T - 1) >> 1) & 1);
                        if (!__shfl_sync(FULL, ok, 0))
                            break;
                        tc_fence_after();
#pragma unroll 1
                        for (int cc = 0; cc < kD / 32; ++cc) {
                            uint32_t o[32];
                            tmem_ld32(tmem_o + (k & 1) * kD + lane_base + cc * 32, o);
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                            tmem_st32(tmem_o + (k & 1) * kD + lane_base + cc * 32, o);
                        }
                        tmem_st_wait();
                    }
                    // P row: 2^(sl2 x - m_ref), one FMA and one exp2 per token;
                    // 0 where masked.  While the column has seen nothing,
                    // m_ref is -inf: the offset 0 keeps the FMA at -inf.
                    const float neg = m_ref != -INFINITY ? -m_ref : 0.f;
                    uint32_t pw[kTokH / 2];  // this head's tokens as bf16 pairs
                    float lsum = 0.f;
#pragma unroll
                    for (int kq = 0; kq < kTokH / 8; ++kq) {
                        float e[8];
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            e[v] = kZeroScale ? (8 * kq + v < jcount ? 1.f : 0.f)
                                              : exp2_approx(fmaf(x[8 * kq + v], sl2, neg));
                        lsum += ((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7]));
                        pw[4 * kq + 0] = pack_bf16x2(e[0], e[1]);
                        pw[4 * kq + 1] = pack_bf16x2(e[2], e[3]);
                        pw[4 * kq + 2] = pack_bf16x2(e[4], e[5]);
                        pw[4 * kq + 3] = pack_bf16x2(e[6], e[7]);
                    }
                    if constexpr (HP == 1)
                        tmem_st32(tmem_p + lane_base + (T & 1) * 32, pw);
                    else
                        tmem_st16(tmem_p + lane_base + (T & 1) * 32 + hh * 16, pw);
                    tmem_st_wait();
                    l += lsum;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sm.p_full[T & 1]);
            }
            // ---- end of unit: hand this column's (m_ref, l) to the epilogue
            // warps through tensor memory (its slot of unit k - 2 read first)
            const int ob = k & 1;
            if (ok && k >= 2 && lane == 0)
                ok = mbar_wait(&sm.o_free[ob], ((k >> 1) - 1) & 1);
            ok = __shfl_sync(FULL, ok, 0);
            if (!ok)
                break;
            tc_fence_after();
            tmem_st2(tmem + kTmemMlTc + 2 * ob + lane_base, __float_as_uint(m_ref), __float_as_uint(l));
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sm.ml_full[ob]);
            ++k;
        }
        if (threadIdx.x == 0)
            grid_launch_dependents();
    }
    // every role is done with tensor memory before it is freed
    tc_fence_before();
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemColsTc);
    }
}

}  // namespace pa
