// C ABI of the paged-KV decode path (declared in include/pa.h): argument
// validation, launch configuration, TMA descriptor encoding, device error
// word.  One translation unit so that the device error word is a single
// symbol without relocatable device code.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "attend.cuh"
#include "attend_tc.cuh"
#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_fp8.cuh"
#include "kv_ops.cuh"
#include "pa.h"
#include "pa_device.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "";
// Process-wide knobs (pa_decode_set_*); atomics so that a setter on one host
// thread and a call on another do not race.  A call reads each knob once.
std::atomic<int32_t> g_part_tokens_override{0};
std::atomic<int32_t> g_decode_kernel{PA_DECODE_KERNEL_MMA};
std::atomic<int32_t> g_attention_kernel{PA_ATTENTION_KERNEL_AUTO};


int cuda_fail(cudaError_t e, const char *what) {
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", what, cudaGetErrorString(e));
    return PA_ECUDA;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cache(const pa_cache_t *c) {
    if (!c || !c->k_cache || !c->v_cache || c->num_blocks <= 0 || c->num_kv_heads <= 0)
        return PA_EINVAL;
    if (c->head_dim != pa::kD || c->num_kv_heads > 65535)  // heads: a grid dimension, and int row sizes
        return PA_EUNSUPPORTED;
    const int32_t b = c->block_size;
    if (b < 1 || b > 64 || (b & (b - 1)) != 0)
        return PA_EUNSUPPORTED;
    // TMA row coordinates are int32.
    if (c->num_blocks * static_cast<int64_t>(b) > INT32_MAX)
        return PA_EUNSUPPORTED;
    if (!aligned16(c->k_cache) || !aligned16(c->v_cache))
        return PA_EUNSUPPORTED;
    return PA_OK;
}

// SM count of the current device, read once per device through the CUDA
// runtime.  If no device can be queried (a host without a GPU), 148 (B200)
// is assumed and the runtime error the failed query recorded is cleared, so
// that the caller's next error check does not see it.  A host-side call that
// reaches this function (the workspace sizes, the launch shapes) may thereby
// clear a runtime error the caller left pending on this thread.
int sm_count() {
    static std::atomic<int> cached[64] = {};
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    if (dev >= 0 && dev < 64 && (n = cached[dev].load(std::memory_order_relaxed)) > 0)
        return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    if (dev >= 0 && dev < 64)
        cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Unique id of the calling thread's current CUDA context, 0 when there is
// none or it cannot be read.  Ids are never reused within a process, so
// per-device set-up cached under the id is redone after the device's
// primary context is destroyed and created anew (cudaDeviceReset), which
// reloads this library's module and resets kernel attributes.
unsigned long long current_ctx_id() {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Tokens per split-K partition.  One CTA streams its partition at roughly
// 0.7 us per 16-token tile on B200 (a few tiles in flight per CTA), so the
// longest partition bounds the kernel's duration whatever the batch looks
// like: the host only knows max_seq_len, not how lengths are spread.  The
// partition is therefore kept near 640 tokens (one partition for chat-length
// sequences; 8 x {32K, 8K} measured at 83% of the HBM copy bandwidth with
// 640 against 70% with 1792), and grows only when even that would launch
// more than ~16 CTAs per resident slot for max-length sequences (bounding
// the merge work and the workspace).  A multiple of 64 (so of the tile and
// of every block size), and at most the per-CTA table capacity.
int32_t choose_part_tokens(int32_t num_seqs, int32_t num_kv_heads, int32_t max_seq_len,
                           int32_t block_size, bool tensor_core_kernel) {
    const int64_t max_blocks = tensor_core_kernel ? pa::kMaxPartBlocksM : pa::kMaxPartBlocks;
    const int64_t cap = max_blocks * block_size;
    int64_t part;
    const int32_t override_tokens = g_part_tokens_override.load(std::memory_order_relaxed);
    if (override_tokens > 0) {
        part = override_tokens;
    } else {
        const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads;
        const int64_t slots = static_cast<int64_t>(sm_count()) *
                              (tensor_core_kernel ? pa::kMmaCtasPerSm : pa::kDecodeCtasPerSm);
        const int64_t len = max_seq_len > 0 ? max_seq_len : 1;
        part = std::max<int64_t>(640, (len * units + 16 * slots - 1) / (16 * slots));
        if (part >= len)
            part = len;  // a single partition: no merge
    }
    part = round_up(std::max<int64_t>(part, 64), 64);
    if (part > cap)
        part = cap / 64 * 64;
    return static_cast<int32_t>(part);
}

struct WorkspaceLayout {
    int32_t part_tokens, num_parts;
    size_t ml_bytes, acc_offset, total;
};

bool decode_kernel_is_mma() { return g_decode_kernel.load(std::memory_order_relaxed) == PA_DECODE_KERNEL_MMA; }
// The pa_attention kernel for a call with these columns per request
// (max_query_len x group size): the knob, or under PA_ATTENTION_KERNEL_AUTO
// the tcgen05 kernel from PA_ATTENTION_TCGEN05_MIN_COLUMNS columns on.
bool attention_kernel_is_tcgen05(int64_t columns) {
    const int32_t k = g_attention_kernel.load(std::memory_order_relaxed);
    return k == PA_ATTENTION_KERNEL_TCGEN05 ||
           (k == PA_ATTENTION_KERNEL_AUTO && columns >= PA_ATTENTION_TCGEN05_MIN_COLUMNS);
}

WorkspaceLayout workspace_layout(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t max_seq_len, int32_t block_size, bool tensor_core_kernel) {
    WorkspaceLayout w{};
    w.part_tokens = choose_part_tokens(num_seqs, num_kv_heads, max_seq_len, block_size, tensor_core_kernel);
    w.num_parts = max_seq_len > 0 ? static_cast<int32_t>((max_seq_len + w.part_tokens - 1) / w.part_tokens) : 1;
    if (w.num_parts <= 1) {
        w.num_parts = 1;
        return w;
    }
    const size_t units = static_cast<size_t>(num_seqs) * num_q_heads * w.num_parts;
    w.ml_bytes = units * sizeof(float2);
    w.acc_offset = static_cast<size_t>(round_up(static_cast<int64_t>(w.ml_bytes), 256));
    w.total = w.acc_offset + units * pa::kD * sizeof(float);
    return w;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 3-D view of one cache tensor: (dim, kv head, slot).  CUDA-core kernel:
// box (128, 1, min(B, 16)), no swizzle.  Tensor-core kernel: box (64, 1,
// min(B, 16)) with the 128-byte swizzle, loaded as two 64-dim halves.
int encode_cache_map(CUtensorMap *tm, void *base, const pa_cache_t *c, bool swizzled, bool fp8 = false) {
    auto fn = encode_fn();
    if (!fn) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled unavailable");
        return PA_ECUDA;
    }
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(c->head_dim),
                                static_cast<cuuint64_t>(c->num_kv_heads),
                                static_cast<cuuint64_t>(c->num_blocks) * c->block_size};
    const cuuint64_t esz = fp8 ? 1 : 2;
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(c->head_dim) * esz,
                                   static_cast<cuuint64_t>(c->num_kv_heads) * c->head_dim * esz};
    // one row of the box is at most 128 bytes under the 128-byte swizzle
    const cuuint32_t inner = swizzled ? static_cast<cuuint32_t>(128 / esz) : static_cast<cuuint32_t>(c->head_dim);
    // box height: one block, at most one tile (16 tokens of bf16, 32 of fp8)
    const int32_t tile = fp8 ? pa::kTileF : pa::kTile;
    const cuuint32_t box[3] = {inner, 1u, static_cast<cuuint32_t>(c->block_size < tile ? c->block_size : tile)};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(tm, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims,
                    strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled failed (%d)",
                      static_cast<int>(r));
        return PA_ECUDA;
    }
    return PA_OK;
}

// Every kernel of the library is launched with programmatic stream
// serialization: its CTAs may become resident while the preceding kernel of
// the stream is finishing, and each kernel waits for that kernel (to complete
// and flush) before it reads or writes global memory (griddepcontrol.wait),
// so stream order is kept.  What overlaps is launch latency and set-up.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Per-device record of the context a one-time set-up was done in.
using CtxDone = std::atomic<unsigned long long>[64];

// Opt a kernel into its dynamic shared memory and the all-shared carveout
// (so that its CTAs-per-SM target fits), once per device and context.
template <typename K>
int prepare_kernel(K kernel, size_t smem, CtxDone &done) {
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long ctx = current_ctx_id();
    if (ctx != 0 && dev >= 0 && dev < 64 && done[dev].load(std::memory_order_acquire) == ctx)
        return PA_OK;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute(max dynamic smem)");
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute(carveout)");
    if (dev >= 0 && dev < 64)  // the context the attributes were set in (setting them twice is harmless)
        done[dev].store(current_ctx_id(), std::memory_order_release);
    return PA_OK;
}

template <int G>
int launch_decode_g(const CUtensorMap &tk, const CUtensorMap &tv, const pa::DecodeParams &p,
                    int32_t num_kv_heads, bool mma, cudaStream_t stream) {
    dim3 grid(p.num_parts, num_kv_heads, p.num_seqs);
    if (mma) {
        // Three consumer warps for multi-wave grids of ragged work, two
        // otherwise (see decode_mma.cuh).  With at most 16 partitions per
        // sequence, sequences of varied length leave many short CTAs whose
        // latency sets the waves (block-size sweeps on B200: +9-11% with
        // three); with more, nearly every CTA is a full partition and two
        // warps stream best (32K context on B200: 3% slower with three).  A
        // one-wave grid has every CTA resident from the start: two warps.
        const int64_t ctas = static_cast<int64_t>(grid.x) * grid.y * grid.z;
        const bool one_wave = ctas <= static_cast<int64_t>(sm_count()) * pa::kMmaCtasPerSm;
        const bool two = one_wave || p.num_parts > 16;
        static CtxDone done2 = {}, done3 = {};
        int rc = two ? prepare_kernel(pa::decode_partition_mma_kernel<G, 2>, pa::kDecodeSmemBytesM, done2)
                     : prepare_kernel(pa::decode_partition_mma_kernel<G, 3>, pa::kDecodeSmemBytesM, done3);
        if (rc)
            return rc;
        cudaError_t e = two ? launch_pdl(pa::decode_partition_mma_kernel<G, 2>, grid, dim3(pa::mma_threads<2>()),
                                         pa::kDecodeSmemBytesM, stream, tk, tv, p)
                            : launch_pdl(pa::decode_partition_mma_kernel<G, 3>, grid, dim3(pa::mma_threads<3>()),
                                         pa::kDecodeSmemBytesM, stream, tk, tv, p);
        if (e != cudaSuccess)
            return cuda_fail(e, "decode_partition_mma_kernel launch");
    } else {
        static CtxDone done = {};
        int rc = prepare_kernel(pa::decode_partition_kernel<G>, pa::kDecodeSmemBytes, done);
        if (rc)
            return rc;
        cudaError_t e = launch_pdl(pa::decode_partition_kernel<G>, grid, dim3(pa::kDecodeThreads),
                                   pa::kDecodeSmemBytes, stream, tk, tv, p);
        if (e != cudaSuccess)
            return cuda_fail(e, "decode_partition_kernel launch");
    }
    if (p.num_parts > 1) {
        cudaError_t e = launch_pdl(pa::decode_merge_kernel, dim3(p.num_q_heads, p.num_seqs, 1), dim3(pa::kD),
                                   0, stream, p);
        if (e != cudaSuccess)
            return cuda_fail(e, "decode_merge_kernel launch");
    }
    return PA_OK;
}

}  // namespace

namespace {
// pa_attention's grid and scratch: column chunks per request, the split-K
// partition (same heuristic as decode, over requests x chunks), and the
// (m, l), acc and per-row length arrays when there is more than one
// partition.
struct AttendLayout {
    bool tcgen05;  // attend_tc_kernel, else attend_partition_kernel
    int32_t heads_per_unit;  // attend_tc_kernel: 2 KV heads per work unit when each has <= 64 columns
    int32_t warps, chunks, part_tokens, num_parts;
    size_t acc_offset, len_offset, total;
};

AttendLayout attend_layout(int32_t num_reqs, int32_t num_tokens, int32_t max_query_len, int32_t num_q_heads,
                           int32_t num_kv_heads, int32_t max_seq_len, int32_t block_size, bool tcgen05) {
    AttendLayout a{};
    a.tcgen05 = tcgen05;
    const int64_t G = num_q_heads / num_kv_heads;
    const int64_t cols = static_cast<int64_t>(max_query_len) * G;
    a.heads_per_unit = tcgen05 && cols <= pa::kColsTc / 2 && num_kv_heads % 2 == 0 ? 2 : 1;
    a.warps = cols <= 16 ? 2 : 4;  // CTA shape: 16 columns x 4 CTAs/SM, or 32 columns x 2 CTAs/SM
    const int64_t per_cta = tcgen05 ? pa::kColsTc / a.heads_per_unit : 8 * a.warps;
    a.chunks = static_cast<int32_t>(std::max<int64_t>(1, (cols + per_cta - 1) / per_cta));
    const int64_t units = std::min<int64_t>(INT32_MAX, static_cast<int64_t>(num_reqs) * a.chunks);
    a.part_tokens = choose_part_tokens(static_cast<int32_t>(units), num_kv_heads, max_seq_len, block_size, true);
    if (tcgen05)  // its table holds fewer entries
        a.part_tokens = std::min<int32_t>(a.part_tokens, pa::kMaxPartBlocksTc * block_size / 64 * 64);
    a.num_parts = max_seq_len > 0 ? (max_seq_len + a.part_tokens - 1) / a.part_tokens : 1;
    if (a.num_parts <= 1) {
        a.num_parts = 1;
        return a;
    }
    const size_t cells = static_cast<size_t>(num_tokens) * num_q_heads * a.num_parts;
    a.acc_offset = static_cast<size_t>(round_up(static_cast<int64_t>(cells * sizeof(float2)), 256));
    a.len_offset = static_cast<size_t>(round_up(static_cast<int64_t>(a.acc_offset + cells * pa::kD * sizeof(float)), 256));
    a.total = a.len_offset + static_cast<size_t>(num_tokens) * sizeof(int32_t);
    return a;
}

// Split-K: merge the partitions of each query row, with its visible length
// as that row's sequence length.
int launch_row_merge(const pa::AttendParams &ap, cudaStream_t stream) {
    if (ap.d.num_parts <= 1)
        return PA_OK;
    pa::DecodeParams md = ap.d;
    md.seq_lens = ap.row_len;
    md.num_seqs = ap.num_tokens;
    const cudaError_t e = launch_pdl(pa::decode_merge_kernel, dim3(md.num_q_heads, std::min(ap.num_tokens, 65535), 1),
                                     dim3(pa::kD), 0, stream, md);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "decode_merge_kernel launch");
}

template <int G, int W>
int launch_attend_g(const CUtensorMap &tk, const CUtensorMap &tv, const pa::AttendParams &ap, int32_t num_kv_heads,
                    cudaStream_t stream) {
    static CtxDone done = {};
    constexpr size_t smem = pa::attend_smem_bytes<W>();
    int rc = prepare_kernel(pa::attend_partition_kernel<G, W>, smem, done);
    if (rc)
        return rc;
    const dim3 grid(ap.d.num_parts, num_kv_heads, ap.d.num_seqs * ap.chunks);
    cudaError_t e = launch_pdl(pa::attend_partition_kernel<G, W>, grid, dim3(pa::attend_threads<W>()), smem,
                               stream, tk, tv, ap);
    if (e != cudaSuccess)
        return cuda_fail(e, "attend_partition_kernel launch");
    return launch_row_merge(ap, stream);
}

// The q rows as a 3-D tensor (dim, head, row) for the tcgen05 kernel's TMA
// loads of its q tiles: boxes of (64 dims, G heads, 64 / G rows), i.e. 64
// columns, the 128-byte swizzle, rows past num_tokens read as zeros.
int encode_q_map(CUtensorMap *tm, const void *q, int32_t num_tokens, int32_t num_q_heads, int32_t G) {
    auto fn = encode_fn();
    if (!fn) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled unavailable");
        return PA_ECUDA;
    }
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(pa::kD), static_cast<cuuint64_t>(num_q_heads),
                                static_cast<cuuint64_t>(num_tokens)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(pa::kD) * 2,
                                   static_cast<cuuint64_t>(num_q_heads) * pa::kD * 2};
    const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(pa::kColsTc / 2 / G)};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled (q) failed (%d)",
                      static_cast<int>(r));
        return PA_ECUDA;
    }
    return PA_OK;
}

// The tensor-memory variant (attend_tc.cuh): 128 columns per work unit, a
// persistent grid of one CTA per SM walking the units.
template <int G, bool kZeroScale, int HP>
int launch_attend_tc_g(const CUtensorMap &tk, const CUtensorMap &tv, const void *q, pa::AttendParams ap,
                       int32_t num_kv_heads, cudaStream_t stream) {
    static CtxDone done = {};
    int rc = prepare_kernel(pa::attend_tc_kernel<G, kZeroScale, HP>, pa::kAttendTcSmemBytes, done);
    if (rc)
        return rc;
    CUtensorMap tq;
    if ((rc = encode_q_map(&tq, q, ap.num_tokens, ap.d.num_q_heads, G)) != PA_OK)
        return rc;
    const int64_t units = static_cast<int64_t>(ap.d.num_parts) * (num_kv_heads / HP) * ap.d.num_seqs * ap.chunks;
    if (units > INT32_MAX)
        return PA_EUNSUPPORTED;
    ap.num_kv_heads = num_kv_heads;
    ap.head_groups = num_kv_heads / HP;
    ap.num_units = static_cast<int32_t>(units);
    const dim3 grid(static_cast<unsigned>(std::min<int64_t>(units, sm_count())));
    const pa::TcDivs dv = {pa::make_fast_div(static_cast<uint32_t>(ap.d.num_parts)),
                           pa::make_fast_div(static_cast<uint32_t>(ap.head_groups)),
                           pa::make_fast_div(static_cast<uint32_t>(ap.chunks))};
    cudaError_t e = launch_pdl(pa::attend_tc_kernel<G, kZeroScale, HP>, grid, dim3(pa::kTcThreads), pa::kAttendTcSmemBytes,
                               stream, tk, tv, tq, ap, dv);
    if (e != cudaSuccess)
        return cuda_fail(e, "attend_tc_kernel launch");
    return launch_row_merge(ap, stream);
}

template <bool kZeroScale, int HP>
int launch_attend_tc_hp(int32_t G, const CUtensorMap &tk, const CUtensorMap &tv, const void *q,
                        const pa::AttendParams &ap, int32_t nk, cudaStream_t st) {
    switch (G) {
    case 1: return launch_attend_tc_g<1, kZeroScale, HP>(tk, tv, q, ap, nk, st);
    case 2: return launch_attend_tc_g<2, kZeroScale, HP>(tk, tv, q, ap, nk, st);
    case 4: return launch_attend_tc_g<4, kZeroScale, HP>(tk, tv, q, ap, nk, st);
    default: return launch_attend_tc_g<8, kZeroScale, HP>(tk, tv, q, ap, nk, st);
    }
}
// The instantiation for a call: group size, zero scale, KV heads per unit.
int launch_attend_tc(int32_t G, bool zero_scale, int32_t heads_per_unit, const CUtensorMap &tk,
                     const CUtensorMap &tv, const void *q, const pa::AttendParams &ap, int32_t nk, cudaStream_t st) {
    if (heads_per_unit == 2)
        return zero_scale ? launch_attend_tc_hp<true, 2>(G, tk, tv, q, ap, nk, st)
                          : launch_attend_tc_hp<false, 2>(G, tk, tv, q, ap, nk, st);
    return zero_scale ? launch_attend_tc_hp<true, 1>(G, tk, tv, q, ap, nk, st)
                      : launch_attend_tc_hp<false, 1>(G, tk, tv, q, ap, nk, st);
}

pa_cache_t as_cache(const pa_cache_fp8_t *c) {
    pa_cache_t r{};
    r.k_cache = c->k_cache;
    r.v_cache = c->v_cache;
    r.num_blocks = c->num_blocks;
    r.block_size = c->block_size;
    r.num_kv_heads = c->num_kv_heads;
    r.head_dim = c->head_dim;
    return r;
}

int check_cache_fp8(const pa_cache_fp8_t *c) {
    if (!c)
        return PA_EINVAL;
    const pa_cache_t b = as_cache(c);
    const int rc = check_cache(&b);
    if (rc)
        return rc;
    if (!(c->k_scale > 0.f) || !(c->v_scale > 0.f) || !std::isfinite(c->k_scale) || !std::isfinite(c->v_scale))
        return PA_EINVAL;
    return PA_OK;
}

template <int G, int CW>
int launch_decode_fp8_cw(const CUtensorMap &tk, const CUtensorMap &tv, const pa::DecodeParams &p,
                         int32_t num_kv_heads, cudaStream_t stream) {
    static CtxDone done = {};
    int rc = prepare_kernel(pa::decode_partition_fp8_kernel<G, CW>, pa::kDecodeSmemBytesF, done);
    if (rc)
        return rc;
    const cudaError_t e = launch_pdl(pa::decode_partition_fp8_kernel<G, CW>,
                                     dim3(p.num_parts, num_kv_heads, p.num_seqs), dim3(pa::fp8_threads<CW>()),
                                     pa::kDecodeSmemBytesF, stream, tk, tv, p);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "decode_partition_fp8_kernel launch");
}

// Two consumer warps when the grid fits in one wave of 4 CTAs per SM, three
// otherwise (see decode_fp8.cuh).
template <int G>
int launch_decode_fp8_g(const CUtensorMap &tk, const CUtensorMap &tv, const pa::DecodeParams &p,
                        int32_t num_kv_heads, cudaStream_t stream) {
    const int64_t ctas = static_cast<int64_t>(p.num_parts) * num_kv_heads * p.num_seqs;
    const bool one_wave = ctas <= static_cast<int64_t>(sm_count()) * pa::kFp8CtasPerSm;
    int rc = one_wave ? launch_decode_fp8_cw<G, 2>(tk, tv, p, num_kv_heads, stream)
                      : launch_decode_fp8_cw<G, 3>(tk, tv, p, num_kv_heads, stream);
    if (rc)
        return rc;
    cudaError_t e;
    if (p.num_parts > 1) {
        e = launch_pdl(pa::decode_merge_kernel, dim3(p.num_q_heads, p.num_seqs, 1), dim3(pa::kD), 0, stream, p);
        if (e != cudaSuccess)
            return cuda_fail(e, "decode_merge_kernel launch");
    }
    return PA_OK;
}

// The host-side argument checks of pa_decode (and pa_decode_static_ws, which
// runs them before it touches the CUDA runtime).  An empty batch passes.
int check_decode_args(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
                      int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                      int32_t max_seq_len, int32_t num_q_heads, float scale, const void *out) {
    int rc = check_cache(cache);
    if (rc)
        return rc;
    if (num_seqs < 0 || max_seq_len < 0 || num_q_heads <= 0 || max_blocks_per_seq < 0)
        return PA_EINVAL;
    if (num_seqs == 0)
        return PA_OK;
    if (!q || !block_tables || !seq_lens || !out)
        return PA_EINVAL;
    if (num_q_heads % cache->num_kv_heads != 0)
        return PA_EINVAL;
    const int32_t G = num_q_heads / cache->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return PA_EUNSUPPORTED;
    if (!aligned16(q) || !aligned16(out))
        return PA_EUNSUPPORTED;
    if (num_seqs > 65535 || cache->num_kv_heads > 65535)
        return PA_EUNSUPPORTED;
    if (!std::isfinite(scale))
        return PA_EINVAL;
    return PA_OK;
}
}  // namespace

extern "C" {

int pa_write_kv(const void *k, const void *v, const int64_t *slot_mapping, int64_t num_tokens,
                const pa_cache_t *cache, void *stream) {
    int rc = check_cache(cache);
    if (rc)
        return rc;
    if (num_tokens < 0)
        return PA_EINVAL;
    if (num_tokens == 0)
        return PA_OK;
    if (!k || !v || !slot_mapping)
        return PA_EINVAL;
    if (!aligned16(k) || !aligned16(v))
        return PA_EUNSUPPORTED;
    const int row_vecs = cache->num_kv_heads * cache->head_dim * 2 / 16;
    if (num_tokens > INT32_MAX)
        return PA_EUNSUPPORTED;  // beyond any grid (and keeps the size arithmetic below in range)
    const int64_t warps = num_tokens * 2;
    const int64_t blocks = (warps * 32 + pa::kWriteThreads - 1) / pa::kWriteThreads;
    if (blocks > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::write_kv_kernel, dim3(static_cast<unsigned>(blocks)), dim3(pa::kWriteThreads),
                               0, static_cast<cudaStream_t>(stream), static_cast<const uint4 *>(k),
                               static_cast<const uint4 *>(v), slot_mapping, num_tokens,
                               static_cast<uint4 *>(cache->k_cache), static_cast<uint4 *>(cache->v_cache),
                               cache->num_blocks * cache->block_size, row_vecs);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "write_kv_kernel launch");
}

int pa_compute_slot_mapping(const int64_t *positions, const int32_t *req_indices, int64_t num_tokens,
                            const int32_t *block_tables, int32_t max_blocks_per_seq, int32_t num_reqs,
                            int32_t block_size, int64_t num_blocks, int64_t *slot_mapping, void *stream) {
    if (num_tokens < 0 || max_blocks_per_seq < 0 || num_reqs < 0 || num_blocks <= 0 || block_size <= 0)
        return PA_EINVAL;
    if (num_tokens == 0)
        return PA_OK;
    if (!positions || !req_indices || !slot_mapping || (num_reqs > 0 && !block_tables))
        return PA_EINVAL;
    if (num_tokens > INT32_MAX)
        return PA_EUNSUPPORTED;  // beyond any grid (and keeps the size arithmetic below in range)
    const int64_t blocks = (num_tokens + pa::kSlotThreads - 1) / pa::kSlotThreads;
    if (blocks > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::slot_mapping_kernel, dim3(static_cast<unsigned>(blocks)), dim3(pa::kSlotThreads),
                               0, static_cast<cudaStream_t>(stream), positions, req_indices, num_tokens,
                               block_tables, max_blocks_per_seq, num_reqs, block_size, num_blocks, slot_mapping);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "slot_mapping_kernel launch");
}

int pa_map_to_kernel_blocks(const int32_t *block_tables, int32_t num_rows, int32_t width, int32_t blocks_per_alloc,
                            int32_t *kernel_tables, int32_t kernel_width, void *stream) {
    if (num_rows < 0 || width < 0 || blocks_per_alloc < 1 || kernel_width < 0)
        return PA_EINVAL;
    if (static_cast<int64_t>(width) * blocks_per_alloc > kernel_width)
        return PA_EINVAL;
    if (num_rows == 0 || kernel_width == 0)
        return PA_OK;
    if (!kernel_tables || (width > 0 && !block_tables))
        return PA_EINVAL;
    const int64_t blocks = (static_cast<int64_t>(num_rows) * kernel_width + pa::kSlotThreads - 1) / pa::kSlotThreads;
    if (blocks > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::map_to_kernel_blocks_kernel, dim3(static_cast<unsigned>(blocks)),
                               dim3(pa::kSlotThreads), 0, static_cast<cudaStream_t>(stream), block_tables, num_rows,
                               width, blocks_per_alloc, kernel_tables, kernel_width);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "map_to_kernel_blocks_kernel launch");
}

int pa_write_kv_positions(const void *k, const void *v, const int64_t *positions, const int32_t *req_indices,
                          int64_t num_tokens, const int32_t *block_tables, int32_t max_blocks_per_seq,
                          int32_t num_reqs, const pa_cache_t *cache, void *stream) {
    int rc = check_cache(cache);
    if (rc)
        return rc;
    if (num_tokens < 0 || max_blocks_per_seq < 0 || num_reqs < 0)
        return PA_EINVAL;
    if (num_tokens == 0)
        return PA_OK;
    if (!k || !v || !positions || !req_indices || (num_reqs > 0 && !block_tables))
        return PA_EINVAL;
    if (!aligned16(k) || !aligned16(v))
        return PA_EUNSUPPORTED;
    const int row_vecs = cache->num_kv_heads * cache->head_dim * 2 / 16;
    if (num_tokens > INT32_MAX)
        return PA_EUNSUPPORTED;  // beyond any grid (and keeps the size arithmetic below in range)
    const int64_t blocks = (num_tokens * 2 * 32 + pa::kWriteThreads - 1) / pa::kWriteThreads;
    if (blocks > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::write_kv_positions_kernel, dim3(static_cast<unsigned>(blocks)),
                               dim3(pa::kWriteThreads), 0, static_cast<cudaStream_t>(stream),
                               static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), positions,
                               req_indices, num_tokens, block_tables, max_blocks_per_seq, num_reqs,
                               cache->block_size, cache->num_blocks, static_cast<uint4 *>(cache->k_cache),
                               static_cast<uint4 *>(cache->v_cache), row_vecs);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "write_kv_positions_kernel launch");
}

int pa_copy_blocks(const pa_cache_t *cache, const int64_t *src_dst_pairs, int64_t num_pairs,
                   void *stream) {
    int rc = check_cache(cache);
    if (rc)
        return rc;
    if (num_pairs < 0)
        return PA_EINVAL;
    if (num_pairs == 0)
        return PA_OK;
    if (!src_dst_pairs)
        return PA_EINVAL;
    if (num_pairs > INT32_MAX)
        return PA_EUNSUPPORTED;  // beyond any grid (and keeps the size arithmetic below in range)
    const int64_t block_vecs =
        static_cast<int64_t>(cache->block_size) * cache->num_kv_heads * cache->head_dim * 2 / 16;
    const int chunks = static_cast<int>((block_vecs + pa::kCopyChunkVecs - 1) / pa::kCopyChunkVecs);
    const int64_t grid = num_pairs * 2 * chunks;
    if (grid > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::copy_blocks_kernel, dim3(static_cast<unsigned>(grid)), dim3(pa::kCopyThreads),
                               0, static_cast<cudaStream_t>(stream), static_cast<uint4 *>(cache->k_cache),
                               static_cast<uint4 *>(cache->v_cache), src_dst_pairs, cache->num_blocks,
                               block_vecs, chunks);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "copy_blocks_kernel launch");
}

int pa_copy_blocks_layers(const pa_cache_t *caches, int32_t num_layers, const int64_t *src_dst_pairs,
                          int64_t num_pairs, void *stream) {
    if (!caches || num_layers < 0 || num_layers > pa::kMaxLayers || num_pairs < 0)
        return num_layers > pa::kMaxLayers ? PA_EUNSUPPORTED : PA_EINVAL;
    pa::LayerPtrs lp{};
    for (int32_t l = 0; l < num_layers; ++l) {
        const int rc = check_cache(&caches[l]);
        if (rc)
            return rc;
        if (caches[l].num_blocks != caches[0].num_blocks || caches[l].block_size != caches[0].block_size ||
            caches[l].num_kv_heads != caches[0].num_kv_heads)
            return PA_EINVAL;  // one pair list needs one block geometry
        lp.k[l] = static_cast<uint4 *>(caches[l].k_cache);
        lp.v[l] = static_cast<uint4 *>(caches[l].v_cache);
    }
    if (num_layers == 0 || num_pairs == 0)
        return PA_OK;
    if (!src_dst_pairs)
        return PA_EINVAL;
    if (num_pairs > INT32_MAX)
        return PA_EUNSUPPORTED;  // beyond any grid (and keeps the size arithmetic below in range)
    const pa_cache_t *c = &caches[0];
    const int64_t block_vecs = static_cast<int64_t>(c->block_size) * c->num_kv_heads * c->head_dim * 2 / 16;
    const int chunks = static_cast<int>((block_vecs + pa::kCopyChunkVecs - 1) / pa::kCopyChunkVecs);
    const int64_t grid = num_pairs * 2 * chunks;
    if (grid > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::copy_blocks_layers_kernel, dim3(static_cast<unsigned>(grid), num_layers),
                               dim3(pa::kCopyThreads), 0, static_cast<cudaStream_t>(stream), lp, src_dst_pairs,
                               c->num_blocks, block_vecs, chunks);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "copy_blocks_layers_kernel launch");
}


int pa_write_kv_fp8(const void *k, const void *v, const int64_t *slot_mapping, int64_t num_tokens,
                    const pa_cache_fp8_t *cache, void *stream) {
    int rc = check_cache_fp8(cache);
    if (rc)
        return rc;
    if (num_tokens < 0)
        return PA_EINVAL;
    if (num_tokens == 0)
        return PA_OK;
    if (!k || !v || !slot_mapping)
        return PA_EINVAL;
    if (!aligned16(k) || !aligned16(v))
        return PA_EUNSUPPORTED;
    const int row_vecs = cache->num_kv_heads * cache->head_dim * 2 / 16;
    if (num_tokens > INT32_MAX)
        return PA_EUNSUPPORTED;  // beyond any grid (and keeps the size arithmetic below in range)
    const int64_t blocks = (num_tokens * 2 * 32 + pa::kWriteThreads - 1) / pa::kWriteThreads;
    if (blocks > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::write_kv_fp8_kernel, dim3(static_cast<unsigned>(blocks)), dim3(pa::kWriteThreads),
                               0, static_cast<cudaStream_t>(stream), static_cast<const uint4 *>(k),
                               static_cast<const uint4 *>(v), slot_mapping, num_tokens,
                               static_cast<uint2 *>(cache->k_cache), static_cast<uint2 *>(cache->v_cache),
                               cache->num_blocks * cache->block_size, row_vecs, cache->k_scale, cache->v_scale);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "write_kv_fp8_kernel launch");
}

int pa_copy_blocks_fp8(const pa_cache_fp8_t *cache, const int64_t *src_dst_pairs, int64_t num_pairs,
                       void *stream) {
    int rc = check_cache_fp8(cache);
    if (rc)
        return rc;
    if (num_pairs < 0)
        return PA_EINVAL;
    if (num_pairs == 0)
        return PA_OK;
    if (!src_dst_pairs)
        return PA_EINVAL;
    if (num_pairs > INT32_MAX)
        return PA_EUNSUPPORTED;  // beyond any grid (and keeps the size arithmetic below in range)
    // one byte per value: the same byte-level kernel with half the bf16 block size
    const int64_t block_vecs = static_cast<int64_t>(cache->block_size) * cache->num_kv_heads * cache->head_dim / 16;
    const int chunks = static_cast<int>((block_vecs + pa::kCopyChunkVecs - 1) / pa::kCopyChunkVecs);
    const int64_t grid = num_pairs * 2 * chunks;
    if (grid > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::copy_blocks_kernel, dim3(static_cast<unsigned>(grid)), dim3(pa::kCopyThreads),
                               0, static_cast<cudaStream_t>(stream), static_cast<uint4 *>(cache->k_cache),
                               static_cast<uint4 *>(cache->v_cache), src_dst_pairs, cache->num_blocks,
                               block_vecs, chunks);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "copy_blocks_kernel launch (fp8)");
}

int pa_copy_blocks_layers_fp8(const pa_cache_fp8_t *caches, int32_t num_layers, const int64_t *src_dst_pairs,
                              int64_t num_pairs, void *stream) {
    if (!caches || num_layers < 0 || num_layers > pa::kMaxLayers || num_pairs < 0)
        return num_layers > pa::kMaxLayers ? PA_EUNSUPPORTED : PA_EINVAL;
    pa::LayerPtrs lp{};
    for (int32_t l = 0; l < num_layers; ++l) {
        const int rc = check_cache_fp8(&caches[l]);
        if (rc)
            return rc;
        if (caches[l].num_blocks != caches[0].num_blocks || caches[l].block_size != caches[0].block_size ||
            caches[l].num_kv_heads != caches[0].num_kv_heads)
            return PA_EINVAL;  // one pair list needs one block geometry
        lp.k[l] = static_cast<uint4 *>(caches[l].k_cache);
        lp.v[l] = static_cast<uint4 *>(caches[l].v_cache);
    }
    if (num_layers == 0 || num_pairs == 0)
        return PA_OK;
    if (!src_dst_pairs)
        return PA_EINVAL;
    if (num_pairs > INT32_MAX)
        return PA_EUNSUPPORTED;  // beyond any grid (and keeps the size arithmetic below in range)
    const pa_cache_fp8_t *c = &caches[0];
    // one byte per value: the byte-level kernel with the FP8 block size
    const int64_t block_vecs = static_cast<int64_t>(c->block_size) * c->num_kv_heads * c->head_dim / 16;
    const int chunks = static_cast<int>((block_vecs + pa::kCopyChunkVecs - 1) / pa::kCopyChunkVecs);
    const int64_t grid = num_pairs * 2 * chunks;
    if (grid > INT32_MAX)
        return PA_EUNSUPPORTED;
    cudaError_t e = launch_pdl(pa::copy_blocks_layers_kernel, dim3(static_cast<unsigned>(grid), num_layers),
                               dim3(pa::kCopyThreads), 0, static_cast<cudaStream_t>(stream), lp, src_dst_pairs,
                               c->num_blocks, block_vecs, chunks);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "copy_blocks_layers_kernel launch (fp8)");
}

size_t pa_decode_fp8_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t max_seq_len,
                                     const pa_cache_fp8_t *cache) {
    if (check_cache_fp8(cache) != PA_OK || num_seqs <= 0 || num_q_heads <= 0 || max_seq_len < 0)
        return 0;
    return workspace_layout(num_seqs, num_q_heads, cache->num_kv_heads, max_seq_len, cache->block_size, true).total;
}

int pa_decode_fp8(const void *q, const pa_cache_fp8_t *cache, const int32_t *block_tables,
                  int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs, int32_t max_seq_len,
                  int32_t num_q_heads, float scale, void *out, void *workspace, size_t workspace_bytes,
                  void *stream) {
    int rc = check_cache_fp8(cache);
    if (rc)
        return rc;
    if (num_seqs < 0 || max_seq_len < 0 || num_q_heads <= 0 || max_blocks_per_seq < 0)
        return PA_EINVAL;
    if (num_seqs == 0)
        return PA_OK;
    if (!q || !block_tables || !seq_lens || !out)
        return PA_EINVAL;
    if (num_q_heads % cache->num_kv_heads != 0)
        return PA_EINVAL;
    const int32_t G = num_q_heads / cache->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return PA_EUNSUPPORTED;
    if (!aligned16(q) || !aligned16(out))
        return PA_EUNSUPPORTED;
    if (num_seqs > 65535 || cache->num_kv_heads > 65535)
        return PA_EUNSUPPORTED;
    if (!std::isfinite(scale))
        return PA_EINVAL;
    const WorkspaceLayout w =
        workspace_layout(num_seqs, num_q_heads, cache->num_kv_heads, max_seq_len, cache->block_size, true);
    if (w.total > 0 && (workspace == nullptr || workspace_bytes < w.total))
        return PA_EWORKSPACE;
    if (w.total > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return PA_EUNSUPPORTED;
    const pa_cache_t view = as_cache(cache);
    CUtensorMap tk, tv;
    if ((rc = encode_cache_map(&tk, cache->k_cache, &view, true, true)) != PA_OK)
        return rc;
    if ((rc = encode_cache_map(&tv, cache->v_cache, &view, true, true)) != PA_OK)
        return rc;
    pa::DecodeParams p{};
    p.q = static_cast<const uint4 *>(q);
    p.k_cache = cache->k_cache;
    p.v_cache = cache->v_cache;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.part_ml = w.total ? static_cast<float2 *>(workspace) : nullptr;
    p.part_acc = w.total ? reinterpret_cast<float *>(static_cast<char *>(workspace) + w.acc_offset) : nullptr;
    p.num_blocks = cache->num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.max_seq_len = max_seq_len;
    p.num_q_heads = num_q_heads;
    p.block_size = cache->block_size;
    p.part_tokens = w.part_tokens;
    p.num_parts = w.num_parts;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);  // log2(e)
    p.k_scale = cache->k_scale;
    p.v_scale = cache->v_scale;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (G) {
    case 1: return launch_decode_fp8_g<1>(tk, tv, p, cache->num_kv_heads, st);
    case 2: return launch_decode_fp8_g<2>(tk, tv, p, cache->num_kv_heads, st);
    case 4: return launch_decode_fp8_g<4>(tk, tv, p, cache->num_kv_heads, st);
    default: return launch_decode_fp8_g<8>(tk, tv, p, cache->num_kv_heads, st);
    }
}

size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t max_seq_len,
                                 const pa_cache_t *cache) {
    if (check_cache(cache) != PA_OK || num_seqs <= 0 || num_q_heads <= 0 || max_seq_len < 0)
        return 0;
    return workspace_layout(num_seqs, num_q_heads, cache->num_kv_heads, max_seq_len, cache->block_size,
                            decode_kernel_is_mma())
        .total;
}

size_t pa_attention_workspace_bytes(int32_t num_reqs, int32_t num_tokens, int32_t max_query_len,
                                    int32_t num_q_heads, int32_t max_seq_len, const pa_cache_t *cache) {
    if (check_cache(cache) != PA_OK || num_reqs <= 0 || num_tokens <= 0 || max_query_len <= 0 ||
        num_q_heads <= 0 || max_seq_len < 0 || num_q_heads % cache->num_kv_heads != 0)
        return 0;
    const int64_t columns = static_cast<int64_t>(max_query_len) * (num_q_heads / cache->num_kv_heads);
    return attend_layout(num_reqs, num_tokens, max_query_len, num_q_heads, cache->num_kv_heads, max_seq_len,
                         cache->block_size, attention_kernel_is_tcgen05(columns))
        .total;
}

int pa_attention(const void *q, int32_t num_tokens, const int32_t *query_start_loc, int32_t num_reqs,
                 int32_t max_query_len, const pa_cache_t *cache, const int32_t *block_tables,
                 int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t max_seq_len, int32_t num_q_heads,
                 float scale, void *out, void *workspace, size_t workspace_bytes, void *stream) {
    int rc = check_cache(cache);
    if (rc)
        return rc;
    if (num_tokens < 0 || num_reqs < 0 || max_query_len < 0 || max_seq_len < 0 || num_q_heads <= 0 ||
        max_blocks_per_seq < 0)
        return PA_EINVAL;
    if (num_reqs == 0 || num_tokens == 0 || max_query_len == 0)
        return PA_OK;
    if (!q || !query_start_loc || !block_tables || !seq_lens || !out)
        return PA_EINVAL;
    if (num_q_heads % cache->num_kv_heads != 0)
        return PA_EINVAL;
    const int32_t G = num_q_heads / cache->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return PA_EUNSUPPORTED;
    if (!aligned16(q) || !aligned16(out))
        return PA_EUNSUPPORTED;
    if (!std::isfinite(scale))
        return PA_EINVAL;
    const AttendLayout a = attend_layout(num_reqs, num_tokens, max_query_len, num_q_heads, cache->num_kv_heads,
                                         max_seq_len, cache->block_size,
                                         attention_kernel_is_tcgen05(static_cast<int64_t>(max_query_len) * G));
    if (static_cast<int64_t>(num_reqs) * a.chunks > 65535 || cache->num_kv_heads > 65535)
        return PA_EUNSUPPORTED;
    if (a.total > 0 && (workspace == nullptr || workspace_bytes < a.total))
        return PA_EWORKSPACE;
    if (a.total > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return PA_EUNSUPPORTED;

    CUtensorMap tk, tv;
    if ((rc = encode_cache_map(&tk, cache->k_cache, cache, true)) != PA_OK)
        return rc;
    if ((rc = encode_cache_map(&tv, cache->v_cache, cache, true)) != PA_OK)
        return rc;

    pa::AttendParams ap{};
    pa::DecodeParams &p = ap.d;
    p.q = static_cast<const uint4 *>(q);
    p.k_cache = cache->k_cache;
    p.v_cache = cache->v_cache;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.part_ml = a.total ? static_cast<float2 *>(workspace) : nullptr;
    p.part_acc = a.total ? reinterpret_cast<float *>(static_cast<char *>(workspace) + a.acc_offset) : nullptr;
    p.num_blocks = cache->num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_reqs;
    p.max_seq_len = max_seq_len;
    p.num_q_heads = num_q_heads;
    p.block_size = cache->block_size;
    p.part_tokens = a.part_tokens;
    p.num_parts = a.num_parts;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);  // log2(e)
    p.k_scale = 1.f;
    p.v_scale = 1.f;
    ap.query_start_loc = query_start_loc;
    ap.row_len = a.total ? reinterpret_cast<int32_t *>(static_cast<char *>(workspace) + a.len_offset) : nullptr;
    ap.num_tokens = num_tokens;
    ap.max_query_len = max_query_len;
    ap.chunks = a.chunks;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (a.tcgen05) {
        return launch_attend_tc(G, scale == 0.f, a.heads_per_unit, tk, tv, q, ap, cache->num_kv_heads, st);
    }
    const bool w2 = a.warps == 2;
    switch (G) {
    case 1: return w2 ? launch_attend_g<1, 2>(tk, tv, ap, cache->num_kv_heads, st)
                      : launch_attend_g<1, 4>(tk, tv, ap, cache->num_kv_heads, st);
    case 2: return w2 ? launch_attend_g<2, 2>(tk, tv, ap, cache->num_kv_heads, st)
                      : launch_attend_g<2, 4>(tk, tv, ap, cache->num_kv_heads, st);
    case 4: return w2 ? launch_attend_g<4, 2>(tk, tv, ap, cache->num_kv_heads, st)
                      : launch_attend_g<4, 4>(tk, tv, ap, cache->num_kv_heads, st);
    default: return w2 ? launch_attend_g<8, 2>(tk, tv, ap, cache->num_kv_heads, st)
                       : launch_attend_g<8, 4>(tk, tv, ap, cache->num_kv_heads, st);
    }
}

int32_t pa_decode_set_kernel(int32_t kind) {
    if (kind == PA_DECODE_KERNEL_MMA || kind == PA_DECODE_KERNEL_SIMT)
        return g_decode_kernel.exchange(kind);
    return g_decode_kernel.load();
}

int32_t pa_attention_set_kernel(int32_t kind) {
    if (kind == PA_ATTENTION_KERNEL_MMA || kind == PA_ATTENTION_KERNEL_TCGEN05 || kind == PA_ATTENTION_KERNEL_AUTO)
        return g_attention_kernel.exchange(kind);
    return g_attention_kernel.load();
}

int32_t pa_decode_set_partition_tokens(int32_t tokens) {
    return g_part_tokens_override.exchange(tokens > 0 ? tokens : 0);
}

int pa_decode(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
              int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
              int32_t max_seq_len, int32_t num_q_heads, float scale, void *out, void *workspace,
              size_t workspace_bytes, void *stream) {
    int rc = check_decode_args(q, cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, max_seq_len,
                               num_q_heads, scale, out);
    if (rc || num_seqs == 0)
        return rc;
    const int32_t G = num_q_heads / cache->num_kv_heads;

    const bool mma = decode_kernel_is_mma();  // the knob, read once for the whole call
    const WorkspaceLayout w =
        workspace_layout(num_seqs, num_q_heads, cache->num_kv_heads, max_seq_len, cache->block_size, mma);
    if (w.total > 0 && (workspace == nullptr || workspace_bytes < w.total))
        return PA_EWORKSPACE;
    if (w.total > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return PA_EUNSUPPORTED;

    CUtensorMap tk, tv;
    if ((rc = encode_cache_map(&tk, cache->k_cache, cache, mma)) != PA_OK)
        return rc;
    if ((rc = encode_cache_map(&tv, cache->v_cache, cache, mma)) != PA_OK)
        return rc;

    pa::DecodeParams p{};
    p.q = static_cast<const uint4 *>(q);
    p.k_cache = cache->k_cache;
    p.v_cache = cache->v_cache;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.part_ml = w.total ? static_cast<float2 *>(workspace) : nullptr;
    p.part_acc = w.total ? reinterpret_cast<float *>(static_cast<char *>(workspace) + w.acc_offset) : nullptr;
    p.num_blocks = cache->num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.max_seq_len = max_seq_len;
    p.num_q_heads = num_q_heads;
    p.block_size = cache->block_size;
    p.part_tokens = w.part_tokens;
    p.num_parts = w.num_parts;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);  // log2(e)
    p.k_scale = 1.f;
    p.v_scale = 1.f;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (G) {
    case 1: return launch_decode_g<1>(tk, tv, p, cache->num_kv_heads, mma, st);
    case 2: return launch_decode_g<2>(tk, tv, p, cache->num_kv_heads, mma, st);
    case 4: return launch_decode_g<4>(tk, tv, p, cache->num_kv_heads, mma, st);
    default: return launch_decode_g<8>(tk, tv, p, cache->num_kv_heads, mma, st);
    }
}

int pa_get_device_error(int32_t *host_code, int clear) {
    if (!host_code)
        return PA_EINVAL;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaDeviceSynchronize");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, pa::g_device_error, sizeof v);
    if (e != cudaSuccess)
        return cuda_fail(e, "read device error word");
    *host_code = v;
    if (clear) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(pa::g_device_error, &zero, sizeof zero);
        if (e != cudaSuccess)
            return cuda_fail(e, "clear device error word");
    }
    return PA_OK;
}

// ---------------------------------------------------------------------------
// pa_decode_static_ws: pa_decode with its split-K scratch in a fixed device
// array owned by this library, for callers that cannot allocate device
// memory (see include/pa.h).  The array is a file-scope __device__ object: one
// copy per device that loads the library, kept until the process exits.  In
// host code its name only stands in for the object; the device address comes
// from cudaGetSymbolAddress, looked up on the first call made with a device
// current and cached with the id of that device's context (looked up again
// after a device reset).
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_decode_static_scratch[PA_DECODE_STATIC_WS_BYTES];

namespace {
// Per device: the array's device address and the context it was looked up in.
struct StaticScratch {
    void *ptr;
    unsigned long long ctx;
};
std::mutex g_static_scratch_mu;
StaticScratch g_static_scratch[64] = {};
}  // namespace

int pa_decode_static_ws(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
                        int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                        int32_t max_seq_len, int32_t num_q_heads, float scale, void *out,
                        void *stream) {
    // Argument errors and a too-large shape are reported before any CUDA
    // call; an empty batch still does the one-time address lookup below.
    int rc = check_decode_args(q, cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, max_seq_len,
                               num_q_heads, scale, out);
    if (rc)
        return rc;
    if (num_seqs > 0) {
        const size_t need = pa_decode_workspace_bytes(num_seqs, num_q_heads, max_seq_len, cache);
        if (need > PA_DECODE_STATIC_WS_BYTES) {
            std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                          "pa_decode_static_ws: this shape needs %zu bytes of scratch, the static "
                          "array holds %zu",
                          need, static_cast<size_t>(PA_DECODE_STATIC_WS_BYTES));
            return PA_EWORKSPACE;
        }
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64)
        return PA_EUNSUPPORTED;
    void *scratch = nullptr;
    {
        // The address is looked up again whenever the current context is not
        // the one it was found in: a device reset gives the device a new
        // primary context, which loads this module afresh, possibly at other
        // addresses.
        std::lock_guard<std::mutex> lock(g_static_scratch_mu);
        StaticScratch &c = g_static_scratch[dev];
        const unsigned long long ctx = current_ctx_id();
        if (!c.ptr || ctx == 0 || c.ctx != ctx) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_decode_static_scratch);
            if (e != cudaSuccess) {
                c.ptr = nullptr;
                c.ctx = 0;
                return cuda_fail(e, "cudaGetSymbolAddress(static decode scratch)");
            }
            c.ptr = p;
            c.ctx = current_ctx_id();  // the lookup above made the device's context current
        }
        scratch = c.ptr;
    }
    return pa_decode(q, cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, max_seq_len,
                     num_q_heads, scale, out, scratch, PA_DECODE_STATIC_WS_BYTES, stream);
}

const char *pa_last_cuda_error(void) { return g_last_cuda_error; }

const char *pa_status_str(int status) {
    switch (status) {
    case PA_OK: return "ok";
    case PA_EINVAL: return "invalid argument";
    case PA_EUNSUPPORTED: return "unsupported shape, size or alignment";
    case PA_EWORKSPACE: return "workspace too small";
    case PA_ECUDA: return "CUDA error";
    default: return "unknown status";
    }
}

}  // extern "C"
