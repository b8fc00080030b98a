/*
 * pa.h -- C ABI of the paged-KV decode path on NVIDIA B200 (sm_100a).
 *
 * Three device operations keep a block-major KV pool consistent and read it:
 *   pa_write_kv     store this step's K/V rows at their slots;
 *   pa_copy_blocks  copy-on-write block copies;
 *   pa_decode       decode attention gathered through the block table.
 *
 * Memory: every pointer argument named without a host_ prefix is a DEVICE
 * pointer (cudaMalloc / torch CUDA memory) on the current device.  The caller
 * allocates and owns every buffer; the library allocates no device memory.
 * bf16 arrays hold IEEE bfloat16 bit patterns.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream).  Every call only enqueues work and returns; results are ready when
 * the stream reaches that point.
 *
 * Status: 0 = success; a negative PA_E* code = nothing was enqueued.
 * Arguments that live on the device (slots, block ids, lengths, copy pairs)
 * cannot be checked on the host without a synchronisation; the kernels check
 * them instead and never touch memory outside the caller's arrays: an
 * out-of-range value is skipped (write, copy) or replaced by an in-range
 * dummy (decode) and recorded in the device error word read by
 * pa_get_device_error.  No kernel traps.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
    PA_OK = 0,
    PA_EINVAL = -1,       /* null pointer, negative size, num_q_heads % num_kv_heads != 0 */
    PA_EUNSUPPORTED = -2, /* head_dim != 128, block_size not a power of two in [1, 64],
                             group size not in {1, 2, 4, 8}, pointer not 16-byte aligned,
                             num_kv_heads > 65535, or a count past the launch limits
                             (more than INT32_MAX tokens or copy pairs) */
    PA_EWORKSPACE = -3,   /* workspace smaller than pa_decode_workspace_bytes() */
    PA_ECUDA = -4         /* a CUDA call or launch failed (see pa_last_cuda_error) */
};

/* Bits of the device error word. */
enum {
    PA_DEVERR_SLOT = 1,       /* pa_write_kv: slot >= num_blocks * block_size (row skipped) */
    PA_DEVERR_BLOCK_ID = 2,   /* pa_decode: block id outside [0, num_blocks) (block 0 read instead) */
    PA_DEVERR_SEQ_LEN = 4,    /* pa_decode: seq_len < 0, > max_seq_len, or needing more than
                                 max_blocks_per_seq table entries (clamped) */
    PA_DEVERR_COPY_PAIR = 8,  /* pa_copy_blocks: id outside [0, num_blocks) (pair skipped) */
    PA_DEVERR_TIMEOUT = 16,   /* a pipeline wait gave up after its time limit */
    PA_DEVERR_QUERY_LOC = 32  /* pa_attention: query_start_loc not a non-decreasing split of
                                 [0, num_tokens), or a request with more rows than tokens or
                                 than max_query_len (the outputs of that request's rows are
                                 undefined: not written with one partition, merged from
                                 unset partials with split-K; every access stays in bounds) */
};

/* One layer's paged KV cache.  k_cache and v_cache are separate tensors of
 * shape [num_blocks][block_size][num_kv_heads][head_dim] bf16, block-major:
 * block i owns one contiguous range, and row `slot` of the cache viewed as
 * [num_blocks*block_size][num_kv_heads*head_dim] is token slot `slot`
 * ("PagedAttention: fragmentation, blocks, block tables", section 3 "The
 * slot mapping": block-major backing storage; the r7 walkthrough stores the
 * token at row 30,608 of the cache so viewed). */
typedef struct pa_cache {
    void *k_cache;
    void *v_cache;
    int64_t num_blocks;
    int32_t block_size;
    int32_t num_kv_heads;
    int32_t head_dim;
} pa_cache_t;

/*
 * pa_write_kv -- the KV-cache write of one step.
 * Defined by: "PagedAttention: fragmentation, blocks, block tables",
 * section 3 "The slot mapping" (each new token's K and V are stored at the
 * slot that slot_mapping[i] names, the same slot in every layer's own
 * tensor; padding entries hold a sentinel that is not a slot).
 *   k, v          [num_tokens][num_kv_heads][head_dim] bf16, contiguous.
 *   slot_mapping  [num_tokens] int64; row i goes to cache row slot_mapping[i];
 *                 a negative slot is padding and is skipped.  Slots must be
 *                 distinct (two tokens to one slot: either row may win).
 * Bit-exact copy of the rows; no arithmetic.
 */
PA_API int pa_write_kv(const void *k, const void *v, const int64_t *slot_mapping, int64_t num_tokens,
                const pa_cache_t *cache, void *stream);

/*
 * pa_compute_slot_mapping -- the slot mapping of a step, on the device.
 * Defined by: "PagedAttention: fragmentation, blocks, block tables",
 * section 3 "The slot mapping" (recomputed every step from the block table
 * and the scheduled tokens' positions: slot = block_table[req][pos / B] * B
 * + pos % B; tokens that are not written get a PAD value).
 *   positions     [num_tokens] int64: position of each token in its sequence;
 *                 a negative position is padding.
 *   req_indices   [num_tokens] int32: row of block_tables of each token.
 *   block_tables  [num_reqs][max_blocks_per_seq] int32.
 *   slot_mapping  [num_tokens] int64 output; padding -> -1.  A token whose
 *                 request, table entry or block id is out of range also gets
 *                 -1 and sets PA_DEVERR_SLOT.
 */
PA_API int pa_compute_slot_mapping(const int64_t *positions, const int32_t *req_indices, int64_t num_tokens,
                                   const int32_t *block_tables, int32_t max_blocks_per_seq, int32_t num_reqs,
                                   int32_t block_size, int64_t num_blocks, int64_t *slot_mapping, void *stream);

/*
 * pa_write_kv_positions -- pa_write_kv with the slot computed in the kernel
 * from the token's request row and position (same passage as above), so a
 * step needs no host-built slot mapping.  Arguments as pa_write_kv and
 * pa_compute_slot_mapping; cache->block_size and cache->num_blocks give B and
 * the block-id range.  Out-of-range tokens are skipped and set
 * PA_DEVERR_SLOT; negative positions are padding.
 */
PA_API int pa_write_kv_positions(const void *k, const void *v, const int64_t *positions,
                                 const int32_t *req_indices, int64_t num_tokens, const int32_t *block_tables,
                                 int32_t max_blocks_per_seq, int32_t num_reqs, const pa_cache_t *cache,
                                 void *stream);

/*
 * pa_map_to_kernel_blocks -- expand block tables of allocation blocks into
 * block tables of smaller kernel blocks.
 * Defined by: "PagedAttention: fragmentation, blocks, block tables",
 * section 2 "The block table" (append_row maps the ids through
 * map_to_kernel_blocks when the kernel's block is smaller) and the passage
 * on decoupling the allocation block from the kernel's page (allocation in
 * 32-token units, say, while the attention kernel reads 16-token pages).  The cache
 * is block-major, so allocation block a (pages of block_size tokens) owns the
 * bytes of kernel blocks a*m .. a*m + m - 1 (pages of block_size / m tokens),
 * m = blocks_per_alloc: the same memory is a pa_cache_t with num_blocks * m
 * blocks of block_size / m tokens, addressed by the expanded tables.
 *   block_tables   [num_rows][width] int32 on the device; negative = padding.
 *   kernel_tables  [num_rows][kernel_width] int32 on the device, kernel_width
 *                  >= width * m: entry i*m + j of row r is tables[r][i]*m + j,
 *                  -1 for padding and for the columns past width * m.
 * Returns PA_EINVAL for blocks_per_alloc < 1 or kernel_width < width * m.  An
 * id whose kernel ids exceed INT32_MAX is written as -1 and sets
 * PA_DEVERR_BLOCK_ID.
 */
PA_API int pa_map_to_kernel_blocks(const int32_t *block_tables, int32_t num_rows, int32_t width,
                                   int32_t blocks_per_alloc, int32_t *kernel_tables, int32_t kernel_width,
                                   void *stream);

/*
 * pa_copy_blocks -- copy-on-write block copies.
 * Defined by: "PagedAttention: fragmentation, blocks, block tables",
 * copy-on-write passage (the queued (src_block_id, dst_block_id) pairs are
 * executed ahead of the step's attention reads; one assignment
 * blocks[dst] = blocks[src] over the block-major storage).
 *   src_dst_pairs [num_pairs][2] int64 (src, dst).  Every dst must be
 *                 distinct and no dst may also be a src (the pool's pairs
 *                 always are); the whole block -- all block_size slots, K
 *                 and V -- is copied bit for bit.
 */
PA_API int pa_copy_blocks(const pa_cache_t *cache, const int64_t *src_dst_pairs, int64_t num_pairs,
                   void *stream);

/*
 * pa_copy_blocks_layers -- pa_copy_blocks for every layer of a model in one
 * launch.  Same passage as pa_copy_blocks (one batched copy for all layers
 * rather than a loop over them: there the
 * layers alias one storage; here each layer has its own K and V tensors and
 * one grid covers them all).
 *   caches      HOST array of num_layers descriptors (<= 128), all with the
 *               same num_blocks, block_size, num_kv_heads and head_dim.
 *   src_dst_pairs, num_pairs: as pa_copy_blocks, applied to every layer.
 */
PA_API int pa_copy_blocks_layers(const pa_cache_t *caches, int32_t num_layers, const int64_t *src_dst_pairs,
                                 int64_t num_pairs, void *stream);

/*
 * Bytes of scratch pa_decode needs for this batch shape (0 when no sequence
 * is long enough to be split across CTAs).  Depends only on host values, so
 * it can be called once per shape and the buffer reused.
 */
PA_API size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t max_seq_len,
                                 const pa_cache_t *cache);

/*
 * pa_decode -- decode attention over the paged cache, one query token per
 * sequence.
 * Defined by: "PagedAttention: fragmentation, blocks, block tables",
 * attention-metadata passage (an int32 table with one row per request; for
 * request r the gather reads the first ceil(seq_lens[r] / block_size)
 * entries of its row; max_seq_len need only bound the lengths from above)
 * and section 2 "The block table" (token p is found through entry p / B, at
 * offset p % B inside that block); "The pantry of pigeonholes", "The mechanism: blocks, block
 * table and the kernel gather".
 * For sequence s and query head j, with h = j / (num_q_heads / num_kv_heads):
 *   out[s][j] = sum_t softmax_t(scale * q[s][j] . K[s,h,t]) V[s,h,t],
 * over the seq_lens[s] tokens of s in logical order; fp32 accumulation,
 * one rounding to bf16 at the end.  A sequence of length 0 gives zeros.
 *   q             [num_seqs][num_q_heads][head_dim] bf16.
 *   block_tables  [num_seqs][max_blocks_per_seq] int32; only the first
 *                 ceil(seq_lens[s] / block_size) entries of row s are read.
 *   seq_lens      [num_seqs] int32 on the device, each <= max_seq_len.
 *   max_seq_len   host-side upper bound of seq_lens (sizes the grid without
 *                 reading the device).
 *   out           [num_seqs][num_q_heads][head_dim] bf16.
 *   workspace     device scratch of at least pa_decode_workspace_bytes(...)
 *                 bytes (may be NULL when that is 0).  Calls that overlap on
 *                 the GPU must use different workspaces.
 */
PA_API int pa_decode(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
              int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
              int32_t max_seq_len, int32_t num_q_heads, float scale, void *out,
              void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_attention -- attention of several query tokens per request over the
 * paged cache (speculative tokens, chunks of a prefill; one row per request
 * is a decode step).
 * Defined by: "PagedAttention: fragmentation, blocks, block tables", the
 * attention-metadata passage: query_start_loc [num_reqs + 1] gives the start
 * of each request's rows in the query tensor, seq_lens [num_reqs] the
 * computed tokens of each request, max_query_len the longest query, and the
 * block table is walked as for pa_decode.  The pages do not spell the mask
 * out; the reading taken is the causal one: the q_len = query_start_loc[r+1]
 * - query_start_loc[r] rows of request r are its last q_len tokens (their K/V
 * already written and counted in n = seq_lens[r]), and row i attends to
 * positions 0 .. n - q_len + i.  For row i of request r and query head j
 * (h = j / (num_q_heads / num_kv_heads)):
 *   out[q0 + i][j] = sum_{t <= n-q_len+i} softmax_t(scale * q[q0+i][j] . K[r,h,t]) V[r,h,t].
 *   q                [num_tokens][num_q_heads][head_dim] bf16 (16-byte aligned).
 *   query_start_loc  [num_reqs + 1] int32 on the device: 0 = loc[0] <= loc[1]
 *                    <= ... <= loc[num_reqs] = num_tokens, each step at most
 *                    max_query_len and at most that request's seq_len
 *                    (checked on the device: PA_DEVERR_QUERY_LOC).
 *   max_query_len    host-side upper bound of the rows per request (sizes the grid).
 *   block_tables, seq_lens, max_seq_len  as for pa_decode, per request.
 *   out              [num_tokens][num_q_heads][head_dim] bf16.
 *   workspace        device scratch of at least pa_attention_workspace_bytes(...)
 *                    bytes (may be NULL when that is 0).
 * Supports the bf16 cache; group sizes 1, 2, 4, 8.  Returns PA_EUNSUPPORTED
 * when num_reqs * ceil(max_query_len * group / 32) exceeds 65535.
 */
PA_API size_t pa_attention_workspace_bytes(int32_t num_reqs, int32_t num_tokens, int32_t max_query_len,
                                           int32_t num_q_heads, int32_t max_seq_len, const pa_cache_t *cache);
PA_API int pa_attention(const void *q, int32_t num_tokens, const int32_t *query_start_loc, int32_t num_reqs,
                        int32_t max_query_len, const pa_cache_t *cache, const int32_t *block_tables,
                        int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t max_seq_len,
                        int32_t num_q_heads, float scale, void *out, void *workspace, size_t workspace_bytes,
                        void *stream);

/* ------------------------------------------------------------------------
 * Tuning knobs.  The three setters below change one process-wide setting
 * each, which every later call from every host thread reads, including
 * calls made by any other user of this library in the same process.  They
 * exist for measurement and tests; a library user should leave them at their
 * defaults, or set them once at start-up and restore the previous value
 * (each setter returns it) when done.  Each call reads each setting once.
 * ------------------------------------------------------------------------ */

/* Which partition kernel pa_decode runs (process wide; returns the previous
 * value; other values are ignored).  Both compute the same result within
 * the stated tolerance.
 *   PA_DECODE_KERNEL_MMA  (default) QK^T and PV of each 16-token tile on
 *                         tensor cores (mma.m16n8k16, fp32 accumulate), K/V
 *                         tiles staged by 128B-swizzled TMA loads;
 *   PA_DECODE_KERNEL_SIMT QK^T, softmax and PV on CUDA cores with warp
 *                         shuffles (kept for measurement). */
enum { PA_DECODE_KERNEL_MMA = 0, PA_DECODE_KERNEL_SIMT = 1 };
PA_API int32_t pa_decode_set_kernel(int32_t kind);

/* Which kernel pa_attention runs (process wide; returns the previous value;
 * other values are ignored).  pa_attention_workspace_bytes() follows the
 * setting, so query it after choosing.
 *   PA_ATTENTION_KERNEL_MMA     warps of 8 (row, head) columns on
 *                               mma.m16n8k16, 16-token K/V tiles: for a few
 *                               rows per request (speculative decoding);
 *   PA_ATTENTION_KERNEL_TCGEN05 work units of 128 (row, head) columns (two KV
 *                               heads of up to 64 columns each, when the KV
 *                               head count is even) on tcgen05.mma with S, P
 *                               and O in tensor memory, 64-row K/V tiles: for
 *                               requests with many rows (prefill chunks);
 *   PA_ATTENTION_KERNEL_AUTO    (default) per call: the tcgen05 kernel when
 *                               max_query_len x (num_q_heads / num_kv_heads)
 *                               is at least PA_ATTENTION_TCGEN05_MIN_COLUMNS
 *                               (above 16 columns the mma.sync kernel moves to
 *                               its wider CTA shape, and the tcgen05 kernel is
 *                               faster from there on B200), else the mma.sync
 *                               kernel. */
enum { PA_ATTENTION_KERNEL_MMA = 0, PA_ATTENTION_KERNEL_TCGEN05 = 1, PA_ATTENTION_KERNEL_AUTO = 2 };
#define PA_ATTENTION_TCGEN05_MIN_COLUMNS 17
PA_API int32_t pa_attention_set_kernel(int32_t kind);

/* Tokens per split-K partition used by pa_decode: 0 = automatic (the
 * default), otherwise a multiple of 64.  Host-side setting, process wide;
 * returns the previous value.  For tuning and tests. */
PA_API int32_t pa_decode_set_partition_tokens(int32_t tokens);

/*
 * pa_decode_static_ws -- pa_decode without a caller-supplied workspace.
 * The pages have no counterpart for this call: it exists for callers that
 * cannot allocate device memory, such as a plugin whose host application
 * owns every device allocation and hands it no allocator, or a serving loop
 * that must not call cudaMalloc on its hot path (it can synchronize the
 * device and stall other work).  Same arguments and result as pa_decode,
 * minus workspace and workspace_bytes.
 *   Scratch: a fixed array of PA_DECODE_STATIC_WS_BYTES (8 MiB) in this
 *   library's device memory, present on every device that loads the library
 *   until the process exits.  A shape whose pa_decode_workspace_bytes() is
 *   larger returns PA_EWORKSPACE (message in pa_last_cuda_error) and enqueues
 *   nothing.  The call allocates nothing.
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current and caches it with the
 *   id of the device's current context; make that first call before any
 *   stream capture.  A device reset (cudaDeviceReset) gives the device a new
 *   context, in which the library's module is loaded afresh; the next call
 *   sees the new context id and looks the address up again, so make the
 *   first call after a reset outside stream capture too.  A call with
 *   num_seqs = 0 does only this set-up and enqueues nothing.
 *   Errors: the argument checks of pa_decode run first, on the host alone.
 *   The scratch size check follows; it asks the CUDA runtime for the
 *   device's SM count (the split-K partition size depends on it), which
 *   can replace a runtime error the caller left pending on this thread.
 *   Neither check enqueues anything.
 *   Sharing: every call on a device uses the same array, which keeps the last
 *   call's contents (nothing in it needs to start at zero).  Calls that may
 *   overlap on the GPU (other streams, other host threads) race on it:
 *   serialise them, or use pa_decode with separate workspaces.
 */
#define PA_DECODE_STATIC_WS_BYTES (8u * 1024u * 1024u)
PA_API int pa_decode_static_ws(const void *q, const pa_cache_t *cache, const int32_t *block_tables,
                               int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                               int32_t max_seq_len, int32_t num_q_heads, float scale, void *out,
                               void *stream);

/* ------------------------------------------------------------------------
 * FP8 KV cache ("The pantry of pigeonholes", "The 10 knobs", knob 4
 * kv_cache_dtype, and "How it connects to the rest of the stack": one-byte
 * codes take half the bytes of bf16 for every cached token).  Codes are OCP FP8 E4M3 (one byte,
 * bias 7, no infinities, largest finite 448); a code c of the K (V) tensor
 * stands for value(c) * k_scale (v_scale), one scale per tensor.
 * ------------------------------------------------------------------------ */
typedef struct pa_cache_fp8 {
    void *k_cache; /* [num_blocks][block_size][num_kv_heads][head_dim] e4m3 codes */
    void *v_cache;
    int64_t num_blocks;
    int32_t block_size;
    int32_t num_kv_heads;
    int32_t head_dim;
    float k_scale; /* > 0 */
    float v_scale; /* > 0 */
} pa_cache_fp8_t;

/* pa_write_kv into an FP8 cache: each bf16 value x is stored as the code of
 * x / scale, the quotient in fp32 (IEEE division), rounded to the nearest
 * e4m3 value with ties to even and saturated at +-448 (infinities too).
 * Slots as pa_write_kv (negative = padding; out of range flagged). */
PA_API int pa_write_kv_fp8(const void *k, const void *v, const int64_t *slot_mapping, int64_t num_tokens,
                           const pa_cache_fp8_t *cache, void *stream);
/* pa_decode over an FP8 cache: same contract and output as pa_decode, with
 * K = value(code) * k_scale and V = value(code) * v_scale.  q and out stay
 * bf16.  Scratch per pa_decode_fp8_workspace_bytes.  The codes go into e4m3
 * tensor-core MMAs as they are; q (scaled per head by a power of two) and the
 * softmax weights enter as sums of two e4m3 numbers (exact for bf16 q, 8
 * significant bits for the weights, as bf16 weights have in pa_decode), so
 * the result is within pa_decode's tolerance of the exact one.  A scale that
 * is not positive and finite gives PA_EINVAL. */
/* pa_copy_blocks_fp8 -- pa_copy_blocks on an FP8 cache: the same whole-block
 * copy-on-write copies, bit for bit, of block_size * num_kv_heads * head_dim
 * one-byte codes per block and tensor (the scales are not used, but the
 * descriptor must be valid).  Pairs and error behaviour as pa_copy_blocks. */
PA_API int pa_copy_blocks_fp8(const pa_cache_fp8_t *cache, const int64_t *src_dst_pairs, int64_t num_pairs,
                              void *stream);
/* pa_copy_blocks_layers_fp8 -- pa_copy_blocks_fp8 for every layer in one
 * launch, as pa_copy_blocks_layers (caches: HOST array of num_layers <= 128
 * FP8 descriptors with one block geometry). */
PA_API int pa_copy_blocks_layers_fp8(const pa_cache_fp8_t *caches, int32_t num_layers,
                                     const int64_t *src_dst_pairs, int64_t num_pairs, void *stream);
PA_API size_t pa_decode_fp8_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t max_seq_len,
                                            const pa_cache_fp8_t *cache);
PA_API int pa_decode_fp8(const void *q, const pa_cache_fp8_t *cache, const int32_t *block_tables,
                         int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                         int32_t max_seq_len, int32_t num_q_heads, float scale, void *out, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Read (and with clear != 0, reset) the device error word of the current
 * device.  Synchronises the device.  Returns PA_OK or PA_ECUDA. */
PA_API int pa_get_device_error(int32_t *host_code, int clear);

/* The last CUDA error string seen by a PA_ECUDA return (static storage). */
PA_API const char *pa_last_cuda_error(void);
PA_API const char *pa_status_str(int status);

#ifdef __cplusplus
}
#endif
#endif /* PA_H */
