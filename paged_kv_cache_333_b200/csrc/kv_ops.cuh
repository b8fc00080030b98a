// The two data-movement kernels of the path: the slot-mapped KV write and
// the copy-on-write block copy.  Both are pure HBM traffic: 16-byte vector
// loads and stores, several in flight per thread, every access bounds-checked
// against the cache extent.
#pragma once

#include <cuda_fp8.h>

#include "pa_device.cuh"

namespace pa {

// ---------------------------------------------------------------------------
// pa_write_kv: one warp per (token, K|V).  A token's row of num_kv_heads *
// head_dim bf16 values is contiguous both in k/v and in the cache (the cache
// row index is the slot), so each warp moves one contiguous row.
// ("PagedAttention: fragmentation, blocks, block tables", section 3 "The
// slot mapping": the KV-cache write stores the token at flat row slot.)
// ---------------------------------------------------------------------------
constexpr int kWriteThreads = 256;

__global__ void __launch_bounds__(kWriteThreads)
write_kv_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                const int64_t *__restrict__ slot_mapping, int64_t num_tokens,
                uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache, int64_t num_slots,
                int row_vecs) {
    // Programmatic dependent launch: let the next kernel's CTAs get resident
    // now; touch global memory only once the preceding kernel is complete.
    grid_launch_dependents();
    grid_dependency_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kWriteThreads + threadIdx.x) >> 5;
    const int64_t tok = warp >> 1;
    if (tok >= num_tokens)
        return;
    const int64_t slot = slot_mapping[tok];
    if (slot < 0)
        return;  // padding
    if (slot >= num_slots) {
        if (lane == 0 && (warp & 1) == 0)
            flag_error(PA_DEVERR_SLOT);
        return;
    }
    const uint4 *src = ((warp & 1) ? v : k) + tok * row_vecs;
    uint4 *dst = ((warp & 1) ? v_cache : k_cache) + slot * row_vecs;
    // 4 loads in flight per lane before the stores (row_vecs is a multiple of 16).
    for (int base = 0; base < row_vecs; base += 128) {
        uint4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * 32 + lane;
            if (i < row_vecs)
                r[u] = __ldg(src + i);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * 32 + lane;
            if (i < row_vecs)
                dst[i] = r[u];
        }
    }
}

// ---------------------------------------------------------------------------
// Slot of a token from its request row and position ("PagedAttention:
// fragmentation, blocks, block tables", section 3 "The slot mapping":
// slot = block_table[req][pos / B] * B + pos % B; padded tokens get a negative
// PAD value).  Returns -1 for padding (pos < 0) and -2 for an argument that is
// out of range (request, table entry or block id), which the callers flag.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int64_t slot_of_position(int64_t pos, int32_t req,
                                                    const int32_t *__restrict__ block_tables,
                                                    int32_t max_blocks_per_seq, int32_t num_reqs,
                                                    int32_t block_size, int64_t num_blocks) {
    if (pos < 0)
        return -1;
    const int64_t lb = pos / block_size;
    if (req < 0 || req >= num_reqs || lb >= max_blocks_per_seq)
        return -2;
    const int64_t blk = block_tables[static_cast<int64_t>(req) * max_blocks_per_seq + lb];
    if (blk < 0 || blk >= num_blocks)
        return -2;
    return blk * block_size + pos % block_size;
}

constexpr int kSlotThreads = 256;

// pa_compute_slot_mapping: one thread per token.
__global__ void __launch_bounds__(kSlotThreads)
slot_mapping_kernel(const int64_t *__restrict__ positions, const int32_t *__restrict__ req_indices,
                    int64_t num_tokens, const int32_t *__restrict__ block_tables, int32_t max_blocks_per_seq,
                    int32_t num_reqs, int32_t block_size, int64_t num_blocks, int64_t *__restrict__ slot_mapping) {
    grid_launch_dependents();
    grid_dependency_wait();
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kSlotThreads + threadIdx.x;
    if (i >= num_tokens)
        return;
    int64_t slot = slot_of_position(positions[i], req_indices[i], block_tables, max_blocks_per_seq, num_reqs,
                                    block_size, num_blocks);
    if (slot == -2) {
        flag_error(PA_DEVERR_SLOT);
        slot = -1;  // written as padding: a later write skips it
    }
    slot_mapping[i] = slot;
}

// pa_map_to_kernel_blocks: one thread per output entry.  Allocation block a
// of a block-major cache owns the bytes of kernel blocks a*m .. a*m + m - 1,
// so entry i of a row becomes entries i*m .. i*m + m - 1 ("PagedAttention:
// fragmentation, blocks, block tables", section 2 "The block table",
// map_to_kernel_blocks; a 32-token allocation block feeding 16-token kernel
// pages).  Padding (< 0) and the columns past width * m become -1; an id
// whose kernel ids overflow int32 is flagged and written as -1.
__global__ void __launch_bounds__(kSlotThreads)
map_to_kernel_blocks_kernel(const int32_t *__restrict__ tables, int32_t num_rows, int32_t width,
                            int32_t blocks_per_alloc, int32_t *__restrict__ kernel_tables, int32_t kernel_width) {
    grid_launch_dependents();
    grid_dependency_wait();
    const int64_t e = static_cast<int64_t>(blockIdx.x) * kSlotThreads + threadIdx.x;
    if (e >= static_cast<int64_t>(num_rows) * kernel_width)
        return;
    const int64_t r = e / kernel_width;
    const int64_t c = e % kernel_width;
    int32_t id = -1;
    if (c < static_cast<int64_t>(width) * blocks_per_alloc) {
        const int32_t a = tables[r * width + c / blocks_per_alloc];
        if (a >= 0) {
            const int64_t k = static_cast<int64_t>(a) * blocks_per_alloc + c % blocks_per_alloc;
            if (k <= INT32_MAX)
                id = static_cast<int32_t>(k);
            else
                flag_error(PA_DEVERR_BLOCK_ID);
        }
    }
    kernel_tables[e] = id;
}

// pa_write_kv_positions: the KV write with the slot computed in-kernel from
// the token's request row and position (one warp per (token, K|V)).
__global__ void __launch_bounds__(kWriteThreads)
write_kv_positions_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                          const int64_t *__restrict__ positions, const int32_t *__restrict__ req_indices,
                          int64_t num_tokens, const int32_t *__restrict__ block_tables,
                          int32_t max_blocks_per_seq, int32_t num_reqs, int32_t block_size,
                          int64_t num_blocks, uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                          int row_vecs) {
    grid_launch_dependents();
    grid_dependency_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kWriteThreads + threadIdx.x) >> 5;
    const int64_t tok = warp >> 1;
    if (tok >= num_tokens)
        return;
    const int64_t slot = slot_of_position(positions[tok], req_indices[tok], block_tables, max_blocks_per_seq,
                                          num_reqs, block_size, num_blocks);
    if (slot < 0) {
        if (slot == -2 && lane == 0 && (warp & 1) == 0)
            flag_error(PA_DEVERR_SLOT);
        return;
    }
    const uint4 *src = ((warp & 1) ? v : k) + tok * row_vecs;
    uint4 *dst = ((warp & 1) ? v_cache : k_cache) + slot * row_vecs;
    for (int base = 0; base < row_vecs; base += 128) {
        uint4 r[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * 32 + lane;
            if (i < row_vecs)
                r[u] = __ldg(src + i);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = base + u * 32 + lane;
            if (i < row_vecs)
                dst[i] = r[u];
        }
    }
}

// ---------------------------------------------------------------------------
// pa_write_kv_fp8: the KV write into an FP8 (OCP E4M3) cache.  Each bf16
// value x becomes the code of x / scale: the quotient in fp32 (IEEE division),
// rounded to the nearest e4m3 value (ties to even), saturating at +-448.
// One warp per (token, K|V); a lane turns 8 bf16 (16 bytes) into 8 codes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kWriteThreads)
write_kv_fp8_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                    const int64_t *__restrict__ slot_mapping, int64_t num_tokens,
                    uint2 *__restrict__ k_cache, uint2 *__restrict__ v_cache, int64_t num_slots,
                    int row_vecs, float k_scale, float v_scale) {
    grid_launch_dependents();
    grid_dependency_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kWriteThreads + threadIdx.x) >> 5;
    const int64_t tok = warp >> 1;
    if (tok >= num_tokens)
        return;
    const int64_t slot = slot_mapping[tok];
    if (slot < 0)
        return;
    if (slot >= num_slots) {
        if (lane == 0 && (warp & 1) == 0)
            flag_error(PA_DEVERR_SLOT);
        return;
    }
    const bool is_v = warp & 1;
    const uint4 *src = (is_v ? v : k) + tok * row_vecs;
    uint2 *dst = (is_v ? v_cache : k_cache) + slot * row_vecs;
    const float sc = is_v ? v_scale : k_scale;
    for (int i = lane; i < row_vecs; i += 32) {
        const uint4 u = __ldg(src + i);
        float f[8];
        unpack8(u, f);
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t c = __nv_cvt_float_to_fp8(__fdiv_rn(f[e], sc), __NV_SATFINITE, __NV_E4M3);
            w[e >> 2] |= (c & 0xffu) << (8 * (e & 3));
        }
        dst[i] = make_uint2(w[0], w[1]);
    }
}

// ---------------------------------------------------------------------------
// pa_copy_blocks: grid = (num_pairs * 2 tensors * chunks_per_block).  Each CTA
// copies one chunk of up to kCopyChunkVecs 16-byte vectors of one block of one
// tensor; 4 vectors in flight per thread.  Pairs with an id outside
// [0, num_blocks) are skipped and flagged.
// ("PagedAttention: fragmentation, blocks, block tables", copy-on-write
// passage: blocks[dst] = blocks[src] over the block-major storage.)
// ---------------------------------------------------------------------------
constexpr int kCopyThreads = 256;
constexpr int kCopyChunkVecs = kCopyThreads * 4;

__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_kernel(uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                   const int64_t *__restrict__ pairs, int64_t num_blocks, int64_t block_vecs,
                   int chunks_per_block) {
    grid_launch_dependents();
    grid_dependency_wait();
    const int64_t item = blockIdx.x;
    const int chunk = static_cast<int>(item % chunks_per_block);
    const int64_t pt = item / chunks_per_block;  // pair * 2 + tensor
    const int64_t pair = pt >> 1;
    const int64_t src = pairs[2 * pair];
    const int64_t dst = pairs[2 * pair + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && chunk == 0 && (pt & 1) == 0)
            flag_error(PA_DEVERR_COPY_PAIR);
        return;
    }
    uint4 *base = (pt & 1) ? v_cache : k_cache;
    const uint4 *s = base + src * block_vecs;
    uint4 *d = base + dst * block_vecs;
    const int64_t begin = static_cast<int64_t>(chunk) * kCopyChunkVecs;
    const int64_t end = begin + kCopyChunkVecs < block_vecs ? begin + kCopyChunkVecs : block_vecs;
    uint4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t i = begin + u * kCopyThreads + threadIdx.x;
        if (i < end)
            r[u] = __ldcs(s + i);  // read once: streaming
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t i = begin + u * kCopyThreads + threadIdx.x;
        if (i < end)
            d[i] = r[u];
    }
}

// ---------------------------------------------------------------------------
// pa_copy_blocks_layers: the same copy for every layer of a model in one
// launch (grid.y = layer).  The layers' cache pointers travel in the kernel
// parameters.
// ---------------------------------------------------------------------------
constexpr int kMaxLayers = 128;

struct LayerPtrs {
    uint4 *k[kMaxLayers];
    uint4 *v[kMaxLayers];
};

__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_layers_kernel(const __grid_constant__ LayerPtrs layers, const int64_t *__restrict__ pairs,
                          int64_t num_blocks, int64_t block_vecs, int chunks_per_block) {
    grid_launch_dependents();
    grid_dependency_wait();
    const int64_t item = blockIdx.x;
    const int layer = blockIdx.y;
    const int chunk = static_cast<int>(item % chunks_per_block);
    const int64_t pt = item / chunks_per_block;  // pair * 2 + tensor
    const int64_t pair = pt >> 1;
    const int64_t src = pairs[2 * pair];
    const int64_t dst = pairs[2 * pair + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && chunk == 0 && (pt & 1) == 0 && layer == 0)
            flag_error(PA_DEVERR_COPY_PAIR);
        return;
    }
    uint4 *base = (pt & 1) ? layers.v[layer] : layers.k[layer];
    const uint4 *s = base + src * block_vecs;
    uint4 *d = base + dst * block_vecs;
    const int64_t begin = static_cast<int64_t>(chunk) * kCopyChunkVecs;
    const int64_t end = begin + kCopyChunkVecs < block_vecs ? begin + kCopyChunkVecs : block_vecs;
    uint4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t i = begin + u * kCopyThreads + threadIdx.x;
        if (i < end)
            r[u] = __ldcs(s + i);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t i = begin + u * kCopyThreads + threadIdx.x;
        if (i < end)
            d[i] = r[u];
    }
}

}  // namespace pa
