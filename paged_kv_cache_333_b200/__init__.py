"""Paged-KV decode path for NVIDIA B200 (sm_100a).

The device path is the C-ABI library ``libpa.so`` (include/pa.h): slot-mapped
KV write, copy-on-write block copy, paged decode attention (bf16 and FP8
caches) and attention of several query tokens per request, all in
hand-written CUDA kernels.  ``libpa_pool.so`` (include/pa_pool.h) is the host
block pool that produces block tables, slot mappings and copy pairs.  The
Python functions here only marshal arguments; there is no fallback path, and
importing the package fails if the libraries have not been built
(``python paged_kv_cache_333_b200/build.py``).
"""
from ._abi import (PA_DEVERR_BLOCK_ID, PA_DEVERR_COPY_PAIR, PA_DEVERR_QUERY_LOC, PA_DEVERR_SEQ_LEN,
                   PA_DEVERR_SLOT, PA_DEVERR_TIMEOUT, PaError, make_cache, pa_attention,
                   pa_attention_workspace_bytes, pa_compute_slot_mapping, pa_copy_blocks,
                   pa_map_to_kernel_blocks,
                   pa_copy_blocks_layers, pa_decode,
                   pa_decode_set_kernel, pa_attention_set_kernel, pa_decode_set_partition_tokens, pa_decode_static_ws,
                   pa_decode_workspace_bytes, pa_get_device_error,
                   pa_decode_fp8, pa_decode_fp8_workspace_bytes, pa_write_kv, pa_write_kv_fp8, pa_copy_blocks_fp8, pa_copy_blocks_layers_fp8,
                   pa_write_kv_positions, make_cache_fp8)
from .pool import BlockPool, PoolError

__all__ = [
    "pa_attention", "pa_attention_workspace_bytes", "PA_DEVERR_QUERY_LOC", "pa_map_to_kernel_blocks",
    "pa_write_kv", "pa_write_kv_fp8", "pa_copy_blocks_fp8", "pa_copy_blocks_layers_fp8", "pa_decode_fp8", "pa_decode_fp8_workspace_bytes", "make_cache_fp8",
    "pa_write_kv_positions", "pa_compute_slot_mapping", "pa_copy_blocks", "pa_copy_blocks_layers", "pa_decode", "pa_decode_static_ws", "pa_decode_workspace_bytes",
    "pa_decode_set_kernel", "pa_attention_set_kernel", "pa_decode_set_partition_tokens", "pa_get_device_error", "make_cache", "PaError",
    "BlockPool", "PoolError", "PA_DEVERR_SLOT", "PA_DEVERR_BLOCK_ID", "PA_DEVERR_SEQ_LEN",
    "PA_DEVERR_COPY_PAIR", "PA_DEVERR_TIMEOUT",
]
