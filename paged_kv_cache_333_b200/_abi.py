"""ctypes binding of libpa.so (include/pa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (PyTorch provides device memory and
streams); each call passes ``data_ptr()`` and the current stream's handle.
Importing this module fails if libpa.so has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python paged_kv_cache_333_b200/build.py` "
                      "(there is no fallback path)")
lib = ctypes.CDLL(LIB_PATH)

PA_OK, PA_EINVAL, PA_EUNSUPPORTED, PA_EWORKSPACE, PA_ECUDA = 0, -1, -2, -3, -4
PA_DEVERR_SLOT, PA_DEVERR_BLOCK_ID, PA_DEVERR_SEQ_LEN, PA_DEVERR_COPY_PAIR, PA_DEVERR_TIMEOUT = 1, 2, 4, 8, 16
PA_DEVERR_QUERY_LOC = 32

EXPORTED = ("pa_write_kv", "pa_compute_slot_mapping", "pa_write_kv_positions", "pa_copy_blocks",
            "pa_copy_blocks_layers", "pa_decode_workspace_bytes", "pa_decode",
            "pa_map_to_kernel_blocks", "pa_decode_static_ws", "pa_attention_workspace_bytes", "pa_attention", "pa_write_kv_fp8", "pa_copy_blocks_fp8", "pa_copy_blocks_layers_fp8", "pa_decode_fp8", "pa_decode_fp8_workspace_bytes",
            "pa_decode_set_kernel", "pa_attention_set_kernel", "pa_decode_set_partition_tokens", "pa_get_device_error",
            "pa_last_cuda_error", "pa_status_str")
PA_DECODE_KERNEL_MMA, PA_DECODE_KERNEL_SIMT = 0, 1
PA_ATTENTION_KERNEL_MMA, PA_ATTENTION_KERNEL_TCGEN05, PA_ATTENTION_KERNEL_AUTO = 0, 1, 2
PA_ATTENTION_TCGEN05_MIN_COLUMNS = 17  # include/pa.h


class PaCache(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("num_blocks", ctypes.c_int64), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32)]


class PaCacheFp8(ctypes.Structure):
    _fields_ = [("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("num_blocks", ctypes.c_int64), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float)]


_P = ctypes.c_void_p
_i32, _i64 = ctypes.c_int32, ctypes.c_int64
lib.pa_write_kv.argtypes = [_P, _P, _P, _i64, ctypes.POINTER(PaCache), _P]
lib.pa_write_kv.restype = ctypes.c_int
lib.pa_compute_slot_mapping.argtypes = [_P, _P, _i64, _P, _i32, _i32, _i32, _i64, _P, _P]
lib.pa_compute_slot_mapping.restype = ctypes.c_int
lib.pa_write_kv_positions.argtypes = [_P, _P, _P, _P, _i64, _P, _i32, _i32, ctypes.POINTER(PaCache), _P]
lib.pa_write_kv_positions.restype = ctypes.c_int
lib.pa_copy_blocks.argtypes = [ctypes.POINTER(PaCache), _P, _i64, _P]
lib.pa_copy_blocks_layers.argtypes = [ctypes.POINTER(PaCache), _i32, _P, _i64, _P]
lib.pa_copy_blocks_layers.restype = ctypes.c_int
lib.pa_copy_blocks.restype = ctypes.c_int
lib.pa_decode_workspace_bytes.argtypes = [_i32, _i32, _i32, ctypes.POINTER(PaCache)]
lib.pa_decode_workspace_bytes.restype = ctypes.c_size_t
lib.pa_decode.argtypes = [_P, ctypes.POINTER(PaCache), _P, _i32, _P, _i32, _i32, _i32, ctypes.c_float,
                          _P, _P, ctypes.c_size_t, _P]
lib.pa_decode.restype = ctypes.c_int
lib.pa_decode_static_ws.argtypes = [_P, ctypes.POINTER(PaCache), _P, _i32, _P, _i32, _i32, _i32, ctypes.c_float,
                                    _P, _P]
lib.pa_decode_static_ws.restype = ctypes.c_int
lib.pa_map_to_kernel_blocks.argtypes = [_P, _i32, _i32, _i32, _P, _i32, _P]
lib.pa_map_to_kernel_blocks.restype = ctypes.c_int
lib.pa_attention_workspace_bytes.argtypes = [_i32, _i32, _i32, _i32, _i32, ctypes.POINTER(PaCache)]
lib.pa_attention_workspace_bytes.restype = ctypes.c_size_t
lib.pa_attention.argtypes = [_P, _i32, _P, _i32, _i32, ctypes.POINTER(PaCache), _P, _i32, _P, _i32, _i32,
                             ctypes.c_float, _P, _P, ctypes.c_size_t, _P]
lib.pa_attention.restype = ctypes.c_int
PA_DECODE_STATIC_WS_BYTES = 8 * 1024 * 1024
lib.pa_write_kv_fp8.argtypes = [_P, _P, _P, _i64, ctypes.POINTER(PaCacheFp8), _P]
lib.pa_write_kv_fp8.restype = ctypes.c_int
lib.pa_copy_blocks_fp8.argtypes = [ctypes.POINTER(PaCacheFp8), _P, _i64, _P]
lib.pa_copy_blocks_fp8.restype = ctypes.c_int
lib.pa_copy_blocks_layers_fp8.argtypes = [ctypes.POINTER(PaCacheFp8), _i32, _P, _i64, _P]
lib.pa_copy_blocks_layers_fp8.restype = ctypes.c_int
lib.pa_decode_fp8_workspace_bytes.argtypes = [_i32, _i32, _i32, ctypes.POINTER(PaCacheFp8)]
lib.pa_decode_fp8_workspace_bytes.restype = ctypes.c_size_t
lib.pa_decode_fp8.argtypes = [_P, ctypes.POINTER(PaCacheFp8), _P, _i32, _P, _i32, _i32, _i32, ctypes.c_float,
                              _P, _P, ctypes.c_size_t, _P]
lib.pa_decode_fp8.restype = ctypes.c_int
lib.pa_decode_set_kernel.argtypes = [_i32]
lib.pa_decode_set_kernel.restype = _i32
lib.pa_attention_set_kernel.argtypes = [_i32]
lib.pa_attention_set_kernel.restype = _i32
lib.pa_decode_set_partition_tokens.argtypes = [_i32]
lib.pa_decode_set_partition_tokens.restype = _i32
lib.pa_get_device_error.argtypes = [ctypes.POINTER(_i32), ctypes.c_int]
lib.pa_get_device_error.restype = ctypes.c_int
lib.pa_last_cuda_error.argtypes = []
lib.pa_last_cuda_error.restype = ctypes.c_char_p
lib.pa_status_str.argtypes = [ctypes.c_int]
lib.pa_status_str.restype = ctypes.c_char_p


class PaError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = f"{what}: {lib.pa_status_str(code).decode()} ({code})"
        if code == PA_ECUDA:
            msg += f": {lib.pa_last_cuda_error().decode()}"
        super().__init__(msg)
        self.code = code


def _check(rc: int, what: str) -> None:
    if rc != PA_OK:
        raise PaError(rc, what)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    dev = getattr(stream, "device", None)
    if dev is not None and dev.index != torch.cuda.current_device():
        raise ValueError(f"stream is on {dev}, but the current CUDA device is cuda:{torch.cuda.current_device()}")
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str, dtype) -> int:
    """Device pointer of a contiguous CUDA tensor of `dtype` on the current
    device: the library launches on the current device, where a pointer into
    another GPU's memory would be an illegal address."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}; call under torch.cuda.device({t.device})")
    return t.data_ptr()


def make_cache(k_cache: torch.Tensor, v_cache: torch.Tensor) -> PaCache:
    """Describe one layer's K and V caches ([num_blocks, block_size, H_kv, D] bf16)."""
    if k_cache.shape != v_cache.shape or k_cache.dim() != 4:
        raise ValueError("k_cache and v_cache must both be [num_blocks, block_size, num_kv_heads, head_dim]")
    nb, bs, hkv, d = k_cache.shape
    return PaCache(_dev(k_cache, "k_cache", torch.bfloat16), _dev(v_cache, "v_cache", torch.bfloat16),
                   nb, bs, hkv, d)


def make_cache_fp8(k_cache: torch.Tensor, v_cache: torch.Tensor, k_scale: float, v_scale: float) -> PaCacheFp8:
    """Describe one layer's FP8 (E4M3) caches: [num_blocks, block_size, H_kv, D]
    uint8 (or float8_e4m3fn) codes, value = code * scale of its tensor."""
    if k_cache.shape != v_cache.shape or k_cache.dim() != 4:
        raise ValueError("k_cache and v_cache must both be [num_blocks, block_size, num_kv_heads, head_dim]")
    kc = k_cache.view(torch.uint8) if k_cache.dtype != torch.uint8 else k_cache
    vc = v_cache.view(torch.uint8) if v_cache.dtype != torch.uint8 else v_cache
    nb, bs, hkv, d = k_cache.shape
    return PaCacheFp8(_dev(kc, "k_cache", torch.uint8), _dev(vc, "v_cache", torch.uint8), nb, bs, hkv, d,
                      float(k_scale), float(v_scale))


def pa_write_kv_fp8(k, v, slot_mapping, k_cache, v_cache, k_scale: float, v_scale: float, stream=None) -> None:
    """KV write into an FP8 cache: code of (bf16 value / scale), nearest even, saturating."""
    cache = make_cache_fp8(k_cache, v_cache, k_scale, v_scale)
    n = slot_mapping.numel()
    if k.shape != v.shape or k.shape[0] != n or tuple(k.shape[1:]) != tuple(k_cache.shape[2:]):
        raise ValueError("k, v must be [num_tokens, num_kv_heads, head_dim] matching slot_mapping and the cache")
    _check(lib.pa_write_kv_fp8(_dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
                               _dev(slot_mapping, "slot_mapping", torch.int64), n, ctypes.byref(cache),
                               _stream_ptr(stream)), "pa_write_kv_fp8")


def pa_copy_blocks_fp8(k_cache, v_cache, src_dst_pairs, stream=None) -> None:
    """cache[dst] = cache[src] for each (src, dst) row of an int64 [P, 2]
    tensor, on FP8 caches (whole blocks of one-byte codes)."""
    cache = make_cache_fp8(k_cache, v_cache, 1.0, 1.0)
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [num_pairs, 2]")
    p = src_dst_pairs.shape[0]
    ptr = _dev(src_dst_pairs, "src_dst_pairs", torch.int64) if p else None
    _check(lib.pa_copy_blocks_fp8(ctypes.byref(cache), ptr, p, _stream_ptr(stream)), "pa_copy_blocks_fp8")


def pa_copy_blocks_layers_fp8(caches, src_dst_pairs, stream=None) -> None:
    """pa_copy_blocks_fp8 over a list of (k_cache, v_cache) FP8 layers, one launch."""
    arr = (PaCacheFp8 * max(1, len(caches)))(*[make_cache_fp8(k, v, 1.0, 1.0) for k, v in caches])
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [num_pairs, 2]")
    p = src_dst_pairs.shape[0]
    ptr = _dev(src_dst_pairs, "src_dst_pairs", torch.int64) if p else None
    _check(lib.pa_copy_blocks_layers_fp8(arr, len(caches), ptr, p, _stream_ptr(stream)), "pa_copy_blocks_layers_fp8")


def pa_decode_fp8_workspace_bytes(num_seqs: int, num_q_heads: int, max_seq_len: int, k_cache, v_cache,
                                  k_scale: float = 1.0, v_scale: float = 1.0) -> int:
    cache = make_cache_fp8(k_cache, v_cache, k_scale, v_scale)
    return int(lib.pa_decode_fp8_workspace_bytes(num_seqs, num_q_heads, max_seq_len, ctypes.byref(cache)))


def pa_decode_fp8(q, k_cache, v_cache, k_scale: float, v_scale: float, block_tables, seq_lens, scale: float,
                  out=None, max_seq_len: int | None = None, workspace=None, stream=None) -> torch.Tensor:
    """pa_decode over an FP8 cache (q and out bf16)."""
    cache = make_cache_fp8(k_cache, v_cache, k_scale, v_scale)
    if q.dim() != 3 or q.shape[2] != k_cache.shape[3]:
        raise ValueError("q must be [num_seqs, num_q_heads, head_dim]")
    S, Hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be [num_seqs, W] and seq_lens [num_seqs]")
    if max_seq_len is None:
        max_seq_len = int(seq_lens.max().item()) if S else 0
    if out is None:
        out = torch.empty_like(q)
    need = int(lib.pa_decode_fp8_workspace_bytes(S, Hq, max_seq_len, ctypes.byref(cache)))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace", torch.uint8) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib.pa_decode_fp8(_dev(q, "q", torch.bfloat16), ctypes.byref(cache),
                             _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
                             _dev(seq_lens, "seq_lens", torch.int32), S, int(max_seq_len), Hq, float(scale),
                             _dev(out, "out", torch.bfloat16), ws_ptr, ws_bytes, _stream_ptr(stream)),
           "pa_decode_fp8")
    return out


def pa_write_kv(k, v, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """k_cache.view(-1, H_kv, D)[slot_mapping[i]] = k[i] (and V); negative slots skipped."""
    cache = make_cache(k_cache, v_cache)
    n = slot_mapping.numel()
    if k.shape != v.shape or k.shape[0] != n or tuple(k.shape[1:]) != tuple(k_cache.shape[2:]):
        raise ValueError("k, v must be [num_tokens, num_kv_heads, head_dim] matching slot_mapping and the cache")
    _check(lib.pa_write_kv(_dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
                           _dev(slot_mapping, "slot_mapping", torch.int64), n, ctypes.byref(cache),
                           _stream_ptr(stream)), "pa_write_kv")


def pa_compute_slot_mapping(positions, req_indices, block_tables, block_size: int, num_blocks: int,
                            slot_mapping=None, stream=None):
    """slot_mapping[i] = block_tables[req[i]][pos[i] // B] * B + pos[i] % B on
    the device (-1 for padding and for out-of-range tokens)."""
    n = positions.numel()
    if req_indices.numel() != n or block_tables.dim() != 2:
        raise ValueError("positions and req_indices need one entry per token; block_tables is [R, W]")
    if slot_mapping is None:
        slot_mapping = torch.empty(n, dtype=torch.int64, device=positions.device)
    _check(lib.pa_compute_slot_mapping(_dev(positions, "positions", torch.int64),
                                       _dev(req_indices, "req_indices", torch.int32), n,
                                       _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
                                       block_tables.shape[0], int(block_size), int(num_blocks),
                                       _dev(slot_mapping, "slot_mapping", torch.int64), _stream_ptr(stream)),
           "pa_compute_slot_mapping")
    return slot_mapping


def pa_write_kv_positions(k, v, positions, req_indices, block_tables, k_cache, v_cache, stream=None) -> None:
    """pa_write_kv with each token's slot computed in the kernel from its
    request row and position."""
    cache = make_cache(k_cache, v_cache)
    n = positions.numel()
    if k.shape != v.shape or k.shape[0] != n or tuple(k.shape[1:]) != tuple(k_cache.shape[2:]):
        raise ValueError("k, v must be [num_tokens, num_kv_heads, head_dim] matching positions and the cache")
    if req_indices.numel() != n or block_tables.dim() != 2:
        raise ValueError("req_indices needs one entry per token; block_tables is [R, W]")
    _check(lib.pa_write_kv_positions(_dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
                                     _dev(positions, "positions", torch.int64),
                                     _dev(req_indices, "req_indices", torch.int32), n,
                                     _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
                                     block_tables.shape[0], ctypes.byref(cache), _stream_ptr(stream)),
           "pa_write_kv_positions")


def pa_copy_blocks(k_cache, v_cache, src_dst_pairs, stream=None) -> None:
    """cache[dst] = cache[src] for each (src, dst) row of an int64 [P, 2] tensor."""
    cache = make_cache(k_cache, v_cache)
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [num_pairs, 2]")
    p = src_dst_pairs.shape[0]
    ptr = _dev(src_dst_pairs, "src_dst_pairs", torch.int64) if p else None
    _check(lib.pa_copy_blocks(ctypes.byref(cache), ptr, p, _stream_ptr(stream)), "pa_copy_blocks")


def pa_copy_blocks_layers(caches, src_dst_pairs, stream=None) -> None:
    """pa_copy_blocks over a list of (k_cache, v_cache) layers, one launch."""
    arr = (PaCache * max(1, len(caches)))(*[make_cache(k, v) for k, v in caches])
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [num_pairs, 2]")
    p = src_dst_pairs.shape[0]
    ptr = _dev(src_dst_pairs, "src_dst_pairs", torch.int64) if p else None
    _check(lib.pa_copy_blocks_layers(arr, len(caches), ptr, p, _stream_ptr(stream)), "pa_copy_blocks_layers")


def pa_decode_workspace_bytes(num_seqs: int, num_q_heads: int, max_seq_len: int, k_cache, v_cache) -> int:
    cache = make_cache(k_cache, v_cache)
    return int(lib.pa_decode_workspace_bytes(num_seqs, num_q_heads, max_seq_len, ctypes.byref(cache)))


def pa_decode(q, k_cache, v_cache, block_tables, seq_lens, scale: float, out=None,
              max_seq_len: int | None = None, workspace=None, stream=None) -> torch.Tensor:
    """Decode attention over the paged cache; returns ``out`` ([S, H_q, D] bf16).

    ``max_seq_len`` is a host-side upper bound of ``seq_lens``; when omitted it
    is read from the device (a synchronisation).  ``workspace`` (uint8 CUDA
    tensor) is allocated here when omitted and needed."""
    cache = make_cache(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != k_cache.shape[3]:
        raise ValueError("q must be [num_seqs, num_q_heads, head_dim]")
    S, Hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be [num_seqs, W] and seq_lens [num_seqs]")
    if max_seq_len is None:
        max_seq_len = int(seq_lens.max().item()) if S else 0
    if out is None:
        out = torch.empty_like(q)
    need = int(lib.pa_decode_workspace_bytes(S, Hq, max_seq_len, ctypes.byref(cache)))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace", torch.uint8) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib.pa_decode(_dev(q, "q", torch.bfloat16), ctypes.byref(cache),
                         _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
                         _dev(seq_lens, "seq_lens", torch.int32), S, int(max_seq_len), Hq,
                         float(scale), _dev(out, "out", torch.bfloat16), ws_ptr, ws_bytes,
                         _stream_ptr(stream)), "pa_decode")
    return out


def pa_map_to_kernel_blocks(block_tables, blocks_per_alloc: int, out=None, stream=None) -> torch.Tensor:
    """[R, W] int32 allocation-block table -> [R, W * m] kernel-block table
    (entry i*m + j = table[i]*m + j; padding stays -1)."""
    if block_tables.dim() != 2:
        raise ValueError("block_tables must be [num_rows, width]")
    R, W = block_tables.shape
    if out is None:
        out = torch.empty((R, W * blocks_per_alloc), dtype=torch.int32, device=block_tables.device)
    _check(lib.pa_map_to_kernel_blocks(_dev(block_tables, "block_tables", torch.int32), R, W, int(blocks_per_alloc),
                                       _dev(out, "out", torch.int32), out.shape[1], _stream_ptr(stream)),
           "pa_map_to_kernel_blocks")
    return out


def pa_attention_workspace_bytes(num_reqs: int, num_tokens: int, max_query_len: int, num_q_heads: int,
                                 max_seq_len: int, k_cache, v_cache) -> int:
    cache = make_cache(k_cache, v_cache)
    return int(lib.pa_attention_workspace_bytes(num_reqs, num_tokens, max_query_len, num_q_heads, max_seq_len,
                                                ctypes.byref(cache)))


def pa_attention(q, query_start_loc, k_cache, v_cache, block_tables, seq_lens, scale: float,
                 max_query_len: int, out=None, max_seq_len: int | None = None, workspace=None,
                 stream=None) -> torch.Tensor:
    """Attention of several query rows per request (the last q_len tokens of
    each, causal); returns ``out`` ([num_tokens, H_q, D] bf16).

    ``query_start_loc`` is int32 [num_reqs + 1] on the device;
    ``max_query_len`` and ``max_seq_len`` are host-side upper bounds (the
    latter read from the device when omitted, a synchronisation)."""
    cache = make_cache(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != k_cache.shape[3]:
        raise ValueError("q must be [num_tokens, num_q_heads, head_dim]")
    T, Hq, _ = q.shape
    R = seq_lens.shape[0]
    if query_start_loc.shape != (R + 1,) or block_tables.dim() != 2 or block_tables.shape[0] != R:
        raise ValueError("query_start_loc must be [num_reqs + 1], block_tables [num_reqs, W]")
    if max_seq_len is None:
        max_seq_len = int(seq_lens.max().item()) if R else 0
    if out is None:
        out = torch.empty_like(q)
    need = int(lib.pa_attention_workspace_bytes(R, T, int(max_query_len), Hq, int(max_seq_len),
                                                ctypes.byref(cache)))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace", torch.uint8) if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib.pa_attention(_dev(q, "q", torch.bfloat16), T, _dev(query_start_loc, "query_start_loc", torch.int32),
                            R, int(max_query_len), ctypes.byref(cache),
                            _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
                            _dev(seq_lens, "seq_lens", torch.int32), int(max_seq_len), Hq, float(scale),
                            _dev(out, "out", torch.bfloat16), ws_ptr, ws_bytes, _stream_ptr(stream)),
           "pa_attention")
    return out


def pa_decode_static_ws(q, k_cache, v_cache, block_tables, seq_lens, scale: float, out=None,
                        max_seq_len: int | None = None, stream=None) -> torch.Tensor:
    """pa_decode for callers that cannot allocate device memory: the split-K
    scratch lives in the library's fixed device array (8 MiB per device), so
    no workspace is passed or allocated (``out`` is still the caller's).
    Calls that overlap on the GPU share that array and must be serialised."""
    cache = make_cache(k_cache, v_cache)
    if q.dim() != 3 or q.shape[2] != k_cache.shape[3]:
        raise ValueError("q must be [num_seqs, num_q_heads, head_dim]")
    S, Hq, _ = q.shape
    if block_tables.dim() != 2 or block_tables.shape[0] != S or seq_lens.shape != (S,):
        raise ValueError("block_tables must be [num_seqs, W] and seq_lens [num_seqs]")
    if max_seq_len is None:
        max_seq_len = int(seq_lens.max().item()) if S else 0
    if out is None:
        raise ValueError("out must be given: this call allocates nothing")
    _check(lib.pa_decode_static_ws(_dev(q, "q", torch.bfloat16), ctypes.byref(cache),
                                   _dev(block_tables, "block_tables", torch.int32), block_tables.shape[1],
                                   _dev(seq_lens, "seq_lens", torch.int32), S, int(max_seq_len), Hq,
                                   float(scale), _dev(out, "out", torch.bfloat16), _stream_ptr(stream)),
           "pa_decode_static_ws")
    return out


def pa_decode_set_kernel(kind: str) -> str:
    """Select the decode partition kernel: "mma" (default) or "simt"; returns the previous one."""
    prev = lib.pa_decode_set_kernel({"mma": PA_DECODE_KERNEL_MMA, "simt": PA_DECODE_KERNEL_SIMT}[kind])
    return "mma" if prev == PA_DECODE_KERNEL_MMA else "simt"


_ATTENTION_KERNELS = {"mma": PA_ATTENTION_KERNEL_MMA, "tcgen05": PA_ATTENTION_KERNEL_TCGEN05,
                      "auto": PA_ATTENTION_KERNEL_AUTO}


def pa_attention_set_kernel(kind: str) -> str:
    """Select the pa_attention kernel: "auto" (default: "tcgen05" from
    PA_ATTENTION_TCGEN05_MIN_COLUMNS (row, head) columns per request, else
    "mma"), "mma" (8 columns per warp on mma.sync) or "tcgen05" (persistent,
    work units of 128 MMA rows, S, P and O in tensor memory); returns the
    previous setting.  The setting is process-wide."""
    prev = lib.pa_attention_set_kernel(_ATTENTION_KERNELS[kind])
    return {v: k for k, v in _ATTENTION_KERNELS.items()}[prev]


def pa_decode_set_partition_tokens(tokens: int) -> int:
    """0 = automatic split-K partition size; else tokens per partition (multiple of 64)."""
    return int(lib.pa_decode_set_partition_tokens(int(tokens)))


def pa_get_device_error(clear: bool = False) -> int:
    code = _i32(0)
    _check(lib.pa_get_device_error(ctypes.byref(code), 1 if clear else 0), "pa_get_device_error")
    return int(code.value)
