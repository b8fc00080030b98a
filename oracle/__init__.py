"""CPU oracle for the paged-KV decode path (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg (``bench.py --impl reference`` and the ``cpu_baseline`` field) may import
this package.  The product path never does: the CUDA library fails loudly
when it is missing instead of falling back to anything here.

Contents
--------
- ``pa_oracle.c`` (compiled to ``liboracle.so`` by :func:`build`): write,
  copy-on-write block copy, decode attention, attention of several query
  tokens per request (query_start_loc, causal) and the FP8 (E4M3) write and
  decode, in plain C, fp64.
- :func:`slot_of` / :func:`slot_mapping` / :func:`blocks_for` /
  :func:`tail_waste`: the slot, block-count and waste formulas, in Python.
- ``oracle.pool``: a pure-Python model of the block pool (free list,
  reference counts, append with copy-on-write, fork, release).

How each piece is pinned to something other than itself (the tests under
``tests/test_oracle_*.py`` and ``tests/test_pool*.py``):
- write / copy: worked examples, the fancy-index definition of the copy,
  negative-slot skipping, byte-exact NaN payload preservation;
- decode: the contiguous special case against ``torch``'s scaled dot-product
  attention in float64, closed forms (all-equal keys give the mean of V; one
  dominant key gives its V row; a single token gives V_0 exactly), invariance
  under any permutation of physical blocks and any block size, brute force on
  tiny inputs, NaN poison in unused storage;
- multi-token attention: whole and chunked prefill against ``torch``'s causal
  scaled dot-product attention in float64, one row per request equal to the
  decode, running means of V under all-equal keys, placement and block-size
  invariance;
- slot / block / waste formulas: the worked examples printed on the pages
  (slot 30,608 for request r7; cdiv(4097, 16) = 257; tail waste 15/1/0/15;
  the simulator's 4 blocks, 2 slots of slack, 50 slots of contiguous waste);
- pool: the pages' invariants, their CPU-allocator trace, and refcounts under
  sharing and copy-on-write.
No oracle function is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into liboracle.so (plain gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-o", _LIB_PATH, _SRC, "-lm"])
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        # ORACLE_LIB lets the mutation tests load a copy of the oracle with a
        # planted mistake; nothing else sets it.
        path = os.environ.get("ORACLE_LIB")
        if not path:
            build()
            path = _LIB_PATH
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        lib.oracle_write_kv.argtypes = [P, P, P, i64, i64, i64, P, P]
        lib.oracle_write_kv.restype = ctypes.c_int
        lib.oracle_copy_blocks.argtypes = [P, i64, i64, i64, P, P]
        lib.oracle_copy_blocks.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64,
                                      ctypes.c_double, P, i64, P]
        lib.oracle_decode.restype = ctypes.c_int
        lib.oracle_attention.argtypes = [P, P, P, P, i32, P, P, i32, i32, i32, i32, i32, i64,
                                         ctypes.c_double, P]
        lib.oracle_attention.restype = ctypes.c_int
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
        lib.oracle_write_kv_fp8.argtypes = [P, P, P, i64, i64, i64, ctypes.c_float, ctypes.c_float, P, P]
        lib.oracle_write_kv_fp8.restype = ctypes.c_int
        lib.oracle_decode_fp8.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_double, P]
        lib.oracle_decode_fp8.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _req(a, dtype):
    a = np.asarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    assert a.flags.c_contiguous
    return a


# ----------------------------------------------------------------------------
# Formulas of the paging scheme
# ----------------------------------------------------------------------------


def blocks_for(n: int, block_size: int) -> int:
    """ceil(n / B): blocks a sequence of n tokens occupies ("Memory
    management", Maths)."""
    return -(-n // block_size)


def tail_waste(n: int, block_size: int) -> int:
    """B*ceil(n/B) - n unused slots in the last block ("Memory management",
    Maths; "PagedAttention: fragmentation, blocks, block tables", Tail waste
    has a distribution)."""
    return block_size * blocks_for(n, block_size) - n


def slot_of(table_row, pos: int, block_size: int) -> int:
    """slot = table[pos // B] * B + pos % B ("PagedAttention: fragmentation,
    blocks, block tables", section 3 "The slot mapping")."""
    return int(table_row[pos // block_size]) * block_size + pos % block_size


def slot_mapping(table_rows, positions, block_size: int) -> np.ndarray:
    """One int64 slot per (row, position) pair; position -1 marks padding and
    maps to -1 (any negative value means "skip")."""
    out = np.empty(len(positions), dtype=np.int64)
    for i, (row, pos) in enumerate(zip(table_rows, positions)):
        out[i] = -1 if pos < 0 else slot_of(row, pos, block_size)
    return out


def map_to_kernel_blocks(block_table, blocks_per_alloc: int) -> np.ndarray:
    """Block table of allocation blocks -> block table of kernel blocks, m =
    blocks_per_alloc kernel blocks per allocation block ("PagedAttention:
    fragmentation, blocks, block tables": section 2 "The block table", where
    append_row maps the ids through map_to_kernel_blocks when the kernel's
    block is smaller, and the decoupling passage: allocation in larger units,
    say 32 tokens, while the attention kernel reads 16-token pages).  Storage is block-major, so
    allocation block a owns the bytes of kernel blocks a*m .. a*m + m - 1:
    entry i of a row becomes entries i*m .. i*m + m - 1.  Negative entries
    (padding) become m entries of -1."""
    t = np.asarray(block_table, dtype=np.int64)
    rows, width = t.shape
    out = np.full((rows, width * blocks_per_alloc), -1, dtype=np.int64)
    for r in range(rows):
        for i in range(width):
            a = int(t[r, i])
            if a < 0:
                continue
            for j in range(blocks_per_alloc):
                out[r, i * blocks_per_alloc + j] = a * blocks_per_alloc + j
    return out.astype(np.int32)


# ----------------------------------------------------------------------------
# Device operations, on host arrays
# ----------------------------------------------------------------------------


def write_kv(k, v, slots, k_cache, v_cache) -> None:
    """In place: k_cache.reshape(-1, H_kv*D)[slots[i]] = k[i] (same for V);
    negative slots skipped."""
    k = _req(k, np.uint16); v = _req(v, np.uint16); slots = _req(slots, np.int64)
    k_cache = _req(k_cache, np.uint16); v_cache = _req(v_cache, np.uint16)
    row = int(np.prod(k.shape[1:])) if k.ndim > 1 else 1
    num_slots = k_cache.size // row
    rc = _load().oracle_write_kv(_ptr(k), _ptr(v), _ptr(slots), len(slots), row, num_slots,
                                 _ptr(k_cache), _ptr(v_cache))
    if rc:
        raise ValueError("slot out of range")


def copy_blocks(pairs, k_cache, v_cache) -> None:
    """In place: cache[dst] = cache[src] for each (src, dst) pair, all sources
    read before any destination is written."""
    pairs = _req(np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2), np.int64)
    k_cache = _req(k_cache, np.uint16); v_cache = _req(v_cache, np.uint16)
    nb = k_cache.shape[0]
    rc = _load().oracle_copy_blocks(_ptr(pairs), len(pairs), k_cache.size // nb, nb,
                                    _ptr(k_cache), _ptr(v_cache))
    if rc:
        raise ValueError("block id out of range")


def decode(q, k_cache, v_cache, block_tables, seq_lens, scale: float, which=None) -> np.ndarray:
    """fp64 paged decode attention.  q: uint16 [S, H_q, D]; caches uint16
    [NB, B, H_kv, D]; block_tables int32 [S, W]; seq_lens int32 [S].  Returns
    float64 [S, H_q, D] (rows outside ``which`` are NaN)."""
    q = _req(q, np.uint16); k_cache = _req(k_cache, np.uint16); v_cache = _req(v_cache, np.uint16)
    block_tables = _req(np.ascontiguousarray(block_tables, dtype=np.int32), np.int32)
    seq_lens = _req(np.ascontiguousarray(seq_lens, dtype=np.int32), np.int32)
    S, Hq, D = q.shape
    NB, B, Hkv, D2 = k_cache.shape
    assert D2 == D and Hq % Hkv == 0 and len(seq_lens) == S and block_tables.shape[0] == S
    out = np.full((S, Hq, D), np.nan, dtype=np.float64)
    if which is not None:
        w = np.ascontiguousarray(which, dtype=np.int32).reshape(-1, 2)
        wp, nw = _ptr(w), len(w)
    else:
        w, wp, nw = None, None, 0
    rc = _load().oracle_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                               block_tables.shape[1], _ptr(seq_lens), S, Hq, Hkv, D, B, NB,
                               float(scale), wp, nw, _ptr(out))
    if rc == -1:
        raise ValueError("block id out of range or table too narrow")
    if rc:
        raise MemoryError("oracle_decode")
    return out


def attention(q, k_cache, v_cache, block_tables, query_start_loc, seq_lens, scale: float) -> np.ndarray:
    """fp64 attention of several query tokens per request over the paged cache
    (causal within each request: query row i of a request with q_len rows and
    n computed tokens attends to positions 0 .. n - q_len + i).  q: uint16
    [T, H_q, D] with T = query_start_loc[-1]; caches uint16 [NB, B, H_kv, D];
    block_tables int32 [R, W]; query_start_loc int32 [R + 1]; seq_lens int32
    [R].  Returns float64 [T, H_q, D]."""
    q = _req(q, np.uint16); k_cache = _req(k_cache, np.uint16); v_cache = _req(v_cache, np.uint16)
    block_tables = _req(np.ascontiguousarray(block_tables, dtype=np.int32), np.int32)
    qsl = _req(np.ascontiguousarray(query_start_loc, dtype=np.int32), np.int32)
    seq_lens = _req(np.ascontiguousarray(seq_lens, dtype=np.int32), np.int32)
    T, Hq, D = q.shape
    NB, B, Hkv, D2 = k_cache.shape
    R = len(seq_lens)
    assert D2 == D and Hq % Hkv == 0 and len(qsl) == R + 1 and block_tables.shape[0] == R
    assert qsl[0] == 0 and qsl[-1] == T
    out = np.full((T, Hq, D), np.nan, dtype=np.float64)
    rc = _load().oracle_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                  block_tables.shape[1], _ptr(qsl), _ptr(seq_lens), R, Hq, Hkv, D, B, NB,
                                  float(scale), _ptr(out))
    if rc == -1:
        raise ValueError("block id out of range or table too narrow")
    if rc == -3:
        raise ValueError("a request has more query rows than computed tokens")
    if rc:
        raise MemoryError("oracle_attention")
    return out


# ----------------------------------------------------------------------------
# FP8 (OCP E4M3) KV cache ("The pantry of pigeonholes", "The 10 knobs", knob 4)
# ----------------------------------------------------------------------------


def e4m3_to_float64(codes) -> np.ndarray:
    """Exact value of e4m3 codes (uint8 array)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_to_double(int(x)) for x in c.reshape(-1)], np.float64).reshape(c.shape)


def e4m3_from_float32(x) -> np.ndarray:
    """e4m3 codes of float32 values: nearest even, |x| >= 448 saturates, NaN -> 0x7F."""
    lib = _load()
    a = np.asarray(x, dtype=np.float32)
    return np.array([lib.oracle_e4m3_from_float(float(v)) for v in a.reshape(-1)], np.uint8).reshape(a.shape)


def write_kv_fp8(k, v, slots, k_cache, v_cache, k_scale: float, v_scale: float) -> None:
    """In place: codes of (bf16 row) / scale at the slots (negative = skip)."""
    k = _req(k, np.uint16); v = _req(v, np.uint16); slots = _req(slots, np.int64)
    k_cache = _req(k_cache, np.uint8); v_cache = _req(v_cache, np.uint8)
    row = int(np.prod(k.shape[1:]))
    rc = _load().oracle_write_kv_fp8(_ptr(k), _ptr(v), _ptr(slots), len(slots), row, k_cache.size // row,
                                     float(k_scale), float(v_scale), _ptr(k_cache), _ptr(v_cache))
    if rc:
        raise ValueError("slot out of range")


def decode_fp8(q, k_cache, v_cache, block_tables, seq_lens, scale: float, k_scale: float,
               v_scale: float) -> np.ndarray:
    """fp64 decode over an e4m3 cache (value = code value * scale of its tensor)."""
    q = _req(q, np.uint16); k_cache = _req(k_cache, np.uint8); v_cache = _req(v_cache, np.uint8)
    block_tables = _req(np.ascontiguousarray(block_tables, dtype=np.int32), np.int32)
    seq_lens = _req(np.ascontiguousarray(seq_lens, dtype=np.int32), np.int32)
    S, Hq, D = q.shape
    NB, B, Hkv, D2 = k_cache.shape
    assert D2 == D and Hq % Hkv == 0
    out = np.full((S, Hq, D), np.nan, dtype=np.float64)
    rc = _load().oracle_decode_fp8(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                   block_tables.shape[1], _ptr(seq_lens), S, Hq, Hkv, D, B, NB,
                                   float(scale), float(k_scale), float(v_scale), _ptr(out))
    if rc == -1:
        raise ValueError("block id out of range or table too narrow")
    if rc:
        raise MemoryError("oracle_decode_fp8")
    return out
