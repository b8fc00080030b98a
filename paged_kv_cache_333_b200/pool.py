"""ctypes binding of libpa_pool.so (include/pa_pool.h): the host block pool."""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa_pool.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python paged_kv_cache_333_b200/build.py`")
lib = ctypes.CDLL(LIB_PATH)

PA_POOL_OK, PA_POOL_EINVAL, PA_POOL_ENOSPACE, PA_POOL_ENOSEQ, PA_POOL_EEXIST, PA_POOL_EINVARIANT, \
    PA_POOL_ERANGE = 0, -1, -2, -3, -4, -5, -6
PA_COW_SHARED, PA_COW_INHERITED = 0, 1

EXPORTED = ("pa_pool_create", "pa_pool_destroy", "pa_pool_seq_create", "pa_pool_append", "pa_pool_append_batch",
            "pa_pool_step", "pa_pool_fork",
            "pa_pool_release", "pa_pool_num_pending_copies", "pa_pool_take_copies", "pa_pool_num_blocks",
            "pa_pool_block_size", "pa_pool_num_free", "pa_pool_seq_len", "pa_pool_seq_num_blocks",
            "pa_pool_refcount", "pa_pool_pins", "pa_pool_free_list", "pa_pool_block_table",
            "pa_pool_block_table_update", "pa_pool_seq_lens",
            "pa_pool_slots", "pa_pool_step_slots", "pa_pool_check", "pa_pool_status_str")

_P, _i32, _i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
lib.pa_pool_create.argtypes = [_i64, _i32, _P, _i32]
lib.pa_pool_create.restype = _P
lib.pa_pool_destroy.argtypes = [_P]
lib.pa_pool_destroy.restype = None
for _name, _args, _res in [
    ("pa_pool_seq_create", [_P, _i64], ctypes.c_int),
    ("pa_pool_append", [_P, _i64, _i64], ctypes.c_int),
    ("pa_pool_append_batch", [_P, _P, _i32, _i64], ctypes.c_int),
    ("pa_pool_step", [_P, _P, _i32, _i64, _P, _i64, _P, _P, _i32, _P, _P, _P], ctypes.c_int),
    ("pa_pool_fork", [_P, _i64, _i64], ctypes.c_int),
    ("pa_pool_release", [_P, _i64], ctypes.c_int),
    ("pa_pool_num_pending_copies", [_P], _i64),
    ("pa_pool_take_copies", [_P, _P, _i64], _i64),
    ("pa_pool_num_blocks", [_P], _i64),
    ("pa_pool_block_size", [_P], _i32),
    ("pa_pool_num_free", [_P], _i64),
    ("pa_pool_seq_len", [_P, _i64], _i64),
    ("pa_pool_seq_num_blocks", [_P, _i64], _i64),
    ("pa_pool_refcount", [_P, _i64], _i32),
    ("pa_pool_pins", [_P, _i64], _i32),
    ("pa_pool_free_list", [_P, _P, _i64], _i64),
    ("pa_pool_block_table", [_P, _P, _i32, _i32, _i32, _P], ctypes.c_int),
    ("pa_pool_block_table_update", [_P, _P, _i32, _i32, _i32, _P, _P], ctypes.c_int),
    ("pa_pool_seq_lens", [_P, _P, _i32, _P], ctypes.c_int),
    ("pa_pool_slots", [_P, _i64, _i64, _i64, _P], ctypes.c_int),
    ("pa_pool_step_slots", [_P, _P, _i32, _i64, _P], ctypes.c_int),
    ("pa_pool_check", [_P], ctypes.c_int),
]:
    getattr(lib, _name).argtypes = _args
    getattr(lib, _name).restype = _res
lib.pa_pool_status_str.argtypes = [ctypes.c_int]
lib.pa_pool_status_str.restype = ctypes.c_char_p


class PoolError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {lib.pa_pool_status_str(code).decode()} ({code})")
        self.code = code


def _ok(rc: int, what: str) -> int:
    if rc < 0:
        raise PoolError(int(rc), what)
    return rc


def _ptr(a: np.ndarray) -> int:
    """Address of a contiguous array's data, for a void* argument.  The caller
    keeps `a` referenced until the call returns (an address holds no reference)."""
    return a.ctypes.data


class BlockPool:
    """Host KV block pool.  ``append`` returns False (pool unchanged) when too
    few blocks are free; every other failure raises PoolError."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None, rule: str = "shared"):
        rule_id = {"shared": PA_COW_SHARED, "inherited": PA_COW_INHERITED}[rule]
        if free_order is not None:
            self._order = np.ascontiguousarray(free_order, dtype=np.int32)
            if self._order.shape != (num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
            fp = _ptr(self._order)
        else:
            fp = None
        self._h = lib.pa_pool_create(int(num_blocks), int(block_size), fp, rule_id)
        if not self._h:
            raise PoolError(PA_POOL_EINVAL, "pa_pool_create")
        self._destroy = lib.pa_pool_destroy  # kept: module globals may be gone when __del__ runs at exit
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._destroy(h)
            self._h = None

    # -- operations -------------------------------------------------------
    def create(self, seq_id: int) -> None:
        _ok(lib.pa_pool_seq_create(self._h, seq_id), "create")

    def append(self, seq_id: int, n: int) -> bool:
        rc = lib.pa_pool_append(self._h, seq_id, n)
        if rc == PA_POOL_ENOSPACE:
            return False
        _ok(rc, "append")
        return True

    def append_batch(self, seq_ids, n: int) -> bool:
        """append(seq, n) for every listed sequence, all or nothing; False
        (and nothing changed) when the pool cannot hold them all."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        rc = lib.pa_pool_append_batch(self._h, _ptr(ids), len(ids), n)
        if rc == PA_POOL_ENOSPACE:
            return False
        _ok(rc, "append_batch")
        return True

    def step(self, seq_ids, n: int, table: np.ndarray, synced: np.ndarray, slots: np.ndarray | None = None,
             lens: np.ndarray | None = None, pairs: np.ndarray | None = None):
        """The host side of one decode step in one call (pa_pool_step): append
        n tokens to every listed sequence, all or nothing, then hand out the
        queued copy pairs, the step's slot mapping and the lengths, and bring
        `table` (with `synced`, as block_table_update) up to date in place.
        Returns (pairs [k, 2] int64, slots [num_seqs * n] int64, lens int32),
        or None when the pool cannot hold the appends (nothing changed).
        `slots`, `lens` and `pairs` may be passed in to be reused."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        S = len(ids)
        if table.dtype != np.int32 or not table.flags.c_contiguous or table.ndim != 2 or table.shape[0] != S:
            raise ValueError("table must be a C-contiguous int32 [num_seqs, width] array")
        if synced.dtype != np.int32 or synced.shape != (S,) or not synced.flags.c_contiguous:
            raise ValueError("synced must be int32 [num_seqs]")
        if slots is None:
            slots = np.empty(S * n, dtype=np.int64)
        elif slots.dtype != np.int64 or slots.shape != (S * n,) or not slots.flags.c_contiguous:
            raise ValueError("slots must be int64 [num_seqs * n]")
        if lens is None:
            lens = np.empty(S, dtype=np.int32)
        elif lens.dtype != np.int32 or lens.shape != (S,) or not lens.flags.c_contiguous:
            raise ValueError("lens must be int32 [num_seqs]")
        if pairs is None:
            pairs = np.empty((S + _ok(lib.pa_pool_num_pending_copies(self._h), "num_pending_copies"), 2),
                             dtype=np.int64)
        elif pairs.dtype != np.int64 or pairs.ndim != 2 or pairs.shape[1] != 2 or not pairs.flags.c_contiguous:
            raise ValueError("pairs must be a C-contiguous int64 [capacity, 2] array")
        k = ctypes.c_int64(0)
        rc = lib.pa_pool_step(self._h, ids.ctypes.data, S, n, pairs.ctypes.data, pairs.shape[0], ctypes.byref(k),
                              slots.ctypes.data, table.shape[1], table.ctypes.data, synced.ctypes.data,
                              lens.ctypes.data)
        if rc == PA_POOL_ENOSPACE:
            return None
        _ok(rc, "step")
        return pairs[:k.value], slots, lens

    def step_into(self, buf: "StepBuffers") -> int | None:
        """pa_pool_step on a StepBuffers (its sequences, its n_tokens): the
        results land in buf.pairs[:k], buf.slots, buf.table (with buf.synced)
        and buf.lens.  Returns k, the number of copy pairs, or None when the
        pool cannot hold the appends (nothing changed)."""
        rc = lib.pa_pool_step(self._h, *buf._args)
        if rc == PA_POOL_ENOSPACE:
            return None
        _ok(rc, "step")
        return buf._k.value

    def fork(self, src: int, dst: int) -> None:
        _ok(lib.pa_pool_fork(self._h, src, dst), "fork")

    def release(self, seq_id: int) -> None:
        _ok(lib.pa_pool_release(self._h, seq_id), "release")

    def take_cow_pairs(self) -> np.ndarray:
        n = _ok(lib.pa_pool_num_pending_copies(self._h), "num_pending_copies")
        out = np.zeros((max(n, 1), 2), dtype=np.int64)
        got = _ok(lib.pa_pool_take_copies(self._h, _ptr(out), n), "take_copies")
        return out[:got]

    # -- queries ------------------------------------------------------------
    def num_free(self) -> int:
        return _ok(lib.pa_pool_num_free(self._h), "num_free")

    def seq_len(self, seq_id: int) -> int:
        return _ok(lib.pa_pool_seq_len(self._h, seq_id), "seq_len")

    def num_blocks_of(self, seq_id: int) -> int:
        return _ok(lib.pa_pool_seq_num_blocks(self._h, seq_id), "seq_num_blocks")

    def refcount(self, block: int) -> int:
        """Owner references (tables naming the block)."""
        return _ok(lib.pa_pool_refcount(self._h, block), "refcount")

    def pins(self, block: int) -> int:
        """Queued copies naming the block."""
        return _ok(lib.pa_pool_pins(self._h, block), "pins")

    def free_list(self) -> list[int]:
        out = np.zeros(self.num_blocks, dtype=np.int32)
        n = _ok(lib.pa_pool_free_list(self._h, _ptr(out), self.num_blocks), "free_list")
        return out[:n].tolist()

    def table(self, seq_id: int) -> list[int]:
        return self.block_table([seq_id], self.num_blocks_of(seq_id))[0].tolist()

    def block_table(self, seq_ids, width: int, pad: int = -1) -> np.ndarray:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        out = np.empty((len(ids), width), dtype=np.int32)
        _ok(lib.pa_pool_block_table(self._h, _ptr(ids), len(ids), width, pad, _ptr(out)), "block_table")
        return out

    def block_table_update(self, seq_ids, table: np.ndarray, synced: np.ndarray, pad: int = -1) -> None:
        """Bring `table` ([num_seqs, width] int32, C-contiguous) up to date in
        place, writing only the entries that can have changed since `synced`
        (int32 [num_seqs], entries already written per row; updated)."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        if table.dtype != np.int32 or not table.flags.c_contiguous or table.shape[0] != len(ids):
            raise ValueError("table must be a C-contiguous int32 [num_seqs, width] array")
        if synced.dtype != np.int32 or synced.shape != (len(ids),):
            raise ValueError("synced must be int32 [num_seqs]")
        _ok(lib.pa_pool_block_table_update(self._h, _ptr(ids), len(ids), table.shape[1], pad, _ptr(table),
                                           _ptr(synced)), "block_table_update")

    def seq_lens(self, seq_ids) -> np.ndarray:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        out = np.empty(len(ids), dtype=np.int32)
        _ok(lib.pa_pool_seq_lens(self._h, _ptr(ids), len(ids), _ptr(out)), "seq_lens")
        return out

    def slots(self, seq_id: int, pos0: int, count: int) -> np.ndarray:
        out = np.empty(count, dtype=np.int64)
        _ok(lib.pa_pool_slots(self._h, seq_id, pos0, count, _ptr(out)), "slots")
        return out

    def step_slots(self, seq_ids, tokens_per_seq: int) -> np.ndarray:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        out = np.empty(len(ids) * tokens_per_seq, dtype=np.int64)
        _ok(lib.pa_pool_step_slots(self._h, _ptr(ids), len(ids), tokens_per_seq, _ptr(out)), "step_slots")
        return out

    def check(self) -> None:
        _ok(lib.pa_pool_check(self._h), "check")


class StepBuffers:
    """The arrays of pa_pool_step for one fixed batch of sequences, allocated
    once and reused every step (their addresses are taken once, which is most
    of the host cost of a step through ctypes).  The table starts empty
    (synced 0), so the first step writes whole rows.
      ids     int64 [S]            the batch, in order
      table   int32 [S, width]     block table, kept up to date in place (pad -1)
      synced  int32 [S]            entries of each row already written
      slots   int64 [S * n_tokens] the step's slot mapping
      lens    int32 [S]            lengths after the step
      pairs   int64 [capacity, 2]  queued copy pairs handed out by the step"""

    def __init__(self, seq_ids, n_tokens: int, width: int, pairs_capacity: int | None = None):
        self.ids = np.array(seq_ids, dtype=np.int64)
        S = len(self.ids)
        self.n_tokens = int(n_tokens)
        self.table = np.full((S, int(width)), -1, dtype=np.int32)
        self.synced = np.zeros(S, dtype=np.int32)
        self.slots = np.empty(S * self.n_tokens, dtype=np.int64)
        self.lens = np.empty(S, dtype=np.int32)
        self.pairs = np.empty((S if pairs_capacity is None else int(pairs_capacity), 2), dtype=np.int64)
        self._k = ctypes.c_int64(0)
        self._args = (self.ids.ctypes.data, S, self.n_tokens, self.pairs.ctypes.data, self.pairs.shape[0],
                      ctypes.byref(self._k), self.slots.ctypes.data, int(width), self.table.ctypes.data,
                      self.synced.ctypes.data, self.lens.ctypes.data)
