"""Seeded synthetic inputs for the paged-KV decode path.

This module only draws random numbers and decides *which* pool operations a
workload performs (which sequences exist, how long they are, in what order
blocks sit on the free list).  It holds none of the method's arithmetic: no
block-count, slot or attention formula lives here.  Both sides of every parity
test (the CUDA path and the CPU oracle) take their inputs from here, and
nothing here imports either side.

Random stream: ``numpy.random.Generator(PCG64(seed))``.  Floating values are
drawn N(0, 1) in float32 and rounded to bfloat16 (round to nearest even); they
travel as ``uint16`` bit patterns.

Workload shapes follow the pages' setting (Llama-3-8B: 32 query heads, 8 KV
heads, head dim 128, 16-token blocks, a 26,785-block pool; chat turns of 512
prompt tokens and at most 100 generated ones; 32K-token contexts).  See
"PagedAttention: fragmentation, blocks, block tables", introduction, for the
pool and the chat turn, and "The pantry of pigeonholes", "The maths that
matter", for the per-token KV size.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Protocol, Sequence

import numpy as np

# ----------------------------------------------------------------------------
# bf16 bit handling (data conversion only)
# ----------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16
    bits, 0x7FC0 for every NaN.  (Add 0x7FFF plus the kept half's lowest bit,
    then drop the low 16 bits; done in place on one uint32 temporary.)"""
    shape = np.shape(x)
    a = np.ascontiguousarray(x, dtype=np.float32)
    u = a.reshape(-1).view(np.uint32)
    r = u >> 16
    r &= 1
    r += 0x7FFF
    r += u  # wraps only for NaN patterns, which are replaced below
    r >>= 16
    out = r.astype(np.uint16)
    nan = np.isnan(a.reshape(-1))
    if nan.any():
        out[nan] = 0x7FC0
    return out.reshape(shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) to float32 values (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


BF16_NAN = np.uint16(0x7FC1)  # a quiet-NaN payload used to poison unused storage


def make_rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_normal(gen: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) float32 draws rounded to bfloat16, as uint16 bits."""
    return f32_to_bf16_bits(gen.standard_normal(shape, dtype=np.float32))


# ----------------------------------------------------------------------------
# Workload configurations
# ----------------------------------------------------------------------------

LLAMA3_8B_POOL_BLOCKS = 26_785  # 52.32 GiB pool at block_size 16 (page 1 intro)
LLAMA3_8B_POOL_SLOTS = 428_560  # 26,785 x 16 token slots


@dataclasses.dataclass
class Shape:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


@dataclasses.dataclass
class Workload:
    """Everything a config draws.  Pool layouts are produced by replaying
    ``ops`` on a pool object (product or oracle); values are logical, i.e.
    indexed by (sequence, position), never by physical block."""

    name: str
    shape: Shape
    seed: int
    free_order: np.ndarray  # int32 [num_blocks]: initial free list, head first
    seq_ids: list[int]  # the decode batch, in batch order
    ops: Callable  # ops(pool) replays the setup on a pool; returns nothing
    step_tokens: int  # tokens appended per batch sequence in the timed step
    k_values: dict  # seq_id -> uint16 [len_after_step, H_kv, D] logical K
    v_values: dict  # seq_id -> uint16 [len_after_step, H_kv, D] logical V
    q: np.ndarray  # uint16 [S, H_q, D]
    scale: float
    notes: str = ""
    # Positions [0, shared_len) of every batch sequence hold shared_k/v
    # (prefix sharing); k_values/v_values then hold only the positions after.
    shared_len: int = 0
    shared_k: np.ndarray | None = None
    shared_v: np.ndarray | None = None
    suffix_ops: Callable | None = None  # replayed after the shared prefix is written

    def seq_total(self, sid: int) -> int:
        """Length of sequence sid after the step's token."""
        return self.shared_len + len(self.k_values[sid])

    def rows(self, which: str, sid: int, a: int, b: int) -> np.ndarray:
        """Logical K ("k") or V ("v") rows of positions [a, b) of sequence sid."""
        own = self.k_values[sid] if which == "k" else self.v_values[sid]
        if self.shared_len == 0:
            return own[a:b]
        sh = self.shared_k if which == "k" else self.shared_v
        parts = []
        if a < self.shared_len:
            parts.append(sh[a:min(b, self.shared_len)])
        if b > self.shared_len:
            parts.append(own[max(a, self.shared_len) - self.shared_len:b - self.shared_len])
        return parts[0] if len(parts) == 1 else np.concatenate(parts)


class PoolLike(Protocol):
    def create(self, seq_id: int) -> None: ...
    def append(self, seq_id: int, n: int) -> bool: ...
    def fork(self, src: int, dst: int) -> None: ...
    def release(self, seq_id: int) -> None: ...
    def num_free(self) -> int: ...
    def seq_len(self, seq_id: int) -> int: ...
    def num_blocks_of(self, seq_id: int) -> int: ...


def _values_for(gen, lens: dict, shape: Shape):
    k, v = {}, {}
    for sid in sorted(lens):
        k[sid] = bf16_normal(gen, (lens[sid], shape.num_kv_heads, shape.head_dim))
    for sid in sorted(lens):
        v[sid] = bf16_normal(gen, (lens[sid], shape.num_kv_heads, shape.head_dim))
    return k, v


def _scale(head_dim: int) -> float:
    return float(np.float32(1.0 / np.sqrt(head_dim)))


def tiny(seed: int = 333) -> Workload:
    """4 sequences with {1,17,33,100} tokens, 8 q / 2 KV heads, 64-block pool
    placed by a seeded permutation; the step appends one token to each."""
    gen = make_rng(seed)
    shape = Shape(8, 2, 128, 16, 64)
    free_order = gen.permutation(shape.num_blocks).astype(np.int32)
    lens0 = {0: 1, 1: 17, 2: 33, 3: 100}
    ids = [0, 1, 2, 3]

    def ops(pool: PoolLike):
        for sid in ids:
            pool.create(sid)
            assert pool.append(sid, lens0[sid])

    q = bf16_normal(gen, (len(ids), shape.num_q_heads, shape.head_dim))
    k, v = _values_for(gen, {s: lens0[s] + 1 for s in ids}, shape)
    return Workload("tiny", shape, seed, free_order, ids, ops, 1, k, v, q, _scale(128),
                    "4 seqs {1,17,33,100} -> {2,18,34,101}")


def chat(seed: int = 334, batch: int = 64, num_blocks: int = LLAMA3_8B_POOL_BLOCKS) -> Workload:
    """Llama-3-8B chat decode, one layer: batch 64, lengths uniform in
    [512, 612] (512-token prompt + 0..100 outputs) before the step's token,
    blocks drawn from a seeded shuffled free list of the full pool."""
    gen = make_rng(seed)
    shape = Shape(32, 8, 128, 16, num_blocks)
    free_order = gen.permutation(shape.num_blocks).astype(np.int32)
    lens = gen.integers(512, 613, size=batch)
    ids = list(range(batch))
    lens0 = {i: int(lens[i]) - 1 for i in ids}  # the step's token makes it [512, 612]

    def ops(pool: PoolLike):
        for sid in ids:
            pool.create(sid)
            assert pool.append(sid, lens0[sid])

    q = bf16_normal(gen, (batch, shape.num_q_heads, shape.head_dim))
    k, v = _values_for(gen, {s: lens0[s] + 1 for s in ids}, shape)
    return Workload("chat", shape, seed, free_order, ids, ops, 1, k, v, q, _scale(128),
                    "64 seqs, len U[512,612] incl. the step's token")


def long_context(seed: int = 335, lens=(32768,) * 4 + (8192,) * 4,
                 num_blocks: int = LLAMA3_8B_POOL_BLOCKS) -> Workload:
    """Long-context decode: 4 x 32768 and 4 x 8192 tokens (after the step's
    token), blocks scattered randomly over the 26,785-block pool."""
    gen = make_rng(seed)
    shape = Shape(32, 8, 128, 16, num_blocks)
    free_order = gen.permutation(shape.num_blocks).astype(np.int32)
    ids = list(range(len(lens)))
    lens0 = {i: int(lens[i]) - 1 for i in ids}

    def ops(pool: PoolLike):
        for sid in ids:
            pool.create(sid)
            assert pool.append(sid, lens0[sid])

    q = bf16_normal(gen, (len(ids), shape.num_q_heads, shape.head_dim))
    k, v = _values_for(gen, {s: lens0[s] + 1 for s in ids}, shape)
    return Workload("long", shape, seed, free_order, ids, ops, 1, k, v, q, _scale(128),
                    "8 seqs {32768 x4, 8192 x4} incl. the step's token")


def prefix_cow(seed: int = 336, batch: int = 256, prefix: int = 2040, max_suffix: int = 256,
               num_blocks: int = LLAMA3_8B_POOL_BLOCKS) -> Workload:
    """Prefix sharing + copy-on-write: sequence 0 holds a 2040-token prefix
    (127 full blocks + an 8-token tail); sequences 1..255 are forked from it,
    so every prefix block is referenced 256 times.  Each sequence then appends
    a unique suffix of 1..256 tokens (the last of them is the step's token);
    appending into the shared partial tail triggers copy-on-write."""
    gen = make_rng(seed)
    shape = Shape(32, 8, 128, 16, num_blocks)
    free_order = gen.permutation(shape.num_blocks).astype(np.int32)
    suffix = gen.integers(1, max_suffix + 1, size=batch)
    ids = list(range(batch))

    def ops(pool: PoolLike):
        pool.create(0)
        assert pool.append(0, prefix)
        for sid in ids[1:]:
            pool.fork(0, sid)

    def suffix_ops(pool: PoolLike):
        # everything but the step's token: suffix - 1 tokens
        for sid in ids:
            if suffix[sid] > 1:
                assert pool.append(sid, int(suffix[sid]) - 1)

    # The shared prefix values are drawn once; each sequence's logical K/V is
    # that prefix followed by its own suffix.
    pk = bf16_normal(gen, (prefix, shape.num_kv_heads, shape.head_dim))
    pv = bf16_normal(gen, (prefix, shape.num_kv_heads, shape.head_dim))
    q = bf16_normal(gen, (batch, shape.num_q_heads, shape.head_dim))
    k, v = {}, {}
    for sid in ids:
        k[sid] = bf16_normal(gen, (int(suffix[sid]), shape.num_kv_heads, shape.head_dim))
        v[sid] = bf16_normal(gen, (int(suffix[sid]), shape.num_kv_heads, shape.head_dim))
    return Workload("prefix", shape, seed, free_order, ids, ops, 1, k, v, q, _scale(128),
                    "256 seqs sharing a 2040-token prefix; suffix U[1,256]",
                    shared_len=prefix, shared_k=pk, shared_v=pv, suffix_ops=suffix_ops)


def sweep(block_size: int, seed: int = 337, batch: int = 128, mean_len: int = 1000,
          cap: int = 8192, events: int = 10_000, occupancy: float = 0.9,
          slots: int = LLAMA3_8B_POOL_SLOTS) -> Workload:
    """Block-size sweep under fragmentation.  The pool keeps the same token
    capacity for every block size (num_blocks = floor(428,560 / block_size), as
    page 1's list of experiments halves the block count when the block size
    doubles).  Churn: ``events``
    seeded events on background sequences, each either a create with a
    Geometric(1/mean_len) length capped at ``cap`` tokens or the release of a
    random live background sequence; then the batch of ``batch`` sequences
    (same length law) is allocated; then background sequences are added or
    released until exactly floor(occupancy * num_blocks) blocks are in use.

    The random draws do not depend on block_size, so every block size sees
    the same logical sequences and the same K/V values."""
    gen = make_rng(seed)
    nb = slots // block_size
    shape = Shape(32, 8, 128, block_size, nb)
    # Draw everything block-size independent first.
    perm_seed = int(gen.integers(0, 2**31 - 1))
    ev_kind = gen.random(events)
    ev_len = np.minimum(gen.geometric(1.0 / mean_len, size=events), cap)
    ev_pick = gen.random(events)
    batch_len = np.minimum(gen.geometric(1.0 / mean_len, size=batch), cap)
    fill_len = np.minimum(gen.geometric(1.0 / mean_len, size=4096), cap)
    fill_pick = gen.random(4096)
    free_order = make_rng(perm_seed).permutation(nb).astype(np.int32)
    ids = list(range(batch))
    BG = 1_000_000  # background sequence ids start here

    def ops(pool: PoolLike):
        live: list[int] = []
        nxt = BG
        for j in range(events):
            if ev_kind[j] < 0.5 or not live:
                pool.create(nxt)
                if pool.append(nxt, int(ev_len[j])):
                    live.append(nxt)
                else:
                    pool.release(nxt)
                nxt += 1
            else:
                victim = live.pop(int(ev_pick[j] * len(live)))
                pool.release(victim)
        # the decode batch; release background sequences until it fits
        for sid in ids:
            pool.create(sid)
            while not pool.append(sid, int(batch_len[sid]) - 1):
                victim = live.pop(int(fill_pick[sid] * len(live)))
                pool.release(victim)
        # reach exactly floor(occupancy * nb) blocks in use; the 10% left
        # free always covers the step's one new block per batch sequence.
        target = int(occupancy * nb)
        j = 0
        while nb - pool.num_free() > target and live:
            victim = live.pop(int(fill_pick[j % 4096] * len(live)))
            pool.release(victim)
            j += 1
        while nb - pool.num_free() < target:
            need_blocks = target - (nb - pool.num_free())
            want = int(fill_len[j % 4096])
            pool.create(nxt)
            # whole blocks only, never more than needed
            n_tok = min(want, need_blocks * block_size)
            n_tok = max(block_size, (n_tok // block_size) * block_size)
            ok = pool.append(nxt, n_tok)
            assert ok
            live.append(nxt)
            nxt += 1
            j += 1

    q = bf16_normal(gen, (batch, shape.num_q_heads, shape.head_dim))
    lens_after = {i: int(batch_len[i]) for i in ids}
    k, v = _values_for(gen, lens_after, shape)
    return Workload(f"sweep_b{block_size}", shape, seed, free_order, ids, ops, 1, k, v, q,
                    _scale(128), f"B={block_size}, 128 seqs geometric mean {mean_len} cap {cap}")


BUILDERS = {
    "tiny": tiny,
    "chat": chat,
    "long": long_context,
    "prefix": prefix_cow,
}


def by_name(name: str) -> Workload:
    if name.startswith("sweep_b"):
        return sweep(int(name[len("sweep_b"):]))
    return BUILDERS[name]()


# ----------------------------------------------------------------------------
# Small random op streams for allocator property tests
# ----------------------------------------------------------------------------


def random_pool_ops(seed: int, n_ops: int = 200, max_append: int = 9):
    """A replayable list of (op, args) tuples: create / append / fork / release
    over a handful of request ids.  Used by the randomized allocator tests."""
    gen = make_rng(seed)
    out = []
    next_id = 0
    for _ in range(n_ops):
        r = gen.random()
        a = int(gen.integers(0, 1 << 30))
        b = int(gen.integers(1, max_append + 1))
        if r < 0.2:
            out.append(("create", next_id))
            next_id += 1
        elif r < 0.7:
            out.append(("append", a, b))
        elif r < 0.85:
            out.append(("fork", a, next_id))
            next_id += 1
        else:
            out.append(("release", a))
    return out
