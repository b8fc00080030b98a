"""Pure-Python model of the KV block pool (TEST INFRASTRUCTURE).

A slow, list-based restatement of the allocator the pages describe, used to
check the product's C++ pool operation by operation:

- one free queue, allocation pops its head, and a failed allocation changes
  nothing ("PagedAttention: fragmentation, blocks, block tables", section 1
  "The block pool": get_new_blocks pops the head of the free queue and
  refuses when too few blocks are free);
- freeing decrements reference counts and puts blocks that reach zero back at
  the FRONT of the queue, as one run in the order given (same section:
  blocks without a hash go back to the head, so the newest free block is
  reused first); a released request gives its blocks back last block first
  (same section, SingleTypeKVCacheManager.free);
- a sequence owns a list of block ids; position p lives in block p // B at
  offset p % B (section 2 "The block table"), and its slot is
  table[p // B] * B + p % B (section 3 "The slot mapping");
- fork shares every block by reference count; sharing whole blocks takes
  no copy (copy-on-write passage of the same page; the CPU reference
  allocator's fork);
- append allocates ceil((len + n) / B) - len(table) new blocks and, when the
  tail is partial and shared, first redirects the tail to a fresh block and
  queues a (src, dst) copy ("Memory management", Code: copy iff len % B != 0
  and refs[last] > 1; the needed count includes the copy's block; a refused
  append changes nothing).  The alternative trigger of page 1 (copy whenever
  the partial tail was not allocated by this sequence, i.e. on every partial
  hit) is selectable with rule="inherited";
- both endpoints of a queued copy stay retained until the copy is taken for
  execution (copy-on-write passage of page 1: the source and destination
  are held until the copy has been carried out).  Such a retention is kept apart from
  the owner references, as page 1's "Two kinds of references" keeps transfer
  pins apart from owners: the copy-on-write trigger counts owners (tables
  naming the block) only, and a block is free only when it has neither
  owners nor pins.
"""
from __future__ import annotations

import copy
from collections import deque

from . import blocks_for, slot_of

RULE_SHARED = "shared"  # copy iff tail partial and refcount > 1 (page 3)
RULE_INHERITED = "inherited"  # copy iff tail partial and inherited (page 1)


class PoolError(Exception):
    pass


class RefPool:
    def __init__(self, num_blocks: int, block_size: int, free_order=None, rule: str = RULE_SHARED):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        self.rule = rule
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        assert sorted(order) == list(range(num_blocks))
        self.free = deque(order)  # head first
        self.ref = [0] * num_blocks  # owner references: tables naming the block
        self.pin = [0] * num_blocks  # queued copies naming the block
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.tail_owned: dict[int, bool] = {}
        self.pending: list[tuple[int, int]] = []

    # -- primitives --------------------------------------------------------
    def _take(self, n: int) -> list[int]:
        got = [self.free.popleft() for _ in range(n)]
        for b in got:
            assert self.ref[b] == 0 and self.pin[b] == 0
            self.ref[b] = 1
        return got

    def _release_refs(self, ordered: list[int], counts: list[int]) -> None:
        """Drop one reference of each block (from `counts`, which is self.ref
        or self.pin); blocks left with no owner and no pin are pushed back at
        the head of the free queue together, keeping the given order."""
        run = []
        for b in ordered:
            counts[b] -= 1
            assert counts[b] >= 0
            if self.ref[b] == 0 and self.pin[b] == 0:
                run.append(b)
        self.free.extendleft(reversed(run))

    # -- sequence operations ----------------------------------------------
    def create(self, seq_id: int) -> None:
        if seq_id in self.tables:
            raise PoolError("sequence exists")
        self.tables[seq_id] = []
        self.lens[seq_id] = 0
        self.tail_owned[seq_id] = True

    def append(self, seq_id: int, n: int) -> bool:
        table = self.tables[seq_id]
        length = self.lens[seq_id]
        B = self.block_size
        needed = blocks_for(length + n, B) - len(table)
        partial = bool(table) and length % B != 0 and n > 0
        if self.rule == RULE_SHARED:
            cow = partial and self.ref[table[-1]] > 1
        else:
            cow = partial and not self.tail_owned[seq_id]
        if needed + (1 if cow else 0) > len(self.free):
            return False
        if cow:
            src = table[-1]
            (dst,) = self._take(1)
            # the sequence stops owning src; both ends are pinned until the
            # copy is handed to the device
            self.ref[src] -= 1
            self.pin[src] += 1
            self.pin[dst] += 1
            table[-1] = dst
            self.pending.append((src, dst))
            self.tail_owned[seq_id] = True
        if needed > 0:
            table.extend(self._take(needed))
            self.tail_owned[seq_id] = True
        self.lens[seq_id] = length + n
        return True

    def append_batch(self, seq_ids, n: int) -> bool:
        """One scheduler step: append(seq, n) for every listed sequence in
        order, all or nothing (a failed call leaves the state unchanged,
        "PagedAttention: fragmentation, blocks, block tables", the allocator
        invariants).  Written as snapshot, sequential appends, restore."""
        if len(set(seq_ids)) != len(seq_ids):
            raise ValueError("a sequence listed twice")
        for sid in seq_ids:
            if sid not in self.tables:
                raise KeyError(sid)
        saved = copy.deepcopy(self.__dict__)
        for sid in seq_ids:
            if not self.append(sid, n):
                self.__dict__.clear()
                self.__dict__.update(saved)
                return False
        return True

    def fork(self, src: int, dst: int) -> None:
        if dst in self.tables:
            raise PoolError("sequence exists")
        for b in self.tables[src]:
            self.ref[b] += 1
        self.tables[dst] = list(self.tables[src])
        self.lens[dst] = self.lens[src]
        self.tail_owned[dst] = not self.tables[src]  # an empty table owns nothing

    def release(self, seq_id: int) -> None:
        table = self.tables.pop(seq_id)
        del self.lens[seq_id]
        del self.tail_owned[seq_id]
        self._release_refs(list(reversed(table)), self.ref)

    def take_cow_pairs(self) -> list[tuple[int, int]]:
        """Hand the queued copies to the device and drop their pins."""
        out = self.pending
        self.pending = []
        for s, d in out:
            self._release_refs([s, d], self.pin)
        return out

    # -- queries -------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def seq_len(self, seq_id: int) -> int:
        return self.lens[seq_id]

    def num_blocks_of(self, seq_id: int) -> int:
        return len(self.tables[seq_id])

    def refcount(self, block: int) -> int:
        """Owner references (tables naming the block)."""
        return self.ref[block]

    def pins(self, block: int) -> int:
        """Queued copies naming the block."""
        return self.pin[block]

    def free_list(self) -> list[int]:
        return list(self.free)

    def table(self, seq_id: int) -> list[int]:
        return list(self.tables[seq_id])

    def block_table(self, seq_ids, width: int, pad: int = -1):
        import numpy as np
        out = np.full((len(seq_ids), width), pad, dtype=np.int32)
        for r, sid in enumerate(seq_ids):
            t = self.tables[sid]
            if len(t) > width:
                raise PoolError("table wider than width")
            out[r, :len(t)] = t
        return out

    def slots(self, seq_id: int, pos0: int, count: int):
        import numpy as np
        t = self.tables[seq_id]
        return np.array([slot_of(t, p, self.block_size) for p in range(pos0, pos0 + count)],
                        dtype=np.int64)

    def check(self) -> None:
        """The allocator invariants listed under "What should every allocator
        mutation preserve?" on page 1 (owner references only; no pins)."""
        B = self.block_size
        free = set(self.free)
        if len(free) != len(self.free):
            raise PoolError("free list holds a block twice")
        owners = [0] * self.num_blocks
        pinned = [0] * self.num_blocks
        for sid, t in self.tables.items():
            if len(set(t)) != len(t):
                raise PoolError(f"seq {sid}: duplicate block id")
            if len(t) != blocks_for(self.lens[sid], B):
                raise PoolError(f"seq {sid}: non-tail block not full or tail empty")
            for b in t:
                owners[b] += 1
        for s, d in self.pending:
            pinned[s] += 1
            pinned[d] += 1
        for b in range(self.num_blocks):
            if owners[b] != self.ref[b] or pinned[b] != self.pin[b]:
                raise PoolError(f"block {b}: counts ({self.ref[b]}, {self.pin[b]}) != references "
                                f"({owners[b]}, {pinned[b]})")
            if (b in free) == (self.ref[b] + self.pin[b] > 0):
                raise PoolError(f"block {b}: free/allocated sets overlap or miss it")
