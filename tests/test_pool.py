"""Block pool: the oracle pool pinned to the pages, and the product's C++ pool
checked against it operation by operation (tables, refcounts, free-list order,
copy pairs, slots), plus the pages' randomized content test."""
import numpy as np
import pytest

import oracle
import synth
from oracle.pool import RULE_INHERITED, RULE_SHARED, RefPool
from paged_kv_cache_333_b200 import BlockPool


def _pools(nb, B, order=None, rule="shared"):
    return RefPool(nb, B, order, rule), BlockPool(nb, B, order, rule)


def _same_state(ref: RefPool, prod: BlockPool):
    assert ref.free_list() == prod.free_list()
    for b in range(ref.num_blocks):
        assert ref.refcount(b) == prod.refcount(b), b
    for sid in ref.tables:
        assert ref.table(sid) == prod.table(sid), sid
        assert ref.seq_len(sid) == prod.seq_len(sid)
    ref.check()
    prod.check()


# ------------------------------------------------------------ pages' examples


@pytest.mark.parametrize("make", [lambda: RefPool(3, 4), lambda: BlockPool(3, 4)])
def test_pagedkv_trace_without_pin(make, golden):
    """Capacity 3, B=4: create a, append one token, fork b, append to b: the
    partial shared tail is copied before b writes; releasing both frees all."""
    g = golden["pagedkv_trace"]
    pool = make()
    pool.create("a" and 1)
    assert pool.append(1, 1)
    pool.fork(1, 2)
    (src,) = pool.table(1)
    assert pool.refcount(src) == 2
    assert pool.append(2, 1)  # b's tail is partial and shared -> copy
    pairs = [tuple(map(int, p)) for p in pool.take_cow_pairs()]
    assert len(pairs) == 1 and pairs[0][0] == src
    dst = pairs[0][1]
    assert pool.table(1) == [src] and pool.table(2) == [dst]
    assert pool.refcount(src) == 1 and pool.refcount(dst) == 1
    assert pool.seq_len(1) == len(g["read_a"]) and pool.seq_len(2) == len(g["read_b"])
    pool.check()
    pool.release(1)
    pool.release(2)
    assert pool.num_free() == g["capacity"] == g["free_after_release_all"]
    pool.check()


@pytest.mark.parametrize("cls", [RefPool, BlockPool])
def test_one_page_pool_cannot_copy_shared_tail(cls):
    """A failed allocation leaves both sequences intact."""
    pool = cls(1, 4)
    pool.create(1)
    assert pool.append(1, 1)
    pool.fork(1, 2)
    before = (pool.table(1), pool.table(2), pool.seq_len(1), pool.seq_len(2), pool.free_list())
    assert not pool.append(2, 1)
    after = (pool.table(1), pool.table(2), pool.seq_len(1), pool.seq_len(2), pool.free_list())
    assert before == after
    assert pool.refcount(pool.table(1)[0]) == 2
    pool.check()


@pytest.mark.parametrize("cls", [RefPool, BlockPool])
def test_tail_waste_and_block_counts(cls, golden):
    g = golden["tail_waste_b16"]
    pool = cls(64, g["block_size"])
    for i, n in enumerate(g["lengths"]):
        pool.create(i)
        assert pool.append(i, n)
        slack = pool.num_blocks_of(i) * g["block_size"] - pool.seq_len(i)
        assert slack == g["unused_tail_slots"][i]
    s = golden["simulator_step0"]
    pool = cls(s["pool_blocks"], s["block_size"])
    pool.create(0)
    assert pool.append(0, s["tokens"])
    assert s["pool_blocks"] - pool.num_free() == s["blocks_used"]
    assert pool.num_blocks_of(0) * s["block_size"] - s["tokens"] == s["paged_slack"]


@pytest.mark.parametrize("cls", [RefPool, BlockPool])
def test_r7_one_block_appended_and_slot(cls, golden):
    g = golden["r7_decode_step"]
    nb = 4096
    order = list(range(nb))
    order.remove(g["new_physical_block"])
    order.insert(g["held_blocks"], g["new_physical_block"])  # 257th block popped is 1913
    pool = cls(nb, g["block_size"], np.array(order, np.int32))
    pool.create(7)
    assert pool.append(7, g["committed_tokens"])
    assert pool.num_blocks_of(7) == g["held_blocks"]
    free0 = pool.num_free()
    assert pool.append(7, g["new_tokens"])
    assert free0 - pool.num_free() == g["blocks_to_allocate"]
    assert pool.table(7)[g["logical_block"]] == g["new_physical_block"]
    assert int(pool.slots(7, g["position"], 1)[0]) == g["slot"]


@pytest.mark.parametrize("cls", [RefPool, BlockPool])
def test_lifo_reuse_and_reverse_free_order(cls):
    pool = cls(8, 4)
    pool.create(1)
    assert pool.append(1, 12)  # blocks 0, 1, 2
    assert pool.table(1) == [0, 1, 2]
    pool.release(1)  # freed in reverse: 2, 1, 0 prepended as one run
    assert pool.free_list()[:3] == [2, 1, 0]
    pool.create(2)
    assert pool.append(2, 1)
    assert pool.table(2) == [2]  # the tail of the released sequence is reused first


@pytest.mark.parametrize("rule", [RULE_SHARED, RULE_INHERITED])
@pytest.mark.parametrize("cls", [RefPool, BlockPool])
def test_prefix_sharing_refcounts(cls, rule, golden):
    """2040-token prefix, 256 sequences: 127 full blocks shared by all, the
    8-token tail copied on first write (255 copies under the refcount rule;
    256 under the partial-hit rule, whose owner writes in place)."""
    p = golden["prefix_sharing"]
    B, n = p["block_size"], 256
    pool = cls(4096, B, None, rule)
    pool.create(0)
    assert pool.append(0, p["prefix_tokens"])
    for sid in range(1, n):
        pool.fork(0, sid)
    prefix_blocks = pool.table(0)
    assert len(prefix_blocks) == p["shared_full_blocks"] + 1
    assert all(pool.refcount(b) == n for b in prefix_blocks)
    tail = prefix_blocks[-1]
    for sid in range(n):
        assert pool.append(sid, 1)
    pairs = pool.take_cow_pairs()
    copies = n - 1
    assert len(pairs) == copies
    assert all(int(s) == tail for s, _ in pairs)
    assert len({int(d) for _, d in pairs}) == copies
    for b in prefix_blocks[:-1]:
        assert pool.refcount(b) == n
    assert pool.refcount(tail) == 1
    writer = n - 1 if rule == RULE_SHARED else 0  # who writes in place
    assert pool.table(writer)[-1] == tail
    pool.check()


# ------------------------------------------------------------ product vs oracle


def _replay(op, ref, prod, live, content, store, B):
    """Apply one random op to both pools and to the content model."""
    kind = op[0]
    if kind == "create":
        sid = op[1]
        ref.create(sid); prod.create(sid)
        live.append(sid); content[sid] = []
    elif kind == "append" and live:
        sid = live[op[1] % len(live)]
        n = op[2]
        ok_r, ok_p = ref.append(sid, n), prod.append(sid, n)
        assert ok_r == ok_p
        if ok_r:
            pr, pp = ref.take_cow_pairs(), prod.take_cow_pairs()
            assert [tuple(x) for x in pr] == [tuple(map(int, x)) for x in pp]
            # copies: the whole block, all B slots, sources read first
            snap = {(s, o): store.get(s * B + o) for s, _ in pr for o in range(B)}
            for s, d in pr:
                for o in range(B):
                    store[d * B + o] = snap[(s, o)]
            start = len(content[sid])
            slots = prod.slots(sid, start, n)
            assert slots.tolist() == ref.slots(sid, start, n).tolist()
            for i, slot in enumerate(slots):
                val = (sid, start + i)
                store[int(slot)] = val
                content[sid].append(val)
    elif kind == "fork" and live:
        src = live[op[1] % len(live)]
        dst = op[2]
        ref.fork(src, dst); prod.fork(src, dst)
        live.append(dst); content[dst] = list(content[src])
    elif kind == "release" and live:
        sid = live.pop(op[1] % len(live))
        ref.release(sid); prod.release(sid)
        del content[sid]


@pytest.mark.parametrize("rule", [RULE_SHARED, RULE_INHERITED])
@pytest.mark.parametrize("seed", range(25))
def test_random_ops_match_oracle_and_contents(seed, rule):
    """25 fixed seeds x 200 create/append/fork/release ops: after every op the
    two pools agree exactly, the invariants hold, and every sequence's pages
    decode to its own list of tokens (the randomized test described on page 1,
    without transfer pins)."""
    B, nb = 4, 24
    order = synth.make_rng(1000 + seed).permutation(nb).astype(np.int32)
    ref, prod = _pools(nb, B, order, rule)
    live, content, store = [], {}, {}
    for op in synth.random_pool_ops(seed, 200, max_append=9):
        _replay(op, ref, prod, live, content, store, B)
        _same_state(ref, prod)
        for sid in live:
            table = prod.table(sid)
            got = [store.get(table[p // B] * B + p % B) for p in range(len(content[sid]))]
            assert got == content[sid]


@pytest.mark.parametrize("name", ["tiny", "chat", "prefix"])
def test_workload_layouts_match_oracle(name):
    w = synth.by_name(name)
    sh = w.shape
    ref, prod = _pools(sh.num_blocks, sh.block_size, w.free_order)
    w.ops(ref); w.ops(prod)
    if w.suffix_ops:
        w.suffix_ops(ref); w.suffix_ops(prod)
    pr, pp = ref.take_cow_pairs(), prod.take_cow_pairs()
    assert [tuple(x) for x in pr] == [tuple(map(int, x)) for x in pp]
    width = max(ref.num_blocks_of(s) for s in w.seq_ids)
    assert np.array_equal(ref.block_table(w.seq_ids, width), prod.block_table(w.seq_ids, width))
    assert ref.free_list() == prod.free_list()
    prod.check()


@pytest.mark.slow
def test_sweep_churn_layout_matches_oracle():
    w = synth.sweep(16)
    sh = w.shape
    ref, prod = _pools(sh.num_blocks, sh.block_size, w.free_order)
    w.ops(ref); w.ops(prod)
    assert ref.free_list() == prod.free_list()
    used = sh.num_blocks - prod.num_free()
    assert used == int(0.9 * sh.num_blocks)
    width = max(ref.num_blocks_of(s) for s in w.seq_ids)
    assert np.array_equal(ref.block_table(w.seq_ids, width), prod.block_table(w.seq_ids, width))
    prod.check()


def test_errors_and_state_unchanged():
    pool = BlockPool(4, 4)
    pool.create(1)
    with pytest.raises(Exception):
        pool.create(1)
    with pytest.raises(Exception):
        pool.append(99, 1)
    assert pool.append(1, 16)
    assert not pool.append(1, 1)  # full
    assert pool.seq_len(1) == 16 and pool.num_free() == 0
    with pytest.raises(Exception):
        pool.block_table([1], 2)  # 4 blocks do not fit in width 2
    with pytest.raises(Exception):
        BlockPool(4, 4, np.array([0, 1, 1, 2], np.int32))  # not a permutation
    pool.check()


@pytest.mark.parametrize("n", [17, 2**40, 2**62, 2**63 - 1])
def test_appends_beyond_the_pool_are_refused_without_overflow(n):
    """No sequence can hold more than num_blocks * block_size tokens: such an
    append (single or batched) is refused with the pool unchanged, however
    large the count (the length arithmetic never overflows)."""
    pool = BlockPool(4, 4)
    pool.create(1)
    pool.create(2)
    assert pool.append(1, 3)
    free = pool.num_free()
    assert not pool.append(1, n)
    assert not pool.append_batch([1, 2], n)
    assert not pool.append(2, n)
    assert pool.num_free() == free and pool.seq_len(1) == 3 and pool.seq_len(2) == 0
    pool.check()
    assert pool.append(1, 13)  # exactly the rest of the pool still fits
    assert pool.num_free() == 0


def test_step_slots_and_padding():
    pool = BlockPool(16, 4)
    for sid, n in [(1, 5), (2, 8)]:
        pool.create(sid)
        assert pool.append(sid, n)
    sl = pool.step_slots([1, 2], 1)
    assert sl.tolist() == [int(pool.slots(1, 4, 1)[0]), int(pool.slots(2, 7, 1)[0])]
    bt = pool.block_table([1, 2], 3, pad=-7)
    assert bt[0, 2] == -7 and bt[1, 2] == -7
    assert oracle.slot_of(bt[1], 7, 4) == sl[1]


def _snapshot(p, ids, NB=40):
    return (np.asarray(p.block_table(ids, 64)).tolist(), [p.seq_len(i) for i in ids], list(p.free_list()),
            [p.refcount(b) for b in range(NB)], [p.pins(b) for b in range(NB)])


@pytest.mark.parametrize("rule", ["shared", "inherited"])
def test_append_batch_matches_sequential_appends(rule):
    """One call per scheduler step: the C++ batch equals the oracle pool's
    sequential appends, including copy-on-write of a tail several forks
    share (the first sharer copies, the last one may own the tail alone)."""
    for seed in range(8):
        gen = np.random.default_rng(seed)
        NB, B = 40, 4
        order = gen.permutation(NB).astype(np.int32)
        c, r = BlockPool(NB, B, order, rule), RefPool(NB, B, order, rule)
        for p in (c, r):
            p.create(0)
            assert p.append(0, 6)  # partial tail (6 % 4)
            for k in (1, 2, 3):
                p.fork(0, k)
        ids = [3, 0, 2, 1]
        for step in range(6):
            n = int(gen.integers(0, 5))
            ok_c, ok_r = c.append_batch(ids, n), r.append_batch(ids, n)
            assert ok_c == ok_r
            assert _snapshot(c, ids) == _snapshot(r, ids)
            c.check()
            r.check()
            assert np.asarray(c.take_cow_pairs()).reshape(-1, 2).tolist() == \
                np.asarray(r.take_cow_pairs()).reshape(-1, 2).tolist()


def test_append_batch_is_all_or_nothing():
    """When the pool cannot hold every append of the batch, nothing changes
    (and a batch that fits after a smaller step succeeds)."""
    for cls in (BlockPool, RefPool):
        p = cls(10, 4, np.arange(10, dtype=np.int32))
        for k in range(3):
            p.create(k)
            assert p.append(k, 8)  # 2 blocks each -> 6 used, 4 free
        ids = [0, 1, 2]
        before = _snapshot(p, ids, 10)
        assert not p.append_batch(ids, 8)  # needs 6 blocks
        assert _snapshot(p, ids, 10) == before
        assert p.append_batch(ids, 4)  # needs 3 blocks
        p.check()
        with pytest.raises(Exception):
            p.append_batch([0, 0], 1)  # listed twice
        with pytest.raises(Exception):
            p.append_batch([0, 99], 1)  # unknown sequence
        assert _snapshot(p, ids, 10)[1] == [12, 12, 12]


@pytest.mark.parametrize("rule", ["shared", "inherited"])
def test_append_batch_counts_copies_exactly_at_capacity(rule):
    """Four sequences share a partial tail and the pool has room for exactly
    three copies: under either rule three sharers copy and one writes in
    place, so the batch fits (counting a copy for every sharer would refuse)."""
    for cls in (BlockPool, RefPool):
        p = cls(5, 4, np.arange(5, dtype=np.int32), rule)
        p.create(0)
        assert p.append(0, 6)  # blocks 0, 1; tail partial
        for k in (1, 2, 3):
            p.fork(0, k)
        assert p.num_free() == 3
        assert p.append_batch([3, 0, 2, 1], 1)
        assert p.num_free() == 0
        assert len(np.asarray(p.take_cow_pairs()).reshape(-1, 2)) == 3
        p.check()


@pytest.mark.parametrize("rule", ["shared", "inherited"])
def test_incremental_block_table_equals_full_rebuild(rule):
    """Rows kept up to date append-only (only the old tail, which a copy-on-
    write may redirect, and the new entries are written) equal a full
    rebuild after every step, including rows reused for another sequence."""
    for seed in range(10):
        gen = np.random.default_rng(100 + seed)
        NB, B, W = 120, 4, 40
        p = BlockPool(NB, B, gen.permutation(NB).astype(np.int32), rule)
        live = []
        next_id = 0
        for _ in range(4):
            p.create(next_id)
            assert p.append(next_id, int(gen.integers(1, 9)))
            live.append(next_id)
            next_id += 1
        rows = list(live)
        table = np.full((len(rows), W), -1, np.int32)
        synced = np.zeros(len(rows), np.int32)
        for step in range(60):
            op = gen.integers(0, 10)
            if op < 5:
                p.append_batch(rows, int(gen.integers(0, 6)))
            elif op < 7 and len(live) < 8:  # fork a row's sequence into a fresh one (shares its tail)
                src = rows[int(gen.integers(0, len(rows)))]
                p.fork(src, next_id)
                live.append(next_id)
                next_id += 1
            elif op < 9:  # a row starts naming another live sequence: the caller resets it
                free = [i for i in live if i not in rows]
                if free:
                    r = int(gen.integers(0, len(rows)))
                    rows[r] = free[int(gen.integers(0, len(free)))]
                    table[r, :] = -1
                    synced[r] = 0
            else:  # append to one sequence only (copy-on-write of a shared tail)
                p.append(rows[int(gen.integers(0, len(rows)))], int(gen.integers(1, 4)))
            p.take_cow_pairs()
            if max(p.num_blocks_of(i) for i in rows) > W:
                break
            p.block_table_update(rows, table, synced)
            assert np.array_equal(table, p.block_table(rows, W)), (seed, step)
            assert synced.tolist() == [p.num_blocks_of(i) for i in rows]
        p.check()


def test_incremental_block_table_refuses_a_row_that_was_not_reset():
    """A row whose count exceeds its sequence's blocks names another sequence
    now: refused with nothing written (silently keeping the other sequence's
    leading entries would give a wrong table)."""
    p = BlockPool(20, 4, np.arange(20, dtype=np.int32))
    for k, n in ((0, 14), (1, 3)):
        p.create(k)
        assert p.append(k, n)
    table = np.full((1, 6), -1, np.int32)
    synced = np.zeros(1, np.int32)
    p.block_table_update([0], table, synced)
    assert synced.tolist() == [4]
    before = table.copy()
    with pytest.raises(Exception):
        p.block_table_update([1], table, synced)  # same row, other sequence, count not reset
    assert np.array_equal(table, before) and synced.tolist() == [4]
    table[:] = -1
    synced[:] = 0
    p.block_table_update([1], table, synced)
    assert np.array_equal(table, p.block_table([1], 6)) and synced.tolist() == [1]


def _step_by_parts(p, ids, n, table, synced):
    """The reference composition of pa_pool_step: the five separate calls."""
    if not p.append_batch(ids, n):
        return None
    pairs = p.take_cow_pairs()
    slots = p.step_slots(ids, n)
    p.block_table_update(ids, table, synced)
    return np.asarray(pairs, np.int64).reshape(-1, 2), slots, p.seq_lens(ids)


def _full_state(p, NB):
    return (list(p.free_list()), [p.refcount(b) for b in range(NB)], [p.pins(b) for b in range(NB)])


@pytest.mark.parametrize("rule", ["shared", "inherited"])
@pytest.mark.parametrize("seed", range(6))
def test_fused_step_equals_the_separate_calls(rule, seed):
    """pa_pool_step gives the pairs, slots, table, lengths and pool state of
    append_batch + take_copies + step_slots + block_table_update + seq_lens,
    step after step, on forks that share partial tails (copy-on-write under
    either rule) until the pool runs out."""
    gen = np.random.default_rng(seed)
    NB, B = 48, 4
    order = gen.permutation(NB).astype(np.int32)
    a, b = BlockPool(NB, B, order, rule), BlockPool(NB, B, order, rule)
    for p in (a, b):
        p.create(0)
        assert p.append(0, 6)
        for k in (1, 2, 3):
            p.fork(0, k)
        p.create(4)
        assert p.append(4, 3)
    ids = np.array([3, 0, 4, 2, 1], np.int64)
    width = NB
    ta, tb = np.full((5, width), -1, np.int32), np.full((5, width), -1, np.int32)
    sa, sb = np.zeros(5, np.int32), np.zeros(5, np.int32)
    full = False
    for step in range(40):
        n = int(gen.integers(0, 4))
        got = a.step(ids, n, ta, sa)
        want = _step_by_parts(b, ids, n, tb, sb)
        if want is None:
            assert got is None
            full = True
            assert _full_state(a, NB) == _full_state(b, NB)
            break
        pairs, slots, lens = got
        assert np.array_equal(pairs, want[0]) and np.array_equal(slots, want[1]) and np.array_equal(lens, want[2])
        assert np.array_equal(ta, tb) and np.array_equal(sa, sb)
        assert _full_state(a, NB) == _full_state(b, NB)
        a.check()
    assert full  # the run reached the end of the pool


def test_fused_step_matches_the_oracle_pool_on_chat():
    """Three decode steps of the chat workload (64 sequences, the 26,785-block
    pool) through pa_pool_step against the oracle pool's appends, slots,
    tables and lengths."""
    w = synth.chat()
    sh = w.shape
    c, r = BlockPool(sh.num_blocks, sh.block_size, w.free_order), RefPool(sh.num_blocks, sh.block_size, w.free_order)
    for p in (c, r):
        w.ops(p)
        p.take_cow_pairs()
    ids = np.asarray(w.seq_ids, np.int64)
    width = max(c.num_blocks_of(int(i)) for i in ids) + 2
    table, synced = np.full((len(ids), width), -1, np.int32), np.zeros(len(ids), np.int32)
    for _ in range(3):
        pairs, slots, lens = c.step(ids, 1, table, synced)
        assert r.append_batch(ids.tolist(), 1)
        assert len(pairs) == len(r.take_cow_pairs()) == 0
        assert slots.tolist() == [int(r.slots(int(i), r.seq_len(int(i)) - 1, 1)[0]) for i in ids]
        assert lens.tolist() == [r.seq_len(int(i)) for i in ids]
        assert np.array_equal(table, np.asarray(r.block_table(ids.tolist(), width)))


def test_fused_step_refusals_change_nothing():
    """Every refusal of pa_pool_step leaves the pool, the table and synced as
    they were: too few free blocks, too little room for the copy pairs or
    the table row, a row not reset, a sequence listed twice, an unknown one."""
    from paged_kv_cache_333_b200.pool import PoolError
    NB, B = 12, 4
    p = BlockPool(NB, B, np.arange(NB, dtype=np.int32))
    p.create(0)
    assert p.append(0, 6)  # 2 blocks, partial tail
    p.fork(0, 1)           # shares both
    ids = np.array([0, 1], np.int64)
    table, synced = np.full((2, 8), -1, np.int32), np.zeros(2, np.int32)
    p.block_table_update(ids, table, synced)

    def snap():
        return (_full_state(p, NB), table.tolist(), synced.tolist(), [p.seq_len(0), p.seq_len(1)])

    def refused(call, error=True):
        before = snap()
        if error:
            with pytest.raises(PoolError):
                call()
        else:
            assert call() is None
        assert snap() == before

    refused(lambda: p.step(ids, 40, table, synced), error=False)  # not enough free blocks
    # 1 token: sequence 0 copies its shared tail, but there is room for 0 pairs
    refused(lambda: p.step(ids, 1, table, synced, pairs=np.empty((0, 2), np.int64)))
    narrow, nsync = np.full((2, 2), -1, np.int32), np.zeros(2, np.int32)
    refused(lambda: p.step(ids, 3, narrow, nsync))  # a third block each: width 2 is too small
    assert narrow.tolist() == [[-1, -1], [-1, -1]] and nsync.tolist() == [0, 0]
    bad = synced.copy()
    bad[1] = 3  # more entries than the sequence has blocks: the row was not reset
    refused(lambda: p.step(ids, 1, table, bad))
    refused(lambda: p.step(np.array([0, 0], np.int64), 1, table, synced))  # listed twice
    refused(lambda: p.step(np.array([0, 7], np.int64), 1, table, synced))  # unknown sequence
    pairs, slots, lens = p.step(ids, 1, table, synced)  # and the step itself still goes through
    assert len(pairs) == 1 and lens.tolist() == [7, 7]
    p.check()


@pytest.mark.parametrize("rule", ["shared", "inherited"])
@pytest.mark.parametrize("seed", range(4))
def test_fused_step_random_histories_match_the_oracle_pool(rule, seed):
    """Random histories of creates, forks, releases and steps over random
    subsets of the live sequences: after every step, pa_pool_step's copy
    pairs, slots, lengths and incrementally kept table rows equal the oracle
    pool's (each sequence keeps its own row and count between its steps, as
    a scheduler would), and both pools hold the same blocks."""
    gen = np.random.default_rng(100 + seed)
    NB, B, W = 64, 4, 64
    order = gen.permutation(NB).astype(np.int32)
    c, r = BlockPool(NB, B, order, rule), RefPool(NB, B, order, rule)
    rows: dict[int, tuple[np.ndarray, int]] = {}
    live: list[int] = []
    nxt = 0
    for _ in range(300):
        op = gen.random()
        if op < 0.15 or not live:
            for p in (c, r):
                p.create(nxt)
            rows[nxt] = (np.full(W, -1, np.int32), 0)
            live.append(nxt)
            nxt += 1
        elif op < 0.25:
            src = live[int(gen.integers(len(live)))]
            for p in (c, r):
                p.fork(src, nxt)
            rows[nxt] = (np.full(W, -1, np.int32), 0)
            live.append(nxt)
            nxt += 1
        elif op < 0.35:
            victim = live.pop(int(gen.integers(len(live))))
            for p in (c, r):
                p.release(victim)
            del rows[victim]
        else:
            k = int(gen.integers(1, len(live) + 1))
            ids = [live[i] for i in gen.choice(len(live), size=k, replace=False)]
            n = int(gen.integers(0, 4))
            table = np.stack([rows[i][0] for i in ids])
            synced = np.array([rows[i][1] for i in ids], np.int32)
            got = c.step(np.array(ids, np.int64), n, table, synced)
            ok = r.append_batch(ids, n)
            if not ok:
                assert got is None
                continue
            pairs, slots, lens = got
            assert [tuple(x) for x in pairs.tolist()] == [tuple(x) for x in r.take_cow_pairs()]
            want_slots = [int(s) for i in ids for s in r.slots(i, r.seq_len(i) - n, n)]
            assert slots.tolist() == want_slots
            assert lens.tolist() == [r.seq_len(i) for i in ids]
            assert table.tolist() == np.asarray(r.block_table(ids, W)).tolist()
            for j, i in enumerate(ids):
                rows[i] = (table[j].copy(), int(synced[j]))
        assert c.free_list() == r.free_list()
    c.check()
    r.check()


@pytest.mark.parametrize("rule", ["shared", "inherited"])
def test_step_buffers_give_the_same_steps(rule):
    """step_into on reused StepBuffers (addresses taken once, table starting
    empty) matches step() on fresh arrays, step after step, copy-on-write
    included, until the pool is full."""
    from paged_kv_cache_333_b200.pool import StepBuffers
    NB, B = 48, 4
    order = np.random.default_rng(5).permutation(NB).astype(np.int32)
    a, b = BlockPool(NB, B, order, rule), BlockPool(NB, B, order, rule)
    for p in (a, b):
        p.create(0)
        assert p.append(0, 6)
        for k in (1, 2):
            p.fork(0, k)
    ids = [2, 0, 1]
    buf = StepBuffers(ids, 2, NB)
    table, synced = np.full((3, NB), -1, np.int32), np.zeros(3, np.int32)
    for _ in range(30):
        k = a.step_into(buf)
        got = b.step(np.array(ids, np.int64), 2, table, synced)
        if got is None:
            assert k is None
            break
        pairs, slots, lens = got
        assert buf.pairs[:k].tolist() == pairs.tolist()
        assert buf.slots.tolist() == slots.tolist() and buf.lens.tolist() == lens.tolist()
        assert buf.table.tolist() == table.tolist() and buf.synced.tolist() == synced.tolist()
    else:
        pytest.fail("the pool never filled")
    a.check()
