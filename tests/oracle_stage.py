"""Oracle-side replay of a synthetic workload (test helper, not a test file).

The oracle's own pool model lays the workload out, the oracle's write and
copy fill host caches, and the oracle decodes.  Nothing here touches the
product package: the parity tests compare this against the CUDA path run on
the same seeded draws."""
from __future__ import annotations

import numpy as np

import oracle
from oracle.pool import RefPool

POISON = np.uint16(0x7FC1)  # the same poison value the device staging uses


def _write(w, pool, kc, vc, items, chunk=1 << 16):
    ks, vs, ss, n = [], [], [], 0
    for item in items + [None]:
        if item is not None and item[2] > item[1]:
            sid, a, b = item
            ks.append(w.rows("k", sid, a, b)); vs.append(w.rows("v", sid, a, b))
            ss.append(pool.slots(sid, a, b - a)); n += b - a
        if n and (item is None or n >= chunk):
            oracle.write_kv(np.ascontiguousarray(np.concatenate(ks)), np.ascontiguousarray(np.concatenate(vs)),
                            np.concatenate(ss), kc, vc)
            ks, vs, ss, n = [], [], [], 0


def stage_oracle(w, rule: str = "shared", decode: bool = True, which=None) -> dict:
    sh = w.shape
    pool = RefPool(sh.num_blocks, sh.block_size, w.free_order, rule)
    w.ops(pool)
    shape = (sh.num_blocks, sh.block_size, sh.num_kv_heads, sh.head_dim)
    kc = np.full(shape, POISON, dtype=np.uint16)
    vc = np.full(shape, POISON, dtype=np.uint16)
    if w.shared_len:
        _write(w, pool, kc, vc, [(w.seq_ids[0], 0, w.shared_len)])
    if w.suffix_ops is not None:
        w.suffix_ops(pool)
    hist = pool.take_cow_pairs()
    if hist:
        oracle.copy_blocks(np.array(hist, np.int64), kc, vc)
    _write(w, pool, kc, vc, [(sid, w.shared_len, pool.seq_len(sid)) for sid in w.seq_ids])
    for sid in w.seq_ids:
        assert pool.append(sid, w.step_tokens)
    step_pairs = pool.take_cow_pairs()
    if step_pairs:
        oracle.copy_blocks(np.array(step_pairs, np.int64), kc, vc)
    lens = np.array([pool.seq_len(s) for s in w.seq_ids], np.int32)
    slots = np.concatenate([pool.slots(s, int(n) - w.step_tokens, w.step_tokens)
                            for s, n in zip(w.seq_ids, lens)])
    _write(w, pool, kc, vc, [(s, int(n) - w.step_tokens, int(n)) for s, n in zip(w.seq_ids, lens)])
    width = max(1, max(pool.num_blocks_of(s) for s in w.seq_ids))
    bt = pool.block_table(w.seq_ids, width)
    out = oracle.decode(w.q, kc, vc, bt, lens, w.scale, which) if decode else None
    return dict(pool=pool, k_cache=kc, v_cache=vc, block_tables=bt, seq_lens=lens, slots=slots,
                history_pairs=np.array(hist, np.int64).reshape(-1, 2),
                step_pairs=np.array(step_pairs, np.int64).reshape(-1, 2), out=out)
