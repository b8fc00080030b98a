"""The seeded inputs are the recipe the design states: the pages' workload
shapes (Llama-3-8B heads, 16-token blocks, the 26,785-block pool), the
length mixes, and the block-size sweep's pool sized for the same token
capacity and filled to exactly 90%."""
import numpy as np
import pytest

import synth
from oracle.pool import RefPool


def _replayed(w):
    p = RefPool(w.shape.num_blocks, w.shape.block_size, w.free_order)
    w.ops(p)
    if w.suffix_ops is not None:
        w.suffix_ops(p)
    return p


def test_chat_recipe():
    w = synth.chat()
    sh = w.shape
    assert (sh.num_q_heads, sh.num_kv_heads, sh.head_dim, sh.block_size, sh.num_blocks) == (32, 8, 128, 16, 26785)
    p = _replayed(w)
    lens = np.array([p.seq_len(s) for s in w.seq_ids]) + w.step_tokens
    assert len(lens) == 64 and lens.min() >= 512 and lens.max() <= 612
    assert sorted(w.free_order.tolist()) == list(range(26785))


def test_long_recipe():
    w = synth.long_context()
    p = _replayed(w)
    lens = sorted(p.seq_len(s) + w.step_tokens for s in w.seq_ids)
    assert lens == [8192] * 4 + [32768] * 4


def test_prefix_recipe():
    w = synth.prefix_cow()
    assert w.shared_len == 2040
    p = _replayed(w)
    lens = np.array([p.seq_len(s) for s in w.seq_ids]) + w.step_tokens
    assert len(lens) == 256 and lens.min() >= 2041 and lens.max() <= 2040 + 256


@pytest.mark.parametrize("B", [1, 16, 32])
def test_sweep_recipe(B):
    w = synth.sweep(B)
    # the same token capacity at every block size, up to one block's rounding
    assert w.shape.num_blocks == 428_560 // B
    assert 0 <= 428_560 - w.shape.num_blocks * B < B
    p = _replayed(w)
    used = w.shape.num_blocks - p.num_free()
    assert used == int(0.9 * w.shape.num_blocks)
    lens = np.array([p.seq_len(s) for s in w.seq_ids]) + w.step_tokens
    assert len(lens) == 128 and lens.min() >= 1 and lens.max() <= 8192


def test_inputs_are_seeded():
    a, b = synth.chat(), synth.chat()
    assert np.array_equal(a.q, b.q) and np.array_equal(a.free_order, b.free_order)
    assert not np.array_equal(synth.chat(seed=1).q, a.q)
