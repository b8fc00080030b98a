"""Pins for the oracle's paging formulas: the worked examples the pages print."""
import math

import numpy as np

import oracle


def test_r7_walkthrough(golden):
    g = golden["r7_decode_step"]
    B = g["block_size"]
    assert oracle.blocks_for(g["committed_tokens"] + g["new_tokens"], B) == g["required_blocks"]
    assert max(g["required_blocks"] - g["held_blocks"], 0) == g["blocks_to_allocate"]
    # a row holding 256 arbitrary blocks, then block 1913 appended at index 256
    row = list(range(10_000, 10_000 + g["held_blocks"])) + [g["new_physical_block"]]
    assert g["position"] // B == g["logical_block"] and g["position"] % B == g["offset"]
    assert oracle.slot_of(row, g["position"], B) == g["slot"]
    sm = oracle.slot_mapping([row, row], [g["position"], -1], B)
    assert sm.dtype == np.int64 and sm.tolist() == [g["slot"], -1]


def test_tail_waste(golden):
    g = golden["tail_waste_b16"]
    w = [oracle.tail_waste(n, g["block_size"]) for n in g["lengths"]]
    assert w == g["unused_tail_slots"]
    assert sum(w) / len(w) == g["mean_if_equally_likely"]
    # the bound B*ceil(n/B) - n < B, and the uniform-residue mean (B-1)/2
    for B in (1, 4, 16, 32, 128):
        ws = [oracle.tail_waste(n, B) for n in range(1, 4 * B + 1)]
        assert all(0 <= x < B for x in ws)
        assert sum(ws) / len(ws) == (B - 1) / 2


def test_simulator_step0(golden):
    g = golden["simulator_step0"]
    assert g["pool_blocks"] * g["block_size"] == g["pool_tokens"]
    assert oracle.blocks_for(g["tokens"], g["block_size"]) == g["blocks_used"]
    assert oracle.tail_waste(g["tokens"], g["block_size"]) == g["paged_slack"]
    assert g["slab_tokens"] - g["tokens"] == g["contiguous_waste"]


def test_kv_bytes_per_token(golden):
    g = golden["kv_bytes_per_token"]
    for key in ("llama3_8b", "llama70b"):
        m = g[key]
        assert 2 * m["L"] * m["h_kv"] * m["d"] * m["s"] == m["bytes"]
    # the page's "16 x 320 KB = 5.12 MB": 320 KB is 327680 / 1024, and 5.12 is in units of 1000 KB
    assert g["llama70b"]["bytes"] / 1024 == 320
    assert 16 * (g["llama70b"]["bytes"] / 1024) / 1000 == g["llama70b"]["block16_bytes_approx_mb"]


def test_h100_pool_arithmetic(golden):
    g = golden["h100_pool"]
    per_tok = 131072
    assert g["blocks"] * g["block_size"] == g["slots"]
    assert g["max_model_len"] * per_tok == g["reservation_gib"] * 2**30
    assert math.floor(g["pool_gib"] / g["reservation_gib"]) == g["reservations"]
    assert round(100 * (1 - g["chat_tokens"] / g["max_model_len"]), 2) == g["chat_waste_pct"]
    per_seq = oracle.blocks_for(g["chat_tokens"], g["block_size"])
    assert per_seq == 39
    assert g["blocks"] // per_seq == g["paged_ceiling_seqs"]


def test_internal_fragmentation(golden):
    g = golden["internal_fragmentation"]
    per_tok = 131072
    for B in (16, 128):
        worst = (B - 1) * per_tok  # at most B-1 unused slots per sequence
        assert worst / 2**20 == g["per_seq_mib"][str(B)]
        assert round(686 * worst / 2**30, 1) == g["at_686_gib"][str(B)]
        assert round(100 * 686 * worst / 2**30 / 52.32, 1 if B == 16 else 0) == g["pct_of_pool"][str(B)]


def test_block_table_metadata(golden):
    g = golden["block_table_metadata"]
    assert g["max_num_reqs"] * g["width"] * 4 == g["bytes"]
    assert g["width"] == 32768 // 16


def test_partial_hit_and_prefix(golden):
    g = golden["partial_hit"]
    assert g["hit_tokens"] // g["block_size"] == g["shared_logical_block"]
    assert g["hit_tokens"] % g["block_size"] == g["valid_slots"]
    p = golden["prefix_sharing"]
    assert p["prefix_tokens"] // p["block_size"] == p["shared_full_blocks"]
    assert p["prefix_tokens"] % p["block_size"] == p["partial_tail_tokens"]
    assert oracle.blocks_for(p["prefix_tokens"], p["block_size"]) == p["shared_full_blocks"] + 1


# ---- kernel block != allocation block ("PagedAttention: fragmentation,
# blocks, block tables", section 2 and the decoupling passage)

def test_kernel_blocks_page_example():
    """A 32-token allocation block feeding 16-token kernel pages: block 7
    becomes kernel blocks 14 and 15; padding stays padding."""
    got = oracle.map_to_kernel_blocks(np.array([[7, 0, -1]], np.int32), 2)
    assert got.tolist() == [[14, 15, 0, 1, -1, -1]]


def test_kernel_blocks_cover_the_same_bytes():
    """Block-major storage: allocation block a of a pages of P_a bytes is the
    byte range [a*P_a, (a+1)*P_a); the kernel blocks it maps to must tile
    exactly that range with pages of P_a / m."""
    gen = np.random.default_rng(3)
    for m in (1, 2, 4, 8, 16):
        page_a = 4096 * m
        t = gen.integers(-1, 200, size=(5, 7)).astype(np.int32)
        k = oracle.map_to_kernel_blocks(t, m)
        page_k = page_a // m
        for r in range(5):
            for i in range(7):
                ids = k[r, i * m:(i + 1) * m]
                if t[r, i] < 0:
                    assert np.all(ids == -1)
                    continue
                starts = ids.astype(np.int64) * page_k
                assert starts[0] == int(t[r, i]) * page_a
                assert np.all(np.diff(starts) == page_k)
                assert starts[-1] + page_k == (int(t[r, i]) + 1) * page_a


def test_kernel_blocks_preserve_every_slot():
    """Every position maps to the same flat slot through (allocation table,
    B_a) and through (kernel table, B_a / m)."""
    gen = np.random.default_rng(4)
    for m, B_a in ((2, 32), (4, 16), (8, 64), (16, 16)):
        t = gen.permutation(300)[:40].reshape(4, 10).astype(np.int32)
        k = oracle.map_to_kernel_blocks(t, m)
        B_k = B_a // m
        for r in range(4):
            for pos in range(10 * B_a):
                assert oracle.slot_of(t[r], pos, B_a) == oracle.slot_of(k[r], pos, B_k)


def test_kernel_blocks_decode_invariance():
    """Decode through the kernel table over the cache viewed with kernel
    blocks equals decode through the allocation table (bit-identical)."""
    import synth
    gen = synth.make_rng(41)
    H_q, H_kv, D, B_a, m = 8, 2, 128, 32, 4
    NB = 16
    lens = [1, 33, 100, 250]
    kc = synth.bf16_normal(gen, (NB, B_a, H_kv, D))
    vc = synth.bf16_normal(gen, (NB, B_a, H_kv, D))
    t = np.full((4, 8), -1, np.int32)
    perm = gen.permutation(NB)
    used = 0
    for r, n in enumerate(lens):
        nb = oracle.blocks_for(n, B_a)
        t[r, :nb] = perm[used:used + nb]
        used += nb
    q = synth.bf16_normal(gen, (4, H_q, D))
    n = np.array(lens, np.int32)
    a = oracle.decode(q, kc, vc, t, n, 0.088)
    b = oracle.decode(q, kc.reshape(NB * m, B_a // m, H_kv, D), vc.reshape(NB * m, B_a // m, H_kv, D),
                      oracle.map_to_kernel_blocks(t, m), n, 0.088)
    assert np.array_equal(a, b)
