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
