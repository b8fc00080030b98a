"""Pins for the oracle's decode attention, write and copy, checked against
things other than the oracle itself: torch's scaled dot-product attention on
the contiguous special case, closed forms, invariances, a 40-digit decimal
brute force, and numpy's fancy-index definition of the scatter and copy."""
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
import synth


def _paged(k_log, v_log, B, NB, H_kv, D, placement_gen=None, poison=True):
    """Place logical per-sequence K/V into a paged cache through the oracle's
    own write; return caches and an int32 block table.  Physical blocks are
    drawn without replacement from a permutation (or in order)."""
    S = len(k_log)
    W = max(1, max(oracle.blocks_for(len(k), B) for k in k_log))
    order = np.arange(NB) if placement_gen is None else placement_gen.permutation(NB)
    bt = np.full((S, W), -1, dtype=np.int32)
    nxt = 0
    fill = synth.BF16_NAN if poison else np.uint16(0)
    kc = np.full((NB, B, H_kv, D), fill, dtype=np.uint16)
    vc = np.full((NB, B, H_kv, D), fill, dtype=np.uint16)
    for s in range(S):
        nb = oracle.blocks_for(len(k_log[s]), B)
        bt[s, :nb] = order[nxt:nxt + nb]
        nxt += nb
        slots = oracle.slot_mapping([bt[s]] * len(k_log[s]), list(range(len(k_log[s]))), B)
        oracle.write_kv(np.ascontiguousarray(k_log[s]), np.ascontiguousarray(v_log[s]), slots, kc, vc)
    return kc, vc, bt


def _logical(gen, lens, H_kv, D):
    k = [synth.bf16_normal(gen, (n, H_kv, D)) for n in lens]
    v = [synth.bf16_normal(gen, (n, H_kv, D)) for n in lens]
    return k, v


def _sdpa(q_bits, k_log, v_log, scale, H_q, H_kv):
    """torch scaled_dot_product_attention in float64 on the contiguous K/V."""
    G = H_q // H_kv
    out = []
    for s in range(len(k_log)):
        q = torch.from_numpy(synth.bf16_bits_to_f32(q_bits[s]).astype(np.float64))  # [H_q, D]
        k = torch.from_numpy(synth.bf16_bits_to_f32(k_log[s]).astype(np.float64))  # [n, H_kv, D]
        v = torch.from_numpy(synth.bf16_bits_to_f32(v_log[s]).astype(np.float64))
        k = k.permute(1, 0, 2).repeat_interleave(G, dim=0)  # [H_q, n, D]
        v = v.permute(1, 0, 2).repeat_interleave(G, dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(
            q[:, None, :], k, v, scale=scale)  # [H_q, 1, D]
        out.append(o[:, 0, :].numpy())
    return np.stack(out)


@pytest.mark.parametrize("placement", ["contiguous", "scattered"])
def test_decode_matches_torch_sdpa(placement):
    gen = synth.make_rng(11)
    H_q, H_kv, D, B = 8, 2, 128, 16
    lens = [1, 17, 40, 100]
    k_log, v_log = _logical(gen, lens, H_kv, D)
    q = synth.bf16_normal(gen, (len(lens), H_q, D))
    pg = None if placement == "contiguous" else synth.make_rng(5)
    kc, vc, bt = _paged(k_log, v_log, B, 64, H_kv, D, pg)
    scale = float(np.float32(1 / np.sqrt(D)))
    got = oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), scale)
    ref = _sdpa(q, k_log, v_log, scale, H_q, H_kv)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_gqa_head_mapping():
    """q head j reads kv head j // G: give each kv head a constant V."""
    gen = synth.make_rng(12)
    H_q, H_kv, D, B = 8, 2, 128, 16
    k_log, v_log = _logical(gen, [30], H_kv, D)
    consts = [synth.f32_to_bf16_bits(np.float32(c)) for c in (0.5, -2.0)]
    for h in range(H_kv):
        v_log[0][:, h, :] = consts[h]
    q = synth.bf16_normal(gen, (1, H_q, D))
    kc, vc, bt = _paged(k_log, v_log, B, 4, H_kv, D)
    got = oracle.decode(q, kc, vc, bt, np.array([30], np.int32), 0.1)
    for j in range(H_q):
        assert np.all(got[0, j] == (0.5 if j < 4 else -2.0))


def test_permutation_invariance_is_bitwise():
    gen = synth.make_rng(13)
    H_q, H_kv, D, B = 8, 2, 128, 16
    lens = [3, 16, 33, 97]
    k_log, v_log = _logical(gen, lens, H_kv, D)
    q = synth.bf16_normal(gen, (len(lens), H_q, D))
    outs = []
    for seed in (None, 1, 2, 3):
        pg = None if seed is None else synth.make_rng(seed)
        kc, vc, bt = _paged(k_log, v_log, B, 64, H_kv, D, pg)
        outs.append(oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), 0.088))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_block_size_invariance_is_bitwise():
    gen = synth.make_rng(14)
    H_q, H_kv, D = 4, 1, 128
    lens = [1, 15, 16, 17, 64, 65]
    k_log, v_log = _logical(gen, lens, H_kv, D)
    q = synth.bf16_normal(gen, (len(lens), H_q, D))
    outs = []
    for B in (1, 2, 16, 32, 64):
        NB = sum(oracle.blocks_for(n, B) for n in lens) + 3
        kc, vc, bt = _paged(k_log, v_log, B, NB, H_kv, D, synth.make_rng(B))
        outs.append(oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), 0.088))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_all_equal_keys_give_mean_of_v():
    gen = synth.make_rng(15)
    H_q, H_kv, D, B, n = 2, 1, 128, 16, 37
    k_log, v_log = _logical(gen, [n], H_kv, D)
    k_log[0][:] = k_log[0][0]  # every key equal
    q = synth.bf16_normal(gen, (1, H_q, D))
    kc, vc, bt = _paged(k_log, v_log, B, 8, H_kv, D)
    got = oracle.decode(q, kc, vc, bt, np.array([n], np.int32), 0.088)
    mean_v = synth.bf16_bits_to_f32(v_log[0][:, 0, :]).astype(np.float64).mean(axis=0)
    for j in range(H_q):
        np.testing.assert_allclose(got[0, j], mean_v, rtol=1e-13, atol=1e-14)


def test_one_dominant_key_gives_its_value():
    gen = synth.make_rng(16)
    H_q, H_kv, D, B, n, star = 1, 1, 128, 16, 50, 23
    k_log, v_log = _logical(gen, [n], H_kv, D)
    k_log[0][:] = 0
    k_log[0][star, 0, 0] = synth.f32_to_bf16_bits(np.float32(64.0))
    q = np.zeros((1, H_q, D), np.uint16)
    q[0, 0, 0] = synth.f32_to_bf16_bits(np.float32(8.0))
    # logit of the star key: 8*64*scale = 512*0.125 = 64 above every other (0)
    kc, vc, bt = _paged(k_log, v_log, B, 8, H_kv, D)
    got = oracle.decode(q, kc, vc, bt, np.array([n], np.int32), 0.125)
    v_star = synth.bf16_bits_to_f32(v_log[0][star, 0]).astype(np.float64)
    bound = n * np.exp(-64.0) * 8  # every other weight <= e^-64, |v| <= 8
    assert np.max(np.abs(got[0, 0] - v_star)) <= bound


def test_single_token_returns_v0_exactly_and_empty_returns_zero():
    gen = synth.make_rng(17)
    H_q, H_kv, D, B = 8, 2, 128, 16
    k_log, v_log = _logical(gen, [1, 5], H_kv, D)
    q = synth.bf16_normal(gen, (3, H_q, D))
    k_log.append(np.zeros((0, H_kv, D), np.uint16))
    v_log.append(np.zeros((0, H_kv, D), np.uint16))
    kc, vc, bt = _paged(k_log, v_log, B, 8, H_kv, D)
    got = oracle.decode(q, kc, vc, bt, np.array([1, 5, 0], np.int32), 0.088)
    for j in range(H_q):
        assert np.array_equal(got[0, j], synth.bf16_bits_to_f32(v_log[0][0, j // 4]).astype(np.float64))
    assert np.all(got[2] == 0.0)


def test_brute_force_decimal_tiny():
    """40-digit decimal arithmetic on tiny inputs (n <= 8, D = 8)."""
    getcontext().prec = 40
    gen = synth.make_rng(18)
    H_q, H_kv, D, B = 4, 2, 8, 2
    lens = [1, 2, 5, 8]
    k_log, v_log = _logical(gen, lens, H_kv, D)
    q = synth.bf16_normal(gen, (len(lens), H_q, D))
    kc, vc, bt = _paged(k_log, v_log, B, 16, H_kv, D, synth.make_rng(3))
    scale = 0.35355339059327373  # any double
    got = oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), scale)
    dec = lambda x: Decimal(float(x))  # noqa: E731  (exact: every float is a finite decimal)
    for s, n in enumerate(lens):
        K = synth.bf16_bits_to_f32(k_log[s]); V = synth.bf16_bits_to_f32(v_log[s])
        Q = synth.bf16_bits_to_f32(q[s])
        for j in range(H_q):
            h = j // (H_q // H_kv)
            logits = [dec(scale) * sum(dec(Q[j, d]) * dec(K[t, h, d]) for d in range(D)) for t in range(n)]
            w = [x.exp() for x in logits]
            tot = sum(w)
            for d in range(D):
                o = sum(w[t] * dec(V[t, h, d]) for t in range(n)) / tot
                assert abs(float(o) - got[s, j, d]) <= 1e-14 * max(1.0, abs(float(o)))


def test_poison_in_unused_storage_is_never_read():
    gen = synth.make_rng(19)
    H_q, H_kv, D, B = 8, 2, 128, 16
    lens = [5, 16, 31]
    k_log, v_log = _logical(gen, lens, H_kv, D)
    q = synth.bf16_normal(gen, (3, H_q, D))
    kc, vc, bt = _paged(k_log, v_log, B, 16, H_kv, D, synth.make_rng(4), poison=True)
    got = oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), 0.088)
    kc0, vc0, bt0 = _paged(k_log, v_log, B, 16, H_kv, D, synth.make_rng(4), poison=False)
    ref = oracle.decode(q, kc0, vc0, bt0, np.array(lens, np.int32), 0.088)
    assert np.all(np.isfinite(got)) and np.array_equal(got, ref)


def test_decode_rejects_bad_block_ids_and_narrow_tables():
    kc = np.zeros((4, 16, 1, 128), np.uint16)
    q = np.zeros((1, 1, 128), np.uint16)
    with pytest.raises(ValueError):
        oracle.decode(q, kc, kc, np.array([[7]], np.int32), np.array([3], np.int32), 0.1)
    with pytest.raises(ValueError):
        oracle.decode(q, kc, kc, np.array([[0]], np.int32), np.array([17], np.int32), 0.1)


# ---------------------------------------------------------------- write / copy


def test_write_matches_fancy_index_and_skips_padding():
    gen = synth.make_rng(20)
    NB, B, H_kv, D, T = 32, 16, 2, 128, 40
    kc = synth.bf16_normal(gen, (NB, B, H_kv, D)); vc = synth.bf16_normal(gen, (NB, B, H_kv, D))
    k = synth.bf16_normal(gen, (T, H_kv, D)); v = synth.bf16_normal(gen, (T, H_kv, D))
    k[3, 0, :5] = synth.BF16_NAN  # payload bits must survive
    slots = gen.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[[7, 19]] = -1
    ek, ev = kc.copy(), vc.copy()
    keep = slots >= 0
    ek.reshape(NB * B, H_kv * D)[slots[keep]] = k.reshape(T, -1)[keep]
    ev.reshape(NB * B, H_kv * D)[slots[keep]] = v.reshape(T, -1)[keep]
    oracle.write_kv(k, v, slots, kc, vc)
    assert np.array_equal(kc.view(np.uint16), ek) and np.array_equal(vc, ev)


def test_write_r7_lands_in_block_1913_offset_0(golden):
    g = golden["r7_decode_step"]
    NB, B, H_kv, D = 2000, 16, 1, 8
    kc = np.zeros((NB, B, H_kv, D), np.uint16); vc = kc.copy()
    k = np.arange(1, 9, dtype=np.uint16).reshape(1, 1, 8); v = k + 100
    oracle.write_kv(k, v, np.array([g["slot"]], np.int64), kc, vc)
    assert np.array_equal(kc[g["new_physical_block"], g["offset"], 0], k[0, 0])
    assert np.array_equal(vc[g["new_physical_block"], g["offset"], 0], v[0, 0])
    assert np.count_nonzero(kc) == 8


def test_write_rejects_slot_past_the_end():
    kc = np.zeros((2, 4, 1, 8), np.uint16)
    with pytest.raises(ValueError):
        oracle.write_kv(np.zeros((1, 1, 8), np.uint16), np.zeros((1, 1, 8), np.uint16),
                        np.array([8], np.int64), kc, kc.copy())


def test_copy_matches_fancy_index_assignment():
    gen = synth.make_rng(21)
    NB, B, H_kv, D = 40, 16, 2, 128
    kc = synth.bf16_normal(gen, (NB, B, H_kv, D)); vc = synth.bf16_normal(gen, (NB, B, H_kv, D))
    perm = gen.permutation(NB)
    pairs = np.stack([perm[:10], perm[10:20]], axis=1).astype(np.int64)
    ek, ev = kc.copy(), vc.copy()
    ek[pairs[:, 1]] = ek[pairs[:, 0]]
    ev[pairs[:, 1]] = ev[pairs[:, 0]]
    oracle.copy_blocks(pairs, kc, vc)
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def test_copy_reads_all_sources_before_writing():
    """A chain 0->1, 1->2: the fancy-index definition gives block 2 the OLD block 1."""
    kc = np.arange(3 * 4 * 1 * 8, dtype=np.uint16).reshape(3, 4, 1, 8)
    vc = kc + 1000
    old1k, old1v = kc[1].copy(), vc[1].copy()
    old0k = kc[0].copy()
    oracle.copy_blocks(np.array([[0, 1], [1, 2]], np.int64), kc, vc)
    assert np.array_equal(kc[2], old1k) and np.array_equal(vc[2], old1v)
    assert np.array_equal(kc[1], old0k)


def test_copy_rejects_out_of_range():
    kc = np.zeros((3, 4, 1, 8), np.uint16)
    with pytest.raises(ValueError):
        oracle.copy_blocks(np.array([[0, 3]], np.int64), kc, kc.copy())
