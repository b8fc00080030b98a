"""Pins for the oracle's FP8 (OCP E4M3) KV cache: code values and the
encoder against torch's float8_e4m3fn and the format's definition; the fp8
decode against the bf16 decode and torch's attention."""
import numpy as np
import pytest
import torch

import oracle
import synth


def test_all_256_code_values_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_float64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.isnan(ours[[0x7F, 0xFF]]).all() and np.isnan(ours).sum() == 2
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0 and ours[0x08] == 2.0 ** -6


def test_encoder_matches_torch_inside_the_range():
    gen = synth.make_rng(5)
    x = np.concatenate([
        gen.standard_normal(4000).astype(np.float32) * 10,
        (gen.random(2000) * 2.0 ** -5).astype(np.float32),          # subnormal region
        (gen.random(2000) * 440).astype(np.float32) * np.sign(gen.standard_normal(2000)).astype(np.float32),
        oracle.e4m3_to_float64(np.arange(0, 0x7E)).astype(np.float32),  # every positive code value
    ])
    # exact ties: the midpoints between neighbouring positive codes
    vals = oracle.e4m3_to_float64(np.arange(0, 0x7F))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    ours = oracle.e4m3_from_float32(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_encoder_saturates_at_448():
    x = np.array([448.0, 463.9, 464.0, 500.0, 1e9, np.inf, -500.0, -np.inf], np.float32)
    assert oracle.e4m3_from_float32(x).tolist() == [0x7E] * 6 + [0xFE, 0xFE]
    assert oracle.e4m3_from_float32(np.array([np.nan], np.float32))[0] == 0x7F


def _paged_pair(gen, lens, B, Hkv, D, NB):
    """Logical K/V whose values are e4m3-representable, laid out in a bf16
    cache and an fp8 cache (scale 1) with the same table."""
    code_vals = oracle.e4m3_to_float64(np.arange(0, 0x7E))
    bt = np.full((len(lens), max(oracle.blocks_for(n, B) for n in lens)), -1, np.int32)
    perm = gen.permutation(NB)
    kb = np.zeros((NB, B, Hkv, D), np.uint16); vb = kb.copy()
    k8 = np.zeros((NB, B, Hkv, D), np.uint8); v8 = k8.copy()
    used = 0
    for s, n in enumerate(lens):
        nb = oracle.blocks_for(n, B)
        bt[s, :nb] = perm[used:used + nb]; used += nb
        kv = gen.choice(code_vals, size=(2, n, Hkv, D)) * np.where(gen.random((2, n, Hkv, D)) < 0.5, -1, 1)
        kv = (kv / 16).astype(np.float32)  # keep scores moderate; still exact
        slots = oracle.slot_mapping([bt[s]] * n, list(range(n)), B)
        oracle.write_kv(synth.f32_to_bf16_bits(kv[0]), synth.f32_to_bf16_bits(kv[1]), slots, kb, vb)
        oracle.write_kv_fp8(synth.f32_to_bf16_bits(kv[0]), synth.f32_to_bf16_bits(kv[1]), slots, k8, v8,
                            1.0 / 16, 1.0 / 16)
    return bt, kb, vb, k8, v8


def test_fp8_decode_equals_bf16_decode_on_representable_values():
    gen = synth.make_rng(6)
    lens = [1, 16, 40, 77]
    Hq, Hkv, D, B = 8, 2, 128, 16
    bt, kb, vb, k8, v8 = _paged_pair(gen, lens, B, Hkv, D, 32)
    q = synth.bf16_normal(gen, (len(lens), Hq, D))
    ref = oracle.decode(q, kb, vb, bt, np.array(lens, np.int32), 0.088)
    got = oracle.decode_fp8(q, k8, v8, bt, np.array(lens, np.int32), 0.088, 1.0 / 16, 1.0 / 16)
    assert np.array_equal(got, ref)


def test_fp8_scales_are_exact_powers_of_two_and_match_sdpa():
    gen = synth.make_rng(7)
    lens = [5, 33]
    Hq, Hkv, D, B = 4, 1, 128, 16
    bt, kb, vb, k8, v8 = _paged_pair(gen, lens, B, Hkv, D, 8)
    q = synth.bf16_normal(gen, (2, Hq, D))
    n = np.array(lens, np.int32)
    base = oracle.decode_fp8(q, k8, v8, bt, n, 0.1, 1.0, 1.0)
    assert np.array_equal(oracle.decode_fp8(q, k8, v8, bt, n, 0.1, 1.0, 4.0), 4.0 * base)
    assert np.array_equal(oracle.decode_fp8(q, k8, v8, bt, n, 0.1, 2.0, 1.0),
                          oracle.decode_fp8(q, k8, v8, bt, n, 0.2, 1.0, 1.0))
    # torch attention on the dequantised contiguous K/V
    for s, m in enumerate(lens):
        blk = bt[s, np.arange(m) // B]
        K = oracle.e4m3_to_float64(k8[blk, np.arange(m) % B, 0]) * 3.0
        V = oracle.e4m3_to_float64(v8[blk, np.arange(m) % B, 0]) * 0.5
        Q = torch.from_numpy(synth.bf16_bits_to_f32(q[s]).astype(np.float64))
        o = torch.nn.functional.scaled_dot_product_attention(Q[:, None, :], torch.from_numpy(K)[None].expand(Hq, -1, -1),
                                                             torch.from_numpy(V)[None].expand(Hq, -1, -1), scale=0.1)
        got = oracle.decode_fp8(q, k8, v8, bt, n, 0.1, 3.0, 0.5)[s]
        np.testing.assert_allclose(got, o[:, 0].numpy(), rtol=1e-12, atol=1e-13)


def test_fp8_write_round_trips_representable_values():
    gen = synth.make_rng(8)
    vals = oracle.e4m3_to_float64(np.arange(0, 0x7E)).astype(np.float32)
    x = gen.choice(vals, size=(10, 2, 128)).astype(np.float32) * 8  # representable after / 8
    slots = np.arange(10, dtype=np.int64) * 3
    kc = np.zeros((8, 4, 2, 128), np.uint8); vc = kc.copy()
    xb = synth.f32_to_bf16_bits(x)
    oracle.write_kv_fp8(xb, xb, slots, kc, vc, 8.0, 8.0)
    rows = kc.reshape(-1, 256)[slots]
    assert np.array_equal(oracle.e4m3_to_float64(rows).reshape(x.shape) * 8, x.astype(np.float64))
    with pytest.raises(ValueError):
        oracle.write_kv_fp8(xb[:1], xb[:1], np.array([32], np.int64), kc, vc, 1.0, 1.0)
