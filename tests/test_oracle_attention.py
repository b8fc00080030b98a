"""Pins for the oracle's attention over several query tokens per request
(query_start_loc / seq_lens / max_query_len of "PagedAttention: fragmentation,
blocks, block tables", the attention-metadata passage), checked against
things other than the oracle: torch's causal scaled dot-product attention in
float64, the already pinned single-token decode, a closed form (all-equal keys
give running means of V), and invariance under physical placement and block
size."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_oracle_decode import _logical, _paged


def _causal_sdpa(q_rows, k_log, v_log, scale, H_q, H_kv):
    """torch's causal SDPA (float64) of the LAST len(q_rows) positions of a
    sequence whose K/V are k_log/v_log: the full-length query is padded at the
    front with zeros (rows that do not affect the others under the causal
    mask), and the bottom rows are returned."""
    G = H_q // H_kv
    n, qn = len(k_log), len(q_rows)
    q = np.zeros((n, H_q, q_rows.shape[-1]), np.float64)
    q[n - qn:] = synth.bf16_bits_to_f32(q_rows)
    qt = torch.from_numpy(q).permute(1, 0, 2)  # [H_q, n, D]
    k = torch.from_numpy(synth.bf16_bits_to_f32(k_log).astype(np.float64)).permute(1, 0, 2)
    v = torch.from_numpy(synth.bf16_bits_to_f32(v_log).astype(np.float64)).permute(1, 0, 2)
    k = k.repeat_interleave(G, dim=0)
    v = v.repeat_interleave(G, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, k, v, is_causal=True, scale=scale)
    return o.permute(1, 0, 2).numpy()[n - qn:]  # [qn, H_q, D]


def _case(seed, lens, q_lens, H_q=8, H_kv=2, D=128, B=16, placement_seed=5):
    gen = synth.make_rng(seed)
    k_log, v_log = _logical(gen, lens, H_kv, D)
    NB = sum(oracle.blocks_for(n, B) for n in lens) + 3
    kc, vc, bt = _paged(k_log, v_log, B, NB, H_kv, D, synth.make_rng(placement_seed))
    qsl = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = synth.bf16_normal(gen, (int(qsl[-1]), H_q, D))
    return k_log, v_log, kc, vc, bt, qsl, q


SCALE = float(np.float32(1 / np.sqrt(128)))


@pytest.mark.parametrize("B", [1, 16])
def test_whole_prefill_matches_causal_sdpa(B):
    """q_len = n: every position of every request attends to its prefix."""
    lens = [1, 5, 17, 40]
    k_log, v_log, kc, vc, bt, qsl, q = _case(21, lens, lens, B=B)
    got = oracle.attention(q, kc, vc, bt, qsl, np.array(lens, np.int32), SCALE)
    for r, n in enumerate(lens):
        ref = _causal_sdpa(q[qsl[r]:qsl[r + 1]], k_log[r], v_log[r], SCALE, 8, 2)
        np.testing.assert_allclose(got[qsl[r]:qsl[r + 1]], ref, rtol=1e-12, atol=1e-13)


def test_chunk_matches_bottom_rows_of_causal_sdpa():
    """q_len < n (a chunk of a prefill, or a few speculative tokens): the rows
    are the last q_len positions, aligned to the end of the sequence."""
    lens = [9, 33, 70, 4]
    q_lens = [3, 1, 16, 4]
    k_log, v_log, kc, vc, bt, qsl, q = _case(22, lens, q_lens)
    got = oracle.attention(q, kc, vc, bt, qsl, np.array(lens, np.int32), SCALE)
    for r in range(len(lens)):
        ref = _causal_sdpa(q[qsl[r]:qsl[r + 1]], k_log[r], v_log[r], SCALE, 8, 2)
        np.testing.assert_allclose(got[qsl[r]:qsl[r + 1]], ref, rtol=1e-12, atol=1e-13)


def test_one_row_per_request_is_decode():
    """q_len = 1 everywhere reduces to one decode step (bit-identical)."""
    lens = [1, 16, 17, 100]
    k_log, v_log, kc, vc, bt, qsl, q = _case(23, lens, [1] * 4)
    n = np.array(lens, np.int32)
    got = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    ref = oracle.decode(q, kc, vc, bt, n, SCALE)
    assert np.array_equal(got, ref)


def test_equal_keys_give_running_means():
    """All keys equal: row i of a request attends uniformly to positions
    0..n-q_len+i, so its output is the mean of those V rows."""
    gen = synth.make_rng(24)
    H_q, H_kv, D, B, n, ql = 4, 1, 128, 4, 13, 6
    k_log, v_log = _logical(gen, [n], H_kv, D)
    k_log[0][:] = k_log[0][0]
    kc, vc, bt = _paged(k_log, v_log, B, 8, H_kv, D, synth.make_rng(1))
    q = synth.bf16_normal(gen, (ql, H_q, D))
    got = oracle.attention(q, kc, vc, bt, np.array([0, ql], np.int32), np.array([n], np.int32), SCALE)
    v = synth.bf16_bits_to_f32(v_log[0]).astype(np.float64)[:, 0, :]
    for i in range(ql):
        mean = v[:n - ql + i + 1].mean(axis=0)
        for j in range(H_q):
            np.testing.assert_allclose(got[i, j], mean, rtol=1e-13, atol=1e-14)


def test_placement_and_block_size_invariance():
    lens, q_lens = [20, 50], [7, 50]
    outs = []
    for B, ps in [(16, 5), (16, 9), (1, 3), (32, 4)]:
        _, _, kc, vc, bt, qsl, q = _case(25, lens, q_lens, B=B, placement_seed=ps)
        outs.append(oracle.attention(q, kc, vc, bt, qsl, np.array(lens, np.int32), SCALE))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_empty_queries_and_bad_lengths():
    lens = [5, 8]
    _, _, kc, vc, bt, qsl, q = _case(26, lens, [0, 3])
    got = oracle.attention(q, kc, vc, bt, qsl, np.array(lens, np.int32), SCALE)
    assert got.shape == (3, 8, 128) and np.all(np.isfinite(got))
    with pytest.raises(ValueError):
        oracle.attention(q, kc, vc, bt, qsl, np.array([5, 2], np.int32), SCALE)  # 3 rows, 2 tokens
