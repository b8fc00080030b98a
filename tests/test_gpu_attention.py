"""pa_attention (several query rows per request, causal) on the GPU against
the oracle: within the decode tolerance on every output element, for
speculative-decode-sized and prefill-chunk-sized queries, every group size
and block size, split-K, requests without rows, and unused storage poisoned
with NaN.  Every case runs on both attention kernels: the mma.sync kernel
(8 (row, head) columns per warp) and the tcgen05 kernel (128 columns per work
unit, S, P and O in tensor memory)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 1.5e-2, 1e-3
SCALE = float(np.float32(1 / np.sqrt(128)))


@pytest.fixture(scope="module", params=["mma", "tcgen05"])
def pa(request):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_333_b200 as m
    m.pa_get_device_error(clear=True)
    prev = m.pa_attention_set_kernel(request.param)
    yield m
    m.pa_attention_set_kernel(prev)
    m.pa_decode_set_partition_tokens(0)


def _bits_to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def _case(seed, lens, q_lens, B, Hq, Hkv):
    """Logical K/V per request written by the oracle into a NaN-poisoned
    cache at shuffled blocks; q rows for the last q_len tokens of each."""
    gen = synth.make_rng(seed)
    D = 128
    nblk = [oracle.blocks_for(n, B) for n in lens]
    NB = sum(nblk) + 5
    perm = gen.permutation(NB).astype(np.int32)
    bt = np.full((len(lens), max(1, max(nblk))), -1, np.int32)
    kc = np.full((NB, B, Hkv, D), synth.BF16_NAN, np.uint16)
    vc = kc.copy()
    used = 0
    for r, n in enumerate(lens):
        bt[r, :nblk[r]] = perm[used:used + nblk[r]]
        used += nblk[r]
        k = synth.bf16_normal(gen, (n, Hkv, D))
        v = synth.bf16_normal(gen, (n, Hkv, D))
        oracle.write_kv(k, v, oracle.slot_mapping([bt[r]] * n, list(range(n)), B), kc, vc)
    qsl = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = synth.bf16_normal(gen, (int(qsl[-1]), Hq, D))
    return q, kc, vc, bt, qsl, np.array(lens, np.int32)


def _run(pa, q, kc, vc, bt, qsl, lens, scale=SCALE):
    out = pa.pa_attention(_bits_to_dev(q), torch.from_numpy(qsl).cuda(), _bits_to_dev(kc), _bits_to_dev(vc),
                          torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), scale,
                          max_query_len=int(np.diff(qsl).max()), max_seq_len=int(lens.max()))
    torch.cuda.synchronize()
    return synth.bf16_bits_to_f32(out.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def _check(got, ref, what):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [1, 2, 8, 16, 32, 64])
def test_attention_block_and_group_sizes(pa, G, B):
    # 1 row (a decode step), 2..5 speculative rows, a 33-row chunk (several
    # column chunks), a whole short prefill, and a request with no rows
    lens = [1, 2, 17, 40, 100, 7, 33]
    q_lens = [1, 2, 5, 4, 33, 7, 0]
    q, kc, vc, bt, qsl, n = _case(500 + 10 * G + B, lens, q_lens, B, 2 * G, 2)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    _check(_run(pa, q, kc, vc, bt, qsl, n), ref, f"G={G} B={B}")
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [1, 4, 16, 64])
def test_attention_small_queries(pa, G, B):
    """At most 16 (row, head) columns per request: the two-warp CTA shape,
    whose warps split the tiles of a group when it has 8 columns or fewer."""
    rmax = 16 // G
    lens = [1, 9, 40, 130, 700, 3]
    q_lens = [min(q, n) for q, n in zip([1, rmax, max(1, rmax - 1), rmax, max(1, rmax // 2), 0], lens)]
    q, kc, vc, bt, qsl, n = _case(600 + 10 * G + B, lens, q_lens, B, 2 * G, 2)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    _check(_run(pa, q, kc, vc, bt, qsl, n), ref, f"G={G} B={B}")
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("part", [64, 256, 1024])
def test_attention_split_k(pa, part):
    lens = [1, 300, 1000, 2049, 3000]
    q_lens = [1, 3, 64, 17, 200]
    q, kc, vc, bt, qsl, n = _case(77, lens, q_lens, 16, 32, 8)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    prev = pa.pa_decode_set_partition_tokens(part)
    try:
        _check(_run(pa, q, kc, vc, bt, qsl, n), ref, f"part={part}")
    finally:
        pa.pa_decode_set_partition_tokens(prev)
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("scale", [-SCALE, 2 * SCALE, 0.0])
def test_attention_negative_and_large_scale(pa, scale):
    """Any finite scale is the caller's: a negative one flips which keys
    dominate (the tcgen05 kernel takes the tile minimum of the raw scores), a
    large one sharpens the softmax, zero makes it the mean of the visible V
    rows (masked tokens still weigh 0); split into partitions so the merge
    sees the same domain."""
    lens = [5, 70, 300, 1000]
    q, kc, vc, bt, qsl, n = _case(83, lens, [5, 9, 40, 100], 16, 32, 8)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, scale)
    prev = pa.pa_decode_set_partition_tokens(256)
    try:
        _check(_run(pa, q, kc, vc, bt, qsl, n, scale=scale), ref, f"scale={scale}")
    finally:
        pa.pa_decode_set_partition_tokens(prev)
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("scale", [SCALE, -SCALE, 0.0])
@pytest.mark.parametrize("part", [0, 128])
def test_attention_up_to_64_columns(pa, G, scale, part):
    """At most 64 (row, head) columns per request (the bench's many-row case
    has 64): requests of one tile and of many, whole or split into 128-token
    partitions (work units of one or two tiles back to back), positive,
    negative and zero scale."""
    rmax = 64 // G
    lens = [1, 3, 64, 65, 100, 129, 700, 5, 2000, 64, 20, 190]
    q_lens = [min(n, r) for n, r in zip(lens, [1, 3, rmax, rmax, rmax - 1, rmax, rmax, 5, rmax // 2, 0, rmax, 2])]
    q, kc, vc, bt, qsl, n = _case(900 + 10 * G + part, lens, q_lens, 16, 2 * G, 2)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, scale)
    prev = pa.pa_decode_set_partition_tokens(part)
    try:
        _check(_run(pa, q, kc, vc, bt, qsl, n, scale=scale), ref, f"G={G} scale={scale} part={part}")
    finally:
        pa.pa_decode_set_partition_tokens(prev)
    assert pa.pa_get_device_error(clear=True) == 0


def test_attention_odd_kv_heads(pa):
    """Three KV heads (group size 2) and at most 64 columns per request: the
    tcgen05 kernel cannot pair the heads and keeps one head per work unit."""
    lens = [1, 40, 300, 77, 129]
    q, kc, vc, bt, qsl, n = _case(95, lens, [1, 12, 32, 5, 32], 16, 6, 3)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    _check(_run(pa, q, kc, vc, bt, qsl, n), ref, "3 KV heads")
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("B,part", [(16, 3072), (8, 1536)])
def test_attention_partition_fills_the_table_slice(pa, B, part):
    """Partitions of exactly 192 blocks, the most a tcgen05 CTA stages: a
    request that fills one partition exactly, one that spills a single token
    into a second, and longer ones, 16 rows each."""
    lens = [part, part + 1, part + part // 2, 2 * part]
    q, kc, vc, bt, qsl, n = _case(79 + B, lens, [16] * 4, B, 32, 8)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    prev = pa.pa_decode_set_partition_tokens(part)
    try:
        _check(_run(pa, q, kc, vc, bt, qsl, n), ref, f"B={B} part={part}")
    finally:
        pa.pa_decode_set_partition_tokens(prev)
    assert pa.pa_get_device_error(clear=True) == 0


def test_attention_whole_prefill(pa):
    """q_len = n: the first rows see a handful of tokens, the last all."""
    lens = [1, 16, 31, 160]
    q, kc, vc, bt, qsl, n = _case(78, lens, lens, 16, 8, 2)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    _check(_run(pa, q, kc, vc, bt, qsl, n), ref, "prefill")


def test_attention_one_row_matches_decode(pa):
    """One row per request is a decode step: pa_attention and pa_decode agree
    within the tolerance (both against the oracle, and each other)."""
    lens = [1, 15, 16, 17, 600, 2000]
    q, kc, vc, bt, qsl, n = _case(79, lens, [1] * len(lens), 16, 32, 8)
    got = _run(pa, q, kc, vc, bt, qsl, n)
    dec = pa.pa_decode(_bits_to_dev(q), _bits_to_dev(kc), _bits_to_dev(vc), torch.from_numpy(bt).cuda(),
                       torch.from_numpy(n).cuda(), SCALE, max_seq_len=int(n.max()))
    torch.cuda.synchronize()
    dec = synth.bf16_bits_to_f32(dec.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    ref = oracle.decode(q, kc, vc, bt, n, SCALE)
    _check(got, ref, "attention")
    _check(dec, ref, "decode")
    assert np.abs(got - dec).max() <= MAX_ABS


def test_attention_spec_decode_full_size(pa):
    """Chat-sized batch (64 requests, 512..612 tokens, Llama-3-8B heads) with
    4 query rows each (3 speculative tokens + 1), sampled rows checked."""
    gen = synth.make_rng(80)
    lens = gen.integers(512, 613, size=64).tolist()
    q, kc, vc, bt, qsl, n = _case(81, lens, [4] * 64, 16, 32, 8)
    got = _run(pa, q, kc, vc, bt, qsl, n)
    ref = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    _check(got, ref, "spec decode 64 x 4")
    assert pa.pa_get_device_error(clear=True) == 0


def test_attention_chunk16_full_size(pa):
    """Chat-sized batch (64 requests, 512..612 tokens, Llama-3-8B heads) with
    16 query rows each: 64 columns per request, the bench's many-row case.
    Eight requests are checked against the oracle row by row."""
    gen = synth.make_rng(84)
    lens = gen.integers(512, 613, size=64).tolist()
    q, kc, vc, bt, qsl, n = _case(85, lens, [16] * 64, 16, 32, 8)
    got = _run(pa, q, kc, vc, bt, qsl, n)
    assert pa.pa_get_device_error(clear=True) == 0
    for r in gen.choice(64, size=8, replace=False).tolist():
        rows = slice(int(qsl[r]), int(qsl[r + 1]))
        ref = oracle.attention(q[rows], kc, vc, bt[r:r + 1], np.array([0, 16], np.int32), n[r:r + 1], SCALE)
        _check(got[rows], ref, f"request {r}")


def test_attention_rejects_bad_query_start_loc(pa):
    """A request with more rows than tokens is flagged on the device; with a
    single partition its rows are not written, and the other requests are
    still computed."""
    lens = [3, 50]
    q, kc, vc, bt, qsl, n = _case(82, lens, [2, 5], 16, 8, 2)
    bad_lens = np.array([1, 50], np.int32)  # request 0: 2 rows but 1 token
    ref = oracle.attention(q, kc, vc, bt, qsl, n, SCALE)
    pa.pa_get_device_error(clear=True)
    out = torch.full((int(qsl[-1]), 8, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    pa.pa_attention(_bits_to_dev(q), torch.from_numpy(qsl).cuda(), _bits_to_dev(kc), _bits_to_dev(vc),
                    torch.from_numpy(bt).cuda(), torch.from_numpy(bad_lens).cuda(), SCALE, max_query_len=5,
                    max_seq_len=50, out=out)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_QUERY_LOC
    got = out.float().cpu().numpy()
    assert np.all(got[:2] == 7.0)  # request 0's rows untouched
    _check(got[2:].astype(np.float64), ref[2:], "valid request")
