"""FP8 (E4M3) KV cache on the GPU against the oracle: the quantising write
bit-exact (every code byte of both caches), decode within the same tolerance
as the bf16 path (both sides read the same codes)."""
import gc

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 1.5e-2, 1e-3
KS, VS = 1.0 / 64, 1.0 / 64


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_333_b200 as m
    m.pa_get_device_error(clear=True)
    yield m
    m.pa_decode_set_partition_tokens(0)


def _to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def _close(got_bf16, ref, what=""):
    got = synth.bf16_bits_to_f32(got_bf16.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"


def _case(seed, lens, B, Hq, Hkv, poison=True):
    """Logical bf16 K/V written into an FP8 cache by the oracle at random blocks."""
    gen = synth.make_rng(seed)
    D = 128
    nblk = [oracle.blocks_for(n, B) for n in lens]
    NB = sum(nblk) + 5
    perm = gen.permutation(NB).astype(np.int32)
    bt = np.full((len(lens), max(1, max(nblk))), -1, np.int32)
    fill = np.uint8(0x7F) if poison else np.uint8(0)
    kc = np.full((NB, B, Hkv, D), fill, np.uint8); vc = kc.copy()
    used = 0
    for s, n in enumerate(lens):
        bt[s, :nblk[s]] = perm[used:used + nblk[s]]; used += nblk[s]
        k = synth.bf16_normal(gen, (n, Hkv, D)); v = synth.bf16_normal(gen, (n, Hkv, D))
        oracle.write_kv_fp8(k, v, oracle.slot_mapping([bt[s]] * n, list(range(n)), B), kc, vc, KS, VS)
    q = synth.bf16_normal(gen, (len(lens), Hq, D))
    return q, kc, vc, bt, np.array(lens, np.int32)


def _run(pa, q, kc, vc, bt, lens, scale=0.08838834764831845):
    out = pa.pa_decode_fp8(_to_dev(q), torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda(), KS, VS,
                           torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), scale,
                           max_seq_len=int(lens.max()))
    torch.cuda.synchronize()
    return out


def test_fp8_write_is_bit_exact(pa):
    gen = synth.make_rng(31)
    NB, B, H, D, T = 64, 16, 8, 128, 400
    k = synth.bf16_normal(gen, (T, H, D)); v = synth.bf16_normal(gen, (T, H, D))
    k[0, 0, :8] = synth.f32_to_bf16_bits(np.array([1000, -1000, 448 / 64, 7.0, 2 ** -16, -2 ** -16, 0, 3.0],
                                                  np.float32))  # saturation, tiny, zero
    slots = gen.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[::37] = -1
    kc = gen.integers(0, 256, size=(NB, B, H, D), dtype=np.uint8); vc = kc.copy()
    dk, dv = torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda()
    pa.pa_write_kv_fp8(_to_dev(k), _to_dev(v), torch.from_numpy(slots).cuda(), dk, dv, KS, VS)
    oracle.write_kv_fp8(k, v, slots, kc, vc, KS, VS)
    torch.cuda.synchronize()
    assert np.array_equal(dk.cpu().numpy(), kc) and np.array_equal(dv.cpu().numpy(), vc)
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("B", [1, 2, 8, 16, 32, 64])
def test_fp8_decode_block_and_group_sizes(pa, G, B):
    lens = [0, 1, 2, 15, 16, 17, 33, 64, 65, 300, 1000]
    q, kc, vc, bt, n = _case(300 + 10 * G + B, lens, B, 2 * G, 2)
    ref = oracle.decode_fp8(q, kc, vc, bt, n, 0.08838834764831845, KS, VS)
    _close(_run(pa, q, kc, vc, bt, n), ref, f"G={G} B={B}")
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("G", [1, 8])
def test_fp8_multi_wave_grid(pa, G):
    """A grid of more than 4 CTAs per SM (160 sequences x 2 KV heads x 5
    partitions) runs the three-consumer-warp kernel."""
    q, kc, vc, bt, n = _case(90 + G, [300] * 150 + [1, 17, 64, 250, 299, 33, 31, 32, 2, 5], 16, 2 * G, 2)
    ref = oracle.decode_fp8(q, kc, vc, bt, n, 0.08838834764831845, KS, VS)
    prev = pa.pa_decode_set_partition_tokens(64)
    try:
        _close(_run(pa, q, kc, vc, bt, n), ref, f"multi-wave G={G}")
    finally:
        pa.pa_decode_set_partition_tokens(prev)
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("part", [64, 256, 1024])
def test_fp8_split_k(pa, part):
    q, kc, vc, bt, n = _case(77, [1, 100, 777, 2049, 5000], 16, 32, 8)
    ref = oracle.decode_fp8(q, kc, vc, bt, n, 0.08838834764831845, KS, VS)
    prev = pa.pa_decode_set_partition_tokens(part)
    try:
        _close(_run(pa, q, kc, vc, bt, n), ref, f"part={part}")
    finally:
        pa.pa_decode_set_partition_tokens(prev)


def test_fp8_scales_fold_exactly(pa):
    """Doubling v_scale doubles the output exactly; a power-of-two k_scale is
    the same as that factor on the softmax scale."""
    q, kc, vc, bt, n = _case(78, [40, 200], 16, 8, 2)
    dq, dk, dv = _to_dev(q), torch.from_numpy(kc).cuda(), torch.from_numpy(vc).cuda()
    dbt, dn = torch.from_numpy(bt).cuda(), torch.from_numpy(n).cuda()
    a = pa.pa_decode_fp8(dq, dk, dv, KS, VS, dbt, dn, 0.1, max_seq_len=200).float()
    b = pa.pa_decode_fp8(dq, dk, dv, KS, 2 * VS, dbt, dn, 0.1, max_seq_len=200).float()
    c = pa.pa_decode_fp8(dq, dk, dv, 2 * KS, VS, dbt, dn, 0.05, max_seq_len=200).float()
    torch.cuda.synchronize()
    assert torch.equal(b, 2 * a)
    assert torch.equal(c, a)


def _scale_heads(q, factors):
    f = np.asarray(factors, np.float32)[None, :, None]
    return synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(q) * f)


def test_fp8_query_magnitudes_per_head(pa):
    """The kernel scales each query head by a power of two before splitting
    it into two e4m3 terms; heads 10^-6 .. 10^3 apart, in one KV group and in
    different groups, must all match the oracle."""
    fac = [1e-6, 3e-3, 1.0, 40.0, 2e-4, 7.0, 0.5, 900.0]
    q, kc, vc, bt, n = _case(81, [1, 31, 32, 33, 500, 1500], 16, 8, 2)
    q = _scale_heads(q, fac)
    ref = oracle.decode_fp8(q, kc, vc, bt, n, 0.08838834764831845 / 64, KS, VS)
    _close(_run(pa, q, kc, vc, bt, n, scale=0.08838834764831845 / 64), ref, "per-head magnitudes")


def test_fp8_query_wide_dynamic_range(pa):
    """One query element 2^12 larger than the rest of its head: the small
    elements fall below the split's exact range and must still not matter."""
    q, kc, vc, bt, n = _case(82, [77, 640], 32, 8, 8)
    qf = synth.bf16_bits_to_f32(q) * np.float32(1e-3)
    qf[:, :, 5] = 4.0
    q = synth.f32_to_bf16_bits(qf)
    ref = oracle.decode_fp8(q, kc, vc, bt, n, 0.5, KS, VS)
    _close(_run(pa, q, kc, vc, bt, n, scale=0.5), ref, "wide dynamic range")


@pytest.mark.parametrize("scale", [1e-4, 0.3, 2.0])
def test_fp8_flat_and_peaked_softmax(pa, scale):
    """Nearly uniform weights (small scale) and nearly one-hot ones (large
    scale): the probabilities' two-term split covers both ends."""
    q, kc, vc, bt, n = _case(83, [5, 64, 999, 3000], 16, 16, 4)
    ref = oracle.decode_fp8(q, kc, vc, bt, n, scale, KS, VS)
    _close(_run(pa, q, kc, vc, bt, n, scale=scale), ref, f"scale={scale}")


@pytest.mark.parametrize("name", ["chat", "sweep_b1", "long"])
def test_fp8_workload_parity(pa, name):
    """A full-size workload staged into FP8 caches by the GPU write: codes
    equal the oracle's, decode within tolerance of the fp8 oracle."""
    from paged_kv_cache_333_b200.workload import run_step, stage
    from oracle.pool import RefPool
    w = synth.by_name(name)
    st = stage(w, "cuda", kv_dtype="fp8", k_scale=KS, v_scale=VS)
    out = run_step(st)
    torch.cuda.synchronize()
    # the oracle's own layout and FP8 caches
    sh = w.shape
    pool = RefPool(sh.num_blocks, sh.block_size, w.free_order)
    w.ops(pool)
    kc = np.full((sh.num_blocks, sh.block_size, sh.num_kv_heads, sh.head_dim), 0x7F, np.uint8)
    vc = kc.copy()
    for sid in w.seq_ids:
        assert pool.append(sid, 1)
        m = pool.seq_len(sid)
        oracle.write_kv_fp8(np.ascontiguousarray(w.rows("k", sid, 0, m)), np.ascontiguousarray(w.rows("v", sid, 0, m)),
                            pool.slots(sid, 0, m), kc, vc, KS, VS)
    bt = pool.block_table(w.seq_ids, st.block_tables_np.shape[1])
    assert np.array_equal(bt, st.block_tables_np)
    assert np.array_equal(st.caches[0][0].cpu().numpy(), kc) and np.array_equal(st.caches[0][1].cpu().numpy(), vc)
    ref = oracle.decode_fp8(w.q, kc, vc, bt, st.seq_lens_np, w.scale, KS, VS)
    _close(out, ref, name)
    assert pa.pa_get_device_error(clear=True) == 0
    del st
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,Hkv", [(16, 8), (1, 2), (64, 1)])
def test_fp8_copy_blocks_bit_exact(pa, B, Hkv):
    """pa_copy_blocks_fp8 copies whole blocks of codes bit for bit: every byte
    of both caches equals the oracle's copy (applied to the same bytes, read
    as 16-bit words); an out-of-range pair is skipped and flagged."""
    gen = synth.make_rng(7100 + B + Hkv)
    NB, D = 40, 128
    k8 = gen.integers(0, 256, size=(NB, B, Hkv, D), dtype=np.uint8)
    v8 = gen.integers(0, 256, size=(NB, B, Hkv, D), dtype=np.uint8)
    pairs = np.array([[3, 10], [3, 11], [7, 12], [0, 39], [21, 2]], np.int64)  # distinct dsts, none a src
    dk, dv = torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda()
    pa.pa_get_device_error(clear=True)
    pa.pa_copy_blocks_fp8(dk, dv, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    ek, ev = k8.copy(), v8.copy()
    oracle.copy_blocks(pairs, ek.view(np.uint16), ev.view(np.uint16))
    assert np.array_equal(dk.cpu().numpy(), ek) and np.array_equal(dv.cpu().numpy(), ev)
    assert pa.pa_get_device_error(clear=True) == 0
    # a pair naming a block past the pool is skipped; the valid one still runs
    bad = torch.tensor([[5, NB], [6, 30]], dtype=torch.int64, device="cuda")
    pa.pa_copy_blocks_fp8(dk, dv, bad)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(clear=True) == pa.PA_DEVERR_COPY_PAIR
    oracle.copy_blocks(np.array([[6, 30]], np.int64), ek.view(np.uint16), ev.view(np.uint16))
    assert np.array_equal(dk.cpu().numpy(), ek) and np.array_equal(dv.cpu().numpy(), ev)


def test_fp8_prefix_copy_on_write_workload(pa):
    """The prefix workload (256 sequences forked from a 2040-token prefix,
    copy-on-write on first write) staged into FP8 caches: the copies run
    through pa_copy_blocks_fp8, every code byte of both caches equals the
    oracle's (which applies the same copies to the same bytes), and decode is
    within tolerance of the fp8 oracle."""
    from paged_kv_cache_333_b200.workload import run_step, stage
    from oracle.pool import RefPool
    w = synth.by_name("prefix")
    st = stage(w, "cuda", kv_dtype="fp8", k_scale=KS, v_scale=VS)
    assert st.history_pairs_np.shape[0] > 0  # the copies really ran
    out = run_step(st)
    torch.cuda.synchronize()
    sh = w.shape
    pool = RefPool(sh.num_blocks, sh.block_size, w.free_order)
    w.ops(pool)
    kc = np.full((sh.num_blocks, sh.block_size, sh.num_kv_heads, sh.head_dim), 0x7F, np.uint8)
    vc = kc.copy()

    def write(items):
        for sid, a, b in items:
            if b > a:
                oracle.write_kv_fp8(np.ascontiguousarray(w.rows("k", sid, a, b)),
                                    np.ascontiguousarray(w.rows("v", sid, a, b)), pool.slots(sid, a, b - a),
                                    kc, vc, KS, VS)

    def copy(pairs):
        if len(pairs):
            oracle.copy_blocks(np.array(pairs, np.int64), kc.view(np.uint16), vc.view(np.uint16))

    write([(w.seq_ids[0], 0, w.shared_len)])
    w.suffix_ops(pool)
    copy(pool.take_cow_pairs())
    write([(sid, w.shared_len, pool.seq_len(sid)) for sid in w.seq_ids])
    for sid in w.seq_ids:
        assert pool.append(sid, w.step_tokens)
    copy(pool.take_cow_pairs())
    lens = np.array([pool.seq_len(s) for s in w.seq_ids], np.int32)
    write([(s, int(n) - w.step_tokens, int(n)) for s, n in zip(w.seq_ids, lens)])
    bt = pool.block_table(w.seq_ids, st.block_tables_np.shape[1])
    assert np.array_equal(bt, st.block_tables_np) and np.array_equal(lens, st.seq_lens_np)
    assert np.array_equal(st.caches[0][0].cpu().numpy(), kc) and np.array_equal(st.caches[0][1].cpu().numpy(), vc)
    # decode checked on every 11th sequence (24 of 256; the oracle reads the same caches)
    pick = np.arange(0, len(w.seq_ids), 11)
    ref = oracle.decode_fp8(np.ascontiguousarray(w.q[pick]), kc, vc, np.ascontiguousarray(bt[pick]),
                            np.ascontiguousarray(lens[pick]), w.scale, KS, VS)
    _close(out[torch.from_numpy(pick).cuda()], ref, "prefix")
    assert pa.pa_get_device_error(clear=True) == 0
    del st
    gc.collect()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("B,Hkv", [(16, 8), (2, 2)])
def test_fp8_copy_blocks_layers_bit_exact(pa, B, Hkv):
    """pa_copy_blocks_layers_fp8: one launch copies the pairs in every layer's
    FP8 caches, each layer bit-exact against the oracle's copy of its bytes."""
    gen = synth.make_rng(7200 + B + Hkv)
    NB, D, L = 24, 128, 3
    pairs = np.array([[1, 20], [4, 21], [4, 22], [9, 0]], np.int64)
    host = [(gen.integers(0, 256, size=(NB, B, Hkv, D), dtype=np.uint8),
             gen.integers(0, 256, size=(NB, B, Hkv, D), dtype=np.uint8)) for _ in range(L)]
    dev = [(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda()) for k, v in host]
    pa.pa_get_device_error(clear=True)
    pa.pa_copy_blocks_layers_fp8(dev, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    for (k, v), (dk, dv) in zip(host, dev):
        ek, ev = k.copy(), v.copy()
        oracle.copy_blocks(pairs, ek.view(np.uint16), ev.view(np.uint16))
        assert np.array_equal(dk.cpu().numpy(), ek) and np.array_equal(dv.cpu().numpy(), ev)
    assert pa.pa_get_device_error(clear=True) == 0
