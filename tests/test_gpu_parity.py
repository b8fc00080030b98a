"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bar: pa_write_kv and pa_copy_blocks bit-exact (every byte of both caches,
poisoned unused storage included); pa_decode within max |err| <= 1.5e-2 and
mean |err| <= 1e-3 of the fp64 oracle (bf16 output, fp32 accumulation)."""
import gc

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from tests.oracle_stage import stage_oracle  # noqa: E402

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 1.5e-2, 1e-3


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_333_b200 as m
    m.pa_get_device_error(clear=True)
    yield m
    m.pa_decode_set_partition_tokens(0)
    m.pa_decode_set_kernel("mma")


@pytest.fixture(params=["mma", "simt"])
def kernel(request, pa):
    """Run the test with each decode partition kernel."""
    prev = pa.pa_decode_set_kernel(request.param)
    yield request.param
    pa.pa_decode_set_kernel(prev)


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def _close(got_bf16: torch.Tensor, ref: np.ndarray, what=""):
    got = synth.bf16_bits_to_f32(_bits(got_bf16)).astype(np.float64)
    assert got.shape == ref.shape
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    return float(err.max()), float(err.mean())


CONFIGS = ["tiny", "chat", "long", "prefix", "sweep_b1", "sweep_b16", "sweep_b32"]


@pytest.mark.parametrize("name", CONFIGS)
def test_config_parity(pa, name):
    _config_parity(pa, name)


@pytest.mark.parametrize("name", ["tiny", "chat", "sweep_b1"])
def test_config_parity_simt_kernel(pa, name):
    prev = pa.pa_decode_set_kernel("simt")
    try:
        _config_parity(pa, name)
    finally:
        pa.pa_decode_set_kernel(prev)


def _config_parity(pa, name):
    """Full-size workloads: layouts identical, caches bit-exact after the
    history writes, the copy-on-write copies and the step's write, decode
    within tolerance for every (sequence, head)."""
    from paged_kv_cache_333_b200.workload import run_step, stage
    w = synth.by_name(name)
    ref = stage_oracle(w)
    st = stage(w, "cuda")
    assert np.array_equal(st.block_tables_np, ref["block_tables"])
    assert np.array_equal(st.seq_lens_np, ref["seq_lens"])
    assert np.array_equal(st.slot_mapping_np, ref["slots"])
    assert np.array_equal(st.history_pairs_np, ref["history_pairs"])
    assert np.array_equal(st.cow_pairs_np, ref["step_pairs"])
    out = run_step(st)
    torch.cuda.synchronize()
    kc, vc = st.caches[0]
    assert np.array_equal(_bits(kc), ref["k_cache"]), "K cache differs"
    assert np.array_equal(_bits(vc), ref["v_cache"]), "V cache differs"
    _close(out, ref["out"], name)
    # a second identical step gives bit-identical results
    out2 = run_step(st, out=torch.empty_like(out))
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    assert pa.pa_get_device_error(clear=True) == 0
    del st, ref
    gc.collect()
    torch.cuda.empty_cache()


def test_tiny_before_and_after_the_step(pa):
    """Lengths {1,17,33,100} (history only) and {2,18,34,101} (with the step's token)."""
    w = synth.tiny()
    ref = stage_oracle(w)
    B = w.shape.block_size
    lens0 = ref["seq_lens"] - 1
    out0 = oracle.decode(w.q, ref["k_cache"], ref["v_cache"], ref["block_tables"], lens0, w.scale)
    kc, vc = _to_dev(ref["k_cache"]), _to_dev(ref["v_cache"])
    q = _to_dev(w.q)
    bt = torch.from_numpy(ref["block_tables"]).cuda()
    for lens, expect in [(lens0, out0), (ref["seq_lens"], ref["out"])]:
        got = pa.pa_decode(q, kc, vc, bt, torch.from_numpy(lens).cuda(), w.scale, max_seq_len=int(lens.max()))
        _close(got, expect, f"lens {lens.tolist()}")
    assert B == 16


def _random_case(seed, lens, B, Hq, Hkv, NB=None, poison=True):
    """Logical K/V laid out at random physical blocks (oracle write)."""
    gen = synth.make_rng(seed)
    D = 128
    nblk = [oracle.blocks_for(n, B) for n in lens]
    NB = NB or sum(nblk) + 5
    perm = gen.permutation(NB).astype(np.int32)
    W = max(1, max(nblk))
    bt = np.full((len(lens), W), -1, np.int32)
    fill = np.uint16(0x7FC1) if poison else np.uint16(0)
    kc = np.full((NB, B, Hkv, D), fill, np.uint16)
    vc = np.full((NB, B, Hkv, D), fill, np.uint16)
    used = 0
    for s, n in enumerate(lens):
        bt[s, :nblk[s]] = perm[used:used + nblk[s]]
        used += nblk[s]
        k = synth.bf16_normal(gen, (n, Hkv, D)); v = synth.bf16_normal(gen, (n, Hkv, D))
        slots = oracle.slot_mapping([bt[s]] * n, list(range(n)), B)
        oracle.write_kv(k, v, slots, kc, vc)
    q = synth.bf16_normal(gen, (len(lens), Hq, D))
    return q, kc, vc, bt, np.array(lens, np.int32)


def _run_case(pa, q, kc, vc, bt, lens, scale=0.08838834764831845, max_len=None):
    dq, dk, dv = _to_dev(q), _to_dev(kc), _to_dev(vc)
    out = pa.pa_decode(dq, dk, dv, torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), scale,
                       max_seq_len=int(lens.max()) if max_len is None else max_len)
    torch.cuda.synchronize()
    return out


EDGE_LENS = [0, 1, 2, 15, 16, 17, 31, 33, 63, 64, 65, 127, 129, 300, 1000]


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [1, 2, 4, 8, 16, 32, 64])
def test_group_and_block_sizes(pa, kernel, G, B):
    Hkv = 2
    q, kc, vc, bt, lens = _random_case(100 + 10 * G + B, EDGE_LENS, B, G * Hkv, Hkv)
    ref = oracle.decode(q, kc, vc, bt, lens, 0.08838834764831845)
    _close(_run_case(pa, q, kc, vc, bt, lens), ref, f"{kernel} G={G} B={B}")
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("part", [64, 128, 192, 256, 512, 1024, 4096])
def test_split_k_partitions_and_merge(pa, kernel, part):
    lens = [1, 64, 65, 200, 777, 2049, 4100]
    q, kc, vc, bt, lens_np = _random_case(7, lens, 16, 32, 8)
    ref = oracle.decode(q, kc, vc, bt, lens_np, 0.08838834764831845)
    prev = pa.pa_decode_set_partition_tokens(part)
    try:
        _close(_run_case(pa, q, kc, vc, bt, lens_np), ref, f"part={part}")
    finally:
        pa.pa_decode_set_partition_tokens(prev)


def test_max_seq_len_upper_bound_is_only_a_bound(pa):
    """A loose max_seq_len (more partitions than needed) changes nothing but
    the launch shape."""
    lens = [5, 300, 1000]
    q, kc, vc, bt, lens_np = _random_case(8, lens, 16, 8, 2)
    ref = oracle.decode(q, kc, vc, bt, lens_np, 0.08838834764831845)
    for m in (1000, 1024, 5000, 32768):
        bt_wide = np.full((3, oracle.blocks_for(m, 16)), -1, np.int32)
        bt_wide[:, :bt.shape[1]] = bt
        _close(_run_case(pa, q, kc, vc, bt_wide, lens_np, max_len=m), ref, f"max_seq_len={m}")


def test_single_token_returns_v0_bit_exact(pa, kernel):
    q, kc, vc, bt, lens = _random_case(9, [1, 1, 1], 16, 8, 2)
    out = _bits(_run_case(pa, q, kc, vc, bt, lens))
    for s in range(3):
        blk = bt[s, 0]
        for j in range(8):
            assert np.array_equal(out[s, j], vc[blk, 0, j // 4])


def test_physical_placement_does_not_change_a_bit(pa, kernel):
    """Same logical K/V, four different placements: identical output bits."""
    lens = [3, 16, 40, 500, 1500]
    outs = []
    for seed in (1, 2, 3, 4):
        gen = synth.make_rng(55)
        B, Hkv, Hq, D = 16, 2, 8, 128
        k = [synth.bf16_normal(gen, (n, Hkv, D)) for n in lens]
        v = [synth.bf16_normal(gen, (n, Hkv, D)) for n in lens]
        q = synth.bf16_normal(gen, (len(lens), Hq, D))
        nblk = [oracle.blocks_for(n, B) for n in lens]
        NB = sum(nblk) + 7
        perm = synth.make_rng(seed).permutation(NB).astype(np.int32)
        bt = np.full((len(lens), max(nblk)), -1, np.int32)
        kc = np.full((NB, B, Hkv, D), 0x7FC1, np.uint16); vc = kc.copy()
        used = 0
        for s, n in enumerate(lens):
            bt[s, :nblk[s]] = perm[used:used + nblk[s]]; used += nblk[s]
            oracle.write_kv(k[s], v[s], oracle.slot_mapping([bt[s]] * n, list(range(n)), B), kc, vc)
        outs.append(_bits(_run_case(pa, q, kc, vc, bt, np.array(lens, np.int32))))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_block_size_invariance_within_tolerance(pa):
    lens = [1, 100, 1000]
    gen = synth.make_rng(66)
    Hkv, Hq, D = 2, 8, 128
    k = [synth.bf16_normal(gen, (n, Hkv, D)) for n in lens]
    v = [synth.bf16_normal(gen, (n, Hkv, D)) for n in lens]
    q = synth.bf16_normal(gen, (len(lens), Hq, D))
    results = []
    for B in (1, 16, 32):
        nblk = [oracle.blocks_for(n, B) for n in lens]
        bt = np.full((3, max(nblk)), -1, np.int32)
        kc = np.zeros((sum(nblk), B, Hkv, D), np.uint16); vc = kc.copy()
        used = 0
        for s, n in enumerate(lens):
            bt[s, :nblk[s]] = np.arange(used, used + nblk[s]); used += nblk[s]
            oracle.write_kv(k[s], v[s], oracle.slot_mapping([bt[s]] * n, list(range(n)), B), kc, vc)
        if B == 1:
            ref = oracle.decode(q, kc, vc, bt, np.array(lens, np.int32), 0.0884)
        results.append(_run_case(pa, q, kc, vc, bt, np.array(lens, np.int32), scale=0.0884))
    for r in results:
        _close(r, ref, "block size")


def test_write_and_copy_bit_exact_random(pa):
    gen = synth.make_rng(77)
    NB, B, Hkv, D, T = 300, 16, 8, 128, 1000
    kc = synth.bf16_normal(gen, (NB, B, Hkv, D)); vc = synth.bf16_normal(gen, (NB, B, Hkv, D))
    k = synth.bf16_normal(gen, (T, Hkv, D)); v = synth.bf16_normal(gen, (T, Hkv, D))
    k[5, 1, :7] = 0x7FC3  # NaN payloads are copied as bits
    slots = gen.choice(NB * B, size=T, replace=False).astype(np.int64)
    slots[gen.choice(T, size=50, replace=False)] = -1
    dk, dv = _to_dev(kc), _to_dev(vc)
    pa.pa_write_kv(_to_dev(k), _to_dev(v), torch.from_numpy(slots).cuda(), dk, dv)
    oracle.write_kv(k, v, slots, kc, vc)
    perm = gen.permutation(NB)
    pairs = np.stack([perm[:120], perm[120:240]], axis=1).astype(np.int64)
    pa.pa_copy_blocks(dk, dv, torch.from_numpy(pairs).cuda())
    oracle.copy_blocks(pairs, kc, vc)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dk), kc) and np.array_equal(_bits(dv), vc)
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("B,Hkv", [(1, 8), (32, 8), (64, 1), (16, 3)])
def test_write_and_copy_shapes(pa, B, Hkv):
    gen = synth.make_rng(78 + B)
    NB, D, T = 64, 128, 50
    kc = synth.bf16_normal(gen, (NB, B, Hkv, D)); vc = synth.bf16_normal(gen, (NB, B, Hkv, D))
    k = synth.bf16_normal(gen, (T, Hkv, D)); v = synth.bf16_normal(gen, (T, Hkv, D))
    slots = gen.choice(NB * B, size=T, replace=False).astype(np.int64)
    dk, dv = _to_dev(kc), _to_dev(vc)
    pa.pa_write_kv(_to_dev(k), _to_dev(v), torch.from_numpy(slots).cuda(), dk, dv)
    oracle.write_kv(k, v, slots, kc, vc)
    pairs = np.stack([np.arange(0, 10), np.arange(20, 30)], axis=1).astype(np.int64)
    pa.pa_copy_blocks(dk, dv, torch.from_numpy(pairs).cuda())
    oracle.copy_blocks(pairs, kc, vc)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dk), kc) and np.array_equal(_bits(dv), vc)


def test_empty_inputs(pa):
    kc = torch.zeros((4, 16, 2, 128), dtype=torch.bfloat16, device="cuda"); vc = kc.clone()
    e = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    pa.pa_write_kv(e, e, torch.empty(0, dtype=torch.int64, device="cuda"), kc, vc)
    pa.pa_copy_blocks(kc, vc, torch.empty((0, 2), dtype=torch.int64, device="cuda"))
    q = torch.randn((3, 8, 128), device="cuda").to(torch.bfloat16)
    bt = torch.zeros((3, 1), dtype=torch.int32, device="cuda")
    out = pa.pa_decode(q, kc, vc, bt, torch.zeros(3, dtype=torch.int32, device="cuda"), 0.1, max_seq_len=0)
    torch.cuda.synchronize()
    assert torch.all(out == 0)
    assert torch.all(kc == 0)


def test_device_checks_flag_bad_inputs_without_faulting(pa):
    """Out-of-range slots, block ids, lengths and copy ids are skipped or
    clamped by the kernels' own bounds checks and reported in the error word."""
    NB, B, Hkv, D = 8, 16, 2, 128
    kc = torch.zeros((NB, B, Hkv, D), dtype=torch.bfloat16, device="cuda"); vc = kc.clone()
    pa.pa_get_device_error(clear=True)
    k = torch.ones((2, Hkv, D), dtype=torch.bfloat16, device="cuda")
    pa.pa_write_kv(k, k, torch.tensor([NB * B, 3], dtype=torch.int64, device="cuda"), kc, vc)
    assert pa.pa_get_device_error(clear=True) == pa.PA_DEVERR_SLOT
    assert int((kc != 0).sum()) == Hkv * D  # only slot 3 was written
    pa.pa_copy_blocks(kc, vc, torch.tensor([[0, NB]], dtype=torch.int64, device="cuda"))
    assert pa.pa_get_device_error(clear=True) == pa.PA_DEVERR_COPY_PAIR
    q = torch.ones((1, 4, D), dtype=torch.bfloat16, device="cuda")
    bt = torch.tensor([[NB + 5, -3]], dtype=torch.int32, device="cuda")
    pa.pa_decode(q, kc, vc, bt, torch.tensor([20], dtype=torch.int32, device="cuda"), 0.1, max_seq_len=20)
    assert pa.pa_get_device_error(clear=True) == pa.PA_DEVERR_BLOCK_ID
    bt = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    pa.pa_decode(q, kc, vc, bt, torch.tensor([40], dtype=torch.int32, device="cuda"), 0.1, max_seq_len=32)
    assert pa.pa_get_device_error(clear=True) == pa.PA_DEVERR_SEQ_LEN
