"""Device-side slot mapping and the KV write fused with it, against the
oracle's slot formula and write (bit-exact)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from oracle.pool import RefPool  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_333_b200 as m
    m.pa_get_device_error(clear=True)
    return m


def _to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _layout(seed, B, R=12, max_len=300):
    gen = synth.make_rng(seed)
    NB = R * (max_len // B + 1) + 16  # room for every sequence at any block size
    pool = RefPool(NB, B, gen.permutation(NB).astype(np.int32))
    lens = gen.integers(1, max_len, size=R)
    for r in range(R):
        pool.create(r)
        assert pool.append(r, int(lens[r]))
    W = max(pool.num_blocks_of(r) for r in range(R))
    return gen, pool, lens, pool.block_table(list(range(R)), W)


@pytest.mark.parametrize("B", [1, 4, 16, 32])
def test_slot_mapping_matches_the_formula(pa, B):
    gen, pool, lens, bt = _layout(10 + B, B)
    T = 700
    req = gen.integers(0, len(lens), size=T).astype(np.int32)
    pos = np.array([gen.integers(0, lens[r]) for r in req], np.int64)
    pos[gen.choice(T, size=40, replace=False)] = -1  # padding
    expect = oracle.slot_mapping([bt[r] for r in req], pos.tolist(), B)
    got = pa.pa_compute_slot_mapping(torch.from_numpy(pos).cuda(), torch.from_numpy(req).cuda(),
                                     torch.from_numpy(bt).cuda(), B, pool.num_blocks)
    assert np.array_equal(got.cpu().numpy(), expect)
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("B", [1, 16])
def test_fused_write_matches_oracle_write(pa, B):
    gen, pool, lens, bt = _layout(20 + B, B, R=8, max_len=200)
    H, D = 8, 128
    T = 300
    req = gen.integers(0, len(lens), size=T).astype(np.int32)
    # distinct (request, position) pairs so that no two tokens share a slot
    pairs = sorted({(int(r), int(gen.integers(0, lens[r]))) for r in req})
    req = np.array([p[0] for p in pairs], np.int32)
    pos = np.array([p[1] for p in pairs], np.int64)
    pos[::17] = -1
    k = synth.bf16_normal(gen, (len(pos), H, D)); v = synth.bf16_normal(gen, (len(pos), H, D))
    kc = synth.bf16_normal(gen, (pool.num_blocks, B, H, D)); vc = synth.bf16_normal(gen, (pool.num_blocks, B, H, D))
    dk, dv = _to_dev(kc), _to_dev(vc)
    pa.pa_write_kv_positions(_to_dev(k), _to_dev(v), torch.from_numpy(pos).cuda(), torch.from_numpy(req).cuda(),
                             torch.from_numpy(bt).cuda(), dk, dv)
    slots = oracle.slot_mapping([bt[r] for r in req], pos.tolist(), B)
    oracle.write_kv(k, v, slots, kc, vc)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(dk), kc) and np.array_equal(_bits(dv), vc)
    assert pa.pa_get_device_error(clear=True) == 0


def test_decode_step_slots_equal_the_pools(pa):
    """For a decode step (position = new length - 1, one token per request),
    the device slots equal the host pool's step slots and the oracle's."""
    from paged_kv_cache_333_b200 import BlockPool
    w = synth.chat()
    pool = BlockPool(w.shape.num_blocks, w.shape.block_size, w.free_order)
    w.ops(pool)
    for sid in w.seq_ids:
        assert pool.append(sid, 1)
    lens = pool.seq_lens(w.seq_ids)
    W = max(pool.num_blocks_of(s) for s in w.seq_ids)
    bt = pool.block_table(w.seq_ids, W)
    pos = (lens - 1).astype(np.int64)
    req = np.arange(len(lens), dtype=np.int32)
    got = pa.pa_compute_slot_mapping(torch.from_numpy(pos).cuda(), torch.from_numpy(req).cuda(),
                                     torch.from_numpy(bt).cuda(), w.shape.block_size, w.shape.num_blocks)
    host = pool.step_slots(w.seq_ids, 1)
    ref = oracle.slot_mapping([bt[r] for r in req], pos.tolist(), w.shape.block_size)
    assert np.array_equal(got.cpu().numpy(), host) and np.array_equal(host, ref)


def test_out_of_range_tokens_are_flagged_and_skipped(pa):
    B, NB, H, D = 16, 8, 2, 128
    bt = torch.tensor([[0, 1], [2, NB + 3]], dtype=torch.int32, device="cuda")
    pos = torch.tensor([5, 40, 20, 3, -4], dtype=torch.int64, device="cuda")  # 40: past the table width
    req = torch.tensor([0, 0, 1, 7, 0], dtype=torch.int32, device="cuda")     # 20 -> bad block id; 7 -> bad request
    pa.pa_get_device_error(clear=True)
    s = pa.pa_compute_slot_mapping(pos, req, bt, B, NB)
    assert s.cpu().tolist() == [5, -1, -1, -1, -1]
    assert pa.pa_get_device_error(clear=True) == pa.PA_DEVERR_SLOT
    kc = torch.zeros((NB, B, H, D), dtype=torch.bfloat16, device="cuda"); vc = kc.clone()
    k = torch.ones((5, H, D), dtype=torch.bfloat16, device="cuda")
    pa.pa_write_kv_positions(k, k, pos, req, bt, kc, vc)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(clear=True) == pa.PA_DEVERR_SLOT
    assert int((kc != 0).sum()) == H * D and bool((kc[0, 5] == 1).all())


def test_copy_blocks_for_all_layers_in_one_launch(pa):
    gen = synth.make_rng(99)
    L, NB, B, H, D = 5, 40, 16, 8, 128
    host = [(synth.bf16_normal(gen, (NB, B, H, D)), synth.bf16_normal(gen, (NB, B, H, D))) for _ in range(L)]
    dev = [(_to_dev(k), _to_dev(v)) for k, v in host]
    perm = gen.permutation(NB)
    pairs = np.stack([perm[:9], perm[9:18]], axis=1).astype(np.int64)
    pa.pa_copy_blocks_layers(dev, torch.from_numpy(pairs).cuda())
    for k, v in host:
        oracle.copy_blocks(pairs, k, v)
    torch.cuda.synchronize()
    for (k, v), (dk, dv) in zip(host, dev):
        assert np.array_equal(_bits(dk), k) and np.array_equal(_bits(dv), v)
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("m", [1, 2, 4, 8, 16])
def test_map_to_kernel_blocks_bit_exact(pa, m):
    """Allocation-block tables expanded to kernel-block tables on the device
    equal the oracle's definition, padding and the extra columns included."""
    gen = synth.make_rng(60 + m)
    t = gen.integers(-1, 5000, size=(33, 41)).astype(np.int32)
    expect = np.full((33, 41 * m + 7), -1, np.int32)
    expect[:, :41 * m] = oracle.map_to_kernel_blocks(t, m)
    out = torch.full((33, 41 * m + 7), 12345, dtype=torch.int32, device="cuda")
    pa.pa_map_to_kernel_blocks(torch.from_numpy(t).cuda(), m, out=out)
    assert np.array_equal(out.cpu().numpy(), expect)
    assert pa.pa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("B_a,m", [(32, 2), (64, 4), (16, 16), (8, 8)])
def test_kernel_block_view_decodes_and_maps_slots_the_same(pa, B_a, m):
    """The cache allocated in B_a-token blocks, seen as kernel blocks of B_a/m
    tokens through the expanded tables: the device slot mapping gives the same
    slots and decode the same outputs (within the tolerance of the oracle)."""
    gen, pool, lens, bt = _layout(70 + m, B_a, R=10, max_len=400)
    NB, H_kv, H_q, D = pool.num_blocks, 2, 8, 128
    kc = synth.bf16_normal(gen, (NB, B_a, H_kv, D))
    vc = synth.bf16_normal(gen, (NB, B_a, H_kv, D))
    q = synth.bf16_normal(gen, (len(lens), H_q, D))
    n = lens.astype(np.int32)
    dkc, dvc = _to_dev(kc), _to_dev(vc)
    kt = pa.pa_map_to_kernel_blocks(torch.from_numpy(bt).cuda(), m)
    # slots: every position of every request, through both tables
    req = np.repeat(np.arange(len(lens)), lens).astype(np.int32)
    pos = np.concatenate([np.arange(x) for x in lens]).astype(np.int64)
    s_a = pa.pa_compute_slot_mapping(torch.from_numpy(pos).cuda(), torch.from_numpy(req).cuda(),
                                     torch.from_numpy(bt).cuda(), B_a, NB)
    s_k = pa.pa_compute_slot_mapping(torch.from_numpy(pos).cuda(), torch.from_numpy(req).cuda(), kt, B_a // m,
                                     NB * m)
    assert torch.equal(s_a, s_k)
    # decode through both views of the same memory
    ref = oracle.decode(q, kc, vc, bt, n, 0.088)
    out_a = pa.pa_decode(_to_dev(q), dkc, dvc, torch.from_numpy(bt).cuda(), torch.from_numpy(n).cuda(), 0.088,
                         max_seq_len=int(n.max()))
    shape_k = (NB * m, B_a // m, H_kv, D)
    out_k = pa.pa_decode(_to_dev(q), dkc.view(shape_k), dvc.view(shape_k), kt, torch.from_numpy(n).cuda(), 0.088,
                         max_seq_len=int(n.max()))
    torch.cuda.synchronize()
    for out in (out_a, out_k):
        got = synth.bf16_bits_to_f32(_bits(out)).astype(np.float64)
        err = np.abs(got - ref)
        assert err.max() <= 1.5e-2 and err.mean() <= 1e-3
    assert pa.pa_get_device_error(clear=True) == 0
