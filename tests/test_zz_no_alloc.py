"""pa_decode_static_ws: decode for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc, for example a plugin
whose host application owns every device allocation, or a serving loop that
must not allocate on its hot path.  For them pa_decode_static_ws keeps
pa_decode's split-K scratch in a fixed device array inside the library.
These tests call it through the C ABI and check its output against pa_decode
given a workspace from the caller, on two calls in a row, with shapes that
really use the scratch.  Both run the same kernels with the same split-K
partitions on the same inputs, so the outputs must be identical bit for bit:
a stale or misplaced partial left in the shared array by the previous call
would show up even where it stays inside the numeric tolerance.  The first
call is also checked against the CPU oracle at the decode tolerance.  The
file name makes pytest collect it last.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 1.5e-2, 1e-3  # the tolerance of the decode parity tests


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import paged_kv_cache_333_b200 as m
    m.pa_decode_set_kernel("mma")
    m.pa_decode_set_partition_tokens(0)
    m.pa_get_device_error(clear=True)
    return m


def _to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def _case(seed, lens, B=16, Hq=32, Hkv=8):
    """Random logical K/V laid out at random physical blocks."""
    gen = synth.make_rng(seed)
    D = 128
    nblk = [oracle.blocks_for(n, B) for n in lens]
    NB = sum(nblk) + 3
    perm = gen.permutation(NB).astype(np.int32)
    bt = np.full((len(lens), max(nblk)), -1, np.int32)
    kc = np.zeros((NB, B, Hkv, D), np.uint16)
    vc = np.zeros((NB, B, Hkv, D), np.uint16)
    used = 0
    for s, n in enumerate(lens):
        bt[s, :nblk[s]] = perm[used:used + nblk[s]]
        used += nblk[s]
        k = synth.bf16_normal(gen, (n, Hkv, D))
        v = synth.bf16_normal(gen, (n, Hkv, D))
        oracle.write_kv(k, v, oracle.slot_mapping([bt[s]] * n, list(range(n)), B), kc, vc)
    q = synth.bf16_normal(gen, (len(lens), Hq, D))
    host = (q, kc, vc, bt, np.array(lens, np.int32))
    return (_to_dev(q), _to_dev(kc), _to_dev(vc), torch.from_numpy(bt).cuda(),
            torch.from_numpy(np.array(lens, np.int32)).cuda(), max(lens)), host


def _close(a, b, what):
    x = a.to(torch.float64).cpu().numpy()
    y = b.to(torch.float64).cpu().numpy()
    err = np.abs(x - y)
    assert np.all(np.isfinite(x)), what
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (what, err.max(), err.mean())


def test_static_scratch_matches_pa_decode_on_two_calls_in_a_row(pa):
    scale = 0.08838834764831845
    cases = [_case(901, [3000, 5000, 1000, 8000]), _case(902, [7000, 64, 2500, 1])]
    for i, ((q, kc, vc, bt, lens, max_len), host) in enumerate(cases):
        need = pa.pa_decode_workspace_bytes(q.shape[0], q.shape[1], max_len, kc, vc)
        assert 0 < need <= pa._abi.PA_DECODE_STATIC_WS_BYTES  # the scratch is really used
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        ref = pa.pa_decode(q, kc, vc, bt, lens, scale, out=torch.empty_like(q), max_seq_len=max_len,
                           workspace=ws)
        got = pa.pa_decode_static_ws(q, kc, vc, bt, lens, scale, out=torch.empty_like(q), max_seq_len=max_len)
        torch.cuda.synchronize()
        if not torch.equal(got.view(torch.int16), ref.view(torch.int16)):
            _close(got, ref, f"call {i + 1}")  # says how far apart they are
            raise AssertionError(f"call {i + 1}: static-scratch output differs from pa_decode's")
        if i == 0:
            oq, okc, ovc, obt, olens = host
            exact = oracle.decode(oq, okc, ovc, obt, olens, scale)
            _close(got, torch.from_numpy(exact), "call 1 against the oracle")
    assert pa.pa_get_device_error(clear=True) == 0


def test_static_scratch_rejects_shapes_that_do_not_fit(pa):
    """A shape needing more than the fixed array is refused before any work."""
    kc = torch.zeros((16, 16, 8, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    q = torch.zeros((4, 32, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((4, 2048), dtype=torch.int32, device="cuda")
    lens = torch.ones(4, dtype=torch.int32, device="cuda")
    prev = pa.pa_decode_set_partition_tokens(64)  # 512 partitions of 64 tokens at 32K
    try:
        need = pa.pa_decode_workspace_bytes(4, 32, 32768, kc, vc)
        assert need > pa._abi.PA_DECODE_STATIC_WS_BYTES
        with pytest.raises(pa.PaError) as ei:
            pa.pa_decode_static_ws(q, kc, vc, bt, lens, 0.1, out=torch.empty_like(q), max_seq_len=32768)
        assert ei.value.code == pa._abi.PA_EWORKSPACE
    finally:
        pa.pa_decode_set_partition_tokens(prev)
