"""The C-ABI libraries load on a machine without a GPU and export every
function their headers declare; argument validation runs on the host."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header: str) -> set:
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text))


@pytest.mark.parametrize("header,lib", [("pa.h", "libpa.so"), ("pa_pool.h", "libpa_pool.so")])
def test_library_exports_every_declared_function(header, lib):
    names = _declared(header)
    assert len(names) >= 8
    so = ctypes.CDLL(os.path.join(ROOT, "paged_kv_cache_333_b200", lib))
    missing = [n for n in sorted(names) if not hasattr(so, n)]
    assert not missing, missing


def test_binding_lists_match_headers():
    from paged_kv_cache_333_b200 import _abi, pool
    assert set(_abi.EXPORTED) == _declared("pa.h")
    assert set(pool.EXPORTED) == _declared("pa_pool.h")


def test_host_side_validation_without_gpu():
    """Calls rejected on the host never touch the device."""
    from paged_kv_cache_333_b200._abi import PA_EINVAL, PA_EUNSUPPORTED, PaCache, lib
    ok = PaCache(16, 16, 64, 16, 2, 128)  # fake, aligned pointers: never dereferenced
    assert lib.pa_write_kv(16, 16, 16, -1, ctypes.byref(ok), None) == PA_EINVAL
    bad_d = PaCache(16, 16, 64, 16, 2, 64)
    assert lib.pa_write_kv(16, 16, 16, 1, ctypes.byref(bad_d), None) == PA_EUNSUPPORTED
    bad_b = PaCache(16, 16, 64, 12, 2, 128)
    assert lib.pa_copy_blocks(ctypes.byref(bad_b), 16, 1, None) == PA_EUNSUPPORTED
    unaligned = PaCache(18, 16, 64, 16, 2, 128)
    assert lib.pa_copy_blocks(ctypes.byref(unaligned), 16, 1, None) == PA_EUNSUPPORTED
    assert lib.pa_decode(16, ctypes.byref(ok), 16, 4, 16, 1, 64, 5, 0.1, 16, None, 0, None) == PA_EINVAL
    assert lib.pa_decode(16, ctypes.byref(ok), 16, 4, 16, 1, 64, 6, 0.1, 16, None, 0, None) == PA_EUNSUPPORTED
    assert lib.pa_decode(16, ctypes.byref(ok), 16, 4, 16, 1, 64, 32, 0.1, 16, None, 0, None) == PA_EUNSUPPORTED
    # empty work is a successful no-op
    assert lib.pa_write_kv(None, None, None, 0, ctypes.byref(ok), None) == 0
    assert lib.pa_copy_blocks(ctypes.byref(ok), None, 0, None) == 0
    assert lib.pa_decode(None, ctypes.byref(ok), None, 0, None, 0, 0, 4, 0.1, None, None, 0, None) == 0
    # one partition per sequence -> no workspace; long sequences -> some
    assert lib.pa_decode_workspace_bytes(64, 32, 0, ctypes.byref(PaCache(16, 16, 26785, 16, 8, 128))) == 0
    assert lib.pa_decode_workspace_bytes(8, 32, 32768, ctypes.byref(PaCache(16, 16, 26785, 16, 8, 128))) > 0
    assert lib.pa_status_str(-3) == b"workspace too small"


def test_host_side_validation_of_the_widened_entry_points():
    """pa_attention, the FP8 entry points and pa_map_to_kernel_blocks reject
    bad arguments on the host (and treat empty work as a no-op) without
    touching the device."""
    from paged_kv_cache_333_b200._abi import (PA_EINVAL, PA_EUNSUPPORTED, PA_EWORKSPACE, PaCache, PaCacheFp8,
                                              lib)
    ok = PaCache(16, 16, 26785, 16, 8, 128)  # fake, aligned pointers: never dereferenced
    c = ctypes.byref(ok)

    def attn(q=16, T=4, qsl=16, R=1, maxq=4, cache=c, W=64, maxlen=600, Hq=32, scale=0.1, out=16, ws=None,
             ws_bytes=0):
        return lib.pa_attention(q, T, qsl, R, maxq, cache, 16, W, 16, maxlen, Hq, scale, out, ws, ws_bytes, None)

    assert attn(T=-1) == PA_EINVAL
    assert attn(R=0) == 0 and attn(T=0) == 0 and attn(maxq=0) == 0  # nothing to do
    assert attn(q=None) == PA_EINVAL and attn(qsl=None) == PA_EINVAL
    assert attn(Hq=30) == PA_EINVAL                       # not a multiple of the KV heads
    assert attn(Hq=24) == PA_EUNSUPPORTED                 # group size 3
    assert attn(q=18) == PA_EUNSUPPORTED                  # q not 16-byte aligned
    assert attn(scale=float("nan")) == PA_EINVAL
    # requests x column chunks > 65535: 40000 x 2 chunks of 32 columns (48 per request) on the mma.sync
    # kernel (chosen by the knob), 70000 x 1 chunk of 16 columns on it (the automatic choice below 17
    # columns), and 70000 x 1 unit of two heads' 64 columns on the tcgen05 kernel
    from paged_kv_cache_333_b200._abi import PA_ATTENTION_KERNEL_MMA
    prev = lib.pa_attention_set_kernel(PA_ATTENTION_KERNEL_MMA)
    try:
        assert attn(R=40000, T=40000, maxq=12) == PA_EUNSUPPORTED
    finally:
        lib.pa_attention_set_kernel(prev)
    assert attn(R=70000, T=70000, maxq=4) == PA_EUNSUPPORTED
    assert attn(R=70000, T=70000, maxq=16) == PA_EUNSUPPORTED
    assert attn(maxlen=32768) == PA_EWORKSPACE            # split-K needs scratch, none given
    assert lib.pa_attention_workspace_bytes(64, 256, 4, 32, 600, c) == 0
    assert lib.pa_attention_workspace_bytes(8, 32, 4, 32, 32768, c) > 0
    assert lib.pa_attention_workspace_bytes(8, 32, 4, 32, 32768, ctypes.byref(PaCache(16, 16, 8, 16, 8, 64))) == 0

    f8 = PaCacheFp8(16, 16, 64, 16, 2, 128, 1.0 / 64, 1.0 / 64)
    assert lib.pa_write_kv_fp8(16, 16, 16, -1, ctypes.byref(f8), None) == PA_EINVAL
    assert lib.pa_write_kv_fp8(None, None, None, 0, ctypes.byref(f8), None) == 0
    for k_scale in (0.0, -1.0, float("inf"), float("nan")):
        bad = PaCacheFp8(16, 16, 64, 16, 2, 128, k_scale, 1.0)
        assert lib.pa_write_kv_fp8(16, 16, 16, 1, ctypes.byref(bad), None) == PA_EINVAL
    assert lib.pa_copy_blocks_fp8(ctypes.byref(f8), None, 0, None) == 0
    assert lib.pa_copy_blocks_fp8(ctypes.byref(f8), None, 3, None) == PA_EINVAL
    assert lib.pa_copy_blocks_fp8(ctypes.byref(f8), 16, -1, None) == PA_EINVAL
    assert lib.pa_copy_blocks_fp8(ctypes.byref(f8), 16, 2**31, None) == PA_EUNSUPPORTED
    assert lib.pa_copy_blocks_fp8(ctypes.byref(PaCacheFp8(16, 16, 64, 12, 2, 128, 1.0, 1.0)), 16, 1,
                                  None) == PA_EUNSUPPORTED  # block size not a power of two
    assert lib.pa_copy_blocks_fp8(ctypes.byref(PaCacheFp8(16, 16, 64, 16, 2, 128, 0.0, 1.0)), 16, 1,
                                  None) == PA_EINVAL        # the descriptor's scales must be valid
    layers8 = (PaCacheFp8 * 2)(f8, f8)
    assert lib.pa_copy_blocks_layers_fp8(layers8, 2, None, 0, None) == 0
    assert lib.pa_copy_blocks_layers_fp8(layers8, 2, None, 4, None) == PA_EINVAL
    assert lib.pa_copy_blocks_layers_fp8(None, 2, 16, 4, None) == PA_EINVAL
    assert lib.pa_copy_blocks_layers_fp8(layers8, 129, 16, 4, None) == PA_EUNSUPPORTED
    assert lib.pa_copy_blocks_layers_fp8(layers8, 2, 16, 2**31, None) == PA_EUNSUPPORTED
    mixed8 = (PaCacheFp8 * 2)(f8, PaCacheFp8(32, 32, 64, 16, 4, 128, 1.0, 1.0))  # two geometries
    assert lib.pa_copy_blocks_layers_fp8(mixed8, 2, 16, 4, None) == PA_EINVAL
    bad_d = PaCacheFp8(16, 16, 64, 16, 2, 96, 1.0, 1.0)
    assert lib.pa_decode_fp8(16, ctypes.byref(bad_d), 16, 4, 16, 1, 64, 4, 0.1, 16, None, 0, None) == PA_EUNSUPPORTED
    assert lib.pa_decode_fp8(16, ctypes.byref(f8), 16, 4, 16, 1, 64, 6, 0.1, 16, None, 0, None) == PA_EUNSUPPORTED

    assert lib.pa_map_to_kernel_blocks(16, 4, 10, 0, 16, 40, None) == PA_EINVAL    # m < 1
    assert lib.pa_map_to_kernel_blocks(16, 4, 10, 4, 16, 39, None) == PA_EINVAL    # too narrow
    assert lib.pa_map_to_kernel_blocks(16, 4, 10, 4, None, 40, None) == PA_EINVAL
    assert lib.pa_map_to_kernel_blocks(None, 0, 10, 4, None, 40, None) == 0       # no rows


@pytest.mark.parametrize("missing", ["libpa.so", "libpa_pool.so"])
def test_package_refuses_to_import_without_its_libraries(tmp_path, missing):
    """No fallback path: a copy of the package without one of its built
    libraries fails at import, naming the library."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "paged_kv_cache_333_b200"
    shutil.copytree(os.path.join(ROOT, "paged_kv_cache_333_b200"), pkg,
                    ignore=shutil.ignore_patterns("csrc", "__pycache__"))
    os.remove(pkg / missing)
    r = subprocess.run([sys.executable, "-c", "import paged_kv_cache_333_b200"], cwd=tmp_path,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert missing in r.stderr


def test_split_k_partition_choice_through_the_workspace_sizes():
    """The partition heuristic, seen through the public workspace sizes (no
    device: the SM count falls back to B200's 148).  Chat lengths (<= 612
    tokens) take one partition, so no scratch; 32K context takes 640-token
    partitions: 52 per sequence, (m, l) float2 + 128 fp32 per (sequence,
    query head, partition)."""
    from paged_kv_cache_333_b200._abi import PaCache, lib
    c = ctypes.byref(PaCache(16, 16, 26785, 16, 8, 128))
    assert lib.pa_decode_workspace_bytes(64, 32, 612, c) == 0
    units = 8 * 32 * 52
    ml = units * 8
    expect = -(-ml // 256) * 256 + units * 128 * 4
    assert lib.pa_decode_workspace_bytes(8, 32, 32768, c) == expect
    # pa_attention over the same sequences, 4 rows each: per (row, head, partition)
    rows = 8 * 4
    cells = rows * 32 * 52
    acc_off = -(-cells * 8 // 256) * 256
    len_off = -(-(acc_off + cells * 128 * 4) // 256) * 256
    assert lib.pa_attention_workspace_bytes(8, rows, 4, 32, 32768, c) == len_off + rows * 4


def test_host_side_validation_of_the_remaining_entry_points():
    """Slot mapping, the fused positions write, the all-layer copy, the
    static-scratch decode and the process-wide knobs: every rejection below
    happens on the host, before any CUDA call (this machine has no device)."""
    from paged_kv_cache_333_b200._abi import (PA_DECODE_KERNEL_MMA, PA_DECODE_KERNEL_SIMT,
                                              PA_DECODE_STATIC_WS_BYTES, PA_EINVAL, PA_EUNSUPPORTED,
                                              PA_EWORKSPACE, PaCache, lib)
    ok = PaCache(16, 16, 26785, 16, 8, 128)  # fake, aligned pointers: never dereferenced
    c = ctypes.byref(ok)

    def slots(pos=16, req=16, T=4, bt=16, W=8, R=2, B=16, NB=64, out=16):
        return lib.pa_compute_slot_mapping(pos, req, T, bt, W, R, B, NB, out, None)

    assert slots(T=-1) == PA_EINVAL and slots(W=-1) == PA_EINVAL and slots(R=-1) == PA_EINVAL
    assert slots(B=0) == PA_EINVAL and slots(NB=0) == PA_EINVAL
    assert slots(T=0) == 0
    assert slots(pos=None) == PA_EINVAL and slots(req=None) == PA_EINVAL and slots(out=None) == PA_EINVAL
    assert slots(bt=None) == PA_EINVAL        # requests but no tables

    def wpos(k=16, v=16, pos=16, req=16, T=4, bt=16, W=8, R=2, cache=c):
        return lib.pa_write_kv_positions(k, v, pos, req, T, bt, W, R, cache, None)

    assert wpos(T=-1) == PA_EINVAL and wpos(R=-1) == PA_EINVAL
    assert wpos(T=0) == 0
    assert wpos(k=None) == PA_EINVAL and wpos(req=None) == PA_EINVAL and wpos(bt=None) == PA_EINVAL
    assert wpos(v=24) == PA_EUNSUPPORTED      # v not 16-byte aligned
    assert wpos(cache=ctypes.byref(PaCache(16, 16, 64, 16, 2, 64))) == PA_EUNSUPPORTED
    assert wpos(cache=ctypes.byref(PaCache(None, 16, 64, 16, 2, 128))) == PA_EINVAL

    layers = (PaCache * 3)(ok, ok, ok)
    assert lib.pa_copy_blocks_layers(layers, 3, None, 0, None) == 0
    assert lib.pa_copy_blocks_layers(layers, 0, 16, 5, None) == 0
    assert lib.pa_copy_blocks_layers(layers, 3, None, 5, None) == PA_EINVAL
    assert lib.pa_copy_blocks_layers(layers, 3, 16, -1, None) == PA_EINVAL
    assert lib.pa_copy_blocks_layers(None, 3, 16, 5, None) == PA_EINVAL
    assert lib.pa_copy_blocks_layers(layers, 129, 16, 5, None) == PA_EUNSUPPORTED
    mixed = (PaCache * 2)(ok, PaCache(16, 16, 26784, 16, 8, 128))  # one pair list, two geometries
    assert lib.pa_copy_blocks_layers(mixed, 2, 16, 5, None) == PA_EINVAL

    def static(q=16, S=4, maxlen=600, Hq=32, scale=0.1, out=16):
        return lib.pa_decode_static_ws(q, c, 16, 64, 16, S, maxlen, Hq, scale, out, None)

    assert static(S=-1) == PA_EINVAL and static(Hq=30) == PA_EINVAL and static(q=None) == PA_EINVAL
    assert static(Hq=24) == PA_EUNSUPPORTED and static(out=8) == PA_EUNSUPPORTED
    assert static(scale=float("inf")) == PA_EINVAL
    big = lib.pa_decode_workspace_bytes(64, 32, 32768, c)
    assert big > PA_DECODE_STATIC_WS_BYTES
    assert static(S=64, maxlen=32768) == PA_EWORKSPACE
    assert b"static" in lib.pa_last_cuda_error()

    prev = lib.pa_decode_set_kernel(PA_DECODE_KERNEL_SIMT)
    try:
        assert prev == PA_DECODE_KERNEL_MMA
        assert lib.pa_decode_set_kernel(7) == PA_DECODE_KERNEL_SIMT   # ignored, reports the current
        assert lib.pa_decode_set_kernel(PA_DECODE_KERNEL_MMA) == PA_DECODE_KERNEL_SIMT
    finally:
        lib.pa_decode_set_kernel(prev)
    prev = lib.pa_decode_set_partition_tokens(256)
    try:
        assert lib.pa_decode_set_partition_tokens(-5) == 256
        assert lib.pa_decode_set_partition_tokens(0) == 0            # negative means automatic
    finally:
        lib.pa_decode_set_partition_tokens(prev)
    for code, text in ((0, b"ok"), (-1, b"invalid argument"), (-2, b"unsupported"), (-4, b"CUDA"), (9, b"unknown")):
        assert text in lib.pa_status_str(code)


def test_attention_kernel_knob_and_the_tensor_memory_chunking():
    """pa_attention_set_kernel is a process-wide host setting that returns the
    previous choice; the tensor-memory kernel takes 128 (row, head) columns
    per CTA instead of 32, which the workspace size shows through the split-K
    partition heuristic (fewer column chunks -> fewer units -> more, shorter
    partitions).  Only sizes are computed here: nothing is launched."""
    from paged_kv_cache_333_b200._abi import (PA_ATTENTION_KERNEL_AUTO, PA_ATTENTION_KERNEL_MMA,
                                              PA_ATTENTION_KERNEL_TCGEN05, PA_ATTENTION_TCGEN05_MIN_COLUMNS,
                                              PaCache, lib)
    c = ctypes.byref(PaCache(16, 16, 26785, 16, 8, 128))

    def ws_bytes(rows, parts):
        cells = rows * 32 * parts
        acc_off = -(-cells * 8 // 256) * 256
        len_off = -(-(acc_off + cells * 128 * 4) // 256) * 256
        return len_off + rows * 4

    R, maxq, L = 8, 64, 32768          # 8 requests of 32K tokens, 64 rows each, G = 4: 256 columns
    slots = 148 * 4                    # no device: B200's SM count x the heuristic's 4 CTAs per SM

    def parts(units):
        part = max(640, -(-(L * units * 8) // (16 * slots)))
        part = -(-part // 64) * 64
        return -(-L // part)

    prev = lib.pa_attention_set_kernel(PA_ATTENTION_KERNEL_MMA)
    try:
        assert lib.pa_attention_workspace_bytes(R, R * maxq, maxq, 32, L, c) == ws_bytes(R * maxq, parts(R * 8))
        assert lib.pa_attention_set_kernel(PA_ATTENTION_KERNEL_TCGEN05) == PA_ATTENTION_KERNEL_MMA
        assert lib.pa_attention_set_kernel(9) == PA_ATTENTION_KERNEL_TCGEN05   # ignored
        assert lib.pa_attention_workspace_bytes(R, R * maxq, maxq, 32, L, c) == ws_bytes(R * maxq, parts(R * 2))
        assert parts(R * 2) == 52 and parts(R * 8) == 19
        # chat lengths stay one partition either way: no scratch
        assert lib.pa_attention_workspace_bytes(64, 64 * 16, 16, 32, 612, c) == 0
        # automatic choice: the tensor-memory kernel from the column threshold on
        assert lib.pa_attention_set_kernel(PA_ATTENTION_KERNEL_AUTO) == PA_ATTENTION_KERNEL_TCGEN05
        assert maxq * 4 >= PA_ATTENTION_TCGEN05_MIN_COLUMNS
        assert lib.pa_attention_workspace_bytes(R, R * maxq, maxq, 32, L, c) == ws_bytes(R * maxq, parts(R * 2))
        few = PA_ATTENTION_TCGEN05_MIN_COLUMNS // 4 - 1  # rows per request just below the threshold at G = 4
        assert lib.pa_attention_workspace_bytes(R, R * few, few, 32, L, c) == ws_bytes(
            R * few, parts(R * -(-(few * 4) // 32)))
    finally:
        lib.pa_attention_set_kernel(prev)
    assert lib.pa_attention_set_kernel(prev) == prev == PA_ATTENTION_KERNEL_AUTO


def test_binding_refuses_tensors_of_another_device(monkeypatch):
    """The library launches on the current device; the binding refuses a
    tensor (or stream) that lives on another GPU instead of passing its
    pointer.  Checked on CPU with a tensor that reports cuda:1 while the
    current device is cuda:0 (nothing is launched)."""
    import torch
    from paged_kv_cache_333_b200 import _abi

    class OnGpu1(torch.Tensor):
        @property
        def is_cuda(self):
            return True

        @property
        def device(self):
            return torch.device("cuda", 1)

    t = torch.Tensor._make_subclass(OnGpu1, torch.zeros(8, dtype=torch.bfloat16))
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="current CUDA device is cuda:0"):
        _abi._dev(t, "q", torch.bfloat16)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    assert _abi._dev(t, "q", torch.bfloat16) == t.data_ptr()
    with pytest.raises(TypeError, match="must be torch.int32"):
        _abi._dev(t, "q", torch.int32)

    class Stream1:
        device = torch.device("cuda", 1)
        cuda_stream = 1234
    assert _abi._stream_ptr(Stream1()) == 1234
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="stream is on cuda:1"):
        _abi._stream_ptr(Stream1())
    assert _abi._stream_ptr(5678) == 5678      # a raw handle: nothing to check


def test_counts_past_the_launch_limits_are_refused_on_the_host():
    """Token and pair counts above INT32_MAX, and more than 65535 KV heads,
    are refused before any size arithmetic could overflow (fake pointers:
    nothing is launched)."""
    from paged_kv_cache_333_b200._abi import PA_EUNSUPPORTED, PaCache, PaCacheFp8, lib
    c = ctypes.byref(PaCache(16, 16, 64, 16, 2, 128))
    for n in (2**31, 2**40, 2**62, 2**63 - 1):
        assert lib.pa_write_kv(16, 16, 16, n, c, None) == PA_EUNSUPPORTED
        assert lib.pa_write_kv_positions(16, 16, 16, 16, n, 16, 8, 2, c, None) == PA_EUNSUPPORTED
        assert lib.pa_compute_slot_mapping(16, 16, n, 16, 8, 2, 16, 64, 16, None) == PA_EUNSUPPORTED
        assert lib.pa_write_kv_fp8(16, 16, 16, n, ctypes.byref(PaCacheFp8(16, 16, 64, 16, 2, 128, 1.0, 1.0)),
                                   None) == PA_EUNSUPPORTED
        assert lib.pa_copy_blocks(c, 16, n, None) == PA_EUNSUPPORTED
        assert lib.pa_copy_blocks_layers((PaCache * 2)(PaCache(16, 16, 64, 16, 2, 128),
                                                       PaCache(32, 32, 64, 16, 2, 128)), 2, 16, n,
                                         None) == PA_EUNSUPPORTED
    wide = ctypes.byref(PaCache(16, 16, 4, 16, 70000, 128))
    assert lib.pa_write_kv(16, 16, 16, 1, wide, None) == PA_EUNSUPPORTED
    assert lib.pa_copy_blocks(wide, 16, 1, None) == PA_EUNSUPPORTED
    assert lib.pa_decode(16, wide, 16, 4, 16, 1, 64, 70000, 0.1, 16, None, 0, None) == PA_EUNSUPPORTED
