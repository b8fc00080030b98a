"""bench.py's measurement helpers on the CPU: the algorithmic bytes it
divides by, the ncu traffic it reports (only while the captured kernel
sources are unchanged), and the host timing of the scheduler step."""
import os
import shutil
import types

import numpy as np

import bench
import synth


def _step(tables, lens, B=4, H=2, D=128, dtype="bf16", T=2, P=0):
    return types.SimpleNamespace(
        num_kv_heads=H, head_dim=D, block_size=B, kv_dtype=dtype, ids=list(range(len(lens))),
        seq_lens_np=np.array(lens, np.int32), block_tables_np=np.array(tables, np.int32),
        slot_mapping_np=np.zeros(T, np.int64), cow_pairs_np=np.zeros((P, 2), np.int64),
        q=types.SimpleNamespace(numel=lambda: len(lens) * 8 * D))


def test_algorithmic_bytes_count_shared_blocks_once():
    # sequence 1 shares block 7 (positions 0..3) with sequence 0
    st = _step([[7, 2, -1], [7, 9, -1]], [6, 5])
    b = bench.algorithmic_bytes(st)
    row = 2 * 128 * 2
    unique = 4 + 2 + 1  # block 7 (4 slots), block 2 (2 of its slots), block 9 (1 slot)
    assert b["decode_kv"] == unique * row * 2
    assert b["decode_kv_logical"] == 11 * row * 2
    assert b["table"] == (2 + 2) * 4
    assert b["write"] == 2 * 2 * 128 * 2 * 2 + 2 * row * 2
    fp8 = bench.algorithmic_bytes(_step([[7, 2, -1], [7, 9, -1]], [6, 5], dtype="fp8"))
    assert fp8["decode_kv"] == b["decode_kv"] // 2
    rows4 = bench.algorithmic_bytes(st, rows_per_seq=4)
    assert rows4["q_out"] == 4 * b["q_out"] and rows4["decode_kv"] == b["decode_kv"]


def test_profiled_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    for kind in ("bf16", "fp8", "rows4", "rows16_tcgen05"):
        t = bench.profiled_traffic("chat", kind)
        assert isinstance(t, int) and t > 0, kind
    assert bench.profiled_traffic("long", "bf16") is None  # captured on chat only
    assert bench.profiled_traffic("chat", "rows8") is None
    assert bench.profiled_traffic("sweep_b1", "fp8") > 0  # a second capture of the same kind
    # a copy of the tree with one kernel source edited: no traffic reported
    root = tmp_path / "tree"
    shutil.copytree(os.path.join(bench.ROOT, "profiles"), root / "profiles")
    shutil.copytree(os.path.join(bench.ROOT, "paged_kv_cache_333_b200", "csrc"),
                    root / "paged_kv_cache_333_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.profiled_traffic("chat", "bf16") is not None
    with open(root / "paged_kv_cache_333_b200" / "csrc" / "decode_mma.cuh", "a") as f:
        f.write("\n")
    assert bench.profiled_traffic("chat", "bf16") is None
    assert bench.profiled_traffic("chat", "fp8") is None  # also hashes decode_mma.cuh


def test_host_pool_step_timing_runs_the_step():
    r = bench.host_pool_step_us(synth.tiny(), steps=20)
    assert r["steps"] == 20 and r["sequences"] == 4 and r["us"] > 0


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the CPU oracle on a bounded sample of the
    chat workload, split over the host's cores) prints exactly one JSON line
    with the contract's keys, its metric and unit matching the GPU arm's."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["vs_baseline"] is None and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == bench.host_cores() and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_clock_samples_give_median_max_and_active_reasons():
    """The bench line's `clocks` field from nvidia-smi samples: median SM clock
    under load, the max clock, the throttle reasons seen Active, and only
    this GPU's rows when the sampler knows its UUID (other GPUs ignored)."""
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.uuid = "GPU-aaa"
    s.proc = types.SimpleNamespace(terminate=lambda: None, wait=lambda timeout=None: 0, kill=lambda: None)
    row = "{u}, {sm}, 1965, 700.5, 0x0, Not Active, Not Active, {swt}, {cap}"
    s.lines = [row.format(u="GPU-aaa", sm=1965, swt="Not Active", cap="Not Active"),
               row.format(u="GPU-aaa", sm=1900, swt="Not Active", cap="Active"),
               row.format(u="GPU-aaa", sm=1800, swt="Not Active", cap="Not Active"),
               row.format(u="GPU-bbb", sm=300, swt="Active", cap="Active"),   # another GPU on the host
               "garbage line"]
    c = bench.ClockSampler.stop(s)
    assert c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965 and c["samples"] == 3
    assert c["reasons"] == ["sw_power_cap"]
    # rows only for other GPUs (a UUID format this sampler does not match):
    # no clock is reported, and nothing of the other GPUs leaks in
    s.uuid = "MIG-ccc"
    c = bench.ClockSampler.stop(s)
    assert c["sm_mhz"] is None and c["sm_max_mhz"] is None and c["samples"] == 0
    assert c["reasons"] == ["uuid not matched"]
    s.proc = None
    assert bench.ClockSampler.stop(s)["reasons"] == ["nvidia-smi unavailable"]


def test_roofline_peak_reads_the_measured_file_else_falls_back(tmp_path, monkeypatch):
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peak, how = bench.measured_peak()
    assert peak == bench.FALLBACK_HBM_GBS and how.startswith("fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6558.4, "bf16_tflops": 1590}))
    peak, how = bench.measured_peak()
    assert peak == 6558.4 and how.startswith("measured")


def test_cpu_baseline_states_cores_and_keeps_the_one_thread_timing():
    """The oracle fanned out over every host core (the reported value, its
    thread count stated) and on one thread, on the same workload."""
    cb = bench.cpu_baseline(synth.tiny(), 0.4)
    assert cb["kind"] == "oracle" and cb["cores"] == cb["cores_available"] == bench.host_cores()
    assert cb["value"] > 0 and cb["single_thread"]["cores"] == 1 and cb["single_thread"]["value"] > 0


def test_split_oracle_layer_computes_every_pair_once(monkeypatch):
    """The all-cores timing splits a layer's (sequence, head) pairs into
    disjoint shares that together cover every pair exactly once."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    w = synth.tiny()
    seen = []
    monkeypatch.setattr(oracle, "decode", lambda *a: seen.append(np.asarray(a[-1]).copy()))
    with ThreadPoolExecutor(max_workers=3) as pool:
        bench._oracle_layer_threads(w, {"k_cache": None, "v_cache": None, "block_tables": None, "seq_lens": None},
                                    pool, 3)
    pairs = np.concatenate(seen)
    assert len(seen) == 3
    expect = {(s, j) for s in range(len(w.seq_ids)) for j in range(w.shape.num_q_heads)}
    assert len(pairs) == len(expect) and {tuple(p) for p in pairs} == expect


def test_related_runs_default_to_fp8_and_sixteen_rows():
    args = bench.argparse.Namespace(related="auto", config="chat", queries=1, kv_dtype="bf16", part_tokens=0)
    assert bench.related_runs(args) == ["fp8", "rows16"]
    for change in ({"config": "long"}, {"queries": 4}, {"kv_dtype": "fp8"}, {"part_tokens": 640}):
        assert bench.related_runs(bench.argparse.Namespace(**{**vars(args), **change})) == []
    assert bench.related_runs(bench.argparse.Namespace(**{**vars(args), "related": "none"})) == []
    assert bench.related_runs(bench.argparse.Namespace(**{**vars(args), "related": "rows16,other"})) == ["rows16"]


def test_extra_configs_default_to_the_long_context_decode():
    args = bench.argparse.Namespace(extra_configs="auto", config="chat", queries=1, kv_dtype="bf16", part_tokens=0)
    assert bench.extra_configs(args) == ["long"]
    for change in ({"config": "long"}, {"queries": 4}, {"kv_dtype": "fp8"}, {"part_tokens": 640}):
        assert bench.extra_configs(bench.argparse.Namespace(**{**vars(args), **change})) == []
    assert bench.extra_configs(bench.argparse.Namespace(**{**vars(args), "extra_configs": "none"})) == []
    assert bench.extra_configs(bench.argparse.Namespace(**{**vars(args), "extra_configs": "long,chat,sweep_b1"})) == [
        "long", "sweep_b1"]
