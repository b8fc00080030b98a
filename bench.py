#!/usr/bin/env python
"""Benchmark: one decode step of Llama-3-8B-shaped paged attention on B200.

A step runs, for each of --layers layers (distinct KV caches of the full
26,785-block pool, so the timed inputs are far larger than L2): the
copy-on-write copies the step queued (none for the chat workload), the
slot-mapped KV write of one new token per sequence, and paged decode
attention.  Inputs are resident in HBM when the timed region starts.

  value  = algorithmic bytes of the step (unique KV bytes the decode reads
           + the write's and the copies' bytes) / step time, in GB/s;
  e2e    = the same bytes / time of the same step driven from pinned host
           buffers (per layer: q, k, v in; out back), copies included;
  roofline = the decode kernel alone: unique KV bytes per launch / its mean
           duration (CUDA events on its stream) vs. measured HBM peak.

--impl reference times the CPU oracle (its (sequence, head) pairs split over
the host's cores) on a bounded sample of the same workload.  The default run
also reports the oracle in cpu_baseline, with a one-thread timing beside it,
and times, under per_config, the 32K long-context decode and two variants of
the chat step: the FP8 cache's decode and 16 query rows per sequence through
pa_attention.  With torchrun
(N > 1) every rank runs its own replica (the path does not shard; no
collective is needed) and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import copy
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "paged decode attention: KV HBM GB/s & % of B200 peak; decode tokens/s per layer"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0

WORKLOAD_TEXT = {
    "chat": "Llama-3-8B chat decode: 64 seqs, len U[512,612], 32 q / 8 KV heads, d=128, block 16, "
            "26,785-block pool, shuffled free list",
    "long": "Long-context decode: 8 seqs {32768 x4, 8192 x4}, 32 q / 8 KV heads, d=128, block 16, "
            "26,785-block pool",
    "prefix": "Prefix sharing + CoW: 256 seqs, 2040-token shared prefix, suffix U[1,256], "
              "32 q / 8 KV heads, d=128, block 16",
    "tiny": "Tiny: 4 seqs {2,18,34,101}, 8 q / 2 KV heads, d=128, block 16, 64-block pool",
    "sweep_b1": "Block-size sweep, B=1: 128 seqs, geometric lengths (mean 1000, cap 8192), pool of "
                "428,560 blocks at 90% occupancy after 10k seeded alloc/free events",
    "sweep_b16": "Block-size sweep, B=16: 128 seqs, geometric lengths (mean 1000, cap 8192), pool of "
                 "26,785 blocks at 90% occupancy after 10k seeded alloc/free events",
    "sweep_b32": "Block-size sweep, B=32: 128 seqs, geometric lengths (mean 1000, cap 8192), pool of "
                 "13,392 blocks at 90% occupancy after 10k seeded alloc/free events",
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="chat")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-op", action="store_true")
    ap.add_argument("--part-tokens", type=int, default=0, help="split-K partition size (0 = automatic)")
    ap.add_argument("--queries", type=int, default=1,
                    help="query rows per request: 1 = decode (pa_decode); Q > 1 = the last Q tokens of every "
                         "request are its rows (speculative decode / prefill chunk; pa_attention)")
    ap.add_argument("--attention-kernel", choices=["default", "mma", "tcgen05"], default="default",
                    help="pa_attention kernel for --queries > 1 (default = the library's own choice)")
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8"], default="bf16",
                    help="KV cache element type (fp8 = OCP E4M3 codes with per-tensor scales)")
    ap.add_argument("--extra-configs", default="auto",
                    help="comma-separated workloads whose bf16 decode is also timed in this run and reported "
                         "under per_config (auto = the 32K long-context one when the main run is the chat "
                         "decode; none = no extra)")
    ap.add_argument("--related", default="auto",
                    help="comma-separated variants of the main workload also timed in this run and reported "
                         "under per_config: fp8 (the FP8 cache's decode), rows16 (16 query rows per sequence "
                         "through pa_attention); auto = both when the main run is the chat bf16 decode; none")
    args = ap.parse_args()
    if args.queries > 1 and args.kv_dtype == "fp8":
        ap.error("--queries > 1 runs pa_attention, which reads a bf16 cache: use --kv-dtype bf16")
    return args


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device) -> float:
    """Max of a per-rank number over all ranks (identity without a process
    group).  Device times of the replicas are combined this way."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, bytes_per_replica: float, seconds: float) -> float:
    """GB/s of the whole job: every replica moves bytes_per_replica in the
    (max over ranks) time."""
    return world * bytes_per_replica / seconds / 1e9


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, torch copy_ read+write)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier measurement on this pool)"


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.uuid = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            pass
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [r.split(", ") for r in self.lines if r.count(",") >= 8]
        if self.uuid:
            mine = [r for r in rows if r[0].strip() == self.uuid]
            if rows and not mine:
                # Samples came back, none of them for this GPU: report no
                # clock rather than other jobs' clocks and throttle reasons.
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["uuid not matched"],
                        "samples": 0, "uuid": self.uuid}
            rows = mine
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- ncu traffic
PROFILE_FOR = {"bf16": ("decode_mma_chat_full.md",),
               "fp8": ("decode_fp8_chat_full.md", "decode_fp8_sweep_b1_full.md"),
               "rows4": ("attention_q4_chat_full.md",), "rows16_tcgen05": ("attention_tc_q16_chat_full.md",)}


def profiled_traffic(config: str, kind: str = "bf16"):
    """DRAM bytes (read + write) per launch of the timed kernel from the
    committed ncu capture of that kernel (kind: "bf16" decode, "fp8" decode,
    "rows4" = pa_attention with 4 rows per sequence on the mma.sync kernel,
    "rows16_tcgen05" = 16 rows on the tcgen05 kernel), if a capture of that
    kind was of this workload and of the kernel sources as they are now;
    otherwise None."""
    import hashlib
    for name in PROFILE_FOR.get(kind, ()):
        try:
            text = open(os.path.join(ROOT, "profiles", name)).read()
        except OSError:
            continue
        fields = {}
        for line in text.splitlines():
            line = line.strip()
            if ":" in line and line.split(":")[0] in ("kernel_sources_sha256_16", "workload",
                                                       "traffic_bytes_per_launch"):
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
        if fields.get("workload") != config or "traffic_bytes_per_launch" not in fields:
            continue
        csrc = os.path.join(ROOT, "paged_kv_cache_333_b200", "csrc")
        current = True
        for item in fields.get("kernel_sources_sha256_16", "").split():
            fname, digest = item.split("=")
            with open(os.path.join(csrc, fname), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest()[:16] != digest:
                    current = False
        if current:
            return int(fields["traffic_bytes_per_launch"])
    return None


# --------------------------------------------------------------------------- bytes
def algorithmic_bytes(st, rows_per_seq: int = 1) -> dict:
    """Bytes the step must move, per layer (rows_per_seq new K/V rows and
    query rows per sequence)."""
    H, D, B = st.num_kv_heads, st.head_dim, st.block_size
    esz = 1 if st.kv_dtype == "fp8" else 2
    row = H * D * esz  # one token's K (or V) row in the cache
    slots = []
    for s in range(len(st.ids)):
        n = int(st.seq_lens_np[s])
        pos = np.arange(n, dtype=np.int64)
        slots.append(st.block_tables_np[s, pos // B].astype(np.int64) * B + pos % B)
    uniq = np.unique(np.concatenate(slots)).size if slots else 0
    logical = int(st.seq_lens_np.sum())
    T = st.slot_mapping_np.size * rows_per_seq
    P = st.cow_pairs_np.shape[0]
    return {
        "decode_kv": uniq * row * 2,  # K and V, each unique slot once
        "decode_kv_logical": logical * row * 2,
        "write": T * H * D * 2 * 2 + T * row * 2,  # bf16 K and V rows read, cache rows written
        "copy": P * B * row * 2 * 2,  # K and V blocks read and written
        "q_out": 2 * st.q.numel() * rows_per_seq * 2,
        "table": int(sum(-(-int(n) // B) for n in st.seq_lens_np)) * 4,
    }


def host_pool_step_us(w, steps: int = 200) -> dict:
    """Host time of the scheduler-side step (the block table and slot
    mapping build) on the C++ pool, as one pa_pool_step call: append one
    token to every sequence, take the queued copy pairs, build the step's
    slot mapping and lengths, and update the block table kept across steps
    (append-only).  The step's arrays are allocated once for the batch
    (StepBuffers) and reused.  Timed on a fresh pool laid out as the workload
    (the timed device step uses its own)."""
    from paged_kv_cache_333_b200.pool import BlockPool, StepBuffers
    sh = w.shape
    pool = BlockPool(sh.num_blocks, sh.block_size, w.free_order, "shared")
    w.ops(pool)
    if w.suffix_ops is not None:
        w.suffix_ops(pool)
    pool.take_cow_pairs()
    ids = np.asarray(w.seq_ids, dtype=np.int64)
    width = max(pool.num_blocks_of(int(i)) for i in ids) + steps // sh.block_size + 2
    buf = StepBuffers(ids, 1, width)
    pool.step_into(buf)  # the first step writes whole table rows; the timed ones are incremental
    done = 0
    t0 = time.perf_counter()
    for _ in range(steps):
        if pool.step_into(buf) is None:
            break
        done += 1
    dt = time.perf_counter() - t0
    return {"us": round(dt / max(done, 1) * 1e6, 2), "steps": done, "sequences": int(len(ids)),
            "what": "pa_pool_step: append 1 token per sequence + copy pairs + slot mapping + block table "
                    "(updated append-only) + lengths, one ctypes call on arrays allocated once, one host thread"}


# --------------------------------------------------------------------------- timing
def capture_graph(fn, dev):
    """One CUDA graph of `fn`'s launches (no host work in the timed loop)."""
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            fn()
    torch.cuda.current_stream(dev).wait_stream(side)
    return g


def timed_replays(g, reps, dev, world):
    """Device milliseconds of `reps` replays of graph g, with CUDA events on
    the replay stream, a barrier and a synchronize on both sides; the max over
    ranks."""
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0.record()
    for _ in range(reps):
        g.replay()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    return reduce_max(t0.elapsed_time(t1), dev)


# --------------------------------------------------------------------------- ours
def run_ours(args, world, rank, local):
    import synth
    import paged_kv_cache_333_b200 as pa
    from paged_kv_cache_333_b200.workload import stage

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.part_tokens:
        pa.pa_decode_set_partition_tokens(args.part_tokens)
    if args.attention_kernel != "default":
        pa.pa_attention_set_kernel(args.attention_kernel)
    w = synth.by_name(args.config)
    fp8 = args.kv_dtype == "fp8"
    st = stage(w, dev, layers=args.layers, kv_dtype=args.kv_dtype)
    L = args.layers
    Q = args.queries
    if Q > 1 and (fp8 or st.cow_pairs.shape[0] > 0):
        raise SystemExit("--queries > 1 is measured on bf16 caches of workloads without copy-on-write pairs")
    S = len(st.ids)
    # The step's inputs.  Decode: one new token per sequence.  --queries Q: the
    # last Q tokens of every sequence are its query rows; their K/V rows are
    # written again (same values, same slots) and pa_attention reads them.
    inp = {"q": st.q, "k": st.k_new, "v": st.v_new, "slots": st.slot_mapping, "bt": st.block_tables,
           "lens": st.seq_lens, "out": st.out, "ws": st.workspace}
    if Q > 1:
        lens_np = st.seq_lens_np.astype(np.int64)
        if int(lens_np.min()) < Q:
            raise SystemExit("--queries exceeds a sequence length")
        pos = np.concatenate([np.arange(n - Q, n) for n in lens_np])
        req = np.repeat(np.arange(S), Q)
        slots_np = st.block_tables_np[req, pos // st.block_size].astype(np.int64) * st.block_size + pos % st.block_size
        k_rows = np.concatenate([w.rows("k", sid, int(n) - Q, int(n)) for sid, n in zip(st.ids, lens_np)])
        v_rows = np.concatenate([w.rows("v", sid, int(n) - Q, int(n)) for sid, n in zip(st.ids, lens_np)])
        q_rows = synth.bf16_normal(synth.make_rng(900 + Q), (S * Q, st.num_q_heads, st.head_dim))
        to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(dev).view(
            torch.bfloat16)
        inp.update(q=to_dev(q_rows), k=to_dev(k_rows), v=to_dev(v_rows), slots=torch.from_numpy(slots_np).to(dev),
                   qsl=torch.arange(0, S * Q + 1, Q, dtype=torch.int32, device=dev))
        inp["out"] = torch.empty_like(inp["q"])
        need = pa.pa_attention_workspace_bytes(S, S * Q, Q, st.num_q_heads, st.max_seq_len, *st.caches[0])
        inp["ws"] = torch.empty(need, dtype=torch.uint8, device=dev) if need else None
    # which pa_attention kernel runs (the library's automatic choice unless forced)
    group = st.num_q_heads // st.num_kv_heads
    attention_tc = Q > 1 and (args.attention_kernel == "tcgen05" or (
        args.attention_kernel == "default" and Q * group >= pa._abi.PA_ATTENTION_TCGEN05_MIN_COLUMNS))
    nbytes = algorithmic_bytes(st, rows_per_seq=Q)
    step_bytes = L * (nbytes["decode_kv"] + nbytes["write"] + nbytes["copy"])
    stream = torch.cuda.current_stream(dev)
    has_pairs = st.cow_pairs.shape[0] > 0
    split = inp["ws"] is not None
    launches_per_layer = 2 + (1 if split else 0) + (1 if has_pairs else 0)

    def write_op(k, v, slots, kc, vc):
        if fp8:
            pa.pa_write_kv_fp8(k, v, slots, kc, vc, st.k_scale, st.v_scale)
        else:
            pa.pa_write_kv(k, v, slots, kc, vc)

    def copy_op(kc, vc, pairs):
        if fp8:
            pa.pa_copy_blocks_fp8(kc, vc, pairs)
        else:
            pa.pa_copy_blocks(kc, vc, pairs)

    def decode_op(q, kc, vc, bt, lens, qsl=None, out=None, ws=None):
        out = inp["out"] if out is None else out
        ws = inp["ws"] if ws is None else ws
        if Q > 1:
            pa.pa_attention(q, qsl, kc, vc, bt, lens, st.scale, max_query_len=Q, out=out,
                            max_seq_len=st.max_seq_len, workspace=ws)
        elif fp8:
            pa.pa_decode_fp8(q, kc, vc, st.k_scale, st.v_scale, bt, lens, st.scale, out=out,
                             max_seq_len=st.max_seq_len, workspace=ws)
        else:
            pa.pa_decode(q, kc, vc, bt, lens, st.scale, out=out, max_seq_len=st.max_seq_len, workspace=ws)

    def layer_ops(l, with_decode=True, with_write=True):
        kc, vc = st.caches[l]
        if with_write:
            if has_pairs:
                copy_op(kc, vc, st.cow_pairs)
            write_op(inp["k"], inp["v"], inp["slots"], kc, vc)
        if with_decode:
            decode_op(inp["q"], kc, vc, inp["bt"], inp["lens"], inp.get("qsl"))

    capture = lambda fn: capture_graph(fn, dev)
    timed = lambda g, reps: timed_replays(g, reps, dev, world)

    # eager warm-up (kernel attributes, tensor maps), then graphs
    for l in range(L):
        layer_ops(l)
    torch.cuda.synchronize()
    g_step = capture(lambda: [layer_ops(l) for l in range(L)])
    g_dec = capture(lambda: [layer_ops(l, with_write=False) for l in range(L)])
    for _ in range(args.warmup):
        g_step.replay()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(clear=True) == 0

    K = args.steps
    clocks = ClockSampler(local)
    clocks.start()
    ms_total = timed(g_step, K)
    clk = clocks.stop()
    for _ in range(args.warmup):
        g_dec.replay()
    dec_ms_total = timed(g_dec, K)
    ms_step = ms_total / K
    value = whole_job_rate(world, step_bytes, ms_step * 1e-3)
    dec_mean_ms = dec_ms_total / (K * L)
    peak, peak_src = measured_peak()
    achieved = nbytes["decode_kv"] / (dec_mean_ms * 1e-3) / 1e9

    # ---- per-op times (graphs of one launch per layer) -------------------------
    per_op = {"pool_step_host": host_pool_step_us(w)}
    if Q > 1:
        per_op["attention"] = {"us": round(dec_mean_ms * 1e3, 3), "GB/s": round(achieved, 2),
                               "rows_per_s": round(S * Q / (dec_mean_ms * 1e-3), 1)}
    if not args.no_per_op and not fp8 and Q == 1:
        row = st.num_kv_heads * st.head_dim * 2
        T = st.slot_mapping.numel()
        pos = st.seq_lens.to(torch.int64) - 1  # decode step: the new token is the last
        req = torch.arange(len(st.ids), dtype=torch.int32, device=dev)
        used = st.block_tables_np[st.block_tables_np >= 0]
        free = np.array(st.pool.free_list(), dtype=np.int64)
        P = int(min(255, len(np.unique(used)), len(free)))  # a prefix-sharing CoW burst: 255 pairs
        pairs = torch.from_numpy(np.stack([np.unique(used)[:P].astype(np.int64), free[:P]], 1).copy()).to(dev)
        blk_bytes = st.block_size * row

        def time_ops(fn, launches):
            g = capture(fn)
            g.replay()
            torch.cuda.synchronize()
            return timed(g, K) / (K * launches) * 1e3  # us per launch

        us = time_ops(lambda: [pa.pa_write_kv(st.k_new, st.v_new, st.slot_mapping, *st.caches[l])
                               for l in range(L)], L)
        per_op["write_kv"] = {"us": round(us, 3), "GB/s": round(T * row * 4 / us / 1e3, 2)}
        us = time_ops(lambda: [pa.pa_write_kv_positions(st.k_new, st.v_new, pos, req, st.block_tables,
                                                        *st.caches[l]) for l in range(L)], L)
        per_op["write_kv_positions"] = {"us": round(us, 3), "GB/s": round(T * row * 4 / us / 1e3, 2)}
        if P:
            us = time_ops(lambda: [pa.pa_copy_blocks(*st.caches[l], pairs) for l in range(L)], L)
            per_op["copy_blocks"] = {"pairs": P, "us": round(us, 3),
                                     "GB/s": round(P * blk_bytes * 4 / us / 1e3, 2)}
            us = time_ops(lambda: pa.pa_copy_blocks_layers(st.caches, pairs), 1)
            per_op["copy_blocks_layers"] = {"pairs": P, "layers": L, "us": round(us, 3),
                                            "GB/s": round(L * P * blk_bytes * 4 / us / 1e3, 2)}
        per_op["decode"] = {"us": round(dec_mean_ms * 1e3, 3), "GB/s": round(achieved, 2)}
        assert pa.pa_get_device_error(clear=True) == 0

    # ---- end to end: the same step from pinned host buffers -------------------
    e2e = None
    if not args.no_e2e:
        # The step as a serving loop would run it from pinned host memory:
        # the per-step metadata and every layer's q, k, v rows go in on a copy
        # stream (into per-layer device buffers; a layer's q, k and v sit back
        # to back in one pinned buffer, so they cross in one copy), layer l's
        # kernels wait only for layer l's inputs, and layer l's output goes
        # back on a second copy stream while the later layers compute.
        nq, nk, nv = inp["q"].numel(), inp["k"].numel(), inp["v"].numel()
        qkv_h = torch.empty(nq + nk + nv, dtype=inp["q"].dtype).pin_memory()
        qkv_h[:nq].copy_(inp["q"].reshape(-1))
        qkv_h[nq:nq + nk].copy_(inp["k"].reshape(-1))
        qkv_h[nq + nk:].copy_(inp["v"].reshape(-1))
        q_h, k_h, v_h = qkv_h[:nq], qkv_h[nq:nq + nk], qkv_h[nq + nk:]
        sm_h = inp["slots"].cpu().pin_memory()
        bt_h, sl_h = inp["bt"].cpu().pin_memory(), inp["lens"].cpu().pin_memory()
        qsl_h = inp["qsl"].cpu().pin_memory() if Q > 1 else None
        out_h = [torch.empty(inp["out"].shape, dtype=inp["out"].dtype).pin_memory() for _ in range(L)]
        qkv_d = [torch.empty_like(qkv_h, device=dev) for _ in range(L)]
        q_d = [b[:nq].view(inp["q"].shape) for b in qkv_d]
        k_d = [b[nq:nq + nk].view(inp["k"].shape) for b in qkv_d]
        v_d = [b[nq + nk:].view(inp["v"].shape) for b in qkv_d]
        out_d = [torch.empty_like(inp["out"]) for _ in range(L)]
        ws_d = [torch.empty_like(inp["ws"]) if inp["ws"] is not None else None for _ in range(L)]
        sm_d, bt_d, sl_d = (torch.empty_like(inp["slots"]), torch.empty_like(inp["bt"]),
                            torch.empty_like(inp["lens"]))
        qsl_d = torch.empty_like(inp["qsl"]) if Q > 1 else None
        pairs_h = st.cow_pairs.cpu().pin_memory() if has_pairs else None
        pairs_d = torch.empty_like(st.cow_pairs) if has_pairs else None
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_step():
            main = torch.cuda.current_stream(dev)
            s_in.wait_stream(main)
            ready = []
            with torch.cuda.stream(s_in):
                sm_d.copy_(sm_h, non_blocking=True)
                bt_d.copy_(bt_h, non_blocking=True)
                sl_d.copy_(sl_h, non_blocking=True)
                if Q > 1:
                    qsl_d.copy_(qsl_h, non_blocking=True)
                if has_pairs:
                    pairs_d.copy_(pairs_h, non_blocking=True)
                for l in range(L):
                    qkv_d[l].copy_(qkv_h, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(s_in)
                    ready.append(ev)
            for l in range(L):
                kc, vc = st.caches[l]
                main.wait_event(ready[l])
                if has_pairs:
                    copy_op(kc, vc, pairs_d)
                write_op(k_d[l], v_d[l], sm_d, kc, vc)
                decode_op(q_d[l], kc, vc, bt_d, sl_d, qsl_d, out=out_d[l], ws=ws_d[l])
                done = torch.cuda.Event()
                done.record(main)
                s_out.wait_event(done)
                with torch.cuda.stream(s_out):
                    out_h[l].copy_(out_d[l], non_blocking=True)
            main.wait_stream(s_out)

        e2e_step()
        torch.cuda.synchronize()
        g_e2e = capture(e2e_step)
        for _ in range(args.warmup):
            g_e2e.replay()
        e_ms = timed(g_e2e, K)
        h2d = (sm_h.numel() * 8 + bt_h.numel() * 4 + sl_h.numel() * 4 + (pairs_h.numel() * 8 if has_pairs else 0)
               + (qsl_h.numel() * 4 if Q > 1 else 0)
               + L * (q_h.numel() + k_h.numel() + v_h.numel()) * 2)
        d2h = L * out_h[0].numel() * 2
        e2e = {"value": round(whole_job_rate(world, step_bytes, e_ms / K * 1e-3), 2), "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e_ms / K, 4),
               "how": "CUDA graph of the step with its pinned-host copies: per layer q, k, v in (one copy) on "
                      "a copy stream and out back on another, overlapping the other layers' kernels"}
        assert pa.pa_get_device_error(clear=True) == 0

    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 (fp8 e4m3 KV cache)" if fp8 else "bf16",
        "data": "synthetic (seeded N(0,1) bf16 K/V/q; seeded shuffled free list)",
        "config": {
            "workload": WORKLOAD_TEXT.get(args.config, args.config)
                        + (f"; {Q} query rows per sequence (its last {Q} tokens, causal), pa_attention" if Q > 1
                           else ""),
            "query_rows_per_seq": Q,
            "attention_kernel": ("tcgen05" if attention_tc else "mma") if Q > 1 else None,
            "layers_per_step": L,
            "batch": S,
            "block_size": st.block_size,
            "num_blocks": st.num_blocks,
            "num_q_heads": st.num_q_heads,
            "num_kv_heads": st.num_kv_heads,
            "head_dim": st.head_dim,
            "max_seq_len": st.max_seq_len,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "kv_cache": f"fp8 e4m3, k_scale {st.k_scale}, v_scale {st.v_scale}" if fp8 else "bf16",
            "l2": f"inputs larger than L2: {L} distinct layer caches, "
                  f"{L * nbytes['decode_kv'] / 1e9:.2f} GB of KV touched per step",
            "timing": "CUDA graph of the whole step (all layers), replayed --steps times",
        },
        "pct_of_peak": {"measured": round(100 * value / world / peak, 2),
                        "nominal_8tbs": round(100 * value / world / NOMINAL_HBM_GBS, 2)},
        "decode_tokens_per_s_per_layer": round(world * S * Q / (ms_step / L * 1e-3), 1),
        "per_op_bytes_per_layer": nbytes,
        "per_op": per_op,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": None if args.part_tokens else profiled_traffic(
                         args.config, "fp8" if fp8 else "bf16" if Q == 1 else
                         f"rows{Q}" + ("_tcgen05" if attention_tc else "")),
                     "kernel": ("pa_attention" if Q > 1 else "pa_decode_fp8" if fp8 else "pa_decode")
                               + " (partition kernel"
                               + (" + LSE merge)" if split else ")"),
                     "mean_launch_us": round(dec_mean_ms * 1e3, 3),
                     "how": f"CUDA graph of {L} back-to-back {'pa_attention' if Q > 1 else 'pa_decode'} calls "
                            f"(one per layer cache), "
                            f"{K} replays timed with CUDA events on the replay stream; mean per call",
                     "bytes_per_launch": nbytes["decode_kv"], "peak_source": peak_src},
        "e2e": e2e,
        "gpu_launches": K * L * launches_per_layer,
        "clocks": clk,
    }
    return result, w


def extra_configs(args) -> list:
    """Workloads timed after the main one: by default the long-context
    decode, the second configuration the bandwidth target names, when the
    main run is the bf16 chat decode."""
    if args.extra_configs == "auto":
        default = args.config == "chat" and args.queries == 1 and args.kv_dtype == "bf16" and not args.part_tokens
        return ["long"] if default else []
    if args.extra_configs in ("", "none"):
        return []
    names = [n.strip() for n in args.extra_configs.split(",") if n.strip()]
    return [n for n in names if n != args.config]


def related_runs(args) -> list:
    """Variants of the main workload timed after it: by default the FP8
    cache's decode and 16 query rows per sequence (pa_attention), when the
    main run is the bf16 chat decode."""
    if args.related == "auto":
        default = args.config == "chat" and args.queries == 1 and args.kv_dtype == "bf16" and not args.part_tokens
        return ["fp8", "rows16"] if default else []
    if args.related in ("", "none"):
        return []
    return [n.strip() for n in args.related.split(",") if n.strip() in ("fp8", "rows16")]


def time_related(name, args, world, rank, local) -> dict:
    """The main workload with the FP8 cache (name "fp8") or with 16 query
    rows per sequence (name "rows16"), staged and timed as the main run is,
    without its end-to-end, per-op and CPU legs.  Returns the per_config
    record."""
    sub = copy.copy(args)
    sub.no_e2e, sub.no_per_op, sub.no_cpu_baseline = True, True, True
    sub.extra_configs, sub.related = "none", "none"
    if name == "fp8":
        sub.kv_dtype = "fp8"
    else:
        sub.queries = 16
    r, _ = run_ours(sub, world, rank, local)
    rec = {"workload": r["config"]["workload"]}
    for key in ("value", "unit", "ms_per_step", "dtype", "decode_tokens_per_s_per_layer", "roofline",
                "gpu_launches", "clocks"):
        if key in r:
            rec[key] = r[key]
    if "attention" in r.get("per_op", {}):
        rec["attention"] = r["per_op"]["attention"]
    rec["attention_kernel"] = r["config"].get("attention_kernel")
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


def time_decode_config(name, args, world, local) -> dict:
    """The bf16 decode step of workload `name`, staged and timed like the main
    one: --layers distinct layer caches, a CUDA graph of the whole step
    (queued copies, the KV write, pa_decode per layer) and one of the decode
    calls alone, each replayed --steps times after --warmup replays, clocks
    sampled during the step replays.  Returns the per-config record."""
    import synth
    import paged_kv_cache_333_b200 as pa
    from paged_kv_cache_333_b200.workload import stage

    dev = torch.device("cuda", local)
    w = synth.by_name(name)
    st = stage(w, dev, layers=args.layers)
    L, K = args.layers, args.steps
    nbytes = algorithmic_bytes(st)
    step_bytes = L * (nbytes["decode_kv"] + nbytes["write"] + nbytes["copy"])
    has_pairs = st.cow_pairs.shape[0] > 0
    split = st.workspace is not None

    def layer_ops(l, with_write=True):
        kc, vc = st.caches[l]
        if with_write:
            if has_pairs:
                pa.pa_copy_blocks(kc, vc, st.cow_pairs)
            pa.pa_write_kv(st.k_new, st.v_new, st.slot_mapping, kc, vc)
        pa.pa_decode(st.q, kc, vc, st.block_tables, st.seq_lens, st.scale, out=st.out,
                     max_seq_len=st.max_seq_len, workspace=st.workspace)

    for l in range(L):
        layer_ops(l)
    torch.cuda.synchronize()
    g_step = capture_graph(lambda: [layer_ops(l) for l in range(L)], dev)
    g_dec = capture_graph(lambda: [layer_ops(l, with_write=False) for l in range(L)], dev)
    for _ in range(args.warmup):
        g_step.replay()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error(clear=True) == 0
    clocks = ClockSampler(local)
    clocks.start()
    ms_total = timed_replays(g_step, K, dev, world)
    clk = clocks.stop()
    for _ in range(args.warmup):
        g_dec.replay()
    dec_ms_total = timed_replays(g_dec, K, dev, world)
    assert pa.pa_get_device_error(clear=True) == 0
    ms_step = ms_total / K
    dec_mean_ms = dec_ms_total / (K * L)
    peak, peak_src = measured_peak()
    achieved = nbytes["decode_kv"] / (dec_mean_ms * 1e-3) / 1e9
    value = whole_job_rate(world, step_bytes, ms_step * 1e-3)
    S = len(st.ids)
    rec = {
        "workload": WORKLOAD_TEXT.get(name, name),
        "batch": S, "block_size": st.block_size, "num_blocks": st.num_blocks, "max_seq_len": st.max_seq_len,
        "layers_per_step": L, "steps": K, "warmup": args.warmup,
        "value": round(value, 2), "unit": "GB/s", "ms_per_step": round(ms_step, 4),
        "decode_us_per_layer": round(dec_mean_ms * 1e3, 3),
        "decode_tokens_per_s_per_layer": round(world * S / (dec_mean_ms * 1e-3), 1),
        "pct_of_peak": {"measured": round(100 * achieved / peak, 2),
                        "nominal_8tbs": round(100 * achieved / NOMINAL_HBM_GBS, 2)},
        "per_op_bytes_per_layer": nbytes,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": profiled_traffic(name, "bf16"),
                     "kernel": "pa_decode (partition kernel" + (" + LSE merge)" if split else ")"),
                     "mean_launch_us": round(dec_mean_ms * 1e3, 3), "bytes_per_launch": nbytes["decode_kv"],
                     "how": f"CUDA graph of {L} back-to-back pa_decode calls (one per layer cache), {K} replays "
                            "timed with CUDA events on the replay stream; mean per call",
                     "peak_source": peak_src},
        "l2": f"inputs larger than L2: {L} distinct layer caches, {L * nbytes['decode_kv'] / 1e9:.2f} GB of KV "
              "touched per step",
        "gpu_launches": K * L * (2 + (1 if split else 0) + (1 if has_pairs else 0)),
        "clocks": clk,
    }
    del g_step, g_dec, st
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return rec


# --------------------------------------------------------------------------- oracle
def _oracle_setup(w):
    from tests.oracle_stage import stage_oracle
    ref = stage_oracle(w, decode=False)
    n = ref["seq_lens"]
    B = w.shape.block_size
    row = w.shape.num_kv_heads * w.shape.head_dim * 2
    pos_slots = [ref["block_tables"][s, np.arange(int(x)) // B].astype(np.int64) * B + np.arange(int(x)) % B
                 for s, x in enumerate(n)]
    uniq = np.unique(np.concatenate(pos_slots)).size
    return ref, uniq * row * 2


def _oracle_layer(w, ref, sample_seqs):
    import oracle
    which = np.array([(s, j) for s in sample_seqs for j in range(w.shape.num_q_heads)], np.int32)
    oracle.decode(w.q, ref["k_cache"], ref["v_cache"], ref["block_tables"], ref["seq_lens"], w.scale, which)


def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def _oracle_layer_threads(w, ref, pool, threads: int):
    """One layer of the oracle's decode, its (sequence, head) pairs split into
    `threads` disjoint contiguous shares, one oracle call per share on a
    worker thread.  The oracle is unchanged: a C call through ctypes, which
    releases the interpreter lock and keeps no global state, so the calls
    run in parallel on the host's cores."""
    import oracle
    pairs = np.array([(s, j) for s in range(len(w.seq_ids)) for j in range(w.shape.num_q_heads)], np.int32)
    shares = [a for a in np.array_split(pairs, threads) if len(a)]
    futs = [pool.submit(oracle.decode, w.q, ref["k_cache"], ref["v_cache"], ref["block_tables"], ref["seq_lens"],
                        w.scale, a) for a in shares]
    for f in futs:
        f.result()


def cpu_baseline(w, seconds: float) -> dict:
    """The oracle (plain C, fp64) on bounded samples of the same workload:
    whole layers, repeated until `seconds` have passed, fanned out over all
    the host's cores (the reported value), and on one thread."""
    from concurrent.futures import ThreadPoolExecutor
    ref, kv_bytes = _oracle_setup(w)
    S = len(w.seq_ids)
    cores = host_cores()

    def run(fn, budget):
        t0 = time.perf_counter()
        layers = 0
        while True:
            fn()
            layers += 1
            if time.perf_counter() - t0 >= budget:
                break
        return layers, time.perf_counter() - t0

    with ThreadPoolExecutor(max_workers=cores) as pool:
        ln, dt = run(lambda: _oracle_layer_threads(w, ref, pool, cores), seconds / 2)
    l1, dt1 = run(lambda: _oracle_layer(w, ref, range(S)), seconds / 2)
    what = f"({S} seqs x {w.shape.num_q_heads} heads), decode only"
    return {"value": round(ln * kv_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "cores_available": cores,
            "sample": f"{ln} full layer(s) of the same workload {what}, {dt:.1f} s; its (sequence, head) pairs "
                      f"split over {cores} threads, one oracle call each",
            "single_thread": {"value": round(l1 * kv_bytes / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"{l1} full layer(s) {what}, {dt1:.1f} s, one thread"}}


def run_reference(args, world, rank):
    if rank != 0:
        return
    from concurrent.futures import ThreadPoolExecutor
    import synth
    w = synth.by_name(args.config)
    ref, kv_bytes = _oracle_setup(w)
    S = len(w.seq_ids)
    cores = host_cores()
    # one step = one full layer of the workload's decode, its (sequence,
    # head) pairs split over the host's cores
    times = []
    with ThreadPoolExecutor(max_workers=cores) as pool:
        for _ in range(args.warmup):
            _oracle_layer(w, ref, range(min(S, 8)))
        for _ in range(args.steps):
            t = time.perf_counter()
            _oracle_layer_threads(w, ref, pool, cores)
            times.append(time.perf_counter() - t)
    ms_step = 1e3 * statistics.mean(times)
    value = kv_bytes / (ms_step * 1e-3) / 1e9
    sample = (f"{args.steps} steps of one full layer ({S} seqs x {w.shape.num_q_heads} heads, split over {cores} "
              "threads), decode only")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT.get(args.config, args.config), "layers_per_step": 1},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "decode_tokens_per_s_per_layer": round(S / (ms_step * 1e-3), 2),
    }), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_env()
    if world > 1 and args.impl == "ours":
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            result, w = run_ours(args, world, rank, local)
            # the other configurations the bandwidth target names, each timed
            # the same way in this process after the main one's caches are freed
            for name in extra_configs(args):
                torch.cuda.empty_cache()
                result.setdefault("per_config", {})[name] = time_decode_config(name, args, world, local)
            for name in related_runs(args):
                torch.cuda.empty_cache()
                result.setdefault("per_config", {})[name] = time_related(name, args, world, rank, local)
            if rank == 0 and world == 1 and not args.no_cpu_baseline and args.queries == 1:
                result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
            if rank == 0:
                print(json.dumps(result), flush=True)
    finally:
        if world > 1 and torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
