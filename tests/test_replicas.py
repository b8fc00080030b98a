"""The multi-GPU path is replicas only: every rank runs the whole step on its
own GPU, the device times are combined as a max over ranks, and only rank 0
prints.  These tests run that host-side plumbing as two gloo ranks on CPU."""
import datetime
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    # a short timeout: a rank whose peer is gone fails instead of waiting
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=30))
    try:
        # per-rank device times differ; the job time is the slowest rank's
        ms = bench.reduce_max(10.0 + 5.0 * rank, "cpu")
        rate = bench.whole_job_rate(world, 2e9, ms * 1e-3)
        # the reference arm prints on rank 0 only
        args = type("A", (), {"config": "tiny", "steps": 1, "warmup": 0})()
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.run_reference(args, world, rank)
        dist.barrier()
        q.put((rank, ms, rate, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_rank0_prints():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(2):
            rank, ms, rate, text = q.get(timeout=120)
            out[rank] = (ms, rate, text)
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    finally:
        for p in procs:  # the workers this test started, if any is still running
            if p.is_alive():
                p.terminate()
                p.join(timeout=10)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] == pytest.approx(2 * 2e9 / 15e-3 / 1e9)
    line = json.loads(out[0][2])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert out[1][2] == ""


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.reduce_max(3.5, "cpu") == 3.5
    assert bench.whole_job_rate(1, 1e9, 1.0) == 1.0
