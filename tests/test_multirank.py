"""The multi-rank host logic of bench.py on CPU (gloo, world size 2).

bench.py --gpus N runs one independent replica per GPU: no collective on the
data path, only the timing reduction (each rank's times, maximum over ranks)
and rank 0 printing the one JSON line. These checks run that logic with two
gloo ranks on the host, and launch the reference arm under torch.distributed.run
with two ranks (rank 0 alone works and prints).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        got = bench._max_over_ranks([1.0 + rank, 10.0 - rank, 3.5], world, "cpu")
        out.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_times_reduce_to_the_slowest_rank_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0, 3.5]


def test_single_rank_needs_no_process_group():
    assert bench._max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]


def test_job_value_is_weak_scaling_aggregate():
    # two ranks, 1000 tokens per step each, 10 steps in 2000 ms (slowest rank)
    assert bench._job_value(2, 1000.0, 10, 2000.0) == pytest.approx(10000.0)
    assert bench._job_value(1, 1000.0, 10, 2000.0) == pytest.approx(5000.0)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "tiny"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0


def test_prefill_reference_arm_prints_its_metric():
    # the oracle arm of the prefill workload (batch shrunk to keep the CPU sample short)
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "prefill", "--batch", "1", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "query-tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["config"]["batch"] == 1
