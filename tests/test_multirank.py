"""The multi-process host logic of bench.py on the CPU (gloo, world size 2).

Under torchrun every rank runs the same step on its own GPU and rank 0 prints
one line whose times are the maximum over ranks; the reference arm runs on
rank 0 only while the other ranks exit cleanly.  Neither needs a GPU to check.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # rank r reports times (r + 1.5, 10 - r): the maximum is taken per entry
        got = bench.max_over_ranks([rank + 1.5, 10.0 - rank], dist, torch.device("cpu"))
        results[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_takes_each_entry_from_the_slowest_rank():
    world = 2
    with mp.Manager() as manager:
        results = manager.dict()
        mp.spawn(_max_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        got = dict(results)
    assert got[0] == got[1] == [2.5, 10.0]


def test_max_over_ranks_without_a_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3, 4.5], None, torch.device("cpu")) == [3.0, 4.5]


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero(oracle_lib):
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["sample"].startswith("the whole tiny step")


def test_reference_arm_falls_back_to_a_sample_beyond_its_budget(oracle_lib):
    """With a budget too small for the whole step, each step is the first
    sequences of the workload, and the line says so."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
           "--warmup", "3", "--workload", "ragged", "--ref-budget-s", "0.01"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][0])
    assert line["cpu_baseline"]["sample"].startswith("first 1 of 64 sequences of ragged")
    assert line["config"]["workload"] == "ragged"


@pytest.mark.parametrize("steps,copies", [(200, 4), (201, 4), (3, 4), (1, 2), (7, 3), (0, 4)])
def test_timed_region_replays_exactly_k_steps(steps, copies):
    """The step region replays graphs of `copies` steps and then one-step
    graphs: exactly K steps, each KV copy in turn."""
    sys.path.insert(0, ROOT)
    import bench
    seen = []
    n = bench.replay_steps(steps, copies, lambda: seen.extend(range(copies)),
                           [lambda c=c: seen.append(c) for c in range(copies)])
    assert n == steps == len(seen)
    assert seen == [k % copies for k in range(steps)]
