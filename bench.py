"""Benchmark of one MLRA decode step on B200: KV-cache read GB/s.

A step is the whole hot path on one batch: split-KV decode attention with its
log-sum-exp merge (mlra_decode, one kernel: paged gather, per-branch scores
against the branch latent plus the shared RoPE key, per-(head, branch)
softmax, value-absorbed output, split merge, out_scale) followed by the
per-branch W_UV up-projection and branch sum (mlra_up_proj, one kernel).

value: algorithmic KV bytes of all ranks' steps / device time (GB/s), the
KV cache resident in HBM, the steps replayed from a CUDA graph holding one
step (both kernels) per KV copy.
L2 cannot serve the cache: each step reads the next of k copies of the
pools, k * KV bytes >= 4x the L2 size.
roofline: the decode kernel alone, a graph of back-to-back decode launches
(one per KV copy, same rotation) replayed until at least K launches, CUDA
events around the region, algorithmic KV bytes / mean duration per launch.
e2e: the same metric through the public Python API (DecodeStep: one graph
launch per step) with the step's inputs (queries, block table, seqlens)
brought in from pinned host memory (one mlra_copy_ranges launch) and the
result y written back into pinned host memory by the up-projection, inside
the timed region, one host synchronisation per step.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
       [--impl ours|reference]
Under torchrun every rank runs the same workload on its own GPU (replicas,
weak scaling); rank 0 prints one JSON line.  --impl reference times the fp64
CPU oracle on the same workload on the host cores (the whole step unless
W + K steps would exceed --ref-budget-s, then the first sequences).
workloads (one GPU): the decode kernel alone on the other decode workloads,
timed like the roofline region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from branch_latent_kv_b200 import binding as b  # noqa: E402
from branch_latent_kv_b200.inputs import WORKLOADS, make_inputs  # noqa: E402
from branch_latent_kv_b200.step import DecodeStep  # noqa: E402

METRIC = "MLRA decode-attention KV GB/s and tokens/s at 1 B200; % of HBM roofline"
# The other decode workloads whose decode-kernel figures ride along in the
# line (the step itself is timed on --workload).
OTHER_WORKLOADS = ["long_context", "ragged", "mla_equal_bytes", "mlra4_equal_bytes", "tp_shard",
                   "mlra2_equal_bytes", "context_2m", "heads_64"]
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic of the decode split kernel per launch on decode_2p9b, from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the
# hash of the kernel sources it was taken on.  Reported as null whenever the
# kernel sources differ from the captured ones.
TRAFFIC_CAPTURE = {"workload": "decode_2p9b", "sources_sha1": "986c9c488856f853531d268efd1ab4d111935fab",
                   "bytes_per_launch": 151393280 + 3135232}
KERNEL_SOURCES = ["branch_latent_kv_b200/csrc/decode_tc.cu", "branch_latent_kv_b200/csrc/sm100.cuh",
                  "branch_latent_kv_b200/csrc/common.cuh"]


def kernel_sources_sha1() -> str:
    h = hashlib.sha1()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is busy."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 100):
        self.gpu_index, self.period_ms = gpu_index, period_ms
        self.proc, self.lines, self.thread = None, [], None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", f"-lms={self.period_ms}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)

    def summary(self, t0=None, t1=None):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if t0 is not None and not (t0 <= ts <= t1):
                continue
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def replay_steps(steps, copies, chain_replay, step_replays):
    """Replay exactly `steps` steps: whole graphs of `copies` steps (one per
    KV copy), then the remainder as one-step graphs.  Returns the count."""
    n_chain, n_rest = divmod(steps, copies)
    for _ in range(n_chain):
        chain_replay()
    for k in range(n_rest):
        step_replays[k]()
    return n_chain * copies + n_rest


def max_over_ranks(values, dist, device):
    """Element-wise max of a list of floats over all ranks (a no-op without a
    process group)."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def kv_bytes_of(x) -> int:
    return x.kv_bytes


def reference_inputs(w, n_seqs=None):
    """The workload's inputs on the host (all sequences, or the first n_seqs)."""
    if n_seqs is None or n_seqs >= w.batch:
        return make_inputs(w, with_w_uv=True)
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    from branch_latent_kv_b200.inputs import draw_seqlens
    seqlens = draw_seqlens(w, gen)[:n_seqs]
    ws = w.with_(batch=int(seqlens.numel()), seqlen=None, seqlen_range=None)
    return make_inputs(ws, seqlens=seqlens, with_w_uv=True)


def l2_copies(kv_bytes):
    """KV copies the GPU arm rotates over so that L2 cannot serve the cache."""
    l2 = 126 * 1024 * 1024
    if torch.cuda.is_available():
        l2 = torch.cuda.get_device_properties(0).L2_cache_size
    return max(2, math.ceil(4 * l2 / kv_bytes))


def run_reference(args, world, rank):
    """The fp64 oracle on the host cores, each step the whole workload
    (decode + up-projection of every sequence), unless W + K such steps
    would take longer than --ref-budget-s: then each step is the first
    sequences of the workload, as many as fit."""
    if rank != 0:
        return
    from oracle import oracle
    w = WORKLOADS[args.workload]
    threads = len(os.sched_getaffinity(0))
    oracle.set_num_threads(threads)
    x = reference_inputs(w)

    def make_step(xx):
        def step():
            out, _, _ = oracle.decode(xx.q_lat, xx.q_rope, xx.latent_cache, xx.rope_cache, xx.block_table,
                                      xx.seqlens, xx.scale, xx.out_scale)
            oracle.up_proj(out, xx.w_uv, w.d_h)
        return step

    step = make_step(x)
    t0 = time.perf_counter()
    step()
    one = time.perf_counter() - t0
    n_steps = args.steps + max(args.warmup - 1, 0)
    if one * n_steps > args.ref_budget_s:
        keep = max(1, int(w.batch * args.ref_budget_s / (one * n_steps)))
        x = reference_inputs(w, keep)
        step = make_step(x)
    for _ in range(max(args.warmup - 1, 0)):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    kv = x.kv_bytes
    gbs = kv * args.steps / dt / 1e9
    n = x.workload.batch
    sample = (f"the whole {w.name} step (all {w.batch} sequences, {int(x.seqlens.sum())} tokens), "
              f"decode + up-projection" if n == w.batch else
              f"first {n} of {w.batch} sequences of {w.name} ({int(x.seqlens.sum())} tokens), "
              f"decode + up-projection per step")
    gen = torch.Generator(device="cpu").manual_seed(w.seed)
    from branch_latent_kv_b200.inputs import draw_seqlens
    full_kv = int(draw_seqlens(w, gen).to(torch.int64).sum()) * (w.branches * w.d_c + w.d_r) * 2
    line = {"impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, l2_copies(full_kv)),
            "tokens_per_s": n * args.steps / dt,
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def prestep_time_us(x, w, dev, stream, steps):
    """Mean duration of mlra_prepare on the workload's batch: CUDA events
    around replays of a graph of 20 back-to-back launches, after warm-up."""
    g = torch.Generator(device="cpu").manual_seed(w.seed + 1)
    N, H, B, d_c = x.q_lat.shape
    d_r, d_h = x.q_rope.shape[2], w.d_h

    def draw(shape, fan):
        return (torch.randn(shape, generator=g) / math.sqrt(fan)).to(torch.bfloat16).to(dev)
    q_c, q_r, w_uk = draw((N, H, d_h), d_h), draw((N, H, d_r), d_r), draw((B, H, d_h, d_c), d_h)
    c_new, kr_new = draw((N, B, d_c), d_c), draw((N, d_r), d_r)
    q_lat, q_rope = torch.empty_like(x.q_lat), torch.empty_like(x.q_rope)
    lat, rope = x.latent_cache.clone(), x.rope_cache.clone()  # the pre-step writes one row per sequence

    def call(st):
        b.mlra_prepare(q_c, q_r, w_uk, c_new, kr_new, x.seqlens, x.block_table, lat, rope,
                       q_lat=q_lat, q_rope=q_rope, stream=st)
    for _ in range(3):
        call(stream)
    # a few microseconds of kernel: 20 launches per graph replay so that the
    # host's replay path does not starve the GPU between launches
    per_graph = 20
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        for _ in range(per_graph):
            call(cap)
    torch.cuda.synchronize(dev)
    for _ in range(3):
        graph.replay()
    reps = max(1, steps // per_graph)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    del lat, rope
    return e0.elapsed_time(e1) / (reps * per_graph) * 1e3


def decode_only_figure(name, dev, stream, hbm_peak, min_launches=24):
    """The decode kernel alone on another workload, timed like the roofline
    region: a graph of one decode launch per KV copy (copies * KV bytes >= 4x
    L2), replayed until at least min_launches launches, CUDA events around the
    region."""
    w = WORKLOADS[name]
    x = make_inputs(w, device=str(dev), with_w_uv=False)
    kv = x.kv_bytes
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(2, math.ceil(4 * l2 / kv))
    lat = [x.latent_cache] + [x.latent_cache.clone() for _ in range(copies - 1)]
    rope = [x.rope_cache] + [x.rope_cache.clone() for _ in range(copies - 1)]
    dims = b.decode_dims(x.q_lat, x.q_rope, x.latent_cache, x.block_table)
    ws = torch.zeros(b.mlra_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    out = torch.empty_like(x.q_lat)

    def call(i, st):
        b.mlra_decode(x.q_lat, x.q_rope, lat[i], rope[i], x.block_table, x.seqlens, x.scale, x.out_scale,
                      out=out, workspace=ws, stream=st)
    call(0, stream)
    torch.cuda.synchronize(dev)
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for c in range(copies):
            call(c, cap)
    torch.cuda.synchronize(dev)
    for _ in range(3):
        g.replay()
    reps = -(-min_launches // copies)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    e0.record(stream)
    for _ in range(reps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    us = e0.elapsed_time(e1) / (reps * copies) * 1e3
    err = b.mlra_read_device_error(ws)
    if err != 0:
        raise RuntimeError(f"device error on {name}: {b.mlra_status_string(err)}")
    del g
    gbs = kv / (us * 1e-6) / 1e9
    return {"tokens": int(x.seqlens.to(torch.int64).sum()), "kv_bytes_per_launch": kv,
            "us_per_launch": us, "decode_gbs": gbs, "frac": gbs / hbm_peak,
            "launches": reps * copies, "kv_copies": copies}, (t0, t1)


def workload_config(w, copies):
    cfg = {"workload": w.name, "batch": w.batch, "heads": w.heads, "branches": w.branches,
           "d_c": w.d_c, "d_r": w.d_r, "page_size": w.page_size, "d_h": w.d_h,
           "seq_len": w.seqlen if w.seqlen is not None else f"U{{{w.seqlen_range[0]}..{w.seqlen_range[1]}}}",
           "page_order": w.page_order, "parallelism": "replicas (one independent step per GPU)",
           "step": "mlra_decode_up_proj (one launch: split-KV attention, in-kernel LSE merge, per-branch "
                   "W_UV up-projection and branch sum); batch > 64: mlra_decode + mlra_up_proj"}
    if copies is not None:
        cfg["l2"] = f"inputs larger than L2: {copies} rotating copies of the KV pools"
    return cfg


def cpu_baseline(w, x_dev, min_seconds=3.0):
    """The oracle on the whole step of the workload (decode + up-projection of
    every sequence), repeated for at least min_seconds on all host cores."""
    from oracle import oracle
    threads = len(os.sched_getaffinity(0))
    oracle.set_num_threads(threads)
    host = [t.cpu() for t in (x_dev.q_lat, x_dev.q_rope, x_dev.latent_cache, x_dev.rope_cache,
                              x_dev.block_table, x_dev.seqlens)]
    w_uv = x_dev.w_uv.cpu()
    reps, t0 = 0, time.perf_counter()
    while True:
        out, _, _ = oracle.decode(*host, x_dev.scale, x_dev.out_scale)
        oracle.up_proj(out, w_uv, w.d_h)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    return {"value": x_dev.kv_bytes * reps / dt / 1e9, "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"the whole {w.name} step (all {w.batch} sequences, decode + up-projection), "
                      f"{reps} repetitions in {dt:.1f} s"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode_2p9b", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-budget-s", type=float, default=150.0,
                    help="reference arm: longest oracle run before it falls back to a sample")
    ap.add_argument("--workloads", default=",".join(OTHER_WORKLOADS),
                    help="decode-kernel figures of these workloads in the line ('' for none)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--two-kernel-step", action="store_true",
                    help="time the step as mlra_decode + mlra_up_proj (two launches) instead of the fused launch")
    ap.add_argument("--profile", action="store_true",
                    help="run W + K device-resident steps only and print nothing (for profilers)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup()

    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    b.library()
    w = WORKLOADS[args.workload]
    x = make_inputs(w, device=str(dev))
    kv = x.kv_bytes
    tokens = w.batch
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(2, math.ceil(4 * l2 / kv))
    lat = [x.latent_cache] + [x.latent_cache.clone() for _ in range(copies - 1)]
    rope = [x.rope_cache] + [x.rope_cache.clone() for _ in range(copies - 1)]
    dims = b.decode_dims(x.q_lat, x.q_rope, x.latent_cache, x.block_table)
    ws = torch.zeros(b.mlra_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    out = torch.empty_like(x.q_lat)
    y = torch.empty((w.batch, w.heads * w.d_h), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def decode_call(i):
        b.mlra_decode(x.q_lat, x.q_rope, lat[i % copies], rope[i % copies], x.block_table,
                      x.seqlens, x.scale, x.out_scale, out=out, workspace=ws)

    def up_call():
        b.mlra_up_proj(out, x.w_uv, y=y)

    # the step: one launch of the fused decode + up-projection where it covers
    # the shape (batch <= 64), else the two kernels
    fused = w.batch <= 64 and not args.two_kernel_step

    def step(i):
        if fused:
            b.mlra_decode_up_proj(x.q_lat, x.q_rope, lat[i % copies], rope[i % copies], x.block_table,
                                  x.seqlens, x.scale, x.out_scale, x.w_uv, out=out, y=y, workspace=ws)
        else:
            decode_call(i)
            up_call()

    if args.profile:
        for i in range(args.warmup + args.steps):
            step(i)
        torch.cuda.synchronize(dev)
        if pg:
            pg.destroy_process_group()
        return

    # The device-resident steps are replayed from CUDA graphs.  One graph
    # holds one step per KV copy (`copies` steps, both kernels each), the way
    # a serving loop launches its kernels back to back from a graph rather
    # than one graph launch per kernel; within a step the up-projection
    # (launched as a programmatic dependent) loads its weights on SMs the
    # decode kernel has released while the decode kernel finishes.  Steps
    # left over when K is not a multiple of `copies` replay one-step graphs.
    # The decode kernel's own duration (the roofline figure) is timed in a
    # second region: a graph of `copies` decode launches, replayed until at
    # least K launches, events around the region, divided by the launches.
    step(0)
    torch.cuda.synchronize(dev)
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    step_graphs = []
    for c in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            step(c)
        step_graphs.append(g)
    chain_steps, chain_decode = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(chain_steps, stream=cap):
        for c in range(copies):
            step(c)
    with torch.cuda.graph(chain_decode, stream=cap):
        for c in range(copies):
            decode_call(c)
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(local)
    sampler.start()
    # warm-up: at least W steps and ~1.5 s of load so the clock sampler sees it
    t_warm = time.time()
    i = 0
    while i < args.warmup or time.time() - t_warm < 1.5:
        chain_steps.replay()
        i += copies
        if i % 256 < copies:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    replay_steps(args.steps, copies, chain_steps.replay, [g.replay for g in step_graphs])
    end.record(stream)
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    elapsed_ms = start.elapsed_time(end)
    # decode kernel alone: at least K launches, events around the region
    reps = -(-args.steps // copies)
    d_start, d_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d_start.record(stream)
    for _ in range(reps):
        chain_decode.replay()
    d_end.record(stream)
    torch.cuda.synchronize(dev)
    t_load1 = time.time()
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    decode_launches = reps * copies
    decode_ms = d_start.elapsed_time(d_end) / decode_launches
    elapsed_ms, decode_ms = max_over_ranks([elapsed_ms, decode_ms], pg, dev)
    del step_graphs, chain_steps, chain_decode

    # end to end through the public API, host buffers: a DecodeStep per KV
    # copy (the same bound device inputs), each step one graph launch that
    # reads the inputs from pinned host memory (one copy launch), runs both
    # kernels and writes y into pinned host memory; the host waits for every
    # step
    h_in = {"q_lat": x.q_lat.cpu().pin_memory(), "q_rope": x.q_rope.cpu().pin_memory(),
            "block_table": x.block_table.cpu().pin_memory(), "seqlens": x.seqlens.cpu().pin_memory()}
    h_y = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    d_in = {k: torch.empty_like(v, device=dev) for k, v in h_in.items()}
    for k in d_in:
        d_in[k].copy_(h_in[k])
    steps_e2e = [DecodeStep(d_in["q_lat"], d_in["q_rope"], lat[c], rope[c], d_in["block_table"],
                            d_in["seqlens"], x.scale, x.out_scale, w_uv=x.w_uv, host_inputs=h_in,
                            host_output=h_y) for c in range(copies)]
    h2d, d2h = steps_e2e[0].h2d_bytes(), steps_e2e[0].d2h_bytes()

    def e2e_step(i):
        steps_e2e[i % copies]()
        stream.synchronize()

    for k in range(args.warmup):
        e2e_step(k)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for k in range(args.steps):
        e2e_step(k)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms, = max_over_ranks([e_start.elapsed_time(e_end)], pg, dev)

    # the decode pre-step (query absorption, rotary embedding, append) on the
    # same batch, its own timed loop: events around each launch
    pre_us = prestep_time_us(x, w, dev, stream, args.steps)

    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    # the decode kernel alone on the other workloads (one GPU runs only)
    others = {}
    names = [n for n in args.workloads.split(",") if n and n != args.workload] if world == 1 else []
    if names:
        del steps_e2e, lat, rope
        torch.cuda.empty_cache()
    for name in names:
        fig, (t0, t1) = decode_only_figure(name, dev, stream, hbm_peak)
        fig["sm_mhz"] = sampler.summary(t0, t1)["sm_mhz"]
        others[name] = fig
        torch.cuda.empty_cache()
    sampler.stop()

    err = b.mlra_read_device_error(ws)
    if err != 0:
        raise RuntimeError(f"device error during the benchmark: {b.mlra_status_string(err)}")

    clocks = sampler.summary(t_warm, t_load1)
    gbs = kv * world * args.steps / (elapsed_ms / 1e3) / 1e9
    achieved = kv / (decode_ms / 1e3) / 1e9
    traffic = None
    if TRAFFIC_CAPTURE["workload"] == args.workload and TRAFFIC_CAPTURE["sources_sha1"] == kernel_sources_sha1():
        traffic = TRAFFIC_CAPTURE["bytes_per_launch"]
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, copies),
        "tokens_per_s": tokens * world * args.steps / (elapsed_ms / 1e3),
        "hbm_roofline_frac": gbs / world / hbm_peak,
        "kv_bytes_per_step": kv,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "kernel": "decode_tc_kernel (mlra_decode: split-KV decode with its in-kernel "
                               "LSE merge), CUDA events around a region of >= K back-to-back decode "
                               "launches (graphs of one launch per KV copy) timed after the step "
                               "region, same KV rotation",
                     "peak_source": f"{peak_kind} hbm_gbs"},
        "e2e": {"value": kv * world * args.steps / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        # per step: the fused decode + up-projection kernel, or the two kernels
        "gpu_launches": (1 if fused else 2) * args.steps,
        "prestep": {"kernel": "prepare_kernel (mlra_prepare: query absorption, rotary embedding, "
                              "append of the new token)", "us_per_launch": pre_us,
                    "note": "not part of the step above; timed in its own loop on the same batch "
                            "(back-to-back launches in a graph)"},
        "clocks": clocks,
    }
    if others:
        line["workloads"] = {
            "what": "decode kernel alone (mlra_decode) on the other decode workloads: graphs of one "
                    "launch per KV copy (copies x KV bytes >= 4x L2) replayed back to back, CUDA events "
                    "around >= 24 launches; frac = decode_gbs / the same measured peak",
            **others}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, x)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
