"""Benchmark of the GSA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one full decode step (routing scores, top-k, unfolding, hybrid
attention) for the whole batch of the workload, through gsa_decode_step.
The default workload is the Llama-3-8B-shaped decode layer (batch 8, 32 query
/ 8 KV heads, d 128, 32768 raw tokens in chunks of 16, top-k 16, tail 64,
bf16).  Inputs are synthetic (seeded normals with planted needle chunks).

Device timing: the K timed steps are one CUDA graph that rotates over L
layer replicas whose bytes touched per rotation exceed 4x the L2 size, timed
with CUDA events on the launching stream, max over ranks.  e2e: the same K
steps through the C ABI from Python with the step's query copied host->device
from pinned memory and the result copied back every step.

With --gpus N > 1 (torchrun, one process per GPU) every rank runs its own
replica set (the path shards by independent sequences; no collective on the
data path), so scaling is weak and `value` is the steps of all ranks divided
by the slowest rank's time.

--impl reference times the CPU oracle (fp64, OpenMP over rows) on the host
cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "GSA decode steps/sec (batch×heads) and achieved HBM GB/s as % of B200 peak"


def algorithmic_bytes(s: synth.DecodeShape) -> int:
    """Bytes a decode step must move: q, every gist key, gist values (all or
    the selected ones), raw K/V of the selected chunks, tail K/V, output."""
    e = 4 if s.dtype == "f32" else 2
    row = s.head_dim * e
    per_kv = s.n_chunks * row                                           # gist keys
    per_kv += (s.n_chunks if s.mode == synth.ALL_GISTS else s.top_k) * row   # gist values
    per_kv += 2 * s.top_k * s.chunk * row                               # unfolded raw K, V
    per_kv += 2 * s.tail_len * row                                      # tail K, V
    return s.rows * per_kv + 2 * s.batch * s.n_q_heads * row            # + q and out


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


KERNEL_SOURCES = ("gsa_fused.cu", "gsa_fused.h", "gsa_device.cuh", "gsa_tc.cuh")


def measured_traffic(workload: str):
    """DRAM bytes per launch of the decode step from a committed ncu summary
    under profiles/, or None when none covers this workload or the kernel
    sources have changed since the counters were taken."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "kv_cache_routing_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    digest = h.hexdigest()
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        kv = {}
        for line in open(path):
            if ":" in line and not line.startswith(("#", "|", "-", " ")):
                k, _, v = line.partition(":")
                kv[k.strip()] = v.strip()
        if kv.get("workload") == workload and kv.get("sources_sha256") == digest:
            try:
                return int(kv["dram_bytes_per_step"]) / int(kv["launches_per_step"])
            except (KeyError, ValueError):
                return None
    return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            self.proc.wait(timeout=5)

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun env).  Only the barrier and the timing
    reduction use the process group; the data path has no collective."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank value (device time) over all ranks."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(steps_per_rank: int, world: int, ms_max: float) -> float:
    """Steps of all ranks divided by the slowest rank's time (weak scaling)."""
    return world * steps_per_rank / (ms_max / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- ours ----
def run_ours(args, world, rank, local):
    import torch

    import kv_cache_routing_b200 as gsa
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from gsa_check import desc_of, dev, tdtype

    s = synth.WORKLOADS[args.workload]
    torch.cuda.set_device(local)
    dev_props = torch.cuda.get_device_properties(local)
    l2 = dev_props.L2_cache_size
    nbytes_step = algorithmic_bytes(s)
    L = max(2, -(-4 * l2 // nbytes_step))                 # replicas: touched bytes per rotation >= 4 x L2
    if args.replicas:
        L = args.replicas
    x = synth.decode_inputs(s, synth.seed_for(args.workload) + 17 * rank)
    base = {k: dev(v) for k, v in x.tensors().items()}
    reps = []
    for r in range(L):
        t = {k: (v if r == 0 else v.clone()) for k, v in base.items()}
        if r:
            # a distinct query per replica (distinct selections); caches are separate copies
            qn = synth.normal(synth.seed_for(args.workload) + 1000 * r + rank, synth.S_Q, x.q.shape, s.dtype)
            t["q"] = dev(qn)
        reps.append(t)
    desc = desc_of(s)
    wsz = gsa.gsa_decode_workspace_size(desc)
    launches = gsa.gsa_decode_launch_count(desc)
    outs = [torch.empty((s.batch, s.n_q_heads, s.head_dim), dtype=tdtype(s.dtype), device="cuda") for _ in range(L)]
    idxs = [torch.empty((s.batch, s.n_kv_heads, s.top_k), dtype=torch.int32, device="cuda") for _ in range(L)]
    ws = torch.zeros(wsz, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    def step(i, st):
        t = reps[i % L]
        gsa.gsa_decode_step(desc, t["q"], t["k_gist"], t["v_gist"], t["k_raw"], t["v_raw"], t["k_tail"],
                            t["v_tail"], idxs[i % L], None, outs[i % L], ws, stream=st)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, stream)
    stream.synchronize()
    # K timed steps captured as one graph
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(args.steps):
                step(i, stream)
    with torch.cuda.stream(stream):
        g.replay()                                   # untimed replay: instantiate / warm the graph
    stream.synchronize()
    assert gsa.gsa_workspace_error(ws, stream=stream) == 0

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world)
    clocks = clk.summary()

    # e2e through the C ABI: per step, H2D of the query from pinned memory,
    # the decode step, D2H of the output and the selection.
    q_host = [torch.empty_like(reps[r]["q"], device="cpu").pin_memory() for r in range(L)]
    for r in range(L):
        q_host[r].copy_(reps[r]["q"].cpu())
    out_host = torch.empty_like(outs[0], device="cpu").pin_memory()
    idx_host = torch.empty_like(idxs[0], device="cpu").pin_memory()
    q_dev = [reps[r]["q"] for r in range(L)]
    barrier(world)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for i in range(args.steps):
            r = i % L
            q_dev[r].copy_(q_host[r], non_blocking=True)
            step(i, stream)
            out_host.copy_(outs[r], non_blocking=True)
            idx_host.copy_(idxs[r], non_blocking=True)
            stream.synchronize()                     # the host reads the step's result
        f1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world)

    per_step_ms = ms_max / args.steps
    steps_per_s = whole_job_rate(args.steps, world, ms_max)
    gbs = nbytes_step / (per_step_ms / 1e3) / 1e9
    peak, peak_kind = peaks()
    line = {
        "metric": METRIC,
        "value": round(steps_per_s, 2),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(per_step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": s.dtype,
        "data": "synthetic",
        "config": {"workload": args.workload, "batch": s.batch, "n_q_heads": s.n_q_heads,
                   "n_kv_heads": s.n_kv_heads, "head_dim": s.head_dim, "raw_tokens": s.n_chunks * s.chunk,
                   "chunk": s.chunk, "n_gists": s.n_chunks, "top_k": s.top_k, "tail": s.tail_len,
                   "mode": "ALL_GISTS" if s.mode == synth.ALL_GISTS else "SELECTED_PAIRS",
                   "parallelism": f"replicas x{world}",
                   "l2": f"rotating {L} layer replicas, {L * nbytes_step / 1e6:.0f} MB touched per rotation "
                         f"(L2 {l2 / 1e6:.0f} MB)"},
        "head_steps_per_s": round(steps_per_s * s.batch * s.n_q_heads, 1),
        "algorithmic_bytes_per_step": nbytes_step,
        "roofline": {"bound": "hbm",
                     "kernel": f"gsa_decode_step: {launches} launches per step of one kernel "
                               f"(per launch: half the step's algorithmic bytes in half the step's time)",
                     "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s", "frac": round(gbs / peak, 4),
                     "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": nbytes_step / launches,
                     "traffic": measured_traffic(args.workload)},
        "e2e": {"value": round(whole_job_rate(args.steps, world, e2e_ms), 2), "unit": "steps/s",
                "h2d_bytes_per_step": q_host[0].numel() * q_host[0].element_size(),
                "d2h_bytes_per_step": out_host.numel() * out_host.element_size()
                + idx_host.numel() * idx_host.element_size()},
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(s, x, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g


# ------------------------------------------------------------ CPU oracle ----
def cpu_baseline(s, x, budget_s: float):
    """The fp64 oracle, as it stands, on the host cores: whole decode steps of
    the same workload until the time budget is spent (at least one)."""
    import oracle
    t = x.tensors()
    oracle.decode(t, s.top_k, s.mode)  # load + warm
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.decode(t, s.top_k, s.mode)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(n / el, 4), "unit": "steps/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} full decode steps of the workload ({s.rows} (batch, kv-head) rows each), "
                      f"fp64, OpenMP over rows, {el:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    s = synth.WORKLOADS[args.workload]
    x = synth.decode_inputs(s, synth.seed_for(args.workload))
    import oracle
    t = x.tensors()
    oracle.decode(t, s.top_k, s.mode)
    times = []
    for _ in range(args.warmup):
        oracle.decode(t, s.top_k, s.mode)
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.decode(t, s.top_k, s.mode)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    v = args.steps / total
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "batch": s.batch, "n_q_heads": s.n_q_heads,
                       "n_kv_heads": s.n_kv_heads, "head_dim": s.head_dim, "raw_tokens": s.n_chunks * s.chunk,
                       "top_k": s.top_k, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(v, 4), "unit": "steps/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} full decode steps, fp64 oracle, OpenMP over "
                                       f"{s.rows} rows"},
            "e2e": {"value": round(v, 4), "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama8b_decode",
                    choices=[k for k, v in synth.WORKLOADS.items() if isinstance(v, synth.DecodeShape)])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--replicas", type=int, default=0,
                    help="layer replicas to rotate over (default: enough to exceed 4x L2); 1 for profiling captures")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
