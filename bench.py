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
steps through the C ABI from Python, each one gsa_decode_step_host call (the
query copied host->device from pinned memory, the step, the output and the
selection copied back) followed by a wait for the result.

With --gpus N > 1 (torchrun, one process per GPU) every rank runs its own
replica set (the path shards by independent sequences; no collective on the
data path), so scaling is weak and `value` is the steps of all ranks divided
by the slowest rank's time.

--impl reference times the CPU oracle (fp64, OpenMP over rows) on the host
cores on a bounded sample of the same workload.

Other workloads: --workload NAME for every decode shape of synth.WORKLOADS
(the sweeps), llama8b_paged (the same step over a shared page pool of
documents through gsa_decode_step_paged), hier_1m (two-level descent, steps/s
against the HBM roofline), hier3_1m (three-level descent through
gsa_levels_decode) and suffix_stage2 (the stage-2 selective-finetuning
forward over a 512-token suffix, positions/s and algorithmic TFLOP/s) and gist_prefill (the gist-causal prefill,
algorithmic TFLOP/s against the bf16 tensor roofline).
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


def paged_bytes(ps: synth.PagedShape, seq_chunks: np.ndarray) -> int:
    """algorithmic_bytes with each sequence's own chunk count nb: nb gist
    keys (and values), the raw K/V of min(k, nb) chunks, the tail."""
    s = ps.base
    e = 4 if s.dtype == "f32" else 2
    row = s.head_dim * e
    total = 2 * s.batch * s.n_q_heads * row
    for nb in seq_chunks.tolist():
        kk = min(s.top_k, nb)
        per_kv = nb * row + (nb if s.mode == synth.ALL_GISTS else kk) * row + 2 * kk * s.chunk * row
        total += s.n_kv_heads * (per_kv + 2 * s.tail_len * row)
    return total


MODE_NAMES = {synth.ALL_GISTS: "ALL_GISTS", synth.SELECTED_PAIRS: "SELECTED_PAIRS", synth.SR_ONLY: "SR_ONLY",
              synth.UNSELECTED_GISTS: "UNSELECTED_GISTS"}


def _dev(a: np.ndarray):
    """Host array -> device tensor (bf16 bit patterns become torch.bfloat16)."""
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def _tdtype(dt: str):
    import torch
    return torch.float32 if dt == "f32" else torch.bfloat16


def _desc_of(s):
    import kv_cache_routing_b200 as gsa
    return gsa.decode_desc(s.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, s.n_chunks, s.chunk, s.top_k,
                           s.tail_len, gsa.GSA_F32 if s.dtype == "f32" else gsa.GSA_BF16, s.mode, s.scale)


B200_L2_BYTES = 132644864   # reported by the device; used for the replica count when no GPU is visible


def l2_bytes(local: int = 0) -> int:
    try:
        import torch
        if torch.cuda.is_available():
            return int(torch.cuda.get_device_properties(local).L2_cache_size)
    except Exception:
        pass
    return B200_L2_BYTES


def replicas_for(nbytes_step: int, l2: int, override: int = 0) -> int:
    """Layer replicas to rotate over so that one rotation touches >= 4x L2."""
    return override if override else max(2, -(-4 * l2 // nbytes_step))


def decode_config(s, workload: str, world: int, L: int, nbytes_step: int, l2: int) -> dict:
    """The `config` of a flat decode line (both arms print the same one)."""
    return {"workload": workload, "batch": s.batch, "n_q_heads": s.n_q_heads, "n_kv_heads": s.n_kv_heads,
            "head_dim": s.head_dim, "raw_tokens": s.n_chunks * s.chunk, "chunk": s.chunk, "n_gists": s.n_chunks,
            "top_k": s.top_k, "tail": s.tail_len, "mode": MODE_NAMES[s.mode],
            "parallelism": f"replicas x{world}",
            "l2": f"rotating {L} layer replicas, {L * nbytes_step / 1e6:.0f} MB touched per rotation "
                  f"(L2 {l2 / 1e6:.0f} MB)"}


def paged_config(ps, x, workload: str, world: int, L: int, nbytes_step: int, l2: int) -> dict:
    c = decode_config(ps.base, workload, world, L, nbytes_step, l2)
    c.update({"n_pages": int(x.k_pages.shape[0]), "n_docs": ps.n_docs,
              "doc_chunks": f"{ps.doc_min}..{ps.doc_max}",
              "seq_chunks_mean": round(float(np.mean(x.seq_chunks)), 1),
              "pages_shared": int(x.table[x.table >= 0].size - np.unique(x.table[x.table >= 0]).size)})
    return c


def hier_config(h, workload: str, world: int, L: int, nbytes: int, l2: int) -> dict:
    s = h.l1
    return {"workload": workload, "batch": s.batch, "n_q_heads": s.n_q_heads, "n_kv_heads": s.n_kv_heads,
            "head_dim": s.head_dim, "raw_tokens": s.n_chunks * s.chunk, "chunk": s.chunk, "n_l2": h.n_l2,
            "group": h.group, "top_k2": h.top_k2, "top_k1": s.top_k, "tail": s.tail_len,
            "parallelism": f"replicas x{world}",
            "l2": f"rotating {L} replicas (own level-2 gists and query), {L * nbytes / 1e6:.0f} MB touched "
                  f"per rotation (L2 {l2 / 1e6:.0f} MB)"}


def suffix_flops(ss) -> float:
    """Algorithmic FLOPs of a suffix forward: per selection row (b, hk, p)
    the routing scores (2 G N d) and the attention over the position's
    context (4 G n_ctx d: QK and PV), n_ctx = the mode's gists + k c + p + 1."""
    s = ss.base
    gists = {synth.ALL_GISTS: s.n_chunks, synth.SELECTED_PAIRS: s.top_k, synth.SR_ONLY: 0,
             synth.UNSELECTED_GISTS: s.n_chunks - s.top_k}[s.mode]
    G, d, S = s.group, s.head_dim, s.tail_len
    ctx_sum = S * (gists + s.top_k * s.chunk) + S * (S + 1) / 2
    return float(s.rows * (S * 2 * G * s.n_chunks * d + 4 * G * d * ctx_sum))


def suffix_replicas(ss, l2: int, override: int = 0) -> int:
    """Replicas of the per-step tensors (queries, gists, suffix K/V) to
    rotate over so that one rotation touches >= 4x L2."""
    s = ss.base
    e = 4 if s.dtype == "f32" else 2
    per_rep = e * s.head_dim * (s.batch * s.tail_len * s.n_q_heads + 2 * s.rows * (s.n_chunks + s.tail_len))
    return override if override else max(2, -(-4 * l2 // per_rep))


def suffix_config(ss, workload: str, world: int, L: int, l2: int) -> dict:
    c = decode_config(ss.base, workload, world, L, 0, l2)
    c.pop("tail")
    c["suffix_len"] = ss.base.tail_len
    c["l2"] = f"rotating {L} replicas (own queries, gists and suffix K/V); raw chunks shared (L2 {l2 / 1e6:.0f} MB)"
    return c


def levels_config(h, workload: str, world: int, L: int, nbytes: int, l2: int) -> dict:
    s = h.l1
    return {"workload": workload, "batch": s.batch, "n_q_heads": s.n_q_heads, "n_kv_heads": s.n_kv_heads,
            "head_dim": s.head_dim, "raw_tokens": s.n_chunks * s.chunk, "chunk": s.chunk,
            "levels": len(h.counts), "gists_per_level": h.counts, "groups": list(h.groups),
            "top_k_per_level": [s.top_k] + list(h.top_ks), "tail": s.tail_len,
            "parallelism": f"replicas x{world}",
            "l2": f"rotating {L} replicas (own top-level gists and query), {L * nbytes / 1e6:.0f} MB touched "
                  f"per rotation (L2 {l2 / 1e6:.0f} MB)"}


def prefill_config(p, workload: str, world: int, l2: int) -> dict:
    qkv = (p.batch * p.n_q_heads + 2 * p.batch * p.n_kv_heads) * p.positions * p.head_dim * 2
    return {"workload": workload, "batch": p.batch, "n_q_heads": p.n_q_heads, "n_kv_heads": p.n_kv_heads,
            "head_dim": p.head_dim, "n_chunks": p.n_chunks, "chunk": p.chunk, "positions": p.positions,
            "parallelism": f"replicas x{world}",
            "l2": f"q, k, v of {qkv / 1e6:.0f} MB per step (L2 {l2 / 1e6:.0f} MB)"}


REPLAYS = 10


def timed_replays(run, stream, n: int = REPLAYS):
    """Device time (ms) of `run()` on `stream`, once per replay, CUDA events
    on the launching stream, synchronised on both sides of every replay."""
    import torch
    ms = []
    for _ in range(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record(stream)
            run()
            e1.record(stream)
        stream.synchronize()
        ms.append(e0.elapsed_time(e1))
    return ms


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    """Measured bf16 dense TFLOP/s, sustained (a kernel timed back to back for a
    long stretch runs under the power cap), else the recipe's fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["bf16_tflops_sustained"]), "measured (sustained)"
    return 1400.0, "fallback (sustained)"


PREFILL_METRIC = "gist-causal prefill: algorithmic TFLOP/s (4 d per allowed query-key pair) and % of bf16 tensor peak"
HIER_METRIC = "GSA hierarchical decode steps/sec and achieved HBM GB/s as % of B200 peak"


def prefill_pairs(n_chunks: int, chunk: int) -> int:
    """Allowed (query, key) pairs of one (sequence, head) under the gist mask:
    a gist sees the earlier gists, itself and its chunk's raw tokens; raw token
    i of a chunk sees the earlier gists and raw tokens 0..i of its chunk."""
    n, c = n_chunks, chunk
    earlier = n * (n - 1) // 2
    return earlier + n + n * c + c * earlier + n * c * (c + 1) // 2


def prefill_row_pairs(pos: int, chunk: int) -> int:
    j, i = divmod(pos, chunk + 1)
    return j + (chunk + 1 if i == chunk else i + 1)


def hier_bytes(h) -> int:
    """Bytes a hierarchical step must move: q, every level-2 gist K and V, the
    K and V of the selected groups' level-1 gists, the raw K/V of the k1
    chunks, the tail K/V, out."""
    s = h.l1
    row = s.head_dim * (4 if s.dtype == "f32" else 2)
    per_kv = 2 * h.n_l2 * row + 2 * h.top_k2 * h.group * row + 2 * s.top_k * s.chunk * row + 2 * s.tail_len * row
    return s.rows * per_kv + 2 * s.batch * s.n_q_heads * row


def levels_bytes(h) -> int:
    """Bytes a descent of any depth must move: q, every top-level gist K and
    V, the K and V of every lower level's candidates, the raw K/V of the k1
    chunks, the tail K/V, out."""
    s = h.l1
    row = s.head_dim * (4 if s.dtype == "f32" else 2)
    n = h.counts
    ks = (s.top_k,) + tuple(h.top_ks)
    per_kv = 2 * n[-1] * row
    for lv in range(len(n) - 1):
        per_kv += 2 * min(ks[lv + 1] * h.groups[lv], n[lv]) * row
    per_kv += 2 * s.top_k * s.chunk * row + 2 * s.tail_len * row
    return s.rows * per_kv + 2 * s.batch * s.n_q_heads * row


KERNEL_SOURCES = ("gsa_fused.cu", "gsa_fused.h", "gsa_device.cuh", "gsa_tc.cuh")


def measured_traffic(workload: str):
    """DRAM bytes per launch of the decode step stored in a committed ncu
    summary under profiles/ (it is not measured by this run), or None when
    none covers this workload or the kernel sources have changed since the
    counters were taken.  See traffic_source() for the file it came from."""
    return _stored_traffic(workload)[0]


def traffic_source(workload: str) -> str:
    """Where roofline.traffic comes from: the stored profile's file name."""
    path = _stored_traffic(workload)[1]
    return f"stored ncu profile {os.path.relpath(path, ROOT)}" if path else "none (no profile of these sources)"


def _stored_traffic(workload: str):
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
                return int(kv["dram_bytes_per_step"]) / int(kv["launches_per_step"]), path
            except (KeyError, ValueError):
                return None, None
    return None, None


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

    w = synth.WORKLOADS[args.workload]
    paged = isinstance(w, synth.PagedShape)
    s = w.base if paged else w
    torch.cuda.set_device(local)
    l2 = l2_bytes(local)
    if paged:
        x = synth.paged_inputs(w, synth.seed_for(args.workload) + 17 * rank)
        nbytes_step = paged_bytes(w, x.seq_chunks)
    else:
        x = synth.decode_inputs(s, synth.seed_for(args.workload) + 17 * rank)
        nbytes_step = algorithmic_bytes(s)
    L = replicas_for(nbytes_step, l2, args.replicas)
    base = {k: _dev(v) for k, v in x.tensors().items()}
    if paged:
        # every replica has its own pool (its own layer's caches); the table is shared
        base["k_pages"], base["v_pages"] = _dev(x.k_pages), _dev(x.v_pages)
        table = torch.from_numpy(x.table).cuda()
        nch = torch.from_numpy(x.seq_chunks).cuda()
        n_pages = int(x.k_pages.shape[0])
    reps = []
    for r in range(L):
        t = {k: (v if r == 0 else v.clone()) for k, v in base.items()}
        if r:
            # a distinct query per replica (distinct selections); caches are separate copies
            qn = synth.normal(synth.seed_for(args.workload) + 1000 * r + rank, synth.S_Q, x.q.shape, s.dtype)
            t["q"] = _dev(qn)
        reps.append(t)
    desc = _desc_of(s)
    wsz = gsa.gsa_decode_workspace_size(desc)
    launches = gsa.gsa_decode_launch_count(desc)
    outs = [torch.empty((s.batch, s.n_q_heads, s.head_dim), dtype=_tdtype(s.dtype), device="cuda") for _ in range(L)]
    idxs = [torch.empty((s.batch, s.n_kv_heads, s.top_k), dtype=torch.int32, device="cuda") for _ in range(L)]
    ws = torch.zeros(wsz, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    def step(i, st):
        t = reps[i % L]
        if paged:
            gsa.gsa_decode_step_paged(desc, t["q"], t["k_gist"], t["v_gist"], t["k_pages"], t["v_pages"], n_pages,
                                      table, nch, t["k_tail"], t["v_tail"], idxs[i % L], None, outs[i % L], ws,
                                      stream=st)
        else:
            gsa.gsa_decode_step(desc, t["q"], t["k_gist"], t["v_gist"], t["k_raw"], t["v_raw"], t["k_tail"],
                                t["v_tail"], idxs[i % L], None, outs[i % L], ws, stream=st)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, stream)
    stream.synchronize()
    # K timed steps captured as one graph, replayed REPLAYS times
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(args.steps):
                step(i, stream)
    with torch.cuda.stream(stream):
        g.replay()                                   # untimed replay: instantiate / warm the graph
    stream.synchronize()
    assert gsa.gsa_workspace_error(ws, stream=stream) == 0

    with ClockSampler(local) as clk:
        barrier(world)
        reps_ms = timed_replays(g.replay, stream)
        barrier(world)
    ms = statistics.median(reps_ms)
    ms_max = max_over_ranks(ms, world)
    clocks = clk.summary()
    assert gsa.gsa_workspace_error(ws, stream=stream) == 0

    # e2e through the C ABI: per step, H2D of the query from pinned memory,
    # the decode step, D2H of the output and the selection.
    q_host = [torch.empty_like(reps[r]["q"], device="cpu").pin_memory() for r in range(L)]
    for r in range(L):
        q_host[r].copy_(reps[r]["q"].cpu())
    out_host = torch.empty_like(outs[0], device="cpu").pin_memory()
    idx_host = torch.empty_like(idxs[0], device="cpu").pin_memory()
    q_dev = [reps[r]["q"] for r in range(L)]

    def e2e_run():
        for i in range(args.steps):
            r = i % L
            if paged:
                q_dev[r].copy_(q_host[r], non_blocking=True)
                step(i, stream)
                out_host.copy_(outs[r], non_blocking=True)
                idx_host.copy_(idxs[r], non_blocking=True)
            else:
                # one C-ABI call: the query in, the step, the output and the selection out
                t = reps[r]
                gsa.gsa_decode_step_host(desc, q_host[r], t["q"], t["k_gist"], t["v_gist"], t["k_raw"], t["v_raw"],
                                         t["k_tail"], t["v_tail"], idxs[r], idx_host, outs[r], out_host, ws,
                                         stream=stream)
            stream.synchronize()                     # the host reads the step's result

    barrier(world)
    e2e_ms = max_over_ranks(statistics.median(timed_replays(e2e_run, stream, 3)), world)

    per_step_ms = ms_max / args.steps
    steps_per_s = whole_job_rate(args.steps, world, ms_max)
    gbs = nbytes_step / (per_step_ms / 1e3) / 1e9
    peak, peak_kind = peaks()
    entry = "gsa_decode_step_paged" if paged else "gsa_decode_step"
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
        "config": (paged_config(w, x, args.workload, world, L, nbytes_step, l2) if paged else
                   decode_config(s, args.workload, world, L, nbytes_step, l2)),
        "timing": {"replays": len(reps_ms), "statistic": "median over replays of the K-step graph",
                   "ms_per_step_min": round(min(reps_ms) / args.steps, 5),
                   "ms_per_step_max": round(max(reps_ms) / args.steps, 5)},
        "head_steps_per_s": round(steps_per_s * s.batch * s.n_q_heads, 1),
        "algorithmic_bytes_per_step": nbytes_step,
        "roofline": {"bound": "hbm",
                     "kernel": (f"{entry}: one launch of fused_decode_kernel per step" if launches == 1 else
                                f"{entry}: {launches} launches per step (per launch: 1/{launches} of the "
                                f"step's algorithmic bytes in 1/{launches} of its time)"),
                     "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s", "frac": round(gbs / peak, 4),
                     "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": nbytes_step / launches,
                     "traffic": measured_traffic(args.workload) if not args.n_chunks else None,
                     "traffic_source": traffic_source(args.workload) if not args.n_chunks else "none"},
        "e2e": {"value": round(whole_job_rate(args.steps, world, e2e_ms), 2), "unit": "steps/s",
                "h2d_bytes_per_step": q_host[0].numel() * q_host[0].element_size(),
                "d2h_bytes_per_step": out_host.numel() * out_host.element_size()
                + idx_host.numel() * idx_host.element_size()},
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(s, x, args.cpu_seconds, w if paged else None)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g


# ------------------------------------------------------------- prefill ----
def run_prefill(args, world, rank, local):
    """The gist-causal prefill: K launches back to back (each reads its q, k,
    v, together far larger than L2), timed with CUDA events on the stream,
    median over REPLAYS replays of the K launches."""
    import torch

    import kv_cache_routing_b200 as gsa

    p = synth.WORKLOADS[args.workload]
    torch.cuda.set_device(local)
    x = synth.prefill_inputs(p, synth.seed_for(args.workload) + 17 * rank)
    d = {k: _dev(v) for k, v in x.tensors().items()}
    P = p.positions
    desc = gsa.prefill_desc(p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.n_chunks, p.chunk, gsa.GSA_BF16,
                            p.scale)
    out = torch.empty((p.batch, p.n_q_heads, P, p.head_dim), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()
    step = lambda: gsa.gsa_gist_prefill(desc, d["q"], d["k"], d["v"], out, None, stream=stream)

    def run_k():
        for _ in range(args.steps):
            step()

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    with ClockSampler(local) as clk:
        barrier(world)
        reps_ms = timed_replays(run_k, stream)
        barrier(world)
    ms_max = max_over_ranks(statistics.median(reps_ms), world)
    assert gsa.gsa_device_error() == 0
    flops = 4.0 * p.head_dim * prefill_pairs(p.n_chunks, p.chunk) * p.batch * p.n_q_heads
    per_ms = ms_max / args.steps
    tflops = world * flops / (per_ms / 1e3) / 1e12
    # e2e: q, k, v from pinned host memory, out back, every step
    hq = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in d.items()}
    for k in d:
        hq[k].copy_(d[k].cpu())
    ho = torch.empty_like(out, device="cpu").pin_memory()
    steps_e2e = max(1, min(args.steps, 5))

    def e2e_run():
        for _ in range(steps_e2e):
            for k in d:
                d[k].copy_(hq[k], non_blocking=True)
            step()
            ho.copy_(out, non_blocking=True)
            stream.synchronize()

    barrier(world)
    e2e_ms = max_over_ranks(statistics.median(timed_replays(e2e_run, stream, 3)), world) / steps_e2e
    peak, peak_kind = tensor_peak()
    line = {
        "metric": PREFILL_METRIC, "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": prefill_config(p, args.workload, world, l2_bytes(local)),
        "timing": {"replays": len(reps_ms), "statistic": "median over replays of K back-to-back launches",
                   "ms_per_step_min": round(min(reps_ms) / args.steps, 5),
                   "ms_per_step_max": round(max(reps_ms) / args.steps, 5)},
        "algorithmic_flop_per_step": flops,
        "roofline": {"bound": "tensor", "kernel": "gist_prefill_kernel (one launch per step)",
                     "achieved": round(tflops / world, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(tflops / world / peak, 4), "peak_kind": peak_kind, "traffic": None,
                     "traffic_source": "none"},
        "e2e": {"value": round(world * flops / (e2e_ms / 1e3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in d.values()),
                "d2h_bytes_per_step": out.numel() * out.element_size()},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(p, x, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)


def cpu_baseline_prefill(p, x, budget_s: float):
    """The fp64 oracle on random query rows until the time budget is spent,
    in the metric's unit (algorithmic FLOP of the rows done / time)."""
    import oracle
    rng = np.random.default_rng(7)
    t = x.tensors()
    P = p.positions
    done_flop, n, t0 = 0.0, 0, time.perf_counter()
    while True:
        rows = np.stack([rng.integers(p.batch, size=64), rng.integers(p.n_q_heads, size=64),
                         rng.integers(P, size=64)], axis=1).astype(np.int64)
        oracle.prefill_rows(t, p.n_chunks, p.chunk, rows, p.scale)
        done_flop += sum(4.0 * p.head_dim * prefill_row_pairs(int(r[2]), p.chunk) for r in rows)
        n += len(rows)
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(done_flop / el / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} random query rows of the workload, fp64, {el:.1f} s"}


# -------------------------------------------------------- hierarchical ----
def run_hier(args, world, rank, local):
    """The two-level descent: K steps captured as one graph rotating over L
    replicas (own level-2 gists and query each; level-1 gists and raw chunks
    shared, distinct queries select distinct children) so that the bytes a
    rotation touches exceed 4x L2; median over REPLAYS replays."""
    import torch

    import kv_cache_routing_b200 as gsa

    h = synth.WORKLOADS[args.workload]
    s = h.l1
    torch.cuda.set_device(local)
    l2 = l2_bytes(local)
    nbytes = hier_bytes(h)
    L = replicas_for(nbytes, l2, args.replicas)
    seed = synth.seed_for(args.workload) + 17 * rank
    x = synth.hier_inputs(h, seed)
    base = {k: _dev(v) for k, v in x.tensors().items()}
    reps = []
    for r in range(L):
        t = dict(base)
        if r:
            t["q"] = _dev(synth.normal(seed + 1000 * r, synth.S_Q, x.q.shape, s.dtype))
            t["k_g2"] = base["k_g2"].clone()
            t["v_g2"] = base["v_g2"].clone()
        reps.append(t)
    hd = gsa.hier_desc(_desc_of(s), h.n_l2, h.group, h.top_k2)
    ws = torch.zeros(max(256, gsa.gsa_hier_workspace_size(hd)), dtype=torch.uint8, device="cuda")
    outs = [torch.empty((s.batch, s.n_q_heads, s.head_dim), dtype=_tdtype(s.dtype), device="cuda") for _ in range(L)]
    i2 = torch.empty((s.batch, s.n_kv_heads, h.top_k2), dtype=torch.int32, device="cuda")
    i1 = torch.empty((s.batch, s.n_kv_heads, s.top_k), dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()

    def step(i, st):
        t = reps[i % L]
        gsa.gsa_hier_decode(hd, t["q"], t["k_g2"], t["v_g2"], t["k_g1"], t["v_g1"], t["k_raw"], t["v_raw"],
                            t["k_tail"], t["v_tail"], i2, i1, outs[i % L], ws, stream=st)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(args.steps):
                step(i, stream)
        g.replay()
    stream.synchronize()
    with ClockSampler(local) as clk:
        barrier(world)
        reps_ms = timed_replays(g.replay, stream)
        barrier(world)
    ms_max = max_over_ranks(statistics.median(reps_ms), world)
    assert gsa.gsa_workspace_error(ws, stream=stream) == 0
    per_ms = ms_max / args.steps
    gbs = nbytes / (per_ms / 1e3) / 1e9
    qh = torch.empty_like(reps[0]["q"], device="cpu").pin_memory()
    qh.copy_(reps[0]["q"].cpu())
    oh = torch.empty_like(outs[0], device="cpu").pin_memory()

    def e2e_run():
        for i in range(args.steps):
            reps[i % L]["q"].copy_(qh, non_blocking=True)
            step(i, stream)
            oh.copy_(outs[i % L], non_blocking=True)
            stream.synchronize()

    barrier(world)
    e2e_ms = max_over_ranks(statistics.median(timed_replays(e2e_run, stream, 3)), world)
    peak, peak_kind = peaks()
    line = {
        "metric": HIER_METRIC, "value": round(whole_job_rate(args.steps, world, ms_max), 2), "unit": "steps/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": s.dtype, "data": "synthetic",
        "config": hier_config(h, args.workload, world, L, nbytes, l2),
        "timing": {"replays": len(reps_ms), "statistic": "median over replays of the K-step graph",
                   "ms_per_step_min": round(min(reps_ms) / args.steps, 5),
                   "ms_per_step_max": round(max(reps_ms) / args.steps, 5)},
        "algorithmic_bytes_per_step": nbytes,
        "roofline": {"bound": "hbm", "kernel": f"gsa_hier_decode (whole step)", "achieved": round(gbs, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(gbs / peak, 4), "peak_kind": peak_kind,
                     "traffic": measured_traffic(args.workload) if not args.n_chunks else None,
                     "traffic_source": traffic_source(args.workload) if not args.n_chunks else "none"},
        "e2e": {"value": round(whole_job_rate(args.steps, world, e2e_ms), 2), "unit": "steps/s",
                "h2d_bytes_per_step": qh.numel() * qh.element_size(),
                "d2h_bytes_per_step": oh.numel() * oh.element_size()},
        "gpu_launches": gsa.gsa_hier_launch_count(hd) * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_hier(h, x, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g


SUFFIX_METRIC = "GSA stage-2 suffix forward positions/s and achieved TFLOP/s against the B200 bf16 peak"


def run_suffix(args, world, rank, local):
    """The stage-2 forward: K steps (each the whole suffix of every sequence)
    as one graph rotating over L replicas, median over REPLAYS replays."""
    import torch

    import kv_cache_routing_b200 as gsa

    ss = synth.WORKLOADS[args.workload]
    s = ss.base
    torch.cuda.set_device(local)
    l2 = l2_bytes(local)
    seed = synth.seed_for(args.workload) + 17 * rank
    x = synth.suffix_inputs(ss, seed)
    shared = {k: _dev(v) for k, v in (("k_raw", x.k_raw), ("v_raw", x.v_raw))}
    own = {k: _dev(getattr(x, k)) for k in ("q", "k_gist", "v_gist", "k_suf", "v_suf")}
    L = suffix_replicas(ss, l2, args.replicas)
    reps = [own] + [{k: v.clone() for k, v in own.items()} for _ in range(L - 1)]
    desc = _desc_of(s)
    ws = torch.zeros(max(256, gsa.gsa_suffix_workspace_size(desc)), dtype=torch.uint8, device="cuda")
    outs = [torch.empty((s.batch, s.tail_len, s.n_q_heads, s.head_dim), dtype=_tdtype(s.dtype), device="cuda")
            for _ in range(L)]
    stream = torch.cuda.Stream()

    def step(i, st):
        t = reps[i % L]
        gsa.gsa_suffix_attn(desc, t["q"], t["k_gist"], t["v_gist"], shared["k_raw"], shared["v_raw"], t["k_suf"],
                            t["v_suf"], None, None, outs[i % L], ws, stream=st)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(args.steps):
                step(i, stream)
        g.replay()
    stream.synchronize()
    with ClockSampler(local) as clk:
        barrier(world)
        reps_ms = timed_replays(g.replay, stream)
        barrier(world)
    ms_max = max_over_ranks(statistics.median(reps_ms), world)
    assert gsa.gsa_workspace_error(ws, stream=stream) == 0
    per_ms = ms_max / args.steps
    flops = suffix_flops(ss)
    tflops = flops / (per_ms / 1e3) / 1e12
    positions = s.batch * s.tail_len
    qh = torch.empty_like(own["q"], device="cpu").pin_memory()
    qh.copy_(own["q"].cpu())
    oh = torch.empty_like(outs[0], device="cpu").pin_memory()
    steps_e2e = max(1, min(args.steps, 20))

    def e2e_run():
        for i in range(steps_e2e):
            reps[i % L]["q"].copy_(qh, non_blocking=True)
            step(i, stream)
            oh.copy_(outs[i % L], non_blocking=True)
            stream.synchronize()

    barrier(world)
    e2e_ms = max_over_ranks(statistics.median(timed_replays(e2e_run, stream, 3)), world) / steps_e2e
    peak, peak_kind = tensor_peak()
    launches = gsa.gsa_suffix_launch_count(desc)
    line = {
        "metric": SUFFIX_METRIC, "value": round(whole_job_rate(args.steps, world, ms_max) * positions, 1),
        "unit": "positions/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": s.dtype, "data": "synthetic", "config": suffix_config(ss, args.workload, world, L, l2),
        "timing": {"replays": len(reps_ms), "statistic": "median over replays of the K-step graph",
                   "ms_per_step_min": round(min(reps_ms) / args.steps, 5),
                   "ms_per_step_max": round(max(reps_ms) / args.steps, 5)},
        "algorithmic_flop_per_step": flops,
        "roofline": {"bound": "tensor", "kernel": f"gsa_suffix_attn (whole step, {launches} launches, CUDA cores)",
                     "achieved": round(tflops, 2), "peak": peak, "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                     "peak_kind": peak_kind, "traffic": None, "traffic_source": "none"},
        "e2e": {"value": round(positions * 1e3 / e2e_ms, 1), "unit": "positions/s",
                "h2d_bytes_per_step": qh.numel() * qh.element_size(),
                "d2h_bytes_per_step": oh.numel() * oh.element_size()},
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_suffix(ss, x, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g


def run_levels(args, world, rank, local):
    """The descent of any depth through gsa_levels_decode, timed like the
    two-level one: K steps as one graph rotating over L replicas (own
    top-level gists and query each)."""
    import torch

    import kv_cache_routing_b200 as gsa

    h = synth.WORKLOADS[args.workload]
    s = h.l1
    torch.cuda.set_device(local)
    l2 = l2_bytes(local)
    nbytes = levels_bytes(h)
    L = replicas_for(nbytes, l2, args.replicas)
    seed = synth.seed_for(args.workload) + 17 * rank
    x = synth.levels_inputs(h, seed)
    kg = [_dev(a) for a in x.k_g]
    vg = [_dev(a) for a in x.v_g]
    raw = [_dev(a) for a in (x.k_raw, x.v_raw, x.k_tail, x.v_tail)]
    q0 = _dev(x.q)
    reps = []
    for r in range(L):
        q = q0 if r == 0 else _dev(synth.normal(seed + 1000 * r, synth.S_Q, x.q.shape, s.dtype))
        top_k, top_v = (kg[-1], vg[-1]) if r == 0 else (kg[-1].clone(), vg[-1].clone())
        reps.append((q, kg[:-1] + [top_k], vg[:-1] + [top_v]))
    desc = gsa.levels_desc(_desc_of(s), h.groups, h.top_ks)
    ws = torch.zeros(max(256, gsa.gsa_levels_workspace_size(desc)), dtype=torch.uint8, device="cuda")
    outs = [torch.empty((s.batch, s.n_q_heads, s.head_dim), dtype=_tdtype(s.dtype), device="cuda") for _ in range(L)]
    stream = torch.cuda.Stream()

    def step(i, st):
        q, kl, vl = reps[i % L]
        gsa.gsa_levels_decode(desc, q, kl, vl, *raw, None, outs[i % L], ws, stream=st)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(args.steps):
                step(i, stream)
        g.replay()
    stream.synchronize()
    with ClockSampler(local) as clk:
        barrier(world)
        reps_ms = timed_replays(g.replay, stream)
        barrier(world)
    ms_max = max_over_ranks(statistics.median(reps_ms), world)
    assert gsa.gsa_workspace_error(ws, stream=stream) == 0
    per_ms = ms_max / args.steps
    gbs = nbytes / (per_ms / 1e3) / 1e9
    qh = torch.empty_like(q0, device="cpu").pin_memory()
    qh.copy_(q0.cpu())
    oh = torch.empty_like(outs[0], device="cpu").pin_memory()

    def e2e_run():
        for i in range(args.steps):
            reps[i % L][0].copy_(qh, non_blocking=True)
            step(i, stream)
            oh.copy_(outs[i % L], non_blocking=True)
            stream.synchronize()

    barrier(world)
    e2e_ms = max_over_ranks(statistics.median(timed_replays(e2e_run, stream, 3)), world)
    peak, peak_kind = peaks()
    launches = gsa.gsa_levels_launch_count(desc)
    line = {
        "metric": HIER_METRIC, "value": round(whole_job_rate(args.steps, world, ms_max), 2), "unit": "steps/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": s.dtype, "data": "synthetic",
        "config": levels_config(h, args.workload, world, L, nbytes, l2),
        "timing": {"replays": len(reps_ms), "statistic": "median over replays of the K-step graph",
                   "ms_per_step_min": round(min(reps_ms) / args.steps, 5),
                   "ms_per_step_max": round(max(reps_ms) / args.steps, 5)},
        "algorithmic_bytes_per_step": nbytes,
        "roofline": {"bound": "hbm",
                     "kernel": (f"gsa_levels_decode: one launch of fused_decode_kernel per step" if launches == 1 else
                                f"gsa_levels_decode (whole step, {launches} launches)"),
                     "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s", "frac": round(gbs / peak, 4),
                     "peak_kind": peak_kind, "traffic": None, "traffic_source": "none"},
        "e2e": {"value": round(whole_job_rate(args.steps, world, e2e_ms), 2), "unit": "steps/s",
                "h2d_bytes_per_step": qh.numel() * qh.element_size(),
                "d2h_bytes_per_step": oh.numel() * oh.element_size()},
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_levels(h, x, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g


# ------------------------------------------------------------ CPU oracle ----
def _oracle_step(s, x, ps=None):
    """One whole decode step of the oracle on the workload's inputs."""
    import oracle
    t = x.tensors()
    if ps is not None:
        return lambda: oracle.decode_paged(t, x.k_pages, x.v_pages, x.table, s.top_k, s.mode,
                                           seq_chunks=x.seq_chunks)
    return lambda: oracle.decode(t, s.top_k, s.mode)


def cpu_baseline(s, x, budget_s: float, ps=None):
    """The fp64 oracle, as it stands, on the host cores: whole decode steps of
    the same workload until the time budget is spent (at least one)."""
    run = _oracle_step(s, x, ps)
    run()  # load + warm
    n, t0 = 0, time.perf_counter()
    while True:
        run()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(n / el, 4), "unit": "steps/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} full decode steps of the workload ({s.rows} (batch, kv-head) rows each), "
                      f"fp64, OpenMP over rows, {el:.1f} s"}


def cpu_baseline_hier(h, x, budget_s: float):
    """The fp64 oracle of the two-level descent, as it stands, on the host
    cores: whole steps until the time budget is spent (at least one).  A step
    has batch x kv-heads rows (8 for the 1M-token workload), so OpenMP over
    rows uses at most that many threads."""
    import oracle
    t = x.tensors()
    s = h.l1
    oracle.hier_decode(t, h.group, h.top_k2, s.top_k)   # load + warm
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.hier_decode(t, h.group, h.top_k2, s.top_k)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    cores = min(s.rows, int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)))
    return {"value": round(n / el, 4), "unit": "steps/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} full hierarchical steps of the workload ({s.rows} (batch, kv-head) rows each, so at "
                      f"most {s.rows} OpenMP threads), fp64, {el:.1f} s"}


def _oracle_levels(h, x):
    import oracle
    ks = (h.l1.top_k,) + tuple(h.top_ks)
    return lambda: oracle.hier_levels(x.q, x.k_g, x.v_g, x.k_raw, x.v_raw, x.k_tail, x.v_tail, h.groups, ks)


def cpu_baseline_levels(h, x, budget_s: float):
    """The fp64 oracle of the descent of any depth, as it stands, on the host
    cores: whole steps until the time budget is spent (at least one)."""
    run = _oracle_levels(h, x)
    s = h.l1
    run()
    n, t0 = 0, time.perf_counter()
    while True:
        run()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    cores = min(s.rows, int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)))
    return {"value": round(n / el, 4), "unit": "steps/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} full {len(h.counts)}-level steps of the workload ({s.rows} (batch, kv-head) rows each, "
                      f"so at most {s.rows} OpenMP threads), fp64, {el:.1f} s"}


def _oracle_suffix_sample(ss, x, n_pos: int):
    """The oracle on the first n_pos suffix positions of every sequence (a
    causal prefix of the suffix is a complete problem of its own)."""
    import oracle
    s = ss.base
    q = np.ascontiguousarray(x.q[:, :n_pos])
    ks, vs = np.ascontiguousarray(x.k_suf[:, :, :n_pos]), np.ascontiguousarray(x.v_suf[:, :, :n_pos])
    return lambda: oracle.suffix_attn(q, x.k_gist, x.v_gist, x.k_raw, x.v_raw, ks, vs, s.top_k, s.mode)


def cpu_baseline_suffix(ss, x, budget_s: float):
    s = ss.base
    n_pos = min(s.tail_len, 16)
    run = _oracle_suffix_sample(ss, x, n_pos)
    n, t0 = 0, time.perf_counter()
    while True:
        run()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 1000:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(n * s.batch * n_pos / el, 3), "unit": "positions/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} runs of the first {n_pos} suffix positions of each of the {s.batch} sequences, fp64, "
                      f"OpenMP over (b, kv head, position), {el:.1f} s"}


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle as it stands, on the host cores, on
    the same workload, metric, unit and config as the GPU arm; each step is
    a bounded sample of the workload (whole decode steps; for the prefill,
    random query rows).  Under torchrun only rank 0 runs it."""
    if rank != 0:
        return
    import oracle
    w = synth.WORKLOADS[args.workload]
    l2 = l2_bytes(0)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    seed = synth.seed_for(args.workload)
    if isinstance(w, synth.PrefillShape):
        x = synth.prefill_inputs(w, seed)
        t = x.tensors()
        rng = np.random.default_rng(7)
        rows = np.stack([rng.integers(w.batch, size=512), rng.integers(w.n_q_heads, size=512),
                         rng.integers(w.positions, size=512)], axis=1).astype(np.int64)
        flop = sum(4.0 * w.head_dim * prefill_row_pairs(int(r[2]), w.chunk) for r in rows)
        run = lambda: oracle.prefill_rows(t, w.n_chunks, w.chunk, rows, w.scale)
        metric, unit, dtype = PREFILL_METRIC, "TFLOP/s", "f64"
        config = prefill_config(w, args.workload, world, l2)
        sample = f"512 random query rows of the workload per step ({flop / 1e9:.2f} GFLOP algorithmic), fp64"
        rate = lambda sec: flop / sec / 1e12
    elif isinstance(w, synth.HierShape):
        x = synth.hier_inputs(w, seed)
        t = x.tensors()
        run = lambda: oracle.hier_decode(t, w.group, w.top_k2, w.l1.top_k)
        metric, unit, dtype = HIER_METRIC, "steps/s", "f64"
        nb = hier_bytes(w)
        config = hier_config(w, args.workload, world, replicas_for(nb, l2, args.replicas), nb, l2)
        sample = f"one full hierarchical step per step ({w.l1.rows} rows, OpenMP over rows), fp64"
        cores = min(cores, w.l1.rows)
        rate = lambda sec: 1.0 / sec
    elif isinstance(w, synth.SuffixShape):
        x = synth.suffix_inputs(w, seed)
        n_pos = min(w.base.tail_len, 16)
        run = _oracle_suffix_sample(w, x, n_pos)
        metric, unit, dtype = SUFFIX_METRIC, "positions/s", "f64"
        config = suffix_config(w, args.workload, world, suffix_replicas(w, l2, args.replicas), l2)
        sample = f"the first {n_pos} suffix positions of each of the {w.base.batch} sequences per step, fp64"
        rate = lambda sec: w.base.batch * n_pos / sec
    elif isinstance(w, synth.LevelsShape):
        x = synth.levels_inputs(w, seed)
        run = _oracle_levels(w, x)
        metric, unit, dtype = HIER_METRIC, "steps/s", "f64"
        nb = levels_bytes(w)
        config = levels_config(w, args.workload, world, replicas_for(nb, l2, args.replicas), nb, l2)
        sample = f"one full {len(w.counts)}-level step per step ({w.l1.rows} rows, OpenMP over rows), fp64"
        cores = min(cores, w.l1.rows)
        rate = lambda sec: 1.0 / sec
    elif isinstance(w, synth.PagedShape):
        x = synth.paged_inputs(w, seed)
        run = _oracle_step(w.base, x, w)
        metric, unit, dtype = METRIC, "steps/s", "f64"
        nb = paged_bytes(w, x.seq_chunks)
        config = paged_config(w, x, args.workload, world, replicas_for(nb, l2, args.replicas), nb, l2)
        sample = f"one full decode step per step ({w.base.rows} rows, OpenMP over rows), fp64"
        rate = lambda sec: 1.0 / sec
    else:
        x = synth.decode_inputs(w, seed)
        t = x.tensors()
        run = lambda: oracle.decode(t, w.top_k, w.mode)
        metric, unit, dtype = METRIC, "steps/s", "f64"
        nb = algorithmic_bytes(w)
        config = decode_config(w, args.workload, world, replicas_for(nb, l2, args.replicas), nb, l2)
        sample = f"one full decode step per step ({w.rows} rows, OpenMP over rows), fp64"
        rate = lambda sec: 1.0 / sec
    run()
    for _ in range(args.warmup):
        run()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    v = rate(total / args.steps)
    line = {"impl": "reference", "metric": metric, "value": round(v, 6), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
            "config": config,
            "cpu_baseline": {"value": round(v, 6), "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} steps; {sample}"},
            "e2e": {"value": round(v, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _with_chunks(w, n: int):
    """The workload with n level-1 chunks (profiling captures of a smaller case)."""
    import dataclasses
    if isinstance(w, synth.DecodeShape):
        return dataclasses.replace(w, n_chunks=n, n_needles=min(w.n_needles, n))
    if isinstance(w, synth.HierShape):
        return dataclasses.replace(w, l1=_with_chunks(w.l1, n), n_l2=-(-n // w.group))
    if isinstance(w, (synth.LevelsShape,)):
        return dataclasses.replace(w, l1=_with_chunks(w.l1, n))
    if isinstance(w, (synth.SuffixShape, synth.PagedShape)):
        return dataclasses.replace(w, base=_with_chunks(w.base, n))
    raise SystemExit("--n-chunks applies to decode-shaped workloads")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama8b_decode", choices=list(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--n-chunks", type=int, default=0,
                    help="profiling captures only: a smaller case of the same kernel (level-1 chunks of a decode "
                         "or hierarchical workload; the upper levels shrink with it)")
    ap.add_argument("--replicas", type=int, default=0,
                    help="layer replicas to rotate over (default: enough to exceed 4x L2); 1 for profiling captures")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.n_chunks:
        synth.WORKLOADS[args.workload] = _with_chunks(synth.WORKLOADS[args.workload], args.n_chunks)
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        w = synth.WORKLOADS[args.workload]
        if isinstance(w, synth.PrefillShape):
            run_prefill(args, world, rank, local)
        elif isinstance(w, synth.HierShape):
            run_hier(args, world, rank, local)
        elif isinstance(w, synth.LevelsShape):
            run_levels(args, world, rank, local)
        elif isinstance(w, synth.SuffixShape):
            run_suffix(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
