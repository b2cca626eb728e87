"""The multi-rank host logic of bench.py on CPU: two gloo ranks, one process
each (the GPU runs use the same code with NCCL).  Checks the max-over-ranks
timing reduction, the whole-job rate, that only rank 0 prints, and the keys of
the reference arm's line."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo")
    ms = bench.max_over_ranks(10.0 + 5.0 * r, w)       # rank 1 is the slow one
    bench.barrier(w)
    rate = bench.whole_job_rate(100, w, ms)
    dist.destroy_process_group()
    q.put((r, w, ms, rate))


def test_two_gloo_ranks_reduce_max_time_and_whole_job_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, ms, rate in res:
        assert w == 2 and ms == 15.0                  # the max over ranks
        assert abs(rate - 2 * 100 / 0.015) < 1e-6     # all ranks' steps / slowest time


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--workload", "tiny_f32"], env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


@pytest.mark.parametrize("workload", ["tiny_f32", "suffix_stage2"])
def test_reference_arm_line_carries_the_contract_keys(workload):
    """Rank 0 of the reference arm prints one JSON line with the contract's
    keys, its cpu_baseline and e2e repeating the line's own value, and the
    same config keys as the GPU arm's line for that workload."""
    import json
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--workload", workload], env=env, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["config"]["workload"] == workload
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.WORKLOADS[workload]
    if isinstance(w, synth.SuffixShape):
        gpu_cfg = bench.suffix_config(w, workload, 1, 2, bench.l2_bytes())
    else:
        gpu_cfg = bench.decode_config(w, workload, 1, 2, bench.algorithmic_bytes(w), bench.l2_bytes())
    assert set(d["config"]) == set(gpu_cfg)
