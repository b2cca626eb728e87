"""The multi-rank host logic of bench.py on CPU: two gloo ranks, one process
each (the GPU runs use the same code with NCCL).  Checks the max-over-ranks
timing reduction, the whole-job rate, and that only rank 0 prints."""
import os
import socket
import subprocess
import sys

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
