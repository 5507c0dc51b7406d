"""The N > 1 host logic of bench.py on CPU, with world_size-2 gloo process groups.

The projection shards by tokens with no exchange (replicas), so the only cross-rank logic is
the timing: every rank times its own replica, the job takes the maximum over ranks, and the
whole-job throughput counts every rank's tokens.  These tests run that logic, and the
reference arm under torch.distributed.run, without a GPU."""
import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        # rank 1 is the slow one: the job time is its time
        mine = 1.0 + 2.0 * rank
        t = bench.reduce_max(mine, world)
        value = bench.aggregate_throughput(64, 10, world, t)
        out.put((rank, t, value))
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_aggregate_throughput_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29611
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, value in got:
        assert t == 3.0                          # max over ranks (rank 1: 1 + 2)
        assert value == pytest.approx(64 * 10 * 2 / 3.0)   # every rank's tokens / job time


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(2.5, 1) == 2.5
    assert bench.aggregate_throughput(8, 100, 1, 0.5) == 1600.0


def test_reference_arm_under_torchrun_two_ranks():
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", "29612", "bench.py", "--impl",
           "reference", "--workload", "tiny_single_t16", "--gpus", "2", "--steps", "2",
           "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1                       # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0
