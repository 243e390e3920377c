"""Multi-rank host logic of the bench (replicas, one process per GPU), run as two
gloo ranks on CPU: times are combined as the max over ranks, the job value is the
aggregate over ranks, and non-zero ranks of the reference arm print nothing."""

import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)]
        got = bench.max_over_ranks(times, torch.device("cpu"))
        q.put((rank, got, bench.job_gbs(world, 1e9, got[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, gbs in res:
        assert got == [2.0, 5.0, 0.5]
        # 2 ranks x 1 GB per step in 2 ms (the slowest rank) = 1000 GB/s
        assert gbs == pytest.approx(1000.0)


def test_single_process_is_identity():
    import torch
    import bench
    assert bench.max_over_ranks([3.0, 1.5], torch.device("cpu")) == [3.0, 1.5]


def test_reference_arm_other_ranks_print_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "1"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_gpus_flag_launches_one_rank_per_gpu():
    # `bench.py --gpus 2` run directly starts two ranks through torch.distributed.run;
    # in the reference arm rank 0 alone works and prints the one JSON line.
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--config", "0", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["n_gpus"] == 2
    assert j["config"]["workload"] == "tiny-d128-k4v4"
    assert j["cpu_baseline"]["cores"] >= 1


def test_mismatched_world_size_is_refused():
    import bench
    env = dict(os.environ, WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--steps", "1"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode != 0
