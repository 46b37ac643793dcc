"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): timings are
max-reduced over ranks and the weak-scaling aggregate counts every rank's step."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measured" 10 + r ms and 20 - r ms
        got = bench.max_over_ranks([10.0 + rank, 20.0 - rank], world)
        out[rank] = torch.tensor(got)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        assert out[r].tolist() == [11.0, 20.0]


def test_weak_scaling_aggregate():
    import bench
    # 10,510,336 B per step in 17.6 us: one rank ~597 GB/s, two ranks twice that
    one = bench.aggregate_gbs(10_510_336, 17.6e-6, 1)
    two = bench.aggregate_gbs(10_510_336, 17.6e-6, 2)
    assert abs(one - 597.178) < 0.01 and abs(two - 2 * one) < 1e-9
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]


def _bench_env():
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    return env


def test_bench_gpus_flag_spawns_ranks():
    """`bench.py --gpus 2` with no launcher starts two local ranks itself (gloo on a
    host without GPUs) and rank 0 reports the max over both ranks."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--launcher-check"], cwd=root,
                       capture_output=True, text=True, timeout=600, env=_bench_env())
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    got = json.loads(lines[0])
    assert got["n_gpus"] == 2 and got["backend"] == "gloo"
    assert got["max_over_ranks"] == [2.0, 10.0]


def test_bench_refuses_world_size_mismatch():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = _bench_env()
    env.update(RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "3", "--launcher-check"], cwd=root,
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 2 and "WORLD_SIZE=2" in r.stderr
