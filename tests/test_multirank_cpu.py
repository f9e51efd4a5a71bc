"""The N > 1 host logic of bench.py on two gloo ranks (CPU): every rank its own
inputs, the slowest rank's time for everyone, whole-job throughput."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import synthetic
        ms = [120.0, 150.0][rank]
        m = bench.reduce_max(ms, world, torch.device("cpu"))
        q, _, _ = synthetic.qkv_bf16(1, 8, 1, 16, seed=bench.rank_seed(rank))
        out[rank] = (m, int(q.astype(np.int64).sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 150.0           # everyone reports the slowest rank
    assert out[0][1] != out[1][1]                    # each rank its own clip
    import bench
    # two ranks, 1e12 FLOPs per rank-step, 4 steps in 150 ms -> 53.3 TFLOP/s for the job
    assert abs(bench.job_throughput(2, 1e12, 4, 150.0) - 2 * 4 / 0.150) < 1e-9


def test_bench_gpus_flag_starts_the_ranks():
    """`bench.py --gpus 2` outside torchrun starts two local ranks itself
    (torch.distributed.run on 127.0.0.1); each joins the group and rank 0
    reports that it saw both.  Host-only: gloo, no GPU, nothing timed."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--launcher-check"],
                         cwd=root, env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    assert json.loads(lines[0]) == {"launcher_check": True, "world": 2, "ranks_seen": 2}


def test_bench_refuses_a_world_size_other_than_gpus(monkeypatch):
    import pytest
    import bench
    monkeypatch.setenv("WORLD_SIZE", "3")
    with pytest.raises(SystemExit):
        bench.check_world(2)
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.check_world(2) == 2
