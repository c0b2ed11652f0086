"""Multi-rank host logic of bench.py on CPU (gloo, world size 2)."""
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    # rank r took (10 + r) ms for a step and did (r + 1) units of work
    mx, sm = bench.reduce_over_ranks([10.0 + rank, 3.0 - rank, 0.5 * rank], [float(rank + 1)], "cpu")
    out[rank] = (tuple(mx), tuple(sm))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_over_ranks_takes_max_time_and_summed_work():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    port = 29500 + os.getpid() % 1000
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == ((11.0, 3.0, 0.5), (3.0,))


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                         env=env, capture_output=True, text=True, timeout=120)
    assert res.returncode == 0 and res.stdout.strip() == ""
