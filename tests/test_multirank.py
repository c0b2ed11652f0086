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


# ---------------- Ulysses sequence <-> head exchange (gloo, world size 2 and 4) ----------------

def _ulysses_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    from block_sparse_video_rearrange_b200 import ulysses
    g = torch.Generator().manual_seed(7)
    ok = []
    # BNSD: B=2, N=8, L=12, D=3 held in row slices of L/P per rank
    full = torch.randn(2, 8, 12, 3, generator=g)
    ls = 12 // world
    mine = full[:, :, rank * ls:(rank + 1) * ls].contiguous()
    heads = ulysses.seq_to_head(mine, "BNSD")
    nh = 8 // world
    ok.append(torch.equal(heads, full[:, rank * nh:(rank + 1) * nh]))
    ok.append(torch.equal(ulysses.head_to_seq(heads, "BNSD"), mine))
    # TND: T=16 packed rows, N=4 heads
    full_t = torch.randn(16, 4, 5, generator=g)
    ts = 16 // world
    mine_t = full_t[rank * ts:(rank + 1) * ts].contiguous()
    heads_t = ulysses.seq_to_head(mine_t, "TND")
    nh = 4 // world
    ok.append(torch.equal(heads_t, full_t[:, rank * nh:(rank + 1) * nh]))
    ok.append(torch.equal(ulysses.head_to_seq(heads_t, "TND"), mine_t))
    out[rank] = ok
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_exchange_matches_head_slices_and_round_trips(world):
    mgr = mp.Manager()
    out = mgr.dict()
    port = 28500 + (os.getpid() + 97 * world) % 1000
    mp.spawn(_ulysses_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        assert all(out[r]), (r, out[r])


def test_ulysses_shardability_rules():
    sys.path.insert(0, ROOT)
    from block_sparse_video_rearrange_b200 import ulysses
    ulysses.check_shardable([(512, 21, 30, 52)], 40, 40, "BNSD", 1, 8)          # 33,272 rows = 8 x 4,159
    ulysses.check_shardable([(256, 13, 32, 48), (384, 21, 24, 40)], 32, 8, "TND", 1, 8)
    with pytest.raises(ValueError):
        ulysses.check_shardable([(512, 21, 30, 52)], 40, 40, "BNSD", 1, 16)     # rows do not divide
    with pytest.raises(ValueError):
        ulysses.check_shardable([(256, 13, 32, 48)], 32, 8, "TND", 1, 16)       # 8 kv heads over 16 ranks
