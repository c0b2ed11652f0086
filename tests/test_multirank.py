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


# ---------------- UlyssesAttention composition (gloo, world size 2 and 4) ----------------
#
# Each rank runs the layer on its row slices; the per-rank path is replaced by the CPU
# oracle (injected by the test: the product never imports it).  The reassembled output
# must equal the oracle's whole path over all heads, because every step of the path is
# independent per (sequence, head) and a query head stays with its key/value head.

ULYSSES_CASES = {
    # BNSD, G = 2, 32 sparse blocks (not dense), L = 4,160 rows
    "bnsd": dict(layout="BNSD", dtype="bf16", seqs=[(64, 8, 16, 32)], n1=8, n2=4, d=64, sparsity=0.8),
    # TND varlen, G = 2: a sparse sequence next to a short dense one, T = 6,676 rows
    "tnd": dict(layout="TND", dtype="fp16", seqs=[(32, 8, 16, 32), (100, 9, 16, 17)], n1=8, n2=4, d=64,
                sparsity=0.7),
}


def _oracle_path(plan, qh, kh, vh, scale):
    import numpy as np
    from block_sparse_video_rearrange_b200 import synth
    from oracle import rainfusion as orc
    p = orc.make_problem(plan.layout, plan.batch, plan.seqs, plan.n1, plan.n2, plan.d, plan.sparsity)
    f = [synth.bits_to_float64(x.contiguous().view(torch.int16).numpy().view(np.uint16), plan.dtype)
         for x in (qh, kh, vh)]
    return torch.from_numpy(orc.run_path(p, *f, scale)["o"])


def _case_inputs(c):
    import numpy as np
    from block_sparse_video_rearrange_b200 import synth
    specs = tuple(synth.SeqSpec(*s) for s in c["seqs"])
    w = synth.Workload("ulysses", c["layout"], c["dtype"], 1, specs, c["n1"], c["n2"], c["d"], c["sparsity"], 77)
    bits = synth.generate_qkv(w)
    tdt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float16
    return [torch.from_numpy(b.view(np.int16)).view(tdt) for b in bits]


def _ulysses_layer_worker(rank, world, port, name, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    from block_sparse_video_rearrange_b200 import ulysses
    c = ULYSSES_CASES[name]
    q, k, v = _case_inputs(c)
    axis = 2 if c["layout"] == "BNSD" else 0
    rows = q.shape[axis] // world
    mine = [x.narrow(axis, rank * rows, rows).contiguous() for x in (q, k, v)]
    layer = ulysses.UlyssesAttention(c["seqs"], c["n1"], c["n2"], c["d"], c["layout"], c["dtype"], c["sparsity"],
                                     path=_oracle_path)
    o = layer(*mine, scale=0.125)
    out[rank] = o.numpy()
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(ULYSSES_CASES))
@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_layer_equals_the_oracle_over_all_heads(name, world):
    import numpy as np
    sys.path.insert(0, ROOT)
    from block_sparse_video_rearrange_b200 import rf
    mgr = mp.Manager()
    out = mgr.dict()
    port = 27500 + (os.getpid() + 31 * world + 7 * len(name)) % 1000
    mp.spawn(_ulysses_layer_worker, args=(world, port, name, out), nprocs=world, join=True)
    c = ULYSSES_CASES[name]
    q, k, v = _case_inputs(c)
    plan = rf.Plan(c["seqs"], c["n1"], c["n2"], c["d"], c["layout"], c["dtype"], c["sparsity"])
    full = _oracle_path(plan, q, k, v, 0.125).numpy()
    axis = 2 if c["layout"] == "BNSD" else 0
    got = np.concatenate([out[r] for r in range(world)], axis=axis)
    assert got.shape == full.shape
    assert np.max(np.abs(got - full)) <= 1e-12
