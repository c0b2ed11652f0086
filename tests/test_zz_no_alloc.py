"""The allocation-free selection entry point, rf_pool_select_noalloc.

It serves callers that cannot allocate device memory (a plugin inside a host
framework that owns all device memory, or a latency-critical path where a
cudaMalloc is not acceptable): its scratch is a static array inside librf.
It must give exactly what rf_pool_select gives when it recomputes the block
means, call after call, even though every call reuses the same array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_video_rearrange_b200 import rf, synth
from tests import parity

pytestmark = pytest.mark.gpu

W, S = synth.Workload, synth.SeqSpec
CASES = {
    "ragged_d128": W("ragged_d128", "BNSD", "bf16", 1, (S(77, 9, 17, 33),), 2, 2, 128, 0.8, 11),
    "tnd_gqa_small": W("tnd_gqa_small", "TND", "fp16", 1, (S(64, 9, 16, 32), S(200, 10, 19, 21)), 4, 2, 128, 0.8, 13),
    "wan": synth.workload("wan"),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


@pytest.mark.parametrize("name,block_kv", [(n, 128) for n in CASES] + [("tnd_gqa_small", 64), ("wan", 64)])
def test_noalloc_selection_equals_workspace_selection_twice(name, block_kv):
    w = CASES[name]
    bits = synth.generate_qkv(w)
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch,
                   block_kv=block_kv)
    assert plan.workspace_bytes <= 32 << 20
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    b = rf.Buffers(plan)
    rf.rearrange(plan, q, k, v, b.q_r, b.k_r, b.v_r, b.ws)
    rf.pool_select(plan, b.q_r, b.k_r, b.select_idx, b.select_num, b.ws, pool_mode="recompute")
    ref_idx, ref_num = b.select_idx.clone(), b.select_num.clone()
    for _ in range(2):                       # the second call starts from the first call's leftovers
        idx = torch.full_like(b.select_idx, 7)
        num = torch.full_like(b.select_num, 7)
        rf.pool_select_noalloc(plan, b.q_r, b.k_r, idx, num)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)     # integer outputs: bit-exact
        assert torch.equal(num, ref_num)


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Too large for the static scratch: a clear error from the C ABI before any device work."""
    w = synth.workload("aligned")            # needs about 89 MB of selection scratch
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity)
    assert plan.workspace_bytes > 32 << 20
    t = torch.empty(64, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    st = rf.lib().rf_pool_select_noalloc(plan.handle, p, p, p, p, None)
    assert st == 1                            # RF_ERR_INVALID_ARG
    assert b"scratch" in rf.lib().rf_last_error()
    # a successful call right after the rejection leaves no stale error text
    w = CASES["ragged_d128"]
    bits = synth.generate_qkv(w)
    small = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch)
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    b = rf.Buffers(small)
    rf.rearrange(small, q, k, v, b.q_r, b.k_r, b.v_r, b.ws)
    st = rf.lib().rf_pool_select_noalloc(plan.handle, p, p, p, p, None)
    assert st == 1
    rf.pool_select_noalloc(small, b.q_r, b.k_r, b.select_idx, b.select_num)
    assert rf.lib().rf_last_error() == b""
    torch.cuda.synchronize()


@pytest.mark.parametrize("precision", ["mix", "mxfp4"])
def test_noalloc_accepts_a_quantized_plan_whose_selection_part_fits(precision):
    """A mix or mxfp4 plan's workspace also holds quantized copies of Q' and K'
    (and V'); selection needs only the part before them, which is what must fit."""
    w = CASES["wan"]
    bits = synth.generate_qkv(w)
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, precision=precision)
    first = min(o for o in (plan.info.ws_q8, plan.info.ws_q_mx) if o >= 0)   # the first quantized region
    assert plan.workspace_bytes > 32 << 20 and first <= 32 << 20
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    b = rf.Buffers(plan)
    rf.rearrange(plan, q, k, v, b.q_r, b.k_r, b.v_r, b.ws)
    rf.pool_select(plan, b.q_r, b.k_r, b.select_idx, b.select_num, b.ws, pool_mode="recompute")
    idx = torch.full_like(b.select_idx, 7)
    num = torch.full_like(b.select_num, 7)
    rf.pool_select_noalloc(plan, b.q_r, b.k_r, idx, num)
    torch.cuda.synchronize()
    assert torch.equal(idx, b.select_idx) and torch.equal(num, b.select_num)
