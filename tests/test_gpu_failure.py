"""Failure detection on a B200 without a GPU fault: a bounded wait that nothing
completes runs out after its limit (about a second), is recorded in the
workspace status words, is reported by rf_check_device_status, and leaves the
CUDA context usable; an attention launch that finds an expiry already recorded
skips its work instead of waiting on anything."""
import numpy as np
import pytest
import torch

from block_sparse_video_rearrange_b200 import rf, synth
from oracle import rainfusion as orc
from tests import parity
from tests.test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def test_expired_wait_is_reported_then_cleared_and_the_context_stays_usable():
    w = SMALL["tiny"]
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity)
    b = rf.Buffers(plan)
    rf.selftest_expired_wait(plan, b.ws)
    st, flags = rf.check_device_status(plan, b.ws)
    assert st == 5 and flags[0] == 0 and flags[1] == 1 << 31
    assert rf.check_device_status(plan, b.ws) == (0, (0, 0))      # read and cleared
    bits = synth.generate_qkv(w)
    gpu = parity.run_gpu(w, bits)                                   # the context still works
    p = parity.problem(w)
    parity.check_attention(p, w, parity_rearranged(p, bits), gpu)


def parity_rearranged(p, bits):
    return [orc.rearrange(p, x) for x in bits]


def test_attention_after_a_recorded_expiry_skips_its_work():
    w = SMALL["ragged_d128"]
    bits = synth.generate_qkv(w)
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity)
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    b = rf.Buffers(plan)
    rf.rearrange(plan, q, k, v, b.q_r, b.k_r, b.v_r, b.ws)
    rf.pool_select(plan, b.q_r, b.k_r, b.select_idx, b.select_num, b.ws)
    rf.selftest_expired_wait(plan, b.ws)                            # an expiry is now on record
    b.o_r.fill_(1.0)
    rf.block_sparse_attn(plan, b.q_r, b.k_r, b.v_r, b.select_idx, b.select_num, 0.088, b.o_r, b.ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(b.o_r).item() == 0                   # every CTA stopped: zero rows
    st, flags = rf.check_device_status(plan, b.ws)
    assert st == 5 and flags[1] == 1 << 31
    rf.block_sparse_attn(plan, b.q_r, b.k_r, b.v_r, b.select_idx, b.select_num, 0.088, b.o_r, b.ws)
    assert rf.check_device_status(plan, b.ws) == (0, (0, 0))
    # with the record cleared the same launch computes the rows again
    gpu = dict(idx=b.select_idx.cpu().numpy(), num=b.select_num.cpu().numpy(), scale=0.088,
               o_r=parity.to_bits(b.o_r))
    p = parity.problem(w)
    parity.check_attention(p, w, parity_rearranged(p, bits), gpu)


def test_public_call_raises_on_a_recorded_fault_and_the_next_call_succeeds():
    """rainfusion_attention reads the status words after every call (check=True): an
    expiry recorded in its workspace raises RfError(RF_ERR_DEVICE_FAULT), the words are
    cleared, and the next call computes the right result."""
    w = SMALL["ragged_d128"]
    bits = synth.generate_qkv(w)
    ref = parity.run_gpu(w, bits)
    seqs = parity.seqs_of(w)
    plan = rf.Plan(seqs, w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity)
    b = rf.Buffers(plan)
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    rf.selftest_expired_wait(plan, b.ws)
    with pytest.raises(rf.RfError) as e:
        rf.rainfusion_attention(q, k, v, seqs, w.sparsity, plan=plan, bufs=b)
    assert e.value.status == 5
    out = rf.rainfusion_attention(q, k, v, seqs, w.sparsity, plan=plan, bufs=b)
    torch.cuda.synchronize()
    assert np.array_equal(parity.to_bits(out), ref["o"])

    # the same through the host pipeline (host tensors): the fault is recorded in one of
    # the pipeline's workspaces, the next call raises, the call after it succeeds
    hq, hk, hv = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in bits)
    first = rf.rainfusion_attention(hq, hk, hv, seqs, w.sparsity)
    assert np.array_equal(first.view(torch.int16).numpy().view(np.uint16), ref["o"])
    pipe = next(pp for key, pp in rf._PIPELINES.items() if key[0] == tuple(map(tuple, seqs)))
    rf.selftest_expired_wait(pipe.plan, pipe.workspaces()[-1])
    with pytest.raises(rf.RfError) as e:
        rf.rainfusion_attention(hq, hk, hv, seqs, w.sparsity)
    assert e.value.status == 5
    again = rf.rainfusion_attention(hq, hk, hv, seqs, w.sparsity)
    assert np.array_equal(again.view(torch.int16).numpy().view(np.uint16), ref["o"])
