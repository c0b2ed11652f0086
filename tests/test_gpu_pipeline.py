"""Host tensors through the public call: head chunks whose copies overlap the
compute must give the one-pass result bit for bit (heads are independent in
every step), for BNSD with a batch and for TND (strided head slices)."""
import numpy as np
import pytest
import torch

from block_sparse_video_rearrange_b200 import pipeline, rf, synth
from tests import parity

pytestmark = pytest.mark.gpu

W, S = synth.Workload, synth.SeqSpec
CASES = {
    # BNSD, batch 2, GQA 8/4, ragged grid with a partial prefix block
    "bnsd_b2": W("bnsd_b2", "BNSD", "bf16", 2, (S(77, 9, 17, 33),), 8, 4, 128, 0.8, 21),
    # TND, two sequences, GQA 8/4, fp16
    "tnd": W("tnd", "TND", "fp16", 1, (S(64, 9, 16, 32), S(200, 10, 19, 21)), 8, 4, 128, 0.8, 22),
    # D = 64, one kv head per chunk
    "d64": W("d64", "BNSD", "bf16", 1, (S(128, 9, 16, 32),), 4, 4, 64, 0.9, 23),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def _host(bits, dtype):
    t = torch.float16 if dtype == "fp16" else torch.bfloat16
    return [torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(t).pin_memory() for x in bits]


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("chunks", [None, 2, 1])
def test_chunked_host_call_equals_one_pass(name, chunks):
    w = CASES[name]
    bits = synth.generate_qkv(w)
    ref = parity.run_gpu(w, bits)["o"]
    q, k, v = _host(bits, w.dtype)
    for _ in range(2):   # a second call reuses the cached pipeline and its buffers
        out = rf.rainfusion_attention(q, k, v, parity.seqs_of(w), w.sparsity, w.layout, chunks=chunks)
        assert not out.is_cuda
        assert np.array_equal(out.view(torch.int16).numpy().view(np.uint16), ref)


def test_pipeline_status_and_default_chunks():
    w = CASES["bnsd_b2"]
    pipe = pipeline.HostPipeline(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, w.batch)
    assert pipe.chunks == 4 and pipe.plan.n1 == 2 and pipe.plan.n2 == 1
    q, k, v = _host(synth.generate_qkv(w), w.dtype)
    out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    pipe(q, k, v, out)
    assert pipe.check_status() == (0, (0, 0))


@pytest.mark.parametrize("precision", ["mix", "mxfp4"])
def test_chunked_host_call_with_a_reduced_precision_equals_one_pass(precision):
    """Quantization groups never cross heads, so chunking by heads leaves the
    reduced-precision result unchanged too."""
    w = CASES["tnd"]
    bits = synth.generate_qkv(w)
    ref = parity.run_gpu(w, bits, precision=precision)["o"]
    q, k, v = _host(bits, w.dtype)
    out = rf.rainfusion_attention(q, k, v, parity.seqs_of(w), w.sparsity, w.layout, precision=precision,
                                  chunks=2)
    assert np.array_equal(out.view(torch.int16).numpy().view(np.uint16), ref)
