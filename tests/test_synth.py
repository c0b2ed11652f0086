"""The seeded input generator shared by the CUDA path and the oracle (CPU only)."""
import numpy as np
import torch

from block_sparse_video_rearrange_b200 import synth


def test_rounding_matches_torch_casts():
    x = np.random.default_rng(0).standard_normal(100_000).astype(np.float32) * 3
    x[:4] = [1.00390625, 1.01171875, -2.0000001, 65504.0]      # ties and edge values
    bf = synth.float32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf, ref)
    hf = synth.float32_to_fp16_bits(x)
    ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(hf, ref)
    assert np.array_equal(synth.bits_to_float64(bf, "bf16"),
                          torch.from_numpy(bf.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_generator_is_seeded_and_shaped():
    w = synth.workload("tiny")
    a = synth.generate_qkv(w)
    b = synth.generate_qkv(w.with_sparsity(0.5))
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert a[0].shape == (1, 2, 128 + 9 * 16 * 32, 64)
    tnd = synth.WORKLOADS["tnd_gqa"]
    small = synth.Workload("t", "TND", "fp16", 1, (synth.SeqSpec(16, 2, 8, 16), synth.SeqSpec(8, 1, 9, 8)),
                           4, 2, 16, 0.8, 7)
    q, k, v = synth.generate_qkv(small)
    assert q.shape == (16 + 256 + 8 + 72, 4, 16) and k.shape == (352, 2, 16)
    assert tnd.n1 % tnd.n2 == 0


def test_video_rows_share_their_cell_offset():
    # rows of one 8x8 cell are strongly correlated (shared offset), rows of different cells are not
    w = synth.Workload("c", "BNSD", "bf16", 1, (synth.SeqSpec(0, 1, 16, 16),), 1, 1, 256, 0.8, 3)
    q = synth.bits_to_float64(synth.generate_qkv(w)[0][0, 0], "bf16")
    same = np.corrcoef(q[0], q[1])[0, 1]          # (0,0) and (0,1): same cell
    other = np.corrcoef(q[0], q[8])[0, 1]         # (0,0) and (0,8): neighbouring cell
    assert same > 0.6 and abs(other) < 0.3


def test_pipeline_default_chunks_divide_the_heads():
    from block_sparse_video_rearrange_b200 import pipeline
    for n2 in (1, 2, 3, 4, 6, 8, 12, 24, 40, 7, 9, 32):
        c = pipeline.default_chunks(n2)
        assert n2 % c == 0 and 1 <= c <= 20
    assert pipeline.default_chunks(40) == 20 and pipeline.default_chunks(24) == 12 and pipeline.default_chunks(9) == 9
    assert pipeline.default_chunks(7) == 7 and pipeline.default_chunks(64) == 16
