"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200."""
import math

import numpy as np
import pytest
import torch

from block_sparse_video_rearrange_b200 import rf, synth
from oracle import mxattention as mxo
from oracle import rainfusion as orc
from tests import parity

pytestmark = pytest.mark.gpu

W = synth.Workload
S = synth.SeqSpec

# Small cases the oracle finishes in seconds; each spans several tiles and a ragged tail.
SMALL = {
    # the Tiny workload itself (D = 64, aligned grid, 4 sink blocks)
    "tiny": synth.WORKLOADS["tiny"],
    # ragged h and w, partial last prefix block (Lp = 518), D = 128
    "ragged_d128": W("ragged_d128", "BNSD", "bf16", 1, (S(77, 9, 17, 33),), 2, 2, 128, 0.8, 11),
    # batch of two, D = 64, higher sparsity
    "batch2_d64": W("batch2_d64", "BNSD", "bf16", 2, (S(128, 9, 16, 32),), 2, 2, 64, 0.9, 12),
    # varlen TND, fp16, GQA G = 2; the second sequence is short (20 blocks) and runs dense
    "tnd_gqa_small": W("tnd_gqa_small", "TND", "fp16", 1, (S(64, 9, 16, 32), S(200, 10, 19, 21)),
                       4, 2, 128, 0.8, 13),
    # sparsity 0 must equal dense attention
    "dense": W("dense", "BNSD", "bf16", 1, (S(100, 8, 16, 32),), 2, 1, 128, 0.0, 14),
    # sparsity 1: prefix + sinks only
    "s_one": W("s_one", "BNSD", "bf16", 1, (S(40, 9, 16, 32),), 2, 2, 128, 1.0, 15),
    # no text prefix at all, odd tile column count
    "no_prefix": W("no_prefix", "BNSD", "fp16", 1, (S(0, 6, 24, 40),), 2, 2, 64, 0.5, 16),
    # text only: no video at all, three prefix blocks, the last one partial (44 rows)
    "text_only": W("text_only", "BNSD", "bf16", 1, (S(300, 0, 0, 0),), 2, 2, 64, 0.8, 31),
    # TND: a grid under 8 rows high (every video token promoted) next to a 2-block video
    "all_promoted": W("all_promoted", "TND", "fp16", 1, (S(64, 3, 5, 9), S(0, 2, 16, 16)), 2, 1, 128, 0.8, 32),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


@pytest.mark.parametrize("name", list(SMALL))
def test_small_full_parity(name):
    w = SMALL[name]
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits)
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    parity.check_pooled(p, qbars, kbars, gpu)
    stats = parity.check_selection(p, qbars, kbars, gpu)
    assert stats["near_tie"] <= max(1, stats["rows"] // 100)
    err = parity.check_attention(p, w, rbits, gpu)
    if name == "dense":
        assert np.all(gpu["num"] == p.geoms[0].n_blocks)
        # against a library dense attention on the original order, per head
        q, k, v = (synth.bits_to_float64(x, w.dtype) for x in bits)
        o = synth.bits_to_float64(gpu["o"], w.dtype)
        for n in range(w.n1):
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[0, n]), torch.from_numpy(k[0, n // 2]), torch.from_numpy(v[0, n // 2]),
                scale=gpu["scale"]).numpy()
            assert np.max(np.abs(o[0, n] - ref)) <= parity.MAX_ABS


def test_pool_recompute_mode_matches_fused_pool():
    w = SMALL["ragged_d128"]
    bits = synth.generate_qkv(w)
    a = parity.run_gpu(w, bits, pool_mode="from_ws")
    b = parity.run_gpu(w, bits, pool_mode="recompute")
    assert np.array_equal(a["pooled_q"], b["pooled_q"]) and np.array_equal(a["pooled_k"], b["pooled_k"])
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["num"], b["num"])
    assert np.array_equal(a["o"], b["o"])


def test_deterministic_repeat():
    w = SMALL["tnd_gqa_small"]
    bits = synth.generate_qkv(w)
    a = parity.run_gpu(w, bits)
    b = parity.run_gpu(w, bits)
    for key in ("q_r", "idx", "num", "o_r", "o"):
        assert np.array_equal(a[key], b[key]), key


def test_handmade_selection_with_padding_and_bad_entries():
    """Any valid selectIdx is accepted; -1 slots are skipped; out-of-range entries are
    skipped and counted in the status words; selectNum 0 gives zeros."""
    w = SMALL["ragged_d128"]
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    g = p.geoms[0]
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity)
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    b = rf.Buffers(plan)
    rf.rearrange(plan, q, k, v, b.q_r, b.k_r, b.v_r, b.ws)
    rng = np.random.default_rng(0)
    T, N, M = b.select_idx.shape
    idx = np.full((T, N, M), -1, dtype=np.int32)
    num = np.zeros((T, N), dtype=np.int32)
    clean = np.full((T, N, M), -1, dtype=np.int32)
    clean_num = np.zeros((T, N), dtype=np.int32)
    bad = 0
    for t in range(T):
        for n in range(N):
            if (t + n) % 7 == 3:
                continue  # selectNum 0 -> zero output rows
            chosen = sorted(rng.choice(g.n_blocks, size=int(rng.integers(1, g.n_blocks - 2)), replace=False).tolist())
            row = list(chosen)
            if t % 3 == 0:
                row.insert(1, -1)
            if t % 5 == 0:
                row.append(g.n_blocks + 3)   # out of range
                bad += 1
            idx[t, n, :len(row)] = row
            num[t, n] = len(row)
            clean[t, n, :len(chosen)] = chosen
            clean_num[t, n] = len(chosen)
    b.select_idx.copy_(torch.from_numpy(idx))
    b.select_num.copy_(torch.from_numpy(num))
    scale = 0.09
    rf.block_sparse_attn(plan, b.q_r, b.k_r, b.v_r, b.select_idx, b.select_num, scale, b.o_r, b.ws)
    st, flags = rf.check_device_status(plan, b.ws)
    assert st == 5                                      # RF_ERR_DEVICE_FAULT
    assert flags[0] == bad * 1 and flags[1] == 0
    st, flags = rf.check_device_status(plan, b.ws)
    assert st == 0 and flags == (0, 0)                  # cleared
    gpu = dict(idx=clean, num=clean_num, scale=scale, o_r=parity.to_bits(b.o_r))
    rbits = [orc.rearrange(p, x) for x in bits]
    items = [(t, n) for t in range(T) for n in range(N) if clean_num[t, n] > 0]
    parity.check_attention(p, w, rbits, gpu, items)
    o_r = synth.bits_to_float64(gpu["o_r"], w.dtype)
    for t in range(T):
        for n in range(N):
            if clean_num[t, n] == 0:
                r = orc.block_rows(g, t)
                assert np.all(o_r[0, n, r.start:r.stop] == 0)


def test_forward_entry_point_equals_step_calls():
    w = SMALL["tnd_gqa_small"]
    bits = synth.generate_qkv(w)
    steps = parity.run_gpu(w, bits)
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity)
    b = rf.Buffers(plan)
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    out = rf.forward(plan, q, k, v, b)
    torch.cuda.synchronize()
    assert np.array_equal(parity.to_bits(out), steps["o"])


def test_user_call_with_host_tensors():
    w = SMALL["batch2_d64"]
    bits = synth.generate_qkv(w)
    steps = parity.run_gpu(w, bits)
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in bits)
    out = rf.rainfusion_attention(q, k, v, parity.seqs_of(w), sparsity=w.sparsity)
    assert not out.is_cuda
    assert np.array_equal(out.view(torch.int16).numpy().view(np.uint16), steps["o"])


# ------------------------------------------------------------------------------------------
# Full-size workloads in the bench's launch configuration: permutation bit-exact over
# everything, pooling and selection over every row, attention on sampled items.
# ------------------------------------------------------------------------------------------

FULL = [("wan", None), ("minimax", 0.8), ("minimax", 0.5), ("minimax", 0.9), ("tnd_gqa", None),
        ("aligned", 0.8), ("aligned", 0.0), ("aligned", 0.5), ("aligned", 0.9)]


@pytest.mark.parametrize("name,s", FULL)
def test_full_size_parity(name, s):
    w = synth.workload(name, s)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits)
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    parity.check_pooled(p, qbars, kbars, gpu)
    stats = parity.check_selection(p, qbars, kbars, gpu)
    assert stats["near_tie"] <= max(1, stats["rows"] // 1000), stats
    items = parity.sample_items(p, np.random.default_rng(7), per_kind=3)
    parity.check_attention(p, w, rbits, gpu, items)


# Whole heads at full size: every query block of the first and the last query head
# against the oracle, one full-size configuration per precision.
WHOLE_HEADS = [("aligned", 0.8, "native"), ("wan", None, "mix"), ("wan", None, "mxfp4")]


@pytest.mark.parametrize("name,s,precision", WHOLE_HEADS)
def test_full_size_whole_heads(name, s, precision):
    w = synth.workload(name, s)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, precision=precision)
    rbits = [orc.rearrange(p, x) for x in bits]
    items = [(t, n) for t in range(p.t_qblk) for n in (0, w.n1 - 1)]
    if precision == "native":
        err = parity.check_attention(p, w, rbits, gpu, items)
    elif precision == "mix":
        parity.check_mix_quantization(p, w, rbits, gpu)
        err = parity.check_attention(p, w, rbits, gpu, items, values=parity.mix_reference_inputs(p, w, gpu, rbits))
    else:
        ref = parity.oracle_mx_inputs(p, w, rbits)
        parity.check_mx_quantization(p, w, ref, gpu)
        err = parity.check_attention(p, w, rbits, gpu, items, values=ref, oracle_fn=mxo.attention_mx)
    print(f"{name}@{w.sparsity:g} {precision}: {err['items']} items (two whole heads), "
          f"max abs {err['max_abs']:.3e}, rel L2 {err['rel_l2']:.3e}")
    assert err["items"] == 2 * p.t_qblk


# ------------------------------------------------------------------------------------------
# Frame-pair token order (xllm PR #1867, frame-pairing approach): the whole path with the
# permutation of rf_plan_create_ex(RF_ORDER_FRAME_PAIR), against the oracle in the same order.
# ------------------------------------------------------------------------------------------

FRAME_PAIR = [
    ("tiny", SMALL["tiny"]),                      # 9 frames: 4 pairs after frame 0
    ("ragged_d128", SMALL["ragged_d128"]),        # ragged edge promoted, 9 frames
    ("no_prefix", SMALL["no_prefix"]),            # 6 frames: the last one is unpaired
    ("tnd_gqa_small", SMALL["tnd_gqa_small"]),    # two sequences, 9 and 10 frames
]


@pytest.mark.parametrize("name,w", FRAME_PAIR, ids=[n for n, _ in FRAME_PAIR])
def test_frame_pair_small_full_parity(name, w):
    bits = synth.generate_qkv(w)
    p = parity.problem(w, order="frame_pair")
    gpu = parity.run_gpu(w, bits, order="frame_pair")
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    parity.check_pooled(p, qbars, kbars, gpu)
    stats = parity.check_selection(p, qbars, kbars, gpu)
    assert stats["near_tie"] <= max(1, stats["rows"] // 100)
    parity.check_attention(p, w, rbits, gpu)


@pytest.mark.parametrize("name,s", [("wan", None), ("minimax", 0.8)])
def test_frame_pair_full_size_parity(name, s):
    w = synth.workload(name, s)
    bits = synth.generate_qkv(w)
    p = parity.problem(w, order="frame_pair")
    gpu = parity.run_gpu(w, bits, order="frame_pair")
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    parity.check_pooled(p, qbars, kbars, gpu)
    stats = parity.check_selection(p, qbars, kbars, gpu)
    assert stats["near_tie"] <= max(1, stats["rows"] // 1000), stats
    items = parity.sample_items(p, np.random.default_rng(8), per_kind=3)
    parity.check_attention(p, w, rbits, gpu, items)


# ------------------------------------------------------------------------------------------
# Precision "mix" (E4M3 Q K^T, 16-bit P V): the E4M3 copies and scales bit-exact against the
# oracle's quantization; the output against the oracle run on the dequantized Q', K' (the
# inputs this precision defines) within the same bars as the native path.
# ------------------------------------------------------------------------------------------

MIX_SMALL = ["ragged_d128", "tnd_gqa_small", "dense", "s_one", "all_promoted"]


@pytest.mark.parametrize("name", MIX_SMALL)
def test_mix_small_parity(name):
    w = SMALL[name]
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, precision="mix")
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    parity.check_mix_quantization(p, w, rbits, gpu)
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    parity.check_pooled(p, qbars, kbars, gpu)             # pooling still reads the 16-bit values
    parity.check_selection(p, qbars, kbars, gpu)
    parity.check_attention(p, w, rbits, gpu, values=parity.mix_reference_inputs(p, w, gpu, rbits))


@pytest.mark.parametrize("name,s", [("wan", None), ("tnd_gqa", None)])
def test_mix_full_size_parity(name, s):
    w = synth.workload(name, s)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, precision="mix")
    rbits = [orc.rearrange(p, x) for x in bits]
    parity.check_mix_quantization(p, w, rbits, gpu)
    items = parity.sample_items(p, np.random.default_rng(9), per_kind=3)
    parity.check_attention(p, w, rbits, gpu, items, values=parity.mix_reference_inputs(p, w, gpu, rbits))
    # the quantization error itself, against the unquantized oracle: reported, and bounded
    # loosely (E4M3 keeps 3 mantissa bits)
    err = parity.check_attention(p, w, rbits, gpu, items, check=False)
    assert err["rel_l2"] <= 0.1, err


def test_mix_quantize_entry_point_equals_fused_quantization():
    w = SMALL["tnd_gqa_small"]
    bits = synth.generate_qkv(w)
    fused = parity.run_gpu(w, bits, precision="mix")
    plan = fused["plan"]
    b = rf.Buffers(plan)
    q_r = parity.to_device(fused["q_r"], w.dtype)
    k_r = parity.to_device(fused["k_r"], w.dtype)
    rf.quantize_qk(plan, q_r, k_r, b.ws)
    torch.cuda.synchronize()
    alone = parity.mix_buffers(plan, b.ws)
    for key in ("q8", "k8", "q_scale", "k_scale"):
        assert np.array_equal(alone[key], fused[key]), key


# ------------------------------------------------------------------------------------------
# Precision "mxfp4" (MXAttention abstract: MXFP4 attention, UOS scaling with Qmax = 7.25,
# Pre-Normalization Quantization): the MXFP4 copies of Q', K', V' equal the oracle's rounding
# value for value; the output against the oracle's PNQ attention on those values within the
# same bars as the native path.
# ------------------------------------------------------------------------------------------

MX_SMALL = ["tiny", "ragged_d128", "tnd_gqa_small", "dense", "s_one", "no_prefix", "text_only",
            "all_promoted"]


@pytest.mark.parametrize("name", MX_SMALL)
def test_mxfp4_small_parity(name):
    w = SMALL[name]
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, precision="mxfp4")
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    ref = parity.oracle_mx_inputs(p, w, rbits)
    parity.check_mx_quantization(p, w, ref, gpu)
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    parity.check_pooled(p, qbars, kbars, gpu)             # pooling reads the unrounded values
    parity.check_selection(p, qbars, kbars, gpu)
    parity.check_attention(p, w, rbits, gpu, values=ref, oracle_fn=mxo.attention_mx)


@pytest.mark.parametrize("name,s", [("wan", None), ("tnd_gqa", None), ("minimax", 0.8)])
def test_mxfp4_full_size_parity(name, s):
    w = synth.workload(name, s)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, precision="mxfp4")
    rbits = [orc.rearrange(p, x) for x in bits]
    ref = parity.oracle_mx_inputs(p, w, rbits)
    parity.check_mx_quantization(p, w, ref, gpu)
    items = parity.sample_items(p, np.random.default_rng(10), per_kind=3)
    parity.check_attention(p, w, rbits, gpu, items, values=ref, oracle_fn=mxo.attention_mx)
    # the quantization error itself, against the unquantized oracle: reported, bounded loosely
    err = parity.check_attention(p, w, rbits, gpu, items, check=False)
    assert err["rel_l2"] <= 0.25, err


def test_mxfp4_with_frame_pair_order():
    w = SMALL["tnd_gqa_small"]
    bits = synth.generate_qkv(w)
    p = parity.problem(w, order="frame_pair")
    gpu = parity.run_gpu(w, bits, order="frame_pair", precision="mxfp4")
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    ref = parity.oracle_mx_inputs(p, w, rbits)
    parity.check_mx_quantization(p, w, ref, gpu)
    parity.check_attention(p, w, rbits, gpu, values=ref, oracle_fn=mxo.attention_mx)


def test_mxfp4_quantize_entry_point_equals_fused_quantization():
    w = SMALL["ragged_d128"]
    bits = synth.generate_qkv(w)
    fused = parity.run_gpu(w, bits, precision="mxfp4")
    plan = fused["plan"]
    b = rf.Buffers(plan)
    q_r, k_r, v_r = (parity.to_device(fused[n], w.dtype) for n in ("q_r", "k_r", "v_r"))
    rf.quantize_mx(plan, q_r, k_r, v_r, b.ws)
    torch.cuda.synchronize()
    alone = parity.mx_buffers(plan, b.ws)
    for key in ("qx", "kx", "vx"):
        assert np.array_equal(alone[key], fused[key]), key


def test_maximum_size_sequence():
    """One sequence at the largest sizes the kernels take: 2,048 sparse blocks (the top-k
    kernel's widest rows) and 2,048 key blocks per selectIdx row (the attention kernel's
    list), 64 first-frame sinks, k = 410."""
    w = W("maxsize", "BNSD", "bf16", 1, (S(0, 32, 64, 128),), 1, 1, 64, 0.8, 33)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    g = p.geoms[0]
    assert (g.nb, g.n_blocks, g.ns, g.k) == (2048, 2048, 64, 410)
    gpu = parity.run_gpu(w, bits)
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    parity.check_pooled(p, qbars, kbars, gpu)
    stats = parity.check_selection(p, qbars, kbars, gpu)
    assert stats["near_tie"] <= max(1, stats["rows"] // 1000), stats
    items = [(0, 0), (63, 0), (64, 0), (1000, 0), (2047, 0)]     # sink, last sink, first sparse, middle, last
    parity.check_attention(p, w, rbits, gpu, items)


def test_exp2_polynomial_against_mufu_and_exact():
    """The FMA-pipe exponential the softmax uses for part of its columns:
    relative error <= 2e-4 against the exact 2^x and against ex2.approx,
    over the range the softmax feeds it (x <= 8)."""
    x = torch.cat([torch.linspace(-125.0, 8.0, 2_000_001, dtype=torch.float32),
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, -8.0, 8.0, -20.25], dtype=torch.float32)]).cuda()
    yp, ym = rf.selftest_exp2(x)
    torch.cuda.synchronize()
    exact = torch.exp2(x.double())
    rel_poly = ((yp.double() - exact).abs() / exact).max().item()
    rel_mufu = ((ym.double() - exact).abs() / exact).max().item()
    assert rel_poly <= 2e-4, rel_poly
    assert rel_mufu <= 1e-5, rel_mufu
    # integers map to exact powers of two
    xi = torch.arange(-120, 9, dtype=torch.float32).cuda()
    yi, _ = rf.selftest_exp2(xi)
    assert torch.equal(yi.double(), torch.exp2(xi.double()))


# ------------------------------------------------------------------------------------------
# blockShape 128 x 64 (aclnnRainFusionAttention "Formula": blocks of blockShapeX x
# blockShapeY): key/value blocks of 64 rows, paired by the kernel into 128-key tiles.
# ------------------------------------------------------------------------------------------

KV64 = ["ragged_d128", "tnd_gqa_small", "tiny", "text_only", "all_promoted", "no_prefix"]


def _kv64_run(w, q_r, k_r, v_r, idx, num, scale):
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch,
                   block_kv=64)
    b = rf.Buffers(plan)
    assert tuple(b.select_idx.shape) == idx.shape
    b.select_idx.copy_(torch.from_numpy(idx))
    b.select_num.copy_(torch.from_numpy(num))
    rf.block_sparse_attn(plan, q_r, k_r, v_r, b.select_idx, b.select_num, scale, b.o_r, b.ws)
    st, flags = rf.check_device_status(plan, b.ws)
    assert st == 0, (st, flags)
    return parity.to_bits(b.o_r)


@pytest.mark.parametrize("name", KV64)
def test_kv64_halves_of_a_128_selection_give_the_128_result_bit_for_bit(name):
    """Listing both 64-row halves of every selected 128-row block rebuilds the same
    128-key tiles (the partial prefix block alone when it is one half), so the
    output equals the 128 x 128 path's bit for bit -- except in a sequence whose
    dense prefix ends 64 rows into a 128-row block: there the last prefix block
    is a whole 64-row block, pairs with the next selected block, and the tiles
    (hence the summation order) differ; those rows are held to the parity bar."""
    w = SMALL[name]
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits)
    plan64 = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch,
                     block_kv=64)
    idx64, num64 = parity.expand_to_kv64(p, gpu["idx"], gpu["num"], int(plan64.info.max_kv_blocks))
    q_r, k_r, v_r = (parity.to_device(gpu[n], w.dtype) for n in ("q_r", "k_r", "v_r"))
    o64 = _kv64_run(w, q_r, k_r, v_r, idx64, num64, gpu["scale"])
    a64 = synth.bits_to_float64(o64, w.dtype)
    a128 = synth.bits_to_float64(gpu["o_r"], w.dtype)
    regrouped = 0
    for s_id, g in p.sequences():
        for n in range(w.n1):
            x, y = p.head_rows(a64, s_id, n), p.head_rows(a128, s_id, n)
            if g.lp % 128 == 64:
                regrouped += 1
                assert np.max(np.abs(x - y)) <= parity.MAX_ABS
            else:
                assert np.array_equal(x, y), (s_id, n)
    assert regrouped < len(p.sequences()) * w.n1      # most rows are checked bit for bit


@pytest.mark.parametrize("name", KV64)
def test_kv64_random_selection_against_the_oracle(name):
    """Arbitrary ascending 64-row selections (odd counts, gaps, the partial prefix
    block at even and odd positions, -1 slots) against the oracle with 64-row key blocks."""
    w = SMALL[name]
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits)
    table = orc.qblock_table(p)
    plan64 = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch,
                     block_kv=64)
    T, N = gpu["num"].shape
    M = int(plan64.info.max_kv_blocks)
    rng = np.random.default_rng(5)
    idx = np.full((T, N, M), -1, dtype=np.int32)
    num = np.zeros((T, N), dtype=np.int32)
    clean = np.full((T, N, M), -1, dtype=np.int32)
    clean_num = np.zeros((T, N), dtype=np.int32)
    for t in range(T):
        s, g, _ = table[t]
        n64 = orc.kv_block_count(g, 64)
        for n in range(N):
            size = int(rng.integers(1, n64 + 1))
            chosen = sorted(rng.choice(n64, size=size, replace=False).tolist())
            row = list(chosen)
            if (t + n) % 4 == 1 and len(row) < M:
                row.insert(int(rng.integers(0, len(row) + 1)), -1)   # an unused slot
            idx[t, n, :len(row)] = row
            num[t, n] = len(row)
            clean[t, n, :len(chosen)] = chosen
            clean_num[t, n] = len(chosen)
    q_r, k_r, v_r = (parity.to_device(gpu[n], w.dtype) for n in ("q_r", "k_r", "v_r"))
    o64 = _kv64_run(w, q_r, k_r, v_r, idx, num, gpu["scale"])
    rbits = [orc.rearrange(p, x) for x in bits]
    got = dict(idx=clean, num=clean_num, scale=gpu["scale"], o_r=o64)
    parity.check_attention(p, w, rbits, got, block_kv=64)


@pytest.mark.parametrize("name", KV64 + ["batch2_d64", "dense", "s_one"])
def test_kv64_selection_small_full_parity(name):
    """blockShape 128 x 64 end to end (reading R26): K pooled over 64-row key blocks,
    those ranked against the 128-row query means, the attention on that selection."""
    w = SMALL[name]
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, block_kv=64)
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    qbars, kbars = parity.oracle_pooled(p, w, rbits, 64)
    parity.check_pooled(p, qbars, kbars, gpu)
    stats = parity.check_selection(p, qbars, kbars, gpu, block_kv=64)
    assert stats["near_tie"] <= max(1, stats["rows"] // 100)
    parity.check_attention(p, w, rbits, gpu, block_kv=64)
    if name == "dense":
        assert np.all(gpu["num"] == orc.kv_block_count(p.geoms[0], 64))


def test_kv64_recompute_forward_and_noalloc_equal_the_step_calls():
    w = SMALL["tnd_gqa_small"]
    bits = synth.generate_qkv(w)
    a = parity.run_gpu(w, bits, block_kv=64)
    b = parity.run_gpu(w, bits, pool_mode="recompute", block_kv=64)
    assert np.array_equal(a["pooled_k"], b["pooled_k"])
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["num"], b["num"])
    assert np.array_equal(a["o"], b["o"])
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, block_kv=64)
    bufs = rf.Buffers(plan)
    q, k, v = (parity.to_device(x, w.dtype) for x in bits)
    out = rf.forward(plan, q, k, v, bufs)
    torch.cuda.synchronize()
    assert np.array_equal(parity.to_bits(out), a["o"])


def test_kv64_user_call_with_host_tensors_equals_the_step_calls():
    """rainfusion_attention(block_kv=64) on host tensors (the chunked host pipeline)
    gives the step calls' output bit for bit."""
    w = SMALL["batch2_d64"]
    bits = synth.generate_qkv(w)
    steps = parity.run_gpu(w, bits, block_kv=64)
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in bits)
    out = rf.rainfusion_attention(q, k, v, parity.seqs_of(w), sparsity=w.sparsity, block_kv=64)
    assert np.array_equal(out.view(torch.int16).numpy().view(np.uint16), steps["o"])


@pytest.mark.parametrize("name,s", [("wan", None), ("aligned", 0.8)])
def test_kv64_full_size_parity(name, s):
    """The 128 x 64 path at full size in the bench's launch configuration: 64-row K
    means and the selection over every row, the attention on sampled items."""
    w = synth.workload(name, s)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, block_kv=64)
    rbits = [orc.rearrange(p, x) for x in bits]
    qbars, kbars = parity.oracle_pooled(p, w, rbits, 64)
    parity.check_pooled(p, qbars, kbars, gpu)
    stats = parity.check_selection(p, qbars, kbars, gpu, block_kv=64)
    assert stats["near_tie"] <= max(1, stats["rows"] // 1000), stats
    items = parity.sample_items(p, np.random.default_rng(8), per_kind=3)
    parity.check_attention(p, w, rbits, gpu, items, block_kv=64)


# ------------------------------------------------------------------------------------------
# Precision "fp8" (user guide "Configuration": precision "fp8"; reading R24): E4M3 Q K^T as
# in mix, E4M3 V' on power-of-two scales, probabilities rounded to E4M3 for P V.  Codes and
# exponents bit-exact; output within the oracle's bound on the probability rounding.
# ------------------------------------------------------------------------------------------

FP8_SMALL = ["ragged_d128", "tnd_gqa_small", "dense", "s_one", "all_promoted"]


@pytest.mark.parametrize("name", FP8_SMALL)
def test_fp8_small_parity(name):
    w = SMALL[name]
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, precision="fp8")
    parity.check_permutation(p, bits, gpu)
    rbits = [orc.rearrange(p, x) for x in bits]
    parity.check_fp8_quantization(p, w, rbits, gpu)
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    parity.check_pooled(p, qbars, kbars, gpu)             # pooling still reads the 16-bit values
    parity.check_selection(p, qbars, kbars, gpu)
    err = parity.check_fp8_attention(p, w, rbits, gpu)
    print(f"fp8 {name}: {err}")


@pytest.mark.parametrize("name,s", [("wan", None), ("tnd_gqa", None), ("aligned", 0.8)])
def test_fp8_full_size_parity(name, s):
    w = synth.workload(name, s)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    gpu = parity.run_gpu(w, bits, precision="fp8")
    rbits = [orc.rearrange(p, x) for x in bits]
    parity.check_fp8_quantization(p, w, rbits, gpu)
    items = parity.sample_items(p, np.random.default_rng(11), per_kind=3)
    err = parity.check_fp8_attention(p, w, rbits, gpu, items)
    print(f"fp8 {name}: {err}")
    # the quantization error itself, against the unquantized oracle: reported, bounded loosely
    err = parity.check_attention(p, w, rbits, gpu, items, check=False)
    assert err["rel_l2"] <= 0.1, err


def test_fp8_quantize_entry_point_equals_fused_quantization():
    w = SMALL["tnd_gqa_small"]
    bits = synth.generate_qkv(w)
    fused = parity.run_gpu(w, bits, precision="fp8")
    plan = fused["plan"]
    b = rf.Buffers(plan)
    q_r, k_r, v_r = (parity.to_device(fused[n], w.dtype) for n in ("q_r", "k_r", "v_r"))
    rf.quantize(plan, q_r, k_r, v_r, b.ws)
    torch.cuda.synchronize()
    alone = parity.mix_buffers(plan, b.ws)
    alone.update(parity.fp8_buffers(plan, b.ws, parity.problem(w)))
    for key in ("q8", "k8", "q_scale", "k_scale", "v8_raw", "v_exp"):
        assert np.array_equal(alone[key], fused[key]), key
