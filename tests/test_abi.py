"""C-ABI checks that need no GPU: the library loads, exports what include/rf.h
declares, validates arguments on the host, and derives the oracle's geometry."""
import ctypes
import os
import re

import numpy as np
import pytest

from block_sparse_video_rearrange_b200 import rf, synth
from oracle import rainfusion as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "rf.h")).read()
    return sorted(set(re.findall(r"RF_API\s+[\w\s\*]+?\b(rf_\w+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 12
    lib = ctypes.CDLL(rf.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(rf.EXPORTED)


def test_status_strings():
    for code in range(7):
        assert rf.lib().rf_status_string(code)
    assert rf.lib().rf_status_string(99) == b"unknown status"


@pytest.mark.parametrize("kwargs,status", [
    (dict(n1=6, n2=4), 1),                     # N1 = G * N2 violated
    (dict(block_q=0), 1),                      # blockShape entries must be > 0
    (dict(block_kv=-3), 1),
    (dict(block_q=64), 6),                     # valid per the pages, not built here
    (dict(sparsity=1.5), 1),
    (dict(sparsity=float("nan")), 1),
    (dict(sparsity=-0.1), 1),
    (dict(d=96), 6),
    (dict(d=0), 1),
    (dict(batch=0), 1),
    (dict(batch=33), 1),
    (dict(seqs=[(0, 0, 0, 0)]), 1),            # empty sequence
    (dict(seqs=[(-1, 2, 8, 8)]), 1),
    (dict(seqs=[(0, 2, 8, 8), (0, 2, 8, 8)]), 1),  # BNSD takes one geometry
    (dict(layout="TND", batch=2), 1),
    (dict(seqs=[(0, 33, 64, 128)]), 6),       # 2,112 sparse blocks: beyond the 2,048 the kernels take
])
def test_plan_validation(kwargs, status):
    args = dict(seqs=[(128, 9, 16, 32)], n1=2, n2=2, d=64, layout="BNSD", dtype="bf16", sparsity=0.8,
                batch=1, block_q=128, block_kv=128)
    args.update(kwargs)
    with pytest.raises(rf.RfError) as e:
        rf.Plan(**args)
    assert e.value.status == status


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_plan_geometry_matches_oracle(name):
    w = synth.WORKLOADS[name]
    seqs = [(s.prefix_len, s.t, s.h, s.w) for s in w.seqs]
    plan = rf.Plan(seqs, w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch)
    prob = orc.make_problem(w.layout, w.batch, seqs, w.n1, w.n2, w.d, w.sparsity)
    assert plan.info.t_qblk == prob.t_qblk
    assert plan.info.max_kv_blocks == prob.max_kv_blocks
    row = 0
    for si, g in zip(plan.seq_info, prob.geoms):
        assert (si.length, si.lp, si.sparse, si.promoted) == (g.length, g.lp, g.sparse, g.promoted)
        assert (si.n_pb, si.nb, si.ns, si.k, si.dense) == (g.n_pb, g.nb, g.ns, g.k, int(g.dense))
        if w.layout == "TND":
            assert si.row_offset == row
        row += g.length
    assert plan.info.rows_total == (prob.geoms[0].length if w.layout == "BNSD" else row)


@pytest.mark.parametrize("s", [0.0, 0.5, 0.8, 0.9, 1.0, 0.37])
def test_keep_count_matches_oracle(s):
    for nb in (32, 36, 157, 189, 465, 630, 2048):
        t, h, w = 1, 8, nb * 16   # nb blocks of two 8x8 tiles
        plan = rf.Plan([(0, t, h, w)], 1, 1, 64, sparsity=s)
        assert plan.seq_info[0].nb == nb
        assert plan.seq_info[0].k == orc.keep_count(nb, s)


def test_keep_count_of_the_plan_equals_the_pinned_values():
    """The host plan's k against the hand-worked values of reading R4 (not the oracle)."""
    from tests.test_oracle_geometry import PINNED_K
    for (p, t, h, w, s, nb, k) in PINNED_K:
        plan = rf.Plan([(p, t, h, w)], 1, 1, 128, sparsity=s)
        assert (plan.seq_info[0].nb, plan.seq_info[0].k) == (nb, k), (p, t, h, w, s)


def test_host_validation_runs_before_any_device_call():
    plan = rf.Plan([(128, 9, 16, 32)], 2, 2, 64)
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced: validation fails first
    # bf16 allows only the fp32 softmax (inner_precise 0)
    st = rf.lib().rf_block_sparse_attn(plan.handle, fake, fake, fake, fake, fake, ctypes.c_float(0.125), 1,
                                       ctypes.c_void_p(2 << 20), fake, plan.workspace_bytes, None)
    assert st == 1
    st = rf.lib().rf_block_sparse_attn(plan.handle, fake, fake, fake, fake, fake, ctypes.c_float(-1.0), 0,
                                       ctypes.c_void_p(2 << 20), fake, plan.workspace_bytes, None)
    assert st == 1
    # an undersized workspace is rejected before the device is touched
    st = rf.lib().rf_rearrange(plan.handle, fake, fake, fake, ctypes.c_void_p(2 << 20), ctypes.c_void_p(3 << 20),
                               ctypes.c_void_p(4 << 20), fake, 16, None)
    assert st == 3
    # misaligned tensors
    st = rf.lib().rf_inverse_rearrange(plan.handle, ctypes.c_void_p((1 << 20) + 2), fake, None)
    assert st == 1


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
def test_kernel_index_math_equals_oracle_permutation(name):
    """The row mapping the CUDA kernels execute (run here on the host) against the
    oracle's permutation, which is built by sorting keys."""
    w = synth.WORKLOADS[name]
    seqs = [(s.prefix_len, s.t, s.h, s.w) for s in w.seqs]
    plan = rf.Plan(seqs, w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch)
    for i, s in enumerate(seqs):
        g = orc.geometry(*s, w.sparsity)
        assert np.array_equal(plan.permutation(i), orc.permutation(g))


@pytest.mark.parametrize("s", [(77, 9, 17, 33), (0, 6, 24, 40), (200, 10, 19, 21), (5, 3, 7, 9), (1, 2, 8, 8),
                               (0, 1, 3, 3), (64, 4, 31, 9), (384, 21, 24, 40)])
def test_kernel_index_math_ragged_cases(s):
    plan = rf.Plan([s], 1, 1, 64)
    assert np.array_equal(plan.permutation(0), orc.permutation(orc.geometry(*s, 0.8)))


# ---------------- frame-pair token order (rf_plan_create_ex) ----------------

@pytest.mark.parametrize("s", [(512, 21, 30, 52), (256, 62, 24, 42), (128, 9, 16, 32), (384, 21, 24, 40),
                               (77, 9, 17, 33), (0, 6, 24, 40), (5, 3, 7, 9), (1, 2, 8, 8), (0, 1, 3, 3),
                               (64, 4, 31, 9), (0, 8, 16, 16)])
def test_frame_pair_index_math_equals_oracle_permutation(s):
    """The kernels' frame-pair row mapping (run on the host) against the oracle's
    key sort, bit for bit, with the counts unchanged from the tile order."""
    plan = rf.Plan([s], 1, 1, 64, order="frame_pair")
    g = orc.geometry(*s, 0.8, "frame_pair")
    assert np.array_equal(plan.permutation(0), orc.permutation(g))
    tile = rf.Plan([s], 1, 1, 64)
    a, b = plan.seq_info[0], tile.seq_info[0]
    assert (a.length, a.lp, a.sparse, a.promoted, a.n_pb, a.nb, a.ns, a.k) == \
           (b.length, b.lp, b.sparse, b.promoted, b.n_pb, b.nb, b.ns, b.k)


def test_frame_pair_tnd_sequences_each_follow_the_order():
    seqs = [(256, 13, 32, 48), (384, 21, 24, 40)]
    plan = rf.Plan(seqs, 32, 8, 128, "TND", "fp16", 0.8, order="frame_pair")
    for i, s in enumerate(seqs):
        assert np.array_equal(plan.permutation(i), orc.permutation(orc.geometry(*s, 0.8, "frame_pair")))


def _create_ex(opts, d=64):
    arr = (rf.SeqGeom * 1)(rf.SeqGeom(128, 9, 16, 32))
    h = ctypes.c_void_p()
    st = rf.lib().rf_plan_create_ex(arr, 1, 1, 2, 2, d, 0, 0, ctypes.c_double(0.8), 128, 128,
                                    ctypes.byref(opts) if opts is not None else None, ctypes.byref(h))
    if h.value:
        rf.lib().rf_plan_destroy(h)
    return st, bool(h.value)


def test_plan_options_are_validated():
    assert _create_ex(None) == (0, True)                          # NULL options: the defaults
    assert _create_ex(rf.PlanOptions(0, 0)) == (0, True)
    assert _create_ex(rf.PlanOptions(7, 0)) == (1, False)         # unknown token order
    assert _create_ex(rf.PlanOptions(0, 9)) == (1, False)         # unknown precision
    bad = rf.PlanOptions(0, 0)
    bad.reserved[3] = 1
    assert _create_ex(bad) == (1, False)                          # reserved fields must be zero
    assert _create_ex(rf.PlanOptions(0, 2), d=128) == (0, True)   # fp8 (FP8 P V as well)
    assert _create_ex(rf.PlanOptions(0, 2), d=64) == (6, False)   # fp8: head dim 128 only
    assert _create_ex(rf.PlanOptions(0, 1), d=64) == (6, False)   # mix: head dim 128 only
    assert _create_ex(rf.PlanOptions(1, 1), d=128) == (0, True)
    with pytest.raises(ValueError):
        rf.Plan([(128, 9, 16, 32)], 2, 2, 64, order="zigzag")
    with pytest.raises(ValueError):
        rf.Plan([(128, 9, 16, 32)], 2, 2, 128, precision="int4")


@pytest.mark.parametrize("layout,seqs,n1,n2", [("BNSD", [(512, 21, 30, 52)], 40, 40),
                                               ("TND", [(256, 13, 32, 48), (384, 21, 24, 40)], 32, 8)])
def test_mix_precision_workspace_layout(layout, seqs, n1, n2):
    """The E4M3 copies and scales sit after the native workspace, 256-byte aligned,
    sized one byte per element of Q' / K' and one float per (head, query block)."""
    nat = rf.Plan(seqs, n1, n2, 128, layout, "bf16", 0.8)
    mix = rf.Plan(seqs, n1, n2, 128, layout, "bf16", 0.8, precision="mix")
    a, b = nat.info, mix.info
    assert (a.precision, b.precision) == (0, 1)
    assert a.ws_q8 == a.ws_k8 == a.ws_q_scale == a.ws_k_scale == -1
    rows, t = int(b.rows_total), int(b.t_qblk)
    assert b.ws_q8 >= a.workspace_bytes and b.ws_q8 % 256 == 0
    assert b.ws_k8 >= b.ws_q8 + rows * n1 * 128 and b.ws_k8 % 256 == 0
    assert b.ws_q_scale >= b.ws_k8 + rows * n2 * 128
    assert b.ws_k_scale >= b.ws_q_scale + n1 * t * 4
    assert b.workspace_bytes >= b.ws_k_scale + n2 * t * 4
    for f in ("rows_total", "t_qblk", "max_kv_blocks", "pooled_blocks", "ws_pooled_q", "ws_pooled_k"):
        assert getattr(a, f) == getattr(b, f), f


@pytest.mark.parametrize("layout,seqs,n1,n2", [("BNSD", [(512, 21, 30, 52)], 40, 40),
                                               ("TND", [(256, 13, 32, 48), (384, 21, 24, 40)], 32, 8)])
def test_fp8_precision_workspace_layout(layout, seqs, n1, n2):
    """Precision fp8: the mix regions, then the transposed E4M3 V' (one byte per
    element, [n2][t_qblk][128][128]) and its int32 exponents [n2][t_qblk]."""
    mix = rf.Plan(seqs, n1, n2, 128, layout, "bf16", 0.8, precision="mix")
    f8 = rf.Plan(seqs, n1, n2, 128, layout, "bf16", 0.8, precision="fp8")
    a, b = mix.info, f8.info
    assert b.precision == 2
    assert a.ws_v8 == a.ws_v_exp == -1
    for f in ("ws_q8", "ws_k8", "ws_q_scale", "ws_k_scale"):
        assert getattr(a, f) == getattr(b, f), f
    t = int(b.t_qblk)
    assert b.ws_v8 >= a.workspace_bytes and b.ws_v8 % 256 == 0
    assert b.ws_v_exp >= b.ws_v8 + n2 * t * 128 * 128 and b.ws_v_exp % 256 == 0
    assert b.workspace_bytes >= b.ws_v_exp + n2 * t * 4
    with pytest.raises(rf.RfError) as e:
        rf.Plan(seqs, n1, n2, 128, layout, "bf16", 0.8, precision="fp8", block_kv=64)
    assert e.value.status == 6


def test_generic_quantize_entry_point_validates_on_the_host():
    fake = ctypes.c_void_p(1 << 20)
    native = rf.Plan([(128, 9, 16, 32)], 2, 2, 128)
    assert rf.lib().rf_quantize(native.handle, fake, fake, fake, fake, native.workspace_bytes, None) == 1
    f8 = rf.Plan([(128, 9, 16, 32)], 2, 2, 128, precision="fp8")
    assert rf.lib().rf_quantize(f8.handle, fake, fake, None, fake, f8.workspace_bytes, None) == 1   # needs V
    assert rf.lib().rf_quantize(f8.handle, fake, fake, fake, fake, 16, None) == 3   # workspace too small


def test_quantize_needs_a_mix_plan():
    plan = rf.Plan([(128, 9, 16, 32)], 2, 2, 128)
    fake = ctypes.c_void_p(1 << 20)
    st = rf.lib().rf_quantize_qk(plan.handle, fake, fake, fake, plan.workspace_bytes, None)
    assert st == 1


@pytest.mark.parametrize("layout,seqs,n1,n2,d", [("BNSD", [(512, 21, 30, 52)], 40, 40, 128),
                                                 ("TND", [(256, 13, 32, 48), (384, 21, 24, 40)], 32, 8, 128),
                                                 ("BNSD", [(128, 9, 16, 32)], 2, 2, 64)])
def test_mxfp4_precision_workspace_layout(layout, seqs, n1, n2, d):
    """The MXFP4 copies of Q', K', V' sit after the native workspace, 256-byte aligned:
    at head dim 128 as E4M3 carriers (one byte per element of Q' and K' in their layouts,
    V' transposed per block; no scales), else two bytes per element each."""
    nat = rf.Plan(seqs, n1, n2, d, layout, "bf16", 0.8)
    mx = rf.Plan(seqs, n1, n2, d, layout, "bf16", 0.8, precision="mxfp4")
    a, b = nat.info, mx.info
    assert b.precision == 3
    assert a.ws_q_mx == a.ws_k_mx == a.ws_v_mx == -1
    assert b.ws_q_scale == b.ws_k_scale == b.ws_v_exp == -1
    rows = int(b.rows_total)
    if d == 128:
        t = int(b.t_qblk)
        assert b.ws_q_mx == b.ws_k_mx == b.ws_v_mx == -1
        assert b.ws_q8 >= a.workspace_bytes and b.ws_q8 % 256 == 0
        assert b.ws_k8 >= b.ws_q8 + rows * n1 * d and b.ws_k8 % 256 == 0
        assert b.ws_v8 >= b.ws_k8 + rows * n2 * d and b.ws_v8 % 256 == 0
        assert b.workspace_bytes >= b.ws_v8 + n2 * t * 128 * d
        return
    assert b.ws_q8 == b.ws_k8 == b.ws_v8 == -1
    assert b.ws_q_mx >= a.workspace_bytes and b.ws_q_mx % 256 == 0
    assert b.ws_k_mx >= b.ws_q_mx + rows * n1 * d * 2 and b.ws_k_mx % 256 == 0
    assert b.ws_v_mx >= b.ws_k_mx + rows * n2 * d * 2 and b.ws_v_mx % 256 == 0
    assert b.workspace_bytes >= b.ws_v_mx + rows * n2 * d * 2
    for f in ("rows_total", "t_qblk", "max_kv_blocks", "pooled_blocks", "ws_pooled_q", "ws_pooled_k"):
        assert getattr(a, f) == getattr(b, f), f


def test_mxfp4_options_and_quantize_entry_point():
    assert _create_ex(rf.PlanOptions(0, 3), d=64) == (0, True)
    assert _create_ex(rf.PlanOptions(1, 3), d=128) == (0, True)
    fake = ctypes.c_void_p(1 << 20)
    native = rf.Plan([(128, 9, 16, 32)], 2, 2, 128)
    mix = rf.Plan([(128, 9, 16, 32)], 2, 2, 128, precision="mix")
    for plan in (native, mix):   # another precision: rejected before any device work
        assert rf.lib().rf_quantize_mx(plan.handle, fake, fake, fake, fake, plan.workspace_bytes, None) == 1
    mx = rf.Plan([(128, 9, 16, 32)], 2, 2, 128, precision="mxfp4")
    assert rf.lib().rf_quantize_qk(mx.handle, fake, fake, fake, mx.workspace_bytes, None) == 1
    assert rf.lib().rf_quantize_mx(mx.handle, fake, fake, None, fake, mx.workspace_bytes, None) == 1
    unaligned = ctypes.c_void_p((1 << 20) + 8)
    assert rf.lib().rf_quantize_mx(mx.handle, fake, fake, unaligned, fake, mx.workspace_bytes, None) == 1


def test_block_shape_128_by_64_plan():
    """blockShape 128 x 64: key blocks of 64 rows (native precision only); the
    selectIdx width counts them; the key-side selection counts and the 64-row K
    means in the workspace follow the oracle's reading; selection and the
    whole-path call pass host validation (and stop at the device check here)."""
    seqs = [(100, 9, 16, 32)]        # Lp = 100: two 64-row prefix blocks, the second partial
    p128 = rf.Plan(seqs, 2, 2, 128)
    p64 = rf.Plan(seqs, 2, 2, 128, block_kv=64)
    g = orc.geometry(100, 9, 16, 32, 0.8)
    assert int(p128.info.max_kv_blocks) == g.n_blocks
    assert int(p64.info.max_kv_blocks) == orc.kv_block_count(g, 64) == 2 + 2 * g.nb
    assert int(p64.info.t_qblk) == int(p128.info.t_qblk)          # query blocks stay 128 rows
    assert p64.select_shapes()[0][2] == int(p64.info.max_kv_blocks)
    for bq, bkv in ((64, 128), (128, 32), (64, 64), (256, 128)):
        with pytest.raises(rf.RfError) as e:
            rf.Plan(seqs, 2, 2, 128, block_q=bq, block_kv=bkv)
        assert e.value.status == 6
    for precision in ("mix", "mxfp4"):
        with pytest.raises(rf.RfError) as e:
            rf.Plan(seqs, 2, 2, 128, block_kv=64, precision=precision)
        assert e.value.status == 6
    kb = orc.key_blocks(g, 64)
    si = p64.seq_info[0]
    assert (int(si.n_pb_kv), int(si.nb_kv), int(si.ns_kv), int(si.k_kv)) == (kb.n_pb, kb.nb, kb.ns, kb.k) \
        == (2, 2 * g.nb, 8, 15)
    si = p128.seq_info[0]
    assert (int(si.n_pb_kv), int(si.nb_kv), int(si.ns_kv), int(si.k_kv)) == (g.n_pb, g.nb, g.ns, g.k)
    assert int(p128.info.pooled_k_blocks) == int(p128.info.pooled_blocks) == g.nb
    assert int(p64.info.pooled_k_blocks) == 2 * int(p64.info.pooled_blocks) == 2 * g.nb
    # the K means region holds the 64-row means, the scores [N1][nb][2 nb]
    extra = 2 * g.nb * 128 * 4 + 2 * g.nb * g.nb * 4        # n2 * nb more means, n1 * nb * nb more scores
    assert abs(p64.workspace_bytes - p128.workspace_bytes - extra) < 3 * 256   # regions start 256-aligned
    fake = ctypes.c_void_p(1 << 20)
    lib = rf.lib()
    import torch
    if torch.cuda.is_available():         # on a GPU the selection itself is tested in the parity suite
        return
    assert lib.rf_pool_select(p64.handle, fake, fake, fake, fake, fake, p64.workspace_bytes, 0, None) == 2
    f = [ctypes.c_void_p((1 << 24) + (i << 20)) for i in range(11)]   # distinct, 16-byte aligned
    assert lib.rf_forward(p64.handle, *f[:8], ctypes.c_float(0.1), *f[8:], p64.workspace_bytes, None) == 2
    assert lib.rf_pool_select_noalloc(p64.handle, fake, fake, fake, fake, None) == 2


# ---------------- randomized geometry sweep (host-side index math) ----------------

from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(p=st.integers(0, 400), t=st.integers(0, 7), h=st.integers(0, 40), w=st.integers(0, 40),
       order=st.sampled_from(["tile", "frame_pair"]))
def test_random_geometries_match_the_oracle(p, t, h, w, order):
    """For random (prefix, t, h, w) and both token orders: the plan's sizes, the 64-row
    key-block count and the row mapping the kernels execute all equal the oracle's."""
    if p + t * h * w == 0:
        return
    g = orc.geometry(p, t, h, w, 0.8, order)
    plan = rf.Plan([(p, t, h, w)], 1, 1, 64, order=order)
    si = plan.seq_info[0]
    assert (int(si.length), int(si.lp), int(si.sparse), int(si.n_pb), int(si.nb), int(si.ns), int(si.k),
            bool(si.dense)) == (g.length, g.lp, g.sparse, g.n_pb, g.nb, g.ns, g.k, g.dense)
    assert np.array_equal(plan.permutation(0), orc.permutation(g))
    p64 = rf.Plan([(p, t, h, w)], 1, 1, 64, order=order, block_kv=64)
    assert int(p64.info.max_kv_blocks) == orc.kv_block_count(g, 64)
    kb, si = orc.key_blocks(g, 64), p64.seq_info[0]
    assert (int(si.n_pb_kv), int(si.nb_kv), int(si.ns_kv), int(si.k_kv)) == (kb.n_pb, kb.nb, kb.ns, kb.k)
