"""Pins for the oracle's block-sparse attention (CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import rainfusion as rf


def _dense_sdpa(q, k, v, scale, mask=None):
    """Library dense attention in float64 (rows on axis -2)."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=None if mask is None else torch.from_numpy(mask), scale=scale).numpy()


def _problem(seqs, n1=2, n2=2, d=16, s=0.8, layout="BNSD", batch=1):
    return rf.make_problem(layout, batch, seqs, n1, n2, d, s)


def _inputs(p, seed=0, total_rows=None):
    rng = np.random.default_rng(seed)
    if p.layout == "BNSD":
        L = p.geoms[0].length
        mk = lambda n: rng.standard_normal((p.batch, n, L, p.d))
    else:
        T = sum(g.length for g in p.geoms)
        mk = lambda n: rng.standard_normal((T, n, p.d))
    return mk(p.n1), mk(p.n2), mk(p.n2)


def test_sparsity_zero_equals_dense_attention():
    # 100 text rows + (8,16,32) video: the last prefix block is partial, 32 video blocks
    p = _problem([(100, 8, 16, 32)], s=0.0)
    q, k, v = _inputs(p)
    scale = 1 / math.sqrt(p.d)
    out = rf.run_path(p, q, k, v, scale)
    assert np.all(out["num"] == p.geoms[0].n_blocks)
    ref = _dense_sdpa(q, k, v, scale)
    assert np.max(np.abs(out["o"] - ref)) < 1e-12


def test_sparsity_zero_equals_dense_attention_ragged_gqa_tnd():
    p = _problem([(40, 3, 13, 21), (7, 2, 16, 24)], n1=4, n2=2, d=8, s=0.0, layout="TND")
    q, k, v = _inputs(p, seed=1)
    scale = 0.3
    out = rf.run_path(p, q, k, v, scale)
    off = 0
    for g in p.geoms:
        for n in range(p.n1):
            ref = _dense_sdpa(q[off:off + g.length, n], k[off:off + g.length, n // 2],
                              v[off:off + g.length, n // 2], scale)
            assert np.max(np.abs(out["o"][off:off + g.length, n] - ref)) < 1e-12
        off += g.length


def test_block_sparse_equals_masked_formula():
    # Softmax(scale*QK^T + mask)V with the additive mask built from selectIdx by loops
    p = _problem([(100, 8, 16, 32)], s=0.8)
    g = p.geoms[0]
    q, k, v = _inputs(p, seed=2)
    scale = 1 / math.sqrt(p.d)
    out = rf.run_path(p, q, k, v, scale)
    q_r, k_r, v_r, idx, num = out["q_r"], out["k_r"], out["v_r"], out["idx"], out["num"]
    for n in range(p.n1):
        mask = np.full((g.length, g.length), -np.inf)
        for qb in range(g.n_blocks):
            qrows = rf.block_rows(g, qb)
            for b in idx[qb, n, :num[qb, n]]:
                krows = rf.block_rows(g, int(b))
                mask[qrows.start:qrows.stop, krows.start:krows.stop] = 0.0
        ref = _dense_sdpa(q_r[0, n], k_r[0, n], v_r[0, n], scale, mask)
        assert np.max(np.abs(out["o_r"][0, n] - ref)) < 1e-12
    # and the selection really is sparse
    assert num[g.n_pb + g.ns:].max() < g.n_blocks


def test_element_by_element_softmax_loops():
    # tiny geometry with hand-made key block lists, against pure-Python loops
    g = rf.geometry(50, 1, 8, 40, 0.8)      # Lp = 50 + 64 promoted = 114, 2 sparse blocks
    rng = np.random.default_rng(3)
    d = 4
    q = rng.standard_normal((g.length, d))
    k = rng.standard_normal((g.length, d))
    v = rng.standard_normal((g.length, d))
    scale = 0.7
    for qb, blocks in [(0, [0]), (1, [0, 2]), (2, [1]), (1, [0, 1, 2, -1, -1])]:
        got = rf.attend_query_block(q, k, v, g, qb, blocks, scale)
        qrows = list(rf.block_rows(g, qb))
        keys = [r for b in blocks if b >= 0 for r in rf.block_rows(g, b)]
        for a, r in enumerate(qrows):
            logits = []
            for c in keys:
                s = 0.0
                for e in range(d):
                    s += q[r, e] * k[c, e]
                logits.append(scale * s)
            mx = max(logits)
            ex = [math.exp(x - mx) for x in logits]
            den = sum(ex)
            for e in range(d):
                num = 0.0
                for w, c in zip(ex, keys):
                    num += w * v[c, e]
                assert abs(got[a, e] - num / den) < 1e-12


def test_constant_values_give_constant_output():
    p = _problem([(64, 8, 16, 32)], s=0.9)
    q, k, v = _inputs(p, seed=4)
    v[...] = 1.0
    out = rf.run_path(p, q, k, v, 0.125)
    assert np.max(np.abs(out["o"] - 1.0)) < 1e-12


def test_text_order_does_not_change_video_outputs():
    p = _problem([(96, 8, 16, 32)], s=0.8)
    g = p.geoms[0]
    q, k, v = _inputs(p, seed=5)
    a = rf.run_path(p, q, k, v, 0.25)["o"]
    perm = np.random.default_rng(6).permutation(96)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for x in (q2, k2, v2):
        x[:, :, :96] = x[:, :, perm]
    b = rf.run_path(p, q2, k2, v2, 0.25)["o"]
    assert np.max(np.abs(a[:, :, 96:] - b[:, :, 96:])) < 1e-12
    assert np.max(np.abs(a[:, :, perm] - b[:, :, :96])) < 1e-12


def test_kept_flops_dense_closed_form():
    p = _problem([(100, 8, 16, 32)], s=0.0)
    g = p.geoms[0]
    q, k, v = _inputs(p)
    out = rf.run_path(p, q, k, v, 0.25)
    assert rf.kept_flops(p, out["idx"], out["num"]) == 4 * p.d * g.length * g.length * p.n1


# --------------------------------------------------------------------------------------
# Key/value blocks of 64 rows under 128-row query blocks ([API] blockShape X x Y)
# --------------------------------------------------------------------------------------

@pytest.mark.parametrize("geom", [(100, 1, 16, 16), (40, 1, 16, 16), (64, 2, 16, 16), (0, 2, 16, 24),
                                  (300, 0, 0, 0), (77, 9, 17, 33)])
def test_kv64_blocks_partition_the_sequence_and_nest_in_128_blocks(geom):
    g = rf.geometry(*geom, 0.8)
    n64 = rf.kv_block_count(g, 64)
    rows = [r for b in range(n64) for r in rf.kv_block_rows(g, b, 64)]
    assert rows == list(range(g.length))                  # a partition, in order
    assert n64 == -(-g.lp // 64) + 2 * g.nb
    assert rf.kv_block_count(g, 128) == g.n_blocks
    for b in range(g.n_blocks):                           # block_kv = 128 is block_rows itself
        assert rf.kv_block_rows(g, b, 128) == rf.block_rows(g, b)
    # every 128-row block is the union of the 64-row blocks inside it
    for b in range(g.n_blocks):
        r = rf.block_rows(g, b)
        inside = [c for c in range(n64) if rf.kv_block_rows(g, c, 64).start in r]
        assert [x for c in inside for x in rf.kv_block_rows(g, c, 64)] == list(r)
        assert 1 <= len(inside) <= 2


def test_kv64_attention_equals_128_attention_on_the_same_rows():
    g = rf.geometry(100, 1, 16, 16, 0.5)                 # partial 100-row prefix block
    rng = np.random.default_rng(21)
    q, k, v = (rng.standard_normal((g.length, 32)) for _ in range(3))
    # blocks 0 (prefix, rows 0..99) and 2 (rows 228..355) at 128 rows are 64-row blocks
    # 0, 1 (rows 0..63, 64..99) and 4, 5 (rows 228..291, 292..355)
    a = rf.attend_query_block(q, k, v, g, 1, [0, 2], 0.2)
    b = rf.attend_query_block(q, k, v, g, 1, [0, 1, 4, 5], 0.2, block_kv=64)
    assert np.max(np.abs(a - b)) < 1e-13
    # a single 64-row block: exactly the softmax over those rows
    c = rf.attend_query_block(q, k, v, g, 2, [3], 0.2, block_kv=64)
    rows = list(range(164, 228))
    x = 0.2 * q[228:356] @ k[rows].T
    w = np.exp(x - x.max(axis=1, keepdims=True))
    assert np.max(np.abs(c - (w / w.sum(axis=1, keepdims=True)) @ v[rows])) < 1e-13
