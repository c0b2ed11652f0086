"""Pins for the oracle's pooling and block selection (CPU only)."""
import itertools

import numpy as np
import pytest

from oracle import rainfusion as rf


def test_topk_equals_best_subset_by_enumeration():
    rng = np.random.default_rng(1)
    for trial in range(30):
        nb = int(rng.integers(4, 11))
        k = int(rng.integers(0, nb + 1))
        # coarse values so that ties occur
        scores = rng.integers(-3, 4, size=nb).astype(np.float64)
        best = None
        for subset in itertools.combinations(range(nb), k):
            # larger total score wins; among equal totals the lexicographically
            # smallest index set wins (lower block index on ties)
            key = (-sum(scores[list(subset)]), subset)
            if best is None or key < best:
                best = key
        assert sorted(rf.topk_blocks(scores, k)) == list(best[1])


def test_topk_equals_pairwise_rank_definition():
    rng = np.random.default_rng(2)
    for trial in range(20):
        nb = int(rng.integers(30, 80))
        k = int(rng.integers(0, nb))
        scores = np.round(rng.standard_normal(nb), 1)
        beats = lambda a, b: scores[a] > scores[b] or (scores[a] == scores[b] and a < b)
        expect = [j for j in range(nb) if sum(beats(o, j) for o in range(nb) if o != j) < k]
        assert sorted(rf.topk_blocks(scores, k)) == expect


def test_block_means_brute_force_and_constant_blocks():
    g = rf.geometry(100, 8, 16, 32, 0.8)            # Lp = 100 (partial prefix block), 32 blocks
    rng = np.random.default_rng(3)
    x = rng.standard_normal((g.length, 5))
    m = rf.block_means(x, g)
    for i in range(g.nb):
        for c in range(5):
            s = 0.0
            for r in range(g.lp + 128 * i, g.lp + 128 * i + 128):
                s += x[r, c]
            assert abs(m[i, c] - s / 128) < 1e-12
    x[g.lp + 128 * 3: g.lp + 128 * 4] = 2.5
    assert np.all(rf.block_means(x, g)[3] == 2.5)


def _random_select(p, t, h, w, s, n1=2, n2=2, d=8, seed=4):
    g = rf.geometry(p, t, h, w, s)
    rng = np.random.default_rng(seed)
    qbar = rng.standard_normal((n1, g.nb, d))
    kbar = rng.standard_normal((n2, g.nb, d))
    idx, num = rf.select_sequence(qbar, kbar, g)
    return g, qbar, kbar, idx, num


@pytest.mark.parametrize("s", [0.5, 0.8, 0.9])
def test_selection_invariants(s):
    g, qbar, kbar, idx, num = _random_select(100, 9, 16, 32, s)
    assert g.n_pb == 1 and g.nb == 36 and g.ns == 4
    for qb in range(g.n_blocks):
        for n in range(2):
            row = idx[qb, n, :num[qb, n]].tolist()
            assert np.all(idx[qb, n, num[qb, n]:] == -1)
            assert row == sorted(row) and len(set(row)) == len(row)
            assert row[:g.n_pb] == list(range(g.n_pb))              # prefix always kept
            video = [b - g.n_pb for b in row[g.n_pb:]]
            i = qb - g.n_pb
            if qb < g.n_pb or i < g.ns:
                assert num[qb, n] == g.n_blocks                       # dense query blocks
                continue
            assert set(range(g.ns)) <= set(video)                     # sinks kept
            assert g.n_pb + max(g.k, g.ns) <= num[qb, n] <= g.n_pb + min(g.k + g.ns, g.nb)
            sc = qbar[n, i] @ kbar[n, :].T
            ranked = [j for j in video if j >= g.ns or j in rf.topk_blocks(sc, g.k)]
            dropped = [j for j in range(g.nb) if j not in video]
            top = rf.topk_blocks(sc, g.k)
            if dropped and top:
                assert min(sc[top]) >= max(sc[dropped])


def test_sparsity_zero_and_one():
    g, _, _, idx, num = _random_select(64, 9, 16, 32, 0.0)
    assert np.all(num == g.n_blocks)
    g, _, _, idx, num = _random_select(64, 9, 16, 32, 1.0)
    for qb in range(g.n_pb + g.ns, g.n_blocks):
        assert idx[qb, 0, :num[qb, 0]].tolist() == list(range(g.n_pb + g.ns))


def test_planted_key_block_is_selected_per_kv_head():
    g = rf.geometry(64, 9, 16, 32, 0.9)
    rng = np.random.default_rng(5)
    n1, n2, d = 4, 2, 8
    qbar = rng.standard_normal((n1, g.nb, d))
    kbar = rng.standard_normal((n2, g.nb, d)) * 0.01
    i, jstar = 20, 30
    kbar[1, jstar] = 100.0 * qbar[2, i]          # only kv head 1 (q heads 2, 3) sees it
    idx, num = rf.select_sequence(qbar, kbar, g)
    row2 = idx[g.n_pb + i, 2, :num[g.n_pb + i, 2]].tolist()
    assert g.n_pb + jstar in row2
    # q head 0 reads kv head 0, where block jstar is tiny: with k = 4 of 36 it is not forced in
    scores0 = qbar[0, i] @ kbar[0].T
    assert (g.n_pb + jstar in idx[g.n_pb + i, 0].tolist()) == (jstar in rf.topk_blocks(scores0, g.k) or jstar < g.ns)


def test_short_video_selects_everything():
    g, _, _, idx, num = _random_select(64, 2, 16, 16, 0.9)
    assert g.dense and np.all(num == g.n_blocks)


def test_multi_sequence_select_pads_to_max():
    p = rf.make_problem("TND", 1, [(64, 9, 16, 32), (10, 2, 16, 16)], 2, 1, 8, 0.8)
    rng = np.random.default_rng(6)
    qb = [rng.standard_normal((2, g.nb, 8)) for g in p.geoms]
    kb = [rng.standard_normal((1, g.nb, 8)) for g in p.geoms]
    idx, num = rf.select(p, qb, kb)
    assert idx.shape == (p.t_qblk, 2, p.max_kv_blocks)
    g1 = p.geoms[1]
    tail = idx[p.geoms[0].n_blocks:]
    assert np.all(tail[:, :, g1.n_blocks:] == -1)
    assert np.all(num[p.geoms[0].n_blocks:] == g1.n_blocks)
