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


# ---- key blocks of 64 rows (blockShape 128 x 64; reading R26) ----

@pytest.mark.parametrize("geom", [(100, 9, 16, 32, 0.8), (64, 9, 16, 32, 0.9), (0, 21, 48, 80, 0.5),
                                  (10, 2, 16, 16, 0.9), (7, 13, 27, 45, 0.8)])
def test_key_blocks_of_128_rows_are_the_sequence_counts(geom):
    g = rf.geometry(*geom)
    kb = rf.key_blocks(g, 128)
    assert (kb.n_pb, kb.nb, kb.ns, kb.k) == (g.n_pb, g.nb, g.ns, g.k)


def test_key_blocks_of_64_rows_closed_forms():
    # P = 100, (9, 16, 32): Lp = 100, S = 36 * 128 = 4608, first frame 16 * 32 = 512 tokens
    kb = rf.key_blocks(rf.geometry(100, 9, 16, 32, 0.8), 64)
    assert (kb.n_pb, kb.nb, kb.ns, kb.k) == (2, 72, 8, 15)        # ceil(100/64), 4608/64, 512/64, ceil(14.4)
    kb = rf.key_blocks(rf.geometry(64, 9, 16, 32, 0.9), 64)
    assert (kb.n_pb, kb.nb, kb.ns, kb.k) == (1, 72, 8, 8)         # ceil(0.1 * 72) = ceil(7.2)
    kb = rf.key_blocks(rf.geometry(0, 21, 48, 80, 0.8), 64)       # the Aligned grid, no text
    assert (kb.n_pb, kb.nb, kb.ns, kb.k) == (0, 1260, 60, 252)
    kb = rf.key_blocks(rf.geometry(10, 2, 16, 16, 0.9), 64)       # 4 blocks of 128: dense
    assert (kb.n_pb, kb.nb, kb.ns, kb.k) == (1, 8, 4, 8)


def test_block_means_of_64_rows_brute_force():
    g = rf.geometry(100, 8, 16, 32, 0.8)
    rng = np.random.default_rng(13)
    x = rng.standard_normal((g.length, 5))
    m = rf.block_means(x, g, 64)
    assert m.shape == (2 * g.nb, 5)
    for i in range(2 * g.nb):
        for c in range(5):
            s = 0.0
            for r in range(g.lp + 64 * i, g.lp + 64 * i + 64):
                s += x[r, c]
            assert abs(m[i, c] - s / 64) < 1e-12


def _random_select64(p, t, h, w, s, n1=2, n2=2, d=8, seed=14):
    g = rf.geometry(p, t, h, w, s)
    kb = rf.key_blocks(g, 64)
    rng = np.random.default_rng(seed)
    qbar = rng.standard_normal((n1, g.nb, d))
    kbar = rng.standard_normal((n2, kb.nb, d))
    idx, num = rf.select_sequence(qbar, kbar, g, 64)
    return g, kb, qbar, kbar, idx, num


@pytest.mark.parametrize("s", [0.5, 0.8, 0.9])
def test_kv64_selection_invariants(s):
    g, kb, qbar, kbar, idx, num = _random_select64(100, 9, 16, 32, s)
    nkv = kb.n_pb + kb.nb
    assert idx.shape == (g.n_blocks, 2, nkv)
    for qb in range(g.n_blocks):
        for n in range(2):
            row = idx[qb, n, :num[qb, n]].tolist()
            assert np.all(idx[qb, n, num[qb, n]:] == -1)
            assert row == sorted(row) and len(set(row)) == len(row)
            assert row[:kb.n_pb] == list(range(kb.n_pb))            # prefix key blocks always kept
            i = qb - g.n_pb
            if qb < g.n_pb or i < g.ns:                             # dense query blocks (128-row units)
                assert row == list(range(nkv))
                continue
            video = [b - kb.n_pb for b in row[kb.n_pb:]]
            assert set(range(kb.ns)) <= set(video)                   # 64-row sinks kept
            assert kb.n_pb + max(kb.k, kb.ns) <= num[qb, n] <= kb.n_pb + min(kb.k + kb.ns, kb.nb)
            sc = qbar[n, i] @ kbar[n].T                              # 128-row query mean . 64-row key means
            top = rf.topk_blocks(sc, kb.k)
            assert set(top) <= set(video)
            dropped = [j for j in range(kb.nb) if j not in video]
            if dropped and top:
                assert min(sc[top]) >= max(sc[dropped])


@pytest.mark.parametrize("s", [0.5, 0.75])
def test_kv64_selection_of_duplicated_halves_is_the_expanded_128_selection(s):
    """Key rows whose two 64-row halves of every sparse 128-row block are equal give
    equal 64-row means for both halves: the 64-row selection must then be the
    128-row selection with every block replaced by the 64-row blocks that cover its
    rows (here k64 = 2 k and ns64 = 2 ns, so nothing else can differ)."""
    g = rf.geometry(100, 9, 16, 32, s)
    kb = rf.key_blocks(g, 64)
    assert kb.k == 2 * g.k and kb.ns == 2 * g.ns
    rng = np.random.default_rng(15)
    n1, n2, d = 4, 2, 8
    k_r = rng.standard_normal((n2, g.length, d))
    for j in range(g.nb):
        r0 = g.lp + 128 * j
        k_r[:, r0 + 64:r0 + 128] = k_r[:, r0:r0 + 64]
    kbar64 = np.stack([rf.block_means(k_r[n], g, 64) for n in range(n2)])
    assert np.array_equal(kbar64[:, 0::2], kbar64[:, 1::2])
    qbar = rng.standard_normal((n1, g.nb, d))
    idx64, num64 = rf.select_sequence(qbar, kbar64, g, 64)
    idx128, num128 = rf.select_sequence(qbar, kbar64[:, 0::2], g)
    cover = {}
    for b in range(g.n_blocks):
        rows = set(rf.block_rows(g, b))
        cover[b] = [c for c in range(kb.n_pb + kb.nb) if rf.kv_block_rows(g, c, 64).start in rows]
    for qb in range(g.n_blocks):
        for n in range(n1):
            want = [c for b in idx128[qb, n, :num128[qb, n]] for c in cover[int(b)]]
            assert idx64[qb, n, :num64[qb, n]].tolist() == want


def test_kv64_sparsity_zero_one_and_dense_sequence():
    g, kb, _, _, idx, num = _random_select64(64, 9, 16, 32, 0.0)
    assert np.all(num == kb.n_pb + kb.nb)
    g, kb, _, _, idx, num = _random_select64(64, 9, 16, 32, 1.0)
    for qb in range(g.n_pb + g.ns, g.n_blocks):
        assert idx[qb, 0, :num[qb, 0]].tolist() == list(range(kb.n_pb + kb.ns))
    g, kb, _, _, idx, num = _random_select64(10, 2, 16, 16, 0.9)
    assert g.dense and np.all(num == kb.n_pb + kb.nb)


def test_kv64_problem_select_pads_to_the_widest_sequence():
    p = rf.make_problem("TND", 1, [(64, 9, 16, 32), (10, 2, 16, 16)], 2, 1, 8, 0.8)
    rng = np.random.default_rng(16)
    qb = [rng.standard_normal((2, g.nb, 8)) for g in p.geoms]
    kb = [rng.standard_normal((1, 2 * g.nb, 8)) for g in p.geoms]
    idx, num = rf.select(p, qb, kb, 64)
    widths = [rf.kv_block_count(g, 64) for g in p.geoms]
    assert idx.shape == (p.t_qblk, 2, max(widths))
    tail = idx[p.geoms[0].n_blocks:]
    assert np.all(tail[:, :, widths[1]:] == -1)
    assert np.all(num[p.geoms[0].n_blocks:] == widths[1])


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=40, deadline=None)
@given(prefix=st.integers(0, 300), t=st.integers(1, 6), h=st.integers(8, 40), w=st.integers(8, 40),
       s=st.sampled_from([0.0, 0.5, 0.8, 0.9, 1.0]), seed=st.integers(0, 1000))
def test_kv64_selection_invariants_on_random_geometries(prefix, t, h, w, s, seed):
    """Over random grids and sparsities: the key-side counts agree with kv_block_count,
    dense rows list every key block, and every other row lists all prefix key blocks and
    then exactly the sink key blocks together with the k best-scoring 64-row key blocks."""
    g = rf.geometry(prefix, t, h, w, s)
    kb = rf.key_blocks(g, 64)
    assert kb.n_pb + kb.nb == rf.kv_block_count(g, 64)
    if g.nb == 0:
        return
    rng = np.random.default_rng(seed)
    qbar = rng.standard_normal((1, g.nb, 4))
    kbar = rng.standard_normal((1, kb.nb, 4))
    idx, num = rf.select_sequence(qbar, kbar, g, 64)
    for qb in range(g.n_blocks):
        row = idx[qb, 0, :num[qb, 0]].tolist()
        i = qb - g.n_pb
        if g.dense or qb < g.n_pb or i < g.ns:
            assert row == list(range(kb.n_pb + kb.nb))
            continue
        assert row[:kb.n_pb] == list(range(kb.n_pb))
        video = [b - kb.n_pb for b in row[kb.n_pb:]]
        top = rf.topk_blocks(qbar[0, i] @ kbar[0].T, kb.k)
        assert set(video) == set(top) | set(range(kb.ns))
