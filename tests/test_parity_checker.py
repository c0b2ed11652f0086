"""The parity checker's selection rule on planted cases (CPU only): a near-tie swap
is accepted, a swap across a clear score gap and a changed selectNum are not."""
import numpy as np
import pytest

from block_sparse_video_rearrange_b200 import synth
from oracle import rainfusion as orc
from tests import parity


def _setup():
    w = synth.Workload("chk", "BNSD", "bf16", 1, (synth.SeqSpec(64, 9, 16, 32),), 2, 1, 64, 0.8, 41)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    rbits = [orc.rearrange(p, x) for x in bits]
    qbars, kbars = parity.oracle_pooled(p, w, rbits)
    idx, num = orc.select(p, qbars, kbars)
    return p, qbars, kbars, idx, num


def _sparse_row(p, idx, num):
    g = p.geoms[0]
    t = g.n_pb + g.ns + 3                       # a sparse query block
    return g, t, 0


def test_identical_selection_passes():
    p, qb, kb, idx, num = _setup()
    st = parity.check_selection(p, qb, kb, dict(idx=idx.copy(), num=num.copy()))
    assert st["exact"] == st["rows"]


def test_swap_across_a_score_gap_fails():
    p, qb, kb, idx, num = _setup()
    g, t, n = _sparse_row(p, idx, num)
    sc = qb[0][n, t - g.n_pb] @ kb[0][0].T
    row = idx[t, n, :num[t, n]].tolist()
    video = [j - g.n_pb for j in row[g.n_pb:]]
    kept = [j for j in video if j >= g.ns]
    dropped = [j for j in range(g.nb) if j not in video]
    lo = max(kept, key=lambda j: sc[j])           # the best kept block ...
    hi = min(dropped, key=lambda j: sc[j])        # ... swapped for the worst dropped one
    new = sorted(g.n_pb + j for j in (set(video) - {lo}) | {hi})
    bad = idx.copy()
    bad[t, n, :len(row)] = sorted(row[:g.n_pb] + new)
    with pytest.raises(AssertionError):
        parity.check_selection(p, qb, kb, dict(idx=bad, num=num.copy()))


def test_near_tie_swap_passes_and_is_counted():
    p, qb, kb, idx, num = _setup()
    g = p.geoms[0]
    # a sparse row whose k-th and (k+1)-th ranked blocks are both outside the sinks
    for t in range(g.n_pb + g.ns, g.n_blocks):
        sc = qb[0][0, t - g.n_pb] @ kb[0][0].T
        order = sorted(range(g.nb), key=lambda j: (-sc[j], j))
        lo, hi = order[g.k - 1], order[g.k]
        if lo >= g.ns and hi >= g.ns:
            break
    else:
        pytest.skip("no such row")
    n = 0
    row = idx[t, n, :num[t, n]].tolist()
    # make the pair a near tie: move K block hi's mean so that its score is just below lo's
    q = qb[0][n, t - g.n_pb]
    kb2 = [kb[0].copy()]
    kb2[0][0, hi] += (sc[lo] * (1 - 1e-6) - sc[hi]) * q / (q @ q)
    got = dict(idx=idx.copy(), num=num.copy())
    video = [j - g.n_pb for j in row[g.n_pb:]]
    got["idx"][t, n, :len(row)] = sorted(row[:g.n_pb] + [g.n_pb + j for j in (set(video) - {lo}) | {hi}])
    st = parity.check_selection(p, qb, kb2, got, rows=[(t, n)])
    assert st["near_tie"] == 1


def test_changed_select_num_fails():
    p, qb, kb, idx, num = _setup()
    g, t, n = _sparse_row(p, idx, num)
    bad_num = num.copy()
    bad_num[t, n] -= 1
    bad_idx = idx.copy()
    bad_idx[t, n, bad_num[t, n]] = -1
    with pytest.raises(AssertionError):
        parity.check_selection(p, qb, kb, dict(idx=bad_idx, num=bad_num))


def test_kv64_checker_accepts_the_oracle_and_rejects_a_gap_swap():
    """The same rule over 64-row key blocks (reading R26): the oracle's own selection
    passes exactly; swapping the best kept key block for the worst dropped one fails."""
    w = synth.Workload("chk64", "BNSD", "bf16", 1, (synth.SeqSpec(100, 9, 16, 32),), 2, 1, 64, 0.8, 42)
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    rbits = [orc.rearrange(p, x) for x in bits]
    qb, kb = parity.oracle_pooled(p, w, rbits, 64)
    assert kb[0].shape[1] == 2 * p.geoms[0].nb
    idx, num = orc.select(p, qb, kb, 64)
    st = parity.check_selection(p, qb, kb, dict(idx=idx.copy(), num=num.copy()), block_kv=64)
    assert st["exact"] == st["rows"]
    g = p.geoms[0]
    k64 = orc.key_blocks(g, 64)
    t, n = g.n_pb + g.ns + 5, 1
    sc = qb[0][n, t - g.n_pb] @ kb[0][0].T
    row = idx[t, n, :num[t, n]].tolist()
    video = [j - k64.n_pb for j in row[k64.n_pb:]]
    kept = [j for j in video if j >= k64.ns]
    dropped = [j for j in range(k64.nb) if j not in video]
    lo, hi = max(kept, key=lambda j: sc[j]), min(dropped, key=lambda j: sc[j])
    bad = idx.copy()
    bad[t, n, :len(row)] = sorted(row[:k64.n_pb] + [k64.n_pb + j for j in (set(video) - {lo}) | {hi}])
    with pytest.raises(AssertionError):
        parity.check_selection(p, qb, kb, dict(idx=bad, num=num.copy()), block_kv=64)
