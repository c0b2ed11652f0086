"""Host helpers of bench.py (CPU only): the 64-row expansion of a selection that the
--block-kv 64 timing mode feeds the attention must list exactly the rows of the
128-row selection, and must agree with the test suite's own expansion, which is
written from the oracle's geometry rather than the plan's."""
import numpy as np
import pytest

import bench
from block_sparse_video_rearrange_b200 import rf, synth
from oracle import rainfusion as orc
from tests import parity

W, S = synth.Workload, synth.SeqSpec
CASES = [
    W("ragged", "BNSD", "bf16", 2, (S(77, 9, 17, 33),), 2, 2, 128, 0.8, 41),          # batch 2
    W("tnd", "TND", "fp16", 1, (S(64, 9, 16, 32), S(200, 10, 19, 21)), 4, 2, 128, 0.8, 42),
    W("text", "BNSD", "bf16", 1, (S(300, 0, 0, 0),), 2, 2, 64, 0.8, 43),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_kv64_expansion_covers_the_same_rows(w):
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    rbits = [orc.rearrange(p, x) for x in bits]
    qb, kb = parity.oracle_pooled(p, w, rbits)
    idx, num = orc.select(p, qb, kb)
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch)
    plan64 = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch,
                     block_kv=64)
    width = int(plan64.info.max_kv_blocks)
    i64, n64 = bench.expand_selection_kv64(plan, idx, num, width)
    ref_i, ref_n = parity.expand_to_kv64(p, idx, num, width)
    assert np.array_equal(i64, ref_i) and np.array_equal(n64, ref_n)
    table = orc.qblock_table(p)
    for t in range(idx.shape[0]):
        _, g, _ = table[t]
        for n in range(w.n1):
            rows128 = [r for b in idx[t, n, :num[t, n]] for r in orc.block_rows(g, int(b))]
            rows64 = [r for c in i64[t, n, :n64[t, n]] for r in orc.kv_block_rows(g, int(c), 64)]
            assert rows128 == rows64
