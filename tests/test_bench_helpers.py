"""Host helpers of bench.py (CPU only): the kept-FLOP count that the bench divides by
its time must equal the oracle's count over the same selection, for 128-row and for
64-row key blocks (the latter on the oracle's own 64-row selection, reading R26)."""
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


@pytest.mark.parametrize("block_kv", [128, 64])
@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_kept_flops_equal_the_oracle_count(w, block_kv):
    bits = synth.generate_qkv(w)
    p = parity.problem(w)
    rbits = [orc.rearrange(p, x) for x in bits]
    qb, kb = parity.oracle_pooled(p, w, rbits, block_kv)
    idx, num = orc.select(p, qb, kb, block_kv)
    plan = rf.Plan(parity.seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch,
                   block_kv=block_kv)
    assert idx.shape[2] == int(plan.info.max_kv_blocks)
    assert bench.kept_flops_from_selection(plan, idx, num) == orc.kept_flops(p, idx, num, block_kv)
