"""Shared parity checks: the CUDA path (through the C ABI) against the CPU oracle.

Bars (stated for this path): permutation and selectNum bit-exact on every
row; selectIdx bit-exact except where two candidate block scores are within
1e-4 relative (then the GPU's row must still be a valid top-k up to such near
ties); attention output, with the oracle run
on the GPU's own selectIdx, max-abs <= 2e-2 and relative L2 <= 1e-2.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence, Tuple

import numpy as np
import torch

from block_sparse_video_rearrange_b200 import rf, synth
from oracle import mxattention as mxo
from oracle import rainfusion as orc

MAX_ABS = 2e-2
REL_L2 = 1e-2
TIE_REL = 1e-4
POOL_REL = 1e-5


def seqs_of(w: synth.Workload):
    return [(s.prefix_len, s.t, s.h, s.w) for s in w.seqs]


def problem(w: synth.Workload, order: str = "tile") -> orc.Problem:
    return orc.make_problem(w.layout, w.batch, seqs_of(w), w.n1, w.n2, w.d, w.sparsity, order)


def to_device(bits: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16).cuda()


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def run_gpu(w: synth.Workload, bits: Sequence[np.ndarray], pool_mode: str = "from_ws",
            order: str = "tile", precision: str = "native", block_kv: int = 128) -> Dict[str, object]:
    """Whole path through the C ABI, one call per step; returns host copies of every result."""
    plan = rf.Plan(seqs_of(w), w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch, order=order,
                   precision=precision, block_kv=block_kv)
    q, k, v = (to_device(b, w.dtype) for b in bits)
    b = rf.Buffers(plan)
    scale = 1.0 / math.sqrt(w.d)
    rf.rearrange(plan, q, k, v, b.q_r, b.k_r, b.v_r, b.ws)
    rf.pool_select(plan, b.q_r, b.k_r, b.select_idx, b.select_num, b.ws, pool_mode=pool_mode)
    rf.block_sparse_attn(plan, b.q_r, b.k_r, b.v_r, b.select_idx, b.select_num, scale, b.o_r, b.ws)
    rf.inverse_rearrange(plan, b.o_r, b.o)
    st, flags = rf.check_device_status(plan, b.ws)
    assert st == 0, (st, flags)
    torch.cuda.synchronize()
    ws8 = b.ws.view(torch.uint8)
    pooled, pooled_k = int(plan.info.pooled_blocks), int(plan.info.pooled_k_blocks)
    oq, ok_ = int(plan.info.ws_pooled_q), int(plan.info.ws_pooled_k)
    pq = ws8[oq:oq + w.n1 * pooled * w.d * 4].view(torch.float32).reshape(w.n1, pooled, w.d).cpu().numpy()
    pk = ws8[ok_:ok_ + w.n2 * pooled_k * w.d * 4].view(torch.float32).reshape(w.n2, pooled_k, w.d).cpu().numpy()
    out = dict(plan=plan, q_r=to_bits(b.q_r), k_r=to_bits(b.k_r), v_r=to_bits(b.v_r), o_r=to_bits(b.o_r),
               o=to_bits(b.o), idx=b.select_idx.cpu().numpy(), num=b.select_num.cpu().numpy(),
               pooled_q=pq, pooled_k=pk, scale=scale)
    if precision in ("mix", "fp8"):
        out.update(mix_buffers(plan, b.ws))
    if precision == "fp8":
        out.update(fp8_buffers(plan, b.ws, problem(w)))
    if precision == "mxfp4":
        out.update(mx_buffers(plan, b.ws))
    return out


def mx_buffers(plan: rf.Plan, ws: torch.Tensor) -> Dict[str, np.ndarray]:
    """float64 values of the MXFP4 copies of Q', K', V' in the layouts of q_r, k_r, v_r:
    at head dim 128 decoded from their E4M3 carriers (Q', K' one byte per element, V'
    transposed per block), else from the 16-bit copies (Q', K' plan dtype, V' f16)."""
    info = plan.info
    ws8 = ws.view(torch.uint8)
    rows, d = int(info.rows_total), plan.d
    if d == 128:
        def bytes_(off, n):
            return ws8[int(off):int(off) + n].cpu().numpy()
        qx = orc.e4m3_decode(bytes_(info.ws_q8, rows * plan.n1 * d).reshape(plan.tensor_shape(plan.n1)))
        kx = orc.e4m3_decode(bytes_(info.ws_k8, rows * plan.n2 * d).reshape(plan.tensor_shape(plan.n2)))
        t = int(info.t_qblk)
        raw = bytes_(info.ws_v8, plan.n2 * t * 128 * d).reshape(plan.n2, t, d, 128)
        p = problem_of_plan(plan)
        vx = np.zeros(plan.tensor_shape(plan.n2), dtype=np.float64)
        for tb, (s, g, b) in enumerate(orc.qblock_table(p)):
            r = orc.block_rows(g, b)
            for n in range(plan.n2):
                p.head_rows(vx, s, n)[r.start:r.stop] = orc.e4m3_decode(raw[n, tb, :, :len(r)].T)
        return dict(qx=qx, kx=kx, vx=vx)

    def region(off, heads, dt):
        n = rows * heads * d * 2
        bits = ws8[int(off):int(off) + n].cpu().numpy().view(np.uint16).reshape(plan.tensor_shape(heads))
        return synth.bits_to_float64(bits, dt)
    return dict(qx=region(info.ws_q_mx, plan.n1, plan.dtype), kx=region(info.ws_k_mx, plan.n2, plan.dtype),
                vx=region(info.ws_v_mx, plan.n2, "fp16"))


def problem_of_plan(plan: rf.Plan) -> orc.Problem:
    return orc.make_problem(plan.layout, plan.batch, plan.seqs, plan.n1, plan.n2, plan.d, plan.sparsity,
                            plan.order)


def oracle_mx_inputs(p: orc.Problem, w: synth.Workload, rbits: Sequence[np.ndarray]):
    """float64 Q', K', V' rounded to MXFP4 by the oracle (UOS, groups along each product's
    reduction axis) from the exact 16-bit rearranged values."""
    q, k, v = (synth.bits_to_float64(x, w.dtype) for x in rbits)
    return (mxo.quantize_head(p, q, w.n1, "rows"), mxo.quantize_head(p, k, w.n2, "rows"),
            mxo.quantize_head(p, v, w.n2, "keys"))


def check_mx_quantization(p: orc.Problem, w: synth.Workload, ref, gpu) -> None:
    """The MXFP4 copies equal the oracle's rounding value for value (carried as E4M3 at
    head dim 128, else Q', K' in the input type and V' in f16; every MXFP4 value of
    these inputs is exact in each)."""
    for name, x in (("qx", ref[0]), ("kx", ref[1]), ("vx", ref[2])):
        got = gpu[name]
        diff = got != x
        assert not diff.any(), f"{name}: {int(diff.sum())} values differ, e.g. {got[diff][:4]} vs {x[diff][:4]}"


def mix_buffers(plan: rf.Plan, ws: torch.Tensor) -> Dict[str, np.ndarray]:
    """Host copies of the E4M3 copies of Q' / K' and their scales in a mix-precision workspace."""
    info = plan.info
    ws8 = ws.view(torch.uint8)
    rows, t, d = int(info.rows_total), int(info.t_qblk), plan.d

    def region(off, n):
        return ws8[int(off):int(off) + n].cpu().numpy()
    q8 = region(info.ws_q8, rows * plan.n1 * d).reshape(plan.tensor_shape(plan.n1))
    k8 = region(info.ws_k8, rows * plan.n2 * d).reshape(plan.tensor_shape(plan.n2))
    qs = region(info.ws_q_scale, plan.n1 * t * 4).view(np.float32).reshape(plan.n1, t)
    ks = region(info.ws_k_scale, plan.n2 * t * 4).view(np.float32).reshape(plan.n2, t)
    return dict(q8=q8, k8=k8, q_scale=qs, k_scale=ks)


def fp8_buffers(plan: rf.Plan, ws: torch.Tensor, p: orc.Problem) -> Dict[str, np.ndarray]:
    """Precision fp8: the transposed E4M3 V' codes put back into the layout of v_r (rows
    past a partial block's end are dropped) and the int32 exponents [n2, t_qblk]."""
    info = plan.info
    ws8 = ws.view(torch.uint8)
    t, d, n2 = int(info.t_qblk), plan.d, plan.n2
    raw = ws8[int(info.ws_v8):int(info.ws_v8) + n2 * t * 128 * d].cpu().numpy().reshape(n2, t, d, 128)
    exps = ws8[int(info.ws_v_exp):int(info.ws_v_exp) + n2 * t * 4].cpu().numpy().view(np.int32).reshape(n2, t)
    codes = np.zeros(plan.tensor_shape(n2), dtype=np.uint8)
    for tb, (s, g, b) in enumerate(orc.qblock_table(p)):
        r = orc.block_rows(g, b)
        for n in range(n2):
            p.head_rows(codes, s, n)[r.start:r.stop] = raw[n, tb, :, :len(r)].T
    return dict(v8=codes, v_exp=exps, v8_raw=raw)


def check_fp8_quantization(p: orc.Problem, w: synth.Workload, rbits: Sequence[np.ndarray], gpu) -> None:
    """Precision fp8: Q', K' as mix; V' codes and exponents bit-exact against the oracle,
    and the rows past a partial block's end hold code 0."""
    check_mix_quantization(p, w, rbits, gpu)
    vf = synth.bits_to_float64(rbits[2], w.dtype)
    codes, exps = orc.quantize_v_fp8(p, vf, w.n2)
    assert np.array_equal(gpu["v_exp"], exps), "V exponents differ"
    diff = gpu["v8"] != codes
    assert not diff.any(), f"V E4M3 codes differ at {int(diff.sum())} elements"
    for tb, (s, g, b) in enumerate(orc.qblock_table(p)):
        n_valid = len(orc.block_rows(g, b))
        assert not gpu["v8_raw"][:, tb, :, n_valid:].any(), tb


def fp8_reference_inputs(p: orc.Problem, w: synth.Workload, gpu, rbits: Sequence[np.ndarray]):
    """float64 Q', K', V' as precision fp8 sees them (codes x scales)."""
    qf = orc.dequantize_e4m3(p, gpu["q8"], gpu["q_scale"], w.n1)
    kf = orc.dequantize_e4m3(p, gpu["k8"], gpu["k_scale"], w.n2)
    vf = orc.dequantize_v_fp8(p, gpu["v8"], gpu["v_exp"], w.n2)
    return qf, kf, vf


def check_fp8_attention(p: orc.Problem, w: synth.Workload, rbits: Sequence[np.ndarray], gpu,
                        items: Sequence[Tuple[int, int]] | None = None) -> Dict[str, float]:
    """Precision fp8 output against the oracle run on the dequantized Q', K', V' with
    exact probabilities: every element within the oracle's bound on rounding the
    probabilities to E4M3 (fp8_probability_error_bound) plus the output's own 16-bit
    rounding (half an ulp, 2^-8 relative for bf16) and 1e-3 for the fp32 arithmetic;
    relative L2 within the native bar."""
    qf, kf, vf = fp8_reference_inputs(p, w, gpu, rbits)
    if items is None:
        items = [(t, n) for t in range(p.t_qblk) for n in range(w.n1)]
    ref = orc.attention(p, qf, kf, vf, gpu["idx"], gpu["num"], gpu["scale"], items)
    bound = orc.fp8_probability_error_bound(p, qf, kf, vf, gpu["idx"], gpu["num"], gpu["scale"], items,
                                            v_exps=gpu["v_exp"])
    o_r = synth.bits_to_float64(gpu["o_r"], w.dtype)
    table = orc.qblock_table(p)
    num = den = 0.0
    mx = worst = 0.0
    for (t, n), rows in ref.items():
        s, g, b = table[t]
        r = orc.block_rows(g, b)
        got = p.head_rows(o_r, s, n)[r.start:r.stop]
        d = np.abs(got - rows)
        lim = bound[(t, n)] + 2.0 ** -8 * np.abs(rows) + 1e-3
        assert np.all(d <= lim), (t, n, float(np.max(d - lim)))
        mx = max(mx, float(np.max(d)))
        worst = max(worst, float(np.max(d / lim)))
        num += float(np.sum(d * d))
        den += float(np.sum(rows * rows))
    rel = math.sqrt(num / max(den, 1e-300))
    assert rel <= REL_L2, f"rel L2 err {rel}"
    return dict(max_abs=mx, rel_l2=rel, items=len(ref), worst_fraction_of_bound=worst)


def check_mix_quantization(p: orc.Problem, w: synth.Workload, rbits: Sequence[np.ndarray], gpu) -> None:
    """E4M3 codes and scales of Q' and K' bit-exact against the oracle's quantization."""
    for name, x, heads in (("q", rbits[0], w.n1), ("k", rbits[1], w.n2)):
        xf = synth.bits_to_float64(x, w.dtype).astype(np.float32)   # exact: 16-bit values
        codes, scales = orc.quantize_e4m3(p, xf, heads)
        assert np.array_equal(gpu[name + "_scale"], scales), f"{name} scales differ"
        got = gpu[name + "8"]
        diff = got != codes
        assert not diff.any(), f"{name} E4M3 codes differ at {int(diff.sum())} elements"


def mix_reference_inputs(p: orc.Problem, w: synth.Workload, gpu, rbits: Sequence[np.ndarray]):
    """float64 Q', K' as the mix precision sees them (E4M3 code x scale) and exact V'."""
    qf = orc.dequantize_e4m3(p, gpu["q8"], gpu["q_scale"], w.n1)
    kf = orc.dequantize_e4m3(p, gpu["k8"], gpu["k_scale"], w.n2)
    return qf, kf, synth.bits_to_float64(rbits[2], w.dtype)


def expand_to_kv64(p: orc.Problem, idx: np.ndarray, num: np.ndarray, width: int):
    """A 128-row key-block selection rewritten over 64-row key blocks: every
    selected block becomes the one or two 64-row blocks inside it (in order)."""
    table = orc.qblock_table(p)
    T, N, _ = idx.shape
    out = np.full((T, N, width), -1, dtype=np.int32)
    cnt = np.zeros((T, N), dtype=np.int32)
    inside = {}
    for t in range(T):
        s, g, _ = table[t]
        if g not in inside:
            n64 = orc.kv_block_count(g, 64)
            starts = {orc.kv_block_rows(g, c, 64).start: c for c in range(n64)}
            inside[g] = [[starts[r] for r in orc.block_rows(g, b) if r in starts] for b in range(g.n_blocks)]
        for n in range(N):
            row = [c for b in idx[t, n, :num[t, n]] if b >= 0 for c in inside[g][int(b)]]
            out[t, n, :len(row)] = row
            cnt[t, n] = len(row)
    return out, cnt


def oracle_rearranged_bits(p: orc.Problem, bits: np.ndarray) -> np.ndarray:
    """The oracle's permutation applied to raw 16-bit patterns (exact)."""
    return orc.rearrange(p, bits)


def check_permutation(p: orc.Problem, bits: Sequence[np.ndarray], gpu: Dict[str, object]) -> None:
    for name, x in zip(("q_r", "k_r", "v_r"), bits):
        exp = oracle_rearranged_bits(p, x)
        assert np.array_equal(gpu[name], exp), f"{name} differs from the oracle permutation"
    # the inverse is checked against the GPU's own rearranged output: o[orig] == o_r
    assert np.array_equal(orc.inverse_rearrange(p, gpu["o_r"]), gpu["o"]), "inverse permutation differs"


def oracle_pooled(p: orc.Problem, w: synth.Workload, rbits: Sequence[np.ndarray], block_kv: int = 128):
    """Per sequence instance: float64 means of the oracle-rearranged Q ([heads, nb, D],
    128-row query blocks) and K ([heads, S / block_kv, D], key blocks of block_kv rows)."""
    qf = synth.bits_to_float64(rbits[0], w.dtype)
    kf = synth.bits_to_float64(rbits[1], w.dtype)
    return orc.pooled_means(p, qf, w.n1), orc.pooled_means(p, kf, w.n2, block_kv)


def check_pooled(p: orc.Problem, qbars, kbars, gpu) -> None:
    offq = offk = 0
    for (s, g), qb, kb in zip(p.sequences(), qbars, kbars):
        gq = gpu["pooled_q"][:, offq:offq + qb.shape[1]]
        gk = gpu["pooled_k"][:, offk:offk + kb.shape[1]]
        for ref, got in ((qb, gq), (kb, gk)):
            assert got.shape == ref.shape
            if ref.size:
                err = np.max(np.abs(got - ref)) / max(1e-30, np.max(np.abs(ref)))
                assert err < POOL_REL, f"pooled means rel err {err}"
        offq += qb.shape[1]
        offk += kb.shape[1]


def check_selection(p: orc.Problem, qbars, kbars, gpu, rows: Sequence[Tuple[int, int]] | None = None,
                    block_kv: int = 128) -> Dict[str, int]:
    """selectIdx / selectNum against the oracle's selection.  Returns counters.

    selectNum must equal the oracle's on every row (bit-exact).  A selectIdx row
    may differ from the oracle's only by near ties: the GPU's top-k set T (its
    non-sink video blocks, completed with the best-scoring sinks) must be a
    valid top-k of the oracle's float64 scores, in that every block in T scores
    at least as high as every video block outside T, up to TIE_REL relative."""
    idx_o, num_o = orc.select(p, qbars, kbars, block_kv)
    idx_g, num_g = gpu["idx"], gpu["num"]
    assert idx_g.shape == idx_o.shape and num_g.shape == num_o.shape
    table = orc.qblock_table(p)
    G = p.n1 // p.n2
    seq_pos = {s: i for i, (s, _) in enumerate(p.sequences())}
    stats = dict(rows=0, exact=0, near_tie=0)
    todo = rows if rows is not None else [(t, n) for t in range(len(table)) for n in range(p.n1)]
    for t, n in todo:
        stats["rows"] += 1
        assert num_g[t, n] == num_o[t, n], f"selectNum differs at (t={t}, n={n}): {num_g[t, n]} vs {num_o[t, n]}"
        a = idx_g[t, n, :num_g[t, n]].tolist()
        b = idx_o[t, n, :num_o[t, n]].tolist()
        # padding is -1 everywhere past selectNum
        assert np.all(idx_g[t, n, num_g[t, n]:] == -1)
        assert a == sorted(a)
        if a == b:
            stats["exact"] += 1
            continue
        s, g, qb = table[t]
        kb = orc.key_blocks(g, block_kv)
        assert not g.dense and qb >= g.n_pb + g.ns, f"dense row (t={t}, n={n}) differs"
        assert a[:kb.n_pb] == list(range(kb.n_pb)), (t, n, a[:kb.n_pb])
        si = seq_pos[s]
        sc = qbars[si][n, qb - g.n_pb] @ kbars[si][n // G].T
        video = [j - kb.n_pb for j in a[kb.n_pb:]]
        sinks = set(range(kb.ns))
        assert sinks <= set(video), (t, n)
        chosen = [j for j in video if j not in sinks]
        assert len(chosen) <= kb.k, (t, n, len(chosen), kb.k)
        best_sinks = sorted(sinks, key=lambda j: (-sc[j], j))[:kb.k - len(chosen)]
        top = set(chosen) | set(best_sinks)
        rest = [j for j in range(kb.nb) if j not in top]
        if top and rest:
            lo = min(top, key=lambda j: sc[j])
            hi = max(rest, key=lambda j: sc[j])
            assert sc[lo] >= sc[hi] - TIE_REL * max(abs(sc[lo]), abs(sc[hi])), (t, n, lo, hi, sc[lo], sc[hi])
        stats["near_tie"] += 1
    return stats


def check_attention(p: orc.Problem, w: synth.Workload, rbits: Sequence[np.ndarray], gpu,
                    items: Sequence[Tuple[int, int]] | None = None, values=None,
                    check: bool = True, oracle_fn=None, block_kv: int = 128) -> Dict[str, float]:
    """GPU o_r against the oracle run on the GPU's selectIdx, for (q-block, head) items.
    `values` replaces the float64 (Q', K', V') decoded from rbits (mix and mxfp4
    precisions); `oracle_fn` replaces the oracle attention (mxfp4: the PNQ one);
    with check=False the errors are returned without asserting the bars."""
    qf, kf, vf = values if values is not None else (synth.bits_to_float64(x, w.dtype) for x in rbits)
    fn = oracle_fn if oracle_fn is not None else orc.attention
    extra = {} if block_kv == 128 else {"block_kv": block_kv}
    ref = fn(p, qf, kf, vf, gpu["idx"], gpu["num"], gpu["scale"], items, **extra)
    o_r = synth.bits_to_float64(gpu["o_r"], w.dtype)
    table = orc.qblock_table(p)
    num = den = 0.0
    mx = 0.0
    for (t, n), rows in ref.items():
        s, g, b = table[t]
        r = orc.block_rows(g, b)
        got = p.head_rows(o_r, s, n)[r.start:r.stop]
        d = got - rows
        mx = max(mx, float(np.max(np.abs(d))))
        num += float(np.sum(d * d))
        den += float(np.sum(rows * rows))
    rel = math.sqrt(num / max(den, 1e-300))
    if check:
        assert mx <= MAX_ABS, f"max abs err {mx}"
        assert rel <= REL_L2, f"rel L2 err {rel}"
    return dict(max_abs=mx, rel_l2=rel, items=len(ref))


def sample_items(p: orc.Problem, rng: np.random.Generator, per_kind: int = 4) -> List[Tuple[int, int]]:
    """Sampled (q-block, head) items covering prefix, partial-prefix, first-frame and sparse blocks."""
    table = orc.qblock_table(p)
    kinds: Dict[str, List[int]] = {"prefix": [], "partial": [], "sink": [], "sparse": [], "last": []}
    for t, (s, g, b) in enumerate(table):
        if b < g.n_pb:
            kinds["partial" if (b == g.n_pb - 1 and g.lp % 128) else "prefix"].append(t)
        elif b - g.n_pb < g.ns:
            kinds["sink"].append(t)
        elif b == g.n_blocks - 1:
            kinds["last"].append(t)
        else:
            kinds["sparse"].append(t)
    items = []
    for name, ts in kinds.items():
        if not ts:
            continue
        for t in rng.choice(ts, size=min(per_kind, len(ts)), replace=False).tolist():
            items.append((int(t), int(rng.integers(0, p.n1))))
    return items
