#!/usr/bin/env python3
"""Benchmark of the RainFusion v2 block-sparse attention path on B200.

One step = the whole path on one synthetic layer: rf_rearrange (Q, K, V and
the fused block means) -> rf_pool_select -> rf_block_sparse_attn ->
rf_inverse_rearrange, inputs resident in HBM.  The metric is the attention's
kept-block TFLOP/s (FLOPs counted from the selectIdx the step produced) over
the whole step, plus ms per call of every kernel and the attention kernel's
fraction of the measured dense BF16 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan] [--sparsity 0.8]
  python bench.py --impl reference ...   (the CPU oracle on a bounded sample)

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
layer (weak scaling; the path has no data exchange), timing is the max over
ranks, the value is the FLOPs of all ranks over that time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn ms/call & kept-block TFLOP/s (% BF16 peak) at sparsity 0.8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD_DESC = {
    "tiny": "Tiny: B=1 N=2 D=64 bf16 BNSD, text 128 + video (9,16,32)",
    "wan": "Wan2.2-shaped layer: B=1 N=40 D=128 bf16 BNSD, text 512 + video (21,30,52)",
    "minimax": "MiniMax-H3-shaped layer: B=1 N=24 D=128 bf16 BNSD, text 256 + video (62,24,42)",
    "aligned": "Aligned grid: B=1 N=40 D=128 bf16 BNSD, text 512 + video (21,48,80)",
    "tnd_gqa": "TND varlen GQA: N1=32 N2=8 D=128 fp16, seqs (256;13,32,48) and (384;21,24,40)",
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="wan", choices=sorted(WORKLOAD_DESC))
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--precision", default="native", choices=["native", "mix", "mxfp4"],
                    help="kernel precision (mix: E4M3 Q K^T with per-block scales, 16-bit P V; "
                         "mxfp4: MXFP4 operands with UOS scaling and PNQ, on the 16-bit tensor cores)")
    ap.add_argument("--order", default="tile", choices=["tile", "frame_pair"],
                    help="token order of the aligned video (frame_pair: frames paired into 2x8x8 blocks)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--block-kv", type=int, default=128, choices=[128, 64],
                    help="64: time the attention with blockShape 128 x 64 on the 64-row halves of the "
                         "step's 128-row selection (expanded once on the host after warm-up; same kept FLOPs)")
    ap.add_argument("--chunks", type=int, default=None,
                    help="head chunks of the host pipeline in the e2e measurement (default: the library's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--heads", type=int, default=None,
                    help="profiling only: shrink the layer to this many query heads (G kept)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_sha(name):
    with open(os.path.join(ROOT, "block_sparse_video_rearrange_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(workload, sparsity, tag=""):
    """DRAM bytes per attention launch from the committed ncu summary, if it still
    describes the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    sha = kernel_sha("rf_attn.cu")
    with open(path) as f:
        for line in f:
            parts = line.strip().strip("|").split("|")
            parts = [p.strip() for p in parts]
            if len(parts) >= 5 and parts[0] == "rf_attn_kernel" and parts[1] == f"{workload}@{sparsity:g}{tag}" \
                    and parts[2] == sha:
                try:
                    return float(parts[3])
                except ValueError:
                    return None
    return None


# ---------------------------------------------------------------------------------------
# Algorithmic work, counted from the selection the step produced
# ---------------------------------------------------------------------------------------

def kept_flops_from_selection(plan, idx, num):
    """4 * D * (query rows) * (valid key rows) over selected (q-block, head, key block)."""
    total = 0
    for si in plan.seq_info_all():
        nblk = si.n_pb + si.nb
        lp, npb = int(si.lp), int(si.n_pb)
        rows = np.full(nblk + 1, 128, dtype=np.int64)
        rows[npb - 1] = lp - 128 * (npb - 1) if npb > 0 else 128
        rows[nblk] = 0                                   # -1 entries map here
        t0 = int(si.qblk_offset)
        sel = idx[t0:t0 + nblk].astype(np.int64)
        n = num[t0:t0 + nblk]
        valid = np.arange(sel.shape[-1])[None, None, :] < n[:, :, None]
        sel = np.where(valid & (sel >= 0), sel, nblk)
        kv_rows = rows[sel].sum(axis=-1)                 # [nblk, N1]
        q_rows = rows[:nblk][:, None]
        total += int((4 * plan.d * q_rows * kv_rows).sum())
    return total


def expand_selection_kv64(plan, idx, num, width):
    """The 128-row key-block selection rewritten over 64-row key blocks (every
    selected block becomes the one or two 64-row blocks inside it, in order)."""
    infos = plan.seq_info_all()
    T, N, _ = idx.shape
    out = np.full((T, N, width), -1, dtype=np.int32)
    cnt = np.zeros((T, N), dtype=np.int32)
    owner = []                                  # sequence of every global query block
    for si in infos:
        owner += [si] * (int(si.n_pb) + int(si.nb))
    if plan.layout == "BNSD":
        owner *= plan.batch                     # one geometry for every batch element
    for t in range(T):
        si = owner[t]
        lp, n_pb = int(si.lp), int(si.n_pb)
        n_pb64 = -(-lp // 64)
        for n in range(N):
            row = []
            for bb in idx[t, n, :num[t, n]]:
                bb = int(bb)
                if bb < 0:
                    continue
                if bb < n_pb:
                    row.append(2 * bb)
                    if 128 * bb + 64 < lp:
                        row.append(2 * bb + 1)
                else:
                    i = bb - n_pb
                    row += [n_pb64 + 2 * i, n_pb64 + 2 * i + 1]
            out[t, n, :len(row)] = row
            cnt[t, n] = len(row)
    return out, cnt


def algorithmic_bytes(plan, elem=2):
    """Minimum bytes the permute/pool/select steps move: read Q, K, V once, write
    Q', K', V' once, write selectIdx/selectNum; the inverse reads O' and writes O."""
    rows = int(plan.info.rows_total)          # BNSD: B * L, TND: T
    qkv = rows * (plan.n1 + 2 * plan.n2) * plan.d * elem
    t, n, m = plan.select_shapes()[0]
    sel = 4 * t * n * m + 4 * t * n
    inv = 2 * rows * plan.n1 * plan.d * elem
    # precision "mix": the rearrange also writes one-byte copies of Q' and K' and their scales
    quant = rows * (plan.n1 + plan.n2) * plan.d + 4 * t * (plan.n1 + plan.n2) if plan.precision == "mix" else 0
    # precision "mxfp4": 16-bit MXFP4-rounded copies of Q', K' and V'
    if plan.precision == "mxfp4":
        quant = rows * (plan.n1 + 2 * plan.n2) * plan.d * 2
    return 2 * qkv + sel + quant, inv


# ---------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.proc, self.lines = index, None, []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for name, flag in zip(names, parts[3:7]):
                if flag.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------------------
# CPU oracle timing (the reported baseline and the reference arm)
# ---------------------------------------------------------------------------------------

def oracle_step_sample(w, bits, budget_items=24, seed=0):
    """Times the CPU oracle on a bounded sample of one step and extrapolates.

    Rearrangement, pooling and selection run in full over every head; the
    attention runs on `budget_items` sampled (q-block, head) items and its time
    is scaled by the kept-FLOP ratio.  Returns (seconds for a whole step,
    kept FLOPs of the whole step, description)."""
    from oracle import rainfusion as orc
    from block_sparse_video_rearrange_b200 import synth
    seqs = [(s.prefix_len, s.t, s.h, s.w) for s in w.seqs]
    p = orc.make_problem(w.layout, w.batch, seqs, w.n1, w.n2, w.d, w.sparsity)
    t0 = time.perf_counter()
    rq, rk, rv = (orc.rearrange(p, x) for x in bits)
    qf, kf = synth.bits_to_float64(rq, w.dtype), synth.bits_to_float64(rk, w.dtype)
    qbars, kbars = orc.pooled_means(p, qf, w.n1), orc.pooled_means(p, kf, w.n2)
    idx, num = orc.select(p, qbars, kbars)
    t_front = time.perf_counter() - t0
    vf = synth.bits_to_float64(rv, w.dtype)
    rng = np.random.default_rng(seed)
    table = orc.qblock_table(p)
    items = [(int(rng.integers(0, len(table))), int(rng.integers(0, w.n1))) for _ in range(budget_items)]
    t1 = time.perf_counter()
    orc.attention(p, qf, kf, vf, idx, num, 1.0 / math.sqrt(w.d), items)
    t_attn = time.perf_counter() - t1
    flops_total = orc.kept_flops(p, idx, num)
    flops_sample = 0
    for t, n in items:
        s, g, b = table[t]
        mq = len(orc.block_rows(g, b))
        flops_sample += 4 * w.d * mq * sum(len(orc.block_rows(g, int(j))) for j in idx[t, n, :num[t, n]])
    step_s = t_front + t_attn * flops_total / max(1, flops_sample)
    desc = (f"rearrange+pool+select in full ({t_front:.1f} s); attention on {budget_items} sampled "
            f"(q-block, head) items ({t_attn:.1f} s), extrapolated by kept-FLOP ratio")
    return step_s, flops_total, desc, t_front + t_attn


def reduce_over_ranks(maxima, sums, device):
    """Times: the max over ranks (the job ends when the slowest rank does);
    work: the sum over ranks.  Every rank calls this with the same layout."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(maxima), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    u = torch.tensor(list(sums), dtype=torch.float64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()], [float(x) for x in u.tolist()]


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------------------
# Main
# ---------------------------------------------------------------------------------------

def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from block_sparse_video_rearrange_b200 import synth
    w = synth.workload(args.workload, args.sparsity)
    if args.heads:
        g = w.n1 // w.n2
        w = synth.Workload(w.name, w.layout, w.dtype, w.batch, w.seqs, args.heads, max(1, args.heads // g), w.d,
                           w.sparsity, w.seed)
    sparsity = w.sparsity

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, w, world)

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    from block_sparse_video_rearrange_b200 import rf

    # Independent layer per rank (weak scaling): same shapes, rank-dependent seed.
    wr = synth.Workload(w.name, w.layout, w.dtype, w.batch, w.seqs, w.n1, w.n2, w.d, w.sparsity, w.seed + 7919 * rank)
    bits = synth.generate_qkv(wr)
    seqs = [(s.prefix_len, s.t, s.h, s.w) for s in w.seqs]
    plan = rf.Plan(seqs, w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch, order=args.order,
                   precision=args.precision)
    tdt = plan.torch_dtype
    host = [torch.from_numpy(x.view(np.int16)).view(tdt).pin_memory() for x in bits]
    q, k, v = (h.to(dev) for h in host)
    b = rf.Buffers(plan, dev)
    scale = 1.0 / math.sqrt(w.d)
    stream = torch.cuda.current_stream(dev)

    kv64 = None   # --block-kv 64: (plan, selectIdx, selectNum, workspace) over 64-row key blocks

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        rf.rearrange(plan, q, k, v, b.q_r, b.k_r, b.v_r, b.ws)
        if ev is not None:
            ev[1].record(stream)
        rf.pool_select(plan, None, None, b.select_idx, b.select_num, b.ws)
        if ev is not None:
            ev[2].record(stream)
        if kv64 is None:
            rf.block_sparse_attn(plan, b.q_r, b.k_r, b.v_r, b.select_idx, b.select_num, scale, b.o_r, b.ws)
        else:
            rf.block_sparse_attn(kv64[0], b.q_r, b.k_r, b.v_r, kv64[1], kv64[2], scale, b.o_r, kv64[3])
        if ev is not None:
            ev[3].record(stream)
        rf.inverse_rearrange(plan, b.o_r, b.o)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if args.block_kv == 64:
        if args.precision != "native":
            raise SystemExit("--block-kv 64 runs native precision only")
        p64 = rf.Plan(seqs, w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch, order=args.order,
                      block_kv=64)
        i64, n64 = expand_selection_kv64(plan, b.select_idx.cpu().numpy(), b.select_num.cpu().numpy(),
                                         int(p64.info.max_kv_blocks))
        kv64 = (p64, torch.from_numpy(i64).to(dev), torch.from_numpy(n64).to(dev),
                torch.zeros(p64.workspace_bytes, dtype=torch.uint8, device=dev))
        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize(dev)
    st, flags = rf.check_device_status(plan, b.ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {st} {flags}")
    flops = kept_flops_from_selection(plan, b.select_idx.cpu().numpy(), b.select_num.cpu().numpy())
    launches_per_step = 5 if any(not si.dense for si in plan.seq_info_all()) else 4

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if (rank == 0 and not args.no_clocks) else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])  # [steps, 4]
    st, flags = rf.check_device_status(plan, b.ws)
    if st == 0 and kv64 is not None:
        st, flags = rf.check_device_status(kv64[0], kv64[3])
    if st != 0:
        raise RuntimeError(f"device status after timing: {st} {flags}")

    # e2e: pinned host buffers through the public API (rf.rainfusion_attention, which
    # runs head chunks whose copies overlap the compute); copies inside the timed region,
    # the result back on the host at the end of every step.
    e2e = None
    # the public call has no 128 x 64 selection, so --block-kv 64 times the kernels only
    if args.e2e_steps > 0 and kv64 is None:
        out_host = None

        def e2e_step():
            nonlocal out_host
            out_host = rf.rainfusion_attention(host[0], host[1], host[2], seqs, w.sparsity, w.layout, scale,
                                               order=args.order, precision=args.precision, chunks=args.chunks)
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
        h2d = sum(x.numel() * x.element_size() for x in host)
        d2h = out_host.numel() * out_host.element_size()
        e2e = (e2e_ms, h2d, d2h)

    ms_step = total_ms / args.steps
    attn_ms = float(np.mean(per[:, 2]))
    if world > 1:
        (ms_step, attn_ms, e2e_max), (flops_all,) = reduce_over_ranks(
            [ms_step, attn_ms, e2e[0] if e2e else 0.0], [float(flops)], dev)
        if e2e:
            e2e = (e2e_max, e2e[1], e2e[2])
    else:
        flops_all = float(flops)

    if rank == 0:
        peaks, peak_src = load_peaks()
        achieved = flops / (attn_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        peak_note = f"{peak_src} bf16_tflops (burst)" + (" x1.0 (fp16 dense rate = bf16)" if w.dtype == "fp16" else "")
        if args.precision == "mix":
            # Q K^T (half the kept FLOPs) at the fp8 rate, taken as 2x the measured
            # 16-bit rate (the nominal 4.5 / 2.25 PFLOP/s ratio), P V at the 16-bit
            # rate: the harmonic combination is 4/3 of the 16-bit peak.
            peak = round(peak * 4.0 / 3.0, 1)
            peak_note += "; mix: QK^T at 2x (fp8, nominal ratio), PV at 1x -> 4/3 x"
        if args.precision == "mxfp4":
            peak_note += "; mxfp4: both products run on the 16-bit tensor cores -> 1x"
        front_bytes, inv_bytes = algorithmic_bytes(plan)
        front_ms = float(np.mean(per[:, 0] + per[:, 1]))
        inv_ms = float(np.mean(per[:, 3]))
        value = flops_all / (ms_step * 1e-3) / 1e12
        traffic = (profiled_traffic(w.name.split("@")[0], sparsity,
                                    ("" if args.precision == "native" else "/" + args.precision)
                                    + ("/kv64" if args.block_kv == 64 else ""))
                   if args.order == "tile" and not args.heads else None)
        line = {
            "metric": METRIC,
            "value": round(value, 3),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": max(3, args.warmup),
            "ms_per_step": round(ms_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": {"mix": "e4m3+", "mxfp4": "mxfp4 on "}.get(args.precision, "") + ("bf16" if w.dtype == "bf16" else "fp16"),
            "data": "synthetic (seeded smooth-field + noise per 8x8 cell; no real activations available)",
            "config": {"workload": WORKLOAD_DESC[w.name.split("@")[0]] + (f" [reduced to {w.n1} heads]" if args.heads else ""),
                       "sparsity": sparsity,
                       **({"token_order": args.order} if args.order != "tile" else {}),
                       **({"precision": "mix (E4M3 QK^T, 16-bit PV)"} if args.precision == "mix" else {}),
                       **({"block_shape": "128 x 64 (attention on the 64-row halves of the step's 128-row "
                                          "selection, expanded once after warm-up)"} if args.block_kv == 64 else {}),
                       **({"precision": "mxfp4 (UOS Qmax 7.25, PNQ; MXFP4 values on the 16-bit tensor cores)"}
                          if args.precision == "mxfp4" else {}),
                       "global_batch": w.batch * world, "seq_len": int(plan.info.rows_total),
                       "parallelism": f"independent layer per GPU x{world}",
                       "l2": "inputs larger than L2 (Q+K+V %.2f GB vs 126 MB)" % (
                           sum(x.numel() * x.element_size() for x in host) / 1e9),
                       "kept_tflop_per_step_per_gpu": round(flops / 1e12, 4)},
            "kernels_ms": {"rf_rearrange": round(float(np.mean(per[:, 0])), 4),
                           "rf_pool_select": round(float(np.mean(per[:, 1])), 4),
                           "rf_block_sparse_attn": round(attn_ms, 4),
                           "rf_inverse_rearrange": round(inv_ms, 4)},
            "attn_ms_per_call": round(attn_ms, 4),
            "attn_tflops": round(achieved, 2),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4),
                         "traffic": traffic,
                         "peak_source": peak_note},
            "hbm_roofline": {"kernels": "rf_rearrange + rf_pool_select", "achieved": round(front_bytes / (front_ms * 1e-3) / 1e9, 1),
                             "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": round(front_bytes / (front_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                             "algorithmic_bytes": front_bytes,
                             "inverse_gbs": round(inv_bytes / (inv_ms * 1e-3) / 1e9, 1)},
            "gpu_launches": launches_per_step * args.steps,
        }
        if e2e:
            line["e2e"] = {"value": round(flops_all / (e2e[0] * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                           "ms_per_step": round(e2e[0], 3), "h2d_bytes_per_step": e2e[1],
                           "d2h_bytes_per_step": e2e[2]}
        if clocks:
            line["clocks"] = clocks
        if world == 1 and not args.no_cpu_baseline:
            del q, k, v
            # about 10 s of CPU work: the front steps in full, 300 attention items
            step_s, oflops, desc, spent = oracle_step_sample(wr, bits, budget_items=300)
            line["cpu_baseline"] = {"value": round(oflops / step_s / 1e12, 6), "unit": "TFLOP/s",
                                    "cores": oracle_threads(), "kind": "oracle",
                                    "sample": desc, "ms_per_step_extrapolated": round(step_s * 1e3, 1),
                                    "cpu_seconds_spent": round(spent, 1)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_reference(args, w, world):
    """The CPU oracle as the reference arm: each step is a bounded sample of the
    same workload, extrapolated to a whole step."""
    from block_sparse_video_rearrange_b200 import synth
    bits = synth.generate_qkv(w)
    for i in range(args.warmup):
        oracle_step_sample(w, bits, budget_items=2, seed=100 + i)
    times, flops, desc = [], 0, ""
    for i in range(args.steps):
        step_s, flops, desc, _ = oracle_step_sample(w, bits, budget_items=4, seed=i)
        times.append(step_s)
    ms = float(np.mean(times)) * 1e3
    value = flops / (ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": WORKLOAD_DESC[w.name.split("@")[0]], "sparsity": w.sparsity},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
