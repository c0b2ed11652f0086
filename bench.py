#!/usr/bin/env python3
"""Benchmark of the RainFusion v2 block-sparse attention path on B200.

One step = the whole path on one synthetic layer: rf_rearrange (Q, K, V and
the fused block means) -> rf_pool_select -> rf_block_sparse_attn ->
rf_inverse_rearrange, inputs resident in HBM.  The metric is the attention's
kept-block TFLOP/s (FLOPs counted from the selectIdx the step produced) over
the whole step, plus ms per call of every kernel and the attention kernel's
fraction of the measured dense BF16 peak.  The default workload is the largest
single-GPU configuration: the 8x8-aligned grid (21,48,80) with 40 heads at
sparsity 0.8.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload aligned] [--sparsity 0.8]
  python bench.py --impl reference ...   (the CPU oracle on a bounded sample)
  python bench.py --record-traffic ncu_raw.csv --workload aligned [--heads 8]
        (writes the attention kernel's DRAM bytes per launch into profiles/traffic.json)

Multi-GPU (torchrun, one rank per GPU), --mode:
  ulysses      (default for N > 1) one layer sharded by heads: each rank holds
               L/N rows of every head, an NCCL all-to-all gives it every row of
               N1/N query heads (and their key/value heads), the path runs on
               those heads, a second all-to-all returns the output rows; the
               exchanges are inside the timed region ("scaling": "strong");
  independent  every rank runs its own layer, no collective ("scaling": "weak").
Timing is the max over ranks; the value is the kept FLOPs of all ranks over that time.
"""
from __future__ import annotations

import argparse
import csv
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
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")
ORACLE_ITEMS = 320          # sampled (q-block, head) attention items per oracle step


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="aligned", choices=sorted(WORKLOAD_DESC))
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--precision", default="native", choices=["native", "mix", "fp8", "mxfp4"],
                    help="kernel precision (mix: E4M3 Q K^T with per-block scales, 16-bit P V; "
                         "fp8: E4M3 for P V as well; mxfp4: MXFP4 operands with UOS scaling and PNQ)")
    ap.add_argument("--order", default="tile", choices=["tile", "frame_pair"],
                    help="token order of the aligned video (frame_pair: frames paired into 2x8x8 blocks)")
    ap.add_argument("--mode", default="auto", choices=["auto", "plain", "ulysses", "independent"],
                    help="auto: plain at N = 1, ulysses at N > 1")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--block-kv", type=int, default=128, choices=[128, 64],
                    help="64: time the attention with blockShape 128 x 64 on the 64-row halves of the "
                         "step's 128-row selection (expanded once on the host after warm-up; same kept FLOPs)")
    ap.add_argument("--chunks", type=int, default=None,
                    help="head chunks of the host pipeline in the e2e measurement (default: the library's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--oracle-workers", type=int, default=None,
                    help="processes for the CPU oracle (default: every core this process may use)")
    ap.add_argument("--heads", type=int, default=None,
                    help="profiling only: shrink the layer to this many query heads (G kept)")
    ap.add_argument("--record-traffic", default=None, metavar="NCU_RAW_CSV",
                    help="write the attention kernel's DRAM bytes per launch from an ncu raw CSV "
                         "(ncu -i rep --page raw --csv) into profiles/traffic.json, scaled from --heads "
                         "to the workload's heads, and exit")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_sha(name="rf_attn.cu"):
    h = hashlib.sha256()
    for n in (name, "rf_device.cuh"):
        with open(os.path.join(ROOT, "block_sparse_video_rearrange_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_key(workload, sparsity, precision="native", block_kv=128):
    return f"{workload}@{sparsity:g}" + ("" if precision == "native" else "/" + precision) + \
           ("/kv64" if block_kv == 64 else "")


def profiled_traffic(key):
    """DRAM bytes per attention launch recorded in profiles/traffic.json for this
    workload, if the record still describes the current kernel source (else None)."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    with open(TRAFFIC_JSON) as f:
        recs = json.load(f).get("rf_attn_kernel", [])
    sha = kernel_sha()
    for r in recs:
        if r.get("workload") == key and r.get("source_sha") == sha:
            return float(r["dram_bytes_per_launch"])
    return None


def record_traffic(csv_path, key, scale, how):
    """Parse the raw ncu CSV (header row, units row, one row per launch) and store the
    mean DRAM read + write bytes per rf_attn_kernel launch, times `scale`."""
    rows = list(csv.reader(open(csv_path)))
    hdr, units = rows[0], rows[1]
    mult = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    i_name = hdr.index("Kernel Name")
    vals = []
    for r in rows[2:]:
        if "rf_attn_kernel" not in r[i_name]:
            continue
        tot = 0.0
        for m in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            i = hdr.index(m)
            tot += float(r[i].replace(",", "")) * mult[units[i]]
        vals.append(tot)
    if not vals:
        raise SystemExit(f"no rf_attn_kernel launch with DRAM counters in {csv_path}")
    per = float(np.mean(vals)) * scale
    data = {"rf_attn_kernel": []}
    if os.path.exists(TRAFFIC_JSON):
        with open(TRAFFIC_JSON) as f:
            data = json.load(f)
    recs = [r for r in data.get("rf_attn_kernel", []) if not (r.get("workload") == key and
                                                            r.get("source_sha") == kernel_sha())]
    recs.append({"workload": key, "source_sha": kernel_sha(), "dram_bytes_per_launch": round(per),
                 "launches_captured": len(vals), "how": how})
    data["rf_attn_kernel"] = recs
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")
    print(json.dumps(recs[-1]))


# ---------------------------------------------------------------------------------------
# Algorithmic work, counted from the selection the step produced
# ---------------------------------------------------------------------------------------

def kept_flops_from_selection(plan, idx, num):
    """4 * D * (query rows) * (valid key rows) over selected (q-block, head, key block);
    query blocks hold 128 rows, key blocks plan.block_kv (the last prefix block of
    each kind possibly partial)."""
    total = 0
    bk = plan.block_kv
    for si in plan.seq_info_all():
        nblk = si.n_pb + si.nb
        nkv = int(si.n_pb_kv) + int(si.nb_kv)
        lp, npb, npk = int(si.lp), int(si.n_pb), int(si.n_pb_kv)
        qrows = np.full(nblk, 128, dtype=np.int64)
        if npb > 0:
            qrows[npb - 1] = lp - 128 * (npb - 1)
        krows = np.full(nkv + 1, bk, dtype=np.int64)
        if npk > 0:
            krows[npk - 1] = lp - bk * (npk - 1)
        krows[nkv] = 0                                   # -1 entries map here
        t0 = int(si.qblk_offset)
        sel = idx[t0:t0 + nblk].astype(np.int64)
        n = num[t0:t0 + nblk]
        valid = np.arange(sel.shape[-1])[None, None, :] < n[:, :, None]
        sel = np.where(valid & (sel >= 0), sel, nkv)
        kv_rows = krows[sel].sum(axis=-1)                # [nblk, N1]
        total += int((4 * plan.d * qrows[:, None] * kv_rows).sum())
    return total


def algorithmic_bytes(plan, elem=2):
    """Minimum bytes the permute/pool/select steps move: read Q, K, V once, write
    Q', K', V' once, write selectIdx/selectNum; the inverse reads O' and writes O."""
    rows = int(plan.info.rows_total)          # BNSD: B * L, TND: T
    qkv = rows * (plan.n1 + 2 * plan.n2) * plan.d * elem
    t, n, m = plan.select_shapes()[0]
    sel = 4 * t * n * m + 4 * t * n
    inv = 2 * rows * plan.n1 * plan.d * elem
    # precision "mix": the rearrange also writes one-byte copies of Q' and K' and their scales
    quant = rows * (plan.n1 + plan.n2) * plan.d + 4 * t * (plan.n1 + plan.n2) if plan.precision in ("mix", "fp8") else 0
    # precision "fp8": and the transposed one-byte copy of V' (whole blocks) with its exponents
    if plan.precision == "fp8":
        quant += plan.n2 * t * 128 * plan.d + 4 * t * plan.n2
    # precision "mxfp4": the MXFP4-rounded copies of Q', K' and V' (head dim 128: one-byte
    # E4M3 carriers, V' as whole transposed blocks; head dim 64: 16-bit copies)
    if plan.precision == "mxfp4":
        quant = (rows * (plan.n1 + plan.n2) * plan.d + plan.n2 * t * 128 * plan.d if plan.d == 128
                 else rows * (plan.n1 + 2 * plan.n2) * plan.d * 2)
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
# CPU oracle timing on all host cores (the reported baseline and the reference arm)
# ---------------------------------------------------------------------------------------
#
# Every step of the path is independent per key/value head group (its G query heads and
# the key/value head they read), so the oracle's step is split into one task per group
# and run on a pool of single-threaded worker processes.  Each task runs rearrangement,
# pooling and selection of its group in full and the attention on sampled (q-block,
# head) items; the attention time is extrapolated by the kept-FLOP ratio.  The step's
# time is the CPU-seconds of the extrapolated full step divided by the worker count
# (the work divides into many independent items).

_WORKER = {}


def _oracle_worker_init(meta):
    from multiprocessing import shared_memory
    arrays = []
    for name, shape in meta["shm"]:
        shm = shared_memory.SharedMemory(name=name)
        arrays.append((shm, np.ndarray(shape, dtype=np.uint16, buffer=shm.buf)))
    _WORKER.update(meta=meta, arrays=arrays)


def _oracle_group_task(task):
    """One key/value head group: (seconds front, seconds attention sample, kept FLOPs of
    the group's whole step, kept FLOPs of the sampled items)."""
    from oracle import rainfusion as orc
    from block_sparse_video_rearrange_b200 import synth
    grp, n_items, seed = task
    m = _WORKER["meta"]
    G = m["n1"] // m["n2"]
    bnsd = m["layout"] == "BNSD"
    parts = []
    for i, (_, arr) in enumerate(_WORKER["arrays"]):
        h0, h1 = (grp * G, (grp + 1) * G) if i == 0 else (grp, grp + 1)
        parts.append(np.ascontiguousarray(arr[:, h0:h1] if bnsd else arr[:, h0:h1, :]))
    p = orc.make_problem(m["layout"], m["batch"], m["seqs"], G, 1, m["d"], m["sparsity"], m["order"])
    t0 = time.perf_counter()
    rq, rk, rv = (orc.rearrange(p, x) for x in parts)
    qf, kf = synth.bits_to_float64(rq, m["dtype"]), synth.bits_to_float64(rk, m["dtype"])
    qbars, kbars = orc.pooled_means(p, qf, G), orc.pooled_means(p, kf, 1)
    idx, num = orc.select(p, qbars, kbars)
    t_front = time.perf_counter() - t0
    vf = synth.bits_to_float64(rv, m["dtype"])
    rng = np.random.default_rng(seed)
    table = orc.qblock_table(p)
    items = [(int(rng.integers(0, len(table))), int(rng.integers(0, G))) for _ in range(n_items)]
    t1 = time.perf_counter()
    orc.attention(p, qf, kf, vf, idx, num, 1.0 / math.sqrt(m["d"]), items)
    t_attn = time.perf_counter() - t1
    flops_total = orc.kept_flops(p, idx, num)
    flops_sample = 0
    for t, n in items:
        _, g, b = table[t]
        mq = len(orc.block_rows(g, b))
        flops_sample += 4 * m["d"] * mq * sum(len(orc.block_rows(g, int(j))) for j in idx[t, n, :num[t, n]])
    return t_front, t_attn, flops_total, flops_sample


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def usable_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OraclePool:
    """A spawn-context pool of single-threaded processes holding the workload's 16-bit
    inputs in shared memory."""

    def __init__(self, w, bits, workers=None):
        import multiprocessing as mproc
        from multiprocessing import shared_memory
        self.w = w
        self.groups = w.n2 * 1
        self.workers = max(1, min(workers or usable_cores(), self.groups))
        self.shms = []
        shm_meta = []
        for x in bits:
            shm = shared_memory.SharedMemory(create=True, size=max(1, x.nbytes))
            np.ndarray(x.shape, dtype=np.uint16, buffer=shm.buf)[...] = x
            self.shms.append(shm)
            shm_meta.append((shm.name, x.shape))
        meta = dict(shm=shm_meta, layout=w.layout, batch=w.batch, n1=w.n1, n2=w.n2, d=w.d, dtype=w.dtype,
                    sparsity=w.sparsity, order="tile", seqs=[(s.prefix_len, s.t, s.h, s.w) for s in w.seqs])
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        os.environ.update({k: "1" for k in saved})        # one BLAS thread per worker process
        try:
            self.pool = mproc.get_context("spawn").Pool(self.workers, initializer=_oracle_worker_init,
                                                        initargs=(meta,))
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v

    def step(self, items_total, seed):
        """One oracle step over every group, attention on about items_total sampled items.
        Returns (extrapolated step seconds, kept FLOPs, description, wall seconds spent)."""
        per = max(1, round(items_total / self.groups))
        tasks = [(g, per, seed * 1000 + g) for g in range(self.groups)]
        t0 = time.perf_counter()
        res = self.pool.map(_oracle_group_task, tasks, chunksize=1)
        wall = time.perf_counter() - t0
        front = sum(r[0] for r in res)
        attn = sum(r[1] for r in res)
        flops = sum(r[2] for r in res)
        cpu_full = sum(r[0] + r[1] * r[2] / max(1, r[3]) for r in res)
        step_s = cpu_full / self.workers
        desc = (f"{self.groups} key/value head groups on {self.workers} single-threaded processes: "
                f"rearrange+pool+select in full ({front:.1f} CPU-s), attention on {per * self.groups} sampled "
                f"(q-block, head) items ({attn:.1f} CPU-s) extrapolated by kept-FLOP ratio; step time = "
                f"CPU-seconds of the extrapolated full step / {self.workers} processes "
                f"(sample wall time {wall:.1f} s)")
        return step_s, flops, desc, wall

    def close(self):
        self.pool.close()
        self.pool.join()
        for shm in self.shms:
            shm.close()
            shm.unlink()


def cpu_baseline_entry(value, workers, desc, step_s, spent):
    return {"value": value, "unit": "TFLOP/s", "cores": workers, "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": usable_cores(), "threads_per_process": 1,
            "sample": desc, "ms_per_step_extrapolated": round(step_s * 1e3, 1),
            "sample_wall_s": round(spent, 1)}


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


def measure_fp8_gemm_tflops(dev):
    """Context for the mix roofline: a cuBLASLt E4M3 GEMM at 8192^3 (best of 10)."""
    import torch
    try:
        n = 8192
        a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:
        return None


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
    full_heads = w.n1
    if args.heads:
        g = w.n1 // w.n2
        w = synth.Workload(w.name, w.layout, w.dtype, w.batch, w.seqs, args.heads, max(1, args.heads // g), w.d,
                           w.sparsity, w.seed)
    if args.record_traffic:
        scale = full_heads / w.n1
        how = (f"ncu capture of {w.n1} of {full_heads} heads, x{scale:g}" if scale != 1 else "full-size ncu capture")
        record_traffic(args.record_traffic, traffic_key(w.name.split("@")[0], w.sparsity, args.precision,
                                                        args.block_kv), scale, how)
        return 0
    mode = args.mode if args.mode != "auto" else ("plain" if world == 1 else "ulysses")

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

    if mode == "ulysses":
        if world == 1:
            raise SystemExit("--mode ulysses needs torchrun with more than one rank")
        return run_ulysses(args, w, world, rank, dev)

    # Independent layer per rank (weak scaling): same shapes, rank-dependent seed.
    wr = synth.Workload(w.name, w.layout, w.dtype, w.batch, w.seqs, w.n1, w.n2, w.d, w.sparsity, w.seed + 7919 * rank)
    bits = synth.generate_qkv(wr)
    seqs = [(s.prefix_len, s.t, s.h, s.w) for s in w.seqs]
    if args.block_kv == 64 and args.precision != "native":
        raise SystemExit("--block-kv 64 runs native precision only")
    plan = rf.Plan(seqs, w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch, order=args.order,
                   precision=args.precision, block_kv=args.block_kv)
    tdt = plan.torch_dtype
    host = [torch.from_numpy(x.view(np.int16)).view(tdt).pin_memory() for x in bits]
    q, k, v = (h.to(dev) for h in host)
    b = rf.Buffers(plan, dev)
    scale = 1.0 / math.sqrt(w.d)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        rf.rearrange(plan, q, k, v, b.q_r, b.k_r, b.v_r, b.ws)
        if ev is not None:
            ev[1].record(stream)
        rf.pool_select(plan, None, None, b.select_idx, b.select_num, b.ws)
        if ev is not None:
            ev[2].record(stream)
        rf.block_sparse_attn(plan, b.q_r, b.k_r, b.v_r, b.select_idx, b.select_num, scale, b.o_r, b.ws)
        if ev is not None:
            ev[3].record(stream)
        rf.inverse_rearrange(plan, b.o_r, b.o)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    rf.raise_on_device_fault(plan, b.ws, "warm-up")
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
    rf.raise_on_device_fault(plan, b.ws, "timed steps")

    # e2e: pinned host buffers through the public API (rf.rainfusion_attention, which
    # runs head chunks whose copies overlap the compute, then reads the status words);
    # copies inside the timed region, the result back on the host at the end of every step.
    e2e = None
    if args.e2e_steps > 0:
        out_host = None

        def e2e_step():
            nonlocal out_host
            out_host = rf.rainfusion_attention(host[0], host[1], host[2], seqs, w.sparsity, w.layout, scale,
                                               order=args.order, precision=args.precision, chunks=args.chunks,
                                               block_kv=args.block_kv)
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
        from block_sparse_video_rearrange_b200.pipeline import default_chunks
        n_sets = 1 if (args.chunks or default_chunks(w.n2)) == 1 else 2
        d2h = out_host.numel() * out_host.element_size() + 8 * n_sets     # output + status words
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
        extra_roof = {}
        if args.precision == "mix":
            # Q K^T (half the kept FLOPs) at the fp8 rate, taken as 2x the measured
            # 16-bit rate (the nominal 4.5 / 2.25 PFLOP/s ratio), P V at the 16-bit
            # rate: the harmonic combination is 4/3 of the 16-bit peak.
            bf = peak
            peak = round(bf * 4.0 / 3.0, 1)
            peak_note += "; mix: QK^T at 2x (fp8, nominal ratio x measured bf16), PV at 1x -> 4/3 x"
            f8 = measure_fp8_gemm_tflops(dev)
            if f8:
                alt = 1.0 / (0.5 / f8 + 0.5 / bf)
                extra_roof = {"fp8_gemm_tflops_measured_here": round(f8, 1),
                              "peak_with_measured_fp8": round(alt, 1), "frac_with_measured_fp8": round(achieved / alt, 4)}
        if args.precision == "fp8":
            # both products at the fp8 rate: 2x the measured 16-bit rate (nominal 4.5 / 2.25)
            bf = peak
            peak = round(bf * 2.0, 1)
            peak_note += "; fp8: QK^T and PV at 2x (fp8, nominal ratio x measured bf16)"
            f8 = measure_fp8_gemm_tflops(dev)
            if f8:
                extra_roof = {"fp8_gemm_tflops_measured_here": round(f8, 1), "peak_with_measured_fp8": round(f8, 1),
                              "frac_with_measured_fp8": round(achieved / f8, 4)}
        if args.precision == "mxfp4" and w.d == 128:
            # both products on the FP8 tensor cores (MXFP4 values carried exactly in E4M3)
            peak = round(peak * 2.0, 1)
            peak_note += "; mxfp4 at head dim 128: both products on E4M3 carriers at 2x (fp8, nominal ratio)"
        elif args.precision == "mxfp4":
            peak_note += "; mxfp4 at head dim 64: both products run on the 16-bit tensor cores -> 1x"
        front_bytes, inv_bytes = algorithmic_bytes(plan)
        front_ms = float(np.mean(per[:, 0] + per[:, 1]))
        inv_ms = float(np.mean(per[:, 3]))
        value = flops_all / (ms_step * 1e-3) / 1e12
        traffic = (profiled_traffic(traffic_key(w.name.split("@")[0], w.sparsity, args.precision, args.block_kv))
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
            "dtype": {"mix": "e4m3+", "fp8": "e4m3 (from ", "mxfp4": "mxfp4 on "}.get(args.precision, "")
                     + ("bf16" if w.dtype == "bf16" else "fp16") + (")" if args.precision == "fp8" else ""),
            "data": "synthetic (seeded smooth-field + noise per 8x8 cell; no real activations available)",
            "config": {"workload": WORKLOAD_DESC[w.name.split("@")[0]] + (f" [reduced to {w.n1} heads]" if args.heads else ""),
                       "sparsity": w.sparsity,
                       **({"token_order": args.order} if args.order != "tile" else {}),
                       **({"precision": "mix (E4M3 QK^T, 16-bit PV)"} if args.precision == "mix" else {}),
                       **({"precision": "fp8 (E4M3 QK^T and PV; V on power-of-two block scales)"}
                          if args.precision == "fp8" else {}),
                       **({"block_shape": "128 x 64 (64-row key blocks ranked against 128-row query "
                                          "blocks)"} if args.block_kv == 64 else {}),
                       **({"precision": "mxfp4 (UOS Qmax 7.25, PNQ; values carried in E4M3 at head dim 128)"}
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
                         "peak_source": peak_note, **extra_roof},
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
            pool = OraclePool(wr, bits, args.oracle_workers)
            try:
                step_s, oflops, desc, spent = pool.step(ORACLE_ITEMS, seed=0)
            finally:
                pool.close()
            line["cpu_baseline"] = cpu_baseline_entry(round(oflops / step_s / 1e12, 6), pool.workers, desc,
                                                      step_s, spent)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_ulysses(args, w, world, rank, dev):
    """One layer sharded by heads over the process group (strong scaling): row slices
    in, NCCL all-to-all, the path on N1/P heads, all-to-all back, all timed."""
    import torch
    import torch.distributed as dist
    from block_sparse_video_rearrange_b200 import rf, synth, ulysses
    if args.block_kv != 128:
        raise SystemExit("--mode ulysses runs blockShape 128 x 128")
    seqs = [(s.prefix_len, s.t, s.h, s.w) for s in w.seqs]
    ulysses.check_shardable(seqs, w.n1, w.n2, w.layout, w.batch, world)
    bits = synth.generate_qkv(w)                    # the same layer on every rank
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    axis = 2 if w.layout == "BNSD" else 0
    rows = bits[0].shape[axis] // world
    host = [torch.from_numpy(np.ascontiguousarray(np.take(x, range(rank * rows, (rank + 1) * rows), axis=axis))
                             .view(np.int16)).view(tdt).pin_memory() for x in bits]
    del bits
    q, k, v = (h.to(dev) for h in host)
    layer = ulysses.UlyssesAttention(seqs, w.n1, w.n2, w.d, w.layout, w.dtype, w.sparsity, batch=w.batch,
                                     order=args.order, precision=args.precision, device=dev)
    scale = 1.0 / math.sqrt(w.d)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        layer(q, k, v, scale, check=False)
    torch.cuda.synchronize(dev)
    rf.raise_on_device_fault(layer.plan, layer.bufs.ws, "warm-up")
    flops = kept_flops_from_selection(layer.plan, layer.bufs.select_idx.cpu().numpy(),
                                      layer.bufs.select_num.cpu().numpy())
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if (rank == 0 and not args.no_clocks) else None
    dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        layer(q, k, v, scale, events=evs[i], check=False)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop() if sampler else None
    dist.barrier()
    rf.raise_on_device_fault(layer.plan, layer.bufs.ws, "timed steps")
    ms_step = t_start.elapsed_time(t_end) / args.steps
    per = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(6)] for e in evs])   # [steps, 6]
    attn_ms = float(np.mean(per[:, 3]))
    a2a_ms = float(np.mean(per[:, 0] + per[:, 5]))

    # e2e: this rank's row slices from pinned host memory, the layer, the output back
    e2e = None
    if args.e2e_steps > 0:
        def e2e_step():
            qd, kd, vd = (x.to(dev, non_blocking=True) for x in host)
            o = layer(qd, kd, vd, scale)                 # reads the status words (synchronises)
            out = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
            out.copy_(o, non_blocking=True)
            stream.synchronize()
            return out
        for _ in range(2):
            out_host = e2e_step()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            out_host = e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e = (e0.elapsed_time(e1) / args.e2e_steps, sum(x.numel() * x.element_size() for x in host),
               out_host.numel() * out_host.element_size() + 8)
    (ms_max, attn_max, a2a_max, e2e_max), (flops_all,) = reduce_over_ranks(
        [ms_step, attn_ms, a2a_ms, e2e[0] if e2e else 0.0], [float(flops)], dev)
    if rank == 0:
        peaks, peak_src = load_peaks()
        achieved = flops / (attn_ms * 1e-3) / 1e12        # rank 0's own launches
        peak = peaks["bf16_tflops"]
        line = {
            "metric": METRIC, "value": round(flops_all / (ms_max * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_max, 4),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": {"mix": "e4m3+", "mxfp4": "mxfp4 on "}.get(args.precision, "") + ("bf16" if w.dtype == "bf16" else "fp16"),
            "data": "synthetic (seeded smooth-field + noise per 8x8 cell; no real activations available)",
            "config": {"workload": WORKLOAD_DESC[w.name.split("@")[0]], "sparsity": w.sparsity,
                       "global_batch": w.batch, "seq_len": int(layer.plan.info.rows_total),
                       "parallelism": f"Ulysses head sharding x{world} (NCCL all-to-all in and out, timed)",
                       "l2": "inputs larger than L2",
                       "kept_tflop_per_step": round(flops_all / 1e12, 4)},
            "kernels_ms": {"all_to_all_in_out": round(float(np.mean(per[:, 0] + per[:, 5])), 4),
                           "rf_rearrange": round(float(np.mean(per[:, 1])), 4),
                           "rf_pool_select": round(float(np.mean(per[:, 2])), 4),
                           "rf_block_sparse_attn": round(attn_ms, 4),
                           "rf_inverse_rearrange": round(float(np.mean(per[:, 4])), 4),
                           "max_over_ranks": {"rf_block_sparse_attn": round(attn_max, 4),
                                              "all_to_all_in_out": round(a2a_max, 4)}},
            "attn_ms_per_call": round(attn_ms, 4),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "traffic": None,
                         "peak_source": f"{peak_src} bf16_tflops (burst); rank 0's attention launches"},
            "gpu_launches": 5 * args.steps,
        }
        if e2e:
            line["e2e"] = {"value": round(flops_all / (e2e_max * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                           "ms_per_step": round(e2e_max, 3), "h2d_bytes_per_step": e2e[1],
                           "d2h_bytes_per_step": e2e[2], "per": "rank (each rank copies its own row slices)"}
        if clocks:
            line["clocks"] = clocks
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


def run_reference(args, w, world):
    """The CPU oracle as the reference arm: each step is a bounded sample of the
    same workload, extrapolated to a whole step, run on all host cores."""
    from block_sparse_video_rearrange_b200 import synth
    bits = synth.generate_qkv(w)
    pool = OraclePool(w, bits, args.oracle_workers)
    try:
        for i in range(args.warmup):
            pool.step(pool.groups, seed=100 + i)          # one item per group
        times, walls, flops, desc = [], [], 0, ""
        for i in range(args.steps):
            step_s, flops, desc, wall = pool.step(ORACLE_ITEMS, seed=i)
            times.append(step_s)
            walls.append(wall)
    finally:
        pool.close()
    ms = float(np.mean(times)) * 1e3
    value = flops / (ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 1),
            "ms_per_step_kind": "extrapolated from a bounded sample (see cpu_baseline.sample)",
            "sample_wall_ms_per_step": round(float(np.mean(walls)) * 1e3, 1),
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
            "config": {"workload": WORKLOAD_DESC[w.name.split("@")[0]], "sparsity": w.sparsity},
            "cpu_baseline": cpu_baseline_entry(round(value, 6), pool.workers, desc, ms * 1e-3,
                                               float(np.mean(walls))),
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
