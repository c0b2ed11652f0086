"""Ulysses sequence parallelism around the RainFusion path (one process per GPU).

"RainFusion Attention" user guide, "Requirements and compatibility": the
kernel needs the complete key sequence to rank key blocks, so it runs under
Ulysses sequence parallelism (ring degree 1) and not under ring attention.
Under Ulysses each rank holds an equal slice of the token rows of every head;
one all-to-all gives each rank every row of its share of the heads, the whole
RainFusion path (rearrange, pooling, selection, attention, inverse) runs on
those heads unchanged, and a second all-to-all returns the output to the row
slices.  Nothing inside the path exchanges data: ranking and attention are
independent per (sequence, head), and a query head and its key/value head
stay on the same rank when both head counts divide by the world size.

Head h of query, key and value goes to rank h // (heads / world), so rank r
owns query heads [r*N1/P, (r+1)*N1/P) and key/value heads [r*N2/P, (r+1)*N2/P);
with N1 = G*N2 query head n reads key/value head n // G, which is on the same
rank.  Rows are split into P equal contiguous slices in the caller's layout:
BNSD [B, N, L, D] by L (every batch element alike), TND [T, N, D] by T (the
packed rows of all sequences together), so L (BNSD) or T (TND) must divide
by the world size.

The exchanges are torch.distributed all-to-alls (NCCL over NVLink on GPUs,
gloo on CPU for the tests); the path itself is the CUDA library, called
through `rf` exactly as on one GPU.
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import rf


def _world(group) -> Tuple[int, int]:
    return dist.get_world_size(group), dist.get_rank(group)


def seq_to_head(x: torch.Tensor, layout: str, group=None) -> torch.Tensor:
    """All-to-all from this rank's row slice of every head to every row of this
    rank's heads.  BNSD [B, N, L/P, D] -> [B, N/P, L, D]; TND [T/P, N, D] -> [T, N/P, D]."""
    world, _ = _world(group)
    if layout == "BNSD":
        b, n, ls, d = x.shape
        if n % world:
            raise ValueError(f"{n} heads do not split over {world} ranks")
        send = x.reshape(b, world, n // world, ls, d).permute(1, 0, 2, 3, 4).contiguous()
        recv = torch.empty_like(send)                         # [P (source rank), B, N/P, L/P, D]
        dist.all_to_all_single(recv, send, group=group)
        return recv.permute(1, 2, 0, 3, 4).reshape(b, n // world, world * ls, d)
    if layout == "TND":
        ts, n, d = x.shape
        if n % world:
            raise ValueError(f"{n} heads do not split over {world} ranks")
        send = x.reshape(ts, world, n // world, d).permute(1, 0, 2, 3).contiguous()
        recv = torch.empty_like(send)                         # [P (source rank), T/P, N/P, D]
        dist.all_to_all_single(recv, send, group=group)
        return recv.reshape(world * ts, n // world, d)
    raise ValueError(f"unknown layout {layout}")


def head_to_seq(x: torch.Tensor, layout: str, group=None) -> torch.Tensor:
    """Inverse of seq_to_head: BNSD [B, N/P, L, D] -> [B, N, L/P, D]; TND [T, N/P, D] -> [T/P, N, D]."""
    world, _ = _world(group)
    if layout == "BNSD":
        b, nh, l, d = x.shape
        if l % world:
            raise ValueError(f"{l} rows do not split over {world} ranks")
        send = x.reshape(b, nh, world, l // world, d).permute(2, 0, 1, 3, 4).contiguous()
        recv = torch.empty_like(send)                         # [P (source head group), B, N/P, L/P, D]
        dist.all_to_all_single(recv, send, group=group)
        return recv.permute(1, 0, 2, 3, 4).reshape(b, world * nh, l // world, d)
    if layout == "TND":
        t, nh, d = x.shape
        if t % world:
            raise ValueError(f"{t} rows do not split over {world} ranks")
        send = x.reshape(world, t // world, nh, d).contiguous()
        recv = torch.empty_like(send)                         # [P (source head group), T/P, N/P, D]
        dist.all_to_all_single(recv, send, group=group)
        return recv.permute(1, 0, 2, 3).reshape(t // world, world * nh, d)
    raise ValueError(f"unknown layout {layout}")


def check_shardable(seqs: Sequence[Tuple[int, int, int, int]], n1: int, n2: int, layout: str,
                    batch: int, world: int) -> None:
    """Raise ValueError unless both head counts and the row count divide by the world size."""
    if n1 % world or n2 % world:
        raise ValueError(f"heads ({n1}, {n2}) must both divide by the world size {world}")
    if layout == "BNSD":
        rows = seqs[0][0] + seqs[0][1] * seqs[0][2] * seqs[0][3]
    else:
        rows = sum(p + t * h * w for (p, t, h, w) in seqs)
    if rows % world:
        raise ValueError(f"{rows} rows per head must divide by the world size {world}")


class UlyssesAttention:
    """RainFusion attention of one layer sharded by heads over a process group.

    Called with this rank's row slices of q, k, v (original token order; BNSD
    [B, N1, L/P, D] and [B, N2, L/P, D], or TND [T/P, N1, D] and [T/P, N2, D]
    on this rank's GPU); returns this rank's row slice of the output.  The plan
    and the device buffers (for N1/P and N2/P heads) are made once.

    `path`, when given, replaces the CUDA path on the rank's heads: a callable
    (plan, qh, kh, vh, scale) -> output heads in the layout of qh.  It exists
    so that the exchange and the reassembly can be tested on CPU ranks with a
    stand-in computation; without it every step runs in librf.
    """

    def __init__(self, seqs: Sequence[Tuple[int, int, int, int]], n1: int, n2: int, d: int,
                 layout: str = "BNSD", dtype: str = "bf16", sparsity: float = 0.8, batch: int = 1,
                 group=None, order: str = "tile", precision: str = "native", device=None,
                 path: Optional[Callable] = None):
        world, _ = _world(group)
        check_shardable(seqs, n1, n2, layout, batch, world)
        self.group, self.layout, self.world = group, layout, world
        self.plan = rf.Plan(seqs, n1 // world, n2 // world, d, layout, dtype, sparsity, batch=batch,
                            order=order, precision=precision)
        self.path = path
        self.bufs = rf.Buffers(self.plan, device if device is not None else "cuda") if path is None else None

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 scale: Optional[float] = None, events: Optional[Sequence] = None,
                 check: bool = True) -> torch.Tensor:
        """One layer.  `events`, if given, are 7 CUDA events recorded on the current
        stream around the phases: exchange in, rearrange, pool_select, attention,
        inverse, exchange out.  check=True synchronises after the call and raises
        RfError(RF_ERR_DEVICE_FAULT) if a kernel recorded a fault (check=False
        leaves the status words for a later check)."""
        if scale is None:
            scale = 1.0 / math.sqrt(self.plan.d)

        def mark(i):
            if events is not None:
                events[i].record()
        mark(0)
        qh = seq_to_head(q, self.layout, self.group)
        kh = seq_to_head(k, self.layout, self.group)
        vh = seq_to_head(v, self.layout, self.group)
        mark(1)
        if self.path is not None:
            o = self.path(self.plan, qh, kh, vh, scale)
            for i in range(2, 6):
                mark(i)
        else:
            b, p = self.bufs, self.plan
            rf.rearrange(p, qh, kh, vh, b.q_r, b.k_r, b.v_r, b.ws)
            mark(2)
            rf.pool_select(p, None, None, b.select_idx, b.select_num, b.ws)
            mark(3)
            rf.block_sparse_attn(p, b.q_r, b.k_r, b.v_r, b.select_idx, b.select_num, scale, b.o_r, b.ws)
            mark(4)
            rf.inverse_rearrange(p, b.o_r, b.o)
            mark(5)
            o = b.o
        out = head_to_seq(o, self.layout, self.group)
        mark(6)
        if check and self.path is None:
            rf.raise_on_device_fault(self.plan, self.bufs.ws, "UlyssesAttention")
        return out
