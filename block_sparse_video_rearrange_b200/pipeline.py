"""The whole path on host tensors, with host<->device copies overlapping the compute.

Heads are independent in every step of the path (permutation, block means,
ranking, attention), so a layer can run as C chunks of N2/C key/value heads
(and their N1/C query heads) with results identical to one pass.  Chunk i's
inputs go to the GPU on a copy-in stream while chunk i-1 computes on the
compute stream and chunk i-2's output returns on a copy-out stream; two sets of
device buffers alternate between chunks.  On a PCIe-attached GPU the copies
dominate (Q, K, V in and O out), and this hides the compute under them.

Copies are plain cudaMemcpyAsync from pinned memory (one per batch element
for BNSD, whose head slices are contiguous per batch element) or
cudaMemcpy2DAsync for TND (a head slice of [T, N, D] is T rows of a fixed
pitch).  All device work is librf's.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import torch

from . import rf

try:  # strided (TND) head slices need a 2-D copy
    from cuda.bindings import runtime as _cudart
except ImportError:  # pragma: no cover - older cuda-python layout
    try:
        from cuda import cudart as _cudart
    except ImportError:
        _cudart = None


def default_chunks(n2: int, limit: int = 20) -> int:
    """Largest divisor of the key/value head count not above `limit`.

    More chunks shorten the pipeline's fill and drain (the first chunk's copy in
    and the last chunk's compute and copy out run alone), until a chunk holds so
    few heads that its launches stop filling the GPU: on a 40-head layer with
    bf16 D = 128 and 33k rows, 20 chunks beat 8 by about 4 % and 40 chunks lose.
    """
    return max(c for c in range(1, min(n2, limit) + 1) if n2 % c == 0)


def _copy_2d(dst_ptr: int, dpitch: int, src_ptr: int, spitch: int, width: int, height: int,
             kind, stream: torch.cuda.Stream) -> None:
    err = _cudart.cudaMemcpy2DAsync(dst_ptr, dpitch, src_ptr, spitch, width, height, kind,
                                    stream.cuda_stream)
    code = err[0] if isinstance(err, tuple) else err
    if int(code) != 0:
        raise RuntimeError(f"cudaMemcpy2DAsync failed: {code}")


class HostPipeline:
    """RainFusion attention of host (pinned) tensors in head chunks over three streams.

    Call with q, k, v on the host in the caller's layout (original token order)
    and a host output tensor shaped like q; the call enqueues everything, makes
    the caller's current stream wait for the last copy, and returns.
    """

    def __init__(self, seqs: Sequence[Tuple[int, int, int, int]], n1: int, n2: int, d: int,
                 layout: str = "BNSD", dtype: str = "bf16", sparsity: float = 0.8, batch: int = 1,
                 chunks: Optional[int] = None, order: str = "tile", precision: str = "native",
                 device=None, block_kv: int = 128):
        self.chunks = chunks if chunks is not None else default_chunks(n2)
        if n2 % self.chunks or n1 % self.chunks:
            raise ValueError(f"{self.chunks} chunks do not divide the heads ({n1}, {n2})")
        if layout == "TND" and self.chunks > 1 and _cudart is None:
            self.chunks = 1                                   # no 2-D copy available: one chunk
        self.layout, self.n1, self.n2, self.d = layout, n1, n2, d
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.plan = rf.Plan(seqs, n1 // self.chunks, n2 // self.chunks, d, layout, dtype, sparsity, batch=batch,
                            order=order, precision=precision, block_kv=block_kv)
        p = self.plan
        self.sets = []
        for _ in range(2 if self.chunks > 1 else 1):
            self.sets.append(dict(q=torch.empty(p.tensor_shape(p.n1), dtype=p.torch_dtype, device=self.device),
                                  k=torch.empty(p.tensor_shape(p.n2), dtype=p.torch_dtype, device=self.device),
                                  v=torch.empty(p.tensor_shape(p.n2), dtype=p.torch_dtype, device=self.device),
                                  bufs=rf.Buffers(p, self.device)))
        self.s_in = torch.cuda.Stream(self.device)
        self.s_cmp = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)

    # -- head-slice copies ---------------------------------------------------------------
    def _h2d(self, dst: torch.Tensor, src: torch.Tensor, h0: int, hc: int, stream) -> None:
        if self.layout == "BNSD":
            for b in range(src.shape[0]):
                dst[b].copy_(src[b, h0:h0 + hc], non_blocking=True)
        elif self.chunks == 1:
            dst.copy_(src, non_blocking=True)
        else:
            t, n, d = src.shape
            es = src.element_size()
            _copy_2d(dst.data_ptr(), hc * d * es, src.data_ptr() + h0 * d * es, n * d * es, hc * d * es, t,
                     _cudart.cudaMemcpyKind.cudaMemcpyHostToDevice, stream)

    def _d2h(self, dst: torch.Tensor, src: torch.Tensor, h0: int, hc: int, stream) -> None:
        if self.layout == "BNSD":
            for b in range(dst.shape[0]):
                dst[b, h0:h0 + hc].copy_(src[b], non_blocking=True)
        elif self.chunks == 1:
            dst.copy_(src, non_blocking=True)
        else:
            t, n, d = dst.shape
            es = dst.element_size()
            _copy_2d(dst.data_ptr() + h0 * d * es, n * d * es, src.data_ptr(), hc * d * es, hc * d * es, t,
                     _cudart.cudaMemcpyKind.cudaMemcpyDeviceToHost, stream)

    def __call__(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                 scale: Optional[float] = None) -> None:
        if scale is None:
            scale = 1.0 / math.sqrt(self.d)
        c = self.chunks
        hq, hk = self.n1 // c, self.n2 // c
        caller = torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(caller)
        self.s_in.wait_event(start)
        freed = [None] * len(self.sets)
        for i in range(c):
            slot = i % len(self.sets)
            st = self.sets[slot]
            with torch.cuda.stream(self.s_in):
                if freed[slot] is not None:          # this set's previous chunk has left the GPU
                    self.s_in.wait_event(freed[slot])
                self._h2d(st["q"], q, i * hq, hq, self.s_in)
                self._h2d(st["k"], k, i * hk, hk, self.s_in)
                self._h2d(st["v"], v, i * hk, hk, self.s_in)
                ready = torch.cuda.Event()
                ready.record(self.s_in)
            self.s_cmp.wait_event(ready)
            with torch.cuda.stream(self.s_cmp):
                rf.forward(self.plan, st["q"], st["k"], st["v"], st["bufs"], scale, stream=self.s_cmp)
                done = torch.cuda.Event()
                done.record(self.s_cmp)
            self.s_out.wait_event(done)
            with torch.cuda.stream(self.s_out):
                self._d2h(out, st["bufs"].o, i * hq, hq, self.s_out)
                freed[slot] = torch.cuda.Event()
                freed[slot].record(self.s_out)
        for ev in freed:                             # the last chunks' copies out
            if ev is not None:
                caller.wait_event(ev)

    def workspaces(self):
        """The device workspace of every buffer set (status words at their start)."""
        return [st["bufs"].ws for st in self.sets]

    def check_status(self) -> Tuple[int, Tuple[int, int]]:
        """Device status words of every buffer set (synchronises, reads and clears
        them all); the first non-zero one."""
        torch.cuda.synchronize(self.device)
        first = (0, (0, 0))
        for st in self.sets:
            s, flags = rf.check_device_status(self.plan, st["bufs"].ws)
            if s != 0 and first[0] == 0:
                first = (s, flags)
        return first

    def raise_on_device_fault(self) -> None:
        """check_status, raising RfError(RF_ERR_DEVICE_FAULT) if any word was set."""
        s, flags = self.check_status()
        if s != rf.RF_OK:
            raise rf.RfError(s, "rainfusion_attention (host pipeline)",
                             f"device status words: {flags[0]} bad selectIdx entries, "
                             f"expired-wait bits {flags[1]:#x}")
