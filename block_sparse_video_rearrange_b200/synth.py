"""Seeded synthetic inputs for the RainFusion v2 block-sparse attention path.

This module only draws random tensors in the ORIGINAL token order (text prefix,
then the video grid in raster (t, y, x) order).  It holds none of the method's
arithmetic: no permutation, pooling, ranking or attention.  Both the CUDA path
and the CPU oracle consume exactly the arrays it returns.

Recipe (a stand-in for real DiT activations, which are not available):
  * text row, head n, tensor X in {Q, K, V}:   0.5 * N(0, 1) per element;
  * video row (tau, y, x), head n, tensor X:   0.5 * N(0, 1)
                                              + off_X[n, tau, y // 8, x // 8, :]
    where every offset vector is an independent N(0, 1) draw per
    (tensor, head, frame, 8x8 spatial cell); cells cut by the grid edge get
    their own offset like any other cell;
  * values are drawn in float32 and rounded to bf16 (or fp16) with
    round-to-nearest-even; the rounded bit patterns are what both sides read.

The five workloads mirror the shapes of the pages' use cases (Wan2.2 and
MiniMax-H3 video layers, an 8x8-aligned grid, a varlen GQA batch and a tiny
case).
"""
from __future__ import annotations

import dataclasses
from typing import List, Sequence, Tuple

import numpy as np

__all__ = [
    "SeqSpec", "Workload", "WORKLOADS", "workload", "generate_qkv",
    "bits_to_float64", "float32_to_bf16_bits", "float32_to_fp16_bits",
]


@dataclasses.dataclass(frozen=True)
class SeqSpec:
    """One sequence: a text/condition prefix followed by a (t, h, w) video grid."""
    prefix_len: int
    t: int
    h: int
    w: int

    @property
    def length(self) -> int:
        return self.prefix_len + self.t * self.h * self.w


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    layout: str            # "BNSD" or "TND"
    dtype: str             # "bf16" or "fp16"
    batch: int             # B for BNSD (every batch element has seqs[0]'s geometry); 1 for TND
    seqs: Tuple[SeqSpec, ...]
    n1: int                # query heads
    n2: int                # key/value heads
    d: int                 # head dim
    sparsity: float
    seed: int

    def with_sparsity(self, s: float) -> "Workload":
        return dataclasses.replace(self, sparsity=float(s), name=f"{self.name.split('@')[0]}@{s:g}")

    @property
    def total_rows(self) -> int:
        if self.layout == "BNSD":
            return self.seqs[0].length
        return sum(s.length for s in self.seqs)


WORKLOADS = {
    # 128 text tokens + (9,16,32) video: 4,608 video rows = 36 blocks, first frame = 4 blocks.
    "tiny": Workload("tiny", "BNSD", "bf16", 1, (SeqSpec(128, 9, 16, 32),), 2, 2, 64, 0.8, 1000),
    # Wan2.2-shaped layer: h = 30 is not a multiple of 8, so part of the video is promoted.
    "wan": Workload("wan", "BNSD", "bf16", 1, (SeqSpec(512, 21, 30, 52),), 40, 40, 128, 0.8, 1001),
    # MiniMax-H3-shaped layer at 1344x768: grid (62, 24, 42).
    "minimax": Workload("minimax", "BNSD", "bf16", 1, (SeqSpec(256, 62, 24, 42),), 24, 24, 128, 0.8, 1002),
    # 8x8-aligned grid, swept against the dense (sparsity 0) path.
    "aligned": Workload("aligned", "BNSD", "bf16", 1, (SeqSpec(512, 21, 48, 80),), 40, 40, 128, 0.8, 1003),
    # Two sequences of different geometry, packed token-major, grouped-query heads (G = 4).
    "tnd_gqa": Workload("tnd_gqa", "TND", "fp16", 1,
                        (SeqSpec(256, 13, 32, 48), SeqSpec(384, 21, 24, 40)), 32, 8, 128, 0.8, 1004),
}


def workload(name: str, sparsity: float | None = None) -> Workload:
    w = WORKLOADS[name]
    return w if sparsity is None else w.with_sparsity(sparsity)


def float32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def float32_to_fp16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to IEEE half (numpy's cast rounds to nearest even); uint16 bit patterns."""
    return np.ascontiguousarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def bits_to_float64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Decode uint16 bf16/fp16 bit patterns to float64 (exact)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    raise ValueError(dtype)


def _one_sequence(rng: np.random.Generator, spec: SeqSpec, heads: int, d: int) -> np.ndarray:
    """float32 [heads, L, d] for one sequence of one tensor, in original token order."""
    L = spec.length
    out = rng.standard_normal((heads, L, d), dtype=np.float32)
    out *= np.float32(0.5)
    nv = spec.t * spec.h * spec.w
    if nv:
        hc = -(-spec.h // 8)
        wc = -(-spec.w // 8)
        offs = rng.standard_normal((heads, spec.t * hc * wc, d), dtype=np.float32)
        tau = np.arange(spec.t)[:, None, None]
        y = np.arange(spec.h)[None, :, None]
        x = np.arange(spec.w)[None, None, :]
        cell = ((tau * hc + y // 8) * wc + x // 8).reshape(-1)           # raster order of the video
        for n in range(heads):                                           # per head keeps temporaries small
            out[n, spec.prefix_len:, :] += offs[n, cell, :]
    return out


def generate_qkv(w: Workload) -> List[np.ndarray]:
    """Return [Q, K, V] as uint16 bit arrays in the workload's layout.

    BNSD: Q is [B, N1, L, D], K/V are [B, N2, L, D].
    TND:  Q is [T, N1, D], K/V are [T, N2, D] with the sequences packed back to back.
    The seed depends only on the workload's base name, so a sparsity sweep
    reuses identical inputs.
    """
    conv1 = float32_to_bf16_bits if w.dtype == "bf16" else float32_to_fp16_bits

    def conv(x):          # head by head: small temporaries, same bits as one call
        out = np.empty(x.shape, dtype=np.uint16)
        for n in range(x.shape[0]):
            out[n] = conv1(x[n])
        return out
    rng = np.random.Generator(np.random.PCG64(w.seed))
    result = []
    for tensor_idx, heads in enumerate((w.n1, w.n2, w.n2)):
        if w.layout == "BNSD":
            spec = w.seqs[0]
            arr = np.empty((w.batch, heads, spec.length, w.d), dtype=np.uint16)
            for b in range(w.batch):
                arr[b] = conv(_one_sequence(rng, spec, heads, w.d))
        elif w.layout == "TND":
            parts = [conv(_one_sequence(rng, spec, heads, w.d)).transpose(1, 0, 2) for spec in w.seqs]
            arr = np.ascontiguousarray(np.concatenate(parts, axis=0))
        else:
            raise ValueError(w.layout)
        result.append(arr)
    return result


def seq_row_offsets(w: Workload) -> List[int]:
    """Start row of each sequence in the packed (TND) token dimension."""
    offs, acc = [], 0
    for s in w.seqs:
        offs.append(acc)
        acc += s.length
    return offs


def sample_rows(rng: np.random.Generator, n: int, k: int) -> Sequence[int]:
    """k distinct sorted integers from range(n) (used to sample work for big cases)."""
    k = min(k, n)
    return sorted(rng.choice(n, size=k, replace=False).tolist())
