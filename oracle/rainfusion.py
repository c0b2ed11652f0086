"""CPU ORACLE for the RainFusion v2 block-sparse attention path.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg import this module.  It shares no code with the CUDA path:
geometry, permutation, pooling, ranking and attention are written out here from
the pages, in float64, plainly and slowly.

Sources (the web pages this path is described on):
  [UG]  "RainFusion Attention" user guide (vllm-omni docs): the opening
        paragraphs, the "Configuration" table and "Geometry handling".
  [PR]  xllm pull request "feat: add RainFusion sparse attention for wan2.2"
        (#1867): the change summary.
  [API] CANN "aclnnRainFusionAttention" API page: "Formula" and the list of
        constraints.
  [ABS] "RainFusion2.0: Temporal-Spatial Awareness and Hardware-Efficient
        Block-wise Sparse Attention", abstract.

Where the pages leave a step open, the reading taken is stated beside the code
(R1..R26 below are the same readings listed in the design notes).

Pins (what ties this oracle to something other than itself) live in
tests/test_oracle_*.py: the worked MiniMax geometry from [UG] "Geometry
handling", a nested-loop construction of the tile order, round trips,
brute-force top-k by subset enumeration, a library dense attention for
sparsity 0, element-by-element softmax loops on tiny inputs, and invariants.
Parity of the *selection* with the pages' own (unpublished) kernel is
unpinned beyond these invariants: the pages print no worked selection.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

BLOCK = 128          # [UG] opening paragraph: 128-token key blocks; [PR] pool size 128
TILE = 8             # [UG] "Geometry handling": grids aligned to 8x8
DENSE_MIN_BLOCKS = 32  # [UG] opening paragraphs: video segments below 32 blocks run dense
K_EPS = 1e-6         # R4: guards (1 - 0.8) * 465 = 92.99999... against float noise


@dataclasses.dataclass(frozen=True)
class SeqGeometry:
    """Derived sizes of one sequence (all counts in tokens unless named *blocks*)."""
    prefix_len: int   # P: text / condition rows, kept dense
    t: int
    h: int
    w: int
    h8: int           # 8 * floor(h / 8)
    w8: int
    aligned: int      # A = t * h8 * w8 tokens inside whole 8x8 tiles
    sparse: int       # S = 128 * floor(A / 128) rows in the sparse region
    promoted: int     # R = t*h*w - S video rows promoted to the dense prefix
    lp: int           # Lp = P + R, the dense prefix length after promotion
    length: int       # L = Lp + S
    n_pb: int         # prefix blocks = ceil(Lp / 128); the last may be partial
    nb: int           # video (sparse-region) blocks = S / 128
    ns: int           # first-frame sink blocks
    k: int            # ranked key blocks kept per sparse query block
    dense: bool       # the whole sequence runs dense (nb < 32)
    order: str = "tile"  # token order of the aligned video: "tile" or "frame_pair"
    sparsity: float = 0.0  # the nominal dropped fraction the keep counts come from

    @property
    def n_blocks(self) -> int:
        return self.n_pb + self.nb


def keep_count(nb: int, sparsity: float) -> int:
    """Number of ranked video key blocks each sparse query block keeps.

    [UG] "Configuration": sparsity is the nominal fraction of key blocks
    dropped, in [0, 1], and 0 disables sparsity.  Reading R4: keep
    ceil((1 - s) * nb) blocks, computed in double with a 1e-6 guard.
    """
    if not (0.0 <= sparsity <= 1.0) or not math.isfinite(sparsity):
        raise ValueError("sparsity must be finite and in [0, 1]")
    k = math.ceil((1.0 - sparsity) * nb - K_EPS)
    return max(0, min(nb, k))


ORDERS = ("tile", "frame_pair")


def geometry(prefix_len: int, t: int, h: int, w: int, sparsity: float,
             order: str = "tile") -> SeqGeometry:
    """Sizes of one sequence under suffix promotion ([UG] "Geometry handling").

    Video tokens inside whole 8x8 tiles are "aligned".  The sparse region is the
    largest whole number of 128-row blocks of aligned tokens (taken in tile
    order); every other video token (the ragged edge, plus the aligned tokens
    past that last whole block, reading R2) is promoted to the dense prefix.
    Nothing is padded.  The counts do not depend on `order` (it only reorders
    the aligned tokens, and the first frame leads in both orders).
    """
    if order not in ORDERS:
        raise ValueError(f"order must be one of {ORDERS}")
    h8, w8 = TILE * (h // TILE), TILE * (w // TILE)
    aligned = t * h8 * w8
    sparse = BLOCK * (aligned // BLOCK)
    promoted = t * h * w - sparse
    lp = prefix_len + promoted
    nb = sparse // BLOCK
    n_pb = -(-lp // BLOCK)
    ns = min(nb, -(-(h8 * w8) // BLOCK))      # blocks holding first-frame tokens (sinks)
    dense = nb < DENSE_MIN_BLOCKS
    k = nb if dense else keep_count(nb, sparsity)
    return SeqGeometry(prefix_len, t, h, w, h8, w8, aligned, sparse, promoted, lp,
                       lp + sparse, n_pb, nb, ns, k, dense, order, sparsity)


# --------------------------------------------------------------------------------------
# Step 1: the token permutation ([UG] opening paragraph and "Geometry handling";
#         [ABS] insight 2, spatiotemporal-aware token permutation).
# --------------------------------------------------------------------------------------

def video_order(t: int, h: int, w: int, order: str = "tile") -> List[int]:
    """V': video raster indices in rearranged order.

    order == "tile" (reading R1): aligned tokens are ordered by (frame, tile
    row, tile column, row in tile, column in tile), so every 128-row block is
    two 8x8 tiles of one frame.

    order == "frame_pair" ([PR] change summary: the frame-pairing approach,
    with the first frame placed before the rest; reading R17): frame 0 comes
    first, in the single-frame tile order above; frames 1..t-1 are then taken
    two at a time, (1,2), (3,4), ..., and each pair is laid out cube by cube
    (tile row, tile column), a cube holding the 8x8 tile of both frames
    (frame in pair, row in tile, column in tile) -- 128 tokens, one block.  A
    last frame left without a partner (t even) follows alone, in tile order.

    Ragged tokens follow the aligned ones in raster order in both cases.
    Built by sorting keys.
    """
    if order not in ORDERS:
        raise ValueError(f"order must be one of {ORDERS}")
    h8, w8 = TILE * (h // TILE), TILE * (w // TILE)
    n_pairs = (t - 1) // 2 if t > 0 else 0

    def group(tau: int) -> Tuple[int, int]:
        """(frame group, position of the frame inside its group)."""
        if order == "tile":
            return tau, 0
        if tau == 0:
            return 0, 0
        if tau <= 2 * n_pairs:
            return 1 + (tau - 1) // 2, (tau - 1) % 2
        return 1 + n_pairs, 0           # the unpaired last frame

    def key(v: int):
        tau, rem = divmod(v, h * w)
        y, x = divmod(rem, w)
        if y < h8 and x < w8:
            grp, fi = group(tau)
            return (0, grp, y // TILE, x // TILE, fi, y % TILE, x % TILE)
        return (1, v, 0, 0, 0, 0, 0)

    return sorted(range(t * h * w), key=key)


def permutation(g: SeqGeometry) -> np.ndarray:
    """src[r] = original row of rearranged row r, for one sequence.

    Original rows are [text 0..P-1 | video raster].  Rearranged rows are
    [text (original order) | promoted | sparse], reading R3: promoted rows sit
    right after the text and join the always-kept prefix.
    """
    vp = video_order(g.t, g.h, g.w, g.order)
    sparse, promoted = vp[:g.sparse], vp[g.sparse:]
    P = g.prefix_len
    src = list(range(P)) + [P + v for v in promoted] + [P + v for v in sparse]
    return np.asarray(src, dtype=np.int64)


def rearrange_rows(x: np.ndarray, src: np.ndarray) -> np.ndarray:
    """Rearranged sequence: row r takes original row src[r] (rows on axis -2)."""
    return x[..., src, :]


def inverse_rows(y: np.ndarray, src: np.ndarray) -> np.ndarray:
    """Inverse permutation ([PR] inverse rearrange): O[src[r]] = O'[r]."""
    out = np.empty_like(y)
    out[..., src, :] = y
    return out


# --------------------------------------------------------------------------------------
# Step 2: block-mean pooling ([UG] opening paragraph; [ABS] insight 1).
# --------------------------------------------------------------------------------------

def block_rows(g: SeqGeometry, b: int) -> range:
    """Rows of block b of one rearranged sequence.

    Blocks 0..n_pb-1 tile the dense prefix from row 0 (the last may be
    partial, [API] constraints: ceiling division); blocks n_pb.. tile the
    sparse region from row Lp.
    """
    if b < g.n_pb:
        return range(BLOCK * b, min(BLOCK * (b + 1), g.lp))
    i = b - g.n_pb
    return range(g.lp + BLOCK * i, g.lp + BLOCK * (i + 1))


def kv_block_rows(g: SeqGeometry, b: int, block_kv: int = BLOCK) -> range:
    """Rows of key/value block b when key blocks hold block_kv rows ([API] "Formula":
    blocks of blockShapeX x blockShapeY, reading R23: query blocks of blockShapeX =
    128 rows as everywhere else, key/value blocks of blockShapeY rows).  The key
    blocks tile the dense prefix from row 0 (ceiling division, the last may be
    partial) and the sparse region from row Lp, like block_rows."""
    n_pb = -(-g.lp // block_kv)
    if b < n_pb:
        return range(block_kv * b, min(block_kv * (b + 1), g.lp))
    i = b - n_pb
    return range(g.lp + block_kv * i, g.lp + block_kv * (i + 1))


def kv_block_count(g: SeqGeometry, block_kv: int = BLOCK) -> int:
    """Key/value blocks of one sequence: ceil(Lp / block_kv) + S / block_kv."""
    return -(-g.lp // block_kv) + g.sparse // block_kv


@dataclasses.dataclass(frozen=True)
class KeyBlocks:
    """Key-side block counts of one sequence when key blocks hold block_kv rows
    (reading R26).  With block_kv = 128 they are the sequence's own n_pb, nb,
    ns and k."""
    block_kv: int
    n_pb: int         # prefix key blocks, ceil(Lp / block_kv)
    nb: int           # sparse-region key blocks, S / block_kv
    ns: int           # first-frame sink key blocks, min(nb, ceil(h8 * w8 / block_kv))
    k: int            # ranked key blocks kept per sparse query block (nb if dense)


def key_blocks(g: SeqGeometry, block_kv: int = BLOCK) -> KeyBlocks:
    """Reading R26 (blockShape 128 x block_kv, [API] "Formula"): key blocks of
    block_kv rows tile the prefix and the sparse region like kv_block_rows; the
    sinks are the key blocks holding first-frame tokens (the first frame leads
    the sparse region, [UG] opening paragraphs); k keeps the same nominal
    fraction of the key blocks (R4); a dense sequence (fewer than 32 query
    blocks of 128 rows, [UG]) keeps every key block."""
    n_pb = -(-g.lp // block_kv)
    nb = g.sparse // block_kv
    ns = min(nb, -(-(g.h8 * g.w8) // block_kv))
    k = nb if g.dense else keep_count(nb, g.sparsity)
    return KeyBlocks(block_kv, n_pb, nb, ns, k)


def block_means(x_r: np.ndarray, g: SeqGeometry, block_kv: int = BLOCK) -> np.ndarray:
    """[S / block_kv, D] float64 means of each sparse-region block of block_kv rows
    of one head's rows x_r [L, D] (query blocks and, by default, key blocks hold
    128 rows; reading R26 pools key blocks of 64 rows over their own rows)."""
    kb = key_blocks(g, block_kv)
    out = np.zeros((kb.nb, x_r.shape[-1]), dtype=np.float64)
    for i in range(kb.nb):
        rows = kv_block_rows(g, kb.n_pb + i, block_kv)
        out[i] = np.asarray(x_r[rows.start:rows.stop], dtype=np.float64).mean(axis=0)
    return out


# --------------------------------------------------------------------------------------
# Step 3: per-query-block ranking and selection ([UG] opening paragraphs and
#         "Configuration"; [API] selectIdx / selectNum constraints).
# --------------------------------------------------------------------------------------

def topk_blocks(scores: np.ndarray, k: int) -> List[int]:
    """Indices of the k best scores: higher score first, lower index on ties (R9).

    A stable library sort: np.lexsort orders by the last key (descending
    score), then by the first (ascending block index).
    """
    scores = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((np.arange(len(scores)), -scores))
    return order[:k].tolist()


def select_sequence(qbar: np.ndarray, kbar: np.ndarray, g: SeqGeometry,
                    block_kv: int = BLOCK) -> Tuple[np.ndarray, np.ndarray]:
    """selectIdx [n_blocks, N1, key blocks] (-1 padded) and selectNum [n_blocks, N1] for one sequence.

    qbar: [N1, nb, D] float64 means of the 128-row query blocks; kbar: [N2,
    S / block_kv, D] float64 means of the key blocks (block_kv rows, reading
    R26; key-side counts from key_blocks).
    * Prefix query blocks and first-frame query blocks are dense ([UG]: prefix
      rows and first-frame blocks remain dense; reading R6).
    * Every other video query block i on head n ranks video key blocks j by
      the plain dot product of block means, qbar[n, i] . kbar[n // G, j]
      (reading R7; GQA head grouping R8), keeps the top k, adds the
      first-frame sinks (reading R5: sinks do not count toward k), and always
      keeps every prefix block ([UG]: prefix rows are dense).
    * A row lists kept blocks in ascending order, prefix blocks first, padded
      with -1 ([API]: invalid slots are -1).
    """
    n1, n2 = qbar.shape[0], kbar.shape[0]
    G = n1 // n2
    kb = key_blocks(g, block_kv)
    nblk = g.n_blocks
    nkv = kb.n_pb + kb.nb
    idx = np.full((nblk, n1, nkv), -1, dtype=np.int32)
    num = np.zeros((nblk, n1), dtype=np.int32)
    everything = list(range(nkv))
    for n in range(n1):
        scores = qbar[n] @ kbar[n // G].T          # [nb, kb.nb]: scores[i, j] = qbar_i . kbar_j
        for qb in range(nblk):
            i = qb - g.n_pb
            if g.dense or qb < g.n_pb or i < g.ns:
                row = everything
            else:
                keep = set(topk_blocks(scores[i], kb.k)) | set(range(kb.ns))
                row = list(range(kb.n_pb)) + [kb.n_pb + j for j in sorted(keep)]
            idx[qb, n, :len(row)] = row
            num[qb, n] = len(row)
    return idx, num


# --------------------------------------------------------------------------------------
# Step 4: block-sparse attention ([API] "Formula": Softmax(scale * Q K^T + mask) V,
#         restricted to the key blocks each query block selected).
# --------------------------------------------------------------------------------------

def attend_query_block(q_r: np.ndarray, k_r: np.ndarray, v_r: np.ndarray, g: SeqGeometry,
                       qb: int, key_blocks: Sequence[int], scale: float,
                       block_kv: int = BLOCK) -> np.ndarray:
    """float64 output rows of query block qb of one head.

    The keys are the union of the rows of the listed blocks (-1 entries are
    ignored); the only mask is that rows past the dense prefix end do not
    belong to the last prefix block (reading R10: no user mask).  Logits are
    formed in float64 from the exact input values, then a max-subtracted
    softmax, then the weighted sum of values.
    """
    qrows = block_rows(g, qb)
    krows: List[int] = []
    for b in key_blocks:
        if b < 0:
            continue
        krows.extend(kv_block_rows(g, int(b), block_kv))
    q = np.asarray(q_r[qrows.start:qrows.stop], dtype=np.float64)
    k = np.asarray(k_r[krows], dtype=np.float64)
    v = np.asarray(v_r[krows], dtype=np.float64)
    logits = scale * (q @ k.T)
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


# --------------------------------------------------------------------------------------
# Whole-path helpers over a batch in BNSD or TND layout.
# --------------------------------------------------------------------------------------

@dataclasses.dataclass
class Problem:
    """Shapes of one call: per-sequence geometry plus heads and layout."""
    layout: str                       # "BNSD" or "TND"
    batch: int                        # BNSD batch size (1 for TND)
    geoms: List[SeqGeometry]          # one per sequence (BNSD: one, shared by the batch)
    n1: int
    n2: int
    d: int

    def sequences(self) -> List[Tuple[int, SeqGeometry]]:
        """(sequence id, geometry) in q-block order: BNSD batch elements, or TND sequences."""
        if self.layout == "BNSD":
            return [(b, self.geoms[0]) for b in range(self.batch)]
        return list(enumerate(self.geoms))

    def row_offsets(self) -> List[int]:
        offs, acc = [], 0
        for g in self.geoms:
            offs.append(acc)
            acc += g.length
        return offs

    def head_rows(self, x: np.ndarray, seq: int, head: int) -> np.ndarray:
        """View [L, D] of one sequence and head."""
        if self.layout == "BNSD":
            return x[seq, head]
        off = self.row_offsets()[seq]
        return x[off:off + self.geoms[seq].length, head, :]

    @property
    def max_kv_blocks(self) -> int:
        return max(g.n_blocks for g in self.geoms)

    @property
    def t_qblk(self) -> int:
        return sum(g.n_blocks for _, g in self.sequences())


def make_problem(layout: str, batch: int, seqs: Sequence[Tuple[int, int, int, int]],
                 n1: int, n2: int, d: int, sparsity: float, order: str = "tile") -> Problem:
    if n1 % n2:
        raise ValueError("N1 must be a multiple of N2 ([API] constraints)")
    geoms = [geometry(p, t, h, w, sparsity, order) for (p, t, h, w) in seqs]
    return Problem(layout, batch, geoms, n1, n2, d)


def rearrange(p: Problem, x: np.ndarray) -> np.ndarray:
    """Apply the per-sequence permutation to a BNSD [B,N,L,D] or TND [T,N,D] array."""
    y = np.empty_like(x)
    if p.layout == "BNSD":
        src = permutation(p.geoms[0])
        y[...] = x[:, :, src, :]
        return y
    for s, (off, g) in enumerate(zip(p.row_offsets(), p.geoms)):
        src = permutation(g)
        y[off:off + g.length] = x[off + src]
    return y


def inverse_rearrange(p: Problem, y: np.ndarray) -> np.ndarray:
    x = np.empty_like(y)
    if p.layout == "BNSD":
        src = permutation(p.geoms[0])
        x[:, :, src, :] = y
        return x
    for off, g in zip(p.row_offsets(), p.geoms):
        src = permutation(g)
        x[off + src] = y[off:off + g.length]
    return x


def pooled_means(p: Problem, x_r: np.ndarray, heads: int, block_kv: int = BLOCK) -> List[np.ndarray]:
    """Per sequence, [heads, S / block_kv, D] float64 block means of the rearranged x_r."""
    out = []
    for s, g in p.sequences():
        nbk = g.sparse // block_kv
        out.append(np.stack([block_means(p.head_rows(x_r, s, n), g, block_kv) for n in range(heads)])
                   if nbk else np.zeros((heads, 0, p.d)))
    return out


def select(p: Problem, qbars: List[np.ndarray], kbars: List[np.ndarray],
           block_kv: int = BLOCK) -> Tuple[np.ndarray, np.ndarray]:
    """selectIdx [T_qblk, N1, maxKv] and selectNum [T_qblk, N1] over all sequences ([API]);
    with block_kv = 64 the entries and maxKv count 64-row key blocks (reading R26)."""
    maxkv = max(kv_block_count(g, block_kv) for g in p.geoms)
    idx = np.full((p.t_qblk, p.n1, maxkv), -1, dtype=np.int32)
    num = np.zeros((p.t_qblk, p.n1), dtype=np.int32)
    t0 = 0
    for (s, g), qb, kb in zip(p.sequences(), qbars, kbars):
        i_s, n_s = select_sequence(qb, kb, g, block_kv)
        idx[t0:t0 + g.n_blocks, :, :i_s.shape[2]] = i_s
        num[t0:t0 + g.n_blocks] = n_s
        t0 += g.n_blocks
    return idx, num


def qblock_table(p: Problem) -> List[Tuple[int, SeqGeometry, int]]:
    """For each global query block t: (sequence id, geometry, local block index)."""
    out = []
    for s, g in p.sequences():
        out.extend((s, g, b) for b in range(g.n_blocks))
    return out


def attention(p: Problem, q_r: np.ndarray, k_r: np.ndarray, v_r: np.ndarray,
              idx: np.ndarray, num: np.ndarray, scale: float,
              items: Sequence[Tuple[int, int]] | None = None,
              block_kv: int = BLOCK) -> Dict[Tuple[int, int], np.ndarray]:
    """float64 output rows for (global q-block, q-head) items (default: all).

    Inputs are float64 arrays in the rearranged layout.  Head n reads key/value
    head n // G ([API] constraints: N1 = G * N2).
    """
    G = p.n1 // p.n2
    table = qblock_table(p)
    if items is None:
        items = [(t, n) for t in range(len(table)) for n in range(p.n1)]
    out = {}
    for (t, n) in items:
        s, g, b = table[t]
        row = idx[t, n, :num[t, n]]
        out[(t, n)] = attend_query_block(p.head_rows(q_r, s, n), p.head_rows(k_r, s, n // G),
                                         p.head_rows(v_r, s, n // G), g, b, row, scale, block_kv)
    return out


def assemble_output(p: Problem, parts: Dict[Tuple[int, int], np.ndarray], like: np.ndarray) -> np.ndarray:
    """Scatter per-(q-block, head) rows into a rearranged-layout float64 array shaped like `like`."""
    o = np.full(like.shape, np.nan, dtype=np.float64)
    table = qblock_table(p)
    for (t, n), rows in parts.items():
        s, g, b = table[t]
        r = block_rows(g, b)
        p.head_rows(o, s, n)[r.start:r.stop] = rows
    return o


def run_path(p: Problem, q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
             block_kv: int = BLOCK) -> Dict[str, object]:
    """Whole path on float64 inputs in original order: permute, pool, select, attend, un-permute
    (key blocks of block_kv rows, reading R26)."""
    q_r, k_r, v_r = rearrange(p, q), rearrange(p, k), rearrange(p, v)
    qbars, kbars = pooled_means(p, q_r, p.n1), pooled_means(p, k_r, p.n2, block_kv)
    idx, num = select(p, qbars, kbars, block_kv)
    o_r = assemble_output(p, attention(p, q_r, k_r, v_r, idx, num, scale, block_kv=block_kv), q_r)
    return dict(q_r=q_r, k_r=k_r, v_r=v_r, qbar=qbars, kbar=kbars, idx=idx, num=num,
                o_r=o_r, o=inverse_rearrange(p, o_r))


def kept_flops(p: Problem, idx: np.ndarray, num: np.ndarray, block_kv: int = BLOCK) -> int:
    """4 * D * (query rows) * (valid key rows) summed over selected (q-block, head, key block)."""
    table = qblock_table(p)
    total = 0
    for t, (s, g, b) in enumerate(table):
        mq = len(block_rows(g, b))
        for n in range(p.n1):
            kv = sum(len(kv_block_rows(g, int(j), block_kv)) for j in idx[t, n, :num[t, n]])
            total += 4 * p.d * mq * kv
    return total


# --------------------------------------------------------------------------------------
# "mix" kernel precision ([UG] "Configuration": precision "bf16" | "fp8" | "mix";
# "Wan2.2 T2V quantization on Ascend": FP8 block-sparse attention).  The pages give the
# names only; reading R18: in "mix", Q and K are quantized to FP8 E4M3 with one scale per
# (head, 128-row block) and Q K^T runs on those codes; P and V stay 16-bit.
# --------------------------------------------------------------------------------------

E4M3_MAX = 448.0     # largest finite E4M3 magnitude (S.1111.110)


def e4m3_value(code: int) -> float:
    """Value of an FP8 E4M3 code: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
    bits, subnormals at exponent 0, no infinities, S.1111.111 is NaN."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3_POS = np.array([e4m3_value(c) for c in range(0x7F)], dtype=np.float64)  # codes 0..126, increasing


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """uint8 E4M3 codes of x: round to the nearest representable value, ties to the
    even code (mantissa LSB 0), magnitudes beyond 448 saturate to 448; the sign bit
    follows the sign of x (negative zero included)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, len(_E4M3_POS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return code | np.where(np.signbit(x), np.uint8(0x80), np.uint8(0))


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """float64 values of E4M3 codes (finite codes only)."""
    codes = np.asarray(codes, dtype=np.uint8)
    mag = _E4M3_POS[np.minimum(codes & 0x7F, 0x7E)]
    return np.where(codes & 0x80, -mag, mag)


def quantize_block_e4m3(x: np.ndarray) -> Tuple[np.ndarray, np.float32]:
    """One block (rows x D) of 16-bit values, given as float32: E4M3 codes and the
    float32 dequantization scale, in the arithmetic reading R18 fixes:
    amax = max |x|; inv = 448 / amax and scale = amax / 448 (each one float32
    division, round to nearest even); codes = E4M3(x * inv) with the product a
    float32 multiply.  An all-zero block has inv = scale = 1."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    if amax == 0:
        inv, scale = np.float32(1), np.float32(1)
    else:
        inv = np.float32(np.float32(E4M3_MAX) / amax)
        scale = np.float32(amax / np.float32(E4M3_MAX))
    y = (x * inv).astype(np.float32)
    return e4m3_round(y), scale


def quantize_e4m3(p: Problem, x_r: np.ndarray, heads: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per (head, block) E4M3 quantization of a rearranged tensor (float32 values in
    the BNSD or TND layout of x_r): uint8 codes shaped like x_r and float32 scales
    [heads, T_qblk] indexed by global query-block number."""
    codes = np.zeros(x_r.shape, dtype=np.uint8)
    scales = np.ones((heads, p.t_qblk), dtype=np.float32)
    for t, (s, g, b) in enumerate(qblock_table(p)):
        r = block_rows(g, b)
        for n in range(heads):
            src = p.head_rows(x_r, s, n)
            c, sc = quantize_block_e4m3(src[r.start:r.stop])
            p.head_rows(codes, s, n)[r.start:r.stop] = c
            scales[n, t] = sc
    return codes, scales


def dequantize_e4m3(p: Problem, codes: np.ndarray, scales: np.ndarray, heads: int) -> np.ndarray:
    """float64 values code * scale of its (head, block), in the layout of codes."""
    out = np.zeros(codes.shape, dtype=np.float64)
    for t, (s, g, b) in enumerate(qblock_table(p)):
        r = block_rows(g, b)
        for n in range(heads):
            v = e4m3_decode(p.head_rows(codes, s, n)[r.start:r.stop]) * np.float64(scales[n, t])
            p.head_rows(out, s, n)[r.start:r.stop] = v
    return out


# --------------------------------------------------------------------------------------
# "fp8" kernel precision ([UG] "Configuration": precision "fp8"; "Wan2.2 T2V quantization
# on Ascend": FP8 block-sparse attention).  The pages give the name only; reading R24:
# Q and K are quantized as in "mix"; V is quantized to E4M3 with one power-of-two scale
# per (head, 128-row block), 2^e with e the smallest integer for which the block's
# largest magnitude is at most 448 * 2^e (codes E4M3(v * 2^-e): an exact scaling, then
# round to nearest even with saturation; an all-zero block takes the smallest exponent,
# -127, so that it never raises a row's largest one); the softmax probabilities of each
# key block enter the P V product as E4M3 values of P * 2^(e_j - e_max), e_max the
# largest V exponent among the row's selected blocks, while the row sum uses the
# unrounded probabilities.
FP8_ZERO_EXP = -127
# --------------------------------------------------------------------------------------

def pow2_exponent(amax: float, top: float = E4M3_MAX) -> int:
    """Smallest integer e with amax <= top * 2^e (0 for amax == 0).  Exact: the
    comparisons are between float64 values that hold amax and top * 2^e exactly."""
    amax = float(amax)
    if amax == 0.0:
        return 0
    e = math.ceil(math.log2(amax / top))
    while amax > top * 2.0 ** e:
        e += 1
    while amax <= top * 2.0 ** (e - 1):
        e -= 1
    return e


def quantize_block_e4m3_pow2(x: np.ndarray) -> Tuple[np.ndarray, int]:
    """One block (rows x D) of 16-bit values: E4M3 codes of x * 2^-e and the exponent e
    (reading R24); an all-zero block has e = -127 and all codes zero."""
    x = np.asarray(x, dtype=np.float64)
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    if amax == 0.0:
        return np.zeros(x.shape, dtype=np.uint8), FP8_ZERO_EXP
    e = pow2_exponent(amax)
    return e4m3_round(x * 2.0 ** (-e)), e


def quantize_v_fp8(p: Problem, v_r: np.ndarray, heads: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per (head, block) power-of-two E4M3 quantization of a rearranged V: uint8 codes
    shaped like v_r and int32 exponents [heads, T_qblk] by global block number."""
    codes = np.zeros(v_r.shape, dtype=np.uint8)
    exps = np.zeros((heads, p.t_qblk), dtype=np.int32)
    for t, (s, g, b) in enumerate(qblock_table(p)):
        r = block_rows(g, b)
        for n in range(heads):
            c, e = quantize_block_e4m3_pow2(p.head_rows(v_r, s, n)[r.start:r.stop])
            p.head_rows(codes, s, n)[r.start:r.stop] = c
            exps[n, t] = e
    return codes, exps


def dequantize_v_fp8(p: Problem, codes: np.ndarray, exps: np.ndarray, heads: int) -> np.ndarray:
    """float64 values code * 2^e of its (head, block), in the layout of codes."""
    out = np.zeros(codes.shape, dtype=np.float64)
    for t, (s, g, b) in enumerate(qblock_table(p)):
        r = block_rows(g, b)
        for n in range(heads):
            p.head_rows(out, s, n)[r.start:r.stop] = (
                e4m3_decode(p.head_rows(codes, s, n)[r.start:r.stop]) * 2.0 ** int(exps[n, t]))
    return out


def fp8_probability_error_bound(p: Problem, q_r: np.ndarray, k_r: np.ndarray, v_r: np.ndarray,
                                idx: np.ndarray, num: np.ndarray, scale: float,
                                items: Sequence[Tuple[int, int]],
                                v_exps: np.ndarray | None = None) -> Dict[Tuple[int, int], np.ndarray]:
    """Per output element of the listed (q-block, head) items: the largest change that
    rounding every probability to E4M3 can make to softmax(scale q K^T) V when the row
    sum stays exact.  P_i is taken relative to the row's largest logit (P_i <= 1).  In
    the normal range P~_i = P_i (1 + d_i), |d_i| <= 2^-4 (half a step of a 3-bit
    mantissa).  A probability of key block j enters as E4M3(P_i 2^u 2^(e_j - e_max)),
    where 2^u in [1, 2^8] is the kernel's own normalisation; below the normal range
    (2^-6) the rounding error is at most half a subnormal step, 2^-10, in those units,
    so at most min(P_i, 2^-10 2^(e_max - e_j)) in units of P_i (and 0 when v_exps is
    None).  The change is sum_i (P~_i - P_i) V_i / sum_i P_i, so
    |change| <= sum_i (2^-4 P_i + min(P_i, 2^-10 2^(e_max - e_j))) |V_i| / sum_i P_i."""
    G = p.n1 // p.n2
    table = qblock_table(p)
    out = {}
    for (t, n) in items:
        s, g, b = table[t]
        qrows = block_rows(g, b)
        krows: List[int] = []
        for j in idx[t, n, :num[t, n]]:
            if j >= 0:
                krows.extend(block_rows(g, int(j)))
        q = p.head_rows(q_r, s, n)[qrows.start:qrows.stop]
        k = p.head_rows(k_r, s, n // G)[krows]
        v = p.head_rows(v_r, s, n // G)[krows]
        logits = scale * (q @ k.T)
        logits -= logits.max(axis=1, keepdims=True)
        w = np.exp(logits)
        err = 2.0 ** -4 * w
        if v_exps is not None:
            t0 = t - b                                   # first global block of this sequence
            blocks = [int(j) for j in idx[t, n, :num[t, n]] if j >= 0]
            e = np.array([v_exps[n // G, t0 + j] for j in blocks], dtype=np.float64)
            step = np.concatenate([np.full(len(block_rows(g, j)), 2.0 ** (-10 + e.max() - ej))
                                   for j, ej in zip(blocks, e)])
            err = err + np.minimum(w, step[None, :])
        out[(t, n)] = (err @ np.abs(v)) / w.sum(axis=1, keepdims=True)
    return out
