"""Pins for the oracle's geometry and permutation (CPU only).

The worked MiniMax example comes from the "RainFusion Attention" user guide,
section "Geometry handling"; everything else is brute force or a closed form.
"""
import itertools

import numpy as np
import pytest

from oracle import rainfusion as rf
from tests.conftest import read_golden


def test_minimax_geometry_matches_worked_example():
    gold = read_golden("minimax_geometry.txt")
    g = rf.geometry(256, gold["grid_t"], gold["grid_h"], gold["grid_w"], 0.8)
    assert g.t * g.h * g.w == gold["video_rows"]
    assert g.promoted == gold["promoted_rows"]
    assert g.sparse == gold["sparse_rows"]
    assert g.nb == gold["sparse_blocks"]
    src = rf.permutation(g)
    # The promoted rows are real video rows placed in the prefix, right after the text.
    promoted_src = src[256:256 + g.promoted]
    assert np.all(promoted_src >= 256)
    assert len(promoted_src) == gold["promoted_rows"]


def _nested_loop_video_order(t, h, w):
    """Tile order written as explicit loops: frame, tile row, tile column, row, column."""
    h8, w8 = 8 * (h // 8), 8 * (w // 8)
    order = []
    for tau in range(t):
        for hb in range(h8 // 8):
            for wb in range(w8 // 8):
                for hi in range(8):
                    for wi in range(8):
                        order.append(tau * h * w + (8 * hb + hi) * w + 8 * wb + wi)
    for tau in range(t):
        for y in range(h):
            for x in range(w):
                if y >= h8 or x >= w8:
                    order.append(tau * h * w + y * w + x)
    return order


@pytest.mark.parametrize("t,h,w", [(1, 8, 8), (2, 16, 24), (3, 13, 21), (2, 30, 52), (1, 7, 9), (4, 5, 40)])
def test_video_order_equals_nested_loops(t, h, w):
    assert rf.video_order(t, h, w) == _nested_loop_video_order(t, h, w)


@pytest.mark.parametrize("p,t,h,w", [(128, 9, 16, 32), (512, 3, 30, 52), (0, 2, 24, 42), (7, 1, 5, 5),
                                     (384, 2, 24, 40), (1, 3, 17, 9)])
def test_permutation_is_bijection_and_round_trips(p, t, h, w):
    g = rf.geometry(p, t, h, w, 0.8)
    src = rf.permutation(g)
    assert g.length == p + t * h * w
    assert sorted(src.tolist()) == list(range(g.length))
    x = np.random.default_rng(0).standard_normal((2, g.length, 3))
    y = rf.rearrange_rows(x, src)
    assert np.array_equal(rf.inverse_rows(y, src), x)
    # text stays first, in its original order
    assert np.array_equal(src[:p], np.arange(p))


def test_aligned_blocks_are_two_adjacent_tiles_of_one_frame():
    # grid with an even number of tile columns: each 128-row block = 2 whole 8x8 tiles
    p, t, h, w = 64, 3, 16, 32
    g = rf.geometry(p, t, h, w, 0.5)
    src = rf.permutation(g)
    assert g.promoted == 0 and g.nb == t * h * w // 128
    for i in range(g.nb):
        rows = src[g.lp + 128 * i: g.lp + 128 * (i + 1)] - p
        tau = rows // (h * w)
        y = (rows % (h * w)) // w
        x = rows % w
        assert len(set(tau.tolist())) == 1
        cells = sorted(set(zip((y // 8).tolist(), (x // 8).tolist())))
        assert len(cells) == 2 and cells[0][0] == cells[1][0] and cells[1][1] == cells[0][1] + 1
        assert cells[0][1] % 2 == 0


def test_promoted_rows_are_ragged_edge_plus_aligned_leftover():
    # (21, 24, 40): A = 20,160 = 157.5 blocks, so 64 aligned rows are promoted (reading R2).
    p, t, h, w = 384, 21, 24, 40
    g = rf.geometry(p, t, h, w, 0.8)
    assert (g.aligned, g.sparse, g.promoted, g.nb, g.n_pb, g.lp) == (20160, 20096, 64, 157, 4, 448)
    src = rf.permutation(g)
    promoted = (src[p:g.lp] - p).tolist()
    assert len(promoted) == 64
    # the leftover is the last whole 8x8 tile of the last frame, in tile order
    ys = [(v % (h * w)) // w for v in promoted]
    xs = [v % w for v in promoted]
    assert all(v // (h * w) == t - 1 for v in promoted)
    assert set(ys) == set(range(16, 24)) and set(xs) == set(range(32, 40))
    # ragged grid: promoted = every token outside the 8x8-aligned area, in raster order
    p, t, h, w = 512, 21, 30, 52
    g = rf.geometry(p, t, h, w, 0.8)
    assert (g.h8, g.w8, g.aligned, g.sparse, g.promoted) == (24, 48, 24192, 24192, 8568)
    assert (g.lp, g.n_pb, g.nb, g.ns) == (9080, 71, 189, 9)
    src = rf.permutation(g)
    promoted = (src[p:g.lp] - p).tolist()
    raster_ragged = [v for v in range(t * h * w) if (v % (h * w)) // w >= 24 or v % w >= 48]
    assert promoted == raster_ragged


def test_tiny_and_config_counts():
    g = rf.geometry(128, 9, 16, 32, 0.8)
    assert (g.sparse, g.nb, g.ns, g.promoted, g.n_pb, g.length) == (4608, 36, 4, 0, 1, 4736)
    g = rf.geometry(512, 21, 48, 80, 0.8)
    assert (g.nb, g.ns, g.n_pb, g.length, g.k) == (630, 30, 4, 81152, 126)
    g = rf.geometry(256, 13, 32, 48, 0.8)
    assert (g.nb, g.ns, g.n_pb, g.promoted) == (156, 12, 2, 0)


def test_sink_blocks_cover_exactly_the_first_frame():
    for (p, t, h, w) in [(128, 9, 16, 32), (256, 62, 24, 42), (512, 21, 30, 52), (0, 3, 8, 8)]:
        g = rf.geometry(p, t, h, w, 0.8)
        src = rf.permutation(g)
        frame = (src[g.lp:] - p) // (h * w)          # frame of every sparse row
        first_frame_blocks = {i // 128 for i in np.nonzero(frame == 0)[0].tolist()}
        assert first_frame_blocks == set(range(g.ns))


@pytest.mark.parametrize("nb", [32, 36, 189, 465, 630])
def test_keep_count_closed_forms(nb):
    assert rf.keep_count(nb, 0.0) == nb          # sparsity 0 disables sparsity
    assert rf.keep_count(nb, 1.0) == 0
    prev = nb
    for s in np.linspace(0, 1, 21):
        k = rf.keep_count(nb, float(s))
        assert k <= prev
        prev = k
        # nominal: the dropped fraction is s up to one block
        assert abs((nb - k) / nb - s) <= 1.0 / nb + 1e-12
    with pytest.raises(ValueError):
        rf.keep_count(nb, 1.5)
    with pytest.raises(ValueError):
        rf.keep_count(nb, float("nan"))


def test_short_video_runs_dense():
    g = rf.geometry(64, 2, 16, 16, 0.9)             # 512 video tokens = 4 blocks < 32
    assert g.dense and g.k == g.nb
    g = rf.geometry(64, 8, 16, 32, 0.9)             # 32 blocks: not dense
    assert not g.dense and g.nb == 32


# ---------------- frame-pair token order ([PR] change summary, reading R17) ----------------

def _nested_loop_frame_pair_order(t, h, w):
    """Frame-pair order written as explicit loops: frame 0 in tile order, then
    each frame pair cube by cube (frame in pair inside the cube), then an
    unpaired last frame in tile order, then the ragged tokens in raster order."""
    h8, w8 = 8 * (h // 8), 8 * (w // 8)

    def one_frame(tau):
        out = []
        for hb in range(h8 // 8):
            for wb in range(w8 // 8):
                for hi in range(8):
                    for wi in range(8):
                        out.append(tau * h * w + (8 * hb + hi) * w + 8 * wb + wi)
        return out

    order = one_frame(0) if t > 0 else []
    tau = 1
    while tau + 1 < t:
        for hb in range(h8 // 8):
            for wb in range(w8 // 8):
                for fi in range(2):
                    for hi in range(8):
                        for wi in range(8):
                            order.append((tau + fi) * h * w + (8 * hb + hi) * w + 8 * wb + wi)
        tau += 2
    if tau < t:
        order += one_frame(tau)
    for tau in range(t):
        for y in range(h):
            for x in range(w):
                if y >= h8 or x >= w8:
                    order.append(tau * h * w + y * w + x)
    return order


@pytest.mark.parametrize("t,h,w", [(1, 8, 8), (2, 16, 24), (3, 13, 21), (4, 30, 52), (5, 8, 16),
                                   (6, 7, 9), (7, 17, 40), (0, 8, 8)])
def test_frame_pair_order_equals_nested_loops(t, h, w):
    assert rf.video_order(t, h, w, "frame_pair") == _nested_loop_frame_pair_order(t, h, w)


def test_frame_pair_order_of_one_or_two_frames_is_tile_order():
    # with t <= 2 no pair exists: frame 0 alone, then (t = 2) the unpaired frame 1
    for (t, h, w) in [(1, 16, 24), (2, 16, 24), (2, 13, 21)]:
        assert rf.video_order(t, h, w, "frame_pair") == rf.video_order(t, h, w, "tile")


@pytest.mark.parametrize("p,t,h,w", [(128, 9, 16, 32), (512, 3, 30, 52), (0, 4, 24, 42), (7, 1, 5, 5),
                                     (384, 21, 24, 40), (1, 6, 17, 9)])
def test_frame_pair_permutation_round_trips_and_keeps_counts(p, t, h, w):
    g_tile = rf.geometry(p, t, h, w, 0.8)
    g = rf.geometry(p, t, h, w, 0.8, "frame_pair")
    # the order changes nothing but the order: every count is the tile order's
    assert dataclasses_replace_order(g_tile) == g
    src = rf.permutation(g)
    assert sorted(src.tolist()) == list(range(g.length))
    assert np.array_equal(src[:p], np.arange(p))
    x = np.random.default_rng(1).standard_normal((g.length, 2))
    assert np.array_equal(rf.inverse_rows(rf.rearrange_rows(x, src), src), x)
    # the promoted ragged edge is the same set of rows in both orders
    assert set(src[p:g.lp].tolist()) >= set(
        v for v in range(p, g.length) if ((v - p) % (h * w)) // w >= g.h8 or (v - p) % w >= g.w8)


def dataclasses_replace_order(g):
    import dataclasses
    return dataclasses.replace(g, order="frame_pair")


def test_frame_pair_blocks_are_spatiotemporal_cubes():
    # Wan2.2-shaped grid: a frame holds 9 whole blocks, so after the 9 first-frame
    # (sink) blocks every sparse block is one 2x8x8 cube of two consecutive frames.
    p, t, h, w = 512, 21, 30, 52
    g = rf.geometry(p, t, h, w, 0.8, "frame_pair")
    assert (g.nb, g.ns, g.promoted) == (189, 9, 8568)
    src = rf.permutation(g)
    for i in range(g.nb):
        rows = src[g.lp + 128 * i: g.lp + 128 * (i + 1)] - p
        tau = rows // (h * w)
        y = (rows % (h * w)) // w
        x = rows % w
        cells = set(zip((y // 8).tolist(), (x // 8).tolist()))
        frames = sorted(set(tau.tolist()))
        if i < g.ns:
            assert frames == [0] and len(cells) == 2       # first frame: two tiles of frame 0
        else:
            assert len(cells) == 1                          # one 8x8 spatial tile ...
            assert frames == [frames[0], frames[0] + 1] and frames[0] % 2 == 1   # ... of frames (2m+1, 2m+2)
            assert np.array_equal(tau[:64], np.full(64, frames[0]))


def test_frame_pair_sinks_cover_exactly_the_first_frame():
    for (p, t, h, w) in [(128, 9, 16, 32), (256, 62, 24, 42), (512, 21, 30, 52), (0, 4, 8, 16)]:
        g = rf.geometry(p, t, h, w, 0.8, "frame_pair")
        src = rf.permutation(g)
        frame = (src[g.lp:] - p) // (h * w)
        first_frame_blocks = {i // 128 for i in np.nonzero(frame == 0)[0].tolist()}
        assert first_frame_blocks == set(range(g.ns))


def test_unknown_order_is_rejected():
    with pytest.raises(ValueError):
        rf.geometry(0, 2, 8, 8, 0.8, "zigzag")
    with pytest.raises(ValueError):
        rf.video_order(2, 8, 8, "zigzag")


# ---------------- k per configuration (reading R4: k = ceil((1 - s) * nb)) ----------------
#
# "RainFusion Attention" user guide, "Configuration": sparsity is the nominal
# fraction of ranked key blocks dropped.  Reading R4 keeps ceil((1 - s) * nb)
# blocks.  The values below are that rule worked out by hand for every
# configuration of the benchmark, and they are written here as numbers, not
# recomputed: a floor (or round-half-down) implementation fails on Tiny
# (7.2 -> 8), Wan (37.8 -> 38), MiniMax at 0.5 and 0.9 (232.5 -> 233,
# 46.5 -> 47) and both TND sequences (31.2, 31.4 -> 32); the guard against
# float noise is exercised by MiniMax at 0.8 ((1 - 0.8) * 465 = 92.99999...).
PINNED_K = [
    # (prefix, t, h, w, sparsity, nb, k)
    (128, 9, 16, 32, 0.8, 36, 8),          # Tiny
    (512, 21, 30, 52, 0.8, 189, 38),       # Wan2.2-shaped
    (256, 62, 24, 42, 0.5, 465, 233),      # MiniMax-H3-shaped sweep
    (256, 62, 24, 42, 0.8, 465, 93),
    (256, 62, 24, 42, 0.9, 465, 47),
    (512, 21, 48, 80, 0.0, 630, 630),      # Aligned sweep
    (512, 21, 48, 80, 0.5, 630, 315),
    (512, 21, 48, 80, 0.8, 630, 126),
    (512, 21, 48, 80, 0.9, 630, 63),
    (256, 13, 32, 48, 0.8, 156, 32),       # TND sequence 0
    (384, 21, 24, 40, 0.8, 157, 32),       # TND sequence 1
]


@pytest.mark.parametrize("p,t,h,w,s,nb,k", PINNED_K)
def test_keep_count_pinned_per_configuration(p, t, h, w, s, nb, k):
    g = rf.geometry(p, t, h, w, s)
    assert (g.nb, g.k) == (nb, k)
    assert rf.keep_count(nb, s) == k


def test_keep_count_pins_reject_a_floor(monkeypatch):
    """Plant the likeliest mistake (floor instead of ceiling) in the oracle and check
    that the pinned table catches it."""
    import math as _math
    monkeypatch.setattr(rf.math, "ceil", _math.floor)
    wrong = [(p, t, h, w, s) for (p, t, h, w, s, nb, k) in PINNED_K if rf.geometry(p, t, h, w, s).k != k]
    assert len(wrong) >= 6, wrong


# Key-side counts with 64-row key blocks (reading R26), worked out by hand for the same
# configurations: n_pb64 = ceil(Lp / 64), nb64 = 2 nb, ns64 = min(nb64, ceil(h8 w8 / 64)),
# k64 = ceil((1 - s) nb64 - 1e-6).
PINNED_K64 = [
    # (prefix, t, h, w, sparsity, n_pb64, nb64, ns64, k64)
    (128, 9, 16, 32, 0.8, 2, 72, 8, 15),          # Tiny: Lp 128, first frame 512 tokens, 14.4 -> 15
    (512, 21, 30, 52, 0.8, 142, 378, 18, 76),     # Wan2.2-shaped: Lp 9,080, 24 x 48 first frame, 75.6 -> 76
    (256, 62, 24, 42, 0.5, 51, 930, 15, 465),     # MiniMax-H3-shaped: Lp 3,232, 24 x 40 first frame
    (256, 62, 24, 42, 0.8, 51, 930, 15, 186),
    (256, 62, 24, 42, 0.9, 51, 930, 15, 93),
    (512, 21, 48, 80, 0.0, 8, 1260, 60, 1260),    # Aligned: Lp 512, 48 x 80 first frame
    (512, 21, 48, 80, 0.5, 8, 1260, 60, 630),
    (512, 21, 48, 80, 0.8, 8, 1260, 60, 252),
    (512, 21, 48, 80, 0.9, 8, 1260, 60, 126),
    (256, 13, 32, 48, 0.8, 4, 312, 24, 63),       # TND sequence 0: 62.4 -> 63
    (384, 21, 24, 40, 0.8, 7, 314, 15, 63),       # TND sequence 1: Lp 448 (64 promoted), 62.8 -> 63
]


@pytest.mark.parametrize("p,t,h,w,s,npb,nb,ns,k", PINNED_K64)
def test_key_blocks_of_64_rows_pinned_per_configuration(p, t, h, w, s, npb, nb, ns, k):
    kb = rf.key_blocks(rf.geometry(p, t, h, w, s), 64)
    assert (kb.n_pb, kb.nb, kb.ns, kb.k) == (npb, nb, ns, k)
