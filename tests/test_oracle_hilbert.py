"""Pins of the oracle's 3D Hilbert order against properties fixed elsewhere.

Page: DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 1 (a global 3D Hilbert curve keeps
spatiotemporal neighbours adjacent in the 1-D order).
"""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import hilbert

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hilbert_small.json")
CONFIG_GRIDS = [(8, 16, 16), (21, 30, 52), (63, 30, 52), (33, 45, 80)]


def _steps(cells):
    a = np.asarray(cells, dtype=np.int64)
    return np.abs(np.diff(a, axis=0))


def _textbook_2d(n, d):
    """Distance -> (x, y) on the n x n Hilbert curve by the classic
    quadrant-rotation method (independent of the box-splitting recursion)."""
    x = y = 0
    s = 1
    t = d
    while s < n:
        rx = 1 & (t // 2)
        ry = 1 & (t ^ rx)
        if ry == 0:
            if rx == 1:
                x, y = s - 1 - x, s - 1 - y
            x, y = y, x
        x += s * rx
        y += s * ry
        t //= 4
        s *= 2
    return x, y


def test_bijection_and_unit_steps_all_small_grids():
    for T, H, W in itertools.product(range(1, 9), repeat=3):
        cells = hilbert.hilbert_cells(T, H, W)
        assert len(cells) == T * H * W
        assert len(set(cells)) == T * H * W
        a = np.asarray(cells)
        assert a.min() >= 0 and (a.max(axis=0) < np.array([T, H, W])).all()
        if len(cells) > 1:
            # every step moves to a cell that touches the previous one
            assert _steps(cells).max(axis=1).max() == 1, (T, H, W)


@pytest.mark.parametrize("T,H,W", CONFIG_GRIDS)
def test_config_grids_bijection_and_unit_steps(T, H, W):
    perm, inv = hilbert.hilbert_perm(T, H, W)
    N = T * H * W
    assert np.array_equal(np.sort(perm), np.arange(N))
    assert np.array_equal(inv[perm], np.arange(N))
    t, r = np.divmod(perm, H * W)
    h, w = np.divmod(r, W)
    st = np.abs(np.diff(np.stack([t, h, w], 1), axis=0))
    assert st.max(axis=1).max() == 1


def test_even_grids_are_face_adjacent():
    # With every side even a face-adjacent path between the chosen corners
    # exists; the construction must find one.
    for T, H, W in itertools.product(range(2, 13, 2), repeat=3):
        st = _steps(hilbert.hilbert_cells(T, H, W))
        assert st.sum(axis=1).max() == 1, (T, H, W)


def test_tiny_workload_grid_has_no_diagonal_step():
    st = _steps(hilbert.hilbert_cells(8, 16, 16))
    assert int((st.sum(axis=1) > 1).sum()) == 0


def test_diagonal_step_counts_regression():
    # Odd sides force a few diagonal steps; values recorded from the oracle
    # (a regression guard, not an independent pin).
    counts = {}
    for g in CONFIG_GRIDS[1:]:
        st = _steps(hilbert.hilbert_cells(*g))
        counts[g] = int((st.sum(axis=1) > 1).sum())
    assert counts == {(21, 30, 52): 88, (63, 30, 52): 129, (33, 45, 80): 672}


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5])
def test_dyadic_octants_are_contiguous_on_cubes(k):
    # The defining Hilbert property: on a 2^k cube every aligned 2^j sub-cube
    # is visited in one contiguous run, and consecutive cells share a face.
    n = 2 ** k
    a = np.asarray(hilbert.hilbert_cells(n, n, n))
    assert _steps(a).sum(axis=1).max() == 1
    for j in range(1, k + 1):
        s = 2 ** j
        key = (a[:, 0] // s) * n * n + (a[:, 1] // s) * n + a[:, 2] // s
        runs = 1 + np.count_nonzero(np.diff(key))
        assert runs == (n // s) ** 3


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5, 6])
def test_square_reduces_to_textbook_2d_curve(k):
    n = 2 ** k
    mine = [(h, w) for (_, h, w) in hilbert.hilbert_cells(1, n, n)]
    ref = [_textbook_2d(n, d) for d in range(n * n)]
    assert mine == [(y, x) for (x, y) in ref]


def test_golden_small_curves():
    g = json.load(open(GOLDEN))
    assert [list(c) for c in hilbert.hilbert_cells(2, 2, 2)] == g["2x2x2"]
    assert [list(c) for c in hilbert.hilbert_cells(1, 4, 4)] == g["1x4x4"]


def test_lines_are_identity():
    for n in (1, 2, 7, 64):
        assert np.array_equal(hilbert.hilbert_perm(1, 1, n)[0], np.arange(n))
        assert np.array_equal(hilbert.hilbert_perm(1, n, 1)[0], np.arange(n))
        assert np.array_equal(hilbert.hilbert_perm(n, 1, 1)[0], np.arange(n))


@pytest.mark.parametrize("T,H,W", [(3, 5, 7), (8, 16, 16), (21, 30, 52), (4, 4, 9)])
def test_endpoints(T, H, W):
    cells = hilbert.hilbert_cells(T, H, W)
    assert cells[0] == (0, 0, 0)
    a, _, _ = hilbert.top_level_axes(T, H, W)
    end = tuple(max(0, x - 1) for x in a)
    assert cells[-1] == end


def test_permute_roundtrip():
    rng = np.random.default_rng(1)
    T, H, W, nh, D = 3, 4, 5, 2, 8
    x = rng.standard_normal((1, T * H * W, nh, D))
    perm, _ = hilbert.hilbert_perm(T, H, W)
    xp = hilbert.permute_tokens(x, perm)
    for i in range(T * H * W):
        assert np.array_equal(xp[0, :, i, :], x[0, perm[i], :, :])
    assert np.array_equal(hilbert.unpermute_tokens(xp, perm), x)


@pytest.mark.parametrize("order", ["tile2d", "tile3d"])
@pytest.mark.parametrize("T,H,W,blk", [(8, 16, 16, 64), (21, 30, 52, 128), (4, 16, 32, 128), (3, 5, 7, 64)])
def test_tiled_orders(order, T, H, W, blk):
    perm, inv = hilbert.make_perm(order, T, H, W, blk)
    N = T * H * W
    assert np.array_equal(np.sort(perm), np.arange(N)) and np.array_equal(inv[perm], np.arange(N))
    ct, ch, cw = hilbert.tile_dims(order, blk)
    assert ct * ch * cw == blk
    t, r = np.divmod(perm, H * W)
    h, w = np.divmod(r, W)
    # every tile is one contiguous run of the order (tile id from integer division)
    tid = ((t // ct) * (-(-H // ch)) + h // ch) * (-(-W // cw)) + w // cw
    assert 1 + np.count_nonzero(np.diff(tid)) == len(np.unique(tid))
    assert np.all(np.diff(tid) >= 0)                     # tiles in raster order
    if T % ct == 0 and H % ch == 0 and W % cw == 0:
        # then every block of blk consecutive tokens is exactly one full tile
        for b0 in range(0, N, blk):
            sl = slice(b0, b0 + blk)
            assert (t[sl].max() - t[sl].min() + 1, h[sl].max() - h[sl].min() + 1,
                    w[sl].max() - w[sl].min() + 1) == (ct, ch, cw)


def test_tile2d_first_block_by_hand():
    # 1 x 16 x 32 grid, blk 128: the first block is rows 0-7, columns 0-15
    perm, _ = hilbert.make_perm("tile2d", 1, 16, 32, 128)
    assert list(perm[:18]) == list(range(16)) + [32, 33]
    assert perm[127] == 7 * 32 + 15 and perm[128] == 16


@pytest.mark.parametrize("T,k", [(1, 1), (3, 2), (2, 4), (5, 5)])
def test_hilbert2d_frames_follow_the_textbook_curve(T, k):
    """2-D Hilbert order on T x 2^k x 2^k: frame after frame, each frame in the
    order of the textbook 2-D Hilbert curve (quadrant-rotation method)."""
    n = 2 ** k
    perm, inv = hilbert.make_perm("hilbert2d", T, n, n)
    ref = [_textbook_2d(n, d) for d in range(n * n)]
    want = [(t * n + y) * n + x for t in range(T) for (x, y) in ref]
    assert perm.tolist() == want
    assert np.array_equal(inv[perm], np.arange(T * n * n))


@pytest.mark.parametrize("T,H,W", [(3, 5, 7), (2, 30, 52), (4, 45, 80), (2, 1, 9), (3, 6, 2)])
def test_hilbert2d_is_frame_major_and_continuous_in_frames(T, H, W):
    perm, inv = hilbert.make_perm("hilbert2d", T, H, W)
    P = H * W
    assert np.array_equal(np.sort(perm), np.arange(T * P)) and np.array_equal(inv[perm], np.arange(T * P))
    t, r = np.divmod(perm, P)
    assert np.array_equal(t, np.repeat(np.arange(T), P))          # whole frames, in time order
    frames = r.reshape(T, P)
    assert (frames == frames[0]).all()                            # the same path in every frame
    h, w = np.divmod(frames[0], W)
    st = np.abs(np.diff(np.stack([h, w], 1), axis=0))
    if P > 1:
        assert st.max() == 1                                      # each step to a touching cell
    if H % 2 == 0 and W % 2 == 0:
        assert st.sum(axis=1).max() == 1                          # even sides: face steps only
