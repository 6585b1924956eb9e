"""Global 3D Hilbert-curve order of a T x H x W token grid (oracle).

Follows DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 1 (3D Hilbert-curve token reordering): tokens are
reordered along one global 3D Hilbert curve before attention so that
spatiotemporal neighbours stay close in the 1-D sequence.

Reading (the page names the curve but not its construction for grids whose
sides are not powers of two): the generalised Hilbert curve built by
recursive splitting of an arbitrary box (the published "gilbert"
construction), restated here from its description.

Definition. A box is (p, a, b, c): p is a grid cell, a, b, c are mutually
orthogonal axis-parallel integer vectors with lengths w = |a|, h = |b|,
d = |c| and unit directions a^, b^, c^. It covers the cells
p + i a^ + j b^ + k c^ (0 <= i < w, 0 <= j < h, 0 <= k < d). Its curve starts
at p and ends at p + (w - 1) a^, the next cell along the major axis a.

  * A box with two unit sides is walked straight along its third side.
  * Otherwise each side is halved, v' = v/2 rounded toward zero; if |v'| is
    odd and |v| > 2, |v'| grows by one (even halves keep corner parity).
  * (wide)    2w > 3h and 2w > 3d: two boxes (p, a', b, c), (p + a', a - a', b, c).
  * (tall)    else 3h > 4d: three boxes
        (p, b', c, a'),  (p + b', a, b - b', c),
        (p + (a - a^) + (b' - b^), -b', c, -(a - a')).
  * (deep)    else 3d > 4h: three boxes
        (p, c', a', b),  (p + c', a, b, c - c'),
        (p + (a - a^) + (c' - c^), -c', -(a - a'), b).
  * (regular) else five boxes
        (p, b', c', a'),
        (p + b', c, a', b - b'),
        (p + (b' - b^) + (c - c^), a, -b', -(c - c')),
        (p + (a - a^) + b' + (c - c^), -c, -(a - a'), b - b'),
        (p + (a - a^) + (b' - b^), -b', c', -(a - a')).
The sub-boxes tile the box and each one starts next to where the previous
one ends, so the whole box is one path.

Top level: p = (0, 0, 0); a runs along the longest grid side (ties go to W,
then H, then T); b and c are the other two sides in the order W, H, T.
Coordinates here are (t, h, w); the raster index is (t*H + h)*W + w.

This module enumerates the curve by full recursive traversal. It is
independent of the CUDA kernel, which locates each rank by descending the
same definition.
"""
from __future__ import annotations

import sys

import numpy as np

sys.setrecursionlimit(10000)


def _add(u, v):
    return (u[0] + v[0], u[1] + v[1], u[2] + v[2])


def _sub(u, v):
    return (u[0] - v[0], u[1] - v[1], u[2] - v[2])


def _neg(u):
    return (-u[0], -u[1], -u[2])


def _length(u):
    return abs(u[0]) + abs(u[1]) + abs(u[2])


def _unit(u):
    return tuple((x > 0) - (x < 0) for x in u)


def _half(u):
    """Half of an axis vector, rounded toward zero, made even when |u| > 2."""
    n = _length(u)
    h = n // 2
    if h % 2 == 1 and n > 2:
        h += 1
    s = _unit(u)
    return (s[0] * h, s[1] * h, s[2] * h)


def _walk(p, a, b, c, out):
    w, h, d = _length(a), _length(b), _length(c)
    if w == 0 or h == 0 or d == 0:
        raise ValueError("empty sub-box in Hilbert recursion")
    if h == 1 and d == 1:
        step = _unit(a)
        for i in range(w):
            out.append((p[0] + i * step[0], p[1] + i * step[1], p[2] + i * step[2]))
        return
    if w == 1 and d == 1:
        step = _unit(b)
        for i in range(h):
            out.append((p[0] + i * step[0], p[1] + i * step[1], p[2] + i * step[2]))
        return
    if w == 1 and h == 1:
        step = _unit(c)
        for i in range(d):
            out.append((p[0] + i * step[0], p[1] + i * step[1], p[2] + i * step[2]))
        return

    a2, b2, c2 = _half(a), _half(b), _half(c)
    ua, ub, uc = _unit(a), _unit(b), _unit(c)
    a_end = _sub(a, ua)              # a - a^
    if 2 * w > 3 * h and 2 * w > 3 * d:
        _walk(p, a2, b, c, out)
        _walk(_add(p, a2), _sub(a, a2), b, c, out)
    elif 3 * h > 4 * d:
        _walk(p, b2, c, a2, out)
        _walk(_add(p, b2), a, _sub(b, b2), c, out)
        _walk(_add(p, _add(a_end, _sub(b2, ub))), _neg(b2), c, _neg(_sub(a, a2)), out)
    elif 3 * d > 4 * h:
        _walk(p, c2, a2, b, out)
        _walk(_add(p, c2), a, b, _sub(c, c2), out)
        _walk(_add(p, _add(a_end, _sub(c2, uc))), _neg(c2), _neg(_sub(a, a2)), b, out)
    else:
        c_end = _sub(c, uc)
        _walk(p, b2, c2, a2, out)
        _walk(_add(p, b2), c, a2, _sub(b, b2), out)
        _walk(_add(p, _add(_sub(b2, ub), c_end)), a, _neg(b2), _neg(_sub(c, c2)), out)
        _walk(_add(p, _add(a_end, _add(b2, c_end))), _neg(c), _neg(_sub(a, a2)), _sub(b, b2), out)
        _walk(_add(p, _add(a_end, _sub(b2, ub))), _neg(b2), c2, _neg(_sub(a, a2)), out)


def top_level_axes(T, H, W):
    """(a, b, c) of the whole grid in (t, h, w) coordinates."""
    ext = {"w": W, "h": H, "t": T}
    vec = {"w": (0, 0, W), "h": (0, H, 0), "t": (T, 0, 0)}
    order = ["w", "h", "t"]
    major = max(order, key=lambda k: (ext[k], -order.index(k)))
    rest = [k for k in order if k != major]
    return vec[major], vec[rest[0]], vec[rest[1]]


def hilbert_cells(T, H, W):
    """The grid cells (t, h, w) in curve order."""
    if T <= 0 or H <= 0 or W <= 0:
        raise ValueError("grid sides must be positive")
    a, b, c = top_level_axes(T, H, W)
    out = []
    _walk((0, 0, 0), a, b, c, out)
    return out


def raster_index(cells, H, W):
    arr = np.asarray(cells, dtype=np.int64)
    return (arr[:, 0] * H + arr[:, 1]) * W + arr[:, 2]


def hilbert_perm(T, H, W):
    """perm[i] = raster index of the i-th token along the curve; inv[perm[i]] = i."""
    perm = raster_index(hilbert_cells(T, H, W), H, W).astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return perm, inv


def hilbert2d_cells(T, H, W):
    """Frame-major cells with a 2-D Hilbert curve inside every frame.

    Reading of DFSAttn, Results (ablation studies: the 3D Hilbert order is
    compared with raster scans and with 2-D Hilbert curves; the page does not
    define the 2-D variant): frames are kept whole and in time order, as a
    per-frame (spatial-only) curve implies, and every frame's H x W tokens
    follow the generalised Hilbert curve of that rectangle -- the definition
    above applied to the 1 x H x W box, which on 2^k x 2^k squares is the
    textbook 2-D Hilbert curve. Every frame uses the same path."""
    frame = [(h, w) for (_, h, w) in hilbert_cells(1, H, W)]
    return [(t, h, w) for t in range(T) for (h, w) in frame]


def hilbert2d_perm(T, H, W):
    perm = raster_index(hilbert2d_cells(T, H, W), H, W).astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return perm, inv


def raster_perm(T, H, W):
    """The identity order (plain row-major flattening used by standard DiTs)."""
    perm = np.arange(T * H * W, dtype=np.int32)
    return perm, perm.copy()


def tile_dims(order, blk):
    """Tile (t, h, w) extents of the tiled orders: blk tokens per full tile.

    Reading of VMoBA: Mixture of Block Attention for Video Diffusion Models,
    abstract, modification (1) (1-D, 2-D and 3-D block partitions; the
    abstract gives no tile shapes): 2-D tiles are 1 x 8 x (blk/8) patches of
    one frame, 3-D tiles are 2 x 8 x (blk/16) cubes; 1-D is the raster order.
    """
    if order == "tile2d":
        return (1, 8, blk // 8)
    if order == "tile3d":
        return (2, 8, blk // 16)
    raise ValueError(order)


def tiled_cells(T, H, W, tile):
    """Cells in tile-major order: tiles in raster order over the tile grid
    (tiles clipped at the grid's far edges), raster order inside a tile."""
    ct, ch, cw = tile
    out = []
    for t0 in range(0, T, ct):
        for h0 in range(0, H, ch):
            for w0 in range(0, W, cw):
                for t in range(t0, min(t0 + ct, T)):
                    for h in range(h0, min(h0 + ch, H)):
                        for w in range(w0, min(w0 + cw, W)):
                            out.append((t, h, w))
    return out


def tiled_perm(T, H, W, tile):
    perm = raster_index(tiled_cells(T, H, W, tile), H, W).astype(np.int32)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return perm, inv


def make_perm(order, T, H, W, blk=128):
    if order == "hilbert3d":
        return hilbert_perm(T, H, W)
    if order == "hilbert2d":
        return hilbert2d_perm(T, H, W)
    if order == "raster":
        return raster_perm(T, H, W)
    if order in ("tile2d", "tile3d"):
        return tiled_perm(T, H, W, tile_dims(order, blk))
    raise ValueError(order)


def permute_tokens(x, perm):
    """x [B, N, nh, D] (raster) -> xp [B, nh, N, D] with xp[:, h, i] = x[:, perm[i], h]."""
    return np.ascontiguousarray(np.transpose(np.asarray(x)[:, perm, :, :], (0, 2, 1, 3)))


def unpermute_tokens(op, perm):
    """op [B, nh, N, D] (curve order) -> o [B, N, nh, D] with o[:, perm[i], h] = op[:, h, i]."""
    op = np.asarray(op)
    B, nh, N, D = op.shape
    o = np.empty((B, N, nh, D), dtype=op.dtype)
    o[:, perm, :, :] = np.transpose(op, (0, 2, 1, 3))
    return o
