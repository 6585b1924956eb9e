"""Frame-structured block mask of LVSA (oracle).

Follows LVSA: Training-Free Sparse Attention for Long Video Diffusion,
section 2 (core mechanism): query frame t attends to the frame set
A(t) = G u W(t), where
  * G_s are rotating periodic global anchor frames, shifted by s mod T_per at
    denoising step s, so that over T_per consecutive steps every frame is an
    anchor exactly once;
  * W(t) is a local window around t, expanded where it overlaps anchors so
    that |A(t)| stays at the budget C (C = 21 frames for Wan 2.1 1.3B).

Readings:
  * G_s = {f in [0, T): (f - s) mod T_per == 0};
  * the window part is the (C - |G_s|) non-anchor frames nearest to t,
    scanned at distance 0, 1, 2, ... with t - d before t + d and frames
    outside [0, T) skipped, so |A(t)| = C exactly whenever T >= C;
  * tokens keep raster order (frames stay contiguous) and a frame holds
    P = H * W tokens;
  * key block J is kept for query block I when some frame touched by J lies
    in the union of A(t) over the frames t touched by I. Attention is then
    exact for this block mask;
  * frame-exact attention additionally drops, inside the kept blocks, every
    (query, key) pair whose key frame is not in A(query frame), so the
    attended set is exactly A(t) (frame_allowed).
"""
from __future__ import annotations

import numpy as np


def anchors(T, T_per, s):
    """G_s as a sorted list."""
    return [f for f in range(T) if (f - s) % T_per == 0]


def window(T, t, G, C):
    """The expanded window: the (C - |G|) nearest non-anchor frames to t."""
    need = max(0, C - len(G))
    Gs = set(G)
    picked = []
    d = 0
    while len(picked) < need and d < T:
        cands = [t] if d == 0 else [t - d, t + d]
        for f in cands:
            if 0 <= f < T and f not in Gs and len(picked) < need:
                picked.append(f)
        d += 1
    return picked


def frame_set(T, t, T_per, C, s):
    """A(t) at step s."""
    G = anchors(T, T_per, s)
    return sorted(set(G) | set(window(T, t, G, C)))


def block_frames(X, blk, N, P):
    lo = X * blk
    hi = min(lo + blk, N) - 1
    return range(lo // P, hi // P + 1)


def block_mask(T, P, blk, T_per, C, s):
    """Boolean [nb, nb] mask: row I keeps column J."""
    N = T * P
    nb = -(-N // blk)
    A = [set(frame_set(T, t, T_per, C, s)) for t in range(T)]
    m = np.zeros((nb, nb), dtype=bool)
    for I in range(nb):
        allowed = set()
        for t in block_frames(I, blk, N, P):
            allowed |= A[t]
        for J in range(nb):
            m[I, J] = any(f in allowed for f in block_frames(J, blk, N, P))
    return m


def frame_allowed(T, T_per, C, s):
    """Boolean [T, T]: query frame t may attend key frame f iff f in A(t)."""
    m = np.zeros((T, T), dtype=bool)
    for t in range(T):
        m[t, frame_set(T, t, T_per, C, s)] = True
    return m
