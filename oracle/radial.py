"""Log-radial static block mask (DynamicRad static-ratio mode) -- oracle.

Test infrastructure: imported only by the tests, the smoke check and the
CPU baseline of the benchmark.

Follows "DynamicRad" (methodology, components 1 and 2): in the static-ratio
mode each (query frame, key frame) pair keeps a fixed share of tokens set
by the temporal distance d between the frames; the window is radial and
logarithmic, shrinking exponentially as d grows, and a long-range factor
lambda keeps far frames from vanishing. The page gives no formula, so the
plainest reading that fits it is taken (each line below is a reading):

  * tokens in raster order, frame t = n // P, spatial index s = n mod P,
    P = H * W tokens per frame;
  * distance bands double in length: band(d) = bit length of d
    (0 -> 0, 1 -> 1, 2..3 -> 2, 4..7 -> 3, ...);
  * window width omega(d) = max(w0 >> band(d), w_far) tokens, with
    w_far = floor(lambda * w0) computed in fp64 from the fp32 lambda;
  * query token q may attend key token k iff 2 * |s_q - s_k| < omega(d),
    d = |t_q - t_k| (a band around the query's own spatial index; w0 >= 2P
    keeps the whole frame at d = 0);
  * key block J is kept for query block I iff some attendable pair
    (q in I, k in J, both < N) exists. Attention is then exact for this
    block mask (a mask generator, like the LVSA block mask).
"""
from __future__ import annotations

import math

import numpy as np


def band(d):
    """Bit length of the non-negative integer d."""
    return int(d).bit_length()


def w_far_of(lam, w0):
    """floor(lambda * w0) with lambda rounded to fp32 first."""
    return int(math.floor(float(np.float32(lam)) * float(w0)))


def window(d, w0, w_far):
    return max(int(w0) >> band(d), int(w_far))


def pair_allowed(q_pos, k_pos, P, w0, w_far):
    """Boolean [len(q_pos), len(k_pos)]: token-level attendability."""
    q = np.asarray(q_pos, dtype=np.int64)[:, None]
    k = np.asarray(k_pos, dtype=np.int64)[None, :]
    d = np.abs(q // P - k // P)
    ds = np.abs(q % P - k % P)
    T = int(max(q.max(initial=0), k.max(initial=0)) // P) + 1
    om = np.array([window(x, w0, w_far) for x in range(T + 1)], dtype=np.int64)
    return 2 * ds < om[d]


def block_mask(T, P, blk, w0, w_far, rows=None):
    """Boolean [nb, nb] (or [len(rows), nb]): row I keeps column J."""
    N = T * P
    nb = -(-N // blk)
    rows = range(nb) if rows is None else rows
    keys = np.arange(N)
    out = np.zeros((len(rows), nb), dtype=bool)
    for r, I in enumerate(rows):
        qs = np.arange(I * blk, min(N, I * blk + blk))
        a = pair_allowed(qs, keys, P, w0, w_far).any(axis=0)
        pad = np.zeros(nb * blk, dtype=bool)
        pad[:N] = a
        out[r] = pad.reshape(nb, blk).any(axis=1)
    return out
