"""Adaptive keep budget with cached masks (oracle).

Follows DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 3 (sparse-mask caching with adaptive ratios):
the keep budget decreases monotonically over the diffusion steps, masks are
reused between refreshes at a fixed interval, and attention itself is
recomputed at every step.

Reading for the 50-step workload: the keep ratio falls linearly from 40 % at
step 0 to 10 % at step 49, ratio(s) = (1960 - 30 s) / 4900; the mask is
rebuilt at the steps s with s mod R == 0 (R = 5), with the budget of that
step, k(s) = ceil(ratio(s) * nb) in exact integer arithmetic, and reused
unchanged until the next refresh.
"""
from __future__ import annotations


def keep_ratio_fraction(s, n_steps=50, start_pct=40, end_pct=10):
    """ratio(s) as an exact fraction (num, den)."""
    # start + (end - start) * s / (n_steps - 1), in percent
    num = start_pct * (n_steps - 1) + (end_pct - start_pct) * s
    den = 100 * (n_steps - 1)
    return num, den


def refresh_step(s, R=5):
    """The step whose mask is in use at step s."""
    return s - (s % R)


def is_refresh(s, R=5):
    return s % R == 0


def budget(s, nb, n_steps=50, R=5, start_pct=40, end_pct=10):
    """k used at step s: the budget of the last refresh step."""
    r = refresh_step(s, R)
    num, den = keep_ratio_fraction(r, n_steps, start_pct, end_pct)
    return -(-(num * nb) // den)
