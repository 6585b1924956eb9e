"""Keep-budget schedule and mask-refresh rule for the denoising loop (host).

DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 3: the sparsity budget decreases monotonically
over diffusion steps, and masks are cached and refreshed at a fixed
interval while attention is recomputed every step.

The keep ratio falls linearly from start_pct % at step 0 to end_pct % at the
last step; the budget in use at step s is that of the last refresh step
r = s - s mod R, k = ceil(ratio(r) * nb), in integers.
"""
from __future__ import annotations


def is_refresh(step: int, refresh: int = 5) -> bool:
    """True at the steps where the mask is rebuilt."""
    return step % refresh == 0


def keep_budget(step: int, nb: int, n_steps: int = 50, refresh: int = 5,
                start_pct: int = 40, end_pct: int = 10) -> int:
    """Key blocks kept per query block at `step`."""
    r = step - step % refresh
    span = n_steps - 1
    # ratio(r) * nb = nb * (start * span - (start - end) * r) / (100 * span)
    num = nb * (start_pct * span - (start_pct - end_pct) * r)
    den = 100 * span
    return (num + den - 1) // den
