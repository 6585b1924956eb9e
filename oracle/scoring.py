"""Hierarchical block scoring (oracle, fp64).

Follows DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 2 (hierarchical block scoring): each block is
split into sub-blocks, attention scores are computed at sub-block level and
aggregated into one importance per (query block, key block).

Readings (the page names neither the pooling operator nor the aggregation):
  * pooling: the arithmetic mean of the sub-block's valid tokens (the last
    sub-block of a ragged sequence averages only the tokens that exist),
    per head, separately for Q and K;
  * sub-block score: (qbar_i . kbar_j) * scale, scale = 1/sqrt(D) unless
    given;
  * aggregation: the maximum over the query sub-blocks i of block I and the
    key sub-blocks j of block J (sub-blocks past the sequence end do not
    exist). A mean would collapse, by bilinearity, to plain block pooling,
    which is the coarse scheme the item says it improves on; the maximum
    rewards a block that holds any matching centroid.
With sub-block size equal to the block size this is coarse block-mean
pooling, the baseline the same item refines.
"""
from __future__ import annotations

import math

import numpy as np


def pool_subblocks(xp, sb):
    """Mean of each run of sb consecutive tokens: [B, nh, N, D] -> [B, nh, ceil(N/sb), D] (fp64)."""
    x = np.asarray(xp, dtype=np.float64)
    B, nh, N, D = x.shape
    nsb = -(-N // sb)
    out = np.empty((B, nh, nsb, D), dtype=np.float64)
    for j in range(nsb):
        lo, hi = j * sb, min((j + 1) * sb, N)
        out[:, :, j, :] = x[:, :, lo:hi, :].sum(axis=2) / (hi - lo)
    return out


def subblock_scores(qbar, kbar, scale):
    """Pooled logits (qbar_i . kbar_j) * scale: [B, nh, nsb, nsb]."""
    return np.einsum("bhid,bhjd->bhij", qbar, kbar) * scale


def block_scores(qp, kp, blk, sb, scale=None):
    """score[b, h, I, J] = max over sub-blocks i in I, j in J of the pooled logit."""
    if blk % sb != 0:
        raise ValueError("block size must be a multiple of the sub-block size")
    qp = np.asarray(qp)
    B, nh, N, D = qp.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    qbar = pool_subblocks(qp, sb)
    kbar = pool_subblocks(kp, sb)
    r = blk // sb
    nsb = qbar.shape[2]
    nb = -(-N // blk)
    starts = np.arange(0, nsb, r)          # first sub-block of each block
    out = np.empty((B, nh, nb, nb), dtype=np.float64)
    for b in range(B):
        for h in range(nh):
            s = subblock_scores(qbar[b:b + 1, h:h + 1], kbar[b:b + 1, h:h + 1], scale)[0, 0]
            rows = np.maximum.reduceat(s, starts, axis=0)       # max over i in I
            out[b, h] = np.maximum.reduceat(rows, starts, axis=1)  # max over j in J
    return out
