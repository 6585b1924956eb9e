"""The whole hot path, stage by stage, on the CPU in fp64 (oracle).

Order of the stages (DFSAttn: Dynamic Fine-grained Sparse Attention for
Efficient Video Generation, Methodology items 1-3): reorder the tokens along
the 3D Hilbert curve, score blocks hierarchically, select key blocks per
query block, attend over the kept blocks, restore the original token order.
The frame-structured mask of LVSA (section 2) replaces scoring and selection
when ``mode == "lvsa"``.
"""
from __future__ import annotations

import math

import numpy as np

from . import attention, hilbert, lvsa, schedule, scoring, selection


def as_f64(x):
    """bf16 torch tensor or array -> fp64 numpy (exact widening)."""
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def run(q, k, v, *, T, H, W, blk, sb, order, mode, k_keep=0, tau=0.0, cap=0,
        lvsa_T_per=8, lvsa_C=21, lvsa_step=0, scale=None, rows=None, kcap=None):
    """Returns a dict with every intermediate of the path.

    q, k, v: [B, N, nh, D] in raster order. ``rows`` restricts attention to a
    list of (b, h, I) query blocks.
    """
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, N, nh, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    perm, inv = hilbert.make_perm(order, T, H, W, blk)
    qp, kp, vp = (hilbert.permute_tokens(x, perm) for x in (q, k, v))
    nb = -(-N // blk)
    res = {"perm": perm, "inv": inv, "qp": qp, "kp": kp, "vp": vp}
    if mode == "lvsa":
        m = lvsa.block_mask(T, H * W, blk, lvsa_T_per, lvsa_C, lvsa_step)
        mask = np.broadcast_to(m, (B, nh, nb, nb))
        kv_idx, kv_cnt = selection.mask_to_lists(mask, kcap)
        res["scores"] = None
    else:
        s = scoring.block_scores(qp, kp, blk, sb, scale)
        res["scores"] = s
        kv_idx, kv_cnt = selection.select(s, mode, k=k_keep, tau=tau, cap=cap, kcap=kcap)
    res["kv_idx"], res["kv_cnt"] = kv_idx, kv_cnt
    op, lse = attention.block_sparse_attention(qp, kp, vp, kv_idx, kv_cnt, blk, scale, rows=rows)
    res["op"], res["lse"] = op, lse
    res["out"] = hilbert.unpermute_tokens(op, perm)
    return res
