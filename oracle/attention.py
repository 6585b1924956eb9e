"""Block-sparse and dense softmax attention and its gradients (oracle, fp64).

Test infrastructure: imported only by the tests, the smoke check and the
CPU baseline of the benchmark.

Follows DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 3 and Significance (block-wise execution: the
attention output of every query is recomputed over the kept key blocks only).

Definition: for each query token q of query block I,
    O_q = sum_{k in keys(I)} softmax_k(scale * q . k) v_k,
where keys(I) are the tokens of the kept key blocks that exist (index < N).
A query block with no kept key block has an empty sum: O = 0, lse = -inf.
scale defaults to 1/sqrt(D). lse_q = log sum_k exp(scale * q . k).
Inputs are the bf16 tensors widened exactly to fp64.
"""
from __future__ import annotations

import math

import numpy as np


def block_sparse_attention(qp, kp, vp, kv_idx, kv_cnt, blk, scale=None, rows=None, allowed=None):
    """O [B, nh, N, D] and lse [B, nh, N] over the kept blocks (curve order).

    ``rows`` optionally restricts the work to a list of (b, h, I) query
    blocks; the other outputs are left as NaN. ``allowed(q_pos, k_pos)``
    optionally drops (query, key) pairs inside the kept blocks: it maps
    arrays of query and key positions to a boolean matrix.
    """
    q = np.asarray(qp, dtype=np.float64)
    k = np.asarray(kp, dtype=np.float64)
    v = np.asarray(vp, dtype=np.float64)
    B, nh, N, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    nb = -(-N // blk)
    out = np.full((B, nh, N, D), np.nan)
    lse = np.full((B, nh, N), np.nan)
    if rows is None:
        rows = [(b, h, I) for b in range(B) for h in range(nh) for I in range(nb)]
    for (b, h, I) in rows:
        q_lo, q_hi = I * blk, min((I + 1) * blk, N)
        c = int(kv_cnt[b, h, I])
        keys = [np.arange(J * blk, min((J + 1) * blk, N)) for J in kv_idx[b, h, I, :c]]
        if not keys:
            out[b, h, q_lo:q_hi] = 0.0
            lse[b, h, q_lo:q_hi] = -np.inf
            continue
        ks = np.concatenate(keys)
        s = (q[b, h, q_lo:q_hi] @ k[b, h, ks].T) * scale
        if allowed is not None:
            s = np.where(allowed(np.arange(q_lo, q_hi), ks), s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        out[b, h, q_lo:q_hi] = (e / z) @ v[b, h, ks]
        lse[b, h, q_lo:q_hi] = (m + np.log(z))[:, 0]
    return out, lse


def block_sparse_attention_bwd(qp, kp, vp, dop, kv_idx, kv_cnt, blk, scale=None, rows=None):
    """Gradients of the block-sparse attention (fp64), as training through
    block attention needs them (VMoBA: Mixture of Block Attention for Video
    Diffusion Models, abstract: training speed-ups of the block attention).

    For a loss L with dL/dO = dop, the attention of each query block over its
    kept keys (the forward definition above) has, per query row q and kept
    key k (P = softmax of the scaled logits, the reverse-mode rule of the
    softmax-weighted sum):
        dV_k += P_qk dO_q
        dP_qk = dO_q . v_k,   D_q = dO_q . O_q = sum_k P_qk dP_qk
        dS_qk = P_qk (dP_qk - D_q)
        dQ_q  = scale sum_k dS_qk k_k
        dK_k += scale dS_qk q_q
    A key block kept by several query blocks sums their contributions.
    Returns dQ, dK, dV [B, nh, N, D]. ``rows`` restricts the query blocks
    that contribute (dQ of the others is NaN; dK, dV then hold only the
    listed blocks' contributions).
    """
    q = np.asarray(qp, dtype=np.float64)
    k = np.asarray(kp, dtype=np.float64)
    v = np.asarray(vp, dtype=np.float64)
    do = np.asarray(dop, dtype=np.float64)
    B, nh, N, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    nb = -(-N // blk)
    dq = np.full((B, nh, N, D), np.nan)
    dk = np.zeros((B, nh, N, D))
    dv = np.zeros((B, nh, N, D))
    if rows is None:
        rows = [(b, h, I) for b in range(B) for h in range(nh) for I in range(nb)]
    for (b, h, I) in rows:
        q_lo, q_hi = I * blk, min((I + 1) * blk, N)
        c = int(kv_cnt[b, h, I])
        keys = [np.arange(J * blk, min((J + 1) * blk, N)) for J in kv_idx[b, h, I, :c]]
        if not keys:
            dq[b, h, q_lo:q_hi] = 0.0
            continue
        ks = np.concatenate(keys)
        s = (q[b, h, q_lo:q_hi] @ k[b, h, ks].T) * scale
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        o = p @ v[b, h, ks]
        g = do[b, h, q_lo:q_hi]
        dp = g @ v[b, h, ks].T
        Dq = (g * o).sum(axis=1, keepdims=True)
        ds = p * (dp - Dq)
        dq[b, h, q_lo:q_hi] = scale * (ds @ k[b, h, ks])
        np.add.at(dk[b, h], ks, scale * (ds.T @ q[b, h, q_lo:q_hi]))
        np.add.at(dv[b, h], ks, p.T @ g)
    return dq, dk, dv


def dense_attention(qp, kp, vp, scale=None):
    """Full softmax attention, [B, nh, N, D] in and out (fp64)."""
    q = np.asarray(qp, dtype=np.float64)
    k = np.asarray(kp, dtype=np.float64)
    v = np.asarray(vp, dtype=np.float64)
    D = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    s = np.einsum("bhid,bhjd->bhij", q, k) * scale
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return np.einsum("bhij,bhjd->bhid", e / e.sum(axis=-1, keepdims=True), v)
