"""Per-query-block key-block selection (oracle).

Follows
  * DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
    Generation, Methodology item 3: a sparsity budget fixes how many key
    blocks each query block keeps (top-k of the block importance);
  * VMoBA: Mixture of Block Attention for Video Diffusion Models, abstract,
    modification (3): threshold-based selection keeps as many blocks as their
    cumulative similarity requires;
  * VMoBA, abstract, modification (2): global block selection ranks
    query-key block pairs across the whole head.

Readings:
  * global selection keeps, per head, the K highest-scoring (query block, key
    block) pairs over all nb x nb pairs, equal scores going to the lower flat
    index I * nb + J; each query block's kept key blocks are listed in
    ascending order (a query block may keep none); K = ceil(ratio * nb^2);
  * top-k keeps the k largest scores of the row; equal scores go to the lower
    key-block index; no block is forced in (no diagonal or sink block);
  * threshold: p = softmax over the row of the block scores (temperature 1,
    the scores already carry the 1/sqrt(D) factor); blocks are ranked by
    score, ties to the lower index; m is the smallest prefix whose mass
    reaches tau; then m = min(m, cap);
  * k and cap come from a keep ratio as ceil(ratio * nb) in exact integer
    arithmetic;
  * the kept indices of a row are listed in ascending order.
The comparisons that decide the kept set are made on float32 scores, the
precision the scoring kernel produces; the threshold mass is summed in fp64.
"""
from __future__ import annotations

import numpy as np


def ratio_count(num, den, nb):
    """ceil(num/den * nb) in integers."""
    return -(-(num * nb) // den)


def rank_order(row):
    """Indices of the row sorted by descending score, ties to the lower index."""
    row = np.asarray(row)
    return np.lexsort((np.arange(row.size), -row.astype(np.float64)))


def topk_row(row, k):
    """Ascending indices of the k best entries of one row."""
    k = max(0, min(int(k), row.size))
    return np.sort(rank_order(row)[:k]).astype(np.int32)


def threshold_count(row, tau, cap):
    """m = min(smallest prefix with softmax mass >= tau, cap), and the sorted cumsum."""
    s = np.asarray(row, dtype=np.float64)
    order = rank_order(row)
    e = np.exp(s - s.max())
    p = e / e.sum()
    csum = np.cumsum(p[order])
    hit = np.nonzero(csum >= tau)[0]
    m = int(hit[0]) + 1 if hit.size else s.size
    return min(m, int(cap)), csum


def threshold_row(row, tau, cap):
    m, _ = threshold_count(row, tau, cap)
    return np.sort(rank_order(row)[:m]).astype(np.int32)


def select(scores, mode, k=0, tau=0.0, cap=0, kcap=None):
    """Kept lists for every row of scores [B, nh, nb, nb].

    Returns kv_idx [B, nh, nb, kcap] (positions past the count hold -1) and
    kv_cnt [B, nh, nb].
    """
    s32 = np.asarray(scores, dtype=np.float32)
    B, nh, nbq, nbk = s32.shape
    if kcap is None:
        kcap = nbk
    idx = np.full((B, nh, nbq, kcap), -1, dtype=np.int32)
    cnt = np.zeros((B, nh, nbq), dtype=np.int32)
    for b in range(B):
        for h in range(nh):
            for I in range(nbq):
                row = s32[b, h, I]
                if mode == "topk":
                    kept = topk_row(row, k)
                elif mode == "threshold":
                    kept = threshold_row(row, tau, cap)
                else:
                    raise ValueError(mode)
                if kept.size > kcap:
                    raise ValueError("kept count exceeds kcap")
                idx[b, h, I, :kept.size] = kept
                cnt[b, h, I] = kept.size
    return idx, cnt


def global_topk_head(scores_head, K):
    """Boolean [nb, nb] mask of the K best pairs of one head (ties: lower flat index)."""
    s = np.asarray(scores_head, dtype=np.float32)
    nbq, nbk = s.shape
    flat = s.reshape(-1)
    K = max(0, min(int(K), flat.size))
    order = np.lexsort((np.arange(flat.size), -flat.astype(np.float64)))
    m = np.zeros(flat.size, dtype=bool)
    m[order[:K]] = True
    return m.reshape(nbq, nbk)


def select_global(scores, K, kcap=None):
    """Per-head global selection of [B, nh, nb, nb] scores -> (kv_idx, kv_cnt)."""
    s32 = np.asarray(scores, dtype=np.float32)
    B, nh = s32.shape[:2]
    mask = np.stack([np.stack([global_topk_head(s32[b, h], K) for h in range(nh)]) for b in range(B)])
    return mask_to_lists(mask, kcap)


def lists_to_mask(kv_idx, kv_cnt, nbk):
    """Dense boolean block mask [B, nh, nbq, nbk] from kept lists."""
    B, nh, nbq, _ = kv_idx.shape
    m = np.zeros((B, nh, nbq, nbk), dtype=bool)
    for b in range(B):
        for h in range(nh):
            for I in range(nbq):
                c = int(kv_cnt[b, h, I])
                m[b, h, I, kv_idx[b, h, I, :c]] = True
    return m


def mask_to_lists(mask, kcap=None):
    B, nh, nbq, nbk = mask.shape
    if kcap is None:
        kcap = nbk
    idx = np.full((B, nh, nbq, kcap), -1, dtype=np.int32)
    cnt = np.zeros((B, nh, nbq), dtype=np.int32)
    for b in range(B):
        for h in range(nh):
            for I in range(nbq):
                js = np.nonzero(mask[b, h, I])[0]
                idx[b, h, I, :js.size] = js
                cnt[b, h, I] = js.size
    return idx, cnt
