"""Pins of the oracle's block-sparse attention.

Page: DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 3 and Significance (block-wise execution over
the kept blocks). A full mask is plain dense attention.
"""
import math

import numpy as np
import pytest

from oracle import attention, hilbert, pipeline, selection


def _qkv(B, nh, N, D, seed=0):
    r = np.random.default_rng(seed)
    return [r.standard_normal((B, nh, N, D)) for _ in range(3)]


def _full_lists(B, nh, nb):
    idx = np.tile(np.arange(nb, dtype=np.int32), (B, nh, nb, 1))
    cnt = np.full((B, nh, nb), nb, dtype=np.int32)
    return idx, cnt


def _loops_dense(q, k, v, scale):
    """Softmax attention written with scalar loops and math.exp."""
    N, D = q.shape
    out = np.zeros((N, D))
    for i in range(N):
        logits = [scale * sum(q[i, d] * k[j, d] for d in range(D)) for j in range(N)]
        m = max(logits)
        e = [math.exp(x - m) for x in logits]
        z = sum(e)
        for d in range(D):
            out[i, d] = sum(e[j] * v[j, d] for j in range(N)) / z
    return out


def test_dense_matches_scalar_loops():
    q, k, v = _qkv(1, 1, 13, 4)
    ref = _loops_dense(q[0, 0], k[0, 0], v[0, 0], 0.5)
    got = attention.dense_attention(q, k, v, 0.5)[0, 0]
    assert np.abs(got - ref).max() < 1e-12


def test_full_mask_is_dense():
    B, nh, N, D, blk = 1, 2, 37, 8, 8
    q, k, v = _qkv(B, nh, N, D, 1)
    nb = -(-N // blk)
    idx, cnt = _full_lists(B, nh, nb)
    o, lse = attention.block_sparse_attention(q, k, v, idx, cnt, blk)
    assert np.abs(o - attention.dense_attention(q, k, v)).max() < 1e-12
    s = np.einsum("bhid,bhjd->bhij", q, k) / math.sqrt(D)
    assert np.abs(lse - np.log(np.exp(s).sum(-1))).max() < 1e-12


def test_diagonal_mask_is_local_attention():
    B, nh, N, D, blk = 1, 1, 20, 4, 8
    q, k, v = _qkv(B, nh, N, D, 2)
    nb = -(-N // blk)
    idx = np.arange(nb, dtype=np.int32).reshape(1, 1, nb, 1)
    cnt = np.ones((1, 1, nb), dtype=np.int32)
    o, _ = attention.block_sparse_attention(q, k, v, idx, cnt, blk, 0.7)
    for I in range(nb):
        lo, hi = I * blk, min(N, I * blk + blk)
        ref = _loops_dense(q[0, 0, lo:hi], k[0, 0, lo:hi], v[0, 0, lo:hi], 0.7)
        assert np.abs(o[0, 0, lo:hi] - ref).max() < 1e-12


def test_constant_v_gives_constant_output():
    B, nh, N, D, blk = 1, 1, 30, 4, 8
    q, k, _ = _qkv(B, nh, N, D, 3)
    v = np.ones((B, nh, N, D)) * np.array([1.5, -2.0, 0.25, 7.0])
    s = np.random.default_rng(3).standard_normal((B, nh, 4, 4))
    idx, cnt = selection.select(s, "topk", k=2)
    o, _ = attention.block_sparse_attention(q, k, v, idx, cnt, blk)
    assert np.abs(o - v).max() < 1e-12


def test_empty_list_gives_zero():
    q, k, v = _qkv(1, 1, 16, 4, 4)
    idx = np.full((1, 1, 2, 2), -1, dtype=np.int32)
    cnt = np.array([[[0, 1]]], dtype=np.int32)
    idx[0, 0, 1, 0] = 0
    o, lse = attention.block_sparse_attention(q, k, v, idx, cnt, 8)
    assert (o[0, 0, :8] == 0).all() and np.isneginf(lse[0, 0, :8]).all()
    assert np.isfinite(o[0, 0, 8:]).all()


def test_pipeline_tiny_grid_full_keep_is_dense():
    # end to end: Hilbert reorder, scoring, top-k with k = nb, attention,
    # inverse reorder equals dense attention in the raster order
    T, H, W, nh, D = 2, 4, 4, 2, 8
    N = T * H * W
    r = np.random.default_rng(5)
    q, k, v = (r.standard_normal((1, N, nh, D)) for _ in range(3))
    res = pipeline.run(q, k, v, T=T, H=H, W=W, blk=8, sb=4, order="hilbert3d",
                       mode="topk", k_keep=4)
    dense = attention.dense_attention(*(np.transpose(x, (0, 2, 1, 3)) for x in (q, k, v)))
    assert np.abs(res["out"] - np.transpose(dense, (0, 2, 1, 3))).max() < 1e-12


def test_recall_closed_forms():
    from oracle import recall
    rng = np.random.default_rng(9)
    T, H, W, nh, D, blk = 2, 4, 4, 1, 4, 8
    N = T * H * W
    q = rng.standard_normal((1, N, nh, D))
    k = rng.standard_normal((1, N, nh, D))
    perm, _ = hilbert.make_perm("hilbert3d", T, H, W)
    nb = N // blk
    full = np.tile(np.arange(nb, dtype=np.int32), (1, 1, nb, 1))
    cnt = np.full((1, 1, nb), nb, dtype=np.int32)
    qs = [(0, 0, n) for n in range(N)]
    assert abs(recall.recall(q, k, perm, full, cnt, blk, qs) - 1.0) < 1e-12     # everything kept
    none = np.zeros((1, 1, nb), dtype=np.int32)
    assert recall.recall(q, k, perm, full, none, blk, qs) == 0.0               # nothing kept
    # one block kept: the mass of that block's keys, by brute force
    one = np.zeros((1, 1, nb, 1), dtype=np.int32)
    ones = np.ones((1, 1, nb), dtype=np.int32)
    n = 5
    s = [sum(q[0, n, 0, d] * k[0, m, 0, d] for d in range(D)) / 2.0 for m in range(N)]
    e = np.exp(np.array(s) - max(s))
    ref = e[perm[:blk]].sum() / e.sum()
    assert abs(recall.recall(q, k, perm, one, ones, blk, [(0, 0, n)]) - ref) < 1e-12


def _loss(q, k, v, do, idx, cnt, blk, scale):
    o, _ = attention.block_sparse_attention(q, k, v, idx, cnt, blk, scale)
    return float((o * do).sum())


def test_backward_matches_finite_differences():
    # L = sum(dO * O); central differences of the forward oracle, element by element
    B, nh, N, D, blk, scale = 1, 1, 19, 3, 8, 0.7
    rng = np.random.default_rng(11)
    q, k, v, do = (rng.standard_normal((B, nh, N, D)) for _ in range(4))
    idx = np.array([[[[0, 2], [1, -1], [0, 1]]]], dtype=np.int32)   # block 2 is ragged (3 keys)
    cnt = np.array([[[2, 1, 2]]], dtype=np.int32)
    dq, dk, dv = attention.block_sparse_attention_bwd(q, k, v, do, idx, cnt, blk, scale)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for pos in np.ndindex(x.shape):
            old = x[pos]
            x[pos] = old + h
            lp = _loss(q, k, v, do, idx, cnt, blk, scale)
            x[pos] = old - h
            lm = _loss(q, k, v, do, idx, cnt, blk, scale)
            x[pos] = old
            assert abs((lp - lm) / (2 * h) - g[pos]) < 1e-7, (name, pos)


def test_backward_full_mask_matches_autograd():
    import torch
    B, nh, N, D, blk = 1, 2, 21, 4, 8
    q, k, v, do = _qkv(B, nh, N, D, 12) + [np.random.default_rng(13).standard_normal((B, nh, N, D))]
    nb = -(-N // blk)
    idx, cnt = _full_lists(B, nh, nb)
    dq, dk, dv = attention.block_sparse_attention_bwd(q, k, v, do, idx, cnt, blk)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = torch.softmax(tq @ tk.transpose(-1, -2) / math.sqrt(D), dim=-1) @ tv
    o.backward(torch.tensor(do))
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(mine - ref.numpy()).max() < 1e-12


def test_backward_empty_row_contributes_nothing():
    q, k, v, do = _qkv(1, 1, 16, 4, 14) + [np.ones((1, 1, 16, 4))]
    idx = np.array([[[[0], [0]]]], dtype=np.int32)
    cnt = np.array([[[0, 1]]], dtype=np.int32)
    dq, dk, dv = attention.block_sparse_attention_bwd(q, k, v, do, idx, cnt, 8)
    assert (dq[0, 0, :8] == 0).all()
    # only query block 1 reaches key block 0; key block 1 is never kept
    assert (dk[0, 0, 8:] == 0).all() and (dv[0, 0, 8:] == 0).all()
    ref_q, ref_k, ref_v = attention.block_sparse_attention_bwd(q, k, v, do, idx, cnt, 8, rows=[(0, 0, 1)])
    assert np.array_equal(dk, ref_k) and np.array_equal(dv, ref_v)


def test_parallel_rows_equal_the_serial_call():
    """oracle.parallel only deals query blocks out to worker processes: every
    row it returns is bitwise the serial oracle's, with and without the
    frame rule."""
    from oracle import lvsa, parallel
    rng = np.random.default_rng(5)
    B, nh, N, D, blk = 1, 2, 700, 16, 64
    nb = -(-N // blk)
    q, k, v = (rng.standard_normal((B, nh, N, D)) for _ in range(3))
    idx = np.full((B, nh, nb, 5), -1, np.int32)
    cnt = rng.integers(0, 6, size=(B, nh, nb)).astype(np.int32)
    for h in range(nh):
        for I in range(nb):
            idx[0, h, I, :cnt[0, h, I]] = np.sort(rng.choice(nb, cnt[0, h, I], replace=False))
    rows = [(0, h, I) for h in range(nh) for I in range(nb)]
    P = 100
    fa = lvsa.frame_allowed(7, 3, 4, 1)
    for frame in (None, (fa, P)):
        allowed = None if frame is None else (lambda qs, ks: fa[np.asarray(qs)[:, None] // P,
                                                               np.asarray(ks)[None, :] // P])
        ref_o, ref_l = attention.block_sparse_attention(q, k, v, idx, cnt, blk, allowed=allowed)
        got = parallel.block_sparse_attention_rows(q, k, v, idx, cnt, blk, rows, frame=frame, workers=3)
        assert sorted(got) == sorted(rows)
        for (b, h, I), (o, l) in got.items():
            lo, hi = I * blk, min(N, I * blk + blk)
            assert np.array_equal(o, ref_o[b, h, lo:hi], equal_nan=True)
            assert np.array_equal(l, ref_l[b, h, lo:hi])
