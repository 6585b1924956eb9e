"""Pins of the oracle's pooling and hierarchical block score.

Page: DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 2 (sub-block scores aggregated into block
importance; coarse block pooling is the special case it refines).
"""
import math

import numpy as np
import pytest

from oracle import scoring, selection


def _rand(shape, seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


def test_pool_sb1_is_identity():
    x = _rand((1, 2, 37, 8))
    assert np.array_equal(scoring.pool_subblocks(x, 1), x)


def test_pool_closed_forms():
    # constant rows pool to the constant; a linear ramp pools to its midpoint
    N, D = 50, 4
    ramp = np.arange(N, dtype=np.float64)[None, None, :, None] * np.ones((1, 1, 1, D))
    p = scoring.pool_subblocks(ramp, 16)
    assert p.shape == (1, 1, 4, D)
    assert np.allclose(p[0, 0, :, 0], [7.5, 23.5, 39.5, 48.5])   # last sub-block: tokens 48, 49
    c = np.full((1, 1, N, D), 3.25)
    assert np.allclose(scoring.pool_subblocks(c, 7), 3.25)


def test_sb_equal_blk_is_block_mean_pooling():
    # brute force: mean of each block's tokens, dot product, scale
    B, nh, N, D, blk = 1, 2, 45, 6, 8
    q, k = _rand((B, nh, N, D), 1), _rand((B, nh, N, D), 2)
    scale = 0.3
    got = scoring.block_scores(q, k, blk, blk, scale)
    nb = -(-N // blk)
    for h in range(nh):
        for I in range(nb):
            qm = [sum(q[0, h, n, d] for n in range(I * blk, min(N, I * blk + blk))) /
                  (min(N, I * blk + blk) - I * blk) for d in range(D)]
            for J in range(nb):
                kk = range(J * blk, min(N, J * blk + blk))
                km = [sum(k[0, h, n, d] for n in kk) / len(kk) for d in range(D)]
                ref = sum(a * b for a, b in zip(qm, km)) * scale
                assert abs(got[0, h, I, J] - ref) < 1e-12


def test_sb1_is_max_token_pair_logit():
    B, nh, N, D, blk = 1, 1, 21, 5, 4
    q, k = _rand((B, nh, N, D), 3), _rand((B, nh, N, D), 4)
    got = scoring.block_scores(q, k, blk, 1, 1.0 / math.sqrt(D))
    nb = -(-N // blk)
    for I in range(nb):
        for J in range(nb):
            best = -math.inf
            for i in range(I * blk, min(N, I * blk + blk)):
                for j in range(J * blk, min(N, J * blk + blk)):
                    best = max(best, sum(q[0, 0, i, d] * k[0, 0, j, d] for d in range(D)) / math.sqrt(D))
            assert abs(got[0, 0, I, J] - best) < 1e-12


def test_hierarchical_by_hand():
    # D = 1, blk = 4, sb = 2, N = 8: sub-block means and the max are checked by hand.
    q = np.array([1, 3, -2, 0, 5, 5, 1, -1], dtype=np.float64).reshape(1, 1, 8, 1)
    k = np.array([2, 2, -4, 0, 1, 0, 3, 3], dtype=np.float64).reshape(1, 1, 8, 1)
    # qbar = [2, -1, 5, 0]; kbar = [2, -2, 0.5, 3]
    # block (0,0): max(2*2, 2*-2, -1*2, -1*-2) = 4
    # block (0,1): max(2*.5, 2*3, -1*.5, -1*3) = 6
    # block (1,0): max(5*2, 5*-2, 0, 0) = 10
    # block (1,1): max(2.5, 15, 0, 0) = 15
    got = scoring.block_scores(q, k, 4, 2, 1.0)
    assert np.allclose(got[0, 0], [[4, 6], [10, 15]])


def test_scale_only_rescales_topk():
    q, k = _rand((1, 2, 64, 8), 5), _rand((1, 2, 64, 8), 6)
    a = scoring.block_scores(q, k, 8, 2, 1.0)
    b = scoring.block_scores(q, k, 8, 2, 0.125)
    assert np.allclose(a * 0.125, b)
    ia, ca = selection.select(a, "topk", k=3)
    ib, cb = selection.select(b, "topk", k=3)
    assert np.array_equal(ia, ib) and np.array_equal(ca, cb)


def test_ragged_tail_subblocks_absent():
    # N = 10, blk = 4, sb = 2: the last block holds one sub-block (tokens 8, 9)
    q, k = _rand((1, 1, 10, 3), 7), _rand((1, 1, 10, 3), 8)
    got = scoring.block_scores(q, k, 4, 2, 1.0)
    qb = np.array([q[0, 0, 8:10].mean(0)])
    kb = [k[0, 0, 0:2].mean(0), k[0, 0, 2:4].mean(0)]
    assert abs(got[0, 0, 2, 0] - max(float(qb[0] @ kb[0]), float(qb[0] @ kb[1]))) < 1e-12
