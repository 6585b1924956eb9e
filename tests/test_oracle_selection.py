"""Pins of the oracle's top-k and threshold selection.

Pages: DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 3 (sparsity budget per query block); VMoBA:
Mixture of Block Attention for Video Diffusion Models, abstract,
modification (3) (the number of blocks follows their cumulative similarity).
"""
import itertools
import math

import numpy as np
import pytest

from oracle import selection


def _beats(row, a, b):
    """a outranks b: larger score, or equal score and lower index."""
    return row[a] > row[b] or (row[a] == row[b] and a < b)


def test_topk_matches_rank_count_brute_force():
    rng = np.random.default_rng(0)
    for trial in range(300):
        n = int(rng.integers(1, 12))
        row = rng.integers(-3, 4, size=n).astype(np.float32)   # many ties
        k = int(rng.integers(0, n + 1))
        got = selection.topk_row(row, k)
        ref = [j for j in range(n) if sum(_beats(row, i, j) for i in range(n) if i != j) < k]
        assert list(got) == ref


def test_topk_full_and_equal_rows():
    row = np.zeros(9, dtype=np.float32)
    assert list(selection.topk_row(row, 4)) == [0, 1, 2, 3]
    row = np.random.default_rng(1).standard_normal(9).astype(np.float32)
    assert list(selection.topk_row(row, 9)) == list(range(9))


def _softmax(row):
    m = max(row)
    e = [math.exp(float(x) - m) for x in row]
    z = sum(e)
    return [x / z for x in e]


def test_threshold_count_is_minimal_subset_size():
    # brute force over all subsets: the smallest set whose mass reaches tau
    rng = np.random.default_rng(2)
    for trial in range(200):
        n = int(rng.integers(1, 9))
        row = (rng.standard_normal(n) * 2).astype(np.float32)
        tau = float(rng.uniform(0.05, 0.999))
        p = _softmax(row)
        best = n
        for r in range(1, n + 1):
            if any(sum(p[j] for j in S) >= tau for S in itertools.combinations(range(n), r)):
                best = r
                break
        m, _ = selection.threshold_count(row, tau, cap=n)
        assert m == best
        kept = selection.threshold_row(row, tau, cap=n)
        # the kept set is the m best-ranked blocks
        order = sorted(range(n), key=lambda j: (-float(row[j]), j))
        assert list(kept) == sorted(order[:m])


def test_threshold_cap_and_full():
    row = np.zeros(10, dtype=np.float32)           # uniform mass 0.1 each
    assert list(selection.threshold_row(row, 0.85, cap=10)) == list(range(9))
    assert list(selection.threshold_row(row, 0.85, cap=4)) == [0, 1, 2, 3]
    row = np.random.default_rng(3).standard_normal(10).astype(np.float32)
    assert list(selection.threshold_row(row, 1.0 + 1e-9, cap=10)) == list(range(10))
    row = np.array([0, 30, 0, 0], dtype=np.float32)  # one block holds ~all mass
    assert list(selection.threshold_row(row, 0.9, cap=4)) == [1]


def test_ratio_counts():
    # keep 25 % of 32 blocks, 15 % of 256, cap 20 % of 929
    assert selection.ratio_count(25, 100, 32) == 8
    assert selection.ratio_count(15, 100, 256) == math.ceil(0.15 * 256) == 39
    assert selection.ratio_count(20, 100, 929) == math.ceil(0.2 * 929) == 186


def test_select_lists_and_mask_roundtrip():
    s = np.random.default_rng(4).standard_normal((1, 2, 5, 7))
    idx, cnt = selection.select(s, "topk", k=3, kcap=4)
    assert (cnt == 3).all() and (idx[..., 3] == -1).all()
    m = selection.lists_to_mask(idx, cnt, 7)
    assert (m.sum(-1) == 3).all()
    idx2, cnt2 = selection.mask_to_lists(m, 4)
    assert np.array_equal(idx, idx2) and np.array_equal(cnt, cnt2)


def test_global_selection_rank_count_brute_force():
    # pair (I, J) kept iff fewer than K pairs outrank it (higher score, or
    # equal score and lower flat index)
    rng = np.random.default_rng(7)
    for trial in range(60):
        nb = int(rng.integers(1, 7))
        s = rng.integers(-2, 3, size=(nb, nb)).astype(np.float32)
        K = int(rng.integers(0, nb * nb + 1))
        m = selection.global_topk_head(s, K)
        flat = s.reshape(-1)
        for f in range(nb * nb):
            better = sum(1 for g in range(nb * nb) if flat[g] > flat[f] or (flat[g] == flat[f] and g < f))
            assert m.reshape(-1)[f] == (better < K)
        assert m.sum() == K


def test_global_selection_lists():
    s = np.zeros((1, 1, 3, 3), dtype=np.float32)
    s[0, 0, 2, 0] = 5.0
    s[0, 0, 0, 2] = 4.0
    idx, cnt = selection.select_global(s, 3)
    # best two pairs, then the lowest flat index among the zero ties: (0, 0)
    assert list(cnt[0, 0]) == [2, 0, 1]
    assert list(idx[0, 0, 0, :2]) == [0, 2] and idx[0, 0, 2, 0] == 0
