"""Pins of the oracle's log-radial static mask.

Page: DynamicRad (methodology, components 1 and 2): the retained share of a
frame pair depends only on the temporal distance and shrinks exponentially
with it (distance bands that double in length), with a long-range factor
lambda flooring the window of far frames.
"""
import numpy as np
import pytest

from oracle import radial


def test_bands_double_in_length():
    # band r >= 1 covers exactly the 2^(r-1) distances [2^(r-1), 2^r)
    counts = {}
    for d in range(1, 1 << 10):
        counts[radial.band(d)] = counts.get(radial.band(d), 0) + 1
    assert counts == {r: 1 << (r - 1) for r in range(1, 11)}
    assert radial.band(0) == 0


def test_window_halves_per_band_until_the_floor():
    w0, w_far = 640, 40
    prev = None
    for d in range(0, 200):
        w = radial.window(d, w0, w_far)
        if d in (0,):
            assert w == w0
        if prev is not None and radial.band(d) != radial.band(d - 1):
            assert w == max(prev // 2, w_far)
        prev = w
    assert radial.window(1000, w0, w_far) == w_far
    assert radial.window(1000, w0, 0) == 0


def _brute_block_mask(T, P, blk, w0, w_far):
    """Scalar loops over every token pair."""
    N = T * P
    nb = -(-N // blk)
    m = np.zeros((nb, nb), dtype=bool)
    for q in range(N):
        for k in range(N):
            d = abs(q // P - k // P)
            om = w0
            r = 0
            while (d >> r) > 0:       # r = bit length of d
                r += 1
            om = max(w0 // (2 ** r), w_far)
            if 2 * abs(q % P - k % P) < om:
                m[q // blk, k // blk] = True
    return m


@pytest.mark.parametrize("T,P,blk,w0,w_far", [(6, 10, 8, 12, 2), (9, 7, 16, 20, 0), (5, 24, 16, 48, 3),
                                              (4, 5, 4, 3, 1)])
def test_block_mask_brute_force(T, P, blk, w0, w_far):
    assert np.array_equal(radial.block_mask(T, P, blk, w0, w_far), _brute_block_mask(T, P, blk, w0, w_far))


def test_rows_argument_matches_full_mask():
    full = radial.block_mask(7, 30, 16, 40, 4)
    rows = [0, 3, full.shape[0] - 1]
    assert np.array_equal(radial.block_mask(7, 30, 16, 40, 4, rows=rows), full[rows])


def test_special_cases():
    T, P, blk = 5, 16, 16                      # one block per frame
    # a window of 2P everywhere keeps every pair: dense
    assert radial.block_mask(T, P, blk, 2 * P, 2 * P).all()
    # w0 = 1, no floor: only d = 0 with equal spatial index -> block diagonal
    assert np.array_equal(radial.block_mask(T, P, blk, 1, 0), np.eye(T, dtype=bool))
    # w0 = 2: d = 0 keeps the same index, d = 1 gets window 1 (same index), d >= 2 nothing
    m = radial.block_mask(T, P, blk, 2, 0)
    ref = np.abs(np.arange(T)[:, None] - np.arange(T)[None, :]) <= 1
    assert np.array_equal(m, ref)


def test_symmetric_and_monotone():
    T, P, blk = 8, 40, 32
    for w0, w_far in [(80, 0), (50, 6), (33, 33)]:
        m = radial.block_mask(T, P, blk, w0, w_far)
        assert np.array_equal(m, m.T)          # same partition, symmetric rule
    a = radial.block_mask(T, P, blk, 60, 0)
    b = radial.block_mask(T, P, blk, 60, 10)
    c = radial.block_mask(T, P, blk, 120, 10)
    assert (a <= b).all() and (b <= c).all()


def test_lambda_floor_rounding():
    # lambda goes through fp32: 0.1f * 1000 = 100.0000014.. -> 100
    assert radial.w_far_of(0.1, 1000) == 100
    assert radial.w_far_of(0.0625, 3120) == 195
    assert radial.w_far_of(0.0, 3120) == 0
