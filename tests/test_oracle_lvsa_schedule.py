"""Pins of the oracle's LVSA frame mask and the adaptive budget schedule.

Pages: LVSA: Training-Free Sparse Attention for Long Video Diffusion,
section 2 (rotating anchors, every frame an anchor exactly once per T_per
steps; expanded windows keep |A(t)| at the budget C); DFSAttn: Dynamic
Fine-grained Sparse Attention for Efficient Video Generation, Methodology
item 3 (budget decreasing monotonically over steps, masks refreshed at a
fixed interval).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import lvsa, schedule


@pytest.mark.parametrize("T,T_per", [(63, 8), (21, 4), (10, 3)])
def test_each_frame_is_anchor_once_per_period(T, T_per):
    seen = []
    for s in range(5, 5 + T_per):           # any T_per consecutive steps
        seen += lvsa.anchors(T, T_per, s)
    assert sorted(seen) == list(range(T))


def test_anchor_counts_at_63_frames():
    assert [len(lvsa.anchors(63, 8, s)) for s in range(8)] == [8, 8, 8, 8, 8, 8, 8, 7]


@pytest.mark.parametrize("s", range(8))
def test_frame_set_has_exactly_budget(s):
    T, T_per, C = 63, 8, 21
    G = set(lvsa.anchors(T, T_per, s))
    for t in range(T):
        A = lvsa.frame_set(T, t, T_per, C, s)
        assert len(A) == C
        assert G <= set(A)
        assert t in A
        # the window part is the set of non-anchors closest to t
        W = sorted(set(A) - G, key=lambda f: abs(f - t))
        others = [f for f in range(T) if f not in A and f not in G]
        if others:
            assert max(abs(f - t) for f in W) <= min(abs(f - t) for f in others)


def test_window_tie_prefers_earlier_frame():
    # T = 10, no anchor near t = 5 (T_per = 10, s = 0 -> anchor 0 only),
    # C = 4: window needs 3 frames: 5, then 4 before 6
    assert lvsa.window(10, 5, [0], 4) == [5, 4, 6]


def test_block_mask_brute_force_toy():
    # token-level pairs on a 6-frame toy (P = 2 x 3 tokens), blocks of 4
    T, P, blk = 6, 6, 4
    N = T * P
    for s in range(3):
        m = lvsa.block_mask(T, P, blk, 3, 4, s)
        nb = -(-N // blk)
        A = [set(lvsa.frame_set(T, t, 3, 4, s)) for t in range(T)]
        ref = np.zeros((nb, nb), dtype=bool)
        for qi in range(N):
            for ki in range(N):
                if ki // P in A[qi // P]:
                    ref[qi // blk, ki // blk] = True
        assert np.array_equal(m, ref)


def test_lvsa_workload_density():
    # 63 x (30 x 52) tokens, blocks of 128: about a third of the blocks kept
    m = lvsa.block_mask(63, 30 * 52, 128, 8, 21, 0)
    assert m.shape == (768, 768)
    frac = m.sum() / m.size
    assert 21 / 63 <= frac < 0.36


def test_schedule_closed_form():
    nb = 256
    ks = [schedule.budget(s, nb) for s in range(50)]
    # exact: ceil(nb * (0.40 + (0.10 - 0.40) * r / 49)) with r the last refresh step
    for s in range(50):
        r = s - s % 5
        ratio = Fraction(40, 100) + (Fraction(10, 100) - Fraction(40, 100)) * Fraction(r, 49)
        assert ks[s] == math.ceil(ratio * nb)
    assert [ks[s] for s in range(0, 50, 5)] == [103, 95, 87, 79, 72, 64, 56, 48, 40, 32]
    assert all(a >= b for a, b in zip(ks, ks[1:]))
    # the budget only changes at refresh steps
    for s in range(1, 50):
        if ks[s] != ks[s - 1]:
            assert schedule.is_refresh(s)


def test_frame_exact_attention_toy():
    # token-level brute force on a 5-frame toy (P = 6, blk 4): frame-exact
    # attention equals dense attention restricted to A(t) frame by frame
    from oracle import attention, selection
    T, P, blk, T_per, C, s = 5, 6, 4, 3, 3, 1
    N = T * P
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, 1, N, 4)) for _ in range(3))
    m = lvsa.block_mask(T, P, blk, T_per, C, s)
    idx, cnt = selection.mask_to_lists(m[None, None])
    fa = lvsa.frame_allowed(T, T_per, C, s)
    allowed = lambda qs, ks: fa[np.asarray(qs)[:, None] // P, np.asarray(ks)[None, :] // P]
    got, _ = attention.block_sparse_attention(q, k, v, idx, cnt, blk, 0.5, allowed=allowed)
    for n in range(N):
        keys = [j for j in range(N) if fa[n // P, j // P]]
        lg = np.array([0.5 * float(q[0, 0, n] @ k[0, 0, j]) for j in keys])
        e = np.exp(lg - lg.max())
        ref = (e[:, None] * v[0, 0, keys]).sum(0) / e.sum()
        assert np.abs(got[0, 0, n] - ref).max() < 1e-12
