"""GPU key-block selection against the oracle.

Pages: DFSAttn, Methodology item 3 (top-k budget); VMoBA abstract,
modifications (2) (global selection) and (3) (cumulative-mass threshold);
LVSA section 2 (frame mask); DynamicRad methodology (log-radial static
mask). Given the same fp32 scores, top-k and global lists are bit-exact
(ties included); a threshold row may differ only where the oracle's
cumulative mass at the cut lies within 1e-5 of tau (counted); LVSA and
log-radial lists are bit-exact."""
import numpy as np
import pytest
import torch

from oracle import lvsa, radial, selection
from tests.parity import compare_masks

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib(cuda_device):
    from block_sparse_attention_36_b200 import dfsattn
    return dfsattn


def _select(lib, scores, shape, params, kcap):
    B, nh, nb = shape.B, shape.nh, shape.nb
    idx = torch.full((B, nh, nb, kcap), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, nh, nb), -7, dtype=torch.int32, device="cuda")
    sc = None if scores is None else torch.from_numpy(np.ascontiguousarray(scores, dtype=np.float32)).cuda()
    lib.dfs_select_mask(shape, sc, params, idx, cnt, kcap)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy()


def _shape_for(lib, nb, nh=2, B=1):
    # N chosen so that nb = ceil(N / 128)
    return lib.Shape(B, nh, 128, 1, 1, nb * 128 - 5, 128, 32)


def _lists_equal(gi, gc, oi, oc):
    gi, oi = gi.reshape(-1, gi.shape[-1]), oi.reshape(-1, oi.shape[-1])
    gc, oc = gc.reshape(-1), oc.reshape(-1)
    assert np.array_equal(gc, oc)
    for r in range(len(gc)):
        assert np.array_equal(gi[r, :gc[r]], oi[r, :oc[r]]), r


@pytest.mark.parametrize("nb,k", [(32, 8), (256, 39), (929, 186), (1, 1), (33, 0), (40, 40), (70, 100),
                                  (1500, 300), (2048, 7)])
def test_topk_bit_exact(lib, nb, k):
    rng = np.random.default_rng(nb + k)
    s = (rng.standard_normal((1, 2, nb, nb)) * 3).astype(np.float32)
    s[0, 0, : nb // 2] = np.round(s[0, 0, : nb // 2])     # many exact ties
    s[0, 1, 0] = 0.0                                      # an all-equal row
    shape = _shape_for(lib, nb)
    kcap = max(1, min(k, nb))
    gi, gc = _select(lib, s, shape, lib.select_params("topk", k=k), kcap)
    oi, oc = selection.select(s, "topk", k=k, kcap=kcap)
    _lists_equal(gi, gc, oi, oc)


def test_topk_negative_zero_ties(lib):
    s = np.zeros((1, 1, 40, 40), dtype=np.float32)
    s[..., ::3] = -0.0
    shape = _shape_for(lib, 40, nh=1)
    gi, gc = _select(lib, s, shape, lib.select_params("topk", k=5), 5)
    assert (gc == 5).all() and (gi[..., :5] == np.arange(5)).all()


@pytest.mark.parametrize("nb,tau,cap", [(929, 0.9, 186), (256, 0.5, 256), (64, 0.99, 10), (100, 0.0, 50),
                                        (100, 1.5, 100), (300, 0.9, 0)])
def test_threshold_matches_with_excusal(lib, nb, tau, cap):
    rng = np.random.default_rng(nb)
    s = (rng.standard_normal((1, 2, nb, nb)) * rng.uniform(0.5, 4, size=(1, 2, nb, 1))).astype(np.float32)
    s[0, 1, :5] = 1.0                                     # uniform rows
    shape = _shape_for(lib, nb)
    kcap = max(1, min(cap, nb))
    gi, gc = _select(lib, s, shape, lib.select_params("threshold", cap=cap, tau=tau), kcap)
    oi, oc = selection.select(s, "threshold", tau=tau, cap=cap, kcap=kcap)
    res = compare_masks(gi, gc, oi, oc, s.astype(np.float64), "threshold", tau=tau, cap=cap)
    assert res["bad_rows"] == 0, res
    assert res["excused_rows"] <= max(2, res["rows"] // 200), res


@pytest.mark.parametrize("T,H,W,blk,T_per,C", [(63, 30, 52, 128, 8, 21), (21, 30, 52, 128, 4, 9),
                                               (6, 2, 3, 64, 3, 4), (10, 4, 4, 64, 10, 30), (9, 8, 8, 128, 2, 5)])
def test_lvsa_bit_exact(lib, T, H, W, blk, T_per, C):
    nh = 2
    shape = lib.Shape(1, nh, 128, T, H, W, blk, 32)
    for s in range(T_per):
        kcap = shape.nb
        gi, gc = _select(lib, None, shape, lib.select_params("lvsa", lvsa_T_per=T_per, lvsa_C=C, lvsa_step=s), kcap)
        m = lvsa.block_mask(T, H * W, blk, T_per, C, s)
        oi, oc = selection.mask_to_lists(np.broadcast_to(m, (1, nh) + m.shape), kcap)
        _lists_equal(gi, gc, oi, oc)


@pytest.mark.parametrize("T,H,W,blk,w0,lam", [
    (6, 4, 5, 64, 12, 0.2),        # frames smaller than a block (P = 20 < 64)
    (9, 7, 1, 64, 20, 0.0),        # P = 7, many frames per block
    (5, 8, 9, 64, 144, 0.0625),    # P = 72, window of a whole frame at d = 0
    (8, 5, 8, 64, 40, 0.15),       # P = 40 < blk = 64
    (11, 16, 12, 128, 192, 0.125), # P = 1.5 blk
    (7, 10, 13, 128, 1, 0.0),      # w0 = 1: only equal positions in the same frame
    (5, 12, 12, 64, 288, 1.0),     # window 2P everywhere: dense
])
def test_radial_bit_exact(lib, T, H, W, blk, w0, lam):
    nh = 2
    shape = lib.Shape(1, nh, 128, T, H, W, blk, 32)
    kcap = shape.nb
    gi, gc = _select(lib, None, shape, lib.select_params("radial", radial_w0=w0, radial_lambda=lam), kcap)
    m = radial.block_mask(T, H * W, blk, w0, radial.w_far_of(lam, w0))
    oi, oc = selection.mask_to_lists(np.broadcast_to(m, (1, nh) + m.shape), kcap)
    _lists_equal(gi, gc, oi, oc)


def test_radial_wan_grid_sampled_rows(lib):
    T, H, W, blk, w0, lam = 21, 30, 52, 128, 1560, 0.125
    shape = lib.Shape(1, 1, 128, T, H, W, blk, 32)
    gi, gc = _select(lib, None, shape, lib.select_params("radial", radial_w0=w0, radial_lambda=lam), shape.nb)
    rows = [0, 1, 12, 13, 100, 127, 128, 200, 254, 255]
    m = radial.block_mask(T, H * W, blk, w0, radial.w_far_of(lam, w0), rows=rows)
    for r, I in enumerate(rows):
        assert np.array_equal(gi[0, 0, I, :gc[0, 0, I]], np.flatnonzero(m[r])), I


def test_kcap_overflow_is_flagged(lib):
    shape = lib.Shape(1, 1, 128, 63, 30, 52, 128, 32)
    lib.dfs_get_error_flags(clear=True)
    gi, gc = _select(lib, None, shape, lib.select_params("lvsa", lvsa_T_per=8, lvsa_C=21, lvsa_step=0), 16)
    assert (gc <= 16).all()
    assert lib.dfs_get_error_flags(clear=True) & lib.DFS_FLAG_KCAP_OVERFLOW


@pytest.mark.parametrize("nb,K", [(32, 100), (256, 9831), (57, 1), (40, 1600), (40, 0), (300, 4500), (929, 172609)])
def test_global_selection_bit_exact(lib, nb, K):
    rng = np.random.default_rng(nb + K)
    s = (rng.standard_normal((1, 2, nb, nb)) * 2).astype(np.float32)
    s[0, 1] = np.round(s[0, 1])                           # heavy ties across the head
    shape = _shape_for(lib, nb)
    kcap = nb
    gi, gc = _select(lib, s, shape, lib.select_params("global", k=K), kcap)
    oi, oc = selection.select_global(s, K, kcap=kcap)
    _lists_equal(gi, gc, oi, oc)
    assert gc.reshape(2, -1).sum(axis=1).tolist() == [min(K, nb * nb)] * 2
