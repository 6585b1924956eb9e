"""GPU Hilbert index, gather and scatter against the oracle: bit-exact.

Page: DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 1."""
import numpy as np
import pytest
import torch

from oracle import hilbert

pytestmark = pytest.mark.gpu

GRIDS = [(1, 1, 1), (1, 1, 100), (5, 1, 9), (2, 3, 5), (3, 7, 11), (4, 4, 4), (8, 16, 16), (16, 16, 16),
         (6, 10, 3), (21, 30, 52), (63, 30, 52), (33, 45, 80)]


@pytest.fixture(scope="module")
def lib(cuda_device):
    from block_sparse_attention_36_b200 import dfsattn
    return dfsattn


def _index(lib, T, H, W, order):
    N = T * H * W
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty(N, dtype=torch.int32, device="cuda")
    s = lib.Shape(1, 1, 64, T, H, W, 64, 16)
    lib.dfs_hilbert_perm(s, order, perm, inv, 1, None, None, None, None, None, None)
    torch.cuda.synchronize()
    return perm.cpu().numpy(), inv.cpu().numpy()


@pytest.mark.parametrize("grid", GRIDS)
def test_hilbert_index_matches_oracle(lib, grid):
    perm, inv = _index(lib, *grid, "hilbert3d")
    operm, oinv = hilbert.hilbert_perm(*grid)
    assert np.array_equal(perm, operm)
    assert np.array_equal(inv, oinv)


def test_small_grids_exhaustive(lib):
    for T in range(1, 7):
        for H in range(1, 7):
            for W in range(1, 7):
                perm, inv = _index(lib, T, H, W, "hilbert3d")
                operm, oinv = hilbert.hilbert_perm(T, H, W)
                assert np.array_equal(perm, operm), (T, H, W)
                assert np.array_equal(inv, oinv), (T, H, W)


def test_raster_is_identity(lib):
    perm, inv = _index(lib, 5, 6, 7, "raster")
    assert np.array_equal(perm, np.arange(210)) and np.array_equal(inv, np.arange(210))


@pytest.mark.parametrize("B,nh,D,grid", [(1, 2, 64, (8, 16, 16)), (2, 3, 128, (3, 7, 11)),
                                         (1, 12, 128, (21, 30, 52)), (1, 1, 64, (1, 1, 37))])
def test_gather_and_scatter_bit_exact(lib, B, nh, D, grid):
    T, H, W = grid
    N = T * H * W
    g = torch.Generator().manual_seed(N + nh)
    x = [torch.randn((B, N, nh, D), generator=g).to(torch.bfloat16) for _ in range(3)]
    xd = [t.cuda() for t in x]
    s = lib.Shape(B, nh, D, T, H, W, 64, 16)
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    xp = [torch.empty((B, nh, N, D), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    lib.dfs_hilbert_perm(s, "hilbert3d", perm, inv, 1, *xd, *xp)
    back = torch.empty_like(xd[0])
    lib.dfs_unperm(s, perm, xp[1], back)
    torch.cuda.synchronize()
    operm, _ = hilbert.hilbert_perm(T, H, W)
    for t in range(3):
        ref = hilbert.permute_tokens(x[t].view(torch.int16).numpy(), operm)
        assert np.array_equal(xp[t].cpu().view(torch.int16).numpy(), ref)
    assert torch.equal(back.cpu().view(torch.int16), x[1].view(torch.int16))
    ref_back = hilbert.unpermute_tokens(xp[2].cpu().view(torch.int16).numpy(), operm)
    assert np.array_equal(ref_back, x[2].view(torch.int16).numpy())


def test_partial_tensors(lib):
    # only K is reordered; Q and V outputs untouched
    T, H, W, nh, D = 2, 3, 4, 2, 64
    N = T * H * W
    s = lib.Shape(1, nh, D, T, H, W, 64, 16)
    k = torch.randn((1, N, nh, D)).to(torch.bfloat16).cuda()
    kp = torch.empty((1, nh, N, D), dtype=torch.bfloat16, device="cuda")
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    lib.dfs_hilbert_perm(s, "hilbert3d", perm, inv, 1, None, k, None, None, kp, None)
    torch.cuda.synchronize()
    operm, _ = hilbert.hilbert_perm(T, H, W)
    assert np.array_equal(kp.cpu().view(torch.int16).numpy(),
                          hilbert.permute_tokens(k.cpu().view(torch.int16).numpy(), operm))


@pytest.mark.parametrize("order", ["tile2d", "tile3d", "hilbert2d"])
@pytest.mark.parametrize("grid,blk", [((8, 16, 16), 64), ((21, 30, 52), 128), ((3, 5, 7), 64), ((63, 30, 52), 128),
                                      ((33, 45, 80), 128), ((1, 1, 100), 128), ((5, 17, 9), 128)])
def test_tiled_and_2d_orders_match_oracle(lib, order, grid, blk):
    """Tiled orders and the frame-major 2-D Hilbert order: the index kernel's
    perm and inv bit-exact against the oracle's enumeration."""
    T, H, W = grid
    N = T * H * W
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty(N, dtype=torch.int32, device="cuda")
    s = lib.Shape(1, 1, 64, T, H, W, blk, 16)
    lib.dfs_hilbert_perm(s, order, perm, inv, 1, None, None, None, None, None, None)
    torch.cuda.synchronize()
    operm, oinv = hilbert.make_perm(order, T, H, W, blk)
    assert np.array_equal(perm.cpu().numpy(), operm)
    assert np.array_equal(inv.cpu().numpy(), oinv)
