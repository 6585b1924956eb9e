"""GPU pooling and hierarchical block scores against the fp64 oracle.

Page: DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 2. The means are fp32 sums of <= sb bf16
values; the dot products run on the tensor cores as three tf32 products of
split operands (x = x_hi + x_lo, both tf32-rounded), each term within
3 * 2^-22 = 12 u of |a||b| (u = 2^-24), accumulated in fp32 over
3 * D / 8 MMA steps. Both fit the bound used here, (D + 2 sb + 4) u times
the magnitudes summed: 12 + 3 D / 8 <= D for D >= 64."""
import math

import numpy as np
import pytest
import torch

from oracle import scoring

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


@pytest.fixture(scope="module")
def lib(cuda_device):
    from block_sparse_attention_36_b200 import dfsattn
    return dfsattn


def _run(lib, B, nh, D, N, blk, sb, seed=0, scale=0.0):
    g = torch.Generator().manual_seed(seed)
    qp = torch.randn((B, nh, N, D), generator=g).to(torch.bfloat16)
    kp = (torch.randn((B, nh, N, D), generator=g) + 0.3).to(torch.bfloat16)
    s = lib.Shape(B, nh, D, 1, 1, N, blk, sb)
    scores = torch.empty((B, nh, s.nb, s.nb), dtype=torch.float32, device="cuda")
    ws = torch.empty(lib.dfs_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    lib.dfs_block_score(s, qp.cuda(), kp.cuda(), scale, scores, ws)
    torch.cuda.synchronize()
    pooled = ws.view(torch.float32).view(2, B, nh, s.nsb, D).cpu().numpy()
    return qp, kp, scores.cpu().numpy(), pooled, s


CASES = [
    (1, 2, 64, 2048, 64, 16),     # tiny workload
    (1, 3, 128, 1000, 128, 32),   # ragged: last block 104 tokens, last sub-block 8
    (2, 2, 128, 777, 128, 16),    # r = 8
    (1, 2, 64, 300, 64, 32),      # r = 2
    (1, 1, 128, 513, 128, 128),   # r = 1 (coarse block pooling)
    (1, 2, 128, 32760, 128, 32),  # full Wan-layer sequence, two heads
]


@pytest.mark.parametrize("B,nh,D,N,blk,sb", CASES)
def test_pool_and_scores(lib, B, nh, D, N, blk, sb):
    qp, kp, got, pooled, s = _run(lib, B, nh, D, N, blk, sb)
    q64, k64 = qp.double().numpy(), kp.double().numpy()
    oq, ok = scoring.pool_subblocks(q64, sb), scoring.pool_subblocks(k64, sb)
    tol_pool = (sb + 2) * U32 * max(np.abs(q64).max(), np.abs(k64).max())
    assert np.abs(pooled[0] - oq).max() <= tol_pool
    assert np.abs(pooled[1] - ok).max() <= tol_pool
    scale = 1.0 / math.sqrt(D)
    ref = scoring.block_scores(q64, k64, blk, sb, scale)
    # per-entry bound: (D + 2 sb + 4) u * scale * max |qbar| |kbar| summed over d
    mag = scale * D * np.abs(oq).max() * np.abs(ok).max()
    tol = (D + 2 * sb + 4) * U32 * mag
    err = np.abs(got - ref).max()
    assert err <= tol, (err, tol)


def test_explicit_scale(lib):
    qp, kp, got, _, s = _run(lib, 1, 1, 64, 500, 64, 16, seed=3, scale=0.5)
    ref = scoring.block_scores(qp.double().numpy(), kp.double().numpy(), 64, 16, 0.5)
    assert np.abs(got - ref).max() < 1e-4


@pytest.mark.parametrize("B,nh,D,grid,blk,sb", [(1, 2, 64, (8, 16, 16), 64, 16), (2, 3, 128, (3, 7, 11), 128, 32),
                                                (1, 12, 128, (21, 30, 52), 128, 32), (1, 1, 128, (1, 1, 100), 64, 8)])
def test_fused_gather_pool_then_score(lib, B, nh, D, grid, blk, sb):
    """dfs_hilbert_perm_pooled reorders exactly like the oracle and writes the
    sub-block means; dfs_block_score_pooled turns them into block scores."""
    from oracle import hilbert
    T, H, W = grid
    N = T * H * W
    g = torch.Generator().manual_seed(N + D)
    x = [torch.randn((B, N, nh, D), generator=g).to(torch.bfloat16) for _ in range(3)]
    s = lib.Shape(B, nh, D, T, H, W, blk, sb)
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty_like(perm)
    xp = [torch.empty((B, nh, N, D), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    ws = torch.empty(lib.dfs_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    scores = torch.empty((B, nh, s.nb, s.nb), dtype=torch.float32, device="cuda")
    lib.dfs_hilbert_perm_pooled(s, "hilbert3d", perm, inv, 1, *(t.cuda() for t in x), *xp, ws)
    lib.dfs_block_score_pooled(s, 0.0, scores, ws)
    torch.cuda.synchronize()
    operm, _ = hilbert.hilbert_perm(T, H, W)
    assert np.array_equal(perm.cpu().numpy(), operm)
    ref = [hilbert.permute_tokens(t.view(torch.int16).numpy(), operm) for t in x]
    for t in range(3):
        assert np.array_equal(xp[t].cpu().view(torch.int16).numpy(), ref[t])
    q64 = hilbert.permute_tokens(x[0].double().numpy(), operm)
    k64 = hilbert.permute_tokens(x[1].double().numpy(), operm)
    pooled = ws.view(torch.float32)[: 2 * B * nh * s.nsb * D].view(2, B, nh, s.nsb, D).cpu().numpy()
    oq, ok = scoring.pool_subblocks(q64, sb), scoring.pool_subblocks(k64, sb)
    tol_pool = (sb + 2) * U32 * max(np.abs(q64).max(), np.abs(k64).max())
    assert np.abs(pooled[0] - oq).max() <= tol_pool
    assert np.abs(pooled[1] - ok).max() <= tol_pool
    scale = 1.0 / math.sqrt(D)
    ref_s = scoring.block_scores(q64, k64, blk, sb, scale)
    mag = scale * D * np.abs(oq).max() * np.abs(ok).max()
    assert np.abs(scores.cpu().numpy() - ref_s).max() <= (D + 2 * sb + 4) * U32 * mag
