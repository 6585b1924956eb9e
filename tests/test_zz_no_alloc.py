"""The scoring entry point that allocates nothing, against the one that takes
a workspace.

dfs_block_score_noalloc is for callers that cannot allocate device memory --
a plugin whose host gives it only tensors and a stream, or a process whose
caching allocator already holds the whole device -- so its pooled-mean
scratch is a fixed buffer compiled into the library. Both entry points run the
same kernels on the same inputs, so the scores must be bit-identical to
dfs_block_score's, on consecutive calls too: the shared buffer keeps the
previous call's contents, and any of it leaking into the next result would
show as a changed bit. A shape that needs more scratch than the buffer holds
must be rejected before anything is launched.

This file is named to be collected last, so that with -x a failure here
comes after every other test has run.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib(cuda_device):
    from block_sparse_attention_36_b200 import dfsattn
    return dfsattn


def _inputs(B, nh, N, D, seed):
    g = torch.Generator().manual_seed(seed)
    qp = torch.randn((B, nh, N, D), generator=g).to(torch.bfloat16).cuda()
    kp = (torch.randn((B, nh, N, D), generator=g) + 0.25).to(torch.bfloat16).cuda()
    return qp, kp


def _with_workspace(lib, s, qp, kp):
    out = torch.empty((s.B, s.nh, s.nb, s.nb), dtype=torch.float32, device="cuda")
    ws = torch.empty(lib.dfs_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    lib.dfs_block_score(s, qp, kp, 0.0, out, ws)
    return out


def _noalloc(lib, s, qp, kp):
    out = torch.full((s.B, s.nh, s.nb, s.nb), float("nan"), dtype=torch.float32, device="cuda")
    lib.dfs_block_score_noalloc(s, qp, kp, 0.0, out)
    return out


def test_two_calls_in_a_row_match_workspace_version(lib):
    cases = [
        (lib.Shape(1, 12, 128, 21, 30, 52, 128, 32), 1),   # Wan layer: 12.6 MB of scratch
        (lib.Shape(1, 2, 64, 8, 16, 16, 64, 16), 2),       # tiny layer, after the larger one
    ]
    for s, seed in cases:
        qp, kp = _inputs(s.B, s.nh, s.N, s.D, seed)
        got = _noalloc(lib, s, qp, kp)
        ref = _with_workspace(lib, s, qp, kp)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert torch.equal(got, ref)
    # the larger shape again, right after the smaller one: the same bits
    s, seed = cases[0]
    qp, kp = _inputs(s.B, s.nh, s.N, s.D, seed)
    a = _noalloc(lib, s, qp, kp)
    b = _noalloc(lib, s, qp, kp)
    ref = _with_workspace(lib, s, qp, kp)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(a, ref)


def test_oversize_shape_is_rejected(lib):
    # 36 heads on the Wan grid, 32-token sub-blocks: 37.7 MB of pooled means,
    # more than the built-in buffer holds. Every tensor is sized for this
    # shape, so even a check that failed to reject it would stay in bounds.
    s = lib.Shape(1, 36, 128, 21, 30, 52, 128, 32)
    need = 2 * s.B * s.nh * s.nsb * s.D * 4
    assert need > lib.NOALLOC_SCRATCH_BYTES
    qp, kp = _inputs(s.B, s.nh, s.N, s.D, 3)
    out = torch.full((s.B, s.nh, s.nb, s.nb), float("nan"), dtype=torch.float32, device="cuda")
    with pytest.raises(lib.DfsError) as e:
        lib.dfs_block_score_noalloc(s, qp, kp, 0.0, out)
    assert e.value.status == lib.DFS_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.isnan(out).all()                        # nothing was launched
