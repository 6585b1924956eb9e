"""Frame-exact LVSA attention on the GPU against the fp64 oracle.

Page: LVSA: Training-Free Sparse Attention for Long Video Diffusion,
section 2: each query frame t attends exactly the frames of A(t). The kept
blocks are the LVSA block mask (bit-exact against the oracle); inside them
the oracle drops every pair whose key frame is not in A(query frame).
Tolerance as for the block-sparse attention: max abs <= 2e-2, relative
Frobenius <= 5e-3.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import attention, lvsa, selection
from tests.parity import assert_attn_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa(cuda_device):
    import block_sparse_attention_36_b200 as m
    return m


def _qkv(B, N, nh, D, seed):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn((B, N, nh, D), generator=g) * 1.5).to(torch.bfloat16) for _ in range(3)]


def _head(x, b, h):
    return x[b, :, h, :].double().numpy()[None, None]


def _oracle_rows(qkv, layer, b, h, P, fa, rows=None):
    idx, cnt = layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy()
    allowed = lambda qs, ks: fa[np.asarray(qs)[:, None] // P, np.asarray(ks)[None, :] // P]
    return attention.block_sparse_attention(*(_head(x, b, h) for x in qkv), idx[b:b + 1, h:h + 1],
                                            cnt[b:b + 1, h:h + 1], layer.shape.blk, rows=rows, allowed=allowed)


# T, H, W, blk, D, T_per, C
SMALL = [
    (9, 8, 8, 64, 64, 3, 4),        # P = blk: blocks are frames
    (11, 16, 12, 128, 128, 4, 5),   # P = 1.5 blk: blocks straddle frames
    (7, 10, 13, 128, 64, 3, 3),     # P = 130, ragged last block
    (6, 9, 15, 64, 128, 2, 4),      # P = 135 with blk 64, three blocks per frame pair
]


@pytest.mark.parametrize("T,H,W,blk,D,T_per,C", SMALL)
def test_small_geometries_every_row(bsa, T, H, W, blk, D, T_per, C):
    B, nh = 1, 2
    P, N = H * W, T * H * W
    qkv = _qkv(B, N, nh, D, T * 100 + blk)
    for step in range(2):
        s = bsa.Shape(B, nh, D, T, H, W, blk, 16)
        layer = bsa.DfsLayer(s, order="raster", mode="lvsa", lvsa_T_per=T_per, lvsa_C=C, lvsa_step=step,
                             want_lse=True, frame_exact=True)
        out = layer.forward(*(x.cuda() for x in qkv))
        torch.cuda.synchronize()
        assert bsa.dfsattn.dfs_get_error_flags(clear=True) == 0
        m = lvsa.block_mask(T, P, blk, T_per, C, step)
        oi, oc = selection.mask_to_lists(np.broadcast_to(m, (B, nh) + m.shape), layer.kcap)
        assert np.array_equal(layer.kv_cnt.cpu().numpy(), oc)
        fa = lvsa.frame_allowed(T, T_per, C, step)
        got = out.float().cpu().numpy()
        lse = layer.lse.cpu().numpy()
        for h in range(nh):
            ref, ref_lse = _oracle_rows(qkv, layer, 0, h, P, fa)
            assert_attn_close(got[0, :, h], ref[0, 0], f"step {step} head {h}")
            assert np.abs(lse[0, h] - ref_lse[0, 0]).max() < 2e-2


def test_all_frames_allowed_equals_block_sparse(bsa):
    # C >= T: A(t) is every frame, so the frame mask drops nothing and the
    # frame-exact kernel must give the plain kernel's output bit for bit.
    T, H, W, blk, D = 5, 12, 12, 128, 128
    B, nh = 1, 2
    qkv = [x.cuda() for x in _qkv(B, T * H * W, nh, D, 7)]
    s = bsa.Shape(B, nh, D, T, H, W, blk, 16)
    outs = []
    for exact in (False, True):
        layer = bsa.DfsLayer(s, order="raster", mode="lvsa", lvsa_T_per=4, lvsa_C=T, want_lse=True,
                             frame_exact=exact)
        outs.append((layer.forward(*qkv).clone(), layer.lse.clone()))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
    assert torch.equal(outs[0][1], outs[1][1])


def test_long_video_whole_heads(bsa):
    """The 63-frame workload, frame-exact: every query block of the first
    and the last head, in raster order (the output of DfsLayer), against
    the oracle with the frame rule applied per pair."""
    from oracle import parallel
    wl = synth.WORKLOADS["lvsa_long_video"]
    qkv = synth.workload_inputs(wl)
    s = bsa.Shape(wl.B, wl.nh, wl.D, wl.T, wl.H, wl.W, wl.blk, wl.sb)
    layer = bsa.DfsLayer(s, order="raster", mode="lvsa", lvsa_T_per=wl.lvsa_T_per, lvsa_C=wl.lvsa_C,
                         lvsa_step=wl.lvsa_step, frame_exact=True)
    layer.forward(*(x.cuda() for x in (qkv["q"], qkv["k"], qkv["v"])))
    torch.cuda.synchronize()
    assert bsa.dfsattn.dfs_get_error_flags(clear=True) == 0
    P = wl.H * wl.W
    fa = lvsa.frame_allowed(wl.T, wl.lvsa_T_per, wl.lvsa_C, wl.lvsa_step)
    idx, cnt = layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy()
    heads = (0, wl.nh - 1)
    cur = [np.concatenate([_head(x, 0, h) for h in heads], axis=1) for x in (qkv["q"], qkv["k"], qkv["v"])]
    ii = np.concatenate([idx[:, h:h + 1] for h in heads], axis=1)
    cc = np.concatenate([cnt[:, h:h + 1] for h in heads], axis=1)
    rows = [(0, n, I) for n in range(len(heads)) for I in range(wl.nb)]
    res = parallel.block_sparse_attention_rows(*cur, ii, cc, wl.blk, rows, frame=(fa, P))
    out = layer.out.cpu()
    for n, h in enumerate(heads):
        want = np.concatenate([res[(0, n, I)][0] for I in range(wl.nb)])
        got = out[0, :, h, :].float().numpy()
        mx, rel = assert_attn_close(got, want, f"head {h}: every row")
        print(f"frame-exact LVSA head {h}: every row, max abs {mx:.3e}, rel fro {rel:.3e}")


def test_rejects_frames_smaller_than_a_block(bsa):
    lib = bsa.dfsattn
    T, H, W, blk, D = 4, 4, 8, 64, 64          # P = 32 < blk
    s = lib.Shape(1, 1, D, T, H, W, blk, 16)
    N = T * H * W
    x = torch.zeros((1, 1, N, D), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((1, 1, s.nb, 1), dtype=torch.int32, device="cuda")
    cnt = torch.ones((1, 1, s.nb), dtype=torch.int32, device="cuda")
    p = lib.select_params("lvsa", lvsa_T_per=2, lvsa_C=2)
    with pytest.raises(RuntimeError, match="unsupported"):
        lib.dfs_sparse_attn_lvsa_fwd(s, x, x, x, idx, cnt, 1, 0.0, p, torch.empty_like(x))
