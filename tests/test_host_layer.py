"""DfsLayer's host-side set-up, built on the CPU (no kernel runs): buffer
shapes, the per-mode state and the workspace sizes the C library reports."""
import pytest
import torch

MODES = [
    ("topk", dict(k=39)),
    ("threshold", dict(cap=186, tau=0.9)),
    ("global", dict(k=9831)),
    ("lvsa", dict(lvsa_T_per=8, lvsa_C=21)),
    ("radial", dict(radial_w0=1560, radial_lambda=0.125)),
]


@pytest.fixture(scope="module")
def bsa():
    import block_sparse_attention_36_b200 as m
    return m


@pytest.mark.parametrize("mode,kw", MODES)
@pytest.mark.parametrize("order", ["hilbert3d", "raster"])
def test_layer_state(bsa, mode, kw, order):
    s = bsa.Shape(1, 12, 128, 21, 30, 52, 128, 32)
    layer = bsa.DfsLayer(s, order=order, mode=mode, device="cpu", want_lse=True, **kw)
    assert layer.order == order                     # the token order, untouched by the mode
    assert layer.qp.shape == (1, 12, s.N, 128) and layer.out.shape == (1, s.N, 12, 128)
    assert layer.kv_idx.shape == (1, 12, s.nb, layer.kcap) and layer.kv_cnt.shape == (1, 12, s.nb)
    assert layer.lse.shape == (1, 12, s.N)
    if mode in ("lvsa", "radial"):
        assert layer.scores is None and layer.ws is None
    else:
        assert layer.scores.shape == (1, 12, s.nb, s.nb)
        assert layer.ws.numel() >= bsa.dfsattn.dfs_workspace_bytes(s, bsa.dfsattn.DFS_WS_BLOCK_SCORE)
    if mode in ("threshold", "global"):
        assert layer.work_order.shape == (12 * s.nb,) and layer.work_order.dtype == torch.int32
    else:
        assert layer.work_order is None


def test_frame_exact_needs_lvsa_and_raster(bsa):
    s = bsa.Shape(1, 2, 64, 9, 8, 8, 64, 16)
    with pytest.raises(ValueError):
        bsa.DfsLayer(s, order="hilbert3d", mode="lvsa", device="cpu", frame_exact=True)
    with pytest.raises(ValueError):
        bsa.DfsLayer(s, order="raster", mode="topk", k=2, device="cpu", frame_exact=True)
    assert bsa.DfsLayer(s, order="raster", mode="lvsa", device="cpu", frame_exact=True).frame_exact


def test_backward_workspace_size(bsa):
    lib = bsa.dfsattn
    s = bsa.Shape(1, 12, 128, 21, 30, 52, 128, 32)
    nb, bh = s.nb, 12
    r256 = lambda x: (x + 255) // 256 * 256
    want = 2 * r256(bh * nb * 128 * 4) + r256(bh * nb * ((nb + 31) // 32) * 4) + r256(bh * nb * 4) + r256(bh * nb * nb * 4)
    assert lib.dfs_workspace_bytes(s, lib.DFS_WS_ATTN_BWD) == want
    assert lib.dfs_workspace_bytes(bsa.Shape(1, 1, 64, 1, 1, 256, 64, 16), lib.DFS_WS_ATTN_BWD) == 0
