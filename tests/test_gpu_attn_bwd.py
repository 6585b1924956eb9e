"""GPU gradients of the block-sparse attention against the fp64 oracle.

Oracle: the reverse rule of the block-sparse attention over the same kept
lists (pinned there against finite differences and autograd). The GPU
takes O and lse from its own forward and rounds P and dS to bf16 for the
tensor-core products (fp32 accumulation) and stores bf16, so each
gradient carries a few bf16 roundings (unit 2^-9) per term, mostly
independent: the forward's bounds apply, relative Frobenius <= 5e-3 and
max abs <= 2e-2 * max(1, max |reference|) per tensor (measured: 2.3e-3 to
2.6e-3 relative Frobenius on every case).
"""
import numpy as np
import pytest
import torch

from oracle import attention
from tests.parity import attn_errors

pytestmark = pytest.mark.gpu

RTOL_FRO = 5e-3
ATOL_MAX = 2e-2


@pytest.fixture(scope="module")
def lib(cuda_device):
    from block_sparse_attention_36_b200 import dfsattn
    return dfsattn


def _lists(rng, B, nh, nb, kcap, empty_rows=()):
    idx = np.full((B, nh, nb, kcap), -1, dtype=np.int32)
    cnt = np.zeros((B, nh, nb), dtype=np.int32)
    for b in range(B):
        for h in range(nh):
            for I in range(nb):
                c = 0 if I in empty_rows else int(rng.integers(1, min(kcap, nb) + 1))
                js = np.sort(rng.choice(nb, size=c, replace=False)) if c else np.zeros(0, np.int32)
                idx[b, h, I, :c] = js
                cnt[b, h, I] = c
    return idx, cnt


def _inputs(B, nh, N, D, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v = ((torch.randn((B, nh, N, D), generator=g) * 1.3).to(torch.bfloat16) for _ in range(3))
    do = (torch.randn((B, nh, N, D), generator=g) * 0.5).to(torch.bfloat16)
    return q, k, v, do


def _gpu_fwd_bwd(lib, q, k, v, do, idx, cnt, D, N, scale=0.0):
    B, nh = q.shape[0], q.shape[1]
    s = lib.Shape(B, nh, D, 1, 1, N, 128, 16)
    dev = [t.cuda() for t in (q, k, v, do)]
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    op = torch.empty_like(dev[0])
    lse = torch.empty((B, nh, N), dtype=torch.float32, device="cuda")
    lib.dfs_sparse_attn_fwd(s, dev[0], dev[1], dev[2], it, ct, idx.shape[-1], scale, op, lse)
    grads = [torch.empty_like(dev[0]) for _ in range(3)]
    ws = torch.empty(lib.dfs_workspace_bytes(s, lib.DFS_WS_ATTN_BWD), dtype=torch.uint8, device="cuda")
    lib.dfs_sparse_attn_bwd(s, dev[0], dev[1], dev[2], op, dev[3], lse, it, ct, idx.shape[-1], scale, *grads, ws)
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == 0
    return [g.float().cpu().numpy() for g in grads]


def _check(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        mx, rel = attn_errors(g, r)
        bound = ATOL_MAX * max(1.0, float(np.abs(r).max()))
        print(f"{what} {name}: max abs {mx:.3e} (bound {bound:.3e}), rel fro {rel:.3e}")
        assert mx <= bound and rel <= RTOL_FRO, f"{what} {name}: max abs {mx:.3e}, rel fro {rel:.3e}"


CASES = [  # B, nh, D, N, kcap
    (1, 2, 128, 1000, 5),      # ragged last block (104 rows)
    (1, 2, 128, 4096, 12),
    (2, 1, 64, 2048, 16),      # D = 64, full lists possible
    (1, 1, 64, 700, 6),        # ragged (60)
    (1, 1, 128, 128, 1),       # one block
]


@pytest.mark.parametrize("B,nh,D,N,kcap", CASES)
def test_random_lists(lib, B, nh, D, N, kcap):
    nb = -(-N // 128)
    rng = np.random.default_rng(N + D)
    idx, cnt = _lists(rng, B, nh, nb, kcap)
    q, k, v, do = _inputs(B, nh, N, D, N + 7 * D)
    got = _gpu_fwd_bwd(lib, q, k, v, do, idx, cnt, D, N)
    ref = attention.block_sparse_attention_bwd(*(t.double().numpy() for t in (q, k, v, do)), idx, cnt, 128)
    _check(got, ref, f"B{B} nh{nh} D{D} N{N}")


def test_empty_rows_and_unused_keys(lib):
    B, nh, D, N = 1, 1, 128, 1024
    nb = N // 128
    idx = np.full((1, 1, nb, 3), -1, dtype=np.int32)
    cnt = np.zeros((1, 1, nb), dtype=np.int32)
    for I in range(nb):
        if I in (2, 5):
            continue                       # empty rows
        js = [0, 3] if I % 2 else [0, 3, 6]  # key blocks 1, 2, 4, 5, 7 never kept
        idx[0, 0, I, :len(js)] = js
        cnt[0, 0, I] = len(js)
    q, k, v, do = _inputs(B, nh, N, D, 3)
    dq, dk, dv = _gpu_fwd_bwd(lib, q, k, v, do, idx, cnt, D, N)
    for I in (2, 5):
        assert (dq[0, 0, I * 128:(I + 1) * 128] == 0).all()
    for J in (1, 2, 4, 5, 7):
        assert (dk[0, 0, J * 128:(J + 1) * 128] == 0).all() and (dv[0, 0, J * 128:(J + 1) * 128] == 0).all()
    ref = attention.block_sparse_attention_bwd(*(t.double().numpy() for t in (q, k, v, do)), idx, cnt, 128)
    _check((dq, dk, dv), ref, "empty rows")


def test_invalid_entries_are_skipped_and_flagged(lib):
    """Entries outside [0, nb) inside the counted part of a list are skipped
    by both passes (the dQ pass reads the caller's lists, in groups of 32)
    and raise DFS_FLAG_BAD_KV_INDEX; the gradients equal those of the lists
    without them."""
    B, nh, D, N = 1, 2, 128, 5000
    nb = -(-N // 128)                      # 40 blocks: lists span two groups of 32
    kcap = nb
    rng = np.random.default_rng(11)
    idx = np.full((B, nh, nb, kcap), -1, dtype=np.int32)
    cnt = np.zeros((B, nh, nb), dtype=np.int32)
    clean_idx = np.full_like(idx, -1)
    clean_cnt = np.zeros_like(cnt)
    for h in range(nh):
        for I in range(nb):
            c = int(rng.integers(1, 38))   # with up to 3 invalid entries: at most kcap = 40
            js = list(np.sort(rng.choice(nb, size=c, replace=False)))
            row = list(js)
            for pos, bad in ((0, -1), (len(row) // 2, nb), (len(row), nb + 7)):
                if I % 3 == h % 3:
                    row.insert(pos, bad)
            idx[0, h, I, :len(row)] = row
            cnt[0, h, I] = len(row)
            clean_idx[0, h, I, :c] = js
            clean_cnt[0, h, I] = c
    q, k, v, do = _inputs(B, nh, N, D, 21)
    s = lib.Shape(B, nh, D, 1, 1, N, 128, 16)
    dev = [t.cuda() for t in (q, k, v, do)]
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    op = torch.empty_like(dev[0])
    lse = torch.empty((B, nh, N), dtype=torch.float32, device="cuda")
    lib.dfs_get_error_flags(clear=True)
    lib.dfs_sparse_attn_fwd(s, dev[0], dev[1], dev[2], it, ct, kcap, 0.0, op, lse)
    grads = [torch.empty_like(dev[0]) for _ in range(3)]
    ws = torch.empty(lib.dfs_workspace_bytes(s, lib.DFS_WS_ATTN_BWD), dtype=torch.uint8, device="cuda")
    lib.dfs_sparse_attn_bwd(s, dev[0], dev[1], dev[2], op, dev[3], lse, it, ct, kcap, 0.0, *grads, ws)
    torch.cuda.synchronize()
    flags = lib.dfs_get_error_flags(clear=True)
    assert flags & lib.DFS_FLAG_BAD_KV_INDEX
    assert not flags & lib.DFS_FLAG_WAIT_TIMEOUT
    got = [g.float().cpu().numpy() for g in grads]
    ref = attention.block_sparse_attention_bwd(*(t.double().numpy() for t in (q, k, v, do)), clean_idx, clean_cnt,
                                               128)
    _check(got, ref, "invalid entries")
    # The backward over the clean lists, from the same forward outputs, is
    # bitwise the same. (The forward's own results may differ by rounding:
    # a split last-wave CTA halves the counted list, invalid entries included.)
    ic, cc = torch.from_numpy(clean_idx).cuda(), torch.from_numpy(clean_cnt).cuda()
    grads2 = [torch.empty_like(dev[0]) for _ in range(3)]
    lib.dfs_sparse_attn_bwd(s, dev[0], dev[1], dev[2], op, dev[3], lse, ic, cc, kcap, 0.0, *grads2, ws)
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == 0
    for x, y in zip(grads, grads2):
        assert torch.equal(x, y)


def test_maximum_block_count(lib):
    """nb = 8192, the largest the backward takes (1,048,576 tokens at D = 64),
    runs and is right; 8193 is rejected before anything is launched. Query
    block I keeps blocks {0, I}, so key block J >= 1 is kept by query block J
    alone and key block 0 by all 8192 (one dK/dV CTA walks the whole
    transposed list): dQ of query block J and dK, dV of key block J equal
    those of the two-block problem (blocks 0 and J) in the oracle."""
    D, blk = 64, 128
    nb_max = 8192
    N_big = (nb_max + 1) * blk
    N = nb_max * blk
    g = torch.Generator().manual_seed(31)
    host = [(torch.randn((1, 1, N_big, D), generator=g) * 1.3).to(torch.bfloat16) for _ in range(3)]
    host.append((torch.randn((1, 1, N_big, D), generator=g) * 0.5).to(torch.bfloat16))
    dev = [t.cuda() for t in host]
    view = [t[:, :, :N] for t in dev]                        # contiguous: leading dims are 1
    s = lib.Shape(1, 1, D, 1, 1, N, blk, 16)
    idx = np.zeros((1, 1, nb_max, 2), dtype=np.int32)
    idx[0, 0, :, 1] = np.arange(nb_max)
    cnt = np.full((1, 1, nb_max), 2, dtype=np.int32)
    cnt[0, 0, 0] = 1                                         # block 0 keeps only itself
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    op = torch.empty_like(view[0])
    lse = torch.empty((1, 1, N), dtype=torch.float32, device="cuda")
    lib.dfs_get_error_flags(clear=True)
    lib.dfs_sparse_attn_fwd(s, view[0], view[1], view[2], it, ct, 2, 0.0, op, lse)
    grads = [torch.empty_like(view[0]) for _ in range(3)]
    ws = torch.empty(lib.dfs_workspace_bytes(s, lib.DFS_WS_ATTN_BWD), dtype=torch.uint8, device="cuda")
    lib.dfs_sparse_attn_bwd(s, view[0], view[1], view[2], op, view[3], lse, it, ct, 2, 0.0, *grads, ws)
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == 0
    for J in (1, 2, 4095, nb_max - 1):
        rows = np.r_[0:blk, J * blk:(J + 1) * blk]
        mini = [t[:, :, rows].double().numpy() for t in host]
        mi = np.array([[[[0, -1], [0, 1]]]], dtype=np.int32)
        mc = np.array([[[1, 2]]], dtype=np.int32)
        ref = attention.block_sparse_attention_bwd(*mini, mi, mc, blk, rows=[(0, 0, 1)])
        sl = slice(J * blk, (J + 1) * blk)
        got = [x[:, :, sl].float().cpu().numpy() for x in grads]
        _check(got, [r[:, :, blk:] for r in ref], f"nb 8192, block {J}")
    # one more block than the backward takes: rejected on the host side of the launch
    s2 = lib.Shape(1, 1, D, 1, 1, N_big, blk, 16)
    idx2 = torch.zeros((1, 1, nb_max + 1, 2), dtype=torch.int32, device="cuda")
    cnt2 = torch.ones((1, 1, nb_max + 1), dtype=torch.int32, device="cuda")
    lse2 = torch.zeros((1, 1, N_big), dtype=torch.float32, device="cuda")
    out2 = [torch.full_like(dev[0], 3.0) for _ in range(3)]
    ws2 = torch.empty(lib.dfs_workspace_bytes(s2, lib.DFS_WS_ATTN_BWD), dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.DfsError) as e:
        lib.dfs_sparse_attn_bwd(s2, dev[0], dev[1], dev[2], dev[0], dev[3], lse2, idx2, cnt2, 2, 0.0, *out2, ws2)
    assert e.value.status == lib.DFS_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert all(bool((x == 3.0).all()) for x in out2)


def test_full_mask_matches_dense_gradients(lib):
    B, nh, D, N = 1, 2, 64, 640
    nb = N // 128
    idx = np.tile(np.arange(nb, dtype=np.int32), (B, nh, nb, 1))
    cnt = np.full((B, nh, nb), nb, dtype=np.int32)
    q, k, v, do = _inputs(B, nh, N, D, 5)
    got = _gpu_fwd_bwd(lib, q, k, v, do, idx, cnt, D, N, scale=0.1)
    tq, tk, tv = (t.double().requires_grad_(True) for t in (q, k, v))
    o = torch.softmax(tq @ tk.transpose(-1, -2) * 0.1, dim=-1) @ tv
    o.backward(do.double())
    _check(got, [tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()], "full mask vs dense autograd")


def test_deterministic(lib):
    B, nh, D, N = 1, 2, 128, 2000
    nb = -(-N // 128)
    idx, cnt = _lists(np.random.default_rng(1), B, nh, nb, 9)
    q, k, v, do = _inputs(B, nh, N, D, 9)
    a = _gpu_fwd_bwd(lib, q, k, v, do, idx, cnt, D, N)
    b = _gpu_fwd_bwd(lib, q, k, v, do, idx, cnt, D, N)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_rejects_blk64_and_short_workspace(lib):
    s64 = lib.Shape(1, 1, 64, 1, 1, 256, 64, 16)
    assert lib.dfs_workspace_bytes(s64, lib.DFS_WS_ATTN_BWD) == 0
    s = lib.Shape(1, 1, 64, 1, 1, 256, 128, 16)
    x = torch.zeros((1, 1, 256, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 1, 256), dtype=torch.float32, device="cuda")
    idx = torch.zeros((1, 1, 2, 1), dtype=torch.int32, device="cuda")
    cnt = torch.ones((1, 1, 2), dtype=torch.int32, device="cuda")
    # a short view of a buffer large enough for the call: a size check that
    # failed to reject it would still write only memory this test owns
    need = lib.dfs_workspace_bytes(s, lib.DFS_WS_ATTN_BWD)
    big = torch.empty(need, dtype=torch.uint8, device="cuda")
    small = big[:256]
    with pytest.raises(RuntimeError, match="workspace"):
        lib.dfs_sparse_attn_bwd(s, x, x, x, x, x, lse, idx, cnt, 1, 0.0, x, x, x, small)
    idx64 = torch.zeros((1, 1, s64.nb, 1), dtype=torch.int32, device="cuda")
    cnt64 = torch.ones((1, 1, s64.nb), dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError, match="unsupported"):
        lib.dfs_sparse_attn_bwd(s64, x, x, x, x, x, lse, idx64, cnt64, 1, 0.0, x, x, x, small)


def test_layer_backward_wan_sampled(lib):
    """Wan-shaped layer end to end: forward, then backward through
    DfsLayer (dO reordered, gradients scattered back to raster order);
    dQ, dK and dV on every row of the first head (the oracle's whole-head
    gradients), and on sampled blocks of the last head (dK/dV of a key block
    from all query blocks that keep it), by the oracle in curve order."""
    import synth
    import block_sparse_attention_36_b200 as bsa
    wl = synth.WORKLOADS["wan_1p3b_layer"]
    qkv = synth.workload_inputs(wl)
    s = bsa.Shape(wl.B, wl.nh, wl.D, wl.T, wl.H, wl.W, wl.blk, wl.sb)
    layer = bsa.DfsLayer(s, order=wl.order, mode="topk", k=wl.ratio_count(wl.keep_num), want_lse=True)
    layer.forward(*(qkv[n].cuda() for n in ("q", "k", "v")))
    g = torch.Generator().manual_seed(21)
    dout = (torch.randn((wl.B, wl.N, wl.nh, wl.D), generator=g) * 0.5).to(torch.bfloat16)
    dq, dk, dv = layer.backward(dout.cuda())
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == 0
    perm = layer.perm.cpu().numpy().astype(np.int64)
    idx, cnt = layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy()
    rng = np.random.default_rng(2)
    got_q, ref_q, got_kv, ref_kv = [], [], [], []
    for h in (0, wl.nh - 1):
        cur = [x[0, perm, h, :].double().numpy()[None, None] for x in (qkv["q"], qkv["k"], qkv["v"], dout)]
        gq, gk, gv = (x.cpu()[0, perm, h, :].float().numpy() for x in (dq, dk, dv))
        ii, cc = idx[:, h:h + 1], cnt[:, h:h + 1]
        Is = [0, wl.nb - 1] + [int(x) for x in rng.integers(0, wl.nb, 3)]
        rq, _, _ = attention.block_sparse_attention_bwd(*cur, ii, cc, wl.blk, rows=[(0, 0, I) for I in Is])
        for I in Is:
            lo, hi = I * wl.blk, min(wl.N, I * wl.blk + wl.blk)
            got_q.append(gq[lo:hi]); ref_q.append(rq[0, 0, lo:hi])
        for J in [wl.nb - 1, int(rng.integers(0, wl.nb))]:
            keepers = [(0, 0, I) for I in range(wl.nb) if J in set(ii[0, 0, I, :cc[0, 0, I]].tolist())]
            _, rk, rv = attention.block_sparse_attention_bwd(*cur, ii, cc, wl.blk, rows=keepers)
            lo, hi = J * wl.blk, min(wl.N, J * wl.blk + wl.blk)
            got_kv.append(np.concatenate([gk[lo:hi], gv[lo:hi]], 1))
            ref_kv.append(np.concatenate([rk[0, 0, lo:hi], rv[0, 0, lo:hi]], 1))
    _check((np.concatenate(got_q), np.concatenate(got_kv)[:, :wl.D], np.concatenate(got_kv)[:, wl.D:]),
           (np.concatenate(ref_q), np.concatenate(ref_kv)[:, :wl.D], np.concatenate(ref_kv)[:, wl.D:]),
           "Wan layer sampled")
    # every row of head 0: the oracle's gradients of the whole head
    cur = [x[0, perm, 0, :].double().numpy()[None, None] for x in (qkv["q"], qkv["k"], qkv["v"], dout)]
    rq, rk, rv = attention.block_sparse_attention_bwd(*cur, idx[:, :1], cnt[:, :1], wl.blk)
    got = tuple(x.cpu()[0, perm, 0, :].float().numpy() for x in (dq, dk, dv))
    _check(got, (rq[0, 0], rk[0, 0], rv[0, 0]), "Wan layer, every row of head 0")


def test_layer_backward_hunyuan_sampled(lib):
    """The threshold-selected Hunyuan-shaped layer (24 heads, 118,800
    tokens, uneven list lengths): dQ on sampled query blocks and dK/dV on
    sampled key blocks (from every query block that keeps them), one head."""
    import synth
    import block_sparse_attention_36_b200 as bsa
    wl = synth.WORKLOADS["hunyuan_layer"]
    qkv = synth.workload_inputs(wl)
    s = bsa.Shape(wl.B, wl.nh, wl.D, wl.T, wl.H, wl.W, wl.blk, wl.sb)
    layer = bsa.DfsLayer(s, order=wl.order, mode="threshold", cap=wl.ratio_count(wl.cap_num), tau=wl.tau,
                         want_lse=True)
    layer.forward(*(qkv[n].cuda() for n in ("q", "k", "v")))
    g = torch.Generator().manual_seed(22)
    dout = (torch.randn((wl.B, wl.N, wl.nh, wl.D), generator=g) * 0.5).to(torch.bfloat16)
    dq, dk, dv = layer.backward(dout.cuda())
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == 0
    perm = torch.from_numpy(layer.perm.cpu().numpy().astype(np.int64))
    h = 7
    ii, cc = layer.kv_idx.cpu().numpy()[:, h:h + 1], layer.kv_cnt.cpu().numpy()[:, h:h + 1]
    cur = [x[0, perm, h, :].double().numpy()[None, None] for x in (qkv["q"], qkv["k"], qkv["v"], dout)]
    gq, gk, gv = (x.cpu()[0, perm, h, :].float().numpy() for x in (dq, dk, dv))
    rng = np.random.default_rng(5)
    Is = [0, wl.nb - 1] + [int(x) for x in rng.integers(0, wl.nb, 2)]
    rq, _, _ = attention.block_sparse_attention_bwd(*cur, ii, cc, wl.blk, rows=[(0, 0, I) for I in Is])
    Js = [wl.nb - 1, int(rng.integers(0, wl.nb))]
    keep = [set(ii[0, 0, I, :cc[0, 0, I]].tolist()) for I in range(wl.nb)]
    got_q = np.concatenate([gq[I * wl.blk:min(wl.N, I * wl.blk + wl.blk)] for I in Is])
    ref_q = np.concatenate([rq[0, 0, I * wl.blk:min(wl.N, I * wl.blk + wl.blk)] for I in Is])
    got_k, got_v, ref_k, ref_v = [], [], [], []
    for J in Js:
        rows = [(0, 0, I) for I in range(wl.nb) if J in keep[I]]
        _, rk, rv = attention.block_sparse_attention_bwd(*cur, ii, cc, wl.blk, rows=rows)
        lo, hi = J * wl.blk, min(wl.N, J * wl.blk + wl.blk)
        got_k.append(gk[lo:hi]); got_v.append(gv[lo:hi]); ref_k.append(rk[0, 0, lo:hi]); ref_v.append(rv[0, 0, lo:hi])
    _check((got_q, np.concatenate(got_k), np.concatenate(got_v)),
           (ref_q, np.concatenate(ref_k), np.concatenate(ref_v)), "Hunyuan layer sampled")
