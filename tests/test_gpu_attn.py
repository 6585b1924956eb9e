"""GPU block-sparse attention against the fp64 oracle.

Page: DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology item 3 and Significance (block-wise execution over
the kept blocks). Tolerance: max abs <= 2e-2, relative Frobenius <= 5e-3.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention
from tests.parity import assert_attn_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib(cuda_device):
    from block_sparse_attention_36_b200 import dfsattn
    return dfsattn


def _lists(rng, B, nh, nb, kcap, full=False):
    idx = np.full((B, nh, nb, kcap), -1, dtype=np.int32)
    cnt = np.zeros((B, nh, nb), dtype=np.int32)
    for b in range(B):
        for h in range(nh):
            for I in range(nb):
                c = nb if full else int(rng.integers(0, min(kcap, nb) + 1))
                c = min(c, kcap)
                js = np.sort(rng.choice(nb, size=c, replace=False)) if c else np.zeros(0, np.int32)
                idx[b, h, I, :c] = js
                cnt[b, h, I] = c
    return idx, cnt


def _run(lib, q, k, v, idx, cnt, D, blk, N, scale=0.0, want_lse=True):
    B, nh = q.shape[0], q.shape[1]
    s = lib.Shape(B, nh, D, 1, 1, N, blk, 16)
    op = torch.empty((B, nh, N, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, nh, N), dtype=torch.float32, device="cuda") if want_lse else None
    lib.dfs_sparse_attn_fwd(s, q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(idx).cuda(),
                            torch.from_numpy(cnt).cuda(), idx.shape[-1], scale, op, lse)
    torch.cuda.synchronize()
    return op.float().cpu().numpy(), (lse.cpu().numpy() if want_lse else None)


CASES = [  # B, nh, D, blk, N
    (1, 2, 128, 128, 1000),    # ragged last block (104)
    (1, 2, 128, 128, 4096),
    (2, 1, 64, 64, 2048),      # tiny workload geometry
    (1, 2, 64, 64, 1000),      # ragged (40)
    (1, 1, 128, 64, 700),
    (1, 1, 64, 128, 700),
]


@pytest.mark.parametrize("B,nh,D,blk,N", CASES)
def test_random_lists(lib, B, nh, D, blk, N):
    rng = np.random.default_rng(N + D)
    g = torch.Generator().manual_seed(N)
    q = torch.randn((B, nh, N, D), generator=g).to(torch.bfloat16)
    k = torch.randn((B, nh, N, D), generator=g).to(torch.bfloat16)
    v = torch.randn((B, nh, N, D), generator=g).to(torch.bfloat16)
    nb = -(-N // blk)
    kcap = max(1, nb // 2 + 1)
    idx, cnt = _lists(rng, B, nh, nb, kcap)
    got, lse = _run(lib, q, k, v, idx, cnt, D, blk, N)
    ref, rlse = attention.block_sparse_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                                 idx, cnt, blk)
    assert_attn_close(got, ref, "output")
    fin = np.isfinite(rlse)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.abs(lse[fin] - rlse[fin]).max() < 1e-3


@pytest.mark.parametrize("D,blk", [(128, 128), (64, 64)])
def test_full_mask_is_dense(lib, D, blk):
    N = 640 if blk == 128 else 576
    g = torch.Generator().manual_seed(7)
    q, k, v = (torch.randn((1, 2, N, D), generator=g).to(torch.bfloat16) for _ in range(3))
    nb = -(-N // blk)
    idx, cnt = _lists(np.random.default_rng(0), 1, 2, nb, nb, full=True)
    got, _ = _run(lib, q, k, v, idx, cnt, D, blk, N)
    ref = attention.dense_attention(q.double().numpy(), k.double().numpy(), v.double().numpy())
    assert_attn_close(got, ref, "dense")


def test_peaked_logits_and_rescale(lib):
    # Large logits make the running maximum jump between blocks, which
    # exercises the O rescale path; scale is passed explicitly.
    N, D, blk = 1024, 128, 128
    g = torch.Generator().manual_seed(11)
    q = (torch.randn((1, 1, N, D), generator=g) * 3).to(torch.bfloat16)
    k = (torch.randn((1, 1, N, D), generator=g) * 3).to(torch.bfloat16)
    k[:, :, 700:710] *= 4
    v = torch.randn((1, 1, N, D), generator=g).to(torch.bfloat16)
    nb = N // blk
    idx, cnt = _lists(np.random.default_rng(1), 1, 1, nb, nb, full=True)
    got, _ = _run(lib, q, k, v, idx, cnt, D, blk, N, scale=0.2)
    ref, _ = attention.block_sparse_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                              idx, cnt, blk, 0.2)
    assert_attn_close(got, ref, "peaked")


def test_empty_rows_and_bad_indices(lib):
    N, D, blk = 512, 64, 64
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn((1, 1, N, D), generator=g).to(torch.bfloat16) for _ in range(3))
    nb = N // blk
    idx = np.full((1, 1, nb, 4), -1, dtype=np.int32)
    cnt = np.zeros((1, 1, nb), dtype=np.int32)
    idx[0, 0, 1, :3] = [0, 99, 5]          # 99 is out of range: skipped, flagged
    cnt[0, 0, 1] = 3
    idx[0, 0, 2, :2] = [2, 3]
    cnt[0, 0, 2] = 2
    lib.dfs_get_error_flags(clear=True)
    got, lse = _run(lib, q, k, v, idx, cnt, D, blk, N)
    assert lib.dfs_get_error_flags(clear=True) & lib.DFS_FLAG_BAD_KV_INDEX
    clean_idx, clean_cnt = idx.copy(), cnt.copy()
    clean_idx[0, 0, 1, :3] = [0, 5, -1]
    clean_cnt[0, 0, 1] = 2
    ref, rlse = attention.block_sparse_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                                 clean_idx, clean_cnt, blk)
    assert_attn_close(got, ref, "bad indices")
    assert (got[0, 0, :64] == 0).all() and np.isneginf(lse[0, 0, :64]).all()


def test_constant_v(lib):
    N, D, blk = 384, 128, 128
    g = torch.Generator().manual_seed(2)
    q, k = (torch.randn((1, 1, N, D), generator=g).to(torch.bfloat16) for _ in range(2))
    v = torch.full((1, 1, N, D), 0.75).to(torch.bfloat16)
    nb = N // blk
    idx, cnt = _lists(np.random.default_rng(3), 1, 1, nb, 2)
    cnt[cnt == 0] = 1
    idx[..., 0] = np.where(idx[..., 0] < 0, 0, idx[..., 0])
    got, _ = _run(lib, q, k, v, idx, cnt, D, blk, N)
    assert np.abs(got - 0.75).max() < 4e-3


@pytest.mark.parametrize("grid,D", [((3, 7, 11), 64), ((8, 16, 16), 128), ((21, 30, 52), 128)])
def test_scatter_epilogue_equals_fwd_then_unperm(lib, grid, D):
    """The fused inverse reorder writes, bit for bit, what the curve-order
    forward followed by dfs_unperm writes."""
    from oracle import hilbert
    T, H, W = grid
    N, nh, blk = T * H * W, 2, 128
    s = lib.Shape(1, nh, D, T, H, W, blk, 16)
    nb = s.nb
    rng = np.random.default_rng(N)
    idx, cnt = _lists(rng, 1, nh, nb, min(nb, 6))
    g = torch.Generator().manual_seed(N)
    qp, kp, vp = ((torch.randn((1, nh, N, D), generator=g)).to(torch.bfloat16).cuda() for _ in range(3))
    perm = torch.from_numpy(hilbert.make_perm("hilbert3d", T, H, W)[0].astype(np.int32)).cuda()
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    op = torch.empty_like(qp)
    lse_a = torch.empty((1, nh, N), dtype=torch.float32, device="cuda")
    lse_b = torch.empty_like(lse_a)
    lib.dfs_sparse_attn_fwd(s, qp, kp, vp, it, ct, idx.shape[-1], 0.0, op, lse_a)
    ref = torch.empty((1, N, nh, D), dtype=torch.bfloat16, device="cuda")
    lib.dfs_unperm(s, perm, op, ref)
    out = torch.full_like(ref, float("nan"))
    lib.dfs_sparse_attn_fwd_ex(s, qp, kp, vp, it, ct, idx.shape[-1], 0.0, out, lse_b, perm=perm)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(lse_a, lse_b)


@pytest.mark.parametrize("B,nh,D,N,kcap", [(1, 3, 128, 5000, 20), (2, 2, 64, 3000, 24)])
def test_work_order_changes_nothing(lib, B, nh, D, N, kcap):
    """Rows run in count order (dfs_attn_order, dfs_attn_opts.order) give
    bit for bit the rows of the default order (tail split off); the order is
    a permutation sorted by kept count, largest first."""
    blk = 128
    nb = -(-N // blk)
    rng = np.random.default_rng(B * N)
    idx, cnt = _lists(rng, B, nh, nb, kcap)
    s = lib.Shape(B, nh, D, 1, 1, N, blk, 16)
    g = torch.Generator().manual_seed(N + D)
    qp, kp, vp = ((torch.randn((B, nh, N, D), generator=g)).to(torch.bfloat16).cuda() for _ in range(3))
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    order = torch.full((B * nh * nb,), -1, dtype=torch.int32, device="cuda")
    lib.dfs_attn_order(s, ct, kcap, order)
    a, b = torch.empty_like(qp), torch.empty_like(qp)
    la = torch.empty((B, nh, N), dtype=torch.float32, device="cuda")
    lb = torch.empty_like(la)
    # every CTA on two rows in both launches (a split tail would merge
    # different rows in the two orders)
    lib.dfs_sparse_attn_fwd_ex(s, qp, kp, vp, it, ct, kcap, 0.0, a, la, tail_split=False)
    lib.dfs_sparse_attn_fwd_ex(s, qp, kp, vp, it, ct, kcap, 0.0, b, lb, order=order, tail_split=False)
    torch.cuda.synchronize()
    o = order.cpu().numpy()
    assert np.array_equal(o, _per_head_order(cnt, min(kcap, nb)))
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(la, lb)


@pytest.mark.parametrize("nh,D,N,kcap,with_order", [(5, 128, 8192, 9, False), (3, 64, 14158, 7, True)])
def test_tail_split(lib, nh, D, N, kcap, with_order):
    """The last, partial wave of two-row CTAs runs as one-row CTAs whose two
    tiles take one half of the row's list each and merge (m, l, O): those
    rows match the oracle and the unsplit launch up to rounding, every other
    row is bitwise the unsplit one. The split rows include lists of 0, 1, 2
    and 3 entries, an invalid entry that empties the first half, and (with a
    work order) an odd number of rows."""
    blk, B = 128, 1
    nb = -(-N // blk)
    rng = np.random.default_rng(N + nh)
    idx = np.full((B, nh, nb, kcap), -1, dtype=np.int32)
    cnt = np.zeros((B, nh, nb), dtype=np.int32)
    for h in range(nh):
        for I in range(nb):
            c = kcap if I < nb - 4 or h < nh - 1 else I - (nb - 4)      # last rows of the last head: 0, 1, 2, 3
            idx[0, h, I, :c] = np.sort(rng.choice(nb, size=c, replace=False))
            cnt[0, h, I] = c
    ref_idx, ref_cnt = idx.copy(), cnt.copy()
    idx[0, nh - 1, nb - 2, 0] = nb + 5          # the 2-entry row: its first half holds only this
    ref_idx[0, nh - 1, nb - 2, :2] = [idx[0, nh - 1, nb - 2, 1], -1]
    ref_cnt[0, nh - 1, nb - 2] = 1
    g = torch.Generator().manual_seed(N)
    q, k, v = (torch.randn((B, nh, N, D), generator=g).to(torch.bfloat16) for _ in range(3))
    s = lib.Shape(B, nh, D, 1, 1, N, blk, 16)
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    order = None
    if with_order:
        order = torch.empty(B * nh * nb, dtype=torch.int32, device="cuda")
        lib.dfs_attn_order(s, ct, kcap, order)
    outs = []
    for split in (True, False):
        o = torch.empty((B, nh, N, D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, nh, N), dtype=torch.float32, device="cuda")
        lib.dfs_sparse_attn_fwd_ex(s, q.cuda(), k.cuda(), v.cuda(), it, ct, kcap, 0.0, o, lse, order=order,
                                   tail_split=split)
        outs.append((o, lse))
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == lib.DFS_FLAG_BAD_KV_INDEX
    # the rows of the split CTAs, from the launch geometry
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    V = B * nh * nb if with_order else 2 * B * nh * ((nb + 1) // 2)
    pairs = (V + 1) // 2
    rem = pairs % sms
    assert 0 < rem and 2 * rem <= sms, "the case must have a split tail"
    split_rows = np.zeros((B * nh, nb), dtype=bool)
    rows = order.cpu().numpy() if with_order else None
    for vr in range(2 * (pairs - rem), V):
        if with_order:
            r = int(rows[vr])
            split_rows[r // nb, r % nb] = True
        else:
            p, e = divmod(vr, 2)
            bh, x = divmod(p, (nb + 1) // 2)
            if 2 * x + e < nb:
                split_rows[bh, 2 * x + e] = True
    assert split_rows[nh - 1, nb - 4:].all()
    tok = np.repeat(split_rows, blk, axis=1)[:, :N].reshape(B, nh, N)
    a, b = (x[0].float().cpu().numpy() for x in outs)
    la, lb = (x[1].cpu().numpy() for x in outs)
    ref, rlse = attention.block_sparse_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                                 ref_idx, ref_cnt, blk)

    def where(mask):
        pos = np.argwhere(mask.reshape(B * nh, N))[:6]
        return [(int(h), int(t) // blk, int(t), float(la.reshape(-1, N)[h, t]), float(lb.reshape(-1, N)[h, t]),
                 float(rlse.reshape(-1, N)[h, t]), int(cnt.reshape(-1, nb)[h, t // blk])) for h, t in pos]

    rf = np.isfinite(rlse)
    assert np.array_equal(rf, np.isfinite(lb)), where(rf != np.isfinite(lb))
    assert np.array_equal(rf, np.isfinite(la)), where(rf != np.isfinite(la))
    assert np.abs(la[rf] - rlse[rf]).max() < 1e-3
    assert_attn_close(a, ref, "tail-split output")
    assert np.array_equal(a[~tok], b[~tok]) and np.array_equal(la[~tok], lb[~tok])
    assert np.abs(la[tok & rf] - lb[tok & rf]).max() < 1e-4
    assert np.abs(a[tok] - b[tok]).max() <= 2 ** -7 * max(1.0, np.abs(b[tok]).max())


def test_binding_rejects_wrong_tensors(lib):
    """The wrappers check device, dtype, contiguity and size against the
    shape before any pointer reaches the library; a rejected call launches
    nothing (the output keeps its contents)."""
    B, nh, D, blk, N = 1, 2, 64, 64, 512
    s = lib.Shape(B, nh, D, 1, 1, N, blk, 16)
    q = torch.zeros((B, nh, N, D), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((B, nh, s.nb, 2), dtype=torch.int32, device="cuda")
    cnt = torch.ones((B, nh, s.nb), dtype=torch.int32, device="cuda")
    op = torch.full((B, nh, N, D), 7.0, dtype=torch.bfloat16, device="cuda")
    bad = [
        dict(q=q[:, :, : N // 2].contiguous()),                   # too small for the shape
        dict(q=q.float()),                                        # wrong dtype
        dict(q=q.transpose(2, 3)),                                # not contiguous
        dict(idx=idx[..., :1].contiguous()),                      # kv_idx shorter than kcap
        dict(cnt=cnt.to(torch.int64)),
        dict(op=op[:, :1].contiguous()),
    ]
    for case in bad:
        a = dict(q=q, idx=idx, cnt=cnt, op=op)
        a.update(case)
        with pytest.raises(lib.DfsError) as e:
            lib.dfs_sparse_attn_fwd(s, a["q"], q, q, a["idx"], a["cnt"], 2, 0.0, a["op"])
        assert e.value.status == lib.DFS_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((op == 7.0).all())


def test_list_length_limit(lib):
    """The two lists of a CTA are staged in shared memory: for D = 128 and
    blk = 128, min(kcap, nb) = 4202 still fits (232,448 bytes) and 4203 is
    rejected with DFS_ERR_UNSUPPORTED before anything is launched. All
    tensors are sized for the shape, so a regression fails the assertion
    rather than touching memory it does not own."""
    D, nb = 128, 4203
    N = nb * 128
    s = lib.Shape(1, 1, D, 1, 1, N, 128, 16)
    q = torch.zeros((1, 1, N, D), dtype=torch.bfloat16, device="cuda")
    cnt = torch.zeros((1, 1, nb), dtype=torch.int32, device="cuda")      # empty lists
    for kcap, ok in ((4202, True), (4203, False)):
        idx = torch.zeros((1, 1, nb, kcap), dtype=torch.int32, device="cuda")
        op = torch.full((1, 1, N, D), 7.0, dtype=torch.bfloat16, device="cuda")
        if ok:
            lib.dfs_sparse_attn_fwd(s, q, q, q, idx, cnt, kcap, 0.0, op)
            torch.cuda.synchronize()
            assert lib.dfs_get_error_flags(clear=True) == 0
            assert bool((op == 0).all())                    # rows with no kept block
        else:
            with pytest.raises(lib.DfsError) as e:
                lib.dfs_sparse_attn_fwd(s, q, q, q, idx, cnt, kcap, 0.0, op)
            assert e.value.status == lib.DFS_ERR_UNSUPPORTED
            torch.cuda.synchronize()
            assert bool((op == 7.0).all())
        del idx, op


def _per_head_order(cnt, kmax):
    """The rows of each head stably sorted by clamped count, largest first;
    heads in order (flat row indices)."""
    c = np.clip(np.asarray(cnt).reshape(-1, np.asarray(cnt).shape[-1]), 0, kmax)
    nb = c.shape[1]
    return np.concatenate([bh * nb + np.argsort(-c[bh], kind="stable") for bh in range(c.shape[0])])


@pytest.mark.parametrize("nb,kcap,nh", [(929, 186, 24), (2000, 2000, 3), (9000, 9000, 1), (300, 5000, 40)])
def test_work_order_is_a_stable_sort(lib, nb, kcap, nh):
    """dfs_attn_order sorts the rows of each head stably by kept count
    (clamped to min(kcap, nb)), largest first, heads in order: rows of equal
    count in ascending order -- for small and large count ranges (fewer
    histogram segments), counts out of range included."""
    rng = np.random.default_rng(nb + kcap)
    kmax = min(kcap, nb)
    cnt = rng.integers(0, kmax + 1, size=(1, nh, nb)).astype(np.int32)
    cnt.reshape(-1)[::97] = kmax + 3            # clamped to kmax
    cnt.reshape(-1)[5::101] = -2                # clamped to 0
    s = lib.Shape(1, nh, 128, 1, 1, nb * 128, 128, 32)
    order = torch.full((nh * nb,), -1, dtype=torch.int32, device="cuda")
    lib.dfs_attn_order(s, torch.from_numpy(cnt).cuda(), kcap, order)
    torch.cuda.synchronize()
    assert np.array_equal(order.cpu().numpy(), _per_head_order(cnt, kmax))


def test_forward_is_reproducible_with_work_order_and_tail_split(lib):
    """Hunyuan-shaped threshold lists (24 heads, 929 blocks, uneven counts up
    to the cap of 186, many rows of equal count): two launches in the work
    order with the default tail split give the same output and LSE bit for
    bit, and so does a work order built again."""
    B, nh, D, blk, N, kcap = 1, 24, 128, 128, 118800, 186
    nb = -(-N // blk)
    rng = np.random.default_rng(7)
    cnt = rng.integers(1, kcap + 1, size=(B, nh, nb)).astype(np.int32)
    idx = np.full((B, nh, nb, kcap), -1, dtype=np.int32)
    for h in range(nh):
        for I in range(nb):
            idx[0, h, I, :cnt[0, h, I]] = np.sort(rng.choice(nb, size=cnt[0, h, I], replace=False))
    s = lib.Shape(B, nh, D, 1, 1, N, blk, 32)
    g = torch.Generator(device="cuda").manual_seed(11)
    qp, kp, vp = (torch.randn((B, nh, N, D), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    res = []
    for _ in range(2):
        order = torch.empty(B * nh * nb, dtype=torch.int32, device="cuda")
        lib.dfs_attn_order(s, ct, kcap, order)
        for _ in range(2):
            o = torch.empty_like(qp)
            lse = torch.empty((B, nh, N), dtype=torch.float32, device="cuda")
            lib.dfs_sparse_attn_fwd_ex(s, qp, kp, vp, it, ct, kcap, 0.0, o, lse, order=order)
            res.append((order, o, lse))
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == 0
    o0 = res[0]
    for r in res[1:]:
        assert torch.equal(r[0], o0[0])
        assert torch.equal(r[1].view(torch.int16), o0[1].view(torch.int16))
        assert torch.equal(r[2].view(torch.int32), o0[2].view(torch.int32))


@pytest.mark.parametrize("fused", [False, True])
def test_bounded_wait_gives_up_and_reports(lib, fused):
    """A wait that gives up (dfs_attn_opts.test_stall_cycles: the MMA warp of
    every CTA waits on a barrier that nothing arrives at) takes the abort
    path: the call returns, DFS_FLAG_WAIT_TIMEOUT is raised, no row with a
    kept block is written (rows with an empty list need no wait and get
    their zero output), and the context stays usable -- the same launch with
    the default settings then matches the oracle. (The CTAs of this small
    launch run split, so both epilogues take the abort path.)"""
    B, nh, D, blk, N, kcap = 1, 2, 128, 128, 1024, 4
    nb = -(-N // blk)
    rng = np.random.default_rng(3)
    idx, cnt = _lists(rng, B, nh, nb, kcap)
    cnt[0, 0, 0] = max(1, cnt[0, 0, 0])
    cnt[0, 1, 3] = 0                            # an empty row
    s = lib.Shape(B, nh, D, 1, 1, N, blk, 16)
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn((B, nh, N, D), generator=g).to(torch.bfloat16) for _ in range(3))
    qp, kp, vp = q.cuda(), k.cuda(), v.cuda()
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    perm = torch.arange(N, dtype=torch.int32, device="cuda").flip(0).contiguous() if fused else None
    sentinel = -12345
    assert lib.dfs_get_error_flags(clear=True) == 0
    o = torch.full((B, nh, N, D), sentinel, dtype=torch.int16, device="cuda").view(torch.bfloat16)
    lse = None if fused else torch.full((B, nh, N), float("nan"), dtype=torch.float32, device="cuda")
    lib.dfs_sparse_attn_fwd_ex(s, qp, kp, vp, it, ct, kcap, 0.0, o, lse, perm=perm, test_stall_cycles=20000)
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == lib.DFS_FLAG_WAIT_TIMEOUT
    # per token row (curve order) of each head: does its block keep anything?
    kept = np.repeat(cnt[0] > 0, blk, axis=1)[:, :N]                     # [nh, N]
    raw = o.view(torch.int16).cpu().numpy()
    rows = raw.reshape(N, nh, D).transpose(1, 0, 2)[:, perm.cpu().numpy()] if fused else raw[0]
    assert (rows[kept] == sentinel).all()
    assert (rows[~kept] == 0).all()
    if lse is not None:
        l = lse[0].cpu().numpy()
        assert np.isnan(l[kept]).all() and np.isneginf(l[~kept]).all()
    # the same launch with the default settings
    lib.dfs_sparse_attn_fwd_ex(s, qp, kp, vp, it, ct, kcap, 0.0, o, lse, perm=perm)
    torch.cuda.synchronize()
    assert lib.dfs_get_error_flags(clear=True) == 0
    ref, _ = attention.block_sparse_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), idx, cnt,
                                              blk)
    got = o.float().cpu().numpy()
    if fused:     # raster o[b, perm[i], h, :] = row i of head h, o viewed as [B, N, nh, D]
        got = got.reshape(B, N, nh, D)[:, perm.long().cpu().numpy()].transpose(0, 2, 1, 3)
    assert_attn_close(got, ref, "after the abort path")
