"""The whole path on the synthetic workloads against the oracle.

* permutation: bit-exact;
* block scores: fp32 against fp64 within the rounding bound;
* masks: bit-exact except entries within 1e-5 of the row's cut-off score
  (and threshold rows whose cumulative mass at the cut is within 1e-5 of
  tau), counted;
* output: max abs <= 2e-2 and relative Frobenius <= 5e-3 against the fp64
  oracle -- on every row for the tiny workload, on a seeded sample of query
  blocks (computed one by one by the oracle) at full size. The sampled
  attention check uses the GPU's own kept lists, so it tests attention
  independently of near-tie mask decisions (those are checked above).
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import attention, hilbert, lvsa, pipeline, radial, schedule, scoring, selection
from tests.parity import assert_attn_close, compare_global_masks, compare_masks

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa(cuda_device):
    import block_sparse_attention_36_b200 as m
    return m


def _layer(bsa, wl, **kw):
    s = bsa.Shape(wl.B, wl.nh, wl.D, wl.T, wl.H, wl.W, wl.blk, wl.sb)
    if wl.mode == "topk":
        return bsa.DfsLayer(s, order=wl.order, mode="topk", k=wl.ratio_count(wl.keep_num), want_lse=True, **kw)
    if wl.mode == "threshold":
        cap = wl.ratio_count(wl.cap_num)
        return bsa.DfsLayer(s, order=wl.order, mode="threshold", cap=cap, tau=wl.tau, want_lse=True, **kw)
    if wl.mode == "lvsa":
        return bsa.DfsLayer(s, order=wl.order, mode="lvsa", lvsa_T_per=wl.lvsa_T_per, lvsa_C=wl.lvsa_C,
                            lvsa_step=wl.lvsa_step, want_lse=True, **kw)
    if wl.mode == "radial":
        return bsa.DfsLayer(s, order=wl.order, mode="radial", radial_w0=wl.radial_w0,
                            radial_lambda=wl.radial_lambda, want_lse=True, **kw)
    if wl.mode == "global":
        return bsa.DfsLayer(s, order=wl.order, mode="global", k=wl.pair_count(wl.keep_num), kcap=s.nb,
                            want_lse=True, **kw)
    raise ValueError(wl.mode)


def _sample_rows(rng, B, nh, nb, n):
    rows = {(0, 0, 0), (0, nh - 1, nb - 1)}   # first block and the ragged last block
    while len(rows) < n:
        rows.add((int(rng.integers(0, B)), int(rng.integers(0, nh)), int(rng.integers(0, nb))))
    return sorted(rows)


def _head(x, b, h, perm):
    """One head of a raster [B, N, nh, D] tensor, reordered, fp64 [1, 1, N, D]."""
    return x[b, perm, h, :].double().numpy()[None, None]


def _check_sampled_attention(layer, qkv, rows):
    perm = torch.from_numpy(layer.perm.cpu().numpy().astype(np.int64))
    idx, cnt = layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy()
    blk, N = layer.shape.blk, layer.shape.N
    got_rows, ref_rows = [], []
    for (b, h) in sorted({(b, h) for (b, h, _) in rows}):
        qp, kp, vp = (_head(x, b, h, perm) for x in qkv)
        mine = [(0, 0, I) for (bb, hh, I) in rows if (bb, hh) == (b, h)]
        ref, _ = attention.block_sparse_attention(qp, kp, vp, idx[b:b + 1, h:h + 1], cnt[b:b + 1, h:h + 1],
                                                  blk, rows=mine)
        op = layer.op[b, h].float().cpu().numpy()
        for (_, _, I) in mine:
            lo, hi = I * blk, min(N, I * blk + blk)
            got_rows.append(op[lo:hi])
            ref_rows.append(ref[0, 0, lo:hi])
    return assert_attn_close(np.concatenate(got_rows), np.concatenate(ref_rows), "sampled rows")


def _oracle_scores(q, k, perm, wl):
    perm = torch.from_numpy(perm.astype(np.int64))
    out = np.empty((wl.B, wl.nh, wl.nb, wl.nb))
    for b in range(wl.B):
        for h in range(wl.nh):
            out[b, h] = scoring.block_scores(_head(q, b, h, perm), _head(k, b, h, perm), wl.blk, wl.sb)[0, 0]
    return out


def test_tiny_workload_end_to_end(bsa):
    wl = synth.WORKLOADS["tiny"]
    qkv = synth.workload_inputs(wl)
    layer = _layer(bsa, wl)
    out = layer.forward(*(x.cuda() for x in (qkv["q"], qkv["k"], qkv["v"]))).float().cpu().numpy()
    torch.cuda.synchronize()
    k = wl.ratio_count(wl.keep_num)
    res = pipeline.run(qkv["q"], qkv["k"], qkv["v"], T=wl.T, H=wl.H, W=wl.W, blk=wl.blk, sb=wl.sb,
                       order=wl.order, mode="topk", k_keep=k, kcap=layer.kcap)
    assert np.array_equal(layer.perm.cpu().numpy(), res["perm"])
    got_scores = layer.scores.cpu().numpy()
    assert np.abs(got_scores - res["scores"]).max() < 1e-4
    cmp = compare_masks(layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy(), res["kv_idx"], res["kv_cnt"],
                        res["scores"], "topk")
    assert cmp["bad_rows"] == 0, cmp
    if cmp["excused_entries"] == 0:
        assert_attn_close(out, res["out"], "tiny output")
    # with the GPU's lists the oracle output must match on every row
    full = attention.block_sparse_attention(res["qp"], res["kp"], res["vp"], layer.kv_idx.cpu().numpy(),
                                            layer.kv_cnt.cpu().numpy(), wl.blk)[0]
    assert_attn_close(out, hilbert.unpermute_tokens(full, res["perm"]), "tiny output, GPU lists")


@pytest.mark.parametrize("name", ["wan_1p3b_layer", "hunyuan_layer", "lvsa_long_video", "wan_1p3b_global",
                                  "wan_1p3b_radial"])
def test_full_size_workload(bsa, name):
    wl = synth.WORKLOADS[name]
    qkv = synth.workload_inputs(wl)
    layer = _layer(bsa, wl)
    layer.forward(*(x.cuda() for x in (qkv["q"], qkv["k"], qkv["v"])))
    torch.cuda.synchronize()
    assert bsa.dfsattn.dfs_get_error_flags(clear=True) == 0
    operm, _ = hilbert.make_perm(wl.order, wl.T, wl.H, wl.W)
    assert np.array_equal(layer.perm.cpu().numpy(), operm)
    if wl.mode == "lvsa":
        m = lvsa.block_mask(wl.T, wl.H * wl.W, wl.blk, wl.lvsa_T_per, wl.lvsa_C, wl.lvsa_step)
        oi, oc = selection.mask_to_lists(np.broadcast_to(m, (wl.B, wl.nh) + m.shape), layer.kcap)
        assert np.array_equal(layer.kv_cnt.cpu().numpy(), oc)
        gi = layer.kv_idx.cpu().numpy()
        for idx in np.ndindex(oc.shape):
            assert np.array_equal(gi[idx][:oc[idx]], oi[idx][:oc[idx]])
    elif wl.mode == "radial":
        rows = [0, 5, 77, 128, 191, wl.nb - 1]
        m = radial.block_mask(wl.T, wl.H * wl.W, wl.blk, wl.radial_w0, radial.w_far_of(wl.radial_lambda, wl.radial_w0),
                              rows=rows)
        gi, gc = layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy()
        for b in range(wl.B):
            for h in range(wl.nh):
                for r, I in enumerate(rows):
                    assert np.array_equal(gi[b, h, I, :gc[b, h, I]], np.flatnonzero(m[r]))
    else:
        ref_scores = _oracle_scores(qkv["q"], qkv["k"], operm, wl)
        got_scores = layer.scores.cpu().numpy()
        assert np.abs(got_scores - ref_scores).max() < 2e-4
        if wl.mode == "topk":
            oi, oc = selection.select(ref_scores, "topk", k=wl.ratio_count(wl.keep_num), kcap=layer.kcap)
            cmp = compare_masks(layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy(), oi, oc, ref_scores, "topk")
        elif wl.mode == "global":
            K = wl.pair_count(wl.keep_num)
            oi, oc = selection.select_global(ref_scores, K, kcap=layer.kcap)
            cmp = compare_global_masks(layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy(), oi, oc, ref_scores, K)
        else:
            cap = wl.ratio_count(wl.cap_num)
            oi, oc = selection.select(ref_scores, "threshold", tau=wl.tau, cap=cap, kcap=layer.kcap)
            cmp = compare_masks(layer.kv_idx.cpu().numpy(), layer.kv_cnt.cpu().numpy(), oi, oc, ref_scores,
                                "threshold", tau=wl.tau, cap=cap)
        print(name, "mask comparison", cmp)
        assert cmp["bad_rows"] == 0, cmp
    rng = np.random.default_rng(0)
    rows = _sample_rows(rng, wl.B, wl.nh, wl.nb, 12)
    _check_sampled_attention(layer, (qkv["q"], qkv["k"], qkv["v"]), rows)
    # the unpermuted output is the permuted one scattered back
    out = layer.out.cpu().view(torch.int16).numpy()
    back = hilbert.unpermute_tokens(layer.op.cpu().view(torch.int16).numpy(), operm)
    assert np.array_equal(out, back)


def test_schedule_workload_steps(bsa):
    """Adaptive budget with mask caching: masks change only at refresh steps,
    with the budget of that step; attention is recomputed every step."""
    wl = synth.WORKLOADS["wan_schedule_50"]
    s = bsa.Shape(wl.B, wl.nh, wl.D, wl.T, wl.H, wl.W, wl.blk, wl.sb)
    kmax = schedule.budget(0, s.nb)
    layer = bsa.DfsLayer(s, order=wl.order, mode="topk", k=kmax, kcap=kmax, want_lse=True)
    v = synth.field_qkv(wl.T, wl.H, wl.W, wl.nh, wl.D, which=("v",))["v"]
    vd = v.cuda()
    prev_idx = None
    rng = np.random.default_rng(1)
    for step in (0, 3, 5, 45, 49):
        qk = synth.schedule_qk(wl.T, wl.H, wl.W, wl.nh, wl.D, step)
        refresh = schedule.is_refresh(step)
        if refresh:
            layer.set_budget(k=schedule.budget(step, s.nb))
        layer.forward(qk["q"].cuda(), qk["k"].cuda(), vd, refresh_mask=refresh)
        torch.cuda.synchronize()
        cnt = layer.kv_cnt.cpu().numpy()
        assert (cnt == schedule.budget(step, s.nb)).all()
        idx = layer.kv_idx.cpu().numpy()
        if not refresh:
            assert np.array_equal(idx, prev_idx)
        prev_idx = idx.copy()
        rows = _sample_rows(rng, wl.B, wl.nh, s.nb, 6)
        _check_sampled_attention(layer, (qk["q"], qk["k"], v), rows)


def test_graph_replay_matches_eager(bsa):
    """A whole step captured in a CUDA graph gives the eager result."""
    wl = synth.WORKLOADS["tiny"]
    qkv = synth.workload_inputs(wl)
    q, k, v = (qkv[n].cuda() for n in ("q", "k", "v"))
    layer = _layer(bsa, wl)
    eager = layer.forward(q, k, v).clone()
    graph = layer.capture_graph(q, k, v)
    layer.out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(layer.out, eager)


def test_pipelined_host_steps_match_eager(bsa):
    """DfsLayer.run_host_steps (copies of neighbouring steps overlapping the
    kernels on three streams) gives, for every step, the bytes the eager
    forward gives for that step's inputs."""
    wl = synth.WORKLOADS["tiny"]
    sets = [synth.workload_inputs(wl, seed=sd) for sd in (0, 1, 2)]
    host = [tuple(x[n].pin_memory() for n in ("q", "k", "v")) for x in sets]
    order = [0, 1, 2, 0, 2, 1, 1]
    layer = _layer(bsa, wl)
    outs = [torch.empty_like(host[0][0]).pin_memory() for _ in order]
    layer.run_host_steps([host[i] for i in order], outs)
    torch.cuda.synchronize()
    ref = _layer(bsa, wl)
    for i, o in zip(order, outs):
        want = ref.forward(*(t.cuda() for t in host[i])).cpu()
        assert torch.equal(o.view(torch.int16), want.view(torch.int16))
