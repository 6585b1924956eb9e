"""One DFSAttn attention layer on the GPU: buffers plus the five library calls.

DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology items 1-3: reorder tokens along the 3D Hilbert
curve, score blocks hierarchically, select key blocks (the mask may be
cached across denoising steps and refreshed at a fixed interval), attend
over the kept blocks every step, restore the token order.

This class only allocates device buffers (torch) and calls the C entry
points in order; all arithmetic happens in libdfsattn's kernels.
"""
from __future__ import annotations

import math

import torch

from . import dfsattn as lib


# selection modes whose mask needs no block scores
STATIC_MODES = ("lvsa", "radial")


class DfsLayer:
    def __init__(self, shape: lib.Shape, order="hilbert3d", mode="topk", k=0, cap=0, tau=0.0,
                 lvsa_T_per=8, lvsa_C=21, lvsa_step=0, kcap=None, scale=0.0, device="cuda",
                 want_lse=False, frame_exact=False, radial_w0=0, radial_lambda=0.0):
        self.shape = shape
        self.order = order
        self.mode = mode
        # LVSA only: drop the pairs of kept blocks whose key frame is outside
        # A(t); frames must stay contiguous, so the order must be raster.
        if frame_exact and (mode != "lvsa" or order != "raster"):
            raise ValueError("frame_exact needs mode='lvsa' and order='raster'")
        self.frame_exact = bool(frame_exact)
        self.params = lib.select_params(mode, k=k, cap=cap, tau=tau, lvsa_T_per=lvsa_T_per, lvsa_C=lvsa_C,
                                        lvsa_step=lvsa_step, radial_w0=radial_w0, radial_lambda=radial_lambda)
        s = shape
        if kcap is None:
            kcap = {"topk": max(1, min(k, s.nb)), "threshold": max(1, min(cap, s.nb)),
                    "global": max(1, min(k, s.nb))}.get(mode, s.nb)
        self.kcap = int(kcap)
        self.scale = float(scale) if scale and scale > 0 else 1.0 / math.sqrt(s.D)
        dev = torch.device(device)
        bf = torch.bfloat16
        self.perm = torch.empty(s.N, dtype=torch.int32, device=dev)
        self.inv = torch.empty(s.N, dtype=torch.int32, device=dev)
        self.qp = torch.empty((s.B, s.nh, s.N, s.D), dtype=bf, device=dev)
        self.kp = torch.empty_like(self.qp)
        self.vp = torch.empty_like(self.qp)
        self.op = torch.empty_like(self.qp)
        self.out = torch.empty((s.B, s.N, s.nh, s.D), dtype=bf, device=dev)
        self.lse = torch.empty((s.B, s.nh, s.N), dtype=torch.float32, device=dev) if want_lse else None
        self.kv_idx = torch.full((s.B, s.nh, s.nb, self.kcap), -1, dtype=torch.int32, device=dev)
        self.kv_cnt = torch.zeros((s.B, s.nh, s.nb), dtype=torch.int32, device=dev)
        if mode not in STATIC_MODES:
            self.scores = torch.empty((s.B, s.nh, s.nb, s.nb), dtype=torch.float32, device=dev)
            nbytes = lib.dfs_workspace_bytes(s, lib.DFS_WS_BLOCK_SCORE)
            self.ws = torch.empty(max(1, nbytes), dtype=torch.uint8, device=dev)
        else:
            self.scores = None
            self.ws = None
        # longest rows first for list lengths that vary from row to row
        self.work_order = (torch.empty(s.B * s.nh * s.nb, dtype=torch.int32, device=dev)
                           if mode in ("threshold", "global") else None)
        self._index_built = False
        self._bwd = None
        self._pipe = None
        # the fused reorder + pooling needs nh * D / 8 <= 512
        self.fused_pool = s.nh * s.D // 8 <= 512

    def set_budget(self, k=None, cap=None, tau=None, lvsa_step=None):
        p = self.params
        if k is not None:
            if k > self.kcap and self.mode == "topk":
                raise ValueError("k exceeds kcap")
            p.k = int(k)
        if cap is not None:
            p.cap = int(cap)
        if tau is not None:
            p.tau = float(tau)
        if lvsa_step is not None:
            p.lvsa_step = int(lvsa_step)

    def permute(self, q, k, v, stream=None):
        lib.dfs_hilbert_perm(self.shape, self.order, self.perm, self.inv, not self._index_built, q, k, v,
                             None if q is None else self.qp, None if k is None else self.kp,
                             None if v is None else self.vp, stream)
        self._index_built = True

    def build_mask(self, stream=None):
        if self.mode not in STATIC_MODES:
            lib.dfs_block_score(self.shape, self.qp, self.kp, self.scale, self.scores, self.ws, stream)
        lib.dfs_select_mask(self.shape, self.scores, self.params, self.kv_idx, self.kv_cnt, self.kcap, stream)
        self._build_order(stream)

    def _build_order(self, stream=None):
        if self.work_order is not None:
            lib.dfs_attn_order(self.shape, self.kv_cnt, self.kcap, self.work_order, stream)

    def attend(self, stream=None, out=None):
        """Attention and the inverse reorder into ``out`` (default: the
        layer's). Without an LSE (inference) the reorder is fused into the
        attention epilogue; with one, O is kept in curve order in ``op`` for
        the backward and scattered by a separate kernel."""
        dst = self.out if out is None else out
        if self.lse is None and not self.frame_exact:
            self.attention(stream, out=dst, perm=self.perm)
            return
        self.attention(stream)
        lib.dfs_unperm(self.shape, self.perm, self.op, dst, stream)

    def attention(self, stream=None, out=None, perm=None):
        """The attention kernel alone: into ``op`` (curve order), or with
        ``perm`` straight into the raster tensor ``out``. Rows of uneven list
        lengths (threshold, global) run in the layer's work order."""
        if self.frame_exact:
            lib.dfs_sparse_attn_lvsa_fwd(self.shape, self.qp, self.kp, self.vp, self.kv_idx, self.kv_cnt,
                                         self.kcap, self.scale, self.params, self.op, self.lse, stream)
        else:
            lib.dfs_sparse_attn_fwd_ex(self.shape, self.qp, self.kp, self.vp, self.kv_idx, self.kv_cnt, self.kcap,
                                       self.scale, self.op if out is None else out, self.lse, perm=perm,
                                       order=self.work_order, stream=stream)

    def permute_pooled(self, q, k, v, stream=None):
        """Reorder Q, K, V and pool Q, K into the score workspace in one pass."""
        lib.dfs_hilbert_perm_pooled(self.shape, self.order, self.perm, self.inv, not self._index_built, q, k, v,
                                    self.qp, self.kp, self.vp, self.ws, stream)
        self._index_built = True

    def prepare(self, q, k, v, refresh_mask=True, stream=None):
        """Reorder Q, K, V and, if asked, rebuild the mask. When the mask is
        rebuilt from scores, the reorder also pools Q and K (one pass over the
        data) and scoring starts from those means."""
        if refresh_mask and self.mode not in STATIC_MODES and self.fused_pool:
            self.permute_pooled(q, k, v, stream)
            lib.dfs_block_score_pooled(self.shape, self.scale, self.scores, self.ws, stream)
            lib.dfs_select_mask(self.shape, self.scores, self.params, self.kv_idx, self.kv_cnt, self.kcap, stream)
            self._build_order(stream)
        else:
            self.permute(q, k, v, stream)
            if refresh_mask:
                self.build_mask(stream)

    def forward(self, q, k, v, refresh_mask=True, stream=None, out=None):
        """q, k, v: bf16 [B, N, nh, D] on the device (raster order). Returns
        the output buffer (``out`` if given, else the layer's own)."""
        self.prepare(q, k, v, refresh_mask, stream)
        self.attend(stream, out)
        return self.out if out is None else out

    def run_host_steps(self, host_inputs, host_outputs, refresh_mask=True, before_step=None):
        """Runs one step per (q, k, v) of ``host_inputs`` (pinned host bf16
        [B, N, nh, D]) and copies each result into the matching pinned host
        tensor of ``host_outputs``. Steps are pipelined over three streams:
        the host-to-device copy of step i+1 and the device-to-host copy of
        step i-1 overlap the kernels of step i (two device input sets and two
        output buffers, ordered by events). ``refresh_mask`` is one flag for
        every step or a sequence with one flag per step (a denoising loop
        with a cached mask); ``before_step(i)``, if given, is called before
        step i is enqueued (e.g. to set that step's budget). Enqueues the
        work after the current stream's pending work and makes the current
        stream wait for all of it; returns without synchronising."""
        n = len(host_inputs)
        if len(host_outputs) != n:
            raise ValueError("one host output per step")
        refresh = [bool(refresh_mask)] * n if isinstance(refresh_mask, bool) else [bool(r) for r in refresh_mask]
        if len(refresh) != n:
            raise ValueError("one refresh flag per step")
        s = self.shape
        dev = self.qp.device
        if self._pipe is None:
            shape = (s.B, s.N, s.nh, s.D)
            self._pipe = {
                "inp": [[torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(3)] for _ in range(2)],
                "out": [torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(2)],
                "streams": [torch.cuda.Stream(device=dev) for _ in range(3)],
            }
        p = self._pipe
        s_in, s_cmp, s_out = p["streams"]
        start = torch.cuda.current_stream()
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(start)
        cmp_done = [None, None]
        out_done = [None, None]
        for i in range(n):
            b = i & 1
            inp, dout = p["inp"][b], p["out"][b]
            with torch.cuda.stream(s_in):
                if cmp_done[b] is not None:
                    s_in.wait_event(cmp_done[b])       # step i-2 has read this input set
                for d, h in zip(inp, host_inputs[i]):
                    d.copy_(h, non_blocking=True)
                in_ready = torch.cuda.Event()
                in_ready.record(s_in)
            s_cmp.wait_event(in_ready)
            if out_done[b] is not None:
                s_cmp.wait_event(out_done[b])          # step i-2's result has left this buffer
            if before_step is not None:
                before_step(i)
            self.forward(inp[0], inp[1], inp[2], refresh[i], stream=s_cmp, out=dout)
            cmp_done[b] = torch.cuda.Event()
            cmp_done[b].record(s_cmp)
            s_out.wait_event(cmp_done[b])
            with torch.cuda.stream(s_out):
                host_outputs[i].copy_(dout, non_blocking=True)
                out_done[b] = torch.cuda.Event()
                out_done[b].record(s_out)
        for st in (s_in, s_cmp, s_out):
            start.wait_stream(st)

    def capture_graph(self, q, k, v, refresh_mask=True, warmup=2):
        """Record one whole step (prepare + attend) into a CUDA graph over the
        given, fixed input buffers; replay it with ``graph.replay()``. Warm-up
        steps run first (eagerly, on a side stream), so one-time set-up such
        as building the curve index and raising kernel attributes happens
        outside the capture."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(warmup):
                self.forward(q, k, v, refresh_mask)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.forward(q, k, v, refresh_mask)
        return graph

    def backward(self, dout, stream=None):
        """Gradients of the last forward: dout is dL/dout, bf16 [B, N, nh, D]
        in raster order (the layout of ``out``). Returns (dq, dk, dv) in the
        same raster layout. Needs ``want_lse=True`` (the backward reads the
        forward's log-sum-exp) and blk = 128; frame-exact LVSA has no
        backward."""
        if self.lse is None:
            raise ValueError("backward needs the forward's lse: build the layer with want_lse=True")
        if self.frame_exact:
            raise ValueError("frame-exact LVSA attention has no backward")
        s = self.shape
        if self._bwd is None:
            dev = self.qp.device
            nbytes = lib.dfs_workspace_bytes(s, lib.DFS_WS_ATTN_BWD)
            self._bwd = {
                "ws": torch.empty(max(1, nbytes), dtype=torch.uint8, device=dev),
                "dop": torch.empty_like(self.qp), "dqp": torch.empty_like(self.qp),
                "dkp": torch.empty_like(self.qp), "dvp": torch.empty_like(self.qp),
            }
        b = self._bwd
        lib.dfs_hilbert_perm(s, self.order, self.perm, self.inv, 0, dout, None, None, b["dop"], None, None, stream)
        lib.dfs_sparse_attn_bwd(s, self.qp, self.kp, self.vp, self.op, b["dop"], self.lse, self.kv_idx,
                                self.kv_cnt, self.kcap, self.scale, b["dqp"], b["dkp"], b["dvp"], b["ws"], stream)
        outs = []
        for name in ("dqp", "dkp", "dvp"):
            g = torch.empty((s.B, s.N, s.nh, s.D), dtype=torch.bfloat16, device=self.qp.device)
            lib.dfs_unperm(s, self.perm, b[name], g, stream)
            outs.append(g)
        return tuple(outs)

    def kept_pairs(self):
        """Valid (query, key) token pairs the kept blocks cover (for FLOP counts)."""
        s = self.shape
        rows_q = torch.full((s.nb,), s.blk, dtype=torch.int64)
        rows_q[-1] = s.N - (s.nb - 1) * s.blk
        idx = self.kv_idx.cpu().long()
        cnt = self.kv_cnt.cpu().long()
        pos = torch.arange(self.kcap).view(1, 1, 1, -1)
        valid = pos < cnt.unsqueeze(-1)
        keys = torch.where(idx == s.nb - 1, rows_q[-1], torch.full_like(idx, s.blk))
        keys = torch.where(valid, keys, torch.zeros_like(keys)).sum(-1)   # [B, nh, nb]
        return int((keys * rows_q.view(1, 1, -1)).sum())
