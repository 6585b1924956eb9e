"""Benchmark of the DFSAttn hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = the whole path over one layer's synthetic Q/K/V already in HBM:
Hilbert gather of Q, K, V -> pooled sub-block scoring -> top-k / threshold /
LVSA selection -> block-sparse attention -> inverse gather. The curve index
is built once per grid shape before timing (it depends only on the shape).
Metric: kept-block TFLOP/s of the whole step (4 * D FLOPs per kept, valid
query-key pair), with ms per step; the roofline object reports the
attention kernel alone against the measured bf16 tensor peak.

Multi-GPU: one process per GPU (torchrun); every rank runs its own
independent layer (weak scaling, no collective on the data path); the time
is the maximum over ranks.

--impl reference times the fp64 CPU oracle (the only reference this
method has) on the host cores over a bounded sample of the same workload.

--backward times the gradient pass instead: after one forward, each step is
DfsLayer.backward (reorder dO, the block-sparse attention backward, scatter
dQ, dK, dV back); metric: kept-block TFLOP/s at 10 * D FLOPs per kept pair
(the five products of the backward; the implementation executes seven).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "block-sparse attn ms/call & kept-block TFLOP/s vs B200 bf16 TC peak"
# fused gather + pooling (1 launch), score, select, attention with the scatter fused in;
# LVSA / log-radial: 3 gathers, select, attention (frame-exact LVSA: + a separate scatter)
# (threshold and global add the work-order sort)
KERNELS_PER_STEP = {"topk": 4, "threshold": 5, "global": 5, "lvsa": 5, "radial": 5}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per attention launch from one ncu capture of
# that workload, valid only for the attention sources
# whose hash is recorded with it; reported as null once they change.
ATTN_TRAFFIC = {"wan_1p3b_layer": (298_117_376 + 81_682_176, "66a54f472c7b2e82"),
                "hunyuan_layer": (4_672_438_528 + 755_917_056, "66a54f472c7b2e82")}
ATTN_SOURCES = ("attn.cu", "sm100_ptx.cuh", "exp2_poly.cuh", "common.cuh", "lvsa.cuh", "tmap.cuh")


# dram read + write of one backward call (its prep, list and gradient
# launches), from a one-pass ncu capture of these sources
BWD_TRAFFIC = {"wan_1p3b_layer": (1_007_642_880 + 262_761_728, "b85a7531aeaa6e3b"),
               "hunyuan_layer": (19_747_298_560 + 2_204_054_528, "b85a7531aeaa6e3b")}
BWD_SOURCES = ("attn_bwd.cu", "sm100_ptx.cuh", "common.cuh", "tmap.cuh")


def sources_hash(files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "block_sparse_attention_36_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def bwd_traffic(workload):
    entry = BWD_TRAFFIC.get(workload)
    if entry is None or entry[1] != sources_hash(BWD_SOURCES):
        return None
    return entry[0]


def attn_sources_hash():
    import hashlib
    h = hashlib.sha256()
    for f in ATTN_SOURCES:
        with open(os.path.join(ROOT, "block_sparse_attention_36_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def attn_traffic(workload):
    entry = ATTN_TRAFFIC.get(workload)
    if entry is None or entry[1] != attn_sources_hash():
        return None
    return entry[0]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def sustained(peaks, achieved):
    """The same kernel against the sustained bf16 figure (a matmul loop held
    for seconds under the power cap), for kernels that run long enough to
    reach the cap; `peak` and `frac` stay on the burst figure."""
    p = peaks.get("bf16_tflops_sustained")
    if not p:
        return {}
    return {"peak_sustained": float(p), "frac_sustained": round(achieved / float(p), 4)}


def workload_config(wl, k, cap):
    sel = {"topk": f"top-k {k}/{wl.nb}", "threshold": f"threshold tau={wl.tau} cap {cap}/{wl.nb}",
           "global": f"global top {k} of {wl.nb}x{wl.nb} pairs per head",
           "lvsa": f"LVSA T_per={wl.lvsa_T_per} C={wl.lvsa_C} step {wl.lvsa_step}"
                   + (" frame-exact" if wl.frame_exact else ""),
           "radial": f"log-radial w0={wl.radial_w0} lambda={wl.radial_lambda}"}[wl.mode]
    return (f"{wl.name}: B={wl.B} nh={wl.nh} D={wl.D} grid {wl.T}x{wl.H}x{wl.W} (N={wl.N}) "
            f"{wl.order} order, blk {wl.blk}, sb {wl.sb}, {sel}")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self._t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def make_layer(bsa, wl, want_lse=False):
    s = bsa.Shape(wl.B, wl.nh, wl.D, wl.T, wl.H, wl.W, wl.blk, wl.sb)
    k = cap = 0
    kw = {"order": wl.order, "want_lse": want_lse}
    if wl.mode == "topk":
        k = wl.ratio_count(wl.keep_num)
        layer = bsa.DfsLayer(s, mode="topk", k=k, **kw)
    elif wl.mode == "threshold":
        cap = wl.ratio_count(wl.cap_num)
        layer = bsa.DfsLayer(s, mode="threshold", cap=cap, tau=wl.tau, **kw)
    elif wl.mode == "global":
        k = wl.pair_count(wl.keep_num)
        layer = bsa.DfsLayer(s, mode="global", k=k, kcap=s.nb, **kw)
    elif wl.mode == "radial":
        layer = bsa.DfsLayer(s, mode="radial", radial_w0=wl.radial_w0, radial_lambda=wl.radial_lambda, **kw)
    else:
        layer = bsa.DfsLayer(s, mode="lvsa", lvsa_T_per=wl.lvsa_T_per, lvsa_C=wl.lvsa_C,
                             lvsa_step=wl.lvsa_step, frame_exact=wl.frame_exact, **kw)
    return layer, k, cap


def run_ours(args):
    import torch
    import synth
    import block_sparse_attention_36_b200 as bsa
    from block_sparse_attention_36_b200 import dfsattn

    rank, world, local = dist_setup(args.gpus)
    wl = synth.WORKLOADS[args.workload]
    if wl.mode == "schedule":
        return run_schedule(args, wl, rank, world, local)
    qkv = synth.workload_inputs(wl, seed=args.seed + rank)
    q, k, v = (qkv[n].cuda() for n in ("q", "k", "v"))
    layer, kk, cap = make_layer(bsa, wl)
    stream = torch.cuda.current_stream()

    # warm-up (also builds the curve index once)
    for _ in range(args.warmup):
        layer.forward(q, k, v)
    torch.cuda.synchronize()
    kept_pairs = layer.kept_pairs()
    flops_step = 4.0 * wl.D * kept_pairs * 1.0
    dense_flops = 4.0 * wl.D * wl.N * wl.N * wl.nh * wl.B
    assert dfsattn.dfs_get_error_flags(clear=True) == 0

    # timed region: K whole steps; attention kernel bracketed by its own events
    ev_attn = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    graph = layer.capture_graph(q, k, v) if args.graph else None
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        if graph is not None:
            graph.replay()
            continue
        layer.prepare(q, k, v)
        ev_attn[i][0].record(stream)
        layer.attend()          # attention with the inverse reorder fused into its epilogue
        ev_attn[i][1].record(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    ms_total = start.elapsed_time(stop)
    if graph is not None:
        # attention-kernel time from eager launches (events cannot sit inside the graph replay)
        for i in range(args.steps):
            ev_attn[i][0].record(stream)
            layer.attend()
            ev_attn[i][1].record(stream)
        torch.cuda.synchronize()
        del graph
    attn_ms = [a.elapsed_time(b) for a, b in ev_attn]
    ms_total_max = max_over_ranks(ms_total, world)
    flops_all = sum_over_ranks(flops_step * args.steps, world)
    attn_avg = statistics.mean(attn_ms)

    # end to end through the public API from pinned host buffers: every step
    # copies its Q, K, V in and its output back. Pipelined
    # (DfsLayer.run_host_steps: copies of neighbouring steps overlap the
    # kernels) and, for reference, one step after the other on one stream.
    hq, hk, hv = (qkv[n].pin_memory() for n in ("q", "k", "v"))
    hos = [torch.empty_like(hq).pin_memory() for _ in range(2)]
    # as many steps as the device-timed loop: the first step's copy in and
    # the last step's kernels and copy out are not overlapped with anything
    e2e_steps = max(4, args.steps)
    layer.run_host_steps([(hq, hk, hv)] * 2, hos)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    layer.run_host_steps([(hq, hk, hv)] * e2e_steps, [hos[i & 1] for i in range(e2e_steps)])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    barrier(world)
    e0.record(stream)
    for _ in range(e2e_steps):
        q.copy_(hq, non_blocking=True); k.copy_(hk, non_blocking=True); v.copy_(hv, non_blocking=True)
        layer.forward(q, k, v)
        hos[0].copy_(layer.out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    serial_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    e2e_flops = sum_over_ranks(flops_step, world)
    assert dfsattn.dfs_get_error_flags(clear=True) == 0

    if rank == 0:
        peaks, src = load_peaks()
        achieved = flops_step / (attn_avg * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops"])
        ms_step = ms_total_max / args.steps
        value = flops_all / (ms_total_max * 1e-3) / 1e12
        traffic = attn_traffic(wl.name)
        line = {
            "metric": METRIC,
            "value": round(value, 3),
            "unit": "TFLOP/s (kept-block, whole step)",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4),
            "attn_ms_per_call": round(attn_avg, 4),
            "dense_equiv_tflops": round(dense_flops / (ms_step * 1e-3) / 1e12, 3),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded smooth Fourier field + noise, bf16)",
            "config": {"workload": workload_config(wl, kk, cap), "kept_pairs_per_step": kept_pairs,
                       "kept_fraction": round(kept_pairs / (wl.N * wl.N * wl.nh * wl.B), 4),
                       "l2": "inputs larger than L2 (3 x %.1f MB of Q/K/V per step)" % (wl.N * wl.nh * wl.D * 2 / 1e6),
                       "parallelism": f"replicas x{world} (independent layer per GPU)",
                       "launch": "CUDA graph replay" if args.graph else "eager launches"},
            "roofline": {"kernel": "attn_fwd_kernel (inverse reorder fused into the epilogue)", "bound": "tensor", "achieved": round(achieved, 2),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                         "peak_source": f"{src} bf16 burst", "traffic": traffic,
                         **sustained(peaks, achieved)},
            "e2e": {"value": round(e2e_flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s (kept-block, whole step)",
                    "ms_per_step": round(e2e_ms, 3),
                    "h2d_bytes_per_step": int(3 * hq.numel() * hq.element_size()),
                    "d2h_bytes_per_step": int(hq.numel() * hq.element_size()),
                    "api": "DfsLayer.run_host_steps (copies of neighbouring steps overlap the kernels)",
                    "serial_ms_per_step": round(serial_ms, 3)},
            "gpu_launches": (KERNELS_PER_STEP[wl.mode] + (1 if wl.frame_exact else 0)) * args.steps,
            "clocks": clk,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(wl, qkv, kk, cap, budget_s=args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# dO reorder, prep, mask bits, transpose, dQ pass, dK/dV pass, three scatters
BWD_KERNELS_PER_STEP = 8


def run_backward(args):
    import torch
    import synth
    import block_sparse_attention_36_b200 as bsa
    from block_sparse_attention_36_b200 import dfsattn

    rank, world, local = dist_setup(args.gpus)
    wl = synth.WORKLOADS[args.workload]
    qkv = synth.workload_inputs(wl, seed=args.seed + rank)
    q, k, v = (qkv[n].cuda() for n in ("q", "k", "v"))
    layer, kk, cap = make_layer(bsa, wl, want_lse=True)
    layer.forward(q, k, v)
    g = torch.Generator().manual_seed(args.seed + 1000 + rank)
    dout_h = (torch.randn((wl.B, wl.N, wl.nh, wl.D), generator=g) * 0.5).to(torch.bfloat16)
    dout = dout_h.cuda()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        layer.backward(dout)
    torch.cuda.synchronize()
    assert dfsattn.dfs_get_error_flags(clear=True) == 0
    kept_pairs = layer.kept_pairs()
    flops_step = 10.0 * wl.D * kept_pairs
    b = layer._bwd
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    s = layer.shape
    for i in range(args.steps):
        dfsattn.dfs_hilbert_perm(s, layer.order, layer.perm, layer.inv, 0, dout, None, None, b["dop"], None, None)
        ev[i][0].record(stream)
        dfsattn.dfs_sparse_attn_bwd(s, layer.qp, layer.kp, layer.vp, layer.op, b["dop"], layer.lse, layer.kv_idx,
                                    layer.kv_cnt, layer.kcap, layer.scale, b["dqp"], b["dkp"], b["dvp"], b["ws"])
        ev[i][1].record(stream)
        for name in ("dqp", "dkp", "dvp"):
            dfsattn.dfs_unperm(s, layer.perm, b[name], layer.out)
    stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop() if clocks else None
    ms_total_max = max_over_ranks(start.elapsed_time(stop), world)
    bwd_ms = statistics.mean(a.elapsed_time(c) for a, c in ev)
    flops_all = sum_over_ranks(flops_step * args.steps, world)

    # end to end: dO from pinned host memory in, the three gradients out
    dh = dout_h.pin_memory()
    hg = [torch.empty_like(dout_h).pin_memory() for _ in range(3)]
    e2e_steps = max(3, args.steps)
    for _ in range(2):
        dout.copy_(dh, non_blocking=True)
        grads = layer.backward(dout)
        for h, d in zip(hg, grads):
            h.copy_(d, non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        dout.copy_(dh, non_blocking=True)
        grads = layer.backward(dout)
        for h, d in zip(hg, grads):
            h.copy_(d, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    assert dfsattn.dfs_get_error_flags(clear=True) == 0
    if rank == 0:
        peaks, src = load_peaks()
        peak = float(peaks["bf16_tflops"])
        achieved = flops_step / (bwd_ms * 1e-3) / 1e12
        ms_step = ms_total_max / args.steps
        line = {
            "metric": "block-sparse attention backward: kept-block TFLOP/s (10*D FLOP per kept pair) vs B200 bf16 TC peak",
            "value": round(flops_all / (ms_total_max * 1e-3) / 1e12, 3),
            "unit": "TFLOP/s (kept-block backward, whole step)",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4), "bwd_ms_per_call": round(bwd_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded smooth Fourier field + noise, bf16; dO Gaussian)",
            "config": {"workload": workload_config(wl, kk, cap) + ", backward", "kept_pairs_per_step": kept_pairs,
                       "executed_flop_per_pair": 14 * wl.D,
                       "l2": "inputs larger than L2 (Q, K, V, O, dO, dQ, dK, dV: 8 x %.1f MB)"
                             % (wl.N * wl.nh * wl.D * 2 / 1e6),
                       "parallelism": f"replicas x{world} (independent layer per GPU)"},
            "roofline": {"kernel": "dfs_sparse_attn_bwd (prep, mask bits, transpose, dQ pass, dK/dV pass)",
                         "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "peak_source": f"{src} bf16 burst",
                         "traffic": bwd_traffic(wl.name), **sustained(peaks, achieved)},
            "e2e": {"value": round(sum_over_ranks(flops_step, world) / (e2e_ms * 1e-3) / 1e12, 3),
                    "unit": "TFLOP/s (kept-block backward, whole step)", "ms_per_step": round(e2e_ms, 3),
                    "h2d_bytes_per_step": int(dh.numel() * dh.element_size()),
                    "d2h_bytes_per_step": int(3 * dh.numel() * dh.element_size())},
            "gpu_launches": BWD_KERNELS_PER_STEP * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def schedule_config(wl):
    return (f"{wl.name}: B={wl.B} nh={wl.nh} D={wl.D} grid {wl.T}x{wl.H}x{wl.W} (N={wl.N}) {wl.order} order, "
            f"blk {wl.blk}, sb {wl.sb}, {wl.n_steps} steps, top-k 103 -> 32 of {wl.nb}, "
            f"mask refresh every {wl.refresh} steps, attention every step")


def run_schedule(args, wl, rank, world, local):
    """The 50-step denoising loop: Q/K change every step (V is fixed), the
    keep budget falls from 40 % to 10 %, masks are rebuilt every 5 steps and
    attention runs every step. Reports the amortised time per step and the
    kept-block TFLOP/s over all 50 steps; the roofline object reports the
    attention kernel over the loop, e2e the loop through the public API from
    pinned host buffers."""
    import torch
    import synth
    import block_sparse_attention_36_b200 as bsa
    from block_sparse_attention_36_b200 import dfsattn
    from block_sparse_attention_36_b200 import schedule

    s = bsa.Shape(wl.B, wl.nh, wl.D, wl.T, wl.H, wl.W, wl.blk, wl.sb)
    ks = [schedule.keep_budget(st, s.nb, wl.n_steps, wl.refresh) for st in range(wl.n_steps)]
    refresh = [schedule.is_refresh(st, wl.refresh) for st in range(wl.n_steps)]
    layer = bsa.DfsLayer(s, order=wl.order, mode="topk", k=ks[0], kcap=ks[0])
    fields = {n: t.cuda() for n, t in synth.schedule_fields(wl.T, wl.H, wl.W, wl.nh, wl.D, seed=args.seed + rank).items()}
    v = synth.field_qkv(wl.T, wl.H, wl.W, wl.nh, wl.D, seed=args.seed + rank, which=("v",))["v"].cuda()
    steps_qk = [synth.schedule_qk_device(fields, st, seed=args.seed + rank, n_steps=wl.n_steps)
                for st in range(wl.n_steps)]
    del fields
    stream = torch.cuda.current_stream()
    def run_loop(count_flops=False, events=None):
        flops = []
        for st in range(wl.n_steps):
            if refresh[st]:
                layer.set_budget(k=ks[st])
            layer.prepare(steps_qk[st]["q"], steps_qk[st]["k"], v, refresh_mask=refresh[st])
            if events is not None:
                events[st][0].record(stream)
            layer.attend()
            if events is not None:
                events[st][1].record(stream)
            if count_flops:
                torch.cuda.synchronize()
                flops.append(4.0 * wl.D * layer.kept_pairs())
        return flops

    flops_steps = run_loop(count_flops=True)       # also the first warm-up pass
    flops_loop = sum(flops_steps)
    for _ in range(max(0, args.warmup - 1)):
        run_loop()
    torch.cuda.synchronize()
    assert dfsattn.dfs_get_error_flags(clear=True) == 0
    reps = max(1, min(args.steps, 5))
    ev_attn = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(wl.n_steps)] for _ in range(reps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for r in range(reps):
        run_loop(events=ev_attn[r])
    e1.record(stream)
    torch.cuda.synchronize()
    attn_ms = [[a.elapsed_time(b) for a, b in evs] for evs in ev_attn]
    barrier(world)
    clk = clocks.stop() if clocks else None
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    ms_step = ms / (reps * wl.n_steps)
    flops_all = sum_over_ranks(flops_loop * reps, world)
    attn_total_ms = sum(sum(x) for x in attn_ms)

    # end to end through the public API: every step copies its Q, K, V in from
    # pinned host memory and its output back (DfsLayer.run_host_steps with the
    # loop's refresh flags and budgets). Host inputs: the first few steps' Q/K
    # (the kept counts, hence the work, depend only on the budgets).
    n_host = 3
    hv = v.cpu().pin_memory()
    host_sets = [(steps_qk[i]["q"].cpu().pin_memory(), steps_qk[i]["k"].cpu().pin_memory(), hv) for i in range(n_host)]
    hos = [torch.empty_like(hv).pin_memory() for _ in range(2)]
    e2e_inputs = [host_sets[i % n_host] for i in range(wl.n_steps)]
    e2e_outs = [hos[i & 1] for i in range(wl.n_steps)]
    set_k = lambda i: layer.set_budget(k=ks[i]) if refresh[i] else None
    layer.run_host_steps(e2e_inputs, e2e_outs, refresh_mask=refresh, before_step=set_k)
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    layer.run_host_steps(e2e_inputs, e2e_outs, refresh_mask=refresh, before_step=set_k)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / wl.n_steps
    assert dfsattn.dfs_get_error_flags(clear=True) == 0
    if rank == 0:
        peaks, src = load_peaks()
        peak = float(peaks["bf16_tflops"])
        achieved = flops_loop * reps / (attn_total_ms * 1e-3) / 1e12
        line = {"metric": METRIC, "value": round(flops_all / (ms * 1e-3) / 1e12, 3),
                "unit": "TFLOP/s (kept-block, amortised over the 50-step loop)", "n_gpus": world,
                "steps": reps * wl.n_steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
                "attn_ms_per_call": round(attn_total_ms / (reps * wl.n_steps), 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded fields; per-step noise drawn on the device)",
                "config": {"workload": schedule_config(wl), "kept_pairs_per_loop": int(flops_loop / (4.0 * wl.D)),
                           "l2": "inputs larger than L2 (3 x %.1f MB of Q/K/V per step)" % (wl.N * wl.nh * wl.D * 2 / 1e6),
                           "parallelism": f"replicas x{world} (independent layer per GPU)", "launch": "eager launches"},
                "roofline": {"kernel": "attn_fwd_kernel (inverse reorder fused into the epilogue), over the 50 steps",
                             "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                             "frac": round(achieved / peak, 4), "peak_source": f"{src} bf16 burst",
                             "traffic": None, **sustained(peaks, achieved)},
                "e2e": {"value": round(sum_over_ranks(flops_loop, world) / (e2e_ms * wl.n_steps * 1e-3) / 1e12, 3),
                        "unit": "TFLOP/s (kept-block, amortised over the 50-step loop)",
                        "ms_per_step": round(e2e_ms, 3),
                        "h2d_bytes_per_step": int(3 * hv.numel() * hv.element_size()),
                        "d2h_bytes_per_step": int(hv.numel() * hv.element_size()),
                        "api": "DfsLayer.run_host_steps (per-step refresh flags and budgets; copies overlap the kernels)"},
                # per step: 3 gathers (or the fused gather + pooling, score and select) and the attention
                "gpu_launches": 4 * wl.n_steps * reps, "clocks": clk}
        if not args.no_cpu_baseline and world == 1:
            qkv = {"q": steps_qk[0]["q"].cpu(), "k": steps_qk[0]["k"].cpu(), "v": hv}
            wl_sel = synth.Workload(**{**wl.__dict__, "mode": "topk"})
            line["cpu_baseline"] = cpu_baseline(wl_sel, qkv, ks[0], 0, budget_s=args.cpu_seconds,
                                                schedule_ks=(ks, refresh))
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def oracle_masks(wl, qkv, k, cap, heads, permt):
    """Curve-ordered fp64 heads and the oracle's kept lists for them."""
    from oracle import lvsa, radial, scoring, selection
    per_head = []
    m = None
    for h in heads:
        qp, kp, vp = (qkv[n][0, permt, h, :].double().numpy()[None, None] for n in ("q", "k", "v"))
        if wl.mode == "lvsa":
            m = lvsa.block_mask(wl.T, wl.H * wl.W, wl.blk, wl.lvsa_T_per, wl.lvsa_C, wl.lvsa_step) if m is None else m
            idx, cnt = selection.mask_to_lists(m[None, None])
        elif wl.mode == "radial":
            m = (radial.block_mask(wl.T, wl.H * wl.W, wl.blk, wl.radial_w0,
                                   radial.w_far_of(wl.radial_lambda, wl.radial_w0)) if m is None else m)
            idx, cnt = selection.mask_to_lists(m[None, None])
        elif wl.mode == "global":
            sc = scoring.block_scores(qp, kp, wl.blk, wl.sb)
            idx, cnt = selection.select_global(sc, k)
        else:
            sc = scoring.block_scores(qp, kp, wl.blk, wl.sb)
            idx, cnt = selection.select(sc, "threshold" if wl.mode == "threshold" else "topk", k=k, tau=wl.tau,
                                        cap=cap, kcap=wl.nb)
        per_head.append((qp, kp, vp, idx, cnt))
    return per_head


def cpu_baseline(wl, qkv, k, cap, budget_s=20.0, schedule_ks=None):
    """Times the oracle on the host cores over a bounded sample of the
    workload and scales it to a whole step: a sampled estimate, not a run of
    the whole layer.

    Sample: the curve index; scoring and selection head by head (numpy's own
    threads) until about 40 % of the budget is spent, the remaining heads
    scaled from their mean; then fp64 attention of random query blocks of the
    scored heads (at most 4), dealt over all host cores by a pool of spawned
    processes (oracle.parallel), batch after batch until the budget is
    spent; the wall time per query block is scaled to every row of the layer.
    ``schedule_ks`` (one k per denoising step, refresh flags) scales the
    sample, taken at the first step's budget, to the whole loop: masks at the
    refresh steps, attention every step in proportion to its k.
    Returns the estimated whole-step throughput in the bench's unit."""
    import torch
    from oracle import attention, hilbert, parallel
    wall0 = time.perf_counter()
    t0 = time.perf_counter()
    perm, _ = hilbert.make_perm(wl.order, wl.T, wl.H, wl.W)
    permt = torch.from_numpy(perm.astype(np.int64))
    t_perm = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    per_head = []
    t_mask = 0.0
    t0 = time.perf_counter()
    for h in range(wl.nh):
        t1 = time.perf_counter()
        per_head += oracle_masks(wl, qkv, k, cap, [h], permt)
        t_mask += time.perf_counter() - t1
        if time.perf_counter() - t0 > budget_s * 0.4 and h < wl.nh - 1:
            break
    heads_done = len(per_head)
    t_mask = t_mask / heads_done * wl.nh * wl.B
    att_heads = per_head[:4]
    stack = lambda i: np.concatenate([ph[i] for ph in att_heads], axis=1)
    frame = None
    if wl.frame_exact:
        from oracle import lvsa
        frame = (lvsa.frame_allowed(wl.T, wl.lvsa_T_per, wl.lvsa_C, wl.lvsa_step), wl.H * wl.W)
    rows_total = wl.nb * wl.nh * wl.B
    n_rows = kept = 0
    t_attn = 0.0
    with parallel.RowPool(stack(0), stack(1), stack(2), stack(3), stack(4), wl.blk, frame=frame) as pool:
        cores = pool.workers
        # start every worker process (spawned on demand, one per pending task): not timed
        pool.run([(0, 0, I % wl.nb) for I in range(cores)], blocks_per_task=1)
        deadline = time.perf_counter() + max(2.0, budget_s - (time.perf_counter() - t0))
        batch = 4 * cores
        while True:
            rows = sorted({(0, int(rng.integers(0, len(att_heads))), int(rng.integers(0, wl.nb)))
                           for _ in range(batch)})
            t1 = time.perf_counter()
            pool.run(rows)
            dt = time.perf_counter() - t1
            t_attn += dt
            n_rows += len(rows)
            for (_, h, I) in rows:
                idx, cnt = att_heads[h][3], att_heads[h][4]
                rows_q = min(wl.blk, wl.N - I * wl.blk)
                js = idx[0, 0, I, :int(cnt[0, 0, I])]
                kept += rows_q * int(sum(min(wl.blk, wl.N - j * wl.blk) for j in js))
            left = deadline - time.perf_counter()
            if left < 1.5 * dt:
                break
            batch = max(4 * cores, min(32 * cores, int(batch * left / max(dt, 1e-3) / 2)))
    t_attn_full = t_attn / n_rows * rows_total
    kept_full = kept / n_rows * rows_total
    # the curve index is built once per grid shape (the GPU path builds it
    # before timing too); it is reported, not counted in a step
    if schedule_ks is None:
        t_step = t_mask + t_attn_full
        flops = 4.0 * wl.D * kept_full
        unit = "TFLOP/s (kept-block, whole step)"
        what = "one step"
    else:
        ks, refresh = schedule_ks
        k0 = ks[0]
        t_step = (sum(t_mask for r in refresh if r) + sum(t_attn_full * kk / k0 for kk in ks)) / len(ks)
        flops = sum(4.0 * wl.D * kept_full * kk / k0 for kk in ks) / len(ks)
        unit = "TFLOP/s (kept-block, amortised over the 50-step loop)"
        what = f"the {len(ks)}-step loop (sample at k = {k0}, attention scaled by k, masks at {sum(refresh)} refreshes)"
    return {"value": round(flops / t_step / 1e12, 6), "unit": unit, "cores": cores, "kind": "oracle",
            "sampled": True, "ms_per_step": round(t_step * 1e3, 1),
            "wall_s": round(time.perf_counter() - wall0, 2),
            "curve_index_s": round(t_perm, 2),
            "sample": (f"estimate of {what} (the curve index, built once per grid, not counted): gather, scoring+selection on {heads_done}/{wl.nh} heads "
                       f"(numpy threads; rest scaled); fp64 attention of {n_rows} randomly drawn query blocks (the layer has "
                       f"{rows_total}) over {cores} worker processes, wall time scaled to every row")}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import synth
    wl = synth.WORKLOADS[args.workload]
    sched = None
    if wl.mode == "schedule":
        from block_sparse_attention_36_b200 import schedule as hs
        ks = [hs.keep_budget(st, wl.nb, wl.n_steps, wl.refresh) for st in range(wl.n_steps)]
        sched = (ks, [hs.is_refresh(st, wl.refresh) for st in range(wl.n_steps)])
        qkv = dict(synth.schedule_qk(wl.T, wl.H, wl.W, wl.nh, wl.D, 0, seed=args.seed))
        qkv["v"] = synth.field_qkv(wl.T, wl.H, wl.W, wl.nh, wl.D, seed=args.seed, which=("v",))["v"]
        wl_sel = synth.Workload(**{**wl.__dict__, "mode": "topk"})
        k, cap = ks[0], 0
    else:
        qkv = synth.workload_inputs(wl, seed=args.seed)
        wl_sel = wl
        k = (wl.ratio_count(wl.keep_num) if wl.mode == "topk" else
             wl.pair_count(wl.keep_num) if wl.mode == "global" else 0)
        cap = wl.ratio_count(wl.cap_num) if wl.mode == "threshold" else 0
    # seconds of oracle work per timed estimate (warm-up estimates a quarter
    # of it): 2 to 20 s so that the whole run stays within a few minutes, and
    # never more than --cpu-seconds
    budget = max(min(2.0, args.cpu_seconds), min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(wl_sel, qkv, k, cap, budget_s=budget / 4, schedule_ks=sched)
    t0 = time.perf_counter()
    vals = [cpu_baseline(wl_sel, qkv, k, cap, budget_s=budget, schedule_ks=sched) for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    ms = statistics.mean(v["ms_per_step"] for v in vals)
    val = statistics.mean(v["value"] for v in vals)
    unit = vals[0]["unit"]
    cfg = schedule_config(wl) if sched else workload_config(wl, k, cap)
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "sampled": True,
            "sampling": (f"each of the {args.steps} timed steps is one sampled estimate of a whole step "
                         f"(ms_per_step is the estimated whole-step time); the {args.steps} estimates took "
                         f"{wall:.1f} s of wall time"),
            "config": {"workload": cfg, "parallelism": "host cores, rank 0 only"},
            "cpu_baseline": {"value": round(val, 6), "unit": unit, "cores": vals[0]["cores"], "kind": "oracle",
                             "sampled": True, "sample": vals[0]["sample"]},
            "e2e": {"value": round(val, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="hunyuan_layer")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true", help="replay each step as a captured CUDA graph")
    ap.add_argument("--backward", action="store_true", help="time the gradient pass (DfsLayer.backward)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.backward:
        run_backward(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
