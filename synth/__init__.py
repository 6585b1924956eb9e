"""Seeded synthetic inputs for the DFSAttn hot path.

This module only draws inputs. It holds none of the method's arithmetic, so
both the fp64 oracle (through the tests) and the CUDA path (through the tests
and the benchmark) can be fed from it without sharing any computation.

What the inputs stand in for
----------------------------
The pages evaluate on video DiT activations (HunyuanVideo, Wan2.1) that are
not available here. These fields stand in for one attention layer's Q/K/V:
a smooth spatiotemporal field (a few low-frequency Fourier modes over the
T x H x W grid) plus iid noise, normalised to unit variance, rounded to bf16.
Smoothness is what gives the Hilbert reorder and the hierarchical scoring
something to find; the noise keeps the scores from being degenerate.

Recipe (per tensor X in (Q, K, V), per head h; batch b)
-------------------------------------------------------
rng = numpy Generator(PCG64(SeedSequence([seed, b, tensor_id, h])))
  1. 8 mode frequencies: indices drawn uniformly from the 124 integer triples
     (kt, kh, kw) in {-2..2}^3 without (0, 0, 0), in that lexicographic order.
  2. 8 phases phi ~ U[0, 2*pi).
  3. 8 amplitude vectors a_m ~ N(0, I_D)  (shape [8, D], row-major draw).
  4. noise ~ N(0, 1) of shape [N, D] (float32 draw), scaled by 0.3.
field[t,h,w,:] = sum_m a_m * cos(2*pi*(kt*t/T + kh*h/H + kw*w/W) + phi_m)
x = field + 0.3 * noise, then x = (x - mean(x)) / std(x) over all N*D
values of that (tensor, head), then bf16 with round-to-nearest-even.
Layout: [B, N, nh, D] with raster token order n = (t*H + h)*W + w.

Denoising-schedule inputs (the 50-step workload): the per-head field of Q
and K is drawn once as above without noise and normalised to unit variance;
step s adds sigma_s * eps_s with sigma_s = 1.0 - 0.95*s/49 and eps_s drawn
from SeedSequence([seed, b, tensor_id, h, 1000 + s]); no renormalisation.
V is the plain recipe above and does not change with s.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field as dc_field
from typing import Optional

import numpy as np
import torch

TENSOR_IDS = {"q": 0, "k": 1, "v": 2}
N_MODES = 8
NOISE_STD = 0.3


def _freq_table():
    out = []
    for kt in range(-2, 3):
        for kh in range(-2, 3):
            for kw in range(-2, 3):
                if (kt, kh, kw) != (0, 0, 0):
                    out.append((kt, kh, kw))
    return np.array(out, dtype=np.int64)


_FREQS = _freq_table()  # 124 x 3


def _phase_grid(T, H, W):
    t = np.arange(T, dtype=np.float64)[:, None, None]
    h = np.arange(H, dtype=np.float64)[None, :, None]
    w = np.arange(W, dtype=np.float64)[None, None, :]
    return t / T, h / H, w / W


def _smooth_field(rng, T, H, W, D):
    """Draw one head's smooth field, [N, D] float64 (steps 1-3 of the recipe)."""
    idx = rng.integers(0, len(_FREQS), size=N_MODES)
    phi = rng.uniform(0.0, 2.0 * math.pi, size=N_MODES)
    amp = rng.standard_normal((N_MODES, D))
    ft, fh, fw = _phase_grid(T, H, W)
    basis = np.empty((T * H * W, N_MODES), dtype=np.float64)
    for m in range(N_MODES):
        kt, kh, kw = _FREQS[idx[m]]
        arg = 2.0 * math.pi * (kt * ft + kh * fh + kw * fw) + phi[m]
        basis[:, m] = np.cos(arg).reshape(-1)
    return basis @ amp


def _normalise(x):
    mu = x.mean(dtype=np.float64)
    sd = x.std(dtype=np.float64)
    return (x - mu) / sd


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def _one_head(seed, b, tid, h, T, H, W, D):
    rng = np.random.default_rng([seed, b, tid, h])
    f = _smooth_field(rng, T, H, W, D)
    noise = rng.standard_normal((T * H * W, D), dtype=np.float32)
    x = f + NOISE_STD * noise.astype(np.float64)
    return _to_bf16(_normalise(x))


def field_qkv(T, H, W, nh, D, B=1, seed=0, threads=8, which=("q", "k", "v")):
    """Q, K, V as bf16 CPU tensors [B, N, nh, D] (raster order)."""
    N = T * H * W
    out = {}
    jobs = [(b, name, h) for name in which for b in range(B) for h in range(nh)]
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        res = list(ex.map(lambda j: _one_head(seed, j[0], TENSOR_IDS[j[1]], j[2], T, H, W, D), jobs))
    for name in which:
        out[name] = torch.empty((B, N, nh, D), dtype=torch.bfloat16)
    for (b, name, h), x in zip(jobs, res):
        out[name][b, :, h, :] = x
    return out


def schedule_sigma(s: int, n_steps: int = 50) -> float:
    return 1.0 - 0.95 * s / (n_steps - 1)


def _schedule_head(seed, b, tid, h, T, H, W, D, s, n_steps):
    rng = np.random.default_rng([seed, b, tid, h])
    f = _normalise(_smooth_field(rng, T, H, W, D))
    rs = np.random.default_rng([seed, b, tid, h, 1000 + s])
    eps = rs.standard_normal((T * H * W, D), dtype=np.float32).astype(np.float64)
    return _to_bf16(f + schedule_sigma(s, n_steps) * eps)


def schedule_qk(T, H, W, nh, D, s, B=1, seed=0, n_steps=50, threads=8):
    """Q, K of denoising step s for the adaptive-schedule workload."""
    N = T * H * W
    out = {n: torch.empty((B, N, nh, D), dtype=torch.bfloat16) for n in ("q", "k")}
    jobs = [(b, name, h) for name in ("q", "k") for b in range(B) for h in range(nh)]
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        res = list(ex.map(lambda j: _schedule_head(seed, j[0], TENSOR_IDS[j[1]], j[2], T, H, W, D, s, n_steps), jobs))
    for (b, name, h), x in zip(jobs, res):
        out[name][b, :, h, :] = x
    return out


def schedule_fields(T, H, W, nh, D, B=1, seed=0, threads=8):
    """The noise-free, normalised Q and K fields of the schedule workload,
    fp32 CPU tensors [B, N, nh, D] (the part of the recipe shared by all steps)."""
    N = T * H * W
    out = {n: torch.empty((B, N, nh, D), dtype=torch.float32) for n in ("q", "k")}

    def one(j):
        b, name, h = j
        rng = np.random.default_rng([seed, b, TENSOR_IDS[name], h])
        return torch.from_numpy(_normalise(_smooth_field(rng, T, H, W, D)).astype(np.float32))

    jobs = [(b, name, h) for name in ("q", "k") for b in range(B) for h in range(nh)]
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        res = list(ex.map(one, jobs))
    for (b, name, h), x in zip(jobs, res):
        out[name][b, :, h, :] = x
    return out


def schedule_qk_device(fields, s, seed=0, n_steps=50):
    """Q, K of step s for timing runs: the same recipe as schedule_qk, but
    eps_s is drawn on the fields' device by torch's generator seeded with
    (seed, s) -- the same distribution, a different realisation. Parity tests
    use schedule_qk."""
    dev = fields["q"].device
    g = torch.Generator(device=dev)
    g.manual_seed(1_000_003 * (seed + 1) + s)
    sig = schedule_sigma(s, n_steps)
    return {n: (fields[n] + sig * torch.randn(fields[n].shape, generator=g, device=dev)).to(torch.bfloat16)
            for n in ("q", "k")}


def segmented_qk(T, H, W, nh, D, B=1, seed=0, region_tokens=256, share=0.55, t_scale=4.0):
    """Q, K with several semantic centroids per block (bf16 CPU [B, N, nh, D]).

    Stand-in for frames of several objects: the grid is cut into Voronoi
    regions around R = N / region_tokens random sites (time distances
    weighted by t_scale); region r has a centroid c_r ~ N(0, I) shared by Q
    and K of the head, so a query attends mostly to keys of its own region,
    and blocks that straddle a region boundary hold several unrelated
    centroids. Per token: x = sqrt(share) * g_r * c_r + sqrt(1 - share) * z,
    z ~ N(0, I) drawn separately for Q and K, g_r ~ U[0.5, 1.5] a per-region
    strength. Draws: sites and strengths from SeedSequence([seed, b, 7, h]),
    centroids (R x D) from [seed, b, 8, h], z from [seed, b, tensor_id, h, 99].
    """
    N = T * H * W
    t, h, w = (a.reshape(-1).astype(np.float64) for a in np.meshgrid(np.arange(T), np.arange(H), np.arange(W),
                                                                      indexing="ij"))
    out = {n: torch.empty((B, N, nh, D), dtype=torch.bfloat16) for n in ("q", "k")}
    R = max(2, N // region_tokens)
    for b in range(B):
        for hd in range(nh):
            rs = np.random.default_rng([seed, b, 7, hd])
            sites = np.stack([rs.uniform(0, T, R), rs.uniform(0, H, R), rs.uniform(0, W, R)], 1)
            gain = rs.uniform(0.5, 1.5, R)
            cent = np.random.default_rng([seed, b, 8, hd]).standard_normal((R, D))
            label = np.empty(N, dtype=np.int64)
            for lo in range(0, N, 8192):
                sl = slice(lo, min(N, lo + 8192))
                d2 = ((t_scale * (t[sl, None] - sites[None, :, 0])) ** 2 + (h[sl, None] - sites[None, :, 1]) ** 2
                      + (w[sl, None] - sites[None, :, 2]) ** 2)
                label[sl] = d2.argmin(1)
            base = math.sqrt(share) * gain[label, None] * cent[label]
            for name in ("q", "k"):
                z = np.random.default_rng([seed, b, TENSOR_IDS[name], hd, 99]).standard_normal((N, D))
                out[name][b, :, hd, :] = _to_bf16(base + math.sqrt(1.0 - share) * z)
    return out


# ---------------------------------------------------------------------------
# The five workloads (shapes, block sizes and selection settings).
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    nh: int
    D: int
    T: int
    H: int
    W: int
    blk: int
    sb: int
    order: str            # "hilbert3d" or "raster"
    mode: str             # "topk", "threshold", "lvsa", "schedule", "global", "radial"
    keep_num: int = 0     # keep ratio numerator / 100 (top-k)
    tau: float = 0.0
    cap_num: int = 0      # cap ratio numerator / 100 (threshold)
    lvsa_T_per: int = 0
    lvsa_C: int = 0
    lvsa_step: int = 0
    n_steps: int = 0
    refresh: int = 0
    frame_exact: bool = False   # LVSA: mask pairs outside A(t) inside kept blocks
    radial_w0: int = 0          # log-radial mask: window at frame distance 0 (tokens)
    radial_lambda: float = 0.0  # log-radial mask: long-range floor, as a fraction of w0

    @property
    def N(self):
        return self.T * self.H * self.W

    @property
    def nb(self):
        return -(-self.N // self.blk)

    @property
    def nsb(self):
        return -(-self.N // self.sb)

    def ratio_count(self, num: int) -> int:
        """ceil(num/100 * nb) in exact integer arithmetic."""
        return -(-(num * self.nb) // 100)

    def pair_count(self, num: int) -> int:
        """ceil(num/100 * nb^2): block pairs kept per head by global selection."""
        return -(-(num * self.nb * self.nb) // 100)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, 8, 16, 16, 64, 16, "hilbert3d", "topk", keep_num=25),
    "wan_1p3b_layer": Workload("wan_1p3b_layer", 1, 12, 128, 21, 30, 52, 128, 32, "hilbert3d", "topk", keep_num=15),
    "wan_schedule_50": Workload("wan_schedule_50", 1, 12, 128, 21, 30, 52, 128, 32, "hilbert3d", "schedule",
                                n_steps=50, refresh=5),
    "lvsa_long_video": Workload("lvsa_long_video", 1, 12, 128, 63, 30, 52, 128, 32, "raster", "lvsa",
                                lvsa_T_per=8, lvsa_C=21, lvsa_step=0),
    "lvsa_long_video_exact": Workload("lvsa_long_video_exact", 1, 12, 128, 63, 30, 52, 128, 32, "raster", "lvsa",
                                      lvsa_T_per=8, lvsa_C=21, lvsa_step=0, frame_exact=True),
    "wan_1p3b_radial": Workload("wan_1p3b_radial", 1, 12, 128, 21, 30, 52, 128, 32, "raster", "radial",
                                radial_w0=1560, radial_lambda=0.125),
    "wan_1p3b_global": Workload("wan_1p3b_global", 1, 12, 128, 21, 30, 52, 128, 32, "hilbert3d", "global",
                                keep_num=15),
    "hunyuan_layer": Workload("hunyuan_layer", 1, 24, 128, 33, 45, 80, 128, 32, "hilbert3d", "threshold",
                              tau=0.9, cap_num=20),
}


def workload_inputs(wl: Workload, seed: int = 0, threads: int = 8):
    return field_qkv(wl.T, wl.H, wl.W, wl.nh, wl.D, B=wl.B, seed=seed, threads=threads)
