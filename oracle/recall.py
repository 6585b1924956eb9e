"""Attention recall of a block mask (diagnostic, fp64; not a parity gate).

DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
Generation, Methodology (the method is built around a lower bound on
attention recall) and Results (ablations: the 3D Hilbert order beats raster
scans and 2-D Hilbert curves; smaller sub-blocks score better). The pages give no formula
for recall; here it is read as the share of each query's dense softmax mass
that falls on the keys its kept blocks cover, averaged over queries.

Run as a script to compare token orders and scoring granularities on a
synthetic workload at the same keep budget:

    python -m oracle.recall --workload wan_1p3b_layer --queries 256

Pinned by closed forms (tests/test_oracle_attention.py): every block kept
gives 1, none kept gives 0, and a one-block mask gives the kept softmax mass
computed by brute force. There is no GPU counterpart to compare with: the
diagnostic only ranks orders and scoring granularities, and the pages print
no recall values to compare its numbers with.
"""
from __future__ import annotations

import argparse
import math

import numpy as np

from . import hilbert, scoring, selection


def recall(q, k, perm, kv_idx, kv_cnt, blk, queries, scale=None):
    """Mean kept softmax mass over the sampled (b, h, raster query) triples.

    q, k: fp64 [B, N, nh, D] raster; perm: curve order; kv_idx/kv_cnt: lists
    in curve order [B, nh, nb, kcap] / [B, nh, nb].
    """
    B, N, nh, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(N, dtype=perm.dtype)
    out = []
    for (b, h, n) in queries:
        s = (k[b, :, h, :] @ q[b, n, h, :]) * scale          # logits to every key (raster)
        p = np.exp(s - s.max())
        p /= p.sum()
        I = int(inv[n]) // blk
        c = int(kv_cnt[b, h, I])
        pos = np.concatenate([np.arange(J * blk, min(N, J * blk + blk)) for J in kv_idx[b, h, I, :c]]) \
            if c else np.zeros(0, dtype=np.int64)
        out.append(float(p[perm[pos]].sum()))
    return float(np.mean(out))


def variant_recall(q, k, T, H, W, blk, sb, order, k_keep, queries):
    perm, _ = hilbert.make_perm(order, T, H, W, blk)
    qp = hilbert.permute_tokens(q, perm)
    kp = hilbert.permute_tokens(k, perm)
    s = scoring.block_scores(qp, kp, blk, sb)
    idx, cnt = selection.select(s, "topk", k=k_keep)
    return recall(q, k, perm, idx, cnt, blk, queries)


def main():
    import synth   # seeded inputs (no method arithmetic)

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="tiny")
    ap.add_argument("--queries", type=int, default=256, help="sampled queries per head")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--input", default="field", choices=["field", "segmented"],
                    help="smooth fields (the workloads' inputs) or segmented fields with several centroids per block")
    a = ap.parse_args()
    wl = synth.WORKLOADS[a.workload]
    if a.input == "field":
        qkv = synth.field_qkv(wl.T, wl.H, wl.W, wl.nh, wl.D, seed=a.seed, which=("q", "k"))
    else:
        qkv = synth.segmented_qk(wl.T, wl.H, wl.W, wl.nh, wl.D, seed=a.seed)
    q = qkv["q"].double().numpy()
    k = qkv["k"].double().numpy()
    rng = np.random.default_rng(a.seed)
    queries = [(0, h, int(n)) for h in range(wl.nh) for n in rng.integers(0, wl.N, size=a.queries)]
    k_keep = selection.ratio_count(wl.keep_num or 15, 100, wl.nb)
    print(f"workload {wl.name}: N={wl.N}, nb={wl.nb}, keep {k_keep}/{wl.nb}, {len(queries)} sampled queries")
    print("| order | sub-block | recall |\n|---|---|---|")
    for order in ("raster", "tile2d", "tile3d", "hilbert2d", "hilbert3d"):
        for sb in (wl.blk, wl.sb):
            r = variant_recall(q, k, wl.T, wl.H, wl.W, wl.blk, sb, order, k_keep, queries)
            print(f"| {order} | {sb}{' (coarse)' if sb == wl.blk else ''} | {r:.4f} |", flush=True)


if __name__ == "__main__":
    main()
