"""Comparison rules shared by the GPU parity tests.

Masks: bit-exact except entries whose fp64 oracle score lies within EPS of
the row's cut-off score (the last kept score), and, for threshold rows,
whole rows whose oracle cumulative mass at m-1 or m lies within EPS of tau;
both kinds are excused and counted.
Attention output: max abs error <= 2e-2 and relative Frobenius error
<= 5e-3 against the fp64 oracle.
"""
from __future__ import annotations

import numpy as np

from oracle import selection

EPS = 1e-5
ATOL_MAX = 2e-2
RTOL_FRO = 5e-3


def row_sets(idx, cnt):
    return [set(idx[i, :c].tolist()) for i, c in enumerate(cnt)]


def compare_masks(g_idx, g_cnt, o_idx, o_cnt, o_scores, mode, tau=None, cap=None, eps=EPS):
    """Returns dict(bad_rows, excused_entries, excused_rows, rows).

    g_* / o_*: kept lists of the GPU and the oracle, any leading shape.
    o_scores: fp64 oracle scores with the same leading shape + [nb].
    """
    nb = o_scores.shape[-1]
    g_idx = np.asarray(g_idx).reshape(-1, g_idx.shape[-1])
    o_idx = np.asarray(o_idx).reshape(-1, o_idx.shape[-1])
    g_cnt = np.asarray(g_cnt).reshape(-1)
    o_cnt = np.asarray(o_cnt).reshape(-1)
    s64 = np.asarray(o_scores, dtype=np.float64).reshape(-1, nb)
    out = {"bad_rows": 0, "excused_entries": 0, "excused_rows": 0, "rows": len(g_cnt), "bad_examples": []}
    for r in range(len(g_cnt)):
        gi = g_idx[r, :g_cnt[r]].tolist()
        oi = o_idx[r, :o_cnt[r]].tolist()
        if gi == oi:
            continue
        if mode == "threshold":
            m, csum = selection.threshold_count(s64[r].astype(np.float32), tau, nb)
            near = abs(csum[m - 1] - tau) <= eps or (m - 2 >= 0 and abs(csum[m - 2] - tau) <= eps)
            if near:
                out["excused_rows"] += 1
                continue
        cut = s64[r, oi].min() if oi else np.inf
        diff = set(gi) ^ set(oi)
        if len(gi) == len(oi) and all(abs(s64[r, j] - cut) <= eps for j in diff):
            out["excused_entries"] += len(diff)
            continue
        out["bad_rows"] += 1
        if len(out["bad_examples"]) < 5:
            out["bad_examples"].append((r, sorted(set(gi) - set(oi))[:5], sorted(set(oi) - set(gi))[:5]))
    return out


def attn_errors(got, ref):
    g = np.asarray(got, dtype=np.float64)
    f = np.asarray(ref, dtype=np.float64)
    d = g - f
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    den = float(np.linalg.norm(f))
    rel = float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def assert_attn_close(got, ref, what=""):
    mx, rel = attn_errors(got, ref)
    assert mx <= ATOL_MAX and rel <= RTOL_FRO, f"{what}: max abs {mx:.3e}, rel fro {rel:.3e}"
    return mx, rel


def compare_global_masks(g_idx, g_cnt, o_idx, o_cnt, o_scores, K, eps=EPS):
    """Global selection: per head the kept pair sets must match except pairs
    whose fp64 oracle score lies within eps of the head's cut-off score (the
    K-th best), which are excused and counted."""
    from oracle import selection as sel
    nb = o_scores.shape[-1]
    gm = sel.lists_to_mask(np.asarray(g_idx), np.asarray(g_cnt), nb)
    om = sel.lists_to_mask(np.asarray(o_idx), np.asarray(o_cnt), nb)
    s64 = np.asarray(o_scores, dtype=np.float64)
    out = {"bad_rows": 0, "excused_entries": 0, "heads": gm.shape[0] * gm.shape[1], "bad_examples": []}
    for b in range(gm.shape[0]):
        for h in range(gm.shape[1]):
            diff = gm[b, h] ^ om[b, h]
            if not diff.any():
                continue
            cut = s64[b, h][om[b, h]].min() if om[b, h].any() else np.inf
            bad = diff & (np.abs(s64[b, h] - cut) > eps)
            if gm[b, h].sum() == om[b, h].sum() and not bad.any():
                out["excused_entries"] += int(diff.sum())
            else:
                out["bad_rows"] += int(bad.any(axis=1).sum())
                out["bad_examples"].append((b, h, int(diff.sum())))
    return out
