// Frame sets of LVSA (LVSA: Training-Free Sparse Attention for Long Video
// Diffusion, section 2): query frame t attends the anchors
// G_s = {f : (f - s) mod T_per == 0} plus the (C - |G_s|) non-anchor frames
// nearest to t (distance 0, 1, 2, ...; t - d before t + d; frames outside
// [0, T) skipped). Membership is decided by counting, without building the
// set: a non-anchor frame f at distance d from t is in the window iff fewer
// than C - |G_s| non-anchor frames come before it in that scan.
#pragma once

namespace dfs {

__device__ __forceinline__ int floor_div(int a, int b) { return (a >= 0) ? a / b : -((-a + b - 1) / b); }

// Number of anchor frames (f mod T_per == s0) in [lo, hi].
__device__ __forceinline__ int lvsa_anchors_in(int lo, int hi, int T_per, int s0) {
  if (hi < lo) return 0;
  return floor_div(hi - s0, T_per) - floor_div(lo - 1 - s0, T_per);
}

__device__ __forceinline__ int lvsa_anchor_count(int T, int T_per, int s0) {
  return (s0 < T) ? (T - 1 - s0) / T_per + 1 : 0;
}

// Is frame f in A(t)? (nG = |G_s|, s0 = s mod T_per.)
__device__ __forceinline__ bool lvsa_in_frame_set(int f, int t, int T, int T_per, int s0, int C, int nG) {
  if (((f - s0) % T_per + T_per) % T_per == 0) return true;
  const int need = C - nG;
  if (need <= 0) return false;
  const int dist = f > t ? f - t : t - f;
  // non-anchor frames scanned before f: all of (t - dist, t + dist) ...
  const int lo = max(0, t - dist + 1), hi = min(T - 1, t + dist - 1);
  int before = (hi >= lo) ? (hi - lo + 1) - lvsa_anchors_in(lo, hi, T_per, s0) : 0;
  // ... plus t - dist when f = t + dist (the earlier side goes first)
  if (dist > 0 && f > t) {
    const int g = t - dist;
    if (g >= 0 && ((g - s0) % T_per + T_per) % T_per != 0) ++before;
  }
  return before < need;
}

}  // namespace dfs
