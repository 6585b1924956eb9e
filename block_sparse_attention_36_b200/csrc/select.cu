// Per-query-block key-block selection.
//
//  * top-k -- DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient
//    Video Generation, Methodology item 3 (a sparsity budget per query
//    block): the k highest scores of the row, equal scores to the lower
//    block index.
//  * threshold -- VMoBA: Mixture of Block Attention for Video Diffusion
//    Models, abstract, modification (3): p = softmax of the row; the fewest
//    best-ranked blocks whose mass reaches tau, at most cap.
//  * LVSA -- LVSA: Training-Free Sparse Attention for Long Video Diffusion,
//    section 2: rotating global anchors plus an expanded local window of
//    frames, mapped onto key blocks.
//
// One warp per row. Scores live in registers, lane l holding columns
// l, l + 32, l + 64, ... Scores map to order-preserving 32-bit keys; the
// k-th largest key comes from a 32-step bitwise descent with warp-wide
// counts (__reduce_add_sync), the threshold cut from the same descent on
// warp-wide mass sums. Kept columns are emitted in ascending order with
// ballots and popcounts; equal keys at the cut go to the lowest columns.
#include "common.cuh"
#include "lvsa.cuh"

namespace {

__device__ uint32_t g_select_flags;

__device__ __forceinline__ uint32_t order_key(float f) {
  f = f + 0.0f;  // -0 -> +0, so equal values compare equal
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Largest key value K with count(key >= K) >= k (k >= 1, k <= n).
template <int S>
__device__ __forceinline__ uint32_t kth_largest_key(const uint32_t (&key)[S], const bool (&valid)[S], int k) {
  uint32_t K = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = K | (1u << bit);
    uint32_t c = 0;
#pragma unroll
    for (int s = 0; s < S; ++s) c += (valid[s] && key[s] >= cand) ? 1u : 0u;
    c = __reduce_add_sync(0xffffffffu, c);
    if (c >= (uint32_t)k) K = cand;
  }
  return K;
}

// Writes the kept columns of a row in ascending order: every column with
// key > K, plus the first `ties` columns with key == K.
template <int S>
__device__ __forceinline__ int emit_row(const uint32_t (&key)[S], const bool (&valid)[S], uint32_t K,
                                        int ties, int32_t* out, int kcap, int lane) {
  int base = 0, tie_seen = 0;
  const unsigned lt = (1u << lane) - 1u;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const bool gt = valid[s] && key[s] > K;
    const bool eq = valid[s] && key[s] == K;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool take_eq = eq && (tie_seen + __popc(eqb & lt)) < ties;
    tie_seen += __popc(eqb);
    const bool take = gt || take_eq;
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int pos = base + __popc(tb & lt);
    if (take && pos < kcap) out[pos] = s * 32 + lane;
    base += __popc(tb);
  }
  return base;
}

template <int S>
__global__ void __launch_bounds__(256)
select_scores_kernel(const float* __restrict__ scores, int rows, int nb, int mode, int k, int cap,
                     float tau, int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt, int kcap) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* src = scores + row * nb;
  float sc[S];
  uint32_t key[S];
  bool valid[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int j = s * 32 + lane;
    valid[s] = j < nb;
    sc[s] = valid[s] ? __ldg(src + j) : -INFINITY;
    key[s] = valid[s] ? order_key(sc[s]) : 0u;
  }
  int32_t* out = kv_idx + row * (long long)kcap;
  int kept;
  uint32_t K = 0u;
  int ties = 0;
  bool cut_known = false;  // K and ties already found (threshold)
  int take = 0;            // number of blocks to keep
  if (mode == DFS_SEL_TOPK) {
    take = min(k, nb);
  } else {
    // threshold: smallest best-ranked prefix with mass >= tau * Z, at most cap
    float m = -INFINITY;
#pragma unroll
    for (int s = 0; s < S; ++s) m = fmaxf(m, sc[s]);
    m = warp_max(m);
    float p[S];
    float z = 0.f;
#pragma unroll
    for (int s = 0; s < S; ++s) {
      p[s] = valid[s] ? expf(sc[s] - m) : 0.f;
      z += p[s];
    }
    z = warp_sum(z);
    const float target = tau * z;
    const int capn = min(cap, nb);
    if (capn >= 1 && capn < nb) {
      // The cap first: the capn best blocks are every key above the capn-th
      // largest key Kc plus the first ties at Kc. If they hold less than the
      // target, the prefix the rule asks for is longer and the cap decides.
      const uint32_t Kc = kth_largest_key<S>(key, valid, capn);
      uint32_t cg = 0;
      float mg = 0.f, pe = 0.f;
#pragma unroll
      for (int s = 0; s < S; ++s) {
        if (valid[s] && key[s] > Kc) { cg++; mg += p[s]; }
        if (valid[s] && key[s] == Kc) pe = p[s];
      }
      cg = __reduce_add_sync(0xffffffffu, cg);
      mg = warp_sum(mg);
      pe = warp_max(pe);
      float acc = mg;
      for (int u = (int)cg; u < capn; ++u) acc += pe;
      if (acc < target) {
        take = capn;
        K = Kc;
        ties = capn - (int)cg;
        cut_known = true;
      }
    }
    if (!cut_known) {
      // Largest key value KK with mass(key >= KK) >= target (a key of the row:
      // the mass only changes at key values).
      uint32_t KK = 0;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = KK | (1u << bit);
        float ms = 0.f;
#pragma unroll
        for (int s = 0; s < S; ++s) ms += (valid[s] && key[s] >= cand) ? p[s] : 0.f;
        ms = warp_sum(ms);
        if (ms >= target) KK = cand;
      }
      // Blocks strictly above the cut, their mass, and the tie value at the cut.
      uint32_t cgt = 0, ceq = 0;
      float mgt = 0.f, peq = 0.f;
#pragma unroll
      for (int s = 0; s < S; ++s) {
        if (valid[s] && key[s] > KK) { cgt++; mgt += p[s]; }
        if (valid[s] && key[s] == KK) { ceq++; peq = p[s]; }
      }
      cgt = __reduce_add_sync(0xffffffffu, cgt);
      ceq = __reduce_add_sync(0xffffffffu, ceq);
      mgt = warp_sum(mgt);
      peq = warp_max(peq);
      // mgt < target by the choice of KK (the warp sums are monotone in the
      // set summed). Equal scores carry equal mass: add them one at a time,
      // lowest column first, until the target is reached.
      int t = 0;
      float acc = mgt;
      while (t < (int)ceq && acc < target) { acc += peq; ++t; }
      take = max(1, (int)cgt + t);   // the shortest prefix holds at least one block
      take = min(take, capn);
      if (t >= 1 && take == (int)cgt + t) {
        // the cut is KK itself: every key above it and t of its ties
        K = KK;
        ties = t;
        cut_known = true;
      }
    }
  }
  if (take <= 0) {
    kept = 0;
  } else if (take >= nb) {
    // keep all columns
    bool all[S];
#pragma unroll
    for (int s = 0; s < S; ++s) all[s] = valid[s];
    uint32_t zk[S];
#pragma unroll
    for (int s = 0; s < S; ++s) zk[s] = 0u;
    kept = emit_row<S>(zk, all, 0u, nb, out, kcap, lane);
  } else {
    if (!cut_known) {
      K = kth_largest_key<S>(key, valid, take);
      uint32_t cgt = 0;
#pragma unroll
      for (int s = 0; s < S; ++s) cgt += (valid[s] && key[s] > K) ? 1u : 0u;
      cgt = __reduce_add_sync(0xffffffffu, cgt);
      ties = take - (int)cgt;
    }
    kept = emit_row<S>(key, valid, K, ties, out, kcap, lane);
  }
  if (lane == 0) {
    if (kept > kcap) atomicOr(&g_select_flags, (uint32_t)DFS_FLAG_KCAP_OVERFLOW);
    kv_cnt[row] = min(kept, kcap);
  }
}

__global__ void __launch_bounds__(256)
select_lvsa_kernel(int rows, int nb, long long N, int blk, int P, int T, int T_per, int C, int s0,
                   int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt, int kcap) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int I = (int)(row % nb);
  const int nG = dfs::lvsa_anchor_count(T, T_per, s0);
  const int qf0 = (int)(((long long)I * blk) / P);
  const int qf1 = (int)((min((long long)I * blk + blk, N) - 1) / P);
  int32_t* out = kv_idx + row * (long long)kcap;
  const unsigned lt = (1u << lane) - 1u;
  int base = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int J = j0 + lane;
    bool take = false;
    if (J < nb) {
      const int kf0 = (int)(((long long)J * blk) / P);
      const int kf1 = (int)((min((long long)J * blk + blk, N) - 1) / P);
      for (int f = kf0; f <= kf1 && !take; ++f)
        for (int t = qf0; t <= qf1 && !take; ++t)
          take = dfs::lvsa_in_frame_set(f, t, T, T_per, s0, C, nG);
    }
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int pos = base + __popc(tb & lt);
    if (take && pos < kcap) out[pos] = J;
    base += __popc(tb);
  }
  if (lane == 0) {
    if (base > kcap) atomicOr(&g_select_flags, (uint32_t)DFS_FLAG_KCAP_OVERFLOW);
    kv_cnt[row] = min(base, kcap);
  }
}

// Log-radial static mask (DynamicRad, methodology, components 1 and 2):
// query token q may attend key token k iff 2 |s_q - s_k| < omega(d), with
// d the frame distance, s the spatial index in the frame and
// omega(d) = max(w0 >> bitlength(d), w_far). Key block J is kept for query
// block I iff some pair qualifies. Each block splits into per-frame
// segments of spatial indices; two segments have a qualifying pair iff the
// gap between their index intervals is small enough, so a block pair costs
// (segments of I) x (segments of J) tests (2 x 2 when H*W >= blk).
__device__ __forceinline__ bool radial_segments_meet(int t, int a0, int a1, int f, int b0, int b1, int w0,
                                                     int w_far) {
  const unsigned d = (unsigned)(t > f ? t - f : f - t);
  const int band = 32 - __clz((int)d);
  const int om = max(band >= 31 ? 0 : (w0 >> band), w_far);
  const int gap = max(0, max(b0 - a1, a0 - b1));
  return 2LL * gap < (long long)om;
}

__global__ void __launch_bounds__(256)
select_radial_kernel(int rows, int nb, long long N, int blk, int P, int w0, int w_far,
                     int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_cnt, int kcap) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int I = (int)(row % nb);
  const long long q_lo = (long long)I * blk, q_hi = min(q_lo + blk, N) - 1;
  const int qf0 = (int)(q_lo / P), qf1 = (int)(q_hi / P);
  int32_t* out = kv_idx + row * (long long)kcap;
  const unsigned lt = (1u << lane) - 1u;
  int base = 0;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int J = j0 + lane;
    bool take = false;
    if (J < nb) {
      const long long k_lo = (long long)J * blk, k_hi = min(k_lo + blk, N) - 1;
      const int kf0 = (int)(k_lo / P), kf1 = (int)(k_hi / P);
      for (int t = qf0; t <= qf1 && !take; ++t) {
        const long long tb = (long long)t * P;
        const int a0 = (int)(max(q_lo, tb) - tb), a1 = (int)(min(q_hi, tb + P - 1) - tb);
        for (int f = kf0; f <= kf1 && !take; ++f) {
          const long long fb = (long long)f * P;
          const int b0 = (int)(max(k_lo, fb) - fb), b1 = (int)(min(k_hi, fb + P - 1) - fb);
          take = radial_segments_meet(t, a0, a1, f, b0, b1, w0, w_far);
        }
      }
    }
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    const int pos = base + __popc(tb & lt);
    if (take && pos < kcap) out[pos] = J;
    base += __popc(tb);
  }
  if (lane == 0) {
    if (base > kcap) atomicOr(&g_select_flags, (uint32_t)DFS_FLAG_KCAP_OVERFLOW);
    kv_cnt[row] = min(base, kcap);
  }
}

// Global selection (VMoBA, abstract, modification 2): per head (one CTA),
// the K best (query block, key block) pairs of all nb x nb, equal scores to
// the lower flat index I * nb + J; rows list their kept J ascending.
// Radix select on order-preserving 32-bit keys (4 passes of 8 bits with a
// shared-memory histogram) finds the K-th largest key; ties at the cut are
// taken in flat-index order through a per-row tie count and its prefix sum.
__global__ void __launch_bounds__(1024)
select_global_kernel(const float* __restrict__ scores, int nb, int K, int32_t* __restrict__ kv_idx,
                     int32_t* __restrict__ kv_cnt, int kcap) {
  extern __shared__ int tie_before[];   // nb + 1 ints
  __shared__ unsigned hist[256];
  __shared__ uint32_t sh_prefix, sh_mask;
  __shared__ int sh_rem;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const long long bh = blockIdx.x;
  const float* s = scores + bh * (long long)nb * nb;
  const long long n = (long long)nb * nb;
  const bool all = (long long)K >= n, none = K <= 0;
  if (tid == 0) { sh_prefix = 0u; sh_mask = 0u; sh_rem = K; }
  __syncthreads();
  if (!all && !none) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int b = tid; b < 256; b += blockDim.x) hist[b] = 0u;
      __syncthreads();
      const uint32_t prefix = sh_prefix, mask = sh_mask;
      for (long long e = tid; e < n; e += blockDim.x) {
        const uint32_t key = order_key(__ldg(s + e));
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        int rem = sh_rem, cum = 0, b = 255;
        for (; b > 0; --b) {
          if (cum + (int)hist[b] >= rem) break;
          cum += (int)hist[b];
        }
        sh_prefix = prefix | ((uint32_t)b << shift);
        sh_mask = mask | (255u << shift);
        sh_rem = rem - cum;
      }
      __syncthreads();
    }
  }
  const uint32_t cut = sh_prefix;              // the K-th largest key
  const int ties_needed = sh_rem;              // keys == cut to keep, lowest flat index first
  // ties per row, then their exclusive prefix over rows
  for (int r = warp; r < nb; r += nwarps) {
    int c = 0;
    if (!all && !none)
      for (int j = lane; j < nb; j += 32) c += order_key(__ldg(s + (long long)r * nb + j)) == cut ? 1 : 0;
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) tie_before[r] = c;
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int r = 0; r < nb; ++r) {
      const int c = tie_before[r];
      tie_before[r] = run;
      run += c;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int r = warp; r < nb; r += nwarps) {
    int base = 0, ties = tie_before[r];
    int32_t* out = kv_idx + (bh * nb + r) * (long long)kcap;
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      bool take = false, eq = false;
      if (j < nb && !none) {
        const uint32_t key = order_key(__ldg(s + (long long)r * nb + j));
        eq = !all && key == cut;
        take = all || key > cut;
      }
      const unsigned eqb = __ballot_sync(0xffffffffu, eq);
      if (eq && ties + __popc(eqb & lt) < ties_needed) take = true;
      ties += __popc(eqb);
      const unsigned tb = __ballot_sync(0xffffffffu, take);
      const int pos = base + __popc(tb & lt);
      if (take && pos < kcap) out[pos] = j;
      base += __popc(tb);
    }
    if (lane == 0) {
      if (base > kcap) atomicOr(&g_select_flags, (uint32_t)DFS_FLAG_KCAP_OVERFLOW);
      kv_cnt[bh * nb + r] = min(base, kcap);
    }
  }
}

}  // namespace

DFS_DEFINE_FLAG_READER(dfs_detail_flags_select, g_select_flags)

extern "C" int dfs_select_mask(const dfs_shape* shape, const float* scores, const dfs_select_params* prm,
                               int32_t* kv_idx, int32_t* kv_cnt, int kcap, dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, false);
  if (st != DFS_OK) return st;
  if (!prm || !kv_idx || !kv_cnt || kcap < 1) return DFS_ERR_INVALID_ARG;
  const long long rows = d.BH * d.nb;
  if (rows > (1LL << 31) / 8) return DFS_ERR_UNSUPPORTED;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  cudaStream_t cs = (cudaStream_t)stream;
  if (prm->mode == DFS_SEL_LVSA) {
    const long long P = (long long)d.H * d.W;
    if (prm->lvsa_T_per < 1 || prm->lvsa_C < 1 || prm->lvsa_step < 0) return DFS_ERR_INVALID_ARG;
    select_lvsa_kernel<<<grid, 256, 0, cs>>>((int)rows, d.nb, d.N, d.blk, (int)P, d.T, prm->lvsa_T_per,
                                             prm->lvsa_C, prm->lvsa_step % prm->lvsa_T_per, kv_idx,
                                             kv_cnt, kcap);
    return dfs::launch_status();
  }
  if (prm->mode == DFS_SEL_RADIAL) {
    const long long P = (long long)d.H * d.W;
    const double lam = (double)prm->radial_lambda;
    if (prm->radial_w0 < 0 || !(lam >= 0.0) || lam > 1e9) return DFS_ERR_INVALID_ARG;
    const double wf = floor(lam * (double)prm->radial_w0);
    const int w_far = wf >= 2147483647.0 ? 2147483647 : (int)wf;
    select_radial_kernel<<<grid, 256, 0, cs>>>((int)rows, d.nb, d.N, d.blk, (int)P, prm->radial_w0, w_far,
                                               kv_idx, kv_cnt, kcap);
    return dfs::launch_status();
  }
  if (!scores) return DFS_ERR_INVALID_ARG;
  if (!dfs::aligned16(scores)) return DFS_ERR_MISALIGNED;
  if (prm->mode == DFS_SEL_GLOBAL) {
    if (prm->k < 0 || kcap < (prm->k < d.nb ? prm->k : d.nb)) return DFS_ERR_INVALID_ARG;
    if ((long long)d.nb * d.nb > (1LL << 31) - 1 || d.BH > 0x7fffffffLL) return DFS_ERR_UNSUPPORTED;
    const size_t smem = ((size_t)d.nb + 1) * sizeof(int);
    if (smem > 200 * 1024) return DFS_ERR_UNSUPPORTED;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(select_global_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return DFS_ERR_CUDA;
    select_global_kernel<<<(unsigned)d.BH, 1024, smem, cs>>>(scores, d.nb, prm->k, kv_idx, kv_cnt, kcap);
    return dfs::launch_status();
  }
  if (prm->mode == DFS_SEL_TOPK) {
    if (prm->k < 0 || kcap < (prm->k < d.nb ? prm->k : d.nb)) return DFS_ERR_INVALID_ARG;
  } else if (prm->mode == DFS_SEL_THRESHOLD) {
    if (prm->cap < 0 || !(prm->tau >= 0.f) || kcap < (prm->cap < d.nb ? prm->cap : d.nb))
      return DFS_ERR_INVALID_ARG;
  } else {
    return DFS_ERR_INVALID_ARG;
  }
  const int S = (d.nb + 31) / 32;
#define DFS_SEL_LAUNCH(SS)                                                                       \
  select_scores_kernel<SS><<<grid, 256, 0, cs>>>(scores, (int)rows, d.nb, prm->mode, prm->k,      \
                                                 prm->cap, prm->tau, kv_idx, kv_cnt, kcap)
  if (S <= 4) DFS_SEL_LAUNCH(4);
  else if (S <= 8) DFS_SEL_LAUNCH(8);
  else if (S <= 16) DFS_SEL_LAUNCH(16);
  else if (S <= 32) DFS_SEL_LAUNCH(32);
  else if (S <= 64) DFS_SEL_LAUNCH(64);
  else return DFS_ERR_UNSUPPORTED;
#undef DFS_SEL_LAUNCH
  return dfs::launch_status();
}
