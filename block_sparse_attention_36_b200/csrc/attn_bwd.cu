// Block-sparse attention backward over the kept key blocks (sm_100a).
//
// Gradients of the forward in attn.cu for a loss L with dL/dO = dO, as
// training through block attention needs them (VMoBA: Mixture of Block
// Attention for Video Diffusion Models, abstract: training speed-ups of the
// block attention). With P = exp(scale q.k - lse) over the kept keys of the
// query's block, dP = dO V^T, Delta_q = dO_q . O_q and dS = P (dP - Delta):
//   dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO.
// Two deterministic passes (no atomics; every sum runs in a fixed order):
//   attn_bwd_dq_kernel    one CTA per query block, over its kept list:
//                         S = Q K^T, dP = dO V^T, dS, dQ += dS K, with Q
//                         and dO held in tensor memory.
//   attn_bwd_dkdv_kernel  one CTA per key block, over the query blocks that
//                         keep it (the transposed lists, ascending):
//                         S^T = K Q^T, dP^T = V dO^T, dV += P^T dO,
//                         dK += dS^T Q.
// bwd_prep_kernel turns lse and O into two per-row constants, -lse log2(e)
// and -Delta, padded to whole blocks (padding rows get -inf and 0, so P = 0
// there); bwd_mask_bits_kernel and bwd_transpose_kernel build the
// transposed lists through a bitset of the kept mask.
// Both passes: warp 0 loads tiles with TMA (128-byte swizzle, no multicast),
// warp 1 owns tensor memory and issues the tcgen05 MMAs from one elected
// lane, warp 2 stages (dQ) or counts (dK/dV) the list, warps 4-11 are two
// warpgroups that each take one half of the 128 columns of the score tiles
// (one TMEM lane per row). dS goes back as bf16 into the tensor-memory
// columns it was read from; P^T of the dK/dV pass goes to a shared-memory
// tile instead, so that the next S^T need not wait for dV. Keys beyond N
// have zero K and V rows (TMA fill), so they add nothing to dQ, and their dK,
// dV rows are not stored. Every mbarrier wait is bounded (timeout flag,
// early return); copies and MMAs in flight are drained before tensor memory
// is released.
#include "common.cuh"
#include "sm100_ptx.cuh"
#include "tmap.cuh"

namespace {

using namespace dfs::sm100;

__device__ uint32_t g_bwd_flags;

constexpr long long kWaitLimit = 4000000000ll;
constexpr long long kDrainLimit = 2000000000ll;
constexpr int kThreads = 384;
constexpr int kBlk = 128;      // block size = MMA M = N of the score products
constexpr int kRing = 6;       // K/V ring stages of the dQ pass
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Bw {
  static constexpr int kChunks = D / 64;          // 128-byte column slabs per row
  static constexpr int kTile = kBlk * D * 2;      // one 128-row tile
  // dQ pass: shared memory holds the K/V ring only
  static constexpr int kRingOff = 0;
  static constexpr int kQBarOff = kRingOff + kRing * kTile;
  // tensor memory columns
  static constexpr int kS = 0, kDP = 128, kDQ = 256, kQT = 256 + D, kDOT = 256 + D + D / 2;
};

// Untiled bulk copy global -> shared completing on an mbarrier, from
// warp-uniform code (one elected lane issues). 16-byte aligned, size a
// multiple of 16.
__device__ __forceinline__ void bulk_load_warp(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  uint64_t g;
  asm("cvta.to.global.u64 %0, %1;" : "=l"(g) : "l"(reinterpret_cast<uint64_t>(src)));
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}\n" ::"r"(
          smem_addr(dst)),
      "l"(g), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// D = A B^T over the D-long rows of two 128-row K-major tiles (S-like
// products): D/16 MMAs of K = 16.
template <int D>
__device__ __forceinline__ void issue_nt(uint32_t d_tmem, uint64_t da, uint64_t db) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBlk, kBlk, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk >> 2) * (kBlk * 128) + (kk & 3) * 32) >> 4);
    mma_ss_warp(d_tmem, da + off, db + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// D (+)= A B with A (128 x 128 bf16) in tensor memory and B (128 x D) a
// 128-row tile read MN-major. A's two 64-wide K halves sit at columns
// a_tmem + 0 .. 31 and a_tmem + 64 .. 95 (two bf16 per column): each
// softmax warpgroup packs its half over the first columns it read.
template <int D>
__device__ __forceinline__ void issue_tn(uint32_t d_tmem, uint32_t a_tmem, uint64_t db, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBlk, D, 1);
#pragma unroll
  for (int kk = 0; kk < kBlk / 16; ++kk)
    mma_ts_warp(d_tmem, a_tmem + (kk >> 2) * 64 + (kk & 3) * 8, db + (uint64_t)((kk * 2048) >> 4), idesc,
                (accumulate || kk > 0) ? 1u : 0u);
}

// Stores 32 fp32 columns of one row, times mul, as bf16 (16-byte stores).
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&raw)[32], float mul, bool store) {
  uint32_t pk[16];
#pragma unroll
  for (int e = 0; e < 16; ++e)
    pk[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * mul, __uint_as_float(raw[2 * e + 1]) * mul);
  if (store) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int v = 0; v < 4; ++v) d4[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
  }
}

// ------------------------------------------------------------ small kernels
// Per padded row n of head bh: nlse = -lse * log2(e) and ndelta = -dO . O
// (fp32 from bf16), or -inf and 0 for n >= N (and -inf for lse = -inf).
template <int D>
__global__ void __launch_bounds__(256)
bwd_prep_kernel(const __nv_bfloat16* __restrict__ op, const __nv_bfloat16* __restrict__ dop,
                const float* __restrict__ lse, int N, int nb, long long rows, float* __restrict__ nlse,
                float* __restrict__ ndelta) {
  constexpr int kLpr = D / 8;        // lanes per row, 16 bytes each
  constexpr int kRpw = 32 / kLpr;    // rows per warp
  const int lane = threadIdx.x & 31;
  const long long row = ((long long)blockIdx.x * 8 + (threadIdx.x >> 5)) * kRpw + lane / kLpr;
  const int sl = lane & (kLpr - 1);
  const long long padded = (long long)nb * kBlk;
  const long long bh = row / padded;
  const int n = (int)(row - bh * padded);
  const bool valid = row < rows && n < N;
  float acc = 0.f;
  if (valid) {
    const long long off = ((long long)bh * N + n) * D + sl * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(op + off);
    const uint4 b = *reinterpret_cast<const uint4*>(dop + off);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[e]));
      const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[e]));
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int o = kLpr / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (sl == 0 && row < rows) {
    ndelta[row] = valid ? -acc : 0.f;
    const float l = valid ? lse[(long long)bh * N + n] : -INFINITY;
    nlse[row] = (valid && isfinite(l)) ? -l * kLog2e : -INFINITY;
  }
}

// One warp per row (b, h, I): the kept key blocks as a bitset of nw words.
__global__ void __launch_bounds__(256)
bwd_mask_bits_kernel(const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt, int kcap, int nb,
                     long long rows, int nw, uint32_t* __restrict__ bits) {
  extern __shared__ uint32_t sbits[];   // 8 warps x nw words
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + warp;
  uint32_t* mine = sbits + warp * nw;
  for (int k = lane; k < nw; k += 32) mine[k] = 0u;
  __syncwarp();
  bool bad = false;
  if (row < rows) {
    const int cnt = max(0, min(kv_cnt[row], min(kcap, nb)));
    for (int j = lane; j < cnt; j += 32) {
      const int J = kv_idx[row * kcap + j];
      if (J >= 0 && J < nb) atomicOr(&mine[J >> 5], 1u << (J & 31));
      else bad = true;
    }
  }
  __syncwarp();
  if (row < rows)
    for (int k = lane; k < nw; k += 32) bits[row * nw + k] = mine[k];
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_bwd_flags, (uint32_t)DFS_FLAG_BAD_KV_INDEX);
}

// One warp per column (b, h, J): the query blocks that keep J, ascending.
__global__ void __launch_bounds__(256)
bwd_transpose_kernel(const uint32_t* __restrict__ bits, int nb, int nw, long long cols, int32_t* __restrict__ q_idx,
                     int32_t* __restrict__ q_cnt) {
  const int lane = threadIdx.x & 31;
  const long long col = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (col >= cols) return;
  const long long bh = col / nb;
  const int J = (int)(col - bh * nb);
  const uint32_t* base = bits + bh * nb * (long long)nw + (J >> 5);
  const int sh = J & 31;
  int32_t* out = q_idx + col * nb;
  const unsigned lt = (1u << lane) - 1u;
  int cnt = 0;
  for (int I0 = 0; I0 < nb; I0 += 32) {
    const int I = I0 + lane;
    const bool take = I < nb && ((base[(long long)I * nw] >> sh) & 1u);
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (take) out[cnt + __popc(m & lt)] = I;
    cnt += __popc(m);
  }
  if (lane == 0) q_cnt[col] = cnt;
}

// ------------------------------------------------------------ dQ pass
struct __align__(8) BarsQ {
  uint64_t qt_ready;
  uint64_t kv_full[kRing], kv_empty[kRing];
  uint64_t s_full, s_free, dp_full, ds_ready, dq_final, mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int n_kv;
};

// S = Q K^T or dP = dO V^T with the 128 x D left operand resident in tensor
// memory (two bf16 per column, D/2 columns) and K or V a K-major tile.
template <int D>
__device__ __forceinline__ void issue_ts_nt(uint32_t d_tmem, uint32_t a_tmem, uint64_t db) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBlk, kBlk, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk >> 2) * (kBlk * 128) + (kk & 3) * 32) >> 4);
    mma_ts_warp(d_tmem, a_tmem + kk * 8, db + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// Q and dO of the query block live in tensor memory for the whole CTA
// (written once by the dS warps), so both score products read only K or V
// from shared memory. Ring tiles in load (= first use) order: K(0), V(0),
// K(1), V(1), ... (tile u: K(u/2) for even u, V(u/2) for odd u). MMA order:
// S(0) dP(0), then per kept block j: [S(j) read] S(j+1), [dS(j) written
// over dP(j)] dQ += dS(j) K(j), dP(j+1). S(j+1) therefore runs while the
// exponentials of block j are formed, and dQ(j), dP(j+1) while those of
// block j+1 are.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __nv_bfloat16* __restrict__ qp, const __nv_bfloat16* __restrict__ dop,
                   const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt, int kcap, int N, int nb,
                   float scale, float scale_log2, const float* __restrict__ nlse, const float* __restrict__ ndelta,
                   __nv_bfloat16* __restrict__ dq, int max_list) {
  using C = Bw<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BarsQ* bars = reinterpret_cast<BarsQ*>(smem + C::kQBarOff);
  int32_t* list = reinterpret_cast<int32_t*>(smem + C::kQBarOff + sizeof(BarsQ));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int I = blockIdx.x, bh = blockIdx.y;
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qt_ready, 8);
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 8);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->ds_ready, 8);
    mbar_init(&bars->dq_final, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    const long long row_id = (long long)bh * nb + I;
    const int cnt = max(0, min(kv_cnt[row_id], max_list));
    const int32_t* src = kv_idx + row_id * (long long)kcap;
    int base = 0;
    bool bad = false;
    for (int j0 = 0; j0 < cnt; j0 += 32) {
      const int j = j0 + lane;
      const int J = (j < cnt) ? src[j] : -1;
      const bool ok = (j < cnt) && J >= 0 && J < nb;
      bad |= (j < cnt) && !ok;
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      if (ok) list[base + __popc(m & ((1u << lane) - 1u))] = J;
      base += __popc(m);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_bwd_flags, (uint32_t)DFS_FLAG_BAD_KV_INDEX);
    if (lane == 0) bars->n_kv = base;
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n = bars->n_kv;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensor_map(&tm_k);
      prefetch_tensor_map(&tm_v);
    }
    int u = 0;
    for (; u < 2 * n; ++u) {
      const int st = u % kRing;
      if (!mbar_wait_bounded(&bars->kv_empty[st], (uint32_t)(((u / kRing) & 1) ^ 1), abort_flag, kWaitLimit)) break;
      mbar_arrive_expect_tx_warp(&bars->kv_full[st], C::kTile);
      const int J = list[u >> 1];
      const CUtensorMap* map = (u & 1) ? &tm_v : &tm_k;
      uint8_t* dst = smem + C::kRingOff + st * C::kTile;
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d_warp(dst + c * (kBlk * 128), map, &bars->kv_full[st], c * 64, J * kBlk, bh);
    }
    // Drain: a stage is reloaded only after its previous tile was consumed,
    // so only the last kRing loads can still be in flight.
    for (int w = max(0, u - kRing); w < u; ++w)
      mbar_wait_timed(&bars->kv_full[w % kRing], (uint32_t)((w / kRing) & 1), kDrainLimit);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t ring_k = desc_sw128(smem_addr(smem + C::kRingOff), 16, 1024);
    const uint64_t ring_mn = desc_sw128(smem_addr(smem + C::kRingOff), kBlk * 128, 1024);
    auto stage_off = [](int u) { return (uint64_t)(((u % kRing) * C::kTile) >> 4); };
    auto wait_tile = [&](int u) {
      return mbar_wait_bounded(&bars->kv_full[u % kRing], (uint32_t)((u / kRing) & 1), abort_flag, kWaitLimit);
    };
    bool ok = true;
    if (n > 0) {
      // Q and dO were stored into tensor memory with tcgen05.st.
      ok = mbar_wait_bounded(&bars->qt_ready, 0, abort_flag, kWaitLimit);
      tc_fence_after();
      if (ok && (ok = wait_tile(0))) {
        issue_ts_nt<D>(tmem + C::kS, tmem + C::kQT, ring_k + stage_off(0));
        mma_commit_warp(&bars->s_full);
      }
      if (ok && (ok = wait_tile(1))) {
        issue_ts_nt<D>(tmem + C::kDP, tmem + C::kDOT, ring_k + stage_off(1));
        mma_commit_warp(&bars->dp_full);
        mma_commit_warp(&bars->kv_empty[1 % kRing]);
      }
    }
    for (int j = 0; j < n && ok; ++j) {
      if (j + 1 < n) {
        // S(j) has been read into registers: S(j+1) may overwrite it.
        if (!mbar_wait_bounded(&bars->s_free, (uint32_t)(j & 1), abort_flag, kWaitLimit)) { ok = false; break; }
        tc_fence_after();
        const int u = 2 * (j + 1);       // K(j+1)
        if (!wait_tile(u)) { ok = false; break; }
        issue_ts_nt<D>(tmem + C::kS, tmem + C::kQT, ring_k + stage_off(u));
        mma_commit_warp(&bars->s_full);
      }
      // dS(j) was written over dP(j) with tcgen05.st by the dS warps.
      if (!mbar_wait_bounded(&bars->ds_ready, (uint32_t)(j & 1), abort_flag, kWaitLimit)) { ok = false; break; }
      tc_fence_after();
      issue_tn<D>(tmem + C::kDQ, tmem + C::kDP, ring_mn + stage_off(2 * j), j > 0);   // K(j), MN-major
      mma_commit_warp(&bars->kv_empty[(2 * j) % kRing]);
      if (j + 1 < n) {
        const int u = 2 * (j + 1) + 1;   // V(j+1)
        if (!wait_tile(u)) { ok = false; break; }
        issue_ts_nt<D>(tmem + C::kDP, tmem + C::kDOT, ring_k + stage_off(u));
        mma_commit_warp(&bars->dp_full);
        mma_commit_warp(&bars->kv_empty[u % kRing]);
      }
    }
    if (ok && n > 0) mma_commit_warp(&bars->dq_final);
    // Every MMA must finish before tensor memory is released.
    mma_commit_warp(&bars->mma_done);
    mbar_wait_timed(&bars->mma_done, 0, kDrainLimit);
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ dS warps
    const int g = (warp - 4) >> 2;                  // column half
    const int sub = warp & 3;                       // TMEM lane quarter
    const int r = sub * 32 + lane;                  // query row in the block
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const long long qrow = (long long)I * kBlk + r;
    {
      // this row's half of Q and dO into tensor memory (zeros past N)
      constexpr int kHalf = D / 2;                  // elements per warpgroup
      const long long off = ((long long)bh * N + qrow) * D + kHalf * g;
      const bool in = qrow < N;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint4* src = reinterpret_cast<const uint4*>((t == 0 ? qp : dop) + off);
        const uint32_t col = tmem + lane_base + (t == 0 ? C::kQT : C::kDOT) + (kHalf / 2) * g;
        if (kHalf == 64) {
          uint32_t w[32];
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const uint4 x = in ? src[v] : make_uint4(0u, 0u, 0u, 0u);
            w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
          }
          tmem_st32(col, w);
        } else {
          uint32_t w[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 x = in ? src[v] : make_uint4(0u, 0u, 0u, 0u);
            w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
          }
          tmem_st16(col, w);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->qt_ready);
    }
    const long long prow = ((long long)bh * nb + I) * kBlk + r;
    const float nl = nlse[prow], nd = ndelta[prow];
    const float2 sc2 = make_float2(scale_log2, scale_log2), nl2 = make_float2(nl, nl), nd2 = make_float2(nd, nd);
    const uint32_t s_addr = tmem + lane_base + C::kS + 64 * g;
    const uint32_t p_addr = tmem + lane_base + C::kDP + 64 * g;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      // S(j) into registers, release it, then P = 2^(S scale log2 e - lse log2 e)
      if (!mbar_wait_bounded(&bars->s_full, (uint32_t)(j & 1), abort_flag, kWaitLimit)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float pv[64];
      {
        uint32_t sr[64];
        tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), sc2, nl2);
          pv[2 * e] = ex2(x.x);
          pv[2 * e + 1] = ex2(x.y);
        }
      }
      if (!mbar_wait_bounded(&bars->dp_full, (uint32_t)(j & 1), abort_flag, kWaitLimit)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pr[32], out[16];
        tmem_ld32(p_addr + 32 * c, pr);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 t = __fadd2_rn(make_float2(__uint_as_float(pr[2 * e]), __uint_as_float(pr[2 * e + 1])), nd2);
          const float2 ds = __fmul2_rn(make_float2(pv[32 * c + 2 * e], pv[32 * c + 2 * e + 1]), t);
          out[e] = pack_bf16x2(ds.x, ds.y);
        }
        // columns 64g + 16c .. +15 of dP: fp32 columns this thread already read
        tmem_st16(p_addr + 16 * c, out);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready);
    }
    if (ok && n > 0) ok = mbar_wait_bounded(&bars->dq_final, 0, abort_flag, kWaitLimit);
    tc_fence_after();
    const bool store = ok && qrow < N;
    __nv_bfloat16* orow = dq + ((long long)bh * N + qrow) * D + (D / 2) * g;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint32_t raw[32];
      if (n > 0 && ok) {
        tmem_ld32(tmem + lane_base + C::kDQ + (D / 2) * g + 32 * c, raw);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) raw[e] = 0u;
      }
      store_row32(orow + 32 * c, raw, scale, store);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && bars->abort_flag) atomicOr(&g_bwd_flags, (uint32_t)DFS_FLAG_WAIT_TIMEOUT);
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------ dK/dV pass
// Shared memory: K, V, two stages of {Q, dO, -lse log2 e [128], -Delta [128]},
// the P^T tile; then the tensor memory columns.
template <int D>
struct BwKV {
  static constexpr int kTile = kBlk * D * 2;        // one 128-row Q / dO / K / V tile
  static constexpr int kPtBytes = kBlk * kBlk * 2;  // P^T: 128 keys x 128 queries, bf16
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTile;
  static constexpr int kStageOff = 2 * kTile;
  static constexpr int kStageBytes = 2 * kTile + 1024;
  static constexpr int kPtOff = kStageOff + 2 * kStageBytes;
  static constexpr int kTiles = kPtOff + kPtBytes;  // everything that needs 1024-byte alignment
  static constexpr int kST_col = 0, kDPT_col = 128, kDV_col = 256, kDK_col = 256 + D;  // tensor memory
};

struct __align__(8) BarsKV {
  uint64_t kv_full;
  uint64_t qq_full[2], qq_empty[2];  // Q and the two per-query constant rows of a stage
  uint64_t qd_full[2], qd_empty[2];  // dO of a stage
  uint64_t st_full, dpt_full, s_read, p_ready, p_free, ds_ready, kv_final, mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int n_q;
};

// The shared-memory window of a CTA: the 1024-byte-aligned tiles and the
// barriers, placed in whichever of three ways fits tiles + 1008 bytes from
// any 16-byte-aligned base. The window is declared 1024-byte aligned, so
// the first way is the one taken; the others keep the layout in bounds
// should a base ever arrive less aligned.
struct SmemKV {
  uint8_t* tiles;
  BarsKV* bars;
};
template <int D>
__device__ __forceinline__ SmemKV place_smem_kv(uint8_t* raw) {
  const uint32_t a = smem_addr(raw) & 1023u;
  SmemKV r;
  if (a == 0) {
    r.tiles = raw;
    r.bars = reinterpret_cast<BarsKV*>(raw + BwKV<D>::kTiles);
  } else if (a + sizeof(BarsKV) <= 1024u) {
    r.bars = reinterpret_cast<BarsKV*>(raw);
    r.tiles = raw + (1024u - a);
  } else {
    r.tiles = raw + (1024u - a);
    r.bars = reinterpret_cast<BarsKV*>(r.tiles + BwKV<D>::kTiles);
  }
  return r;
}

// D (+)= A B with A (128 x 128 bf16, K-major, 128-byte swizzled) and B a
// 128-row tile read MN-major, both in shared memory.
template <int D>
__device__ __forceinline__ void issue_ss_tn(uint32_t d_tmem, uint64_t da, uint64_t db, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kBlk, D, 1);
#pragma unroll
  for (int kk = 0; kk < kBlk / 16; ++kk) {
    const uint64_t aoff = (uint64_t)(((kk >> 2) * (kBlk * 128) + (kk & 3) * 32) >> 4);
    mma_ss_warp(d_tmem, da + aoff, db + (uint64_t)((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Per query block i of the transposed list the P/dS warps read S^T(i) from
// tensor memory (and report it read, so that S^T(i+1) can start at once),
// form P^T(i) into a shared-memory tile for dV(i), then dS^T(i) over dP^T(i)
// in tensor memory for dK(i). MMA order: S^T(0) dP^T(0), then per i:
// [S^T(i) read] S^T(i+1) [P^T(i)] dV(i) [dS^T(i)] dK(i) dP^T(i+1). The
// exponentials of block i overlap S^T(i+1), dK(i-1) and dP^T(i); P^T(i+1)
// is written once dV(i) has read P^T(i).
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const int32_t* __restrict__ q_idx, const int32_t* __restrict__ q_cnt, int N, int nb,
                        float scale, float scale_log2, const float* __restrict__ nlse,
                        const float* __restrict__ ndelta, __nv_bfloat16* __restrict__ dk,
                        __nv_bfloat16* __restrict__ dv) {
  using C = BwKV<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const SmemKV sp = place_smem_kv<D>(smem_raw);
  uint8_t* smem = sp.tiles;
  BarsKV* bars = sp.bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int J = blockIdx.x, bh = blockIdx.y;
  volatile int* abort_flag = &bars->abort_flag;
  const long long col = (long long)bh * nb + J;
  const int cnt = max(0, min(q_cnt[col], nb));
  const int32_t* src = q_idx + col * nb;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->qq_full[s], 1);
      mbar_init(&bars->qq_empty[s], 1);
      mbar_init(&bars->qd_full[s], 1);
      mbar_init(&bars->qd_empty[s], 1);
    }
    mbar_init(&bars->st_full, 1);
    mbar_init(&bars->dpt_full, 1);
    mbar_init(&bars->s_read, 8);
    mbar_init(&bars->p_ready, 8);
    mbar_init(&bars->p_free, 1);
    mbar_init(&bars->ds_ready, 8);
    mbar_init(&bars->kv_final, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    // valid entries of the list (the producer skips the others in the same order)
    int valid = 0;
    for (int i0 = 0; i0 < cnt; i0 += 32) {
      const int i = i0 + lane;
      const int Iq = (i < cnt) ? src[i] : -1;
      valid += __popc(__ballot_sync(0xffffffffu, Iq >= 0 && Iq < nb));
    }
    if (lane == 0) bars->n_q = valid;
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n = bars->n_q;
  const long long padded = (long long)nb * kBlk;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensor_map(&tm_q);
      prefetch_tensor_map(&tm_k);
      prefetch_tensor_map(&tm_v);
      prefetch_tensor_map(&tm_do);
    }
    if (n > 0) {
      mbar_arrive_expect_tx_warp(&bars->kv_full, 2 * C::kTile);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d_warp(smem + C::kKOff + c * (kBlk * 128), &tm_k, &bars->kv_full, c * 64, J * kBlk, bh);
        tma_load_3d_warp(smem + C::kVOff + c * (kBlk * 128), &tm_v, &bars->kv_full, c * 64, J * kBlk, bh);
      }
    }
    // The list is read 32 entries at a time (one per lane); `pend` holds the
    // lanes of the current group whose entries are valid and not yet used.
    int g0 = -32;
    int mine = -1;
    unsigned pend = 0u;
    int i = 0, nq = 0, nd = 0;  // blocks whose Q / dO copies were issued
    for (; i < n; ++i) {
      while (pend == 0u && g0 + 32 < cnt) {
        g0 += 32;
        mine = (g0 + lane < cnt) ? src[g0 + lane] : -1;
        pend = __ballot_sync(0xffffffffu, mine >= 0 && mine < nb);
      }
      if (pend == 0u) break;  // cannot happen: n counts the valid entries
      const int src_lane = __ffs(pend) - 1;
      pend &= pend - 1u;
      const int Iq = __shfl_sync(0xffffffffu, mine, src_lane);
      const int st = i & 1;
      const uint32_t ep = (uint32_t)(((i >> 1) & 1) ^ 1);
      uint8_t* stage = smem + C::kStageOff + st * C::kStageBytes;
      // dO first: its half of the stage is free once dV(i-2) is done, the
      // Q half (with the constants) only once dK(i-2) is
      if (!mbar_wait_bounded(&bars->qd_empty[st], ep, abort_flag, kWaitLimit)) break;
      mbar_arrive_expect_tx_warp(&bars->qd_full[st], C::kTile);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d_warp(stage + C::kTile + c * (kBlk * 128), &tm_do, &bars->qd_full[st], c * 64, Iq * kBlk, bh);
      nd = i + 1;
      if (!mbar_wait_bounded(&bars->qq_empty[st], ep, abort_flag, kWaitLimit)) break;
      mbar_arrive_expect_tx_warp(&bars->qq_full[st], C::kTile + 1024);
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_3d_warp(stage + c * (kBlk * 128), &tm_q, &bars->qq_full[st], c * 64, Iq * kBlk, bh);
      const long long prow = (long long)bh * padded + (long long)Iq * kBlk;
      bulk_load_warp(stage + 2 * C::kTile, nlse + prow, kBlk * 4, &bars->qq_full[st]);
      bulk_load_warp(stage + 2 * C::kTile + 512, ndelta + prow, kBlk * 4, &bars->qq_full[st]);
      nq = i + 1;
    }
    if (i < n) *abort_flag = 1;
    // copies still in flight: at most the last two of each kind
    for (int w = max(0, nd - 2); w < nd; ++w)
      mbar_wait_timed(&bars->qd_full[w & 1], (uint32_t)((w >> 1) & 1), kDrainLimit);
    for (int w = max(0, nq - 2); w < nq; ++w)
      mbar_wait_timed(&bars->qq_full[w & 1], (uint32_t)((w >> 1) & 1), kDrainLimit);
    if (n > 0) mbar_wait_timed(&bars->kv_full, 0, kDrainLimit);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dk_k = desc_sw128(smem_addr(smem + C::kKOff), 16, 1024);
    const uint64_t dv_k = desc_sw128(smem_addr(smem + C::kVOff), 16, 1024);
    const uint64_t st_k = desc_sw128(smem_addr(smem + C::kStageOff), 16, 1024);
    const uint64_t st_mn = desc_sw128(smem_addr(smem + C::kStageOff), kBlk * 128, 1024);
    const uint64_t pt_k = desc_sw128(smem_addr(smem + C::kPtOff), 16, 1024);
    bool ok = true;
    auto q_off = [](int i) { return (uint64_t)(((i & 1) * C::kStageBytes) >> 4); };
    auto do_off = [](int i) { return (uint64_t)(((i & 1) * C::kStageBytes + C::kTile) >> 4); };
    if (n > 0) {
      ok = mbar_wait_bounded(&bars->kv_full, 0, abort_flag, kWaitLimit) &&
           mbar_wait_bounded(&bars->qq_full[0], 0, abort_flag, kWaitLimit);
      if (ok) {
        issue_nt<D>(tmem + C::kST_col, dk_k, st_k + q_off(0));     // S^T = K Q^T
        mma_commit_warp(&bars->st_full);
        ok = mbar_wait_bounded(&bars->qd_full[0], 0, abort_flag, kWaitLimit);
      }
      if (ok) {
        issue_nt<D>(tmem + C::kDPT_col, dv_k, st_k + do_off(0));   // dP^T = V dO^T
        mma_commit_warp(&bars->dpt_full);
      }
    }
    for (int i = 0; i < n && ok; ++i) {
      if (i + 1 < n) {
        // S^T(i) has been read into registers: S^T(i+1) may overwrite it
        if (!mbar_wait_bounded(&bars->s_read, (uint32_t)(i & 1), abort_flag, kWaitLimit) ||
            !mbar_wait_bounded(&bars->qq_full[(i + 1) & 1], (uint32_t)(((i + 1) >> 1) & 1), abort_flag, kWaitLimit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_nt<D>(tmem + C::kST_col, dk_k, st_k + q_off(i + 1));
        mma_commit_warp(&bars->st_full);
      }
      // P^T(i) was stored by other threads and made visible to the tensor
      // cores (fence.proxy.async) before their arrivals.
      if (!mbar_wait_bounded(&bars->p_ready, (uint32_t)(i & 1), abort_flag, kWaitLimit)) { ok = false; break; }
      issue_ss_tn<D>(tmem + C::kDV_col, pt_k, st_mn + do_off(i), i > 0);   // dV += P^T dO
      mma_commit_warp(&bars->p_free);
      mma_commit_warp(&bars->qd_empty[i & 1]);                                // dO(i) read
      // dS^T(i) was written with tcgen05.st by other threads
      if (!mbar_wait_bounded(&bars->ds_ready, (uint32_t)(i & 1), abort_flag, kWaitLimit)) { ok = false; break; }
      tc_fence_after();
      issue_tn<D>(tmem + C::kDK_col, tmem + C::kDPT_col, st_mn + q_off(i), i > 0);    // dK += dS^T Q
      mma_commit_warp(&bars->qq_empty[i & 1]);                                // Q(i), constants read
      if (i + 1 < n) {
        if (!mbar_wait_bounded(&bars->qd_full[(i + 1) & 1], (uint32_t)(((i + 1) >> 1) & 1), abort_flag, kWaitLimit)) {
          ok = false;
          break;
        }
        issue_nt<D>(tmem + C::kDPT_col, dv_k, st_k + do_off(i + 1));
        mma_commit_warp(&bars->dpt_full);
      }
    }
    if (ok && n > 0) mma_commit_warp(&bars->kv_final);
    mma_commit_warp(&bars->mma_done);
    mbar_wait_timed(&bars->mma_done, 0, kDrainLimit);
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ P/dS warps
    const int g = (warp - 4) >> 2;                  // query-column half
    const int sub = warp & 3;
    const int r = sub * 32 + lane;                  // key row in the block
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const float2 sc2 = make_float2(scale_log2, scale_log2);
    // this thread's row of P^T in slab g (queries 64g .. 64g + 63), 128-byte swizzled
    uint8_t* pt_row = smem + C::kPtOff + g * (kBlk * 128) + (r >> 3) * 1024 + (r & 7) * 128;
    const int sw = r & 7;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int st = i & 1;
      // qq_full: the stage's -lse and -Delta rows, written by the bulk copy
      if (!mbar_wait_bounded(&bars->st_full, (uint32_t)(i & 1), abort_flag, kWaitLimit) ||
          !mbar_wait_bounded(&bars->qq_full[st], (uint32_t)((i >> 1) & 1), abort_flag, kWaitLimit)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* nl = reinterpret_cast<const float*>(smem + C::kStageOff + st * C::kStageBytes + 2 * C::kTile);
      const float* nd = nl + kBlk;
      const uint32_t s_addr = tmem + lane_base + C::kST_col + 64 * g;
      const uint32_t p_addr = tmem + lane_base + C::kDPT_col + 64 * g;
      // phase A: S^T(i) into registers, then P^T = 2^(S^T scale log2 e - lse log2 e)
      uint32_t sr[64];
      {
        uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        tmem_ld32(s_addr, s0);
        tmem_ld32(s_addr + 32, s1);
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_read);
      // dV(i-1) has read P^T(i-1)
      if (i > 0 && !mbar_wait_bounded(&bars->p_free, (uint32_t)((i - 1) & 1), abort_flag, kWaitLimit)) {
        ok = false;
        break;
      }
      float pv[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float4 nl4[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) nl4[v] = *reinterpret_cast<const float4*>(nl + 64 * g + 32 * c + 4 * v);
        uint32_t po[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 nl2 = (e & 1) ? make_float2(nl4[e >> 1].z, nl4[e >> 1].w) : make_float2(nl4[e >> 1].x, nl4[e >> 1].y);
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[32 * c + 2 * e]), __uint_as_float(sr[32 * c + 2 * e + 1])), sc2, nl2);
          pv[32 * c + 2 * e] = ex2(x.x);
          pv[32 * c + 2 * e + 1] = ex2(x.y);
          po[e] = pack_bf16x2(pv[32 * c + 2 * e], pv[32 * c + 2 * e + 1]);
        }
#pragma unroll
        for (int v = 0; v < 4; ++v)
          *reinterpret_cast<uint4*>(pt_row + (((4 * c + v) ^ sw) << 4)) =
              make_uint4(po[4 * v], po[4 * v + 1], po[4 * v + 2], po[4 * v + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready);
      // phase B: dS^T = P^T (dP^T - Delta), packed over dP^T(i)
      if (!mbar_wait_bounded(&bars->dpt_full, (uint32_t)(i & 1), abort_flag, kWaitLimit)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pr[32], so[16];
        tmem_ld32(p_addr + 32 * c, pr);
        float4 nd4[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) nd4[v] = *reinterpret_cast<const float4*>(nd + 64 * g + 32 * c + 4 * v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 nd2 = (e & 1) ? make_float2(nd4[e >> 1].z, nd4[e >> 1].w) : make_float2(nd4[e >> 1].x, nd4[e >> 1].y);
          const float2 t = __fadd2_rn(make_float2(__uint_as_float(pr[2 * e]), __uint_as_float(pr[2 * e + 1])), nd2);
          const float2 ds = __fmul2_rn(make_float2(pv[32 * c + 2 * e], pv[32 * c + 2 * e + 1]), t);
          so[e] = pack_bf16x2(ds.x, ds.y);
        }
        tmem_st16(p_addr + 16 * c, so);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_ready);
    }
    if (ok && n > 0) ok = mbar_wait_bounded(&bars->kv_final, 0, abort_flag, kWaitLimit);
    tc_fence_after();
    const long long krow = (long long)J * kBlk + r;
    const bool store = ok && krow < N;
    const long long roff = ((long long)bh * N + krow) * D + (D / 2) * g;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint32_t raw[32];
      if (n > 0 && ok) {
        tmem_ld32(tmem + lane_base + C::kDV_col + (D / 2) * g + 32 * c, raw);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) raw[e] = 0u;
      }
      store_row32(dv + roff + 32 * c, raw, 1.0f, store);
      if (n > 0 && ok) {
        tmem_ld32(tmem + lane_base + C::kDK_col + (D / 2) * g + 32 * c, raw);
        tmem_wait_ld();
      }
      store_row32(dk + roff + 32 * c, raw, scale, store);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && bars->abort_flag) atomicOr(&g_bwd_flags, (uint32_t)DFS_FLAG_WAIT_TIMEOUT);
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdWs {
  float* nlse;
  float* ndelta;
  uint32_t* bits;
  int32_t* q_cnt;
  int32_t* q_idx;
  size_t bytes;
};

BwdWs carve(const dfs::Dims& d, void* base) {
  const size_t padded = (size_t)d.BH * d.nb * kBlk;
  const int nw = (d.nb + 31) / 32;
  const size_t s0 = round256(padded * 4), s1 = s0, s2 = round256((size_t)d.BH * d.nb * nw * 4),
               s3 = round256((size_t)d.BH * d.nb * 4), s4 = round256((size_t)d.BH * d.nb * d.nb * 4);
  uint8_t* p = static_cast<uint8_t*>(base);
  BwdWs w;
  w.nlse = reinterpret_cast<float*>(p);
  w.ndelta = reinterpret_cast<float*>(p + s0);
  w.bits = reinterpret_cast<uint32_t*>(p + s0 + s1);
  w.q_cnt = reinterpret_cast<int32_t*>(p + s0 + s1 + s2);
  w.q_idx = reinterpret_cast<int32_t*>(p + s0 + s1 + s2 + s3);
  w.bytes = s0 + s1 + s2 + s3 + s4;
  return w;
}

template <int D>
int launch_bwd(const dfs::Dims& d, const void* qp, const void* kp, const void* vp, const void* op, const void* dop,
               const float* lse, const int32_t* kv_idx, const int32_t* kv_cnt, int kcap, float scale, void* dqp,
               void* dkp, void* dvp, const BwdWs& w, cudaStream_t cs) {
  using C = Bw<D>;
  CUtensorMap mq, mk, mv, mdo;
  if (!dfs::make_map_bf16(&mq, qp, d.N, D, d.BH, kBlk) || !dfs::make_map_bf16(&mk, kp, d.N, D, d.BH, kBlk) ||
      !dfs::make_map_bf16(&mv, vp, d.N, D, d.BH, kBlk) || !dfs::make_map_bf16(&mdo, dop, d.N, D, d.BH, kBlk))
    return DFS_ERR_CUDA;
  const int nb = d.nb, nw = (nb + 31) / 32;
  const long long rows = d.BH * nb;                 // list rows (= columns)
  const long long prows = rows * kBlk;              // padded token rows
  const int max_list = min(kcap, nb);
  // A 512-column CTA must be alone on its SM: pad shared memory so that
  // the scheduler never places two.
  const size_t min_smem = 120 * 1024;
  size_t smem_q = 1024 + C::kQBarOff + sizeof(BarsQ) + (size_t)max_list * 4;
  // tiles + the worst case of place_smem_kv: a base 16 bytes past a
  // 1024-byte boundary puts the barriers below the tiles, 1008 bytes on
  static_assert(2 * sizeof(BarsKV) <= 1008, "barrier block too large");
  size_t smem_kv = (size_t)BwKV<D>::kTiles + 1008;
  if (smem_q > 232448 || smem_kv > 232448 || (size_t)8 * nw * 4 > 48 * 1024) return DFS_ERR_UNSUPPORTED;
  smem_q = smem_q < min_smem ? min_smem : smem_q;
  smem_kv = smem_kv < min_smem ? min_smem : smem_kv;
  if (cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_q) !=
          cudaSuccess ||
      cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv) !=
          cudaSuccess)
    return DFS_ERR_CUDA;
  const float scale_log2 = scale * kLog2e;
  constexpr int kRowsPerBlock = 8 * (32 / (D / 8));
  bwd_prep_kernel<D><<<(unsigned)((prows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, cs>>>(
      (const __nv_bfloat16*)op, (const __nv_bfloat16*)dop, lse, (int)d.N, nb, prows, w.nlse, w.ndelta);
  bwd_mask_bits_kernel<<<(unsigned)((rows + 7) / 8), 256, (size_t)8 * nw * 4, cs>>>(kv_idx, kv_cnt, kcap, nb, rows,
                                                                                      nw, w.bits);
  bwd_transpose_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, cs>>>(w.bits, nb, nw, rows, w.q_idx, w.q_cnt);
  const dim3 grid((unsigned)nb, (unsigned)d.BH);
  attn_bwd_dq_kernel<D><<<grid, kThreads, smem_q, cs>>>(mk, mv, (const __nv_bfloat16*)qp, (const __nv_bfloat16*)dop,
                                                         kv_idx, kv_cnt, kcap, (int)d.N, nb, scale, scale_log2,
                                                         w.nlse, w.ndelta, (__nv_bfloat16*)dqp, max_list);
  attn_bwd_dkdv_kernel<D><<<grid, kThreads, smem_kv, cs>>>(mq, mk, mv, mdo, w.q_idx, w.q_cnt, (int)d.N, nb, scale,
                                                            scale_log2, w.nlse, w.ndelta, (__nv_bfloat16*)dkp,
                                                            (__nv_bfloat16*)dvp);
  return dfs::launch_status();
}

}  // namespace

DFS_DEFINE_FLAG_READER(dfs_detail_flags_bwd, g_bwd_flags)

extern "C" size_t dfs_detail_ws_attn_bwd(const dfs_shape* shape) {
  dfs::Dims d;
  if (dfs::check_shape(shape, &d, false) != DFS_OK || d.blk != kBlk) return 0;
  return carve(d, nullptr).bytes;
}

extern "C" int dfs_sparse_attn_bwd(const dfs_shape* shape, const void* qp, const void* kp, const void* vp,
                                   const void* op, const void* dop, const float* lse, const int32_t* kv_idx,
                                   const int32_t* kv_cnt, int kcap, float scale, void* dqp, void* dkp, void* dvp,
                                   void* ws, size_t ws_bytes, dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, false);
  if (st != DFS_OK) return st;
  if (!qp || !kp || !vp || !op || !dop || !lse || !kv_idx || !kv_cnt || !dqp || !dkp || !dvp || kcap < 1)
    return DFS_ERR_INVALID_ARG;
  if (!dfs::aligned16(qp) || !dfs::aligned16(kp) || !dfs::aligned16(vp) || !dfs::aligned16(op) ||
      !dfs::aligned16(dop) || !dfs::aligned16(lse) || !dfs::aligned16(dqp) || !dfs::aligned16(dkp) ||
      !dfs::aligned16(dvp))
    return DFS_ERR_MISALIGNED;
  if (d.blk != kBlk || d.N >= (1LL << 31) || d.BH > 65535 || d.nb > 8192) return DFS_ERR_UNSUPPORTED;
  const BwdWs need = carve(d, nullptr);
  if (!ws || ws_bytes < need.bytes) return DFS_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DFS_ERR_MISALIGNED;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d.D);
  const BwdWs w = carve(d, ws);
  cudaStream_t cs = (cudaStream_t)stream;
  if (d.D == 128) return launch_bwd<128>(d, qp, kp, vp, op, dop, lse, kv_idx, kv_cnt, kcap, scale, dqp, dkp, dvp, w, cs);
  return launch_bwd<64>(d, qp, kp, vp, op, dop, lse, kv_idx, kv_cnt, kcap, scale, dqp, dkp, dvp, w, cs);
}
