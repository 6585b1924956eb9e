// Block-sparse attention forward over the kept key blocks (sm_100a).
//
// DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
// Generation, Methodology item 3 and Significance: after the mask is chosen,
// attention runs block-wise over the kept blocks only, on the reordered,
// contiguous token blocks.
//
// One CTA computes one 128-row query tile (one query block; for 64-token
// blocks the lower 64 rows) of one head against the key blocks of its list.
// Warp roles (192 threads):
//   warp 0     TMA producer: Q once, then K and V tiles of each kept block
//              into a 2-stage ring (128-byte swizzled tiles, no multicast).
//   warp 1     owns tensor memory; one lane issues the tcgen05 MMAs:
//                S_j = Q K_j^T  (SS, into TMEM buffer j % 2)
//                O  += P_j V_j  (TS: P_j read back from TMEM, V_j MN-major)
//              issuing S_{j+1} before waiting for P_j, so the tensor pipe
//              works on the next logits while the softmax runs.
//   warps 2-5  softmax, one thread per query row: fp32 online softmax on S
//              read from TMEM, P_j written back into S_j's columns as bf16;
//              O is rescaled in TMEM only when the running row maximum grows
//              by more than 2^8 (an older maximum is exact as long as the
//              same one is used for P and for the row sum); epilogue
//              normalises O and writes bf16 rows (and the log-sum-exp).
// Tensor memory: S0 | S1 | O  (BLK + BLK + D fp32 columns, 128 lanes).
// Every mbarrier wait is bounded (DFS_FLAG_WAIT_TIMEOUT, early return).
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace {

using namespace dfs::sm100;

__device__ uint32_t g_attn_flags;

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per pipeline wait
constexpr uint64_t kDrainLimitNs = 1000000000ull;  // 1 s per drain wait
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kQRows = 128;  // MMA M

template <int D, int BLK>
struct Cfg {
  static constexpr int kChunks = D / 64;                   // 128-byte column slabs per row
  static constexpr int kQBytes = kQRows * D * 2;
  static constexpr int kKVBytes = BLK * D * 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;
  static constexpr int kVOff = kKOff + kStages * kKVBytes;
  static constexpr int kBarOff = kVOff + kStages * kKVBytes;
  static constexpr int kTmemCols = (2 * BLK + D <= 256) ? 256 : 512;
  static constexpr int kS0 = 0, kS1 = BLK, kO = 2 * BLK;
};

struct __align__(8) Barriers {
  uint64_t q_full;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_ready, o_final;
  uint32_t tmem_base;
  int abort_flag;
  int n_kv;
};

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ kv_idx,
                const int32_t* __restrict__ kv_cnt, int kcap, int N, int nb, float scale_log2,
                __nv_bfloat16* __restrict__ op, float* __restrict__ lse, int max_list) {
  using C = Cfg<D, BLK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled tiles.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::kBarOff);
  int32_t* list = reinterpret_cast<int32_t*>(smem + C::kBarOff + sizeof(Barriers));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int I = blockIdx.x;
  const int bh = blockIdx.y;
  const long long row_id = (long long)bh * nb + I;
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], 4);
    }
    mbar_init(&bars->o_ready, 1);
    mbar_init(&bars->o_final, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    // Compact the kept list into shared memory, dropping invalid indices.
    int cnt = kv_cnt[row_id];
    cnt = max(0, min(cnt, min(kcap, max_list)));
    const int32_t* src = kv_idx + row_id * (long long)kcap;
    int base = 0;
    bool bad = false;
    for (int j0 = 0; j0 < cnt; j0 += 32) {
      const int j = j0 + lane;
      int J = -1;
      if (j < cnt) J = src[j];
      const bool ok = (j < cnt) && J >= 0 && J < nb;
      bad |= (j < cnt) && !ok;
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      if (ok) list[base + __popc(m & ((1u << lane) - 1u))] = J;
      base += __popc(m);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_attn_flags, (uint32_t)DFS_FLAG_BAD_KV_INDEX);
    if (lane == 0) bars->n_kv = base;
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_kv = bars->n_kv;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensor_map(&tm_q);
      prefetch_tensor_map(&tm_k);
      prefetch_tensor_map(&tm_v);
      mbar_arrive_expect_tx(&bars->q_full, C::kQBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d(smem + C::kQOff + c * (kQRows * 128), &tm_q, &bars->q_full, c * 64, I * BLK, bh);
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % kStages;
        const uint32_t ph = (uint32_t)((j / kStages) & 1);
        const int J = list[j];
        if (!mbar_wait_bounded(&bars->k_empty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], C::kKVBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(smem + C::kKOff + s * C::kKVBytes + c * (BLK * 128), &tm_k, &bars->k_full[s], c * 64,
                      J * BLK, bh);
        issued_k = j + 1;
        if (!mbar_wait_bounded(&bars->v_empty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], C::kKVBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(smem + C::kVOff + s * C::kKVBytes + c * (BLK * 128), &tm_v, &bars->v_full[s], c * 64,
                      J * BLK, bh);
        issued_v = j + 1;
      }
      // Drain: every load issued must land before the CTA may exit. A stage
      // is reloaded only after its previous load was consumed, so only the
      // last kStages loads of each ring can still be in flight.
      for (int j = max(0, issued_k - kStages); j < issued_k; ++j)
        mbar_wait_timed(&bars->k_full[j % kStages], (uint32_t)((j / kStages) & 1), kDrainLimitNs);
      for (int j = max(0, issued_v - kStages); j < issued_v; ++j)
        mbar_wait_timed(&bars->v_full[j % kStages], (uint32_t)((j / kStages) & 1), kDrainLimitNs);
      mbar_wait_timed(&bars->q_full, 0, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kQRows, BLK, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kQRows, D, 1);
      const uint32_t q_base = smem_addr(smem + C::kQOff);
      const uint32_t k_base = smem_addr(smem + C::kKOff);
      const uint32_t v_base = smem_addr(smem + C::kVOff);
      bool ok = mbar_wait_bounded(&bars->q_full, 0, abort_flag, kWaitLimitNs);
      auto issue_pv = [&](int jj) -> bool {
        const int b = jj & 1, s = jj % kStages;
        const uint32_t ph = (uint32_t)((jj / kStages) & 1);
        if (!mbar_wait_bounded(&bars->p_full[b], (uint32_t)((jj >> 1) & 1), abort_flag, kWaitLimitNs)) return false;
        if (!mbar_wait_bounded(&bars->v_full[s], ph, abort_flag, kWaitLimitNs)) return false;
        tc_fence_after();
        const uint32_t p_tmem = tmem + (b ? C::kS1 : C::kS0);
        const uint32_t vs = v_base + s * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk) {
          const uint64_t bdesc = desc_sw128(vs + kk * 2048, BLK * 128, 1024);
          mma_ts(tmem + C::kO, p_tmem + kk * 8, bdesc, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars->v_empty[s]);
        mma_commit(&bars->o_ready);
        return true;
      };
      for (int j = 0; ok && j < n_kv; ++j) {
        const int s = j % kStages, b = j & 1;
        const uint32_t ph = (uint32_t)((j / kStages) & 1);
        if (!mbar_wait_bounded(&bars->k_full[s], ph, abort_flag, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ks = k_base + s * C::kKVBytes;
        const uint32_t s_tmem = tmem + (b ? C::kS1 : C::kS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2, w = kk & 3;
          const uint64_t adesc = desc_sw128(q_base + c * (kQRows * 128) + w * 32, 16, 1024);
          const uint64_t bdesc = desc_sw128(ks + c * (BLK * 128) + w * 32, 16, 1024);
          mma_ss(s_tmem, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[b]);
        mma_commit(&bars->k_empty[s]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && n_kv > 0) issue_pv(n_kv - 1);
      mma_commit(&bars->o_final);
      // Every MMA of this CTA must finish before tensor memory is released.
      mbar_wait_timed(&bars->o_final, 0, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int sub = warp & 3;                        // TMEM lane quarter of this warp
    const int r = sub * 32 + lane;                   // query row in the tile
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const int rem = N - (nb - 1) * BLK;              // valid keys in the last block
    float m = -INFINITY;                             // running max (log2 units)
    float l = 0.f;                                   // running row sum
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int b = j & 1;
      if (!mbar_wait_bounded(&bars->s_full[b], (uint32_t)((j >> 1) & 1), abort_flag, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + (b ? C::kS1 : C::kS0);
      float sv[BLK];
#pragma unroll
      for (int c = 0; c < BLK / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(s_addr + c * 32, raw);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(raw[e]);
      }
      const int J = list[j];
      if (J == nb - 1 && rem < BLK) {
#pragma unroll
        for (int e = 0; e < BLK; ++e)
          if (e >= rem) sv[e] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < BLK; ++e) mx = fmaxf(mx, sv[e]);
      const float m_blk = mx * scale_log2;
      // Keep the old maximum unless it is more than 2^8 below the new one
      // somewhere in this warp; then the warp rescales O and its sums.
      bool rescale = false;
      float m_use;
      if (j == 0) {
        m_use = m_blk;
      } else {
        rescale = __any_sync(0xffffffffu, m_blk > m + 8.0f);
        m_use = rescale ? fmaxf(m, m_blk) : m;
      }
      // P = exp2(s * scale_log2 - m), bf16, written over S_j's first columns
      // (S_j is fully read already; PV_{j-1} reads the other buffer).
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < BLK / 64; ++c) {
        uint32_t packed[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2(fmaf(sv[c * 64 + 2 * e], scale_log2, -m_use));
          const float p1 = ex2(fmaf(sv[c * 64 + 2 * e + 1], scale_log2, -m_use));
          rs += p0 + p1;
          packed[e] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_addr + c * 32, packed);
      }
      // One o_ready phase per iteration: PV_{j-1} has finished with O.
      if (j >= 1) {
        if (!mbar_wait_bounded(&bars->o_ready, (uint32_t)((j - 1) & 1), abort_flag, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
      }
      if (rescale) {
        const float alpha = ex2(m - m_use);
        const uint32_t o_addr = tmem + lane_base + C::kO;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(o_addr + c * 32, raw);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
          tmem_st32(o_addr + c * 32, raw);
        }
        l *= alpha;
      }
      tmem_wait_st();
      m = m_use;
      l += rs;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[b]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) ok = mbar_wait_bounded(&bars->o_final, 0, abort_flag, kWaitLimitNs);
    tc_fence_after();
    const long long qrow = (long long)I * BLK + r;
    const bool store = ok && r < BLK && qrow < N;
    __nv_bfloat16* orow = op + ((long long)bh * N + qrow) * D;
    const float inv_l = (n_kv > 0 && l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t raw[32];
      if (n_kv > 0) {
        tmem_ld32(tmem + lane_base + C::kO + c * 32, raw);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) raw[e] = 0u;
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * inv_l, __uint_as_float(raw[2 * e + 1]) * inv_l);
      if (store) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      }
    }
    if (store && lse) {
      // natural-log LSE of the scaled logits: (m + log2 l) * ln 2
      lse[(long long)bh * N + qrow] = (n_kv > 0) ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && bars->abort_flag) atomicOr(&g_attn_flags, (uint32_t)DFS_FLAG_WAIT_TIMEOUT);
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [BH, N, D] bf16 viewed as a 3-D tensor (D fastest); box = 64 x rows x 1.
bool make_map(CUtensorMap* map, const void* base, long long N, int D, long long BH, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int BLK>
int launch_attn(const dfs::Dims& d, const void* qp, const void* kp, const void* vp, const int32_t* kv_idx,
                const int32_t* kv_cnt, int kcap, float scale, void* op, float* lse, cudaStream_t st) {
  using C = Cfg<D, BLK>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, qp, d.N, D, d.BH, kQRows) || !make_map(&mk, kp, d.N, D, d.BH, BLK) ||
      !make_map(&mv, vp, d.N, D, d.BH, BLK))
    return DFS_ERR_CUDA;
  const int max_list = min(kcap, d.nb);
  size_t smem = 1024 + C::kBarOff + sizeof(Barriers) + (size_t)max_list * sizeof(int32_t);
  if (smem > 232448) return DFS_ERR_UNSUPPORTED;
  // Tensor memory per SM is 512 columns: a 512-column CTA must be alone on
  // its SM and a 256-column CTA may share it with one other, so shared
  // memory is padded to make the scheduler place CTAs that way.
  const size_t min_smem = (C::kTmemCols == 512) ? 120 * 1024 : 80 * 1024;
  if (smem < min_smem) smem = min_smem;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return DFS_ERR_CUDA;
  dim3 grid((unsigned)d.nb, (unsigned)d.BH);
  const float scale_log2 = scale * 1.4426950408889634f;
  attn_fwd_kernel<D, BLK><<<grid, kThreads, smem, st>>>(mq, mk, mv, kv_idx, kv_cnt, kcap, (int)d.N, d.nb,
                                                        scale_log2, (__nv_bfloat16*)op, lse, max_list);
  return dfs::launch_status();
}

}  // namespace

DFS_DEFINE_FLAG_READER(dfs_detail_flags_attn, g_attn_flags)

extern "C" int dfs_sparse_attn_fwd(const dfs_shape* shape, const void* qp, const void* kp, const void* vp,
                                   const int32_t* kv_idx, const int32_t* kv_cnt, int kcap, float scale, void* op,
                                   float* lse, dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, false);
  if (st != DFS_OK) return st;
  if (!qp || !kp || !vp || !kv_idx || !kv_cnt || !op || kcap < 1) return DFS_ERR_INVALID_ARG;
  if (!dfs::aligned16(qp) || !dfs::aligned16(kp) || !dfs::aligned16(vp) || !dfs::aligned16(op) ||
      (lse && !dfs::aligned16(lse)))
    return DFS_ERR_MISALIGNED;
  if (d.N >= (1LL << 31) || d.BH > 65535 || d.nb > 0x7fffffff) return DFS_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d.D);
  cudaStream_t cs = (cudaStream_t)stream;
  if (d.D == 128 && d.blk == 128) return launch_attn<128, 128>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, cs);
  if (d.D == 128 && d.blk == 64) return launch_attn<128, 64>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, cs);
  if (d.D == 64 && d.blk == 128) return launch_attn<64, 128>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, cs);
  return launch_attn<64, 64>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, cs);
}
