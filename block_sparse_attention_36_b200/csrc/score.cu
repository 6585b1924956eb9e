// Hierarchical block scoring.
//
// DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
// Generation, Methodology item 2: blocks are split into sub-blocks, scores
// are computed at sub-block level and aggregated into a block importance.
// Here: pooled sub-block means of Q and K (fp32), pooled logits
// qbar_i . kbar_j, and the maximum of the logits over the sub-block pairs of
// each (query block, key block), times the softmax scale.
//
// Kernel 1 (pool): one warp per sub-block streams its sb x D bf16 tile with
// 16-byte loads (8 values per lane) and keeps fp32 sums; HBM-bound.
// Kernel 2 (score): the pooled logits of a 128 x 256 tile of (query,
// key) sub-blocks are one dense product qbar_tile . kbar_tile^T over D, run
// on the tensor cores (tcgen05, kind::tf32, accumulator in tensor memory).
// Each fp32 operand x is split into x_hi = tf32(x) and x_lo = tf32(x - x_hi)
// and the product is taken as a_lo b_hi + a_hi b_lo + a_hi b_hi (the
// dropped a_lo b_lo and the rounding of the lo parts are below 2^-22 of
// |a||b| per term, i.e. fp32-level accuracy). The r x r max-pool runs in the
// epilogue: r columns inside a thread's row, r rows across r lanes.
#include "common.cuh"
#include "sm100_ptx.cuh"

namespace {

__device__ uint32_t g_score_flags;

// pooled[t, bh, j, :] = mean over the tokens of sub-block j of x_t[bh, :, :]
// for t in {0 (Q), 1 (K)}; sums run over tokens in order per lane and the two
// (D = 128) or four (D = 64) partial sums of a column are added pairwise.
template <int D>
__global__ void __launch_bounds__(256)
pool_kernel(const __nv_bfloat16* __restrict__ qp, const __nv_bfloat16* __restrict__ kp,
            float* __restrict__ pooled, long long N, int sb, int nsb, long long BH) {
  constexpr int kLanesPerRow = D / 8;             // 16-byte vectors per token row
  constexpr int kRowsPerIter = 32 / kLanesPerRow; // token rows one warp reads at once
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gw = (long long)blockIdx.x * 8 + warp;   // global sub-block job
  const int t = blockIdx.y;                                  // 0 = Q, 1 = K
  if (gw >= BH * nsb) return;
  const long long bh = gw / nsb;
  const int j = (int)(gw - bh * nsb);
  const __nv_bfloat16* src = (t == 0 ? qp : kp) + (bh * N) * D;
  const long long lo = (long long)j * sb;
  const long long hi = min(lo + sb, N);
  const int cnt = (int)(hi - lo);
  const int col = (lane % kLanesPerRow) * 8;
  const int rsub = lane / kLanesPerRow;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  constexpr int kU = 8;  // loads in flight per lane
  for (long long row0 = lo + rsub; row0 < hi; row0 += (long long)kRowsPerIter * kU) {
    uint4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long long row = row0 + (long long)u * kRowsPerIter;
      v[u] = row < hi ? __ldg(reinterpret_cast<const uint4*>(src + row * D + col))
                      : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int off = kLanesPerRow; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (rsub == 0) {
    float* dst = pooled + (((long long)t * BH + bh) * nsb + j) * D + col;
    const float fc = (float)cnt;
    float4 o0 = make_float4(__fdiv_rn(acc[0], fc), __fdiv_rn(acc[1], fc), __fdiv_rn(acc[2], fc),
                            __fdiv_rn(acc[3], fc));
    float4 o1 = make_float4(__fdiv_rn(acc[4], fc), __fdiv_rn(acc[5], fc), __fdiv_rn(acc[6], fc),
                            __fdiv_rn(acc[7], fc));
    reinterpret_cast<float4*>(dst)[0] = o0;
    reinterpret_cast<float4*>(dst)[1] = o1;
  }
}

using namespace dfs::sm100;

constexpr int kSM = 128;                    // query sub-blocks per tile (MMA M)
constexpr int kSN = 256;                    // key sub-blocks per tile (MMA N)
constexpr int kScoreThreads = 256;
constexpr int kQSlab = kSM * 128;           // one 32-column fp32 slab of the query tile, bytes
constexpr int kKSlab = kSN * 128;           // the same for the key tile
constexpr int kScoreSmem = 1024 + 2 * kQSlab + 2 * kKSlab;   // + alignment slack
constexpr long long kScoreWait = 2000000000ll;   // SM clock cycles per wait (about 1 s)

// scores[bh, I, J] = scale * max_{i in I, j in J} sum_d qbar[bh,i,d] kbar[bh,j,d]
// One CTA per 128 x 256 tile of sub-block pairs (two CTAs per SM, 256
// tensor-memory columns each). The head dimension is walked in slabs of 32
// fp32 columns (one 128-byte row per sub-block): every thread loads its
// share of the slab from global memory into registers, splits it into tf32
// hi and lo parts and stores both into 128-byte-swizzled shared-memory
// tiles (the 16-byte chunk c of row r at r * 128 + ((c ^ (r & 7)) << 4),
// the layout the MMA descriptors expect); one warp then issues the slab's
// 3 x 4 MMAs (K = 8 each) and commits them, and the next slab's loads are
// in flight while they run.
template <int D, int R>
__global__ void __launch_bounds__(kScoreThreads, 2)
score_tc_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar, float* __restrict__ scores,
                int nsb, int nb, float scale) {
  extern __shared__ uint8_t score_smem[];
  __shared__ __align__(8) uint64_t mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  constexpr int kSlabs = D / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long bh = blockIdx.z;
  const int row0 = blockIdx.y * kSM, col0 = blockIdx.x * kSN;
  const uint32_t raw = smem_addr(score_smem);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* tiles = score_smem + (base - raw);
  uint8_t* q_hi = tiles;
  uint8_t* q_lo = tiles + kQSlab;
  uint8_t* k_hi = tiles + 2 * kQSlab;
  uint8_t* k_lo = k_hi + kKSlab;

  if (warp == 0) tmem_alloc(&tmem_slot, 256);
  if (tid == 0) {
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    fence_barrier_init();
  }

  const float* qa = qbar + bh * (long long)nsb * D;
  const float* ka = kbar + bh * (long long)nsb * D;
  // slab s: query rows r < 128 and key rows r < 256, eight 16-byte chunks
  // per row; thread t takes the chunks t, t + 256, ... of the slab
  float4 rq[kSM * 8 / kScoreThreads], rk[kSN * 8 / kScoreThreads];
  auto fetch = [&](int slab) {
#pragma unroll
    for (int u = 0; u < kSM * 8 / kScoreThreads; ++u) {
      const int f = tid + u * kScoreThreads, r = f >> 3, c = f & 7;
      rq[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (row0 + r < nsb) rq[u] = __ldg(reinterpret_cast<const float4*>(qa + (long long)(row0 + r) * D + slab * 32 + c * 4));
    }
#pragma unroll
    for (int u = 0; u < kSN * 8 / kScoreThreads; ++u) {
      const int f = tid + u * kScoreThreads, r = f >> 3, c = f & 7;
      rk[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (col0 + r < nsb) rk[u] = __ldg(reinterpret_cast<const float4*>(ka + (long long)(col0 + r) * D + slab * 32 + c * 4));
    }
  };
  auto split_store = [&](const float4& x, uint8_t* hi, uint8_t* lo, int f) {
    const int r = f >> 3, c = f & 7;
    const int off = r * 128 + ((c ^ (r & 7)) << 4);
    float4 h, l;
    h.x = round_tf32(x.x); l.x = round_tf32(x.x - h.x);
    h.y = round_tf32(x.y); l.y = round_tf32(x.y - h.y);
    h.z = round_tf32(x.z); l.z = round_tf32(x.z - h.z);
    h.w = round_tf32(x.w); l.w = round_tf32(x.w - h.w);
    *reinterpret_cast<float4*>(hi + off) = h;
    *reinterpret_cast<float4*>(lo + off) = l;
  };

  fetch(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  constexpr uint32_t idesc = idesc_tf32_f32(kSM, kSN);
#pragma unroll 1
  for (int slab = 0; slab < kSlabs; ++slab) {
    if (slab > 0) {
      // the previous slab's MMAs have read the tiles
      mbar_wait_bounded(&mma_done, (slab - 1) & 1, &abort_flag, kScoreWait);
      tc_fence_after();
    }
#pragma unroll
    for (int u = 0; u < kSM * 8 / kScoreThreads; ++u) split_store(rq[u], q_hi, q_lo, tid + u * kScoreThreads);
#pragma unroll
    for (int u = 0; u < kSN * 8 / kScoreThreads; ++u) split_store(rk[u], k_hi, k_lo, tid + u * kScoreThreads);
    fence_proxy_async_smem();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t o = kk * 32;   // K = 8 fp32 columns = 32 bytes along the swizzled row
        const uint64_t aq_hi = desc_sw128(smem_addr(q_hi) + o, 16, 1024);
        const uint64_t aq_lo = desc_sw128(smem_addr(q_lo) + o, 16, 1024);
        const uint64_t bk_hi = desc_sw128(smem_addr(k_hi) + o, 16, 1024);
        const uint64_t bk_lo = desc_sw128(smem_addr(k_lo) + o, 16, 1024);
        mma_ss_tf32_warp(tmem, aq_lo, bk_hi, idesc, (slab > 0 || kk > 0) ? 1u : 0u);
        mma_ss_tf32_warp(tmem, aq_hi, bk_lo, idesc, 1u);
        mma_ss_tf32_warp(tmem, aq_hi, bk_hi, idesc, 1u);
      }
      mma_commit_warp(&mma_done);
    }
    if (slab + 1 < kSlabs) fetch(slab + 1);
  }
  if (!mbar_wait_bounded(&mma_done, (kSlabs - 1) & 1, &abort_flag, kScoreWait))
    atomicOr(&g_score_flags, DFS_FLAG_WAIT_TIMEOUT);
  tc_fence_after();

  // epilogue: warp w reads tensor-memory lanes 32 (w & 3) .. + 31 (its
  // query sub-block rows) and columns 128 (w >> 2) .. + 127 in chunks of 32
  const int quarter = warp & 3, half = warp >> 2;
  const int srow = row0 + quarter * 32 + lane;
  const bool row_ok = srow < nsb;
#pragma unroll 1
  for (int ch = 0; ch < 4; ++ch) {
    const int cbase = half * 128 + ch * 32;
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)cbase, v);
    tmem_wait_ld();
    float m[32 / R];
#pragma unroll
    for (int g = 0; g < 32 / R; ++g) {
      m[g] = -INFINITY;
#pragma unroll
      for (int j = 0; j < R; ++j)
        if (row_ok && col0 + cbase + g * R + j < nsb) m[g] = fmaxf(m[g], __uint_as_float(v[g * R + j]));
    }
#pragma unroll
    for (int off = 1; off < R; off <<= 1)
#pragma unroll
      for (int g = 0; g < 32 / R; ++g) m[g] = fmaxf(m[g], __shfl_xor_sync(0xffffffffu, m[g], off));
    const int I = srow / R;
    if (lane % R == 0 && I < nb) {
      float* dst = scores + (bh * nb + I) * (long long)nb;
#pragma unroll
      for (int g = 0; g < 32 / R; ++g) {
        const int J = (col0 + cbase) / R + g;
        if (J < nb) dst[J] = m[g] * scale;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    if (abort_flag) mbar_wait_timed(&mma_done, (kSlabs - 1) & 1, kScoreWait);
    tmem_dealloc(tmem, 256);
  }
}

template <int D, int R>
int launch_score_tc(const dfs::Dims& d, const float* qbar, const float* kbar, float* scores, float scale,
                    cudaStream_t cs) {
  if (cudaFuncSetAttribute(score_tc_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoreSmem) !=
      cudaSuccess)
    return DFS_ERR_CUDA;
  const dim3 grid((unsigned)((d.nsb + kSN - 1) / kSN), (unsigned)((d.nsb + kSM - 1) / kSM), (unsigned)d.BH);
  score_tc_kernel<D, R><<<grid, kScoreThreads, kScoreSmem, cs>>>(qbar, kbar, scores, d.nsb, d.nb, scale);
  return dfs::launch_status();
}

template <int D>
int launch_score_d(const dfs::Dims& d, const float* qbar, const float* kbar, float* scores, float scale,
                   cudaStream_t cs) {
  switch (d.r) {
    case 1: return launch_score_tc<D, 1>(d, qbar, kbar, scores, scale, cs);
    case 2: return launch_score_tc<D, 2>(d, qbar, kbar, scores, scale, cs);
    case 4: return launch_score_tc<D, 4>(d, qbar, kbar, scores, scale, cs);
    default: return launch_score_tc<D, 8>(d, qbar, kbar, scores, scale, cs);
  }
}

// Block scores from pooled means qbar, kbar ([BH, nsb, D] fp32 each).
int launch_score(const dfs::Dims& d, const float* qbar, const float* kbar, float* scores, float scale,
                 cudaStream_t cs) {
  return d.D == 128 ? launch_score_d<128>(d, qbar, kbar, scores, scale, cs)
                    : launch_score_d<64>(d, qbar, kbar, scores, scale, cs);
}

}  // namespace

DFS_DEFINE_FLAG_READER(dfs_detail_flags_score, g_score_flags)

extern "C" size_t dfs_workspace_bytes(const dfs_shape* shape, int which) {
  dfs::Dims d;
  if (which == DFS_WS_ATTN_BWD) return dfs_detail_ws_attn_bwd(shape);
  if (which != DFS_WS_BLOCK_SCORE) return 0;
  if (dfs::check_shape(shape, &d, true) != DFS_OK) return 0;
  return (size_t)2 * d.BH * d.nsb * d.D * sizeof(float);
}

extern "C" int dfs_block_score(const dfs_shape* shape, const void* qp, const void* kp, float scale,
                               float* scores, void* ws, size_t ws_bytes, dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, true);
  if (st != DFS_OK) return st;
  if (!qp || !kp || !scores) return DFS_ERR_INVALID_ARG;
  if (!dfs::aligned16(qp) || !dfs::aligned16(kp) || !dfs::aligned16(scores)) return DFS_ERR_MISALIGNED;
  const size_t need = dfs_workspace_bytes(shape, DFS_WS_BLOCK_SCORE);
  if (!ws || ws_bytes < need) return DFS_ERR_WORKSPACE;
  if (!dfs::aligned16(ws)) return DFS_ERR_MISALIGNED;
  if (d.BH > 65535) return DFS_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d.D);
  cudaStream_t cs = (cudaStream_t)stream;
  float* pooled = (float*)ws;
  const long long jobs = d.BH * d.nsb;
  dim3 pg((unsigned)((jobs + 7) / 8), 2);
  if (d.D == 128)
    pool_kernel<128><<<pg, 256, 0, cs>>>((const __nv_bfloat16*)qp, (const __nv_bfloat16*)kp, pooled,
                                         d.N, d.sb, d.nsb, d.BH);
  else
    pool_kernel<64><<<pg, 256, 0, cs>>>((const __nv_bfloat16*)qp, (const __nv_bfloat16*)kp, pooled,
                                        d.N, d.sb, d.nsb, d.BH);
  st = dfs::launch_status();
  if (st != DFS_OK) return st;
  const float* qbar = pooled;
  const float* kbar = pooled + d.BH * d.nsb * d.D;
  return launch_score(d, qbar, kbar, scores, scale, cs);
}

extern "C" int dfs_block_score_pooled(const dfs_shape* shape, float scale, float* scores, const void* ws,
                                      size_t ws_bytes, dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, true);
  if (st != DFS_OK) return st;
  if (!scores) return DFS_ERR_INVALID_ARG;
  if (!dfs::aligned16(scores)) return DFS_ERR_MISALIGNED;
  const size_t need = (size_t)2 * d.BH * d.nsb * d.D * sizeof(float);
  if (!ws || ws_bytes < need) return DFS_ERR_WORKSPACE;
  if (!dfs::aligned16(ws)) return DFS_ERR_MISALIGNED;
  if (d.BH > 65535) return DFS_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d.D);
  cudaStream_t cs = (cudaStream_t)stream;
  const float* qbar = (const float*)ws;
  const float* kbar = qbar + d.BH * d.nsb * d.D;
  return launch_score(d, qbar, kbar, scores, scale, cs);
}

// ---------------------------------------------------------------------------
// dfs_block_score_noalloc: the same two kernels, with the pooled means kept
// in a buffer compiled into the library instead of a caller workspace, for
// callers that cannot allocate device memory (see include/dfsattn.h).
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr size_t kNoallocScratchBytes = DFS_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DFS_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DFS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DFS_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return DFS_OK;
}

}  // namespace

extern "C" int dfs_block_score_noalloc(const dfs_shape* shape, const void* qp, const void* kp, float scale,
                                       float* scores, dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, true);
  if (st != DFS_OK) return st;
  if (!qp || !kp || !scores) return DFS_ERR_INVALID_ARG;
  if (!dfs::aligned16(qp) || !dfs::aligned16(kp) || !dfs::aligned16(scores)) return DFS_ERR_MISALIGNED;
  const size_t need = (size_t)2 * d.BH * d.nsb * d.D * sizeof(float);
  if (need > kNoallocScratchBytes) return DFS_ERR_WORKSPACE;   // beyond the built-in buffer
  if (d.BH > 65535) return DFS_ERR_UNSUPPORTED;
  float* pooled = nullptr;
  st = noalloc_scratch(&pooled);
  if (st != DFS_OK) return st;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d.D);
  cudaStream_t cs = (cudaStream_t)stream;
  // Every pooled value the score kernel reads is written first by the pool
  // kernel on the same stream, so the buffer needs no clearing.
  const long long jobs = d.BH * d.nsb;
  dim3 pg((unsigned)((jobs + 7) / 8), 2);
  if (d.D == 128)
    pool_kernel<128><<<pg, 256, 0, cs>>>((const __nv_bfloat16*)qp, (const __nv_bfloat16*)kp, pooled,
                                         d.N, d.sb, d.nsb, d.BH);
  else
    pool_kernel<64><<<pg, 256, 0, cs>>>((const __nv_bfloat16*)qp, (const __nv_bfloat16*)kp, pooled,
                                        d.N, d.sb, d.nsb, d.BH);
  st = dfs::launch_status();
  if (st != DFS_OK) return st;
  const float* qbar = pooled;
  const float* kbar = pooled + d.BH * d.nsb * d.D;
  return launch_score(d, qbar, kbar, scores, scale, cs);
}
