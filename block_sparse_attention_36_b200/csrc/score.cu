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
// Kernel 2 (score): a 128 x 128 tile of pooled logits per CTA computed with
// fp32 FMAs from shared-memory staged operands (8 x 8 per thread), followed
// by the r x r max-pool inside each thread's registers (r = blk/sb divides
// 8, so every pooled group lies inside one thread's 8 x 8 patch).
#include "common.cuh"

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

constexpr int kTile = 128;   // sub-blocks per tile side
constexpr int kKStep = 16;   // head-dim slice staged per iteration
constexpr int kPad = 4;      // smem row padding (floats)

// scores[bh, I, J] = scale * max_{i in I, j in J} sum_d qbar[bh,i,d] kbar[bh,j,d]
// Two shared-memory buffers: the next head-dim slice is read from global
// memory into registers while the current one is multiplied, and the 8 x 8
// register tile is updated with paired fp32 FMAs (two columns per
// instruction; each sum is still one fp32 fma chain over d, as before).
// For R <= 4 a thread's eight columns are two runs of four, 4tx and
// 64 + 4tx, so that a warp's 16-byte column loads are contiguous (without
// bank conflicts); an R x R pool group then stays inside one run. For
// R = 8 the eight columns are consecutive.
template <int R>
__device__ __forceinline__ int score_col(int tx, int jj) {
  return R <= 4 ? (jj < 4 ? tx * 4 + jj : 64 + tx * 4 + jj - 4) : tx * 8 + jj;
}

template <int R>
__global__ void __launch_bounds__(256, 2)
score_kernel(const float* __restrict__ qbar, const float* __restrict__ kbar,
             float* __restrict__ scores, int D, int nsb, int nb, float scale) {
  __shared__ __align__(16) float As[2][kKStep][kTile + kPad];
  __shared__ __align__(16) float Bs[2][kKStep][kTile + kPad];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const long long bh = blockIdx.z;
  const int row0 = blockIdx.y * kTile, col0 = blockIdx.x * kTile;
  const float* qa = qbar + bh * (long long)nsb * D;
  const float* ka = kbar + bh * (long long)nsb * D;
  float2 acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.f, 0.f);

  float4 ga[2], gb[2];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int f = tid + u * 256;
      const int r = f >> 2, c4 = (f & 3) * 4;
      ga[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      gb[u] = ga[u];
      if (row0 + r < nsb) ga[u] = *reinterpret_cast<const float4*>(qa + (long long)(row0 + r) * D + k0 + c4);
      if (col0 + r < nsb) gb[u] = *reinterpret_cast<const float4*>(ka + (long long)(col0 + r) * D + k0 + c4);
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int f = tid + u * 256;
      const int r = f >> 2, c4 = (f & 3) * 4;
      As[buf][c4 + 0][r] = ga[u].x; As[buf][c4 + 1][r] = ga[u].y;
      As[buf][c4 + 2][r] = ga[u].z; As[buf][c4 + 3][r] = ga[u].w;
      Bs[buf][c4 + 0][r] = gb[u].x; Bs[buf][c4 + 1][r] = gb[u].y;
      Bs[buf][c4 + 2][r] = gb[u].z; Bs[buf][c4 + 3][r] = gb[u].w;
    }
  };
  fetch(0);
  stash(0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < D; k0 += kKStep) {
    const bool more = k0 + kKStep < D;
    if (more) fetch(k0 + kKStep);
#pragma unroll
    for (int kk = 0; kk < kKStep; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][score_col<R>(tx, 0)]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][score_col<R>(tx, 4)]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float2 b[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                           make_float2(b1.z, b1.w)};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 ai = make_float2(a[i], a[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __ffma2_rn(ai, b[j], acc[i][j]);
      }
    }
    if (more) {
      stash(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }

  // r x r max-pool within the 8 x 8 patch; sub-blocks past nsb do not exist.
  constexpr int G = 8 / R;
#pragma unroll
  for (int gi = 0; gi < G; ++gi) {
#pragma unroll
    for (int gj = 0; gj < G; ++gj) {
      float m = -INFINITY;
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) {
          const int sr = row0 + ty * 8 + gi * R + i, sc = col0 + score_col<R>(tx, gj * R + j);
          const int cc = gj * R + j;
          const float2 pr = acc[gi * R + i][cc >> 1];
          if (sr < nsb && sc < nsb) m = fmaxf(m, (cc & 1) ? pr.y : pr.x);
        }
      const int I = (row0 + ty * 8) / R + gi, J = (col0 + score_col<R>(tx, gj * R)) / R;
      if (I < nb && J < nb) scores[(bh * nb + I) * (long long)nb + J] = m * scale;
    }
  }
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
  const unsigned tiles = (unsigned)((d.nsb + kTile - 1) / kTile);
  dim3 sg(tiles, tiles, (unsigned)d.BH);
  switch (d.r) {
    case 1: score_kernel<1><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    case 2: score_kernel<2><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    case 4: score_kernel<4><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    default: score_kernel<8><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
  }
  return dfs::launch_status();
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
  const unsigned tiles = (unsigned)((d.nsb + kTile - 1) / kTile);
  dim3 sg(tiles, tiles, (unsigned)d.BH);
  switch (d.r) {
    case 1: score_kernel<1><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    case 2: score_kernel<2><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    case 4: score_kernel<4><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    default: score_kernel<8><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
  }
  return dfs::launch_status();
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
  const unsigned tiles = (unsigned)((d.nsb + kTile - 1) / kTile);
  dim3 sg(tiles, tiles, (unsigned)d.BH);
  switch (d.r) {
    case 1: score_kernel<1><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    case 2: score_kernel<2><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    case 4: score_kernel<4><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
    default: score_kernel<8><<<sg, 256, 0, cs>>>(qbar, kbar, scores, d.D, d.nsb, d.nb, scale); break;
  }
  return dfs::launch_status();
}
