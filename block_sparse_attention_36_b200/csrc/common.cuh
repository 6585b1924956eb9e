// Shared host/device helpers of libdfsattn (argument checks, sizes, flags).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "dfsattn.h"

namespace dfs {

struct Dims {
  int B, nh, D, T, H, W, blk, sb;
  long long N;   // tokens
  int nb;        // blocks
  int nsb;       // sub-blocks
  int r;         // sub-blocks per block
  long long BH;  // B * nh
};

// Validates a shape; fills d. Returns DFS_OK or an error status.
inline int check_shape(const dfs_shape* s, Dims* d, bool need_sb) {
  if (!s) return DFS_ERR_INVALID_ARG;
  if (s->B < 1 || s->nh < 1 || s->T < 1 || s->H < 1 || s->W < 1) return DFS_ERR_INVALID_ARG;
  long long N = (long long)s->T * s->H * s->W;
  if (N > (1LL << 30)) return DFS_ERR_UNSUPPORTED;
  if (s->D != 64 && s->D != 128) return DFS_ERR_UNSUPPORTED;
  if (s->blk != 64 && s->blk != 128) return DFS_ERR_UNSUPPORTED;
  if (need_sb) {
    if (s->sb < 1 || s->blk % s->sb != 0) return DFS_ERR_INVALID_ARG;
    int r = s->blk / s->sb;
    if (r != 1 && r != 2 && r != 4 && r != 8) return DFS_ERR_UNSUPPORTED;
  }
  d->B = s->B; d->nh = s->nh; d->D = s->D; d->T = s->T; d->H = s->H; d->W = s->W;
  d->blk = s->blk; d->sb = s->sb;
  d->N = N;
  d->nb = (int)((N + s->blk - 1) / s->blk);
  d->nsb = (s->sb > 0) ? (int)((N + s->sb - 1) / s->sb) : 0;
  d->r = (s->sb > 0) ? s->blk / s->sb : 0;
  d->BH = (long long)s->B * s->nh;
  return DFS_OK;
}

// Unsigned division by a run-time invariant divisor d >= 1 for dividends
// n < 2^31, by multiply-high and shift (Granlund & Montgomery, "Division by
// invariant integers using multiplication", 1994, section 4):
//   l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1,
//   q = (umulhi(m, n) + n) >> l  (the sum taken in 64 bits).
struct FastDiv {
  uint32_t d, m, l;
  FastDiv() : d(1), m(0), l(0) {}
  explicit FastDiv(uint32_t div) : d(div) {
    l = 0;
    while ((1ull << l) < div) ++l;
    m = (uint32_t)((((1ull << l) - div) << 32) / div + 1);
  }
  __host__ __device__ __forceinline__ uint32_t div(uint32_t n) const {
#ifdef __CUDA_ARCH__
    uint32_t t = __umulhi(m, n);
#else
    uint32_t t = (uint32_t)(((uint64_t)m * n) >> 32);
#endif
    return (uint32_t)(((uint64_t)t + n) >> l);
  }
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
  cudaError_t e = cudaPeekAtLastError();
  return e == cudaSuccess ? DFS_OK : DFS_ERR_CUDA;
}

}  // namespace dfs

// Per-translation-unit readers of the device error words (one word per .cu
// file, OR-ed together by dfs_get_error_flags).
extern "C" int dfs_detail_flags_perm(uint32_t* v, int clear);
extern "C" int dfs_detail_flags_score(uint32_t* v, int clear);
extern "C" int dfs_detail_flags_select(uint32_t* v, int clear);
extern "C" int dfs_detail_flags_attn(uint32_t* v, int clear);
extern "C" int dfs_detail_flags_bwd(uint32_t* v, int clear);
// Workspace bytes of dfs_sparse_attn_bwd (0 for an unsupported shape).
extern "C" size_t dfs_detail_ws_attn_bwd(const dfs_shape* shape);

#define DFS_DEFINE_FLAG_READER(NAME, SYMBOL)                                   \
  extern "C" int NAME(uint32_t* v, int clear) {                               \
    uint32_t h = 0;                                                           \
    if (cudaMemcpyFromSymbol(&h, SYMBOL, sizeof(h)) != cudaSuccess)           \
      return DFS_ERR_CUDA;                                                    \
    *v |= h;                                                                  \
    if (clear) {                                                              \
      uint32_t z = 0;                                                         \
      if (cudaMemcpyToSymbol(SYMBOL, &z, sizeof(z)) != cudaSuccess)           \
        return DFS_ERR_CUDA;                                                  \
    }                                                                         \
    return DFS_OK;                                                            \
  }
