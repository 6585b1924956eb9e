// Token reorder along the global 3D Hilbert curve and its inverse.
//
// DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
// Generation, Methodology item 1: tokens are reordered along one global 3D
// Hilbert curve before attention, keeping spatiotemporal neighbours close
// and memory access contiguous.
//
// Curve: the generalised Hilbert curve of an arbitrary box, built by
// recursive splitting (the published "gilbert" construction). A box is an
// entry cell p plus three orthogonal axis-parallel vectors a (major), b, c;
// its path starts at p and ends one step short of p + a. Boxes with two unit
// sides are walked straight; otherwise the sides are halved (rounded toward
// zero, then made even when the side exceeds 2) and the box is cut into 2,
// 3 or 5 sub-boxes depending on its aspect ratio (wide: 2w > 3h and 2w > 3d;
// tall: 3h > 4d; deep: 3d > 4h; else regular). Here each thread finds the
// cell of one curve rank by descending into the sub-box that holds it, so
// the index kernel needs no traversal and no scratch memory.
//
// Gather / scatter: 16-byte vector loads and stores. A token-major row of
// nh*D bf16 values is contiguous in the raster layout; a head's D values of
// consecutive curve positions are contiguous in the head-major layout, so
// both sides move whole 256-byte (D = 128) or 128-byte (D = 64) runs.
#include "common.cuh"

namespace {

__device__ uint32_t g_perm_flags;

// An axis-parallel vector: coordinate index (0 = t, 1 = h, 2 = w) and signed
// length along it.
struct Axis {
  int dim;
  int len;
};

__device__ __forceinline__ int alen(Axis a) { return a.len < 0 ? -a.len : a.len; }
__device__ __forceinline__ int asign(Axis a) { return a.len < 0 ? -1 : 1; }
__device__ __forceinline__ Axis aneg(Axis a) { return Axis{a.dim, -a.len}; }
// a - b for parallel a, b.
__device__ __forceinline__ Axis aminus(Axis a, Axis b) { return Axis{a.dim, a.len - b.len}; }
// a shortened by one unit step (the vector to its last cell).
__device__ __forceinline__ Axis alast(Axis a) { return Axis{a.dim, a.len - asign(a)}; }
__device__ __forceinline__ Axis ahalf(Axis a) {
  int n = alen(a);
  int h = n >> 1;
  if ((h & 1) && n > 2) ++h;
  return Axis{a.dim, a.len < 0 ? -h : h};
}

struct Box {
  int p[3];
  Axis a, b, c;
};

__device__ __forceinline__ long long box_volume(const Box& x) {
  return (long long)alen(x.a) * alen(x.b) * alen(x.c);
}

__device__ __forceinline__ void shift(int p[3], Axis v) { p[v.dim] += v.len; }

__device__ __forceinline__ Box make_box(const int p[3], Axis o1, Axis o2, Axis o3,
                                        Axis a, Axis b, Axis c) {
  Box x;
  x.p[0] = p[0]; x.p[1] = p[1]; x.p[2] = p[2];
  shift(x.p, o1); shift(x.p, o2); shift(x.p, o3);
  x.a = a; x.b = b; x.c = c;
  return x;
}

// Cell (t, h, w) at rank r of the curve over box `top`.
__device__ void hilbert_cell(Box cur, long long r, int out[3]) {
  const Axis zero{0, 0};
  for (int guard = 0; guard < 256; ++guard) {
    const int w = alen(cur.a), h = alen(cur.b), d = alen(cur.c);
    if (h == 1 && d == 1) { cur.p[cur.a.dim] += asign(cur.a) * (int)r; break; }
    if (w == 1 && d == 1) { cur.p[cur.b.dim] += asign(cur.b) * (int)r; break; }
    if (w == 1 && h == 1) { cur.p[cur.c.dim] += asign(cur.c) * (int)r; break; }
    const Axis a2 = ahalf(cur.a), b2 = ahalf(cur.b), c2 = ahalf(cur.c);
    Box kids[5];
    int nk;
    if (2 * w > 3 * h && 2 * w > 3 * d) {
      kids[0] = make_box(cur.p, zero, zero, zero, a2, cur.b, cur.c);
      kids[1] = make_box(cur.p, a2, zero, zero, aminus(cur.a, a2), cur.b, cur.c);
      nk = 2;
    } else if (3 * h > 4 * d) {
      kids[0] = make_box(cur.p, zero, zero, zero, b2, cur.c, a2);
      kids[1] = make_box(cur.p, b2, zero, zero, cur.a, aminus(cur.b, b2), cur.c);
      kids[2] = make_box(cur.p, alast(cur.a), alast(b2), zero, aneg(b2), cur.c,
                         aneg(aminus(cur.a, a2)));
      nk = 3;
    } else if (3 * d > 4 * h) {
      kids[0] = make_box(cur.p, zero, zero, zero, c2, a2, cur.b);
      kids[1] = make_box(cur.p, c2, zero, zero, cur.a, cur.b, aminus(cur.c, c2));
      kids[2] = make_box(cur.p, alast(cur.a), alast(c2), zero, aneg(c2),
                         aneg(aminus(cur.a, a2)), cur.b);
      nk = 3;
    } else {
      kids[0] = make_box(cur.p, zero, zero, zero, b2, c2, a2);
      kids[1] = make_box(cur.p, b2, zero, zero, cur.c, a2, aminus(cur.b, b2));
      kids[2] = make_box(cur.p, alast(b2), alast(cur.c), zero, cur.a, aneg(b2),
                         aneg(aminus(cur.c, c2)));
      kids[3] = make_box(cur.p, alast(cur.a), b2, alast(cur.c), aneg(cur.c),
                         aneg(aminus(cur.a, a2)), aminus(cur.b, b2));
      kids[4] = make_box(cur.p, alast(cur.a), alast(b2), zero, aneg(b2), c2,
                         aneg(aminus(cur.a, a2)));
      nk = 5;
    }
    int pick = nk - 1;
    for (int i = 0; i < nk; ++i) {
      const long long v = box_volume(kids[i]);
      if (r < v) { pick = i; break; }
      r -= v;
    }
    cur = kids[pick];
  }
  out[0] = cur.p[0]; out[1] = cur.p[1]; out[2] = cur.p[2];
}

// Cell of rank i in tile-major order (tiles of ct x ch x cw in raster order,
// clipped at the far edges; raster order inside a tile). Every time slab of
// tiles before the last is full, every row of tiles before the last in a
// slab is full, and so on, so each level is one division.
__device__ __forceinline__ long long tiled_cell(long long i, int T, int H, int W, int ct, int ch, int cw) {
  const long long slab = (long long)ct * H * W;
  const long long a = i / slab;
  long long r = i - a * slab;
  const int tt = min(ct, T - (int)a * ct);
  const long long row = (long long)tt * ch * W;
  const long long b = r / row;
  r -= b * row;
  const int hh = min(ch, H - (int)b * ch);
  const long long cube = (long long)tt * hh * cw;
  const long long c = r / cube;
  r -= c * cube;
  const int ww = min(cw, W - (int)c * cw);
  const long long t = a * ct + r / ((long long)hh * ww);
  const long long h = b * ch + (r / ww) % hh;
  const long long w = c * cw + r % ww;
  return (t * H + h) * W + w;
}

__global__ void hilbert_index_kernel(int T, int H, int W, int order, int ct, int ch, int cw,
                                     int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  const long long N = (long long)T * H * W;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  long long n;
  if (order == DFS_ORDER_RASTER) {
    n = i;
  } else if (order == DFS_ORDER_TILE2D || order == DFS_ORDER_TILE3D) {
    n = tiled_cell(i, T, H, W, ct, ch, cw);
    if (n < 0 || n >= N) n = 0;  // unreachable for valid shapes; keeps the write in bounds
  } else {
    // 3-D: the curve of the whole T x H x W box. 2-D (frame-major): frame
    // t = i / (H W) in time order, its tokens along the curve of the
    // 1 x H x W box (the same path in every frame).
    const bool two_d = order == DFS_ORDER_HILBERT2D;
    const long long P = (long long)H * W;
    const int Tb = two_d ? 1 : T;
    const long long t0 = two_d ? i / P : 0;
    const long long rank = two_d ? i - t0 * P : i;
    // Major axis: the longest side, ties to W, then H, then T; the other two
    // in the order W, H, T.
    Axis aw{2, W}, ah{1, H}, at{0, Tb};
    Box top;
    top.p[0] = top.p[1] = top.p[2] = 0;
    if (W >= H && W >= Tb) { top.a = aw; top.b = ah; top.c = at; }
    else if (H >= Tb) { top.a = ah; top.b = aw; top.c = at; }
    else { top.a = at; top.b = aw; top.c = ah; }
    int cell[3];
    hilbert_cell(top, rank, cell);
    cell[0] += (int)t0;
    n = ((long long)cell[0] * H + cell[1]) * W + cell[2];
    if (cell[0] < 0 || cell[0] >= T || cell[1] < 0 || cell[1] >= H || cell[2] < 0 || cell[2] >= W)
      n = 0;  // unreachable for valid shapes; keeps the write in bounds
  }
  perm[i] = (int32_t)n;
  inv[n] = (int32_t)i;
}

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 8;

// Moves 16-byte vectors between the token-major layout [B, N, nh*D] and the
// head-major layout [B, nh, N, D] through perm.
//   to_curve = true : dst_headmajor[b, h, i, :] = src_tokmajor[b, perm[i], h, :]
//   to_curve = false: dst_tokmajor[b, perm[i], h, :] = src_headmajor[b, h, i, :]
// The flat work index e runs over (b, i, vec) with vec = h * (D/8) + d8
// (e < 2^31, checked on the host); each thread handles kCopyUnroll vectors
// spaced kCopyThreads apart and issues all its loads before its stores.
template <bool kToCurve>
__global__ void __launch_bounds__(kCopyThreads)
permute_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                    const int32_t* __restrict__ perm, uint32_t N, uint32_t nh, uint32_t dvec,
                    dfs::FastDiv div_vpt, dfs::FastDiv div_n, dfs::FastDiv div_dvec,
                    uint32_t total) {
  const uint32_t vpt = nh * dvec;  // vectors per token
  const uint32_t base = blockIdx.x * (kCopyThreads * kCopyUnroll) + threadIdx.x;
  uint4 val[kCopyUnroll];
  long long dst_off[kCopyUnroll];
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u) {
    const uint32_t e = base + (uint32_t)u * kCopyThreads;
    dst_off[u] = -1;
    if (e < total) {
      const uint32_t tok = div_vpt.div(e);      // flat (b, i)
      const uint32_t vec = e - tok * vpt;
      const uint32_t b = div_n.div(tok);
      const uint32_t i = tok - b * N;
      const uint32_t h = div_dvec.div(vec);
      const uint32_t d8 = vec - h * dvec;
      const long long n = perm[i];
      const long long tokmajor = ((long long)b * N + n) * vpt + vec;
      const long long headmajor = (((long long)b * nh + h) * N + i) * dvec + d8;
      if (kToCurve) {
        val[u] = __ldg(src + tokmajor);
        dst_off[u] = headmajor;
      } else {
        val[u] = __ldg(src + headmajor);
        dst_off[u] = tokmajor;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kCopyUnroll; ++u)
    if (dst_off[u] >= 0) dst[dst_off[u]] = val[u];
}

int launch_copy(bool to_curve, const void* src, void* dst, const int32_t* perm, const dfs::Dims& d,
                cudaStream_t st) {
  const int dvec = d.D / 8;
  const long long total = (long long)d.B * d.N * d.nh * dvec;
  if (total >= (1LL << 31)) return DFS_ERR_UNSUPPORTED;
  const long long per_block = (long long)kCopyThreads * kCopyUnroll;
  const unsigned grid = (unsigned)((total + per_block - 1) / per_block);
  const dfs::FastDiv dv((uint32_t)(d.nh * dvec)), dn((uint32_t)d.N), dd((uint32_t)dvec);
  if (to_curve)
    permute_copy_kernel<true><<<grid, kCopyThreads, 0, st>>>(
        (const uint4*)src, (uint4*)dst, perm, (uint32_t)d.N, d.nh, dvec, dv, dn, dd, (uint32_t)total);
  else
    permute_copy_kernel<false><<<grid, kCopyThreads, 0, st>>>(
        (const uint4*)src, (uint4*)dst, perm, (uint32_t)d.N, d.nh, dvec, dv, dn, dd, (uint32_t)total);
  return dfs::launch_status();
}

// Gather of Q, K, V into curve order fused with the sub-block means of Q and
// K. One CTA per (sub-block j, batch b, tensor): thread v owns one 16-byte
// column (head h, eight dims) and walks the sub-block's tokens in order, so
// the column sum needs no cross-thread reduction; loads of eight tokens are
// in flight per thread. pooled: fp32 [2, B, nh, nsb, D] (Q then K).
template <int D>
__global__ void __launch_bounds__(512)
gather_pool_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
                   uint4* __restrict__ qp, uint4* __restrict__ kp, uint4* __restrict__ vp,
                   const int32_t* __restrict__ perm, float* __restrict__ pooled, int N, int nh, int sb, int nsb,
                   int B) {
  constexpr int kDvec = D / 8;
  const int vpt = nh * kDvec;
  const int col = threadIdx.x;
  if (col >= vpt) return;
  const int j = blockIdx.x, b = blockIdx.y, tsel = blockIdx.z;  // tensor: 0 Q, 1 K, 2 V
  const uint4* src = tsel == 0 ? q : (tsel == 1 ? k : v);
  uint4* dst = tsel == 0 ? qp : (tsel == 1 ? kp : vp);
  if (!src) return;
  const int h = col / kDvec, d8 = col - h * kDvec;
  const int i0 = j * sb, i1 = min(i0 + sb, N);
  const uint4* s_base = src + (long long)b * N * vpt + col;
  uint4* d_base = dst + ((long long)(b * nh + h) * N) * kDvec + d8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int i = i0; i < i1; i += 8) {
    uint4 val[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int ii = i + u;
      if (ii < i1) val[u] = __ldg(s_base + (long long)__ldg(perm + ii) * vpt);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int ii = i + u;
      if (ii < i1) {
        d_base[(long long)ii * kDvec] = val[u];
        if (tsel < 2) {
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&val[u]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            acc[2 * e] += f.x;
            acc[2 * e + 1] += f.y;
          }
        }
      }
    }
  }
  if (tsel < 2) {
    const float fc = (float)(i1 - i0);
    float* out = pooled + ((((long long)tsel * B + b) * nh + h) * nsb + j) * D + d8 * 8;
    reinterpret_cast<float4*>(out)[0] =
        make_float4(__fdiv_rn(acc[0], fc), __fdiv_rn(acc[1], fc), __fdiv_rn(acc[2], fc), __fdiv_rn(acc[3], fc));
    reinterpret_cast<float4*>(out)[1] =
        make_float4(__fdiv_rn(acc[4], fc), __fdiv_rn(acc[5], fc), __fdiv_rn(acc[6], fc), __fdiv_rn(acc[7], fc));
  }
}

bool valid_order(int order) {
  return order == DFS_ORDER_RASTER || order == DFS_ORDER_HILBERT3D || order == DFS_ORDER_TILE2D ||
         order == DFS_ORDER_TILE3D || order == DFS_ORDER_HILBERT2D;
}

// Tile extents of the tiled orders (blk tokens per full tile).
void tile_dims(int order, int blk, int* ct, int* ch, int* cw) {
  if (order == DFS_ORDER_TILE2D) { *ct = 1; *ch = 8; *cw = blk / 8; }
  else if (order == DFS_ORDER_TILE3D) { *ct = 2; *ch = 8; *cw = blk / 16; }
  else { *ct = *ch = *cw = 1; }
}

}  // namespace

DFS_DEFINE_FLAG_READER(dfs_detail_flags_perm, g_perm_flags)

extern "C" int dfs_hilbert_perm(const dfs_shape* shape, int order, int32_t* perm, int32_t* inv,
                                int build_index, const void* q, const void* k, const void* v,
                                void* qp, void* kp, void* vp, dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, false);
  if (st != DFS_OK) return st;
  if (!valid_order(order)) return DFS_ERR_INVALID_ARG;
  if (!perm || (build_index && !inv)) return DFS_ERR_INVALID_ARG;
  const void* srcs[3] = {q, k, v};
  void* dsts[3] = {qp, kp, vp};
  for (int t = 0; t < 3; ++t) {
    if ((srcs[t] == nullptr) != (dsts[t] == nullptr)) return DFS_ERR_INVALID_ARG;
    if (srcs[t] && (!dfs::aligned16(srcs[t]) || !dfs::aligned16(dsts[t]))) return DFS_ERR_MISALIGNED;
  }
  cudaStream_t cs = (cudaStream_t)stream;
  if (build_index) {
    const int threads = 256;
    const long long grid = (d.N + threads - 1) / threads;
    int ct = 1, ch = 1, cw = 1;
    tile_dims(order, d.blk, &ct, &ch, &cw);
    hilbert_index_kernel<<<(unsigned)grid, threads, 0, cs>>>(d.T, d.H, d.W, order, ct, ch, cw, perm, inv);
    st = dfs::launch_status();
    if (st != DFS_OK) return st;
  }
  for (int t = 0; t < 3; ++t) {
    if (!srcs[t]) continue;
    st = launch_copy(true, srcs[t], dsts[t], perm, d, cs);
    if (st != DFS_OK) return st;
  }
  return DFS_OK;
}

extern "C" int dfs_unperm(const dfs_shape* shape, const int32_t* perm, const void* op, void* o,
                          dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, false);
  if (st != DFS_OK) return st;
  if (!perm || !op || !o) return DFS_ERR_INVALID_ARG;
  if (!dfs::aligned16(op) || !dfs::aligned16(o)) return DFS_ERR_MISALIGNED;
  return launch_copy(false, op, o, perm, d, (cudaStream_t)stream);
}

extern "C" int dfs_hilbert_perm_pooled(const dfs_shape* shape, int order, int32_t* perm, int32_t* inv,
                                       int build_index, const void* q, const void* k, const void* v, void* qp,
                                       void* kp, void* vp, void* ws, size_t ws_bytes, dfs_stream_t stream) {
  dfs::Dims d;
  int st = dfs::check_shape(shape, &d, true);
  if (st != DFS_OK) return st;
  if (!valid_order(order)) return DFS_ERR_INVALID_ARG;
  if (!perm || (build_index && !inv)) return DFS_ERR_INVALID_ARG;
  if (!q || !k || !qp || !kp) return DFS_ERR_INVALID_ARG;
  if ((v == nullptr) != (vp == nullptr)) return DFS_ERR_INVALID_ARG;
  const void* ptrs[6] = {q, k, v, qp, kp, vp};
  for (const void* p : ptrs)
    if (p && !dfs::aligned16(p)) return DFS_ERR_MISALIGNED;
  const size_t need = (size_t)2 * d.BH * d.nsb * d.D * sizeof(float);
  if (!ws || ws_bytes < need) return DFS_ERR_WORKSPACE;
  if (!dfs::aligned16(ws)) return DFS_ERR_MISALIGNED;
  const int vpt = d.nh * (d.D / 8);
  if (vpt > 512 || d.B > 65535 || d.N >= (1LL << 31)) return DFS_ERR_UNSUPPORTED;
  cudaStream_t cs = (cudaStream_t)stream;
  if (build_index) {
    const int threads = 256;
    const long long grid = (d.N + threads - 1) / threads;
    int ct = 1, ch = 1, cw = 1;
    tile_dims(order, d.blk, &ct, &ch, &cw);
    hilbert_index_kernel<<<(unsigned)grid, threads, 0, cs>>>(d.T, d.H, d.W, order, ct, ch, cw, perm, inv);
    st = dfs::launch_status();
    if (st != DFS_OK) return st;
  }
  const int threads = ((vpt + 31) / 32) * 32;
  dim3 grid((unsigned)d.nsb, (unsigned)d.B, v ? 3u : 2u);
  if (d.D == 128)
    gather_pool_kernel<128><<<grid, threads, 0, cs>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, (uint4*)qp,
                                                      (uint4*)kp, (uint4*)vp, perm, (float*)ws, (int)d.N, d.nh,
                                                      d.sb, d.nsb, d.B);
  else
    gather_pool_kernel<64><<<grid, threads, 0, cs>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, (uint4*)qp,
                                                     (uint4*)kp, (uint4*)vp, perm, (float*)ws, (int)d.N, d.nh,
                                                     d.sb, d.nsb, d.B);
  return dfs::launch_status();
}
