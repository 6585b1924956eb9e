/*
 * libdfsattn -- the DFSAttn hot path on one B200 (sm_100a).
 *
 * Dynamic block-sparse spatiotemporal self-attention for video DiTs, as
 * "DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
 * Generation" describes it (Methodology items 1-3): reorder the T x H x W
 * tokens along a global 3D Hilbert curve, score (query block, key block)
 * pairs hierarchically from pooled sub-blocks, keep a budget of key blocks
 * per query block, run block-sparse attention over the kept blocks only,
 * and restore the token order. Two other selection rules share the path:
 * the cumulative-mass threshold of "VMoBA: Mixture of Block Attention for
 * Video Diffusion Models" (abstract, modification 3) and the frame mask of
 * "LVSA: Training-Free Sparse Attention for Long Video Diffusion" (section 2).
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates or frees memory and keeps no state between
 *     calls except a device-side error word (dfs_get_error_flags).
 *   - Every tensor pointer must be 16-byte aligned; otherwise the call
 *     returns DFS_ERR_MISALIGNED.
 *   - Calls are asynchronous and ordered on `stream` (NULL = legacy default
 *     stream). They never synchronise, print, abort or exit.
 *   - The return value is a dfs_status. Argument errors are reported before
 *     anything is launched; DFS_ERR_CUDA means a launch failed (the CUDA
 *     error is left for cudaGetLastError to report).
 *   - bf16 tensors use the IEEE-style bfloat16 layout (uint16 storage).
 *   - Token order: "raster" index n = (t*H + h)*W + w; "curve" index i is the
 *     position along the chosen order; perm[i] = n, inv[n] = i.
 */
#ifndef DFSATTN_H
#define DFSATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st *dfs_stream_t;

typedef enum {
  DFS_OK = 0,
  DFS_ERR_INVALID_ARG = -1, /* null pointer, bad size, inconsistent shape      */
  DFS_ERR_UNSUPPORTED = -2, /* D, blk, blk/sb or nb outside the supported set  */
  DFS_ERR_MISALIGNED = -3,  /* a tensor pointer is not 16-byte aligned          */
  DFS_ERR_CUDA = -4,        /* a kernel launch or a CUDA runtime call failed    */
  DFS_ERR_TIMEOUT = -5,     /* a bounded device wait gave up (see error flags)  */
  DFS_ERR_WORKSPACE = -6    /* workspace missing or smaller than required       */
} dfs_status;

/* Problem shape.
 *   B, nh, D : batch, heads, head dimension (D in {64, 128}).
 *   T, H, W  : token grid; N = T*H*W tokens (N >= 1).
 *   blk      : block size in tokens (64 or 128); nb = ceil(N / blk).
 *   sb       : sub-block size in tokens; blk % sb == 0 and blk/sb in
 *              {1, 2, 4, 8}; nsb = ceil(N / sb).                            */
typedef struct {
  int B, nh, D;
  int T, H, W;
  int blk, sb;
} dfs_shape;

enum {
  DFS_ORDER_RASTER = 0,
  DFS_ORDER_HILBERT3D = 1,
  DFS_ORDER_TILE2D = 2,
  DFS_ORDER_TILE3D = 3,
  DFS_ORDER_HILBERT2D = 4
};
enum { DFS_SEL_TOPK = 0, DFS_SEL_THRESHOLD = 1, DFS_SEL_LVSA = 2, DFS_SEL_GLOBAL = 3, DFS_SEL_RADIAL = 4 };
enum { DFS_WS_BLOCK_SCORE = 0, DFS_WS_ATTN_BWD = 1 };

/* Device error word bits (dfs_get_error_flags). */
enum {
  DFS_FLAG_WAIT_TIMEOUT = 1u << 0, /* an mbarrier wait in the attention kernel gave up */
  DFS_FLAG_BAD_KV_INDEX = 1u << 1, /* kv_idx held a block outside [0, nb): skipped     */
  DFS_FLAG_KCAP_OVERFLOW = 1u << 2 /* a selected list was longer than kcap: truncated */
};

/* Selection settings for dfs_select_mask.
 *   mode = DFS_SEL_TOPK      : keep the k highest-scoring key blocks of each
 *                              row (equal scores: lower block index first).
 *   mode = DFS_SEL_THRESHOLD : p = softmax over the row of the scores; keep
 *                              the fewest best-ranked blocks whose mass
 *                              reaches tau, at most cap of them.
 *   mode = DFS_SEL_LVSA      : scores ignored (may be NULL). Query frame t
 *                              attends to the anchors G_s = {f : (f - s) mod
 *                              lvsa_T_per == 0} (s = lvsa_step) plus the
 *                              (lvsa_C - |G_s|) nearest non-anchor frames
 *                              (distance 0, 1, ..; t-d before t+d). Key block
 *                              J is kept for query block I when a frame J
 *                              touches lies in the union of the frame sets of
 *                              the frames I touches. A frame is H*W tokens of
 *                              the raster order.
 *   mode = DFS_SEL_GLOBAL    : VMoBA global selection (abstract, modification
 *                              2): per head, the k best (query block, key
 *                              block) pairs over all nb * nb of them (equal
 *                              scores: lower flat index I * nb + J first);
 *                              each query block lists its kept key blocks
 *                              ascending and may keep none. k counts pairs
 *                              per head here.
 *   mode = DFS_SEL_RADIAL    : scores ignored (may be NULL). Log-radial
 *                              static mask of DynamicRad (methodology,
 *                              components 1 and 2; static-ratio mode), raster
 *                              order, frames of P = H*W tokens: query token q
 *                              may attend key token k iff
 *                              2 |s_q - s_k| < max(w0 >> bitlen(d), w_far),
 *                              d = |frame(q) - frame(k)|, s = index inside
 *                              the frame, w0 = radial_w0 (>= 0) and
 *                              w_far = floor((double)radial_lambda * w0)
 *                              (radial_lambda >= 0). Key block J is kept
 *                              for query block I when some pair qualifies. */
typedef struct {
  int mode;
  int k;
  int cap;
  float tau;
  int lvsa_T_per, lvsa_C, lvsa_step;
  int radial_w0;
  float radial_lambda;
} dfs_select_params;

/* dfs_hilbert_perm -- token reorder (DFSAttn, Methodology item 1).
 *
 * If build_index != 0, first writes perm[N] and inv[N] (int32, device) for
 * `order`: DFS_ORDER_HILBERT3D is the generalised 3D Hilbert curve over the
 * whole T x H x W box (recursive box splitting; starts at (0,0,0), its major
 * axis is the longest side, ties W, H, T); DFS_ORDER_RASTER is the identity;
 * DFS_ORDER_TILE2D / DFS_ORDER_TILE3D are the 2-D / 3-D block partitions of
 * "VMoBA: Mixture of Block Attention for Video Diffusion Models" (abstract,
 * modification 1), read as tile-major orders: tiles of 1 x 8 x (blk/8)
 * tokens (one frame) or 2 x 8 x (blk/16) tokens, in raster order over the
 * tile grid, clipped at its far edges, raster order inside each tile;
 * DFS_ORDER_HILBERT2D is the 2-D Hilbert order that the DFSAttn ablation
 * (Results, ablation studies) compares against, read as frame-major: the
 * frames whole and in time order, each frame's H x W tokens along the
 * generalised Hilbert curve of the 1 x H x W box (the same path in every
 * frame; the textbook 2-D Hilbert curve on 2^k x 2^k frames).
 * The index depends only on (T, H, W, order): callers build it once and
 * reuse it with build_index = 0.
 * Then gathers each non-NULL input x in {q, k, v}, bf16 [B, N, nh, D]
 * (raster, token-major), into xp in {qp, kp, vp}, bf16 [B, nh, N, D]
 * (curve order, head-major): xp[b, h, i, :] = x[b, perm[i], h, :].
 * An input and its output must be both NULL or both non-NULL.             */
int dfs_hilbert_perm(const dfs_shape *shape, int order, int32_t *perm, int32_t *inv,
                     int build_index, const void *q, const void *k, const void *v,
                     void *qp, void *kp, void *vp, dfs_stream_t stream);

/* dfs_block_score -- hierarchical block scoring (DFSAttn, Methodology item 2).
 *
 * qp, kp: bf16 [B, nh, N, D] in curve order. Pools every run of sb tokens to
 * its mean over the tokens that exist (fp32), then writes
 *   scores[b, h, I, J] = scale * max_{i in I, j in J} qbar_i . kbar_j
 * (fp32 [B, nh, nb, nb]; sub-blocks past N do not exist).
 * scale <= 0 selects 1/sqrt(D).
 * ws: device workspace of at least dfs_workspace_bytes(shape,
 * DFS_WS_BLOCK_SCORE) bytes (the pooled means, fp32 [2, B, nh, nsb, D]);
 * the call overwrites it, and it must stay untouched until the call's
 * kernels finish.                                                          */
int dfs_block_score(const dfs_shape *shape, const void *qp, const void *kp, float scale,
                    float *scores, void *ws, size_t ws_bytes, dfs_stream_t stream);

/* dfs_hilbert_perm_pooled -- dfs_hilbert_perm fused with the first half of
 * dfs_block_score (DFSAttn, Methodology items 1 and 2).
 *
 * Same reorder as dfs_hilbert_perm (q, k, qp, kp required; v and vp both
 * NULL or both given), and in the same pass over the data it writes the
 * sub-block means of the reordered Q and K to ws, fp32 [2, B, nh, nsb, D]
 * (the layout dfs_block_score keeps in its workspace; ws_bytes >=
 * dfs_workspace_bytes(shape, DFS_WS_BLOCK_SCORE)). Needs nh * D / 8 <= 512.
 * Follow it with dfs_block_score_pooled on the same ws.                    */
int dfs_hilbert_perm_pooled(const dfs_shape *shape, int order, int32_t *perm, int32_t *inv,
                            int build_index, const void *q, const void *k, const void *v,
                            void *qp, void *kp, void *vp, void *ws, size_t ws_bytes,
                            dfs_stream_t stream);

/* dfs_block_score_pooled -- the second half of dfs_block_score: block scores
 * from sub-block means already in ws (as dfs_hilbert_perm_pooled writes
 * them); same scale rule and output as dfs_block_score.                   */
int dfs_block_score_pooled(const dfs_shape *shape, float scale, float *scores, const void *ws,
                           size_t ws_bytes, dfs_stream_t stream);

/* dfs_block_score_noalloc -- dfs_block_score without a caller workspace.
 *
 * Not from the pages (they have no counterpart): an entry point for callers
 * that cannot allocate device memory -- for example a plugin whose host
 * hands it only tensors and a stream, or a serving process whose caching
 * allocator has already reserved the device, where a raw cudaMalloc would
 * fail or stall the stream. Same arguments, arithmetic and output as
 * dfs_block_score, but the pooled means live in a buffer compiled into the
 * library: DFS_NOALLOC_SCRATCH_BYTES bytes of device memory, held by every
 * GPU that loads the library until the process exits. A shape that needs
 * more (2 * B * nh * ceil(N / sb) * D * 4 bytes) returns DFS_ERR_WORKSPACE
 * without launching. The call allocates nothing; the first call on a device
 * looks the buffer's device address up once (cudaGetSymbolAddress) with
 * that device current, so make that first call before any stream capture.
 * All calls in the process share the one buffer and it keeps the last
 * call's contents (each call writes every value it later reads, so nothing
 * needs clearing): calls that may overlap on the GPU -- on different
 * streams, or from different threads -- race and must be serialised by the
 * caller.                                                                  */
#define DFS_NOALLOC_SCRATCH_BYTES (32u << 20)
int dfs_block_score_noalloc(const dfs_shape *shape, const void *qp, const void *kp, float scale,
                            float *scores, dfs_stream_t stream);

/* dfs_select_mask -- key-block selection (DFSAttn, Methodology item 3;
 * VMoBA abstract, modification 3; LVSA section 2).
 *
 * scores: fp32 [B, nh, nb, nb] (NULL allowed for DFS_SEL_LVSA and
 * DFS_SEL_RADIAL).
 * Writes, per row (b, h, I), the kept key-block indices in ascending order
 * to kv_idx[((b*nh + h)*nb + I)*kcap + 0 .. cnt-1] (int32) and cnt to
 * kv_cnt[(b*nh + h)*nb + I]. Slots past cnt are not written. kcap >= 1; for
 * top-k and global kcap >= min(k, nb) and for threshold kcap >= min(cap,
 * nb) are checked on the host; a longer list is truncated to kcap and sets
 * DFS_FLAG_KCAP_OVERFLOW.                                                  */
int dfs_select_mask(const dfs_shape *shape, const float *scores, const dfs_select_params *params,
                    int32_t *kv_idx, int32_t *kv_cnt, int kcap, dfs_stream_t stream);

/* dfs_sparse_attn_fwd -- block-sparse attention over the kept blocks
 * (DFSAttn, Methodology item 3 and Significance: block-wise execution).
 *
 * qp, kp, vp: bf16 [B, nh, N, D], curve order. For every query token q of
 * query block I of head (b, h):
 *   op[q] = sum_{k in kept(I), k < N} softmax_k(scale * q.k) v_k
 * with kept(I) the tokens of the blocks kv_idx[row][0 .. kv_cnt[row]-1].
 * A row with kv_cnt == 0 gets op = 0 (and lse = -inf).
 * op: bf16 [B, nh, N, D]. lse (optional, fp32 [B, nh, N]): natural-log
 * sum of exp of the scaled logits. scale <= 0 selects 1/sqrt(D).
 * The softmax runs in fp32, P is rounded to bf16 for the P.V product,
 * accumulation is fp32. Indices outside [0, nb) are skipped and set
 * DFS_FLAG_BAD_KV_INDEX. The two lists a CTA works on are staged in shared
 * memory beside the tiles: for D = 128 and blk = 128, min(kcap, nb) may be
 * at most 4202 (a little over half that with frame-exact masking); a longer
 * list returns DFS_ERR_UNSUPPORTED before anything is launched. Every
 * device wait is bounded; a wait that gives up sets DFS_FLAG_WAIT_TIMEOUT
 * and the kernel returns early.                                           */
int dfs_sparse_attn_fwd(const dfs_shape *shape, const void *qp, const void *kp, const void *vp,
                        const int32_t *kv_idx, const int32_t *kv_cnt, int kcap, float scale,
                        void *op, float *lse, dfs_stream_t stream);

/* Options of dfs_sparse_attn_fwd_ex (zero / NULL members: the defaults). */
typedef struct {
  /* perm (int32 [N], device; the index of dfs_hilbert_perm): write the row
   * of curve position i straight to its raster place o[b, perm[i], h, :],
   * o bf16 [B, N, nh, D] -- the inverse reorder of dfs_unperm fused into
   * the attention epilogue. NULL: o is op, curve order [B, nh, N, D].    */
  const int32_t *perm;
  /* order (int32 [B * nh * nb], device; a permutation of the query rows
   * (b * nh + h) * nb + I, e.g. from dfs_attn_order): CTA c computes rows
   * order[2c] and order[2c + 1]. Only the scheduling changes; with
   * no_tail_split set, every row's result is bitwise that of the default
   * order. NULL: CTAs take blocks 2x, 2x + 1 of one head, head by head.  */
  const int32_t *order;
  /* no_tail_split: 0 (default) lets the launch turn its last, partial wave
   * of two-row CTAs (when it holds at most half as many CTAs as the GPU
   * has SMs) into one-row CTAs that give each half of the row's kept list
   * to one of their two tiles and merge the two partial softmax states --
   * the same rows in about half the time. The merged rows differ from the
   * unsplit ones by rounding only (the halves are those of the counted
   * list, invalid entries included). Nonzero: every CTA takes two rows.
   * dfs_sparse_attn_fwd and dfs_sparse_attn_lvsa_fwd use the default.      */
  int no_tail_split;
  /* test_stall_cycles: testing only, 0 in normal use. Nonzero makes every
   * CTA's MMA-issuing warp first wait, for at most this many SM cycles, on a
   * barrier that nothing arrives at: the wait gives up, the CTA raises
   * DFS_FLAG_WAIT_TIMEOUT, drains the copies and MMAs it started, releases
   * its tensor memory and writes nothing -- the path any wait takes that
   * gives up (a GPU fault is never needed to test it).                    */
  unsigned int test_stall_cycles;
} dfs_attn_opts;

/* dfs_sparse_attn_fwd_ex -- dfs_sparse_attn_fwd with the options above.
 * lse, if given, stays in curve order.                                     */
int dfs_sparse_attn_fwd_ex(const dfs_shape *shape, const void *qp, const void *kp, const void *vp,
                           const int32_t *kv_idx, const int32_t *kv_cnt, int kcap, float scale,
                           const dfs_attn_opts *opts, void *o, float *lse, dfs_stream_t stream);

/* dfs_attn_order -- a work order for dfs_attn_opts.order: within each head
 * the query rows sorted by kept count (kv_cnt clamped to [0, min(kcap,
 * nb)]), largest first, and the heads in order. The longest rows of a head
 * start first and the two rows of a CTA have equal work (longest-processing-
 * time first for lists of uneven length, as threshold and global selection
 * make), while the CTAs running at any time share the keys and values of
 * about two heads, which stay in L2. The sort is stable: rows of equal
 * count stay in ascending row order, so the order -- and with it which rows
 * a launch's last, split wave takes -- is the same on every run, and so is
 * every output bit. One CTA per head, no workspace; min(kcap, nb) must not
 * exceed 29055 (DFS_ERR_UNSUPPORTED).                                       */
int dfs_attn_order(const dfs_shape *shape, const int32_t *kv_cnt, int kcap, int32_t *order, dfs_stream_t stream);

/* dfs_sparse_attn_lvsa_fwd -- frame-exact LVSA attention (LVSA: Training-Free
 * Sparse Attention for Long Video Diffusion, section 2).
 *
 * As dfs_sparse_attn_fwd over the kept blocks (normally the DFS_SEL_LVSA
 * lists), and inside them every (query, key) pair whose key frame is not in
 * the query frame's set A(t) (the rule of DFS_SEL_LVSA, from lvsa's T_per,
 * C and step) is dropped, so each query attends exactly the frames of A(t).
 * Requires raster order (curve order = raster) and H * W >= blk. A query row
 * with no allowed key gets op = 0, lse = -inf.                             */
int dfs_sparse_attn_lvsa_fwd(const dfs_shape *shape, const void *qp, const void *kp, const void *vp,
                             const int32_t *kv_idx, const int32_t *kv_cnt, int kcap, float scale,
                             const dfs_select_params *lvsa, void *op, float *lse, dfs_stream_t stream);

/* dfs_sparse_attn_bwd -- gradients of dfs_sparse_attn_fwd over the same
 * kept lists, as training through block attention needs them (VMoBA:
 * Mixture of Block Attention for Video Diffusion Models, abstract: training
 * speed-ups of the block attention).
 *
 * For a loss L with dL/dO = dop, and P = exp(scale q.k - lse) over the kept
 * keys of each query's block, dP = dO V^T, Delta_q = dO_q . O_q,
 * dS = P (dP - Delta):
 *   dqp = scale dS K,  dkp = scale dS^T Q,  dvp = P^T dO
 * qp, kp, vp, op, dop, dqp, dkp, dvp: bf16 [B, nh, N, D] (curve order);
 * op and lse (fp32 [B, nh, N], natural log) are the forward's outputs for
 * the same lists and scale. Lists must not repeat a block (as produced by
 * dfs_select_mask). P and dS are rounded to bf16 for the tensor-core
 * products, accumulation is fp32, the sums run in a fixed order (the
 * result is deterministic). blk must be 128 (D 64 or 128), nb <= 8192.
 * Workspace: dfs_workspace_bytes(shape, DFS_WS_ATTN_BWD) bytes, 256-byte
 * aligned, owned by the caller and not read before it is written (the
 * per-row constants and the transposed lists). Invalid list entries are
 * skipped and set DFS_FLAG_BAD_KV_INDEX.                                   */
int dfs_sparse_attn_bwd(const dfs_shape *shape, const void *qp, const void *kp, const void *vp,
                        const void *op, const void *dop, const float *lse, const int32_t *kv_idx,
                        const int32_t *kv_cnt, int kcap, float scale, void *dqp, void *dkp, void *dvp,
                        void *ws, size_t ws_bytes, dfs_stream_t stream);

/* dfs_unperm -- inverse reorder: o[b, perm[i], h, :] = op[b, h, i, :],
 * op bf16 [B, nh, N, D] (curve order) -> o bf16 [B, N, nh, D] (raster).   */
int dfs_unperm(const dfs_shape *shape, const int32_t *perm, const void *op, void *o,
               dfs_stream_t stream);

/* Workspace bytes a call needs (0 if none). which: DFS_WS_*. Returns 0 for
 * an invalid shape.                                                        */
size_t dfs_workspace_bytes(const dfs_shape *shape, int which);

/* Reads the device error word of the current device (DFS_FLAG_* bits) into
 * *flags; clears it when clear != 0. Synchronises the current device.     */
int dfs_get_error_flags(uint32_t *flags, int clear);

/* Static text for a dfs_status value. */
const char *dfs_status_string(int status);

/* Library version, e.g. 100 for 0.1.0. */
int dfs_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DFSATTN_H */
