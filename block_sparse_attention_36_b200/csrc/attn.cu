// Block-sparse attention forward over the kept key blocks (sm_100a).
//
// DFSAttn: Dynamic Fine-grained Sparse Attention for Efficient Video
// Generation, Methodology item 3 and Significance: after the mask is chosen,
// attention runs block-wise over the kept blocks only, on the reordered,
// contiguous token blocks.
//
// A CTA owns two query tiles ("slots" A and B: query blocks 2x and 2x+1 of
// one head, or rows order[2x], order[2x+1] of a work order), each with its
// own kept list. While the softmax of one slot runs, the tensor pipe works
// on the other slot's products, so neither the tensor pipe nor the
// exponential units wait on each other for long. The CTAs of a last,
// partial wave may instead each take one query block and give each slot
// half of its kept list; the two softmax warpgroups then merge their
// (max, sum, O) in the epilogue, so that wave takes about half as long.
// Warp roles (384 threads, three warpgroups):
//   thread 0   initialises the barriers and starts the Q_A, Q_B loads at
//              once (they depend only on the block index).
//   warp 0     TMA producer: the K and V tiles of both lists into a 4-stage
//              ring, in exactly the order the MMAs consume them (128-byte
//              swizzled tiles, no multicast).
//   warp 1     owns tensor memory; one lane issues the tcgen05 MMAs, per
//              slot X and kept block j:
//                S_X = Q_X K_j^T  (SS)            into TMEM S_X
//                O_X += P_X V_j   (TS: P_X from TMEM, V MN-major)
//              ordered S_A(0) S_B(0), then per j: PV_A(j) S_A(j+1)
//              PV_B(j) S_B(j+1); S_X(j+1) overwrites P_X(j) only after
//              PV_X(j) read it (tcgen05 MMAs of one thread run in order).
//              With 128-key blocks, PV_X(j) starts on keys 0-63 of P as
//              soon as the softmax releases them (p_half) and finishes on
//              keys 64-127 after p_full.
//   warps 2-3  compact the two kept lists into shared memory, then idle.
//   warps 4-7  softmax of slot A, warps 8-11 softmax of slot B: one thread
//              per query row; fp32 online softmax on S read from TMEM,
//              P written back as bf16 over S_X; O_X is rescaled in TMEM
//              only when a warp's running maximum grows by more than 2^8
//              (an older maximum stays exact as long as P and the row sum
//              use the same one); epilogue normalises O_X and stores bf16
//              rows (in curve order, or straight to raster order through
//              perm) and the log-sum-exp; in a split CTA slot B passes its
//              (max, sum) through shared memory and slot A reads O_B from
//              tensor memory and writes the merged rows.
// Tensor memory: S_A | S_B | O_A | O_B (BLK, BLK, D, D fp32 columns).
// Every mbarrier wait is bounded (DFS_FLAG_WAIT_TIMEOUT, early return);
// copies and MMAs in flight are drained before tensor memory is released.
#include "common.cuh"
#include "exp2_poly.cuh"
#include "lvsa.cuh"
#include "sm100_ptx.cuh"
#include "tmap.cuh"

// Every DFS_ATTN_EXP2_EMU-th pair of softmax exponentials is computed on the
// FMA pipe (0: all on the special-function unit).
#ifndef DFS_ATTN_EXP2_EMU
#define DFS_ATTN_EXP2_EMU 0
#endif

namespace {

using namespace dfs::sm100;

__device__ uint32_t g_attn_flags;

// Wait limits in SM clock cycles (about 2 s and 1 s at the 2 GHz maximum).
constexpr long long kWaitLimit = 4000000000ll;   // per pipeline wait
constexpr long long kDrainLimit = 2000000000ll;  // per drain wait
constexpr int kRing = 4;                           // K/V ring stages
constexpr int kThreads = 384;                      // 3 warpgroups
// Warp-specialised register split of the 512-column (blk 128) kernels, which
// are launched at the 168-register cap of 384 threads: warpgroup 0
// (producer, MMA issuer, list warps) gives registers back and the two
// softmax warpgroups take them (setmaxnreg), which removes the softmax's
// spills. 128 * 80 + 256 * 208 = 63,488 <= 384 * 168 = 64,512 registers;
// the launch checks the kernel's register count against this before it
// runs (an increase beyond the block's registers would never complete).
constexpr int kRegWg0 = 80;
constexpr int kRegSoftmax = 208;
constexpr int kQRows = 128;                        // MMA M

template <int D, int BLK>
struct Cfg {
  static constexpr int kChunks = D / 64;          // 128-byte column slabs per row
  static constexpr int kQBytes = kQRows * D * 2;  // one slot's Q tile
  static constexpr int kTileBytes = BLK * D * 2;  // one K or V tile
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kQBytes;
  static constexpr int kBarOff = kRingOff + kRing * kTileBytes;
  static constexpr int kCols = 2 * BLK + 2 * D;
  static constexpr int kTmemCols = kCols <= 256 ? 256 : 512;
  __host__ __device__ static constexpr int s_col(int x) { return x * BLK; }
  __host__ __device__ static constexpr int o_col(int x) { return 2 * BLK + x * D; }
};

struct __align__(8) Barriers {
  uint64_t q_full[2];
  uint64_t kv_full[kRing], kv_empty[kRing];
  uint64_t s_full[2], p_half[2], p_full[2], o_final[2];
  uint64_t mma_done;
  uint64_t stall;          // nothing ever arrives here (the abort-path test)
  uint32_t tmem_base;
  int abort_flag;
  int n_kv[2];
};

// S = Q K^T for one 128-row query tile and one key tile: D/16 MMAs of
// K = 16; dq, dk describe the first 16 columns of the 128-byte-swizzled tiles.
template <int D, int BLK>
__device__ __forceinline__ void issue_s(uint32_t d_tmem, uint64_t dq, uint64_t dk) {
  constexpr uint32_t idesc = idesc_bf16_f32(kQRows, BLK, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t oa = (uint64_t)(((kk >> 2) * (kQRows * 128) + (kk & 3) * 32) >> 4);
    const uint64_t ob = (uint64_t)(((kk >> 2) * (BLK * 128) + (kk & 3) * 32) >> 4);
    mma_ss_warp(d_tmem, dq + oa, dk + ob, idesc, kk > 0 ? 1u : 0u);
  }
}

// O (+)= P V for one query tile: P (bf16) from tensor memory, V MN-major in
// shared memory; BLK/16 MMAs of K = 16.
// K steps [KK0, KK1) only: the first half of P can be consumed while the
// second half is still being formed.
template <int D, int BLK, int KK0, int KK1>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t dv, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(kQRows, D, 1);
#pragma unroll
  for (int kk = KK0; kk < KK1; ++kk)
    mma_ts_warp(o_tmem, p_tmem + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// Frame-exact LVSA masking inside the kept blocks (raster token order, P
// tokens per frame, P >= BLK so a block touches at most two frames and the
// 2 * BLK query rows of a CTA at most three). The CTA first tabulates, for
// each of its query frames, the bit set A(t) over all T key frames in
// shared memory; the softmax then masks by two bit lookups per key block.
struct FrameMask {
  int P, T, T_per, s0, C, nG;
};
// Output rows go to op in curve order, or, when perm is set, straight to
// their raster place o[b, perm[i], h, :] (o: [B, N, nh, D]).
// Query rows are numbered by a virtual index v. With a work order, v is the
// row (b * nh + h) * nb + I at order[v] (rows = B * nh * nb entries);
// without one, v = 2 (bh * P + x) + e is block 2x + e of head bh, with
// P = ceil(nb / 2) (block nb: an empty slot). CTA c < split_from takes rows
// 2c and 2c + 1, one per slot. A CTA c >= split_from takes the one row
// 2 split_from + (c - split_from) and gives each slot half of its kept list;
// the epilogue merges the two partial softmax states. The host sets
// split_from so that the last, partial wave of two-row CTAs becomes twice
// as many half-length CTAs (tail_split) or leaves it at the CTA count.
// stall_cycles > 0 (tests only): the MMA-issuing warp first waits that many
// SM cycles on the barrier `stall`, which nothing arrives at, so the launch
// runs the abort path of a bounded wait that gives up.
struct OutMap {
  const int32_t* perm;
  int nh;
  const int32_t* order;
  long long rows;
  int tail_split;
  long long split_from;
  long long stall_cycles;
};

constexpr int kFrameRows = 3;
constexpr int kMaxFrames = 4096;
__host__ __device__ constexpr int frame_words(int T) { return (T + 31) / 32; }

template <int D, int BLK, int EMU, bool FRAME>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ kv_idx,
                const int32_t* __restrict__ kv_cnt, int kcap, int N, int nb, float scale_log2,
                __nv_bfloat16* __restrict__ op, float* __restrict__ lse, int max_list, FrameMask fm,
                OutMap om) {
  using C = Cfg<D, BLK>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Barriers* bars = reinterpret_cast<Barriers*>(smem + C::kBarOff);
  int32_t* lists = reinterpret_cast<int32_t*>(smem + C::kBarOff + sizeof(Barriers));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // (head, query block) of each slot; an empty slot gets block nb
  const long long cta = blockIdx.x;
  const bool split = cta >= om.split_from;          // one row, half of its list per slot
  const long long v0 = split ? 2 * om.split_from + (cta - om.split_from) : 2 * cta;
  const long long v1 = split ? v0 : v0 + 1;
  auto decode = [&](long long v, int& bh, int& I) {
    if (om.order) {
      const int r = v < om.rows ? om.order[v] : -1;
      bh = r >= 0 ? r / nb : 0;
      I = r >= 0 ? r - bh * nb : nb;
    } else {
      const long long P = (nb + 1) >> 1;
      const long long p = v >> 1;
      bh = (int)(p / P);
      I = 2 * (int)(p - bh * P) + (int)(v & 1);
    }
  };
  int bh0, I0, bh1, I1;
  decode(v0, bh0, I0);
  decode(v1, bh1, I1);
  auto slot_bh = [&](int x) { return x ? bh1 : bh0; };
  // frame-exact masking (no order): I1 = I0 + 1, or I1 = I0 in a split CTA
  auto slot_I = [&](int x) { return x ? I1 : I0; };
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->q_full[x], 1);
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_half[x], 4);
      mbar_init(&bars->p_full[x], 4);
      mbar_init(&bars->o_final[x], 1);
    }
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->stall, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
    // Q of each existing slot depends only on its block index: start both
    // loads now, while the lists are being staged.
    for (int x = 0; x < 2; ++x) {
      if (slot_I(x) >= nb) continue;
      mbar_arrive_expect_tx(&bars->q_full[x], C::kQBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d(smem + C::kQOff + x * C::kQBytes + c * (kQRows * 128), &tm_q, &bars->q_full[x], c * 64,
                    slot_I(x) * BLK, slot_bh(x));
    }
  }
  if (warp == 2 || warp == 3) {
    // Compact the slot's kept list into shared memory, dropping invalid indices.
    const int x = warp - 2;
    const int I = slot_I(x);
    int base = 0;
    bool bad = false;
    if (I < nb) {
      const long long row_id = (long long)slot_bh(x) * nb + I;
      const int32_t* src = kv_idx + row_id * (long long)kcap;
      const int lim = min(kcap, max_list);
      const int J_first = lane < lim ? src[lane] : -1;    // fetched alongside the count
      int cnt = kv_cnt[row_id];
      cnt = max(0, min(cnt, lim));
      // entries [lo, hi) of the row: all of it, or one half in a split CTA
      int lo = 0, hi = cnt;
      if (split) {
        const int h0 = (cnt + 1) >> 1;
        lo = x ? h0 : 0;
        hi = x ? cnt : h0;
      }
      int32_t* dst = lists + x * max_list;
      for (int j0 = lo; j0 < hi; j0 += 32) {
        const int j = j0 + lane;
        int J = -1;
        if (j < hi) J = (j0 == 0) ? J_first : src[j];
        const bool ok = (j < hi) && J >= 0 && J < nb;
        bad |= (j < hi) && !ok;
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        if (ok) {
          const int pos = base + __popc(m & ((1u << lane) - 1u));
          dst[pos] = J;
          if (FRAME) {
            // first frame of the key block and the columns that lie in it
            const int k0 = J * BLK;
            const int f0 = k0 / fm.P;
            const int cb = min(BLK, (f0 + 1) * fm.P - k0);
            dst[2 * max_list + pos] = (f0 << 8) | cb;
          }
        }
        base += __popc(m);
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_attn_flags, (uint32_t)DFS_FLAG_BAD_KV_INDEX);
    if (lane == 0) bars->n_kv[x] = base;
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, C::kTmemCols);
  // FRAME only: per list entry (first key frame << 8 | columns in it), then the frame bit sets
  const int32_t* kmeta = lists + 2 * max_list;
  uint32_t* ftab = reinterpret_cast<uint32_t*>(lists + 4 * max_list);
  // split CTAs: slot B's row maxima and sums for the merge (2 x 128 floats)
  float* xch = reinterpret_cast<float*>(lists + (FRAME ? 4 * max_list + kFrameRows * frame_words(fm.T) : 2 * max_list));
  const int qf_lo = FRAME ? (I0 * BLK) / fm.P : 0;
  if (FRAME && warp >= 4) {
    const int words = frame_words(fm.T);
    for (int w = threadIdx.x - 128; w < kFrameRows * words; w += kThreads - 128) {
      const int t = min(fm.T - 1, qf_lo + w / words);
      const int f_base = (w % words) * 32;
      uint32_t bits = 0;
      for (int b = 0; b < 32 && f_base + b < fm.T; ++b)
        if (dfs::lvsa_in_frame_set(f_base + b, t, fm.T, fm.T_per, fm.s0, fm.C, fm.nG)) bits |= 1u << b;
      ftab[w] = bits;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n[2] = {bars->n_kv[0], bars->n_kv[1]};
  const int jmax = max(n[0], n[1]);
  if (warp < 4) {
  if (BLK == 128) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegWg0) : "memory");
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Warp-uniform loop; elect.sync picks the lane that arms a barrier or
    // issues a copy.
    {
      if (lane == 0) {
        prefetch_tensor_map(&tm_q);
        prefetch_tensor_map(&tm_k);
        prefetch_tensor_map(&tm_v);
      }
      // Same step order as the MMA issuer: step -1 loads K_A(0), K_B(0); step
      // j loads, per slot, V(j) and then K(j+1).
      int t = 0;  // ring tiles loaded so far
      bool ok = true;
      for (int step = -1; step < jmax && ok; ++step) {
#pragma unroll 1
        for (int x = 0; x < 2; ++x) {
          const int nx = n[x];
          if (step >= nx) continue;
#pragma unroll 1
          for (int kind = 0; kind < 2; ++kind) {      // 0: V(step), 1: K(step + 1)
            const int jj = kind == 0 ? step : step + 1;
            if (jj < 0 || jj >= nx) continue;
            const int st = t % kRing;
            if (!mbar_wait_bounded(&bars->kv_empty[st], (uint32_t)(((t / kRing) & 1) ^ 1), abort_flag, kWaitLimit)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx_warp(&bars->kv_full[st], C::kTileBytes);
            const int J = lists[x * max_list + jj];
            uint8_t* dst = smem + C::kRingOff + st * C::kTileBytes;
            const CUtensorMap* map = kind == 0 ? &tm_v : &tm_k;
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c)
              tma_load_3d_warp(dst + c * (BLK * 128), map, &bars->kv_full[st], c * 64, J * BLK, slot_bh(x));
            ++t;
          }
          if (!ok) break;
        }
      }
      // Drain: a stage is reloaded only after its previous tile was
      // consumed, so only the last kRing loads can still be in flight.
      for (int u = max(0, t - kRing); u < t; ++u)
        mbar_wait_timed(&bars->kv_full[u % kRing], (uint32_t)((u / kRing) & 1), kDrainLimit);
      for (int x = 0; x < 2; ++x)
        if (slot_I(x) < nb) mbar_wait_timed(&bars->q_full[x], 0, kDrainLimit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (warp-uniform control flow and
    // operands); elect.sync inside each MMA / commit picks the issuing lane.
    {
      // Descriptors are built once; a K step or a ring stage only moves the
      // start-address field (16-byte units), so each MMA costs an add.
      const uint64_t dq = desc_sw128(smem_addr(smem + C::kQOff), 16, 1024);
      const uint64_t dk = desc_sw128(smem_addr(smem + C::kRingOff), 16, 1024);
      const uint64_t dv = desc_sw128(smem_addr(smem + C::kRingOff), BLK * 128, 1024);
      bool ok = true;
      if (om.stall_cycles > 0) ok = mbar_wait_bounded(&bars->stall, 0, abort_flag, om.stall_cycles);
      for (int x = 0; x < 2 && ok; ++x)
        if (n[x] > 0) ok = mbar_wait_bounded(&bars->q_full[x], 0, abort_flag, kWaitLimit);
      // Step -1 issues S_A(0), S_B(0); step j issues, per slot, PV(j) and
      // then S(j+1) (or the slot's final commit).
      int t = 0;  // ring tiles consumed so far
      for (int step = -1; step < jmax && ok; ++step) {
#pragma unroll 1
        for (int x = 0; x < 2; ++x) {
          const int nx = n[x];
          if (step >= nx) continue;
          if (step >= 0) {
            // P_X was written by other threads with tcgen05.st: order this
            // thread's MMAs after their arrival. (TMA-filled tiles need no
            // fence: the mbarrier transaction count orders them.)
            const int st = t % kRing;
            const uint64_t dvs = dv + (uint64_t)((st * C::kTileBytes) >> 4);
            if (BLK == 128) {
              // keys 0-63 of P(step) first, while the softmax forms keys 64-127
              if (!mbar_wait_bounded(&bars->p_half[x], (uint32_t)(step & 1), abort_flag, kWaitLimit)) { ok = false; break; }
              tc_fence_after();
              if (!mbar_wait_bounded(&bars->kv_full[st], (uint32_t)((t / kRing) & 1), abort_flag, kWaitLimit)) { ok = false; break; }
              issue_pv<D, BLK, 0, BLK / 32>(tmem + C::o_col(x), tmem + C::s_col(x), dvs, step > 0);
              if (!mbar_wait_bounded(&bars->p_full[x], (uint32_t)(step & 1), abort_flag, kWaitLimit)) { ok = false; break; }
              tc_fence_after();
              issue_pv<D, BLK, BLK / 32, BLK / 16>(tmem + C::o_col(x), tmem + C::s_col(x), dvs, true);
            } else {
              if (!mbar_wait_bounded(&bars->p_full[x], (uint32_t)(step & 1), abort_flag, kWaitLimit)) { ok = false; break; }
              tc_fence_after();
              if (!mbar_wait_bounded(&bars->kv_full[st], (uint32_t)((t / kRing) & 1), abort_flag, kWaitLimit)) { ok = false; break; }
              issue_pv<D, BLK, 0, BLK / 16>(tmem + C::o_col(x), tmem + C::s_col(x), dvs, step > 0);
            }
            mma_commit_warp(&bars->kv_empty[st]);
            ++t;
          }
          if (step + 1 < nx) {
            const int st = t % kRing;
            if (!mbar_wait_bounded(&bars->kv_full[st], (uint32_t)((t / kRing) & 1), abort_flag, kWaitLimit)) { ok = false; break; }
            issue_s<D, BLK>(tmem + C::s_col(x), dq + (uint64_t)((x * C::kQBytes) >> 4),
                            dk + (uint64_t)((st * C::kTileBytes) >> 4));
            mma_commit_warp(&bars->s_full[x]);
            mma_commit_warp(&bars->kv_empty[st]);
            ++t;
          } else if (step >= 0) {
            mma_commit_warp(&bars->o_final[x]);
          }
        }
      }
      // Every MMA must finish before tensor memory is released.
      mma_commit_warp(&bars->mma_done);
      mbar_wait_timed(&bars->mma_done, 0, kDrainLimit);
    }
    __syncwarp();
  }
  } else {
    // ------------------------------------------------------------ softmax
    if (BLK == 128) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax) : "memory");
    const int x = warp < 8 ? 0 : 1;                 // slot
    const int I = slot_I(x);
    const int bh = slot_bh(x);
    const int sub = warp & 3;                       // TMEM lane quarter of this warp
    const int r = sub * 32 + lane;                  // query row in the tile
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + C::s_col(x);
    const uint32_t o_addr = tmem + lane_base + C::o_col(x);
    const int rem = N - (nb - 1) * BLK;             // valid keys in the last block
    const int32_t* list = lists + x * max_list;
    const int nx = n[x];
    float m = -INFINITY;                            // running max (log2 units)
    float l = 0.f;                                  // running row sum
    bool ok = true;
    const uint32_t* frow = ftab;                    // A(query frame) as bits
    if (FRAME) frow += (min(fm.T - 1, (I * BLK + r) / fm.P) - qf_lo) * frame_words(fm.T);
    for (int j = 0; j < nx; ++j) {
      if (!mbar_wait_bounded(&bars->s_full[x], (uint32_t)(j & 1), abort_flag, kWaitLimit)) { ok = false; break; }
      tc_fence_after();
      float sv[BLK];
#pragma unroll
      for (int c = 0; c < BLK / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(s_addr + c * 32, raw);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(raw[e]);
      }
      tmem_wait_ld();
      if (list[j] == nb - 1 && rem < BLK) {
#pragma unroll
        for (int e = 0; e < BLK; ++e)
          if (e >= rem) sv[e] = -INFINITY;
      }
      if (FRAME) {
        // Keys of this block lie in frames f0 (columns < cb) and f0 + 1;
        // drop the frame(s) outside A(query frame).
        const int mt = kmeta[x * max_list + j];
        const int f0 = mt >> 8, cb = mt & 255;
        const bool a0 = (frow[f0 >> 5] >> (f0 & 31)) & 1u;
        const bool a1 = cb >= BLK || (f0 + 1 < fm.T && ((frow[(f0 + 1) >> 5] >> ((f0 + 1) & 31)) & 1u));
        if (!a0 || !a1) {
#pragma unroll
          for (int e = 0; e < BLK; ++e)
            if (e < cb ? !a0 : !a1) sv[e] = -INFINITY;
        }
      }
      // row maximum: eight independent chains of three-input maxima
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = sv[e];
#pragma unroll
      for (int e = 8; e + 16 <= BLK; e += 16)
#pragma unroll
        for (int c = 0; c < 8; ++c) mx8[c] = fmax3(mx8[c], sv[e + c], sv[e + 8 + c]);
      if ((BLK - 8) % 16 != 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c) mx8[c] = fmaxf(mx8[c], sv[BLK - 8 + c]);
      }
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
      const float m_blk = mx * scale_log2;
      bool rescale = false;
      float m_use;
      if (j == 0) {
        m_use = m_blk;
      } else {
        rescale = __any_sync(0xffffffffu, m_blk > m + 8.0f);
        m_use = rescale ? fmaxf(m, m_blk) : m;
      }
      // P = 2^(s * scale_log2 - m), bf16, written over S_X (fully read).
      const float2 sc2 = make_float2(scale_log2, scale_log2);
      // A row whose keys so far are all masked has no maximum yet: its
      // exponentials are all 2^-inf = 0 whatever is subtracted.
      const float m_sub = (FRAME && m_use == -INFINITY) ? 0.f : m_use;
      const float2 nm2 = make_float2(-m_sub, -m_sub);
      float2 acc[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < BLK / 64; ++c) {
        uint32_t packed[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float2 x2 = __ffma2_rn(make_float2(sv[c * 64 + 2 * e], sv[c * 64 + 2 * e + 1]), sc2, nm2);
          float2 p2;
          if (EMU > 0 && (e % (EMU > 0 ? EMU : 1)) == EMU - 1) {
            p2 = make_float2(dfs::exp2_poly(x2.x), dfs::exp2_poly(x2.y));
          } else {
            p2 = make_float2(ex2(x2.x), ex2(x2.y));
          }
          acc[e & 3] = __fadd2_rn(acc[e & 3], p2);
          packed[e] = pack_bf16x2(p2.x, p2.y);
        }
        tmem_st32(s_addr + c * 32, packed);
        if (BLK == 128 && c == 0 && !rescale) {
          // keys 0-63 of P are in place: release them to the MMAs while the
          // rest is formed (a warp that rescales O releases them after that)
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->p_half[x]);
        }
      }
      const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
      const float2 a = __fadd2_rn(a01, a23);
      const float rs = a.x + a.y;
      // O_X may be rescaled here: s_full(j) was committed after PV_X(j-1)
      // by the same thread, so PV_X(j-1) has completed, and no MMA of PV_X(j)
      // starts before this warp's arrival on p_half.
      if (rescale) {
        // (a row with no unmasked key yet has O = 0 and l = 0)
        const float alpha = (FRAME && m == -INFINITY) ? 0.f : ex2(m - m_use);
        const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t raw[32];
          tmem_ld32(o_addr + c * 32, raw);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(raw[2 * e]), __uint_as_float(raw[2 * e + 1])), al2);
            raw[2 * e] = __float_as_uint(v.x);
            raw[2 * e + 1] = __float_as_uint(v.y);
          }
          tmem_st32(o_addr + c * 32, raw);
        }
        l *= alpha;
        if (BLK == 128) {
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->p_half[x]);
        }
      }
      tmem_wait_st();
      m = m_use;
      l += rs;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[x]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && nx > 0) ok = mbar_wait_bounded(&bars->o_final[x], 0, abort_flag, kWaitLimit);
    tc_fence_after();
    if (split) {
      // Both slots hold the same query rows over disjoint halves of the
      // list: slot B hands its (m, l) to slot A, whose threads read O_B from
      // tensor memory (same lane quarter) and write the merged rows.
      if (x == 1) {
        xch[r] = (nx > 0 && ok) ? m : -INFINITY;
        xch[kQRows + r] = (nx > 0 && ok) ? l : 0.f;
      }
      tc_fence_before();
      asm volatile("bar.sync 1, 256;" ::: "memory");   // the two softmax warpgroups
      tc_fence_after();
    }
    if (split && n[1] > 0) {
      if (x == 0) {
        // O = (2^(m_A - M) O_A + 2^(m_B - M) O_B) / (2^(m_A - M) l_A + 2^(m_B - M) l_B),
        // M = max(m_A, m_B); a half with no unmasked key has m = -inf and weight 0
        const float mA = (nx > 0 && ok) ? m : -INFINITY, lA = (nx > 0 && ok) ? l : 0.f;
        const float mB = xch[r], lB = xch[kQRows + r];
        const float M = fmaxf(mA, mB);
        const float aA = (mA == -INFINITY) ? 0.f : ex2(mA - M);
        const float aB = (mB == -INFINITY) ? 0.f : ex2(mB - M);
        const float L = lA * aA + lB * aB;
        const float inv = L > 0.f ? 1.0f / L : 0.f;
        const float wA = aA * inv, wB = aB * inv;
        const long long qrow = (long long)I * BLK + r;
        const bool store = ok && I < nb && r < BLK && qrow < N;
        __nv_bfloat16* orow;
        if (om.perm) {
          const int b = bh / om.nh, h = bh - b * om.nh;
          const long long tok = (qrow < N) ? om.perm[qrow] : 0;
          orow = op + (((long long)b * N + tok) * om.nh + h) * D;
        } else {
          orow = op + ((long long)bh * N + qrow) * D;
        }
        const uint32_t oB_addr = tmem + lane_base + C::o_col(1);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ra[32], rb[32];
          if (nx > 0) {
            tmem_ld32(o_addr + c * 32, ra);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) ra[e] = 0u;
          }
          tmem_ld32(oB_addr + c * 32, rb);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float v[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              float t = 0.f;
              if (wA != 0.f) t = __uint_as_float(ra[2 * e + u]) * wA;
              if (wB != 0.f) t = fmaf(__uint_as_float(rb[2 * e + u]), wB, t);
              v[u] = t;
            }
            pk[e] = pack_bf16x2(v[0], v[1]);
          }
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        if (store && lse) lse[(long long)bh * N + qrow] = (M + __log2f(L)) * 0.6931471805599453f;
      }
    } else if (!split || x == 0) {
    const long long qrow = (long long)I * BLK + r;
    const bool store = ok && I < nb && r < BLK && qrow < N;
    __nv_bfloat16* orow;
    if (om.perm) {
      const int b = bh / om.nh, h = bh - b * om.nh;
      const long long tok = (qrow < N) ? om.perm[qrow] : 0;
      orow = op + (((long long)b * N + tok) * om.nh + h) * D;
    } else {
      orow = op + ((long long)bh * N + qrow) * D;
    }
    const float inv_l = (nx > 0 && l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t raw[32];
      if (nx > 0 && ok) {
        tmem_ld32(o_addr + c * 32, raw);
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
      lse[(long long)bh * N + qrow] = (nx > 0) ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && bars->abort_flag) atomicOr(&g_attn_flags, (uint32_t)DFS_FLAG_WAIT_TIMEOUT);
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// ------------------------------------------------------------------ host
template <int D, int BLK, int EMU, bool FRAME>
int launch_attn(const dfs::Dims& d, const void* qp, const void* kp, const void* vp, const int32_t* kv_idx,
                const int32_t* kv_cnt, int kcap, float scale, void* op, float* lse, cudaStream_t st,
                FrameMask fm, OutMap om) {
  using C = Cfg<D, BLK>;
  CUtensorMap mq, mk, mv;
  if (!dfs::make_map_bf16(&mq, qp, d.N, D, d.BH, kQRows) || !dfs::make_map_bf16(&mk, kp, d.N, D, d.BH, BLK) ||
      !dfs::make_map_bf16(&mv, vp, d.N, D, d.BH, BLK))
    return DFS_ERR_CUDA;
  const int max_list = min(kcap, d.nb);
  size_t smem = 1024 + C::kBarOff + sizeof(Barriers) + 2 * (size_t)max_list * sizeof(int32_t) +
                2 * kQRows * sizeof(float);
  if (FRAME) smem += 2 * (size_t)max_list * sizeof(int32_t) + (size_t)kFrameRows * frame_words(fm.T) * sizeof(uint32_t);
  if (smem > 232448) return DFS_ERR_UNSUPPORTED;
  // Tensor memory per SM is 512 columns: a 512-column CTA must be alone on
  // its SM and a 256-column CTA may share it with one other, so shared
  // memory is padded to make the scheduler place CTAs that way.
  const size_t min_smem = (C::kTmemCols == 512) ? 120 * 1024 : 80 * 1024;
  if (smem < min_smem) smem = min_smem;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, BLK, EMU, FRAME>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return DFS_ERR_CUDA;
  if (BLK == 128) {
    // the register split must fit the registers the CTA is launched with
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_fwd_kernel<D, BLK, EMU, FRAME>) != cudaSuccess) return DFS_ERR_CUDA;
    const int launched = ((fa.numRegs + 7) / 8) * 8;
    if (128 * kRegWg0 + 256 * kRegSoftmax > launched * kThreads) return DFS_ERR_UNSUPPORTED;
  }
  // virtual rows (see OutMap), two-row CTAs, and the split of the last wave
  const long long V = om.order ? om.rows : 2LL * d.BH * ((d.nb + 1) / 2);
  const long long pairs = (V + 1) / 2;
  om.split_from = pairs;
  if (om.tail_split) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0) {
      // a last wave of rem two-row CTAs (rem <= SMs / 2) becomes 2 rem
      // CTAs of half the work each, which all run at once
      const long long rem = pairs % sms;
      if (rem > 0 && 2 * rem <= sms) om.split_from = pairs - rem;
    }
  }
  // two-row CTAs, plus one CTA per row after them (the last pair may hold
  // one row when V is odd; it is split only together with its wave)
  const long long ctas = om.split_from == pairs ? pairs : om.split_from + (V - 2 * om.split_from);
  if (ctas > 0x7fffffffLL) return DFS_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)ctas);
  const float scale_log2 = scale * 1.4426950408889634f;
  attn_fwd_kernel<D, BLK, EMU, FRAME><<<grid, kThreads, smem, st>>>(
      mq, mk, mv, kv_idx, kv_cnt, kcap, (int)d.N, d.nb, scale_log2, (__nv_bfloat16*)op, lse, max_list, fm, om);
  return dfs::launch_status();
}

}  // namespace

DFS_DEFINE_FLAG_READER(dfs_detail_flags_attn, g_attn_flags)

namespace {

int check_attn_args(const dfs_shape* shape, const void* qp, const void* kp, const void* vp, const int32_t* kv_idx,
                    const int32_t* kv_cnt, int kcap, void* op, float* lse, dfs::Dims* d) {
  int st = dfs::check_shape(shape, d, false);
  if (st != DFS_OK) return st;
  if (!qp || !kp || !vp || !kv_idx || !kv_cnt || !op || kcap < 1) return DFS_ERR_INVALID_ARG;
  if (!dfs::aligned16(qp) || !dfs::aligned16(kp) || !dfs::aligned16(vp) || !dfs::aligned16(op) ||
      (lse && !dfs::aligned16(lse)))
    return DFS_ERR_MISALIGNED;
  if (d->N >= (1LL << 31) || d->BH > 65535) return DFS_ERR_UNSUPPORTED;
  return DFS_OK;
}

template <bool FRAME>
int dispatch_attn(const dfs::Dims& d, const void* qp, const void* kp, const void* vp, const int32_t* kv_idx,
                  const int32_t* kv_cnt, int kcap, float scale, void* op, float* lse, cudaStream_t cs,
                  FrameMask fm, OutMap om) {
  constexpr int kEmu = DFS_ATTN_EXP2_EMU;
  if (d.D == 128 && d.blk == 128)
    return launch_attn<128, 128, kEmu, FRAME>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, cs, fm, om);
  if (d.D == 128 && d.blk == 64)
    return launch_attn<128, 64, kEmu, FRAME>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, cs, fm, om);
  if (d.D == 64 && d.blk == 128)
    return launch_attn<64, 128, kEmu, FRAME>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, cs, fm, om);
  return launch_attn<64, 64, kEmu, FRAME>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, cs, fm, om);
}

}  // namespace

extern "C" int dfs_sparse_attn_fwd(const dfs_shape* shape, const void* qp, const void* kp, const void* vp,
                                   const int32_t* kv_idx, const int32_t* kv_cnt, int kcap, float scale, void* op,
                                   float* lse, dfs_stream_t stream) {
  dfs::Dims d;
  const int st = check_attn_args(shape, qp, kp, vp, kv_idx, kv_cnt, kcap, op, lse, &d);
  if (st != DFS_OK) return st;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d.D);
  return dispatch_attn<false>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, (cudaStream_t)stream,
                              FrameMask{1, 1, 1, 0, 1, 0}, OutMap{nullptr, 1, nullptr, d.BH * d.nb, 1, 0, 0});
}

extern "C" int dfs_sparse_attn_fwd_ex(const dfs_shape* shape, const void* qp, const void* kp, const void* vp,
                                      const int32_t* kv_idx, const int32_t* kv_cnt, int kcap, float scale,
                                      const dfs_attn_opts* opts, void* o, float* lse, dfs_stream_t stream) {
  dfs::Dims d;
  const int st = check_attn_args(shape, qp, kp, vp, kv_idx, kv_cnt, kcap, o, lse, &d);
  if (st != DFS_OK) return st;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d.D);
  OutMap om{nullptr, d.nh, nullptr, d.BH * d.nb, 1, 0, 0};
  if (opts) {
    om.perm = opts->perm;
    om.order = opts->order;
    om.tail_split = opts->no_tail_split ? 0 : 1;
    om.stall_cycles = (long long)opts->test_stall_cycles;
  }
  return dispatch_attn<false>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, o, lse, (cudaStream_t)stream,
                              FrameMask{1, 1, 1, 0, 1, 0}, om);
}

extern "C" int dfs_sparse_attn_lvsa_fwd(const dfs_shape* shape, const void* qp, const void* kp, const void* vp,
                                        const int32_t* kv_idx, const int32_t* kv_cnt, int kcap, float scale,
                                        const dfs_select_params* lvsa, void* op, float* lse, dfs_stream_t stream) {
  dfs::Dims d;
  const int st = check_attn_args(shape, qp, kp, vp, kv_idx, kv_cnt, kcap, op, lse, &d);
  if (st != DFS_OK) return st;
  if (!lvsa || lvsa->lvsa_T_per < 1 || lvsa->lvsa_C < 1 || lvsa->lvsa_step < 0) return DFS_ERR_INVALID_ARG;
  const long long P = (long long)d.H * d.W;
  if (P < d.blk || d.T > kMaxFrames) return DFS_ERR_UNSUPPORTED;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)d.D);
  FrameMask fm;
  fm.P = (int)P;
  fm.T = d.T;
  fm.T_per = lvsa->lvsa_T_per;
  fm.s0 = lvsa->lvsa_step % lvsa->lvsa_T_per;
  fm.C = lvsa->lvsa_C;
  fm.nG = (fm.s0 < d.T) ? (d.T - 1 - fm.s0) / fm.T_per + 1 : 0;
  return dispatch_attn<true>(d, qp, kp, vp, kv_idx, kv_cnt, kcap, scale, op, lse, (cudaStream_t)stream, fm,
                             OutMap{nullptr, 1, nullptr, d.BH * d.nb, 1, 0, 0});
}

namespace {

// Stable counting sort of the query rows of one head (one CTA per head) by
// kept count, descending: rows of equal count stay in ascending order, so
// the order (and every result computed in it) is the same on every run, and
// the heads stay in order, so the CTAs running at any time read the keys and
// values of about two heads (they stay in L2).
//   1. warp w < S takes the contiguous segment w of the head's rows and
//      counts its keys into its own histogram hist[w][key] (only warp w
//      writes it);
//   2. the key totals are scanned from the largest key down, and each
//      histogram entry becomes the first output slot of that warp's rows
//      with that key: base(key) + rows of that key in segments before w;
//   3. each warp walks its segment in order, 32 rows at a time; the lanes
//      with equal keys (__match_any_sync) take consecutive slots in lane
//      order and the group's leader advances hist[w][key].
// S = the number of segments whose histograms fit the shared memory.
constexpr int kOrderThreads = 1024;
constexpr size_t kOrderSmemMax = 200 * 1024;

__host__ __device__ inline int order_segments(int kmax) {
  const long long per = (long long)(kmax + 1) * (long long)sizeof(int);
  const long long s = (long long)kOrderSmemMax / per - 1;    // one row of the table holds the key bases
  return (int)(s < 1 ? 1 : (s > kOrderThreads / 32 ? kOrderThreads / 32 : s));
}

__global__ void __launch_bounds__(kOrderThreads)
attn_order_kernel(const int32_t* __restrict__ kv_cnt, int nb, int kmax, int nseg, int32_t* __restrict__ order) {
  extern __shared__ int hist[];              // [nseg + 1][kmax + 1]; the last row: key bases
  const int K = kmax + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long row0 = (long long)blockIdx.x * nb;   // this head's rows: row0 .. row0 + nb - 1
  const int32_t* cnt = kv_cnt + row0;
  int32_t* out = order + row0;
  int* base = hist + (size_t)nseg * K;
  for (int i = tid; i < (nseg + 1) * K; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int seg = (nb + nseg - 1) / nseg;
  const int lo = warp * seg, hi = min(lo + seg, nb);
  int* mine = hist + (size_t)warp * K;
  if (warp < nseg) {
    for (int r0 = lo; r0 < hi; r0 += 32) {
      const int r = r0 + lane;
      const bool in = r < hi;
      const int c = in ? max(0, min(cnt[r], kmax)) : -1 - lane;
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      if (in && lane == __ffs(peers) - 1) mine[c] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  for (int c = tid; c < K; c += blockDim.x) {
    int tot = 0;
    for (int w = 0; w < nseg; ++w) tot += hist[(size_t)w * K + c];
    base[c] = tot;
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int c = kmax; c >= 0; --c) {
      const int h = base[c];
      base[c] = run;
      run += h;
    }
  }
  __syncthreads();
  for (int c = tid; c < K; c += blockDim.x) {
    int run = base[c];
    for (int w = 0; w < nseg; ++w) {
      const int h = hist[(size_t)w * K + c];
      hist[(size_t)w * K + c] = run;
      run += h;
    }
  }
  __syncthreads();
  if (warp < nseg) {
    for (int r0 = lo; r0 < hi; r0 += 32) {
      const int r = r0 + lane;
      const bool in = r < hi;
      const int c = in ? max(0, min(cnt[r], kmax)) : -1 - lane;
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      const int leader = __ffs(peers) - 1;
      int slot = 0;
      if (in && lane == leader) {
        slot = mine[c];
        mine[c] = slot + __popc(peers);
      }
      slot = __shfl_sync(0xffffffffu, slot, leader);
      if (in) out[slot + __popc(peers & ((1u << lane) - 1u))] = (int32_t)(row0 + r);
      __syncwarp();
    }
  }
}

}  // namespace

extern "C" int dfs_attn_order(const dfs_shape* shape, const int32_t* kv_cnt, int kcap, int32_t* order,
                              dfs_stream_t stream) {
  dfs::Dims d;
  const int st = dfs::check_shape(shape, &d, false);
  if (st != DFS_OK) return st;
  if (!kv_cnt || !order || kcap < 1) return DFS_ERR_INVALID_ARG;
  const int kmax = min(kcap, d.nb);
  if (d.BH * d.nb >= (1LL << 31)) return DFS_ERR_UNSUPPORTED;
  const int nseg = order_segments(kmax);
  const size_t smem = (size_t)(nseg + 1) * (kmax + 1) * sizeof(int);
  if (smem > 232448) return DFS_ERR_UNSUPPORTED;      // two table rows beyond the shared memory: kmax > 29055
  if (cudaFuncSetAttribute(attn_order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return DFS_ERR_CUDA;
  if (d.BH > 0x7fffffffLL) return DFS_ERR_UNSUPPORTED;
  attn_order_kernel<<<(unsigned)d.BH, kOrderThreads, smem, (cudaStream_t)stream>>>(kv_cnt, d.nb, kmax, nseg, order);
  return dfs::launch_status();
}
