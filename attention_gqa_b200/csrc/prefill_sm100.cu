// Prefill attention kernel for sm_100a: gpt-oss-style grouped-query attention
// (64 query heads over 8 key/value heads, head_dim 64) with half-split RoPE,
// a learned sink logit in the softmax denominator, and full-causal or
// sliding-window masks (gpt-oss pages: inteligile techniques map rows
// "Grouped-query attention", "Partial RoPE", "Learnable attention sink",
// "Sliding-window attention"; llm-atlas field tables for the constants).
//
// Work item: batch b, key/value head g, 32 query tokens. The 8 query heads of
// group g are packed into the M dimension, so an item is two M=128 tiles
// (16 tokens x 8 heads) sharing every K/V tile. CTAs are persistent (one per
// SM) and walk a static "snake" order over the items sorted longest first,
// which balances the causal triangle without a global counter.
//
// Roles (512 threads, four warpgroups):
//   WG0 warp 0    TMA producer of Q per item (2-slot buffer, with the
//                 rotary-table rows of its tokens) and of K tiles of 128 keys
//                 through a kStages-deep ring; warp 3 produces the V tiles.
//                 A K stage is released after both M tiles' Q.K^T, a V stage
//                 after both P.V, so K runs further ahead than V.
//   WG0 warps 1-2 one tcgen05 issuer thread per M tile m (warp 1 also owns
//                 the tensor memory): S_m = Q_m K^T (SS, K-major) and
//                 O_m += P_m V (A = P from TMEM, B = V MN-major). Separate
//                 issuers keep each M tile's pipeline independent of the
//                 other's progress; the tensor core interleaves the streams.
//   WG1, WG2      softmax for M tile 0 / 1 (thread = TMEM lane = one query row):
//                 one 128-column TMEM load per tile, sink-seeded online softmax
//                 in log2 units, bf16 P to TMEM; after an item's last tile the
//                 same warpgroup normalises O and stores it (bf16, TMA) through
//                 its half of the item's Q slot.
//   WG3           RoPE: rotates the Q rows of each item in shared memory from
//                 an fp64-built (cos, sin) table. Keys arrive already rotated
//                 (a pre-pass rotates each key once per layer).
// TMEM (512 columns): S0 [0,128), S1 [128,256), P0 [256,320), P1 [320,384),
// O0 [384,448), O1 [448,512). The softmax releases S right after loading it,
// so Q K^T of tile j+1 overlaps the softmax of tile j and P.V of tile j
// overlaps the softmax of tile j+1.
// The running max starts at sigma*log2(e) with l = 1; O is rescaled only when
// the max grows by more than 2^8 (exact: O and l share the reference). The two
// softmax warpgroups take turns on their exp loops (a warpgroup hands over 5/8
// of the way through its loop), which keeps their tiles staggered against the
// tensor core. Query token i of a call sits at key index q_start+i (q_start > 0
// when a chunk is prefilled against a cache): masks and tile ranges use key
// indices, Q rows, positions and outputs use i.
#include <cmath>

#include "prefill_common.cuh"

namespace gqa {
namespace {

constexpr int kBlockQ = 32;      // query tokens per work item
constexpr int kTokensPerM = 16;  // tokens per M=128 tile (x 8 heads)
constexpr int kBlockN = 128;     // keys per K/V tile
constexpr int kStages = 4;
constexpr uint32_t kTileBytes = 128 * 128;  // 128 rows of 64 bf16

// TMEM columns of M tile m: S (fp32, 128 columns), P (bf16 pairs, 64 columns)
// and the O accumulator (fp32, 64 columns). P has columns of its own, so the
// next tile's S = Q K^T can be computed while the softmax still works on the
// current one.
__host__ __device__ constexpr uint32_t tmem_s(int m) { return 128u * static_cast<uint32_t>(m); }
__host__ __device__ constexpr uint32_t tmem_p(int m) { return 256u + 64u * static_cast<uint32_t>(m); }
__host__ __device__ constexpr uint32_t tmem_o(int m) { return 384u + 64u * static_cast<uint32_t>(m); }

// Register budgets after the warpgroup split; launch is 512 x 128.
constexpr uint32_t kRegsLight = 72;     // WG0 and WG3
constexpr uint32_t kRegsSoftmax = 184;  // WG1 and WG2
static_assert(2 * 128 * kRegsLight + 2 * 128 * kRegsSoftmax <= 512 * 128, "register split");

constexpr float kRescaleThreshold = 8.0f;      // log2 units
// Exp-loop step (of 64 column pairs) at which a softmax warpgroup releases the
// exponential unit to the other one (measured best at about 5/8 of the loop).
constexpr int kTurnHandOff = 38;

// Rotary-table rows in shared memory: 32 (cos, sin) pairs plus 16 bytes of
// padding, so the rows of the four tokens a warp touches sit in different banks.
constexpr uint32_t kTabRowBytes = kRopePairs * 8 + 16;

enum : int {
  BAR_Q_FULL = 0,                        // [2] slot loaded
  BAR_Q_READY = BAR_Q_FULL + 2,          // [2] slot rotated
  BAR_Q_EMPTY = BAR_Q_READY + 2,         // [2] slot's outputs stored (both halves)
  BAR_K_FULL = BAR_Q_EMPTY + 2,          // [kStages]
  BAR_V_FULL = BAR_K_FULL + kStages,     // [kStages]
  BAR_K_EMPTY = BAR_V_FULL + kStages,    // [kStages] both M tiles' Q.K^T done with the stage
  BAR_V_EMPTY = BAR_K_EMPTY + kStages,   // [kStages] both M tiles' P.V done with the stage
  BAR_S_FULL = BAR_V_EMPTY + kStages,    // [2] per M tile: S written
  BAR_S_FREE = BAR_S_FULL + 2,           // [2] S read by the softmax
  BAR_P_FULL = BAR_S_FREE + 2,           // [2] P written
  BAR_P_FREE = BAR_P_FULL + 2,           // [2] P.V done (P free)
  BAR_O_FULL = BAR_P_FREE + 2,           // [2] item's O complete
  BAR_STAGED = BAR_O_FULL + 2,           // [2] item's normalised O in shared memory
  BAR_TURN = BAR_STAGED + 2,             // [2] exp-loop turn of softmax warpgroup m
  BAR_MMA_DONE = BAR_TURN + 2,           // [2] per issuer
  NUM_BARS = BAR_MMA_DONE + 2
};

constexpr uint32_t kOffQ = 0;  // [2 slots][2 halves] tiles
constexpr uint32_t kOffK = kOffQ + 4 * kTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffTab = kOffV + kStages * kTileBytes;  // [2 slots][32 tokens] table rows
constexpr uint32_t kTabSlotBytes = kBlockQ * kTabRowBytes;
constexpr uint32_t kOffBar = kOffTab + 2 * kTabSlotBytes;
constexpr uint32_t kOffMisc = kOffBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

struct Ctx {
  uint32_t sbase;
  volatile int* abort_flag;
  int* err;
  __device__ uint32_t bar(int i) const { return sbase + kOffBar + 8u * static_cast<uint32_t>(i); }
  __device__ bool wait(int i, uint32_t parity) const {
    return mbar_wait(bar(i), parity, abort_flag, err, kErrTimeout, kWaitTimeoutNs);
  }
  __device__ bool wait_warp(int i, uint32_t parity) const {
    return mbar_wait_warp(bar(i), parity, abort_flag, err, kErrTimeout, kWaitTimeoutNs);
  }
  __device__ uint32_t q_tile(int slot, int m) const {
    return sbase + kOffQ + static_cast<uint32_t>(2 * slot + m) * kTileBytes;
  }
};

struct Item {
  int b, g, q0, jt0, n_tiles;
};

// The k-th item of CTA `cta` in snake order over items sorted longest first;
// false past the end. Order 0: query tile descending, then kv head, then
// batch. Order C > 0 (long sequences): chunks of C query tiles from the end,
// inside a chunk (batch, kv head) outer and query tile descending inner, so
// the CTAs of a wave stream the keys and values of only a few (b, g) pairs and
// those stay in L2 (with every pair active at once they do not fit).
__device__ __forceinline__ bool item_for(const PrefillArgs& a, int k, int cta, Item* it) {
  const int grid = static_cast<int>(gridDim.x);
  const int idx = (k & 1) ? (k + 1) * grid - 1 - cta : k * grid + cta;
  if (idx >= a.n_items) return false;
  const int n_bg = kNumKvHeads * a.batch;
  int qt, bg;
  if (a.order_chunk == 0) {
    qt = a.n_qtiles - 1 - idx / n_bg;
    bg = idx % n_bg;
  } else {
    const int C = a.order_chunk;
    const int c = idx / (C * n_bg);
    const int r = idx - c * C * n_bg;
    const int top = a.n_qtiles - 1 - c * C;  // highest query tile of the chunk
    const int cc = min(C, top + 1);          // query tiles in the chunk
    bg = r / cc;
    qt = top - r % cc;
  }
  // bg = b * 8 + g
  it->g = bg % kNumKvHeads;
  it->b = bg / kNumKvHeads;
  it->q0 = qt * kBlockQ;
  // key index of the item's first and last query token
  const int kq0 = a.q_start + it->q0;
  const int qlast = a.q_start + min(it->q0 + kBlockQ - 1, a.seqlen - 1);
  const int klo = a.window > 0 ? max(0, kq0 - a.window + 1) : 0;
  it->jt0 = klo / kBlockN;
  it->n_tiles = qlast / kBlockN - it->jt0 + 1;
  return true;
}

// S_m = Q_m K^T for one K/V tile (4 MMAs of K = 16 over head_dim 64).
__device__ __forceinline__ void issue_qk(const Ctx& ctx, uint32_t tmem, int m, int qs, int s) {
  constexpr uint32_t idesc = idesc_bf16(128, kBlockN, false);
  const uint32_t qa = ctx.q_tile(qs, m);
  const uint32_t ka = ctx.sbase + kOffK + s * kTileBytes;
#pragma unroll
  for (int kk = 0; kk < kHeadDim / 16; ++kk)
    mma_bf16_ss(tmem + tmem_s(m), sdesc_sw128(qa + 32 * kk), sdesc_sw128(ka + 32 * kk), idesc,
                kk > 0 ? 1u : 0u);
}

// O_m (+)= P_m V for global tile G, then the commits that release P, this
// M tile's use of the K/V stage and, after an item's last tile, O. The first
// tile of an item overwrites O: the softmax publishes that tile's P only after
// it has read out the previous item's O.
__device__ __forceinline__ bool issue_pv(const Ctx& ctx, uint32_t tmem, int m, int G, bool first,
                                         bool last) {
  constexpr uint32_t idesc = idesc_bf16(128, kHeadDim, true);
  const int s = G % kStages;
  if (!ctx.wait(BAR_V_FULL + s, (G / kStages) & 1)) return false;
  if (!ctx.wait(BAR_P_FULL + m, G & 1)) return false;
  tc_fence_after_sync();
  const uint32_t va = ctx.sbase + kOffV + s * kTileBytes;
#pragma unroll
  for (int kk = 0; kk < kBlockN / 16; ++kk)
    mma_bf16_ts(tmem + tmem_o(m), tmem + tmem_p(m) + 8 * kk, sdesc_sw128(va + 2048 * kk), idesc,
                (!first || kk > 0) ? 1u : 0u);
  mma_commit(ctx.bar(BAR_P_FREE + m));
  if (last) mma_commit(ctx.bar(BAR_O_FULL + m));
  mma_commit(ctx.bar(BAR_V_EMPTY + s));
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillMaps maps, const PrefillArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctx ctx;
  ctx.sbase = smem_u32(smem);
  ctx.abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  ctx.err = args.err;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);

  const int warp = static_cast<int>(threadIdx.x >> 5);
  const int lane = static_cast<int>(threadIdx.x & 31);
  const int cta = static_cast<int>(blockIdx.x);
  const int S = args.seqlen;
  const int W = args.window;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(ctx.bar(BAR_Q_FULL + i), 1);
      mbar_init(ctx.bar(BAR_Q_READY + i), 4);
      mbar_init(ctx.bar(BAR_Q_EMPTY + i), 2);
      mbar_init(ctx.bar(BAR_S_FULL + i), 1);
      mbar_init(ctx.bar(BAR_S_FREE + i), 4);
      mbar_init(ctx.bar(BAR_P_FULL + i), 4);
      mbar_init(ctx.bar(BAR_P_FREE + i), 1);
      mbar_init(ctx.bar(BAR_O_FULL + i), 1);
      mbar_init(ctx.bar(BAR_STAGED + i), 4);
      mbar_init(ctx.bar(BAR_TURN + i), 4);
      mbar_init(ctx.bar(BAR_MMA_DONE + i), 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(ctx.bar(BAR_K_FULL + s), 1);
      mbar_init(ctx.bar(BAR_V_FULL + s), 1);
      mbar_init(ctx.bar(BAR_K_EMPTY + s), 2);
      mbar_init(ctx.bar(BAR_V_EMPTY + s), 2);
    }
    // A pipeline timeout earlier left the error word set: skip the work.
    *ctx.abort_flag = (*reinterpret_cast<volatile int*>(args.err) & kErrTimeout) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *ctx.abort_flag != 0;
  const int wg = warp >> 2;

  if (wg == 0) {
    setmaxnreg_dec<kRegsLight>();
    if (warp == 0) {
      // -------------------------------------------------------------- producer
      if (lane == 0 && !skip) {
        prefetch_tensormap(&maps.q);
        prefetch_tensormap(&maps.k);
        int G = 0, n = 0, nq = 0;
        Item it;
        bool ok = true;
        for (; ok && item_for(args, n, cta, &it); ++n) {
          const int qs = n & 1;
          if (n >= 2 && !(ok = ctx.wait(BAR_Q_EMPTY + qs, ((n >> 1) - 1) & 1))) break;
          const uint32_t tab_bytes = kRopePairs * 8 * static_cast<uint32_t>(min(kBlockQ, S - it.q0));
          mbar_arrive_expect_tx(ctx.bar(BAR_Q_FULL + qs), 2 * kTileBytes + tab_bytes);
          tma_load_4d(ctx.q_tile(qs, 0), &maps.q, ctx.bar(BAR_Q_FULL + qs), 0, it.g * kGroup,
                      it.q0, it.b);
          tma_load_4d(ctx.q_tile(qs, 1), &maps.q, ctx.bar(BAR_Q_FULL + qs), 0, it.g * kGroup,
                      it.q0 + kTokensPerM, it.b);
          stage_rope_rows<kBlockQ, kTabRowBytes>(args, it.b, it.q0,
                                                 ctx.sbase + kOffTab + qs * kTabSlotBytes,
                                                 ctx.bar(BAR_Q_FULL + qs));
          // The rotated keys come from the key-rotation kernel launched just
          // before this one, which may still be running (the launch overlaps
          // this kernel's prologue and first Q loads with its tail).
          if (n == 0) griddep_wait();
          nq = n + 1;
          for (int j = 0; j < it.n_tiles; ++j) {
            const int s = G % kStages;
            if (G >= kStages && !(ok = ctx.wait(BAR_K_EMPTY + s, ((G / kStages) - 1) & 1)))
              break;
            mbar_arrive_expect_tx(ctx.bar(BAR_K_FULL + s), kTileBytes);
            tma_load_4d(ctx.sbase + kOffK + s * kTileBytes, &maps.k, ctx.bar(BAR_K_FULL + s), 0,
                        it.g, (it.jt0 + j) * kBlockN, it.b);
            ++G;
          }
        }
        if (*ctx.abort_flag) {
          // Let every copy this thread started land before shared memory is released.
          volatile int never = 0;
          for (int i = max(0, nq - 2); i < nq; ++i)
            mbar_wait(ctx.bar(BAR_Q_FULL + (i & 1)), (i >> 1) & 1, &never, nullptr, 0,
                      kWaitTimeoutNs);
          for (int i = max(0, G - kStages); i < G; ++i)
            mbar_wait(ctx.bar(BAR_K_FULL + i % kStages), (i / kStages) & 1, &never, nullptr, 0,
                      kWaitTimeoutNs);
        }
      }
    } else if (warp == 3) {
      // -------------------------------------------------------------- V producer
      if (lane == 0 && !skip) {
        prefetch_tensormap(&maps.v);
        int G = 0, n = 0;
        Item it;
        bool ok = true;
        for (; ok && item_for(args, n, cta, &it); ++n) {
          for (int j = 0; j < it.n_tiles; ++j) {
            const int s = G % kStages;
            if (G >= kStages && !(ok = ctx.wait(BAR_V_EMPTY + s, ((G / kStages) - 1) & 1)))
              break;
            mbar_arrive_expect_tx(ctx.bar(BAR_V_FULL + s), kTileBytes);
            tma_load_4d(ctx.sbase + kOffV + s * kTileBytes, &maps.v, ctx.bar(BAR_V_FULL + s), 0,
                        it.g, (it.jt0 + j) * kBlockN, it.b);
            ++G;
          }
        }
        if (*ctx.abort_flag) {
          volatile int never = 0;
          for (int i = max(0, G - kStages); i < G; ++i)
            mbar_wait(ctx.bar(BAR_V_FULL + i % kStages), (i / kStages) & 1, &never, nullptr, 0,
                      kWaitTimeoutNs);
        }
      }
    } else {
      // -------------------------------------------------------------- MMA issuer of M tile m
      const int m = warp - 1;
      if (lane == 0 && !skip) {
        // P.V of tile pv_G is issued after the next tile's Q.K^T: the softmax
        // releases S as soon as it has loaded it, long before P.
        int pv_G = -1;
        bool pv_first = false, pv_last = false;
        int G = 0, n = 0;
        Item it;
        bool ok = true;
        for (; ok && item_for(args, n, cta, &it); ++n) {
          const int qs = n & 1;
          if (!(ok = ctx.wait(BAR_Q_FULL + qs, (n >> 1) & 1) &&
                     ctx.wait(BAR_Q_READY + qs, (n >> 1) & 1)))
            break;
          for (int j = 0; j < it.n_tiles; ++j, ++G) {
            const int s = G % kStages;
            if (!(ok = ctx.wait(BAR_K_FULL + s, (G / kStages) & 1))) break;
            if (G > 0 && !(ok = ctx.wait(BAR_S_FREE + m, (G - 1) & 1))) break;
            tc_fence_after_sync();
            issue_qk(ctx, tmem, m, qs, s);
            mma_commit(ctx.bar(BAR_S_FULL + m));
            mma_commit(ctx.bar(BAR_K_EMPTY + s));
            if (pv_G >= 0 && !(ok = issue_pv(ctx, tmem, m, pv_G, pv_first, pv_last))) break;
            pv_G = G;
            pv_first = j == 0;
            pv_last = j == it.n_tiles - 1;
          }
        }
        if (ok && pv_G >= 0) issue_pv(ctx, tmem, m, pv_G, pv_first, pv_last);
        // Every MMA issued must finish before the tensor memory is released.
        mma_commit(ctx.bar(BAR_MMA_DONE + m));
        volatile int never = 0;
        mbar_wait(ctx.bar(BAR_MMA_DONE + m), 0, &never, nullptr, 0, kWaitTimeoutNs);
      }
    }
  } else if (wg == 1 || wg == 2) {
    // ---------------------------------------------------------------- softmax + epilogue
    setmaxnreg_inc<kRegsSoftmax>();
    const int m = wg - 1;          // M tile
    const int wq = warp & 3;       // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;  // row of the M tile = TMEM lane
    const bool elected = wq == 0 && lane == 0;  // issues this warpgroup's output stores
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + tmem_s(m);
    const uint32_t tP = tmem + lane_off + tmem_p(m);
    const uint32_t tO = tmem + lane_off + tmem_o(m);
    int G = 0, n = 0;
    int store_slot = -1;  // Q slot whose output store may still be reading shared memory
    Item it;
    bool ok = !skip;
    for (; ok && item_for(args, n, cta, &it); ++n) {
      const int qs = n & 1;
      // key index of this row's query token; this warp's tokens are tmin .. tmin+3
      const int tq = args.q_start + it.q0 + m * kTokensPerM + (r >> 3);
      const int tmin = args.q_start + it.q0 + m * kTokensPerM + wq * 4;
      const int tmax = tmin + 3;
      const float sink = __ldg(args.sinks + it.g * kGroup + (r & 7));
      const bool sink_off = isinf(sink) && sink < 0.f;
      float m_ref = sink_off ? -INFINITY : sink * kLog2e;
      float l = sink_off ? 0.f : 1.f;
      for (int j = 0; j < it.n_tiles; ++j, ++G) {
        if (!(ok = ctx.wait_warp(BAR_S_FULL + m, G & 1))) break;
        tc_fence_after_sync();
        uint32_t sv[128];
        tmem_ld128_split(tS, sv);
        // S is in registers: let the next Q.K^T overwrite it.
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(ctx.bar(BAR_S_FREE + m));
        if (store_slot >= 0 && elected) {
          // The previous item's output store has long finished reading its
          // staging tile; hand the Q slot back to the producer.
          tma_store_wait_read();
          mbar_arrive(ctx.bar(BAR_Q_EMPTY + store_slot));
        }
        store_slot = -1;
        const int kb = (it.jt0 + j) * kBlockN;
        const bool wmask = (kb + kBlockN - 1 > tmin) || (W > 0 && kb <= tmax - W);
        if (wmask) {
          // this row sees the tile's columns [c_lo, c_hi] (keys tq-W < j <= tq)
          const int c_hi = tq - kb;
          const int c_lo = W > 0 ? tq - W + 1 - kb : -1;
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i > c_hi || i < c_lo) sv[i] = __float_as_uint(-INFINITY);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; i += 8) {
          mx0 = fmax3(mx0, __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
          mx1 = fmax3(mx1, __uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3]));
          mx2 = fmax3(mx2, __uint_as_float(sv[i + 4]), __uint_as_float(sv[i + 5]));
          mx3 = fmax3(mx3, __uint_as_float(sv[i + 6]), __uint_as_float(sv[i + 7]));
        }
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * kScaleLog2;
        const float m_new = fmaxf(m_ref, mx);
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          if (m_new > m_ref) {
            l *= ex2_approx(m_ref - m_new);
            m_ref = m_new;
          }
        } else if (m_new > m_ref + kRescaleThreshold) {
          alpha = ex2_approx(m_ref - m_new);
          l *= alpha;
          m_ref = m_new;
          rescale = true;
        }
        // The two softmax warpgroups take turns on the exponential unit (M
        // tile 0 of tile G, M tile 1 of tile G, M tile 0 of tile G+1, ...):
        // each one's loads, max and stores overlap the other's exponentials.
        if (G > 0 || m == 1) {
          if (!(ok = ctx.wait_warp(BAR_TURN + m, (m == 0 ? G - 1 : G) & 1))) break;
        }
        // probabilities, packed to bf16 in place: sv[i] <- (p[2i], p[2i+1]);
        // scale-and-subtract and the row sum run on packed fp32 pairs
        const float mr = m_ref == -INFINITY ? 0.f : m_ref;
        const uint64_t c2 = f2_pack(kScaleLog2, kScaleLog2);
        const uint64_t nm2 = f2_pack(-mr, -mr);
        uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          float x0, x1, x2, x3;
          f2_unpack(ffma2(f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), c2,
                          nm2),
                    x0, x1);
          f2_unpack(ffma2(f2_pack(__uint_as_float(sv[2 * i + 2]), __uint_as_float(sv[2 * i + 3])),
                          c2, nm2),
                    x2, x3);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
          acc0 = fadd2(acc0, f2_pack(p0, p1));
          acc1 = fadd2(acc1, f2_pack(p2, p3));
          sv[i] = pack_bf16x2(p0, p1);
          sv[i + 1] = pack_bf16x2(p2, p3);
          if (i == kTurnHandOff) {
            // Hand the exponential unit to the other warpgroup before this
            // loop ends: its wake-up overlaps these last exponentials.
            __syncwarp();
            if (lane == 0) mbar_arrive(ctx.bar(BAR_TURN + (m ^ 1)));
          }
        }
        {
          float a0, a1, a2, a3;
          f2_unpack(acc0, a0, a1);
          f2_unpack(acc1, a2, a3);
          l += (a0 + a1) + (a2 + a3);
        }
        // P is free once the previous tile's P.V has completed.
        if (G > 0 && !(ok = ctx.wait_warp(BAR_P_FREE + m, (G - 1) & 1))) break;
        tc_fence_after_sync();
        {
          uint32_t pw[64];
#pragma unroll
          for (int i = 0; i < 64; ++i) pw[i] = sv[i];
          tmem_st64(tP, pw);
        }
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int ch = 0; ch < kHeadDim / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld32(tO + ch * 32, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
            tmem_st32(tO + ch * 32, ov);
          }
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(ctx.bar(BAR_P_FULL + m));
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 -> this M tile's half of the item's Q slot -> TMA store.
      // O_FULL follows the item's last P.V, so every Q.K^T that read the Q tile is done too.
      if (!(ok = ctx.wait_warp(BAR_O_FULL + m, n & 1))) break;
      tc_fence_after_sync();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      if (args.lse) {
        // natural-log normaliser of this row: (m_ref + log2 l) ln 2
        const int t = it.q0 + m * kTokensPerM + (r >> 3);
        if (t < S)
          args.lse[(static_cast<size_t>(it.b) * S + t) * kNumHeads + it.g * kGroup + (r & 7)] =
              l > 0.f ? (m_ref + __log2f(l)) * kLn2 : -INFINITY;
      }
      uint8_t* stage = smem + kOffQ + (2 * qs + m) * kTileBytes;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t ov[32];
        tmem_ld32(tO + 32 * half, ov);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(ov[8 * cc + 2 * e]) * inv_l,
                               __uint_as_float(ov[8 * cc + 2 * e + 1]) * inv_l);
          const int chunk = 4 * half + cc;
          *reinterpret_cast<uint4*>(stage + r * 128 + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      // O has been read: the next item's first P.V (which overwrites it) is
      // issued only after this warpgroup's next P_FULL.
      tc_fence_before_sync();
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_STAGED + m));
      if (elected) {
        ok = ctx.wait(BAR_STAGED + m, n & 1);
        if (ok && it.q0 + m * kTokensPerM < S)
          tma_store_4d(&maps.o, ctx.q_tile(qs, m), 0, it.g * kGroup, it.q0 + m * kTokensPerM,
                       it.b);
        tma_store_commit();
      }
      store_slot = qs;
      ok = __all_sync(0xffffffffu, ok);
    }
    if (elected) {
      tma_store_wait_all();
      if (ok && store_slot >= 0) mbar_arrive(ctx.bar(BAR_Q_EMPTY + store_slot));
    }
  } else {
    // ---------------------------------------------------------------- RoPE
    setmaxnreg_dec<kRegsLight>();
    const int t = static_cast<int>(threadIdx.x) - 384;  // 0..127: row t of both M tiles
    int n = 0;
    Item it;
    bool ok = !skip;
    for (; ok && item_for(args, n, cta, &it); ++n) {
      const int qs = n & 1;
      if (!(ok = ctx.wait_warp(BAR_Q_FULL + qs, (n >> 1) & 1))) break;
      const uint8_t* tab = smem + kOffTab + qs * kTabSlotBytes;
#pragma unroll 1
      for (int mm = 0; mm < 2; ++mm) {
        const int tl = mm * kTokensPerM + (t >> 3);  // token within the item
        if (it.q0 + tl < S)
          rope_row(smem + kOffQ + (2 * qs + mm) * kTileBytes + t * 128, t,
                   reinterpret_cast<const float2*>(tab + tl * kTabRowBytes));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_Q_READY + qs));
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool prefill_uses_band(int window) { return window > 0 && window <= 128; }

int prefill_items(int batch, int seqlen, int window) {
  const int tokens = prefill_uses_band(window) ? kBandTokens : kBlockQ;
  return (seqlen + tokens - 1) / tokens * kNumKvHeads * batch;
}

// While the keys and values of every (b, g) pair fit in half of L2 (126 MB),
// the plain longest-first order balances best. Beyond that, chunks of C query
// tiles with C large enough that the ~grid/C pairs a wave touches hold at most
// 64 MB of keys and values (256 bytes per key and kv head).
int prefill_order_chunk(int batch, int keys, int grid) {
  const double kv_bytes = 256.0 * keys;  // one (b, g) pair
  if (kv_bytes * kNumKvHeads * batch <= 64.0 * 1024 * 1024) return 0;
  const int c = static_cast<int>(std::ceil(grid * kv_bytes / (64.0 * 1024 * 1024)));
  return c < 1 ? 1 : c;
}

// Both attention kernels are launched with programmatic stream serialization:
// they may start while the key-rotation kernel before them finishes, and only
// the thread that loads rotated keys waits for it (griddep_wait).
cudaError_t launch_prefill(const PrefillMaps& maps, const PrefillArgs& args, cudaStream_t stream) {
  const int grid = args.n_items < args.grid ? args.n_items : args.grid;
  if (prefill_uses_band(args.window)) return launch_prefill_band(maps, args, grid, stream);
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefill_kernel, maps, args);
}

}  // namespace gqa
