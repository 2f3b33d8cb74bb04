// Narrow-band prefill kernel for sm_100a (sliding windows of at most 128 keys,
// the model's W = 128 layers): gpt-oss-style grouped-query attention with
// half-split RoPE and a learned sink logit (gpt-oss pages: inteligile
// techniques map rows "Grouped-query attention", "Partial RoPE", "Learnable
// attention sink", "Sliding-window attention").
#include "prefill_common.cuh"

namespace gqa {
namespace {

// Narrow-band kernel for sliding windows 0 < W <= 128 (the model's W = 128).
//
// Work item: batch b, kv head g, 16 query tokens = one M=128 tile. Query i
// (key index q_start+i) sees keys (i-W, i], so an item needs only the 144 keys
// [q0-128, q0+16): S = Q K^T with N = 144 and a single-tile softmax (no online
// rescaling), then P V over the same keys. Each CTA walks a contiguous run of
// items in (batch, kv head, query tile) order, so consecutive items of one
// (b, g) share 128 of their 144 keys: keys and values sit in a ring of 16-key
// blocks in shared memory and an item loads only its own 16 keys (all 9 blocks
// when the run enters a (b, g)). Q tiles, with the rotary-table rows of their
// tokens, have a ring of their own that Q K^T releases. Keys arrive rotated.
//
// Roles (512 threads):
//   warp 0     TMA producer: per item the Q tile and its table rows, then the
//              item's new key/value blocks.
//   warp 1     tcgen05 issuer (owns TMEM): Q K^T of item k (N = 144, cut in two
//              where the span wraps around the ring) and P V of item k-1 (one
//              K = 16 MMA per key block), in whichever order their inputs land.
//              Its loop does no division and no descriptor encoding: an MMA
//              costs its issuing thread tens of cycles, and with two issues per
//              item this thread sits on every item's critical path.
//   WG1, WG2   softmax of alternate items (thread = TMEM lane = query row):
//              band-edge mask, max with the sink, exp2, bf16 P over S, row sum
//              (and the log-normaliser when asked for); then the output of the
//              warpgroup's previous item: O/l from TMEM -> bf16 -> the thread's
//              128-byte row of `out`, stored from registers.
//   WG3        rotates each item's Q rows in shared memory (as far ahead as the
//              Q ring allows).
// TMEM: S/P of the two softmax warpgroups at columns 0 and 160 (144 each); three
// O accumulators at 320, 384 and 448 (item k's is k % 3), so a warpgroup reads
// its previous item's O while P V of the next items already runs.
namespace band {

constexpr int kTokens = kBandTokens;
constexpr int kSpan = 144;  // 128 keys before the tile + the tile's 16
constexpr int kSpanBlocks = kSpan / 16;
constexpr int kQSlots = 4;
constexpr int kRing = 18;  // key/value blocks of 16 keys
// Register budgets after the warpgroup split (launch is 512 x 128): the
// softmax rows here are 144 scores wide, so it gets more than in prefill_kernel.
constexpr uint32_t kRegsLight = 72;     // WG0 and WG3
constexpr uint32_t kRegsSoftmax = 184;  // WG1 and WG2
static_assert(2 * 128 * kRegsLight + 2 * 128 * kRegsSoftmax <= 512 * 128, "register split");
constexpr uint32_t kQBytes = 128 * 128;
constexpr uint32_t kBlkBytes = 16 * 128;
constexpr uint32_t kTabBytes = kTokens * kRopePairs * 8;  // table rows of the 16 tokens
constexpr uint32_t kOffQ = 0;                                // [kQSlots] Q tiles
constexpr uint32_t kOffK = kOffQ + kQSlots * kQBytes;        // [kRing] key blocks
constexpr uint32_t kOffV = kOffK + kRing * kBlkBytes;        // [kRing] value blocks
constexpr uint32_t kOffTab = kOffV + kRing * kBlkBytes;      // [kQSlots] table rows
constexpr int kOBufs = 3;  // O accumulators: item k's is k % 3
enum : int {
  BAR_Q_FULL = 0,                      // [kQSlots] Q tile and table rows landed
  BAR_Q_READY = BAR_Q_FULL + kQSlots,  // [kQSlots] Q rotated
  BAR_Q_EMPTY = BAR_Q_READY + kQSlots, // [kQSlots] Q K^T done with the slot
  BAR_B_FULL = BAR_Q_EMPTY + kQSlots,  // [kRing] key and value block landed
  BAR_B_EMPTY = BAR_B_FULL + kRing,    // [kRing] last P V over the block done
  BAR_S_FULL = BAR_B_EMPTY + kRing,    // [2] S of softmax warpgroup m
  BAR_P_FULL = BAR_S_FULL + 2,         // [2]
  BAR_O_FULL = BAR_P_FULL + 2,         // [kOBufs] P V done
  BAR_O_EMPTY = BAR_O_FULL + kOBufs,   // [kOBufs] O read out
  BAR_MMA_DONE = BAR_O_EMPTY + kOBufs,
  NUM_BARS
};
constexpr uint32_t kOffBar = kOffTab + kQSlots * kTabBytes;
constexpr uint32_t kOffMisc = kOffBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0, "swizzle atoms");
static_assert(kRing >= 2 * kSpanBlocks, "a run's new (b, g) must not wait on the last span");
__host__ __device__ constexpr uint32_t tmem_s(int m) { return m ? 160u : 0u; }
__host__ __device__ constexpr uint32_t tmem_o(int i) { return 320u + 64u * static_cast<uint32_t>(i); }

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
  __device__ uint32_t q(int s) const { return sbase + kOffQ + s * kQBytes; }
  __device__ uint32_t kblk(int j) const { return sbase + kOffK + j * kBlkBytes; }
  __device__ uint32_t vblk(int j) const { return sbase + kOffV + j * kBlkBytes; }
  __device__ uint32_t tab(int s) const { return sbase + kOffTab + s * kTabBytes; }
};

struct Item {
  int b, g, q0;
};

// This CTA's run: items [lo, lo + n) of the list ordered by batch, kv head and
// query tile (runs differ in length by at most one). Item lo + k is query tile
// (lo + k) % n_t of pair b * 8 + g = (lo + k) / n_t; every role steps these
// coordinates instead of dividing. A run's first item of a (b, g) loads the
// whole span (9 blocks), every other item one block; its last item of a (b, g)
// frees the whole span, every other item the span's oldest block.
struct Run {
  int lo, n, n_t;
  __device__ Run(const PrefillArgs& a, int cta) {
    const long long grid = gridDim.x;
    lo = static_cast<int>(cta * static_cast<long long>(a.n_items) / grid);
    n = static_cast<int>((cta + 1) * static_cast<long long>(a.n_items) / grid) - lo;
    n_t = (a.seqlen + kTokens - 1) / kTokens;
  }
};

}  // namespace band

__global__ void __launch_bounds__(kThreads, 1)
    prefill_band_kernel(const __grid_constant__ PrefillMaps maps, const PrefillArgs args) {
  using namespace band;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  band::Ctx ctx;
  ctx.sbase = smem_u32(smem);
  ctx.abort_flag = reinterpret_cast<volatile int*>(smem + band::kOffMisc + 4);
  ctx.err = args.err;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + band::kOffMisc);

  const int warp = static_cast<int>(threadIdx.x >> 5);
  const int lane = static_cast<int>(threadIdx.x & 31);
  const int cta = static_cast<int>(blockIdx.x);
  const int S = args.seqlen;
  const int W = args.window;
  const band::Run run(args, cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < band::kQSlots; ++s) {
      mbar_init(ctx.bar(band::BAR_Q_FULL + s), 1);
      mbar_init(ctx.bar(band::BAR_Q_READY + s), 4);
      mbar_init(ctx.bar(band::BAR_Q_EMPTY + s), 1);
    }
    for (int j = 0; j < band::kRing; ++j) {
      mbar_init(ctx.bar(band::BAR_B_FULL + j), 1);
      mbar_init(ctx.bar(band::BAR_B_EMPTY + j), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(ctx.bar(band::BAR_S_FULL + i), 1);
      mbar_init(ctx.bar(band::BAR_P_FULL + i), 4);
    }
    for (int i = 0; i < band::kOBufs; ++i) {
      mbar_init(ctx.bar(band::BAR_O_FULL + i), 1);
      mbar_init(ctx.bar(band::BAR_O_EMPTY + i), 4);
    }
    mbar_init(ctx.bar(band::BAR_MMA_DONE), 1);
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
    setmaxnreg_dec<band::kRegsLight>();
    if (warp == 0) {
      // -------------------------------------------------------------- producer
      if (lane == 0 && !skip) {
        prefetch_tensormap(&maps.q);
        prefetch_tensormap(&maps.k_band);
        prefetch_tensormap(&maps.v_band);
        int nq = 0, nb = 0;  // Q tiles and key/value blocks requested
        int qs = 0, bslot = 0;
        uint32_t qpar = 0, bpar = 0;  // phases of the next Q slot / ring slot use
        const int n_t = run.n_t;
        // Positions of an item's tokens are loaded one item ahead into the
        // other of two register sets, so their round trip to memory hides
        // behind the slot waits and the previous item's copies.
        int pa[band::kTokens], pb[band::kTokens];
        auto issue = [&](int k, int t, int bg, const int (&p)[band::kTokens]) -> bool {
          const int b = bg >> 3, g = bg & 7, q0 = t * band::kTokens;
          if (k >= band::kQSlots && !ctx.wait(band::BAR_Q_EMPTY + qs, qpar ^ 1u)) return false;
          const uint32_t tab_bytes =
              kRopePairs * 8 * static_cast<uint32_t>(min(band::kTokens, S - q0));
          mbar_arrive_expect_tx(ctx.bar(band::BAR_Q_FULL + qs), band::kQBytes + tab_bytes);
          tma_load_4d(ctx.q(qs), &maps.q, ctx.bar(band::BAR_Q_FULL + qs), 0, g * kGroup, q0, b);
          stage_rope_rows_at<band::kTokens>(args, p, q0, ctx.tab(qs), ctx.bar(band::BAR_Q_FULL + qs));
          ++nq;
          if (++qs == band::kQSlots) {
            qs = 0;
            qpar ^= 1u;
          }
          // key index of the first new key: the span start for a run's first
          // item of a (b, g), else the item's own first token
          const bool first = k == 0 || t == 0;
          const int kb = args.q_start + q0 - (first ? 128 : 0);
          const int n_new = first ? band::kSpanBlocks : 1;
          for (int j = 0; j < n_new; ++j) {
            if (nb >= band::kRing && !ctx.wait(band::BAR_B_EMPTY + bslot, bpar ^ 1u)) return false;
            // rotated keys: see the same wait in prefill_kernel
            if (nb == 0) griddep_wait();
            const uint32_t fb = ctx.bar(band::BAR_B_FULL + bslot);
            mbar_arrive_expect_tx(fb, 2 * band::kBlkBytes);
            tma_load_4d(ctx.kblk(bslot), &maps.k_band, fb, 0, g, kb + 16 * j, b);
            tma_load_4d(ctx.vblk(bslot), &maps.v_band, fb, 0, g, kb + 16 * j, b);
            ++nb;
            if (++bslot == band::kRing) {
              bslot = 0;
              bpar ^= 1u;
            }
          }
          return true;
        };
        int t = run.lo % n_t, bg = run.lo / n_t;  // query tile and b*8+g of item k
        auto next = [&](int& tt, int& bb) {
          if (++tt == n_t) {
            tt = 0;
            ++bb;
          }
        };
        load_positions(args, bg >> 3, t * band::kTokens, pa);
        for (int k = 0; k < run.n; k += 2) {
          int t1 = t, bg1 = bg;
          next(t1, bg1);
          if (k + 1 < run.n) load_positions(args, bg1 >> 3, t1 * band::kTokens, pb);
          if (!issue(k, t, bg, pa) || k + 1 >= run.n) break;
          int t2 = t1, bg2 = bg1;
          next(t2, bg2);
          if (k + 2 < run.n) load_positions(args, bg2 >> 3, t2 * band::kTokens, pa);
          if (!issue(k + 1, t1, bg1, pb)) break;
          t = t2;
          bg = bg2;
        }
        if (*ctx.abort_flag) {
          // drain the copies still in flight before the CTA exits
          volatile int never = 0;
          for (int i = max(0, nq - band::kQSlots); i < nq; ++i)
            mbar_wait(ctx.bar(band::BAR_Q_FULL + i % band::kQSlots), (i / band::kQSlots) & 1,
                      &never, nullptr, 0, kWaitTimeoutNs);
          for (int j = max(0, nb - band::kRing); j < nb; ++j)
            mbar_wait(ctx.bar(band::BAR_B_FULL + j % band::kRing), (j / band::kRing) & 1, &never,
                      nullptr, 0, kWaitTimeoutNs);
        }
      }
    } else if (warp == 1) {
      // -------------------------------------------------------------- MMA issuer
      // Q.K^T of item kq and P.V of item kp are independent, so they are issued
      // in whichever order their inputs arrive (rotated Q and the item's key
      // blocks for Q.K^T, P for P.V). Q.K^T of item kq overwrites S/P of item
      // kq-2, so it is issued only after that item's P.V (the tensor core runs
      // one thread's MMAs in order).
      if (lane == 0 && !skip) {
        // Everything per MMA is precomputed or stepped: a shared-memory
        // descriptor advances by one per 16 bytes of its start address, ring
        // slots and phases are counters, and the items' (b, g) boundaries come
        // from a tile counter (no division on the issue path).
        constexpr uint32_t idesc_pv = idesc_bf16(128, kHeadDim, true);
        constexpr uint64_t kQStep = band::kQBytes >> 4, kBlkStep = band::kBlkBytes >> 4;
        const uint64_t qdesc0 = sdesc_sw128(ctx.q(0));
        const uint64_t kdesc0 = sdesc_sw128(ctx.kblk(0));
        const uint64_t vdesc0 = sdesc_sw128(ctx.vblk(0));
        const int n_t = run.n_t, last_k = run.n - 1;
        int kq = 0, kp = 0;
        int qs = 0;
        uint32_t qpar = 0;                       // Q slot of item kq and its phase
        int tq = run.lo % n_t, tp = tq;          // query tile of items kq and kp
        int q_end = band::kSpanBlocks;           // blocks through item kq
        int qb0 = 0, pb0 = 0;                    // ring slot of the span start of kq / kp
        int ready = 0, rslot = 0;                // blocks seen landed; ring slot of the next
        uint32_t rpar = 0;
        int ob = 0;                              // O buffer of item kp and its phase
        uint32_t opar = 0;
        bool ok = true;
        uint64_t t_progress = global_timer_ns();
        uint32_t idle = 0;
        while (ok && kp < run.n) {
          bool progressed = false;
          if (kq < run.n && kq <= kp + 1) {
            while (ready < q_end && mbar_test_wait(ctx.bar(band::BAR_B_FULL + rslot), rpar)) {
              ++ready;
              if (++rslot == band::kRing) {
                rslot = 0;
                rpar ^= 1u;
              }
            }
            if (ready >= q_end && mbar_test_wait(ctx.bar(band::BAR_Q_READY + qs), qpar)) {
              tc_fence_after_sync();
              const uint32_t tS = tmem + ((kq & 1) ? band::tmem_s(1) : band::tmem_s(0));
              const uint64_t qd = qdesc0 + static_cast<uint64_t>(qs) * kQStep;
              const uint64_t kd = kdesc0 + static_cast<uint64_t>(qb0) * kBlkStep;
              const int n1 = band::kRing - qb0;  // blocks before the ring wraps
              if (n1 >= band::kSpanBlocks) {
                constexpr uint32_t id = idesc_bf16(128, band::kSpan, false);
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk)
                  mma_bf16_ss(tS, qd + 2 * kk, kd + 2 * kk, id, kk > 0 ? 1u : 0u);
              } else {
                const uint32_t id1 = idesc_bf16(128, 16 * n1, false);
                const uint32_t id2 = idesc_bf16(128, band::kSpan - 16 * n1, false);
                const uint32_t tS2 = tS + 16 * n1;
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) {
                  mma_bf16_ss(tS, qd + 2 * kk, kd + 2 * kk, id1, kk > 0 ? 1u : 0u);
                  mma_bf16_ss(tS2, qd + 2 * kk, kdesc0 + 2 * kk, id2, kk > 0 ? 1u : 0u);
                }
              }
              mma_commit(ctx.bar(band::BAR_S_FULL + (kq & 1)));
              mma_commit(ctx.bar(band::BAR_Q_EMPTY + qs));
              if (++qs == band::kQSlots) {
                qs = 0;
                qpar ^= 1u;
              }
              ++kq;
              if (++tq == n_t) tq = 0;
              const int step = tq == 0 ? band::kSpanBlocks : 1;  // a new (b, g) loads its span
              q_end += step;
              qb0 += step;
              if (qb0 >= band::kRing) qb0 -= band::kRing;
              progressed = true;
            }
          }
          if (kp < kq) {
            const int m = kp & 1;
            if (mbar_test_wait(ctx.bar(band::BAR_P_FULL + m), (kp >> 1) & 1) &&
                (kp < band::kOBufs ||
                 mbar_test_wait(ctx.bar(band::BAR_O_EMPTY + ob), opar ^ 1u))) {
              tc_fence_after_sync();
              const uint32_t tS = tmem + (m ? band::tmem_s(1) : band::tmem_s(0));
              const uint32_t tO = tmem + band::tmem_o(0) + 64u * static_cast<uint32_t>(ob);
              int sl = pb0;
#pragma unroll
              for (int t = 0; t < band::kSpanBlocks; ++t) {
                mma_bf16_ts(tO, tS + 8 * t, vdesc0 + static_cast<uint64_t>(sl) * kBlkStep,
                            idesc_pv, t > 0 ? 1u : 0u);
                sl = sl + 1 == band::kRing ? 0 : sl + 1;
              }
              mma_commit(ctx.bar(band::BAR_O_FULL + ob));
              if (++ob == band::kOBufs) {
                ob = 0;
                opar ^= 1u;
              }
              // the span's oldest block has no later user in this (b, g); at
              // the run's last item of the (b, g) none of the span has
              const bool last = kp == last_k || tp == n_t - 1;
              sl = pb0;
              for (int t = 0; t < (last ? band::kSpanBlocks : 1); ++t) {
                mma_commit(ctx.bar(band::BAR_B_EMPTY + sl));
                sl = sl + 1 == band::kRing ? 0 : sl + 1;
              }
              ++kp;
              if (++tp == n_t) tp = 0;
              pb0 += tp == 0 ? band::kSpanBlocks : 1;
              if (pb0 >= band::kRing) pb0 -= band::kRing;
              progressed = true;
            }
          }
          if (progressed) {
            idle = 0;
          } else {
            if ((++idle & 1023u) == 0u) {
              if (*ctx.abort_flag) {
                ok = false;
              } else if (idle == 1024u) {
                t_progress = global_timer_ns();
              } else if (global_timer_ns() - t_progress > kWaitTimeoutNs) {
                *ctx.abort_flag = 1;
                atomicOr(args.err, kErrTimeout);
                ok = false;
              }
            }
          }
        }
        mma_commit(ctx.bar(band::BAR_MMA_DONE));
        volatile int never = 0;
        mbar_wait(ctx.bar(band::BAR_MMA_DONE), 0, &never, nullptr, 0, kWaitTimeoutNs);
      }
    }
    // warps 2-3 have no role here
  } else if (wg == 1 || wg == 2) {
    // ---------------------------------------------------------------- softmax
    setmaxnreg_inc<band::kRegsSoftmax>();
    const int m = wg - 1;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + band::tmem_s(m);
    bool ok = !skip;
    float l_prev = 1.f;
    // Item k_e's output: O (buffer k_e % 3) / l -> bf16 -> this thread's
    // 128-byte row of `out`, written straight from registers. Its (b*8+g,
    // query tile) are passed in.
    auto epilogue = [&](int k_e, int bg_e, int t_e, float l_e) -> bool {
      const int ob = k_e % band::kOBufs;
      if (!ctx.wait_warp(band::BAR_O_FULL + ob, (k_e / band::kOBufs) & 1)) return false;
      tc_fence_after_sync();
      const int de = r >> 3;
      const int q0e = t_e * band::kTokens;
      const float inv_l = 1.f / l_e;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(args.out) +
                   ((static_cast<size_t>(bg_e >> 3) * S + q0e + de) * kNumHeads +
                    (bg_e & 7) * kGroup + (r & 7)) * kHeadDim);
      const bool in = q0e + de < S;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t ov[32];
        tmem_ld32(tmem + lane_off + band::tmem_o(ob) + 32 * half, ov);
        if (half == 1) {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(ctx.bar(band::BAR_O_EMPTY + ob));
        }
        if (in) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack_bf16x2(__uint_as_float(ov[8 * cc + 2 * e]) * inv_l,
                                 __uint_as_float(ov[8 * cc + 2 * e + 1]) * inv_l);
            dst[4 * half + cc] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      return true;
    };
    // sink logits of this row's head in each kv group
    float sk[kNumKvHeads];
#pragma unroll
    for (int g = 0; g < kNumKvHeads; ++g) sk[g] = __ldg(args.sinks + g * kGroup + (r & 7));
    int t_cur = (run.lo + m) % run.n_t, bg_cur = (run.lo + m) / run.n_t;  // item k = m
    int t_prev = 0, bg_prev = 0;
    for (int k = m, i = 0; ok && k < run.n; k += 2, ++i) {
      band::Item it;
      it.b = bg_cur >> 3;
      it.g = bg_cur & 7;
      it.q0 = t_cur * band::kTokens;
      // row token q0 + d (key index kq0 + d) sees keys (kq0+d-W, kq0+d], i.e.
      // span columns [max(128-kq0, d+129-W), d+128] of the span starting at
      // key kq0-128
      const int d = r >> 3;
      const int kq0 = args.q_start + it.q0;  // key index of the item's first query token
      const int c_lo = max(128 - kq0, d + 129 - W);
      const int c_hi = d + 128;
      float sink = sk[0];
#pragma unroll
      for (int g = 1; g < kNumKvHeads; ++g)
        if (it.g == g) sink = sk[g];
      const bool sink_off = isinf(sink) && sink < 0.f;
      if (!(ok = ctx.wait_warp(band::BAR_S_FULL + m, i & 1))) break;
      tc_fence_after_sync();
      uint32_t sv[band::kSpan];
      tmem_ld144_split(tS, sv);
      // Columns that can be masked: those before c_lo and after c_hi. With
      // W = 128 and q0 >= 128 that is only [0, 17) and [128, 144).
      // (Only the executed branch occupies the instruction cache, so the
      // common case stays short.)
      if (W == 128 && kq0 >= 128) {
#pragma unroll
        for (int c = 0; c < 17; ++c)
          if (c < c_lo) sv[c] = __float_as_uint(-INFINITY);
#pragma unroll
        for (int c = 128; c < band::kSpan; ++c)
          if (c > c_hi) sv[c] = __float_as_uint(-INFINITY);
      } else {
#pragma unroll
        for (int c = 0; c < band::kSpan; ++c)
          if (c < c_lo || c > c_hi) sv[c] = __float_as_uint(-INFINITY);
      }
      float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < band::kSpan; c += 8) {
        m0 = fmax3(m0, __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
        m1 = fmax3(m1, __uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3]));
        m2 = fmax3(m2, __uint_as_float(sv[c + 4]), __uint_as_float(sv[c + 5]));
        m3 = fmax3(m3, __uint_as_float(sv[c + 6]), __uint_as_float(sv[c + 7]));
      }
      const float mx = fmaxf(fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * kScaleLog2,
                             sink_off ? -INFINITY : sink * kLog2e);
      const float mr = mx == -INFINITY ? 0.f : mx;
      const uint64_t c2 = f2_pack(kScaleLog2, kScaleLog2);
      const uint64_t nm2 = f2_pack(-mr, -mr);
      uint64_t acc0 = f2_pack(sink_off ? 0.f : ex2_approx(sink * kLog2e - mr), 0.f);
      uint64_t acc1 = f2_pack(0.f, 0.f);
      // probabilities packed to bf16 in place: sv[c] <- (p[2c], p[2c+1])
#pragma unroll
      for (int c = 0; c < band::kSpan / 2; c += 2) {
        float x0, x1, x2, x3;
        f2_unpack(ffma2(f2_pack(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), c2,
                        nm2),
                  x0, x1);
        f2_unpack(ffma2(f2_pack(__uint_as_float(sv[2 * c + 2]), __uint_as_float(sv[2 * c + 3])),
                        c2, nm2),
                  x2, x3);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
        acc0 = fadd2(acc0, f2_pack(p0, p1));
        acc1 = fadd2(acc1, f2_pack(p2, p3));
        sv[c] = pack_bf16x2(p0, p1);
        sv[c + 1] = pack_bf16x2(p2, p3);
      }
      float l0, l1;
      {
        float a0, a1, a2, a3;
        f2_unpack(acc0, a0, a1);
        f2_unpack(acc1, a2, a3);
        l0 = a0 + a2;
        l1 = a1 + a3;
      }
      if (args.lse && it.q0 + d < S)
        args.lse[(static_cast<size_t>(it.b) * S + it.q0 + d) * kNumHeads + it.g * kGroup +
                 (r & 7)] = (mr + __log2f(l0 + l1)) * kLn2;
      {
        uint32_t a[64], b8[8];
#pragma unroll
        for (int c = 0; c < 64; ++c) a[c] = sv[c];
#pragma unroll
        for (int c = 0; c < 8; ++c) b8[c] = sv[64 + c];
        tmem_st64(tS, a);
        tmem_st8(tS + 64, b8);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(band::BAR_P_FULL + m));
      // output of this warpgroup's previous item (its P V finished long ago)
      if (k >= 2 && !(ok = epilogue(k - 2, bg_prev, t_prev, l_prev))) break;
      l_prev = l0 + l1;
      t_prev = t_cur;
      bg_prev = bg_cur;
      t_cur += 2;
      while (t_cur >= run.n_t) {
        t_cur -= run.n_t;
        ++bg_cur;
      }
    }
    // and of its last item
    const int k_last = run.n - 1 - ((run.n - 1 - m) & 1);
    if (ok && k_last >= 0) epilogue(k_last, bg_prev, t_prev, l_prev);
  } else {
    // ---------------------------------------------------------------- Q rotation
    setmaxnreg_dec<band::kRegsLight>();
    const int r = (warp & 3) * 32 + lane;
    // Rotation work of thread r: chunk pair c (elements 8c..8c+7 and 8c+32..
    // 8c+39) of heads 4h..4h+3 of token t, which share one table chunk. Within
    // a quarter warp the 8 (c, h) combinations of one token and row step hit
    // 8 distinct 16-byte bank groups of the swizzled tile.
    const int rt = r >> 3, rc = r & 3, rh = (r >> 2) & 1;
    int qs = 0;
    uint32_t qpar = 0;
    int t = run.lo % run.n_t;  // query tile of item k
    for (int k = 0; !skip && k < run.n; ++k) {
      if (!ctx.wait_warp(band::BAR_Q_FULL + qs, qpar)) break;
      if (t * band::kTokens + rt < S) {
        const float4* t4 = reinterpret_cast<const float4*>(
            smem + band::kOffTab + qs * band::kTabBytes + rt * kRopePairs * 8 + rc * 64);
        const float4 t0 = t4[0], t1 = t4[1], t2 = t4[2], t3 = t4[3];
        const float cv[8] = {t0.x, t0.z, t1.x, t1.z, t2.x, t2.z, t3.x, t3.z};
        const float sn[8] = {t0.y, t0.w, t1.y, t1.w, t2.y, t2.w, t3.y, t3.w};
        uint8_t* qt = smem + band::kOffQ + qs * band::kQBytes;
#pragma unroll 2
        for (int j = 0; j < 4; ++j) {
          const int row = rt * 8 + rh * 4 + j;
          rope_chunk(qt + row * 128, row, rc, cv, sn);
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(band::BAR_Q_READY + qs));
      if (++qs == band::kQSlots) {
        qs = 0;
        qpar ^= 1u;
      }
      if (++t == run.n_t) t = 0;
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

cudaError_t launch_prefill_band(const PrefillMaps& maps, const PrefillArgs& args, int grid,
                                cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(prefill_band_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(band::kSmemBytes));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = band::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, prefill_band_kernel, maps, args);
}

}  // namespace gqa
