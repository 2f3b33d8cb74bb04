// Prefill attention kernel for sm_100a: gpt-oss-style grouped-query attention
// (64 query heads over 8 key/value heads, head_dim 64) with half-split RoPE,
// a learned sink logit in the softmax denominator, and full-causal or
// sliding-window masks (gpt-oss pages: inteligile techniques map rows
// "Grouped-query attention", "Partial RoPE", "Learnable attention sink",
// "Sliding-window attention"; llm-atlas field tables for the constants).
//
// One CTA handles one work item: batch b, key/value head g, and 32 query
// tokens. The 8 query heads of group g are packed into the M dimension, so a
// work item is two M=128 tiles (16 tokens x 8 heads each) that share every
// K/V tile loaded. Roles (512 threads):
//   warp 0       TMA producer: Q once, then K/V tiles of 128 keys through a
//                kStages-deep ring.
//   warp 1       TMEM owner and tcgen05 issuer (one thread): S = Q K^T
//                (SS, K-major) and O += P V (A = P from TMEM, B = V MN-major).
//   warps 4-7    softmax for M tile 0 (thread = TMEM lane = one query row)
//   warps 8-11   softmax for M tile 1
//   warps 12-15  RoPE: rotate Q rows and every K tile in shared memory.
// Online softmax in log2 units with the running max seeded by the sink,
// m0 = sigma*log2(e) and l0 = 1; O is rescaled only when the max grows by
// more than 2^8 (the result is exact because O and l share the reference).
// Tiles wholly outside the causal/window band are never visited; only
// boundary tiles evaluate the mask per element.
#include <cmath>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {
namespace {

constexpr int kBlockQ = 32;      // query tokens per work item
constexpr int kTokensPerM = 16;  // tokens per M=128 tile (x 8 heads)
constexpr int kBlockN = 128;     // keys per K/V tile
constexpr int kStages = 3;
constexpr int kThreads = 512;
constexpr uint32_t kTileBytes = 128 * 128;  // 128 rows of 64 bf16

constexpr uint32_t kTmemCols = 512;
// TMEM columns of M tile m: S (fp32, 128 columns) with P (bf16) aliased on
// its first 64, and the O accumulator (fp32, 64 columns).
__host__ __device__ constexpr uint32_t tmem_s(int m) { return m ? 128u : 0u; }
__host__ __device__ constexpr uint32_t tmem_o(int m) { return m ? 320u : 256u; }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kScaleLog2 = 0.125f * kLog2e;  // 1/sqrt(64) * log2(e)
constexpr float kRescaleThreshold = 8.0f;      // log2 units

enum : int {
  BAR_Q_FULL = 0,
  BAR_Q_READY,
  BAR_K_FULL,
  BAR_V_FULL = BAR_K_FULL + kStages,
  BAR_K_READY = BAR_V_FULL + kStages,
  BAR_KV_EMPTY = BAR_K_READY + kStages,
  BAR_S_FULL = BAR_KV_EMPTY + kStages,
  BAR_P_FULL = BAR_S_FULL + 2,
  BAR_O_FULL = BAR_P_FULL + 2,
  BAR_MMA_DONE = BAR_O_FULL + 2,
  NUM_BARS
};

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
constexpr uint32_t kOffMisc = kOffBar + NUM_BARS * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment

struct Ctx {
  uint32_t sbase;
  volatile int* abort_flag;
  int* err;
  __device__ uint32_t bar(int i) const { return sbase + kOffBar + 8u * static_cast<uint32_t>(i); }
  __device__ bool wait(int i, uint32_t parity) const {
    return mbar_wait(bar(i), parity, abort_flag, err, kErrTimeout, kWaitTimeoutNs);
  }
};

__device__ __forceinline__ int load_position(const PrefillArgs& a, int b, int t) {
  int p = __ldg(a.pos + static_cast<size_t>(b) * a.seqlen + t);
  if (p < 0 || p >= kMaxPosition) {
    atomicOr(a.err, kErrPosition);
    p = p < 0 ? 0 : kMaxPosition - 1;
  }
  return p;
}

// Rotate one 64-element row stored at `row` (128 bytes, 128B-swizzled with
// row index r) by the table entry of position p, in place.
__device__ __forceinline__ void rope_row(uint8_t* row, int r, const float2* __restrict__ cs) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4* plo = reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4));
    uint4* phi = reinterpret_cast<uint4*>(row + (((c + 4) ^ (r & 7)) << 4));
    const uint4 a = *plo, h = *phi;
    const float4* t4 = reinterpret_cast<const float4*>(cs + 8 * c);
    const float4 t0 = __ldg(t4 + 0), t1 = __ldg(t4 + 1), t2 = __ldg(t4 + 2), t3 = __ldg(t4 + 3);
    const float cv[8] = {t0.x, t0.z, t1.x, t1.z, t2.x, t2.z, t3.x, t3.z};
    const float sv[8] = {t0.y, t0.w, t1.y, t1.w, t2.y, t2.w, t3.y, t3.w};
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
    uint32_t ya[4], yh[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x1l = bf16lo_to_f32(aw[e]), x1h = bf16hi_to_f32(aw[e]);
      const float x2l = bf16lo_to_f32(hw[e]), x2h = bf16hi_to_f32(hw[e]);
      const float cl = cv[2 * e], ch = cv[2 * e + 1], sl = sv[2 * e], sh = sv[2 * e + 1];
      ya[e] = pack_bf16x2(fmaf(x1l, cl, -x2l * sl), fmaf(x1h, ch, -x2h * sh));
      yh[e] = pack_bf16x2(fmaf(x2l, cl, x1l * sl), fmaf(x2h, ch, x1h * sh));
    }
    *plo = make_uint4(ya[0], ya[1], ya[2], ya[3]);
    *phi = make_uint4(yh[0], yh[1], yh[2], yh[3]);
  }
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
  const int qt = args.n_qtiles - 1 - static_cast<int>(blockIdx.x);  // longest rows first
  const int g = static_cast<int>(blockIdx.y);
  const int b = static_cast<int>(blockIdx.z);
  const int S = args.seqlen;
  const int W = args.window;
  const int q0 = qt * kBlockQ;
  const int qlast = min(q0 + kBlockQ - 1, S - 1);
  const int klo = W > 0 ? max(0, q0 - W + 1) : 0;
  const int jt0 = klo / kBlockN;
  const int n_tiles = qlast / kBlockN - jt0 + 1;

  if (threadIdx.x == 0) {
    mbar_init(ctx.bar(BAR_Q_FULL), 1);
    mbar_init(ctx.bar(BAR_Q_READY), 4);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(ctx.bar(BAR_K_FULL + s), 1);
      mbar_init(ctx.bar(BAR_V_FULL + s), 1);
      mbar_init(ctx.bar(BAR_K_READY + s), 4);
      mbar_init(ctx.bar(BAR_KV_EMPTY + s), 1);
    }
    for (int m = 0; m < 2; ++m) {
      mbar_init(ctx.bar(BAR_S_FULL + m), 1);
      mbar_init(ctx.bar(BAR_P_FULL + m), 4);
      mbar_init(ctx.bar(BAR_O_FULL + m), 1);
    }
    mbar_init(ctx.bar(BAR_MMA_DONE), 1);
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

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && !skip) {
      prefetch_tensormap(&maps.q);
      prefetch_tensormap(&maps.k);
      prefetch_tensormap(&maps.v);
      prefetch_tensormap(&maps.o);
      mbar_arrive_expect_tx(ctx.bar(BAR_Q_FULL), 2 * kTileBytes);
      tma_load_4d(ctx.sbase + kOffQ, &maps.q, ctx.bar(BAR_Q_FULL), 0, g * kGroup, q0, b);
      tma_load_4d(ctx.sbase + kOffQ + kTileBytes, &maps.q, ctx.bar(BAR_Q_FULL), 0, g * kGroup,
                  q0 + kTokensPerM, b);
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int s = it % kStages;
        if (it >= kStages && !ctx.wait(BAR_KV_EMPTY + s, ((it / kStages) - 1) & 1)) break;
        const int kb = (jt0 + it) * kBlockN;
        mbar_arrive_expect_tx(ctx.bar(BAR_K_FULL + s), kTileBytes);
        tma_load_4d(ctx.sbase + kOffK + s * kTileBytes, &maps.k, ctx.bar(BAR_K_FULL + s), 0, g, kb,
                    b);
        mbar_arrive_expect_tx(ctx.bar(BAR_V_FULL + s), kTileBytes);
        tma_load_4d(ctx.sbase + kOffV + s * kTileBytes, &maps.v, ctx.bar(BAR_V_FULL + s), 0, g, kb,
                    b);
        issued = it + 1;
      }
      if (*ctx.abort_flag) {
        // Let every copy this CTA started land before its shared memory is released.
        volatile int never = 0;
        mbar_wait(ctx.bar(BAR_Q_FULL), 0, &never, nullptr, 0, kWaitTimeoutNs);
        for (int it = max(0, issued - kStages); it < issued; ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          mbar_wait(ctx.bar(BAR_K_FULL + s), ph, &never, nullptr, 0, kWaitTimeoutNs);
          mbar_wait(ctx.bar(BAR_V_FULL + s), ph, &never, nullptr, 0, kWaitTimeoutNs);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && !skip) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, kBlockN, false);
      constexpr uint32_t idesc_pv = idesc_bf16(128, kHeadDim, true);
      auto issue_qk = [&](int m, int s) {
        const uint32_t qa = ctx.sbase + kOffQ + m * kTileBytes;
        const uint32_t ka = ctx.sbase + kOffK + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          mma_bf16_ss(tmem + tmem_s(m), sdesc_sw128(qa + 32 * kk), sdesc_sw128(ka + 32 * kk),
                      idesc_qk, kk > 0 ? 1u : 0u);
      };
      auto issue_pv = [&](int m, int s, bool accumulate) {
        const uint32_t va = ctx.sbase + kOffV + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          mma_bf16_ts(tmem + tmem_o(m), tmem + tmem_s(m) + 8 * kk, sdesc_sw128(va + 2048 * kk),
                      idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
      };
      bool ok = ctx.wait(BAR_Q_READY, 0);
      tc_fence_after_sync();
      for (int it = 0; ok && it < n_tiles; ++it) {
        const int s = it % kStages;
        if (!(ok = ctx.wait(BAR_K_READY + s, (it / kStages) & 1))) break;
        tc_fence_after_sync();
        const int sp = (it + kStages - 1) % kStages;
        if (it > 0) {
          if (!(ok = ctx.wait(BAR_V_FULL + sp, ((it - 1) / kStages) & 1) &&
                     ctx.wait(BAR_P_FULL + 0, (it - 1) & 1)))
            break;
          tc_fence_after_sync();
          issue_pv(0, sp, it > 1);
        }
        issue_qk(0, s);
        mma_commit(ctx.bar(BAR_S_FULL + 0));
        if (it > 0) {
          if (!(ok = ctx.wait(BAR_P_FULL + 1, (it - 1) & 1))) break;
          tc_fence_after_sync();
          issue_pv(1, sp, it > 1);
          mma_commit(ctx.bar(BAR_KV_EMPTY + sp));
        }
        issue_qk(1, s);
        mma_commit(ctx.bar(BAR_S_FULL + 1));
      }
      if (ok) {
        const int last = n_tiles - 1;
        const int sp = last % kStages;
        if (ctx.wait(BAR_V_FULL + sp, (last / kStages) & 1) && ctx.wait(BAR_P_FULL + 0, last & 1)) {
          tc_fence_after_sync();
          issue_pv(0, sp, last > 0);
          mma_commit(ctx.bar(BAR_O_FULL + 0));
          if (ctx.wait(BAR_P_FULL + 1, last & 1)) {
            tc_fence_after_sync();
            issue_pv(1, sp, last > 0);
            mma_commit(ctx.bar(BAR_KV_EMPTY + sp));
            mma_commit(ctx.bar(BAR_O_FULL + 1));
          }
        }
      }
      // Every MMA issued must finish before the tensor memory is released.
      mma_commit(ctx.bar(BAR_MMA_DONE));
      volatile int never = 0;
      mbar_wait(ctx.bar(BAR_MMA_DONE), 0, &never, nullptr, 0, kWaitTimeoutNs);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------------------------------------------------------------- softmax
    const int m = (warp - 4) >> 2;  // M tile
    const int wq = warp & 3;        // TMEM lane quarter of this warp
    const int r = wq * 32 + lane;   // row of the M tile = TMEM lane
    const int tq = q0 + m * kTokensPerM + (r >> 3);
    const int h = g * kGroup + (r & 7);
    const int tmin = q0 + m * kTokensPerM + wq * 4;  // tokens of this warp: tmin .. tmin+3
    const int tmax = tmin + 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + tmem_s(m);
    const uint32_t tO = tmem + lane_off + tmem_o(m);
    const float sink = __ldg(args.sinks + h);
    const bool sink_off = isinf(sink) && sink < 0.f;
    float m_ref = sink_off ? -INFINITY : sink * kLog2e;
    float l = sink_off ? 0.f : 1.f;
    bool ok = !skip;
    for (int it = 0; ok && it < n_tiles; ++it) {
      if (!(ok = ctx.wait(BAR_S_FULL + m, it & 1))) break;
      tc_fence_after_sync();
      const int kb = (jt0 + it) * kBlockN;
      const bool wmask = (kb + kBlockN - 1 > tmin) || (W > 0 && kb <= tmax - W);
      // pass 1: row maximum of the visible scores
      float mx = -INFINITY;
#pragma unroll
      for (int ch = 0; ch < kBlockN / 32; ++ch) {
        uint32_t sv[32];
        tmem_ld32(tS + ch * 32, sv);
        if (wmask) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int kj = kb + ch * 32 + i;
            const bool vis = kj <= tq && (W <= 0 || kj > tq - W);
            mx = fmaxf(mx, vis ? __uint_as_float(sv[i]) : -INFINITY);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(sv[i]));
        }
      }
      mx *= kScaleLog2;
      const float m_new = fmaxf(m_ref, mx);
      float alpha = 1.f;
      bool rescale = false;
      if (it == 0) {
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
      // pass 2: probabilities, row sum, bf16 P into the S columns
      const float mr = m_ref == -INFINITY ? 0.f : m_ref;
      float rs = 0.f;
#pragma unroll
      for (int ch = 0; ch < kBlockN / 32; ++ch) {
        uint32_t sv[32];
        tmem_ld32(tS + ch * 32, sv);
        uint32_t pw[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0 = fmaf(__uint_as_float(sv[2 * i]), kScaleLog2, -mr);
          float x1 = fmaf(__uint_as_float(sv[2 * i + 1]), kScaleLog2, -mr);
          if (wmask) {
            const int kj = kb + ch * 32 + 2 * i;
            if (!(kj <= tq && (W <= 0 || kj > tq - W))) x0 = -INFINITY;
            if (!(kj + 1 <= tq && (W <= 0 || kj + 1 > tq - W))) x1 = -INFINITY;
          }
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          rs += p0 + p1;
          pw[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + ch * 16, pw);
      }
      l += rs;
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_P_FULL + m));
    }
    // epilogue: O / l -> bf16 -> (swizzled) staging in the Q tile -> TMA store
    uint8_t* stage = smem + kOffQ + m * kTileBytes;
    if (ok && ctx.wait(BAR_O_FULL + m, 0)) {
      tc_fence_after_sync();
      const float inv_l = 1.f / l;
#pragma unroll
      for (int ch = 0; ch < kHeadDim / 32; ++ch) {
        uint32_t ov[32];
        tmem_ld32(tO + ch * 32, ov);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(ov[8 * cc + 2 * e]) * inv_l,
                               __uint_as_float(ov[8 * cc + 2 * e + 1]) * inv_l);
          const int chunk = ch * 4 + cc;
          *reinterpret_cast<uint4*>(stage + r * 128 + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      fence_async_smem();
    }
    named_barrier(1 + m, 128);
    if (r == 0 && !skip && !*ctx.abort_flag && q0 + m * kTokensPerM < S) {
      tma_store_4d(&maps.o, ctx.sbase + kOffQ + m * kTileBytes, 0, g * kGroup,
                   q0 + m * kTokensPerM, b);
      tma_store_commit();
      tma_store_wait_all();
    }
  } else if (warp >= 12) {
    // ---------------------------------------------------------------- RoPE
    const int t = static_cast<int>(threadIdx.x) - 384;  // 0..127
    bool ok = !skip && ctx.wait(BAR_Q_FULL, 0);
    if (ok) {
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        const int tok = q0 + m * kTokensPerM + (t >> 3);
        if (tok < S)
          rope_row(smem + kOffQ + m * kTileBytes + t * 128, t,
                   args.rope + static_cast<size_t>(load_position(args, b, tok)) * kRopePairs);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_Q_READY));
    }
    for (int it = 0; ok && it < n_tiles; ++it) {
      const int s = it % kStages;
      if (!(ok = ctx.wait(BAR_K_FULL + s, (it / kStages) & 1))) break;
      const int key = (jt0 + it) * kBlockN + t;
      if (key < S)
        rope_row(smem + kOffK + s * kTileBytes + t * 128, t,
                 args.rope + static_cast<size_t>(load_position(args, b, key)) * kRopePairs);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_K_READY + s));
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

cudaError_t launch_prefill(const PrefillMaps& maps, const PrefillArgs& args, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(args.n_qtiles), kNumKvHeads,
                  static_cast<unsigned>(args.batch));
  prefill_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps, args);
  return cudaGetLastError();
}

}  // namespace gqa
