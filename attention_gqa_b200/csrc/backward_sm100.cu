// Backward pass of the prefill attention for sm_100a: gradients of
// L = sum(dO * out) with respect to q, k, v and the per-head sink logits
// (the forward of the gpt-oss pages: inteligile "gpt-oss-120b" techniques map
// rows "Grouped-query attention", "Partial RoPE", "Learnable attention sink",
// "Sliding-window attention").
//
// With rotated q' = R(pos) q, k' = R(pos) k, scores s = q'.k'/8, the row
// normaliser lse (sink included, from the forward) and p = exp(s - lse):
//   D_i      = dO_i . out_i
//   dS_ij    = p_ij (dO_i . v_j - D_i)
//   dv_j     = sum_i p_ij dO_i            (the 8 heads of a group summed)
//   dq'_i    = sum_j dS_ij k'_j / 8,  dk'_j = sum_i dS_ij q'_i / 8
//   dsigma_h = -sum_i exp(sigma_h - lse_i) D_i
//   dq = R(pos)^T dq',  dk = R(pos)^T dk'.
//
// Kernels, in stream order:
//   rope_rows_kernel (twice): q' and k' into the workspace (bf16, as the
//     forward rounds them for the tensor cores).
//   bwd_prep_kernel: D and lse in log2 units per row, laid out [b][g][t][8]
//     so a 16-token tile of one group is 128 consecutive floats; the sink
//     gradient (block sums, one atomic per head and block).
//   bwd_dq_kernel: one CTA per (b, g, 16 tokens) = an M=128 tile of 16 tokens
//     x 8 heads; over its 64-key tiles: S = Q'K'^T and dP = dO V^T (tcgen05,
//     fp32 in TMEM), dS by the elementwise warpgroup (bf16 back into S's
//     columns), dQ += dS K' (A from TMEM). dQ stays in TMEM until the item's
//     end, is rotated back and stored as bf16.
//   bwd_dkv_kernel: one CTA per (b, g, 128 keys, chunk of query steps) = M=128
//     keys; over its 8-token (64-row) query steps that see them: S^T = K'Q'^T,
//     dP^T = V dO^T, P^T and dS^T by the elementwise warpgroup, dV += P^T dO and
//     dK += dS^T Q' (A from TMEM, summing over the 8 heads of the group because
//     they are rows of the tile). A key tile's steps are split into chunks of
//     similar length, so the first key tiles of a causal sequence (which see
//     every query) do not set the kernel's length; each chunk adds its fp32
//     dK', dV to zeroed sums in the workspace (vector reductions). When every
//     tile fits one chunk (long sequences, sliding windows) the CTA writes
//     dk = R(pos)^T dK' and dv as bf16 itself.
//   bwd_dkv_finish_kernel (split tiles only): dk = R(pos)^T dK' and dv from the
//     sums, as bf16.
// In both kernels the elementwise warps release S and dP (S^T, dP^T) as soon
// as they have loaded them and write their bf16 results (dS; P^T and dS^T)
// into separate double-buffered columns, so the MMAs of the next step run
// while the elementwise work of this one finishes. A dQ CTA takes 256
// tensor-memory columns and ~100 KB of shared memory (two CTAs per SM); a
// dK/dV CTA takes all 512 columns (one CTA per SM).
// Roles (192 threads): warp 0 TMA producer, warp 1 MMA issuer and TMEM owner,
// warps 2-5 the elementwise warpgroup (thread = TMEM lane; warp w reads lanes
// 32 (w % 4) .. 32 (w % 4) + 31).
// Every pipeline wait is bounded like the forward kernels'.
#include <algorithm>
#include <cmath>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {
namespace {
namespace bwd {

constexpr int kThreads = 192;
constexpr int kTok = 16;      // query tokens per 128-row dQ tile
constexpr int kKeys = 128;    // keys per dK/dV tile
constexpr int kQKeys = 64;    // keys per step of the dQ kernel
constexpr int kKTok = 8;      // query tokens (64 rows) per step of the dK/dV kernel
constexpr int kStages = 3;
constexpr uint32_t kTile = 128 * 128;  // 128 rows of 64 bf16
constexpr uint32_t kHalf = 64 * 128;   // 64 rows of 64 bf16
constexpr uint32_t kTmemCols = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kScaleLog2 = 0.125f * kLog2e;
constexpr float kScale = 0.125f;
// TMEM columns: S (or S^T) [0,64), dP (dP^T) [64,128), dQ or dV [128,192), dK [192,256).
constexpr uint32_t kColS = 0, kColP = 64, kColA = 128, kColB = 192;
// dQ kernel: dS of alternate tiles in two 32-column buffers, so the next
// tile's S and dP may overwrite theirs as soon as the elementwise warps have
// loaded them; dQ accumulates at kColQ.
constexpr uint32_t kColDS = 128, kColQ = 192;
// dK/dV kernel (one CTA per SM, all 512 columns): S^T and dP^T at 0 and 64, then
// two buffers of (P^T, dS^T) as bf16 (32 columns each), dV at 256, dK at 320.
constexpr uint32_t kKTmemCols = 512;
constexpr uint32_t kColPD = 128, kColDV = 256, kColDK = 320;
// one CTA per SM: a shared-memory request above half of the SM's
constexpr uint32_t kDkvSmemBytes = 120 * 1024;

// dq kernel shared memory
constexpr uint32_t kQOffQ = 0, kQOffDO = kTile, kQOffK = 2 * kTile;
constexpr uint32_t kQOffV = kQOffK + kStages * kHalf;
constexpr uint32_t kQOffBar = kQOffV + kStages * kHalf;
// dkv kernel shared memory
constexpr uint32_t kKOffK = 0, kKOffV = kTile, kKOffQ = 2 * kTile;  // [stage]: Q', then dO
constexpr uint32_t kKOffLD = kKOffQ + kStages * 2 * kHalf;           // [stage]: lse2[64], D[64]
constexpr uint32_t kKOffBar = kKOffLD + kStages * 512;
// two CTAs per SM (each takes half of the tensor memory)
constexpr uint32_t kSmemBytes = 100 * 1024;
static_assert(kQOffBar + 256 + 1024 <= kSmemBytes && kKOffBar + 256 + 1024 <= kSmemBytes, "smem");

enum : int {
  BAR_Q_FULL = 0,                        // [2] the query-side tile(s) of a stage
  BAR_Q_EMPTY = BAR_Q_FULL + kStages,    // [2]
  BAR_KV_FULL = BAR_Q_EMPTY + kStages,   // [2]
  BAR_KV_EMPTY = BAR_KV_FULL + kStages,  // [2]
  BAR_S_FULL = BAR_KV_EMPTY + kStages,   // S and dP written
  BAR_E_DONE = BAR_S_FULL + 1,           // elementwise results in TMEM, S/dP read
  BAR_ACC_FULL = BAR_E_DONE + 1,         // the item's accumulators complete
  BAR_MMA_DONE = BAR_ACC_FULL + 1,
  BAR_SP_FREE = BAR_MMA_DONE + 1,        // S and dP (S^T and dP^T) loaded by the elementwise warps
  BAR_DS_FREE = BAR_SP_FREE + 1,         // [2] a bf16 result buffer read by its MMAs
  NUM_BARS = BAR_DS_FREE + 2
};
// the barriers, then the TMEM address slot and the abort flag (8 bytes)
static_assert(NUM_BARS * 8 + 8 <= 256, "barrier region");

struct Ctx {
  uint32_t sbase, obar;
  volatile int* abort_flag;
  int* err;
  __device__ uint32_t bar(int i) const { return sbase + obar + 8u * static_cast<uint32_t>(i); }
  __device__ bool wait(int i, uint32_t parity) const {
    return mbar_wait(bar(i), parity, abort_flag, err, kErrTimeout, kWaitTimeoutNs);
  }
  __device__ bool wait_warp(int i, uint32_t parity) const {
    return mbar_wait_warp(bar(i), parity, abort_flag, err, kErrTimeout, kWaitTimeoutNs);
  }
};

// Common prologue: barriers, abort flag (a timeout left in the error word
// skips the work), tensor memory. Returns the TMEM base address.
__device__ uint32_t setup(Ctx& ctx, uint8_t* smem, uint32_t obar, int* err,
                          uint32_t ncols = kTmemCols) {
  ctx.sbase = smem_u32(smem);
  ctx.obar = obar;
  ctx.abort_flag = reinterpret_cast<volatile int*>(smem + obar + NUM_BARS * 8 + 4);
  ctx.err = err;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + obar + NUM_BARS * 8);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(ctx.bar(BAR_Q_FULL + s), 1);
      mbar_init(ctx.bar(BAR_Q_EMPTY + s), 1);
      mbar_init(ctx.bar(BAR_KV_FULL + s), 1);
      mbar_init(ctx.bar(BAR_KV_EMPTY + s), 1);
    }
    mbar_init(ctx.bar(BAR_S_FULL), 1);
    mbar_init(ctx.bar(BAR_E_DONE), 4);
    mbar_init(ctx.bar(BAR_ACC_FULL), 1);
    mbar_init(ctx.bar(BAR_MMA_DONE), 1);
    mbar_init(ctx.bar(BAR_SP_FREE), 4);
    mbar_init(ctx.bar(BAR_DS_FREE), 1);
    mbar_init(ctx.bar(BAR_DS_FREE + 1), 1);
    *ctx.abort_flag = (*reinterpret_cast<volatile int*>(err) & kErrTimeout) ? 1 : 0;
    fence_barrier_init();
  }
  if ((threadIdx.x >> 5) == 1) {
    tmem_alloc(smem_u32(tmem_slot), ncols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  return *tmem_slot;
}

__device__ void teardown(uint32_t tmem, uint32_t ncols = kTmemCols) {
  tc_fence_before_sync();
  __syncthreads();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, ncols);
  }
}

// D = A B^T over head_dim 64 for a K-major 128-row tile A and a K-major
// 64-row tile B (4 MMAs, K = 16): D is 128 x 64.
__device__ __forceinline__ void mma_abt(uint32_t d_tmem, uint32_t a, uint32_t b) {
  constexpr uint32_t idesc = idesc_bf16(128, 64, false);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_bf16_ss(d_tmem, sdesc_sw128(a + 32 * kk), sdesc_sw128(b + 32 * kk), idesc,
                kk > 0 ? 1u : 0u);
}

// D (+)= A B with A bf16 [128 x 64] in TMEM and B a 64-row tile read
// MN-major (rows = the contraction, 64 bf16 per row = the N columns).
__device__ __forceinline__ void mma_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint32_t b,
                                           bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(128, kHeadDim, true);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_bf16_ts(d_tmem, a_tmem + 8 * kk, sdesc_sw128(b + 2048 * kk), idesc,
                (accumulate || kk > 0) ? 1u : 0u);
}

// Rotates a 64-element gradient row back (R(p)^T) with the table row `cs`
// (global memory) and stores it as bf16 at `dst` (128 bytes, 16-byte aligned).
__device__ __forceinline__ void unrotate_store(const uint32_t (&lo)[32], const uint32_t (&hi)[32],
                                               const float2* cs, uint16_t* dst) {
  uint32_t w[32];
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(cs + k));
    const float y1a = __uint_as_float(lo[k]), y2a = __uint_as_float(hi[k]);
    const float y1b = __uint_as_float(lo[k + 1]), y2b = __uint_as_float(hi[k + 1]);
    w[k / 2] = pack_bf16x2(fmaf(y1a, t.x, y2a * t.y), fmaf(y1b, t.z, y2b * t.w));
    w[16 + k / 2] = pack_bf16x2(fmaf(y2a, t.x, -y1a * t.y), fmaf(y2b, t.z, -y1b * t.w));
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

// Adds 4 floats to global memory at p (16-byte aligned) with one vector reduction.
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// Adds a thread's 64-float accumulator row (lo: columns 0-31, hi: 32-63) to `row`.
__device__ __forceinline__ void red_add_row(float* row, const uint32_t (&lo)[32],
                                            const uint32_t (&hi)[32]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    red_add4(row + 4 * i, __uint_as_float(lo[4 * i]), __uint_as_float(lo[4 * i + 1]),
             __uint_as_float(lo[4 * i + 2]), __uint_as_float(lo[4 * i + 3]));
#pragma unroll
  for (int i = 0; i < 8; ++i)
    red_add4(row + 32 + 4 * i, __uint_as_float(hi[4 * i]), __uint_as_float(hi[4 * i + 1]),
             __uint_as_float(hi[4 * i + 2]), __uint_as_float(hi[4 * i + 3]));
}

__device__ __forceinline__ int clamp_pos(int p, int* err) {
  if (p < 0 || p >= kMaxPosition) {
    atomicOr(err, kErrPosition);
    return p < 0 ? 0 : kMaxPosition - 1;
  }
  return p;
}

}  // namespace bwd

// D and lse2 per row, and the sink gradient. Thread (token lane, head): 256
// threads = 4 token lanes x 64 heads, grid-stride over tokens.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BackwardArgs a) {
  const int h = static_cast<int>(threadIdx.x & 63);
  const int lane_t = static_cast<int>(threadIdx.x >> 6);
  const int g = h / kGroup, hl = h % kGroup;
  const float sig = __ldg(a.sinks + h);
  const bool sink_on = !(isinf(sig) && sig < 0.f);
  const int64_t ntok = static_cast<int64_t>(a.batch) * a.seqlen;
  float acc = 0.f;
  for (int64_t bt = static_cast<int64_t>(blockIdx.x) * 4 + lane_t; bt < ntok;
       bt += static_cast<int64_t>(gridDim.x) * 4) {
    const int64_t row = bt * kNumHeads + h;
    const uint4* po = reinterpret_cast<const uint4*>(a.out + row * kHeadDim);
    const uint4* pd = reinterpret_cast<const uint4*>(a.dout + row * kHeadDim);
    float d = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 o = __ldg(po + i), g4 = __ldg(pd + i);
      const uint32_t ow[4] = {o.x, o.y, o.z, o.w}, gw[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        d = fmaf(bf16lo_to_f32(ow[e]), bf16lo_to_f32(gw[e]),
                 fmaf(bf16hi_to_f32(ow[e]), bf16hi_to_f32(gw[e]), d));
    }
    const float lse2 = __ldg(a.lse + row) * bwd::kLog2e;
    const int64_t b = bt / a.seqlen, t = bt % a.seqlen;
    const int64_t w = ((b * kNumKvHeads + g) * a.seqlen + t) * kGroup + hl;
    a.lse2[w] = lse2;
    a.dd[w] = d;
    if (sink_on) acc -= ex2_approx(sig * bwd::kLog2e - lse2) * d;
  }
  __shared__ float red[4][64];
  red[lane_t][h] = acc;
  __syncthreads();
  if (lane_t == 0) atomicAdd(a.dsinks + h, red[0][h] + red[1][h] + red[2][h] + red[3][h]);
}

// dQ for one (b, g, 16-token) tile per CTA.
__global__ void __launch_bounds__(bwd::kThreads, 2)
    bwd_dq_kernel(const __grid_constant__ BackwardMaps maps, const BackwardArgs a) {
  using namespace bwd;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // the dK/dV kernel does not read this kernel's results: let it start filling
  // the SMs this grid's last CTAs leave idle
  griddep_launch_dependents();
  Ctx ctx;
  const uint32_t tmem = setup(ctx, smem, kQOffBar, a.err);
  const bool skip = *ctx.abort_flag != 0;
  const int warp = static_cast<int>(threadIdx.x >> 5), lane = static_cast<int>(threadIdx.x & 31);
  const int S = a.seqlen, W = a.window;
  // longest first: query tiles from the end of the sequence
  const int per_tile = kNumKvHeads * a.batch;
  const int idx = static_cast<int>(blockIdx.x);
  const int qt = a.n_qt - 1 - idx / per_tile;
  const int g = (idx % per_tile) % kNumKvHeads, b = (idx % per_tile) / kNumKvHeads;
  const int q0 = qt * kTok;
  const int tlast = min(q0 + kTok - 1, S - 1);
  const int jt0 = W > 0 ? max(0, q0 - W + 1) / kQKeys : 0;
  const int n_tiles = tlast / kQKeys - jt0 + 1;

  if (warp == 0) {
    if (lane == 0 && !skip) {
      prefetch_tensormap(&maps.q16);
      prefetch_tensormap(&maps.dout16);
      prefetch_tensormap(&maps.k64);
      prefetch_tensormap(&maps.v64);
      mbar_arrive_expect_tx(ctx.bar(BAR_Q_FULL), 2 * kTile);
      tma_load_4d(ctx.sbase + kQOffQ, &maps.q16, ctx.bar(BAR_Q_FULL), 0, g * kGroup, q0, b);
      tma_load_4d(ctx.sbase + kQOffDO, &maps.dout16, ctx.bar(BAR_Q_FULL), 0, g * kGroup, q0, b);
      int j = 0;
      for (; j < n_tiles; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !ctx.wait(BAR_KV_EMPTY + s, ((j / kStages) - 1) & 1)) break;
        mbar_arrive_expect_tx(ctx.bar(BAR_KV_FULL + s), 2 * kHalf);
        tma_load_4d(ctx.sbase + kQOffK + s * kHalf, &maps.k64, ctx.bar(BAR_KV_FULL + s), 0, g,
                    (jt0 + j) * kQKeys, b);
        tma_load_4d(ctx.sbase + kQOffV + s * kHalf, &maps.v64, ctx.bar(BAR_KV_FULL + s), 0, g,
                    (jt0 + j) * kQKeys, b);
      }
      if (*ctx.abort_flag) {
        volatile int never = 0;
        mbar_wait(ctx.bar(BAR_Q_FULL), 0, &never, nullptr, 0, kWaitTimeoutNs);
        for (int i = max(0, j - kStages); i < j; ++i)
          mbar_wait(ctx.bar(BAR_KV_FULL + i % kStages), (i / kStages) & 1, &never, nullptr, 0,
                    kWaitTimeoutNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && !skip) {
      // S(j) and dP(j) go out as soon as the elementwise warps have loaded
      // S(j-1) and dP(j-1); dQ += dS(j-1) K(j-1) once dS(j-1) is written (into
      // its own columns), so the tensor core works on tile j while the
      // elementwise warps finish tile j-1.
      bool ok = ctx.wait(BAR_Q_FULL, 0);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j % kStages;
          if (!(ok = ctx.wait(BAR_KV_FULL + s, (j / kStages) & 1))) break;
          if (j > 0 && !(ok = ctx.wait(BAR_SP_FREE, (j - 1) & 1))) break;
          tc_fence_after_sync();
          mma_abt(tmem + kColS, ctx.sbase + kQOffQ, ctx.sbase + kQOffK + s * kHalf);
          mma_abt(tmem + kColP, ctx.sbase + kQOffDO, ctx.sbase + kQOffV + s * kHalf);
          mma_commit(ctx.bar(BAR_S_FULL));
        }
        if (j > 0) {
          const int jp = j - 1, sp = jp % kStages;
          if (!(ok = ctx.wait(BAR_E_DONE, jp & 1))) break;
          tc_fence_after_sync();
          mma_tmem_a(tmem + kColQ, tmem + kColDS + 32 * (jp & 1), ctx.sbase + kQOffK + sp * kHalf,
                     jp > 0);
          mma_commit(ctx.bar(BAR_KV_EMPTY + sp));
          mma_commit(ctx.bar(BAR_DS_FREE + (jp & 1)));
          if (jp == n_tiles - 1) mma_commit(ctx.bar(BAR_ACC_FULL));
        }
      }
      mma_commit(ctx.bar(BAR_MMA_DONE));
      volatile int never = 0;
      mbar_wait(ctx.bar(BAR_MMA_DONE), 0, &never, nullptr, 0, kWaitTimeoutNs);
    }
  } else {
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // row: token q0 + r/8, head g*8 + r%8
    const int t = q0 + (r >> 3);
    const bool row_ok = t < S;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    float lse2 = 0.f, dd = 0.f;
    if (row_ok) {
      const int64_t w = ((static_cast<int64_t>(b) * kNumKvHeads + g) * S + t) * kGroup + (r & 7);
      lse2 = a.lse2[w];
      dd = a.dd[w];
    }
    bool ok = !skip;
    for (int j = 0; ok && j < n_tiles; ++j) {
      if (!(ok = ctx.wait_warp(BAR_S_FULL, j & 1))) break;
      tc_fence_after_sync();
      const int kb = (jt0 + j) * kQKeys;
      const int c_hi = t - kb;                           // visible columns [c_lo, c_hi]
      const int c_lo = W > 0 ? t - W + 1 - kb : -1;
      uint32_t sv[64], pv[64], out[32];
      tmem_ld32(tmem + lane_off + kColS, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(tmem + lane_off + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_ld32(tmem + lane_off + kColP, *reinterpret_cast<uint32_t(*)[32]>(pv));
      tmem_ld32(tmem + lane_off + kColP + 32, *reinterpret_cast<uint32_t(*)[32]>(pv + 32));
      // S and dP are in registers: the next tile's may overwrite them
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_SP_FREE));
#pragma unroll
      for (int e = 0; e < 64; e += 2) {
        float ds[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int col = e + u;
          const bool vis = row_ok && col <= c_hi && col >= c_lo;
          const float p = vis ? ex2_approx(__uint_as_float(sv[e + u]) * kScaleLog2 - lse2) : 0.f;
          ds[u] = p * (__uint_as_float(pv[e + u]) - dd) * kScale;
        }
        out[e / 2] = pack_bf16x2(ds[0], ds[1]);
      }
      // this tile's dS buffer was last read by dQ of tile j-2
      if (j >= 2 && !(ok = ctx.wait_warp(BAR_DS_FREE + (j & 1), ((j >> 1) - 1) & 1))) break;
      tc_fence_after_sync();
      {
        uint32_t o16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) o16[i] = out[i];
        tmem_st16(tmem + lane_off + kColDS + 32 * (j & 1), o16);
#pragma unroll
        for (int i = 0; i < 16; ++i) o16[i] = out[16 + i];
        tmem_st16(tmem + lane_off + kColDS + 32 * (j & 1) + 16, o16);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_E_DONE));
    }
    if (ok && (ok = ctx.wait_warp(BAR_ACC_FULL, 0))) {
      tc_fence_after_sync();
      uint32_t lo[32], hi[32];
      tmem_ld32(tmem + lane_off + kColQ, lo);
      tmem_ld32(tmem + lane_off + kColQ + 32, hi);
      if (row_ok) {
        const int p = bwd::clamp_pos(__ldg(a.pos + static_cast<int64_t>(b) * S + t), a.err);
        unrotate_store(lo, hi, a.rope + static_cast<size_t>(p) * kRopePairs,
                       a.dq + ((static_cast<int64_t>(b) * S + t) * kNumHeads + g * kGroup +
                               (r & 7)) * kHeadDim);
      }
    }
  }
  teardown(tmem);
}

// Partial dK and dV for one (b, g, 128-key tile, chunk of query steps) per CTA.
__global__ void __launch_bounds__(bwd::kThreads, 1)
    bwd_dkv_kernel(const __grid_constant__ BackwardMaps maps, const BackwardArgs a) {
  using namespace bwd;
  const int S = a.seqlen, W = a.window;
  // chunk-major, then key tile, then (b, g): full chunks of all tiles first
  const int per_tile = kNumKvHeads * a.batch;
  const int n_kt = (S + kKeys - 1) / kKeys;
  const int idx = static_cast<int>(blockIdx.x);
  const int chunk = idx / (n_kt * per_tile);
  const int kt = (idx / per_tile) % n_kt;
  const int g = (idx % per_tile) % kNumKvHeads, b = (idx % per_tile) / kNumKvHeads;
  const int kb = kt * kKeys;
  // query tokens that see a key of this tile: [kb, t_max], in 8-token steps
  const int t_max = W > 0 ? min(S - 1, kb + kKeys - 1 + W - 1) : S - 1;
  const int j0 = chunk * a.kv_steps;
  const int qt0 = kb / kKTok + j0;  // this CTA's first step
  const int n_tiles = min(t_max / kKTok - kb / kKTok + 1 - j0, a.kv_steps);
  if (n_tiles <= 0) return;  // the tile has fewer chunks than the longest one
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Ctx ctx;
  const uint32_t tmem = setup(ctx, smem, kKOffBar, a.err, kKTmemCols);
  const bool skip = *ctx.abort_flag != 0;
  const int warp = static_cast<int>(threadIdx.x >> 5), lane = static_cast<int>(threadIdx.x & 31);
  const float* lse2_g = a.lse2 + (static_cast<int64_t>(b) * kNumKvHeads + g) * S * kGroup;
  const float* dd_g = a.dd + (static_cast<int64_t>(b) * kNumKvHeads + g) * S * kGroup;

  if (warp == 0) {
    if (lane == 0 && !skip) {
      prefetch_tensormap(&maps.q8);
      prefetch_tensormap(&maps.dout8);
      prefetch_tensormap(&maps.k128);
      prefetch_tensormap(&maps.v128);
      mbar_arrive_expect_tx(ctx.bar(BAR_KV_FULL), 2 * kTile);
      tma_load_4d(ctx.sbase + kKOffK, &maps.k128, ctx.bar(BAR_KV_FULL), 0, g, kb, b);
      tma_load_4d(ctx.sbase + kKOffV, &maps.v128, ctx.bar(BAR_KV_FULL), 0, g, kb, b);
      int j = 0;
      for (; j < n_tiles; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !ctx.wait(BAR_Q_EMPTY + s, ((j / kStages) - 1) & 1)) break;
        const int t0 = (qt0 + j) * kKTok;
        const uint32_t st = ctx.sbase + kKOffQ + s * 2 * kHalf;
        const uint32_t ld = ctx.sbase + kKOffLD + s * 512;
        // lse2 and D of the step's 64 rows: 256 contiguous bytes each (the
        // arrays are padded by one tile, rows past the sequence are masked)
        mbar_arrive_expect_tx(ctx.bar(BAR_Q_FULL + s), 2 * kHalf + 512);
        tma_load_4d(st, &maps.q8, ctx.bar(BAR_Q_FULL + s), 0, g * kGroup, t0, b);
        tma_load_4d(st + kHalf, &maps.dout8, ctx.bar(BAR_Q_FULL + s), 0, g * kGroup, t0, b);
        bulk_load(ld, lse2_g + static_cast<int64_t>(t0) * kGroup, 256, ctx.bar(BAR_Q_FULL + s));
        bulk_load(ld + 256, dd_g + static_cast<int64_t>(t0) * kGroup, 256,
                  ctx.bar(BAR_Q_FULL + s));
      }
      if (*ctx.abort_flag) {
        volatile int never = 0;
        mbar_wait(ctx.bar(BAR_KV_FULL), 0, &never, nullptr, 0, kWaitTimeoutNs);
        for (int i = max(0, j - kStages); i < j; ++i)
          mbar_wait(ctx.bar(BAR_Q_FULL + i % kStages), (i / kStages) & 1, &never, nullptr, 0,
                    kWaitTimeoutNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && !skip) {
      // S^T(j), dP^T(j) go out as soon as the elementwise warps have loaded
      // step j-1's; dV, dK of step j-1 once its P^T and dS^T are written (into
      // buffer (j-1) & 1), so the tensor core works on step j meanwhile.
      bool ok = ctx.wait(BAR_KV_FULL, 0);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j < n_tiles) {
          const int s = j % kStages;
          if (!(ok = ctx.wait(BAR_Q_FULL + s, (j / kStages) & 1))) break;
          if (j > 0 && !(ok = ctx.wait(BAR_SP_FREE, (j - 1) & 1))) break;
          tc_fence_after_sync();
          const uint32_t st = ctx.sbase + kKOffQ + s * 2 * kHalf;
          mma_abt(tmem + kColS, ctx.sbase + kKOffK, st);          // S^T = K' Q'^T
          mma_abt(tmem + kColP, ctx.sbase + kKOffV, st + kHalf);  // dP^T = V dO^T
          mma_commit(ctx.bar(BAR_S_FULL));
        }
        if (j > 0) {
          const int jp = j - 1, sp = jp % kStages;
          if (!(ok = ctx.wait(BAR_E_DONE, jp & 1))) break;
          tc_fence_after_sync();
          const uint32_t st = ctx.sbase + kKOffQ + sp * 2 * kHalf;
          const uint32_t pd = tmem + kColPD + 64 * (jp & 1);
          mma_tmem_a(tmem + kColDV, pd, st + kHalf, jp > 0);  // dV += P^T dO
          mma_tmem_a(tmem + kColDK, pd + 32, st, jp > 0);     // dK += dS^T Q'
          mma_commit(ctx.bar(BAR_Q_EMPTY + sp));
          mma_commit(ctx.bar(BAR_DS_FREE + (jp & 1)));
          if (jp == n_tiles - 1) mma_commit(ctx.bar(BAR_ACC_FULL));
        }
      }
      mma_commit(ctx.bar(BAR_MMA_DONE));
      volatile int never = 0;
      mbar_wait(ctx.bar(BAR_MMA_DONE), 0, &never, nullptr, 0, kWaitTimeoutNs);
    }
  } else {
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // key kb + r
    const int kj = kb + r;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    bool ok = !skip;
    for (int j = 0; ok && j < n_tiles; ++j) {
      const int s = j % kStages;
      if (!(ok = ctx.wait_warp(BAR_S_FULL, j & 1))) break;
      tc_fence_after_sync();
      const int t0 = (qt0 + j) * kKTok;
      const float* ld = reinterpret_cast<const float*>(smem + kKOffLD + s * 512);
      // column col is token t0 + col/8: visible iff kj <= t < S and t < kj + W
      const int lo_t = kj - t0;                              // first visible token offset
      const int hi_t = min(S - 1 - t0, W > 0 ? kj + W - 1 - t0 : 1 << 30);
      uint32_t sv[64], pv[64], pw[32], dw[32];
      tmem_ld32(tmem + lane_off + kColS, *reinterpret_cast<uint32_t(*)[32]>(sv));
      tmem_ld32(tmem + lane_off + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
      tmem_ld32(tmem + lane_off + kColP, *reinterpret_cast<uint32_t(*)[32]>(pv));
      tmem_ld32(tmem + lane_off + kColP + 32, *reinterpret_cast<uint32_t(*)[32]>(pv + 32));
      // S^T and dP^T are in registers: the next step's may overwrite them
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_SP_FREE));
#pragma unroll
      for (int e = 0; e < 64; e += 2) {
        float p[2], ds[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int col = e + u;
          const int tt = col >> 3;
          const bool vis = tt >= lo_t && tt <= hi_t;
          p[u] = vis ? ex2_approx(__uint_as_float(sv[e + u]) * kScaleLog2 - ld[col]) : 0.f;
          // rows past the sequence carry no lse or D: keep them out of dK
          ds[u] = vis ? p[u] * (__uint_as_float(pv[e + u]) - ld[64 + col]) * kScale : 0.f;
        }
        pw[e / 2] = pack_bf16x2(p[0], p[1]);
        dw[e / 2] = pack_bf16x2(ds[0], ds[1]);
      }
      // this step's P^T/dS^T buffer was last read by dV, dK of step j-2
      if (j >= 2 && !(ok = ctx.wait_warp(BAR_DS_FREE + (j & 1), ((j >> 1) - 1) & 1))) break;
      tc_fence_after_sync();
      {
        const uint32_t pd = tmem + lane_off + kColPD + 64 * (j & 1);
        uint32_t t16[16];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int i = 0; i < 16; ++i) t16[i] = pw[16 * h + i];
          tmem_st16(pd + 16 * h, t16);
#pragma unroll
          for (int i = 0; i < 16; ++i) t16[i] = dw[16 * h + i];
          tmem_st16(pd + 32 + 16 * h, t16);
        }
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(ctx.bar(BAR_E_DONE));
    }
    if (ok && (ok = ctx.wait_warp(BAR_ACC_FULL, 0))) {
      tc_fence_after_sync();
      uint32_t lo[32], hi[32];
      const int64_t row = ((static_cast<int64_t>(b) * S + kj) * kNumKvHeads + g) * kHeadDim;
      tmem_ld32(tmem + lane_off + kColDV, lo);
      tmem_ld32(tmem + lane_off + kColDV + 32, hi);
      if (kj < S) {
        if (a.kv_chunks > 1) {
          red_add_row(a.dv32 + row, lo, hi);
        } else {
          // the only chunk of the tile: dv straight to bf16
          uint4* dv4 = reinterpret_cast<uint4*>(a.dv + row);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dv4[i] = make_uint4(
                pack_bf16x2(__uint_as_float(lo[8 * i]), __uint_as_float(lo[8 * i + 1])),
                pack_bf16x2(__uint_as_float(lo[8 * i + 2]), __uint_as_float(lo[8 * i + 3])),
                pack_bf16x2(__uint_as_float(lo[8 * i + 4]), __uint_as_float(lo[8 * i + 5])),
                pack_bf16x2(__uint_as_float(lo[8 * i + 6]), __uint_as_float(lo[8 * i + 7])));
            dv4[4 + i] = make_uint4(
                pack_bf16x2(__uint_as_float(hi[8 * i]), __uint_as_float(hi[8 * i + 1])),
                pack_bf16x2(__uint_as_float(hi[8 * i + 2]), __uint_as_float(hi[8 * i + 3])),
                pack_bf16x2(__uint_as_float(hi[8 * i + 4]), __uint_as_float(hi[8 * i + 5])),
                pack_bf16x2(__uint_as_float(hi[8 * i + 6]), __uint_as_float(hi[8 * i + 7])));
          }
        }
      }
      tmem_ld32(tmem + lane_off + kColDK, lo);
      tmem_ld32(tmem + lane_off + kColDK + 32, hi);
      if (kj < S) {
        if (a.kv_chunks > 1) {
          red_add_row(a.dk32 + row, lo, hi);
        } else {
          const int p = bwd::clamp_pos(__ldg(a.pos + static_cast<int64_t>(b) * S + kj), a.err);
          unrotate_store(lo, hi, a.rope + static_cast<size_t>(p) * kRopePairs, a.dk + row);
        }
      }
    }
  }
  teardown(tmem, kKTmemCols);
}

// dk = R(pos)^T dK' and dv from the fp32 sums, as bf16: one thread per
// (token, kv head) row, grid-stride. Skipped while the error word holds a
// timeout (the dK/dV CTAs then left the sums incomplete).
__global__ void __launch_bounds__(256) bwd_dkv_finish_kernel(const BackwardArgs a) {
  // like the other kernels, skip the work while a timeout is pending
  if (*reinterpret_cast<volatile int*>(a.err) & kErrTimeout) return;
  const int64_t n = static_cast<int64_t>(a.batch) * a.seqlen * kNumKvHeads;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; r < n;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4* k4 = reinterpret_cast<const float4*>(a.dk32 + r * kHeadDim);
    const float4* v4 = reinterpret_cast<const float4*>(a.dv32 + r * kHeadDim);
    uint32_t lo[32], hi[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 x = k4[i], y = k4[8 + i];
      lo[4 * i] = __float_as_uint(x.x);
      lo[4 * i + 1] = __float_as_uint(x.y);
      lo[4 * i + 2] = __float_as_uint(x.z);
      lo[4 * i + 3] = __float_as_uint(x.w);
      hi[4 * i] = __float_as_uint(y.x);
      hi[4 * i + 1] = __float_as_uint(y.y);
      hi[4 * i + 2] = __float_as_uint(y.z);
      hi[4 * i + 3] = __float_as_uint(y.w);
    }
    const int64_t bt = r / kNumKvHeads;  // b * S + t
    const int p = bwd::clamp_pos(__ldg(a.pos + bt), a.err);
    bwd::unrotate_store(lo, hi, a.rope + static_cast<size_t>(p) * kRopePairs, a.dk + r * kHeadDim);
    uint4* d4 = reinterpret_cast<uint4*>(a.dv + r * kHeadDim);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 x = v4[2 * i], y = v4[2 * i + 1];
      d4[i] = make_uint4(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w), pack_bf16x2(y.x, y.y),
                         pack_bf16x2(y.z, y.w));
    }
  }
}

}  // namespace

int backward_q_tiles(int seqlen) { return (seqlen + bwd::kTok - 1) / bwd::kTok; }
int backward_k_tiles(int seqlen) { return (seqlen + bwd::kKeys - 1) / bwd::kKeys; }

void backward_plan(BackwardArgs* a, int target_ctas) {
  const int S = a->seqlen, W = a->window, n_kt = backward_k_tiles(S);
  int64_t total = 0;
  int longest = 1;
  for (int kt = 0; kt < n_kt; ++kt) {
    const int kb = kt * bwd::kKeys;
    const int t_max = W > 0 ? std::min(S - 1, kb + bwd::kKeys - 1 + W - 1) : S - 1;
    const int n = t_max / bwd::kKTok - kb / bwd::kKTok + 1;
    total += n;
    longest = std::max(longest, n);
  }
  total *= static_cast<int64_t>(kNumKvHeads) * a->batch;
  // at least 32 steps per CTA (256 query tokens), so the partial sums stay a
  // small share of the traffic
  int64_t steps = (total + target_ctas - 1) / target_ctas;
  if (steps < 32) steps = 32;
  if (steps > longest) steps = longest;
  a->kv_steps = static_cast<int>(steps);
  a->kv_chunks = (longest + a->kv_steps - 1) / a->kv_steps;
}

cudaError_t launch_backward(const BackwardMaps& maps, const BackwardArgs& args, int num_sms,
                            cudaStream_t stream) {
  const int64_t ntok = static_cast<int64_t>(args.batch) * args.seqlen;
  int64_t prep_blocks = (ntok + 3) / 4;
  if (prep_blocks > 4 * num_sms) prep_blocks = 4 * num_sms;
  bwd_prep_kernel<<<static_cast<unsigned>(prep_blocks), 256, 0, stream>>>(args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bwd::kSmemBytes));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bwd::kDkvSmemBytes));
  if (e != cudaSuccess) return e;
  const unsigned n_dq = static_cast<unsigned>(args.n_qt * kNumKvHeads * args.batch);
  bwd_dq_kernel<<<n_dq, bwd::kThreads, bwd::kSmemBytes, stream>>>(maps, args);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned n_dkv = static_cast<unsigned>(backward_k_tiles(args.seqlen) * kNumKvHeads *
                                              args.batch * args.kv_chunks);
  // programmatic dependent launch: independent of the dQ kernel, it overlaps
  // that kernel's tail (both read only the preparation kernel's results, which
  // are complete before the dQ kernel starts)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_dkv);
  cfg.blockDim = dim3(bwd::kThreads);
  cfg.dynamicSmemBytes = bwd::kDkvSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, bwd_dkv_kernel, maps, args);
  if (e != cudaSuccess || args.kv_chunks == 1) return e;
  const int64_t rows = static_cast<int64_t>(args.batch) * args.seqlen * kNumKvHeads;
  int64_t fin_blocks = (rows + 255) / 256;
  if (fin_blocks > 8 * num_sms) fin_blocks = 8 * num_sms;
  bwd_dkv_finish_kernel<<<static_cast<unsigned>(fin_blocks), 256, 0, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace gqa
