// Rotary embedding (half-split RoPE of the gpt-oss pages: inteligile
// techniques map rows "Partial RoPE" and "Layers without positional encoding
// (NoPE)"; rope_theta = 150000 in the llm-atlas field table).
//
// rope_table_kernel: for every position p < 131072 and pair k < 32 the
//   (cos, sin) of p * theta^(-2k/64). Angles reach 1.3e5 rad, so they are
//   formed and reduced in fp64; only the results are stored as fp32.
//   The YaRN table (techniques map row "YaRN RoPE scaling": factor 32 over the
//   4096-token initial context of the llm-atlas field tables) blends each
//   pair's frequency between theta^(-2k/64) and theta^(-2k/64) / 32 by a ramp
//   linear in the pair index, from 0 at the pair whose wavelength fits 32 times
//   into 4096 tokens to 1 at the pair where it fits once (the transformers yarn
//   initialisation, beta_fast 32 and beta_slow 1, no truncation), and scales
//   cos and sin by the attention factor 0.1 ln 32 + 1, which therefore reaches
//   both the rotated queries and the rotated keys.
// rope_rows_kernel: rotates every key row once per layer into a workspace,
//   so the attention kernels, which read each key tile many times, never
//   rotate keys. HBM bound: 128 bytes read and written per row.
#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {
namespace {

constexpr double kYarnFactor = 32.0;
constexpr double kYarnContext = 4096.0;
constexpr double kYarnTurnsFast = 32.0;  // beta_fast: full turns over the context
constexpr double kYarnTurnsSlow = 1.0;   // beta_slow
constexpr double kTwoPi = 6.283185307179586476925286766559;

// Pair index (fractional) at which theta^(-2k/64) * context / (2 pi) = turns.
__device__ double yarn_pair(double turns) {
  return kHeadDim * log(kYarnContext / (turns * kTwoPi)) / (2.0 * log(kRopeTheta));
}

__global__ void rope_table_kernel(float2* __restrict__ table, int yarn) {
  const int idx = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
  if (idx >= kMaxPosition * kRopePairs) return;
  const int p = idx / kRopePairs;
  const int k = idx % kRopePairs;
  double inv_freq = pow(kRopeTheta, -2.0 * static_cast<double>(k) / kHeadDim);
  double scale = 1.0;
  if (yarn) {
    const double lo = fmax(yarn_pair(kYarnTurnsFast), 0.0);
    const double hi = fmin(yarn_pair(kYarnTurnsSlow), kHeadDim - 1.0);
    const double w = fmin(fmax((static_cast<double>(k) - lo) / (hi - lo), 0.0), 1.0);
    inv_freq = w * (inv_freq / kYarnFactor) + (1.0 - w) * inv_freq;
    scale = 0.1 * log(kYarnFactor) + 1.0;
  }
  double s, c;
  sincos(static_cast<double>(p) * inv_freq, &s, &c);
  table[idx] = make_float2(static_cast<float>(c * scale), static_cast<float>(s * scale));
}

// Four threads per 64-element row; thread c rotates the 16-byte chunks c and
// c+4 (elements 8c..8c+7 pair with 8c+32..8c+39). Rows are [token][head]
// with 2^heads_log2 heads per token, which share one position and table row.
// Source tokens are [batch][n]; token t of sequence b is written to token
// dst_start + t of a destination laid out [batch][dst_len] (a cache), which
// is the same layout when dst_len == n and dst_start == 0.
__global__ void __launch_bounds__(256) rope_rows_kernel(const uint4* __restrict__ k,
                                                        const int32_t* __restrict__ pos,
                                                        const float2* __restrict__ table,
                                                        uint4* __restrict__ k_rot,
                                                        int64_t n_rows, int heads_log2,
                                                        int64_t n, int64_t dst_len,
                                                        int64_t dst_start, int* err) {
  // The attention kernel that follows may launch now; it waits for this
  // kernel's writes before it reads them.
  griddep_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
       idx < n_rows * 4; idx += stride) {
    const int64_t row = idx >> 2;
    const int c = static_cast<int>(idx & 3);
    const int64_t tok = row >> heads_log2;
    const int64_t dst_tok = dst_len == n ? tok + dst_start : tok + (tok / n) * (dst_len - n) + dst_start;
    const int64_t dst_row = (dst_tok << heads_log2) | (row & ((int64_t{1} << heads_log2) - 1));
    int p = __ldg(pos + tok);
    if (p < 0 || p >= kMaxPosition) {
      atomicOr(err, kErrPosition);
      p = p < 0 ? 0 : kMaxPosition - 1;
    }
    const uint4 a = __ldg(k + row * 8 + c);
    const uint4 h = __ldg(k + row * 8 + c + 4);
    const float4* t4 = reinterpret_cast<const float4*>(table + static_cast<int64_t>(p) * kRopePairs +
                                                       8 * c);
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
    k_rot[dst_row * 8 + c] = make_uint4(ya[0], ya[1], ya[2], ya[3]);
    k_rot[dst_row * 8 + c + 4] = make_uint4(yh[0], yh[1], yh[2], yh[3]);
  }
}

// Diagnostic: one thread waits, with the library's bounded wait, on an
// mbarrier that nothing ever arrives at; when the limit runs out the wait
// raises the timeout bit of the error word and the kernel returns.
__global__ void wait_timeout_kernel(int* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(smem_u32(&bar), 0, &abort_flag, err, kErrTimeout, timeout_ns);
}

}  // namespace

cudaError_t launch_wait_timeout(int* err, uint64_t timeout_ns, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(err, timeout_ns);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* table, bool yarn, cudaStream_t stream) {
  const int n = kMaxPosition * kRopePairs;
  rope_table_kernel<<<(n + 255) / 256, 256, 0, stream>>>(table, yarn ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_rope_rows(const void* x, const int32_t* pos, const float2* table, void* x_rot,
                             int batch, int64_t n, int64_t dst_len, int64_t dst_start, int heads,
                             int grid_cap, int* err, cudaStream_t stream) {
  const int heads_log2 = heads == kNumHeads ? 6 : 3;
  const int64_t n_rows = static_cast<int64_t>(batch) * n * heads;
  const int64_t threads = n_rows * 4;
  int64_t blocks = (threads + 255) / 256;
  if (blocks > grid_cap) blocks = grid_cap;
  rope_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint4*>(x), pos, table, static_cast<uint4*>(x_rot), n_rows, heads_log2, n,
      dst_len, dst_start, err);
  return cudaGetLastError();
}

}  // namespace gqa
