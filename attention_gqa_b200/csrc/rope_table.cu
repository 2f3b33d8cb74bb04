// Rotary-embedding table: for every position p < 131072 and pair k < 32 the
// (cos, sin) of p * theta^(-2k/64), theta = 150000 (half-split RoPE of the
// gpt-oss pages: inteligile techniques map row "Partial RoPE"; rope_theta in
// the llm-atlas field table). Angles reach 1.3e5 rad, so they are formed and
// reduced in fp64 and only the results are stored as fp32.
#include "internal.h"

namespace gqa {
namespace {

__global__ void rope_table_kernel(float2* __restrict__ table) {
  const int idx = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
  if (idx >= kMaxPosition * kRopePairs) return;
  const int p = idx / kRopePairs;
  const int k = idx % kRopePairs;
  const double inv_freq = pow(kRopeTheta, -2.0 * static_cast<double>(k) / kHeadDim);
  double s, c;
  sincos(static_cast<double>(p) * inv_freq, &s, &c);
  table[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

}  // namespace

cudaError_t launch_rope_table(float2* table, cudaStream_t stream) {
  const int n = kMaxPosition * kRopePairs;
  rope_table_kernel<<<(n + 255) / 256, 256, 0, stream>>>(table);
  return cudaGetLastError();
}

}  // namespace gqa
