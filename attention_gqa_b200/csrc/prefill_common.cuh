// Pieces shared by the two prefill kernels (full causal in prefill_sm100.cu,
// narrow band in prefill_band_sm100.cu): launch shape, softmax constants, the
// in-place RoPE of 128-byte-swizzled rows, and the staging of rotary-table rows.
#pragma once

#include <cstdint>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {
namespace {

constexpr int kThreads = 512;       // four warpgroups
constexpr uint32_t kTmemCols = 512;  // the whole tensor memory: one CTA per SM
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kScaleLog2 = 0.125f * kLog2e;  // 1/sqrt(64) * log2(e)

// Rotate one 64-element row stored at `row` (128 bytes, 128B-swizzled with
// row index r) by the (cos, sin) table row `cs` of its position, in place.
// Both live in shared memory: the producer stages the table rows an item
// needs (one per token) next to its Q tile.
// Rotates, in place, the 16-byte chunks c and c+4 (elements 8c..8c+7 and
// their partners 8c+32..8c+39) of a 64-element row stored at `row` (128 bytes,
// 128B-swizzled with row index r), with the (cos, sin) of pairs 8c..8c+7.
__device__ __forceinline__ void rope_chunk(uint8_t* row, int r, int c, const float (&cv)[8],
                                           const float (&sv)[8]) {
  uint4* plo = reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4));
  uint4* phi = reinterpret_cast<uint4*>(row + (((c + 4) ^ (r & 7)) << 4));
  const uint4 a = *plo, h = *phi;
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

// Rotates a whole row with the table row `cs` of its position (both in shared memory).
__device__ __forceinline__ void rope_row(uint8_t* row, int r, const float2* cs) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4* t4 = reinterpret_cast<const float4*>(cs + 8 * c);
    const float4 t0 = t4[0], t1 = t4[1], t2 = t4[2], t3 = t4[3];
    const float cv[8] = {t0.x, t0.z, t1.x, t1.z, t2.x, t2.z, t3.x, t3.z};
    const float sv[8] = {t0.y, t0.w, t1.y, t1.w, t2.y, t2.w, t3.y, t3.w};
    rope_chunk(row, r, c, cv, sv);
  }
}

// Stages the rotary-table rows of tokens q0 .. q0+n-1 of sequence b (one
// 256-byte row each, kRowStride bytes apart in shared memory; the 8 heads of
// a token share its position) at `dst`, completing on `bar`. Returns the
// bytes requested; tokens past the sequence end are skipped. Run by one thread.
template <int kTokensPerItem, uint32_t kRowStride>
__device__ __forceinline__ uint32_t stage_rope_rows(const PrefillArgs& a, int b, int q0,
                                                    uint32_t dst, uint32_t bar) {
  constexpr uint32_t kRowBytes = kRopePairs * sizeof(float2);
  constexpr int kGroupTok = 8;  // positions loaded together, then their copies issued
  uint32_t bytes = 0;
#pragma unroll 1
  for (int t0 = 0; t0 < kTokensPerItem && q0 + t0 < a.seqlen; t0 += kGroupTok) {
    int p[kGroupTok];
#pragma unroll
    for (int t = 0; t < kGroupTok; ++t)
      p[t] = q0 + t0 + t < a.seqlen
                 ? __ldg(a.pos + static_cast<size_t>(b) * a.seqlen + q0 + t0 + t) : 0;
#pragma unroll
    for (int t = 0; t < kGroupTok; ++t) {
      if (q0 + t0 + t >= a.seqlen) break;
      int pt = p[t];
      if (pt < 0 || pt >= kMaxPosition) {
        atomicOr(a.err, kErrPosition);
        pt = pt < 0 ? 0 : kMaxPosition - 1;
      }
      bulk_load(dst + (t0 + t) * kRowStride, a.rope + static_cast<size_t>(pt) * kRopePairs,
                kRowBytes, bar);
      bytes += kRowBytes;
    }
  }
  return bytes;
}

// Rotary positions of tokens q0 .. q0+N-1 of sequence b (0 past the sequence
// end). The loads are independent, so they cost one round trip to memory.
template <int N>
__device__ __forceinline__ void load_positions(const PrefillArgs& a, int b, int q0, int (&p)[N]) {
#pragma unroll
  for (int t = 0; t < N; ++t)
    p[t] = q0 + t < a.seqlen ? __ldg(a.pos + static_cast<size_t>(b) * a.seqlen + q0 + t) : 0;
}

// Stages the rotary-table rows of tokens q0 .. q0+N-1 whose positions are p
// (256 bytes each, consecutive in shared memory at `dst`), completing on
// `bar`; tokens past the sequence end are skipped. Consecutive positions (the
// usual p = token index) take one bulk copy, others one copy per row. Returns
// the bytes requested. Run by one thread.
template <int N>
__device__ __forceinline__ uint32_t stage_rope_rows_at(const PrefillArgs& a, const int (&p)[N],
                                                       int q0, uint32_t dst, uint32_t bar) {
  constexpr uint32_t kRowBytes = kRopePairs * sizeof(float2);
  const int n = min(N, a.seqlen - q0);
  bool run = p[0] >= 0 && p[0] + n <= kMaxPosition;
#pragma unroll
  for (int t = 1; t < N; ++t) run = run && (t >= n || p[t] == p[0] + t);
  if (run) {
    bulk_load(dst, a.rope + static_cast<size_t>(p[0]) * kRopePairs, kRowBytes * n, bar);
    return kRowBytes * n;
  }
#pragma unroll
  for (int t = 0; t < N; ++t) {
    if (t >= n) break;
    int pt = p[t];
    if (pt < 0 || pt >= kMaxPosition) {
      atomicOr(a.err, kErrPosition);
      pt = pt < 0 ? 0 : kMaxPosition - 1;
    }
    bulk_load(dst + t * kRowBytes, a.rope + static_cast<size_t>(pt) * kRopePairs, kRowBytes, bar);
  }
  return kRowBytes * n;
}

}  // namespace
}  // namespace gqa
