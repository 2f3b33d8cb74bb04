// Single-token decode attention for sm_100a over a bf16 key/value cache, with
// the gpt-oss learned sink joined once into the softmax denominator
// (inteligile techniques map, row "Learnable attention sink"; the cache is the
// use_cache path of the llm-atlas field table).
//
// Split-KV: CTA (split, g, b) streams its chunk of the visible keys of
// sequence b, key/value head g, through a TMA ring (64 keys of K and V per
// stage), and four consumer warps each take 16 keys of every stage. Scores
// and P.V run on mma.sync m16n8k16 with the 8 query heads of the group as
// rows (rows 8-15 are zero); the work is bound by HBM bandwidth, not by the
// tensor pipe. Each CTA writes an unnormalised partial (max in log2 units,
// sum, O[64]) per head; the combine kernel merges the splits with the sink
// term exp2(sigma*log2 e - M) counted once, and rounds to bf16.
#include <cmath>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace gqa {
namespace {

constexpr int kKeys = 64;  // keys per stage
constexpr int kStages = 4;
constexpr int kWarps = 4;  // consumer warps
constexpr int kThreads = (kWarps + 1) * 32;
constexpr uint32_t kStageBytes = kKeys * 128;  // one of K or V
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kScaleLog2 = 0.125f * kLog2e;
constexpr float kRescaleThreshold = 8.0f;

constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kOffK + kStages * kStageBytes;
constexpr uint32_t kOffQ = kOffV + kStages * kStageBytes;       // bf16 [8][64]
constexpr uint32_t kOffCS = kOffQ + kGroup * kHeadDim * 2;      // float2 [32]
constexpr uint32_t kOffMerge = kOffCS + kRopePairs * 8;         // per warp: [8][64] O + [8] m + [8] l
constexpr uint32_t kMergeWarpBytes = (kGroup * kHeadDim + 2 * kGroup) * 4;
constexpr uint32_t kOffBar = kOffMerge + kWarps * kMergeWarpBytes;
constexpr uint32_t kOffMisc = kOffBar + 2 * kStages * 8;
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16, rows 8-15 zero) * B(16x8) + C, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kThreads)
    decode_kernel(const __grid_constant__ DecodeMaps maps, const DecodeArgs a) {
  // The combine kernel may launch now; it waits for this grid before reading.
  griddep_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc);
  auto full_bar = [&](int s) { return sbase + kOffBar + 8u * s; };
  auto empty_bar = [&](int s) { return sbase + kOffBar + 8u * (kStages + s); };

  const int warp = static_cast<int>(threadIdx.x >> 5);
  const int lane = static_cast<int>(threadIdx.x & 31);
  const int split = static_cast<int>(blockIdx.x);
  const int g = static_cast<int>(blockIdx.y);
  const int b = static_cast<int>(blockIdx.z);

  int L = __ldg(a.len + b);
  if (L < 0 || L > a.max_len) {
    if (threadIdx.x == 0 && split == 0 && g == 0) atomicOr(a.err, kErrLength);
    L = L < 0 ? 0 : a.max_len;
  }
  const int lo = a.window > 0 ? max(0, L - a.window) : 0;
  const int k_begin = lo + split * a.chunk;
  const int k_end = min(L, k_begin + a.chunk);
  const int n_keys = max(0, k_end - k_begin);
  const int n_stages = (n_keys + kKeys - 1) / kKeys;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), kWarps);
    }
    *abort_flag = (*reinterpret_cast<volatile int*>(a.err) & kErrTimeout) ? 1 : 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool skip = *abort_flag != 0;

  if (warp == kWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && !skip) {
      prefetch_tensormap(&maps.k);
      prefetch_tensormap(&maps.v);
      int issued = 0;
      for (int i = 0; i < n_stages; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(empty_bar(s), ((i / kStages) - 1) & 1, abort_flag, a.err,
                                       kErrTimeout, kWaitTimeoutNs))
          break;
        mbar_arrive_expect_tx(full_bar(s), 2 * kStageBytes);
        tma_load_4d(sbase + kOffK + s * kStageBytes, &maps.k, full_bar(s), 0, g, k_begin + i * kKeys,
                    b);
        tma_load_4d(sbase + kOffV + s * kStageBytes, &maps.v, full_bar(s), 0, g, k_begin + i * kKeys,
                    b);
        issued = i + 1;
      }
      if (*abort_flag) {
        volatile int never = 0;
        for (int i = max(0, issued - kStages); i < issued; ++i)
          mbar_wait(full_bar(i % kStages), (i / kStages) & 1, &never, nullptr, 0, kWaitTimeoutNs);
      }
    }
    return;  // the producer takes no part in the merge below
  }

  // ------------------------------------------------------------------ consumers
  const int t = static_cast<int>(threadIdx.x);  // 0..127
  // rotation of the new query at position L-1 (fp64 angles)
  float2* cs = reinterpret_cast<float2*>(smem + kOffCS);
  if (t < kRopePairs) {
    if (a.rope) {
      // a table (YaRN) covers positions below kMaxPosition; the API limits
      // max_len to that, and len is clamped to max_len above
      const int p = min(L > 0 ? L - 1 : 0, kMaxPosition - 1);
      cs[t] = a.rope[static_cast<size_t>(p) * kRopePairs + t];
    } else {
      const double ang = static_cast<double>(L > 0 ? L - 1 : 0) *
                         pow(kRopeTheta, -2.0 * static_cast<double>(t) / kHeadDim);
      double sn, cn;
      sincos(ang, &sn, &cn);
      cs[t] = make_float2(static_cast<float>(cn), static_cast<float>(sn));
    }
  }
  named_barrier(1, kWarps * 32);
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + kOffQ);
  {
    const int hh = t >> 4;          // head within the group
    const int d0 = (t & 15) * 4;    // 4 elements per thread
    const uint16_t* qrow = a.q + (static_cast<size_t>(b) * kNumHeads + g * kGroup + hh) * kHeadDim;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int d = d0 + e;
      const int k = d & 31;
      const float x = __uint_as_float(static_cast<uint32_t>(qrow[d]) << 16);
      const float xp = __uint_as_float(static_cast<uint32_t>(qrow[d ^ 32]) << 16);
      const float2 c = cs[k];
      const float y = d < 32 ? fmaf(x, c.x, -xp * c.y) : fmaf(x, c.x, xp * c.y);
      qs[hh * kHeadDim + d] = static_cast<uint16_t>(pack_bf16x2(y, 0.f) & 0xFFFFu);
    }
  }
  named_barrier(1, kWarps * 32);
  const int gr = lane >> 2, tc = lane & 3;
  uint32_t qa[4][2];  // A fragments (rows = heads) for the 4 k-steps over d
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    qa[kk][0] = *reinterpret_cast<const uint32_t*>(qs + gr * kHeadDim + 16 * kk + 2 * tc);
    qa[kk][1] = *reinterpret_cast<const uint32_t*>(qs + gr * kHeadDim + 16 * kk + 8 + 2 * tc);
  }

  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run = -INFINITY, l_part = 0.f;
  bool ok = !skip;
  for (int i = 0; ok && i < n_stages; ++i) {
    const int s = i % kStages;
    if (!(ok = mbar_wait(full_bar(s), (i / kStages) & 1, abort_flag, a.err, kErrTimeout,
                         kWaitTimeoutNs)))
      break;
    const uint32_t sk = sbase + kOffK + s * kStageBytes;
    const uint32_t sv = sbase + kOffV + s * kStageBytes;
    // scores for keys 16*warp .. 16*warp+15 of this stage
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int j = lane >> 3, row = lane & 7;
      const int kl = 16 * warp + 8 * (j >> 1) + row;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int chunk = 2 * kk + (j & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sk + kl * 128 + ((chunk ^ (kl & 7)) << 4), b0, b1, b2, b3);
        mma_16816(sc[0], qa[kk][0], qa[kk][1], b0, b1);
        mma_16816(sc[1], qa[kk][0], qa[kk][1], b2, b3);
      }
    }
    const int key0 = k_begin + i * kKeys + 16 * warp;
    float x[2][2];
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kj = key0 + 8 * nt + 2 * tc + e;
        x[nt][e] = kj < k_end ? sc[nt][e] * kScaleLog2 : -INFINITY;
        mx = fmaxf(mx, x[nt][e]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    if (m_new > m_run + kRescaleThreshold || (m_run == -INFINITY && m_new > m_run)) {
      const float alpha = m_run == -INFINITY ? 0.f : ex2_approx(m_run - m_new);
      l_part *= alpha;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        o[nt][0] *= alpha;
        o[nt][1] *= alpha;
      }
      m_run = m_new;
    }
    const float mr = m_run == -INFINITY ? 0.f : m_run;
    const float p00 = ex2_approx(x[0][0] - mr), p01 = ex2_approx(x[0][1] - mr);
    const float p10 = ex2_approx(x[1][0] - mr), p11 = ex2_approx(x[1][1] - mr);
    l_part += (p00 + p01) + (p10 + p11);
    const uint32_t pa0 = pack_bf16x2(p00, p01), pa2 = pack_bf16x2(p10, p11);
    // Keys past the end of the sequence have p = 0, but their cache rows may
    // hold anything (never written), and 0 * NaN or 0 * Inf would poison O:
    // zero this warp's V rows of such keys before P.V reads them.
    const bool tail = key0 + 16 > k_end;
    if (tail) {
#pragma unroll
      for (int c = lane; c < 16 * 8; c += 32) {
        const int rr = c >> 3;
        if (key0 + rr >= k_end) {
          const uint32_t addr = sv + (16 * warp + rr) * 128 + (c & 7) * 16;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
        }
      }
      __syncwarp();
    }
    {
      const int j = lane >> 3, row = lane & 7;
      const int kl = 16 * warp + 8 * (j & 1) + row;
#pragma unroll
      for (int dn = 0; dn < 4; ++dn) {
        const int chunk = 2 * dn + (j >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(sv + kl * 128 + ((chunk ^ (kl & 7)) << 4), b0, b1, b2, b3);
        mma_16816(o[2 * dn], pa0, pa2, b0, b1);
        mma_16816(o[2 * dn + 1], pa0, pa2, b2, b3);
      }
    }
    // the zeroing above wrote the stage through the generic proxy; order it
    // before the next TMA write into this stage
    if (tail) fence_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
  }

  // merge the four warps, then write this split's partial for the 8 heads
  float l_row = l_part;
  l_row += __shfl_xor_sync(0xffffffffu, l_row, 1);
  l_row += __shfl_xor_sync(0xffffffffu, l_row, 2);
  float* mo = reinterpret_cast<float*>(smem + kOffMerge + warp * kMergeWarpBytes);
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    mo[gr * kHeadDim + 8 * nt + 2 * tc] = o[nt][0];
    mo[gr * kHeadDim + 8 * nt + 2 * tc + 1] = o[nt][1];
  }
  if (tc == 0) {
    mo[kGroup * kHeadDim + gr] = m_run;
    mo[kGroup * kHeadDim + kGroup + gr] = l_row;
  }
  named_barrier(1, kWarps * 32);
  if (!skip && !*abort_flag) {
    const int hh = t >> 4;
    const int d0 = (t & 15) * 4;
    float mw[kWarps], M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float* mw_base =
          reinterpret_cast<const float*>(smem + kOffMerge + w * kMergeWarpBytes);
      mw[w] = mw_base[kGroup * kHeadDim + hh];
      M = fmaxf(M, mw[w]);
    }
    float lsum = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float* mw_base =
          reinterpret_cast<const float*>(smem + kOffMerge + w * kMergeWarpBytes);
      const float f = mw[w] == -INFINITY ? 0.f : ex2_approx(mw[w] - M);
      lsum += f * mw_base[kGroup * kHeadDim + kGroup + hh];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] += f * mw_base[hh * kHeadDim + d0 + e];
    }
    const size_t head = static_cast<size_t>(b) * kNumHeads + g * kGroup + hh;
    if (a.nsplit == 1) {
      // one split covers the whole visible range: add the sink and normalise
      // here (the combine step below, with a single split)
      const float sink = __ldg(a.sinks + g * kGroup + hh);
      const bool sink_off = isinf(sink) && sink < 0.f;
      const float ms = sink_off ? -INFINITY : sink * kLog2e;
      const float Mf = fmaxf(ms, M);
      float den = 0.f, f = 0.f;
      if (Mf != -INFINITY) {
        den = sink_off ? 0.f : ex2_approx(ms - Mf);
        if (M != -INFINITY) {
          f = ex2_approx(M - Mf);
          den += f * lsum;
        }
      }
      const float scale = den > 0.f ? f / den : 0.f;
      *reinterpret_cast<uint2*>(a.out + head * kHeadDim + d0) =
          make_uint2(pack_bf16x2(acc[0] * scale, acc[1] * scale),
                     pack_bf16x2(acc[2] * scale, acc[3] * scale));
    } else {
      const size_t row = head * a.nsplit + split;
      *reinterpret_cast<float4*>(a.part_o + row * kHeadDim + d0) =
          make_float4(acc[0], acc[1], acc[2], acc[3]);
      if ((t & 15) == 0) a.part_ml[row] = make_float2(M, lsum);
    }
  }
}

// One warp per (b, h): merge the splits and the sink, normalise, round to bf16.
__global__ void __launch_bounds__(256) combine_kernel(const DecodeArgs a) {
  const int wid = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = static_cast<int>(threadIdx.x & 31);
  if (wid >= a.batch * kNumHeads) return;
  griddep_wait();  // partials of the split kernel launched just before
  const int h = wid % kNumHeads;
  if (*reinterpret_cast<volatile int*>(a.err) & kErrTimeout) return;
  const float sink = __ldg(a.sinks + h);
  const bool sink_off = isinf(sink) && sink < 0.f;
  const float ms = sink_off ? -INFINITY : sink * kLog2e;
  const float2* ml = a.part_ml + static_cast<size_t>(wid) * a.nsplit;
  float M = ms;
  for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, ml[s].x);
  float den = 0.f, o0 = 0.f, o1 = 0.f;
  if (M != -INFINITY) {
    den = sink_off ? 0.f : ex2_approx(ms - M);
    for (int s = 0; s < a.nsplit; ++s) {
      const float2 v = ml[s];
      if (v.x == -INFINITY) continue;
      const float f = ex2_approx(v.x - M);
      den += f * v.y;
      const float2 po = *reinterpret_cast<const float2*>(
          a.part_o + (static_cast<size_t>(wid) * a.nsplit + s) * kHeadDim + 2 * lane);
      o0 += f * po.x;
      o1 += f * po.y;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  reinterpret_cast<uint32_t*>(a.out + static_cast<size_t>(wid) * kHeadDim)[lane] =
      pack_bf16x2(o0 * inv, o1 * inv);
}

}  // namespace

void decode_plan(int batch, int max_len, int window, int* nsplit, int* chunk) {
  const int n_plan = window > 0 ? (window < max_len ? window : max_len) : max_len;
  // aim for about four waves of three CTAs per SM on a 148-SM part
  const int target_ctas = 148 * 3 * 4;
  int ns = target_ctas / (batch * kNumKvHeads);
  const int max_ns = (n_plan + kKeys - 1) / kKeys;
  if (ns > max_ns) ns = max_ns;
  // short visible ranges (sliding layers) take one split: each CTA then
  // finishes its heads itself and the combine launch is skipped
  if (n_plan <= 256) ns = 1;
  if (ns < 1) ns = 1;
  int ch = (n_plan + ns - 1) / ns;
  ch = (ch + kKeys - 1) / kKeys * kKeys;
  ns = (n_plan + ch - 1) / ch;
  if (ns < 1) ns = 1;
  *nsplit = ns;
  *chunk = ch;
}

size_t decode_workspace_bytes(int batch, int nsplit) {
  const size_t rows = static_cast<size_t>(batch) * kNumHeads * nsplit;
  return rows * kHeadDim * sizeof(float) + rows * sizeof(float2);
}

cudaError_t launch_decode(const DecodeMaps& maps, const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(a.nsplit), kNumKvHeads, static_cast<unsigned>(a.batch));
  decode_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.nsplit == 1) return cudaSuccess;  // the split kernel wrote the output
  // programmatic dependent launch: the combine grid's launch overlaps the
  // split kernel's tail; its threads wait for the partials (griddep_wait).
  const int warps = a.batch * kNumHeads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((warps * 32 + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, a);
}

}  // namespace gqa
