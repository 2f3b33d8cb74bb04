// Allocation-free decode entry point.
//
// Some callers cannot allocate device memory when they run decode: serving
// engines that hand all device memory to their own pool up front and forbid
// later allocations, and latency-bound loops that cannot afford the implicit
// synchronization of an allocation. For them this entry point runs the same
// split-KV decode as gptoss_attn_decode(), but its scratch (the per-split
// partial results and an error word) lives in a fixed array that is part of
// the library's device image, so the call allocates nothing.
//
// The array is GPTOSS_ATTN_NOALLOC_SCRATCH_BYTES bytes on every GPU that loads
// the library, held until the process exits. Every call shares it, so calls
// whose kernels overlap in time on the GPU race and must be serialized (for
// instance by issuing them on one stream).
#include <cstdint>
#include <mutex>

#include "gptoss_attn.h"
#include "internal.h"
#include "tmap.h"

namespace {

using namespace gqa;

constexpr size_t kScratchBytes = GPTOSS_ATTN_NOALLOC_SCRATCH_BYTES;
constexpr size_t kErrBytes = 256;  // the error word, padded so the partials stay aligned

// [0, 256): error word (int); [256, kScratchBytes): decode partials. In host
// code this name is only a stand-in for the device object: its device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
unsigned char* g_scratch_addr[kMaxDevices];  // device address of g_scratch, per device

// Looks up the device address of the scratch array for `dev`, which must be
// the current device. Done once per device ordinal and cached for the life of
// the process (the address belongs to the device's primary context); no
// allocation.
int scratch_address(int dev, unsigned char** addr) {
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return GPTOSS_ATTN_ERR_LAUNCH;
    g_scratch_addr[dev] = static_cast<unsigned char*>(p);
  }
  *addr = g_scratch_addr[dev];
  return GPTOSS_ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int gptoss_attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                          const float* sinks, const int32_t* len, int window,
                                          void* out, int batch, int max_len, cudaStream_t stream) {
  if (!q || !kcache || !vcache || !sinks || !len || !out) return GPTOSS_ATTN_ERR_NULL_PTR;
  if (batch < 1 || max_len < 1 || batch > 65535) return GPTOSS_ATTN_ERR_BAD_SHAPE;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(sinks) & 3u) || (reinterpret_cast<uintptr_t>(len) & 3u))
    return GPTOSS_ATTN_ERR_BAD_ALIGN;
  int nsplit = 0, chunk = 0;
  decode_plan(batch, max_len, window, &nsplit, &chunk);
  if (decode_workspace_bytes(batch, nsplit) > kScratchBytes - kErrBytes)
    return GPTOSS_ATTN_ERR_SMALL_WORKSPACE;  // these sizes need more than the fixed scratch
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      major != 10)
    return GPTOSS_ATTN_ERR_NO_DEVICE;
  unsigned char* scratch = nullptr;
  int st = scratch_address(dev, &scratch);
  if (st != GPTOSS_ATTN_OK) return st;

  DecodeMaps maps;
  const uint64_t L = static_cast<uint64_t>(max_len), B = static_cast<uint64_t>(batch);
  const uint64_t dims[4] = {kHeadDim, kNumKvHeads, L, B};
  const uint64_t str[3] = {kHeadDim * 2, kNumKvHeads * kHeadDim * 2,
                           L * kNumKvHeads * kHeadDim * 2};
  const uint32_t box[4] = {kHeadDim, 1, 64, 1};
  if (!make_tmap_bf16_4d(&maps.k, kcache, dims, str, box) ||
      !make_tmap_bf16_4d(&maps.v, vcache, dims, str, box))
    return GPTOSS_ATTN_ERR_TENSOR_MAP;

  DecodeArgs a;
  a.q = static_cast<const uint16_t*>(q);
  a.kcache = static_cast<const uint16_t*>(kcache);
  a.vcache = static_cast<const uint16_t*>(vcache);
  a.sinks = sinks;
  a.len = len;
  a.rope = nullptr;  // plain RoPE, evaluated in the kernel
  a.out = static_cast<uint16_t*>(out);
  const size_t rows = static_cast<size_t>(batch) * kNumHeads * nsplit;
  a.part_o = reinterpret_cast<float*>(scratch + kErrBytes);
  a.part_ml = reinterpret_cast<float2*>(scratch + kErrBytes + rows * kHeadDim * 4);
  a.err = reinterpret_cast<int*>(scratch);
  a.batch = batch;
  a.max_len = max_len;
  a.window = window > 0 ? window : 0;
  a.nsplit = nsplit;
  a.chunk = chunk;
  // The error word must start at zero (a stale timeout bit would make the
  // kernels skip their work); the partials are fully written before being read.
  if (cudaMemsetAsync(scratch, 0, sizeof(int), stream) != cudaSuccess)
    return GPTOSS_ATTN_ERR_LAUNCH;
  return launch_decode(maps, a, stream) == cudaSuccess ? GPTOSS_ATTN_OK : GPTOSS_ATTN_ERR_LAUNCH;
}
