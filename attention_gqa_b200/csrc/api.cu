// C-ABI entry points of libgptoss_attn.so: argument validation, per-device
// state (rotary tables, per-stream error words), TMA tensor maps, kernel
// launches.
#include <cstdint>
#include <mutex>

#include "gptoss_attn.h"
#include "internal.h"
#include "tmap.h"

namespace {

using namespace gqa;

constexpr int kMaxDevices = 64;
// Error words per device: one per stream that has launched work, in order of
// first use; streams beyond the last word share it.
constexpr int kErrWords = 64;

struct DeviceState {
  int* err = nullptr;                       // kErrWords 4-byte error words
  cudaStream_t err_stream[kErrWords] = {};  // the stream each word belongs to
  int err_used = 0;
  float2* rope = nullptr;     // [kMaxPosition][32], plain RoPE
  float2* yarn = nullptr;     // [kMaxPosition][32], YaRN (built on first use)
  int num_sms = 0;
};

// Which rotary table a call rotates with.
enum class Rope { kNone, kPlain, kYarn };

std::mutex g_mutex;
DeviceState g_state[kMaxDevices];

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices)
    return GPTOSS_ATTN_ERR_NO_DEVICE;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
      major != 10)
    return GPTOSS_ATTN_ERR_NO_DEVICE;
  return GPTOSS_ATTN_OK;
}

// Builds one rotary table on the current device (legacy default stream, waited on).
int build_table(float2** dst, bool yarn) {
  float2* t = nullptr;
  if (cudaMalloc(&t, sizeof(float2) * kMaxPosition * kRopePairs) != cudaSuccess)
    return GPTOSS_ATTN_ERR_ALLOC;
  if (launch_rope_table(t, yarn, nullptr) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(t);
    return GPTOSS_ATTN_ERR_LAUNCH;
  }
  *dst = t;
  return GPTOSS_ATTN_OK;
}

// Allocates the error words (and, when asked, builds a rotary table) once
// per device. Runs on the legacy default stream and waits for completion.
int ensure_state(int dev, Rope need) {
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_state[dev];
  if (st.num_sms == 0 &&
      cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return GPTOSS_ATTN_ERR_NO_DEVICE;
  if (!st.err) {
    int* e = nullptr;
    if (cudaMalloc(&e, sizeof(int) * kErrWords) != cudaSuccess) return GPTOSS_ATTN_ERR_ALLOC;
    if (cudaMemset(e, 0, sizeof(int) * kErrWords) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess) {
      cudaFree(e);
      return GPTOSS_ATTN_ERR_LAUNCH;
    }
    st.err = e;
  }
  if (need == Rope::kPlain && !st.rope) return build_table(&st.rope, false);
  if (need == Rope::kYarn && !st.yarn) return build_table(&st.yarn, true);
  return GPTOSS_ATTN_OK;
}

// The error word of `stream` on device `dev` (its state already allocated):
// kernels launched on the stream report into it and skip their work while it
// holds a timeout; gptoss_attn_check(stream) reads and clears it.
int* err_word(int dev, cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_state[dev];
  for (int i = 0; i < st.err_used; ++i)
    if (st.err_stream[i] == stream) return st.err + i;
  if (st.err_used < kErrWords) {
    st.err_stream[st.err_used] = stream;
    return st.err + st.err_used++;
  }
  return st.err + (kErrWords - 1);
}

const float2* table_of(int dev, Rope r) {
  return r == Rope::kYarn ? g_state[dev].yarn : g_state[dev].rope;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int gptoss_attn_abi_version(void) { return GPTOSS_ATTN_ABI_VERSION; }

const char* gptoss_attn_status_string(int status) {
  switch (status) {
    case GPTOSS_ATTN_OK: return "ok";
    case GPTOSS_ATTN_ERR_NULL_PTR: return "a required pointer is NULL";
    case GPTOSS_ATTN_ERR_BAD_SHAPE: return "batch, seqlen or max_len out of range";
    case GPTOSS_ATTN_ERR_BAD_ALIGN: return "a tensor base pointer is not 16-byte aligned";
    case GPTOSS_ATTN_ERR_SMALL_WORKSPACE: return "workspace smaller than required";
    case GPTOSS_ATTN_ERR_NO_DEVICE: return "no current CUDA device, or it is not sm_100";
    case GPTOSS_ATTN_ERR_LAUNCH: return "a CUDA call or kernel launch failed";
    case GPTOSS_ATTN_ERR_TENSOR_MAP: return "the driver rejected a TMA tensor map";
    case GPTOSS_ATTN_ERR_ALLOC: return "library-owned device memory could not be allocated";
    case GPTOSS_ATTN_ERR_DEVICE_TIMEOUT: return "a kernel pipeline wait timed out";
    case GPTOSS_ATTN_ERR_BAD_POSITION: return "a rotary position was outside [0, 131072)";
    case GPTOSS_ATTN_ERR_BAD_LENGTH: return "a decode length was outside [0, max_len]";
    default: return "unknown status";
  }
}

int gptoss_attn_init(void) {
  int dev = 0;
  int st = current_device(&dev);
  if (st != GPTOSS_ATTN_OK) return st;
  return ensure_state(dev, Rope::kPlain);
}

int gptoss_attn_init_yarn(void) {
  int dev = 0;
  int st = current_device(&dev);
  if (st != GPTOSS_ATTN_OK) return st;
  return ensure_state(dev, Rope::kYarn);
}

static int rope_table_of(const void** table, Rope r) {
  if (!table) return GPTOSS_ATTN_ERR_NULL_PTR;
  int dev = 0;
  int st = current_device(&dev);
  if (st == GPTOSS_ATTN_OK) st = ensure_state(dev, r);
  if (st != GPTOSS_ATTN_OK) return st;
  *table = table_of(dev, r);
  return GPTOSS_ATTN_OK;
}

int gptoss_attn_rope_table(const void** table) { return rope_table_of(table, Rope::kPlain); }

int gptoss_attn_rope_table_yarn(const void** table) { return rope_table_of(table, Rope::kYarn); }

size_t gptoss_attn_prefill_workspace_bytes(int batch, int seqlen) {
  if (batch < 1 || seqlen < 1 || seqlen > kMaxPosition || batch > 65535) return 0;
  return static_cast<size_t>(batch) * seqlen * kNumKvHeads * kHeadDim * 2;
}

static int prefill_impl(const void* q, const void* k, const void* v, const float* sinks,
                        const int32_t* pos, int window, void* out, int batch, int seqlen,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream, Rope rope,
                        float* lse) {
  if (!q || !k || !v || !sinks || !pos || !out || !workspace) return GPTOSS_ATTN_ERR_NULL_PTR;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GPTOSS_ATTN_ERR_BAD_ALIGN;
  if (batch < 1 || seqlen < 1 || seqlen > kMaxPosition || batch > 65535)
    return GPTOSS_ATTN_ERR_BAD_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(sinks) & 3u) ||
      (reinterpret_cast<uintptr_t>(pos) & 3u))
    return GPTOSS_ATTN_ERR_BAD_ALIGN;
  if (workspace_bytes < gptoss_attn_prefill_workspace_bytes(batch, seqlen))
    return GPTOSS_ATTN_ERR_SMALL_WORKSPACE;
  int dev = 0;
  int st = current_device(&dev);
  if (st == GPTOSS_ATTN_OK) st = ensure_state(dev, rope);
  if (st != GPTOSS_ATTN_OK) return st;

  PrefillMaps maps;
  const uint64_t S = static_cast<uint64_t>(seqlen), B = static_cast<uint64_t>(batch);
  const uint64_t qdims[4] = {kHeadDim, kNumHeads, S, B};
  const uint64_t qstr[3] = {kHeadDim * 2, kNumHeads * kHeadDim * 2, S * kNumHeads * kHeadDim * 2};
  const uint32_t qbox[4] = {kHeadDim, kGroup, 16, 1};
  const uint64_t kdims[4] = {kHeadDim, kNumKvHeads, S, B};
  const uint64_t kstr[3] = {kHeadDim * 2, kNumKvHeads * kHeadDim * 2,
                            S * kNumKvHeads * kHeadDim * 2};
  const uint32_t kbox[4] = {kHeadDim, 1, 128, 1};
  const uint32_t kbox_band[4] = {kHeadDim, 1, 16, 1};  // 16-key blocks of the band kernel
  // the attention kernels read the rotated keys from the workspace
  if (!make_tmap_bf16_4d(&maps.q, q, qdims, qstr, qbox) ||
      !make_tmap_bf16_4d(&maps.o, out, qdims, qstr, qbox) ||
      !make_tmap_bf16_4d(&maps.k, workspace, kdims, kstr, kbox) ||
      !make_tmap_bf16_4d(&maps.v, v, kdims, kstr, kbox) ||
      !make_tmap_bf16_4d(&maps.k_band, workspace, kdims, kstr, kbox_band) ||
      !make_tmap_bf16_4d(&maps.v_band, v, kdims, kstr, kbox_band))
    return GPTOSS_ATTN_ERR_TENSOR_MAP;

  PrefillArgs args;
  args.pos = pos;
  args.sinks = sinks;
  args.rope = table_of(dev, rope);
  args.err = err_word(dev, stream);
  args.out = out;
  args.lse = lse;
  args.batch = batch;
  args.seqlen = seqlen;
  args.q_start = 0;
  // A window covering the whole sequence is full causal.
  args.window = (window > 0 && window < seqlen) ? window : 0;
  args.n_qtiles = (seqlen + 31) / 32;
  args.n_items = prefill_items(batch, seqlen, args.window);
  args.grid = g_state[dev].num_sms;
  args.order_chunk = prefill_order_chunk(batch, seqlen, args.grid);
  if (launch_rope_rows(k, pos, args.rope, workspace, batch, seqlen, seqlen, 0, kNumKvHeads,
                       args.grid * 8, args.err, stream) != cudaSuccess)
    return GPTOSS_ATTN_ERR_LAUNCH;
  return launch_prefill(maps, args, stream) == cudaSuccess ? GPTOSS_ATTN_OK
                                                           : GPTOSS_ATTN_ERR_LAUNCH;
}

static int prefill_chunk_impl(const void* q, const void* k, const void* v, const float* sinks,
                              const int32_t* pos, int window, void* out, void* kcache,
                              void* vcache, int batch, int start, int n, int max_len,
                              cudaStream_t stream, Rope rope) {
  if (!q || !k || !v || !sinks || !pos || !out || !kcache || !vcache)
    return GPTOSS_ATTN_ERR_NULL_PTR;
  if (batch < 1 || batch > 65535 || n < 1 || start < 0 || max_len > kMaxPosition ||
      static_cast<int64_t>(start) + n > max_len)
    return GPTOSS_ATTN_ERR_BAD_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(kcache) ||
      !aligned16(vcache) || (reinterpret_cast<uintptr_t>(sinks) & 3u) ||
      (reinterpret_cast<uintptr_t>(pos) & 3u))
    return GPTOSS_ATTN_ERR_BAD_ALIGN;
  int dev = 0;
  int st = current_device(&dev);
  if (st == GPTOSS_ATTN_OK) st = ensure_state(dev, rope);
  if (st != GPTOSS_ATTN_OK) return st;

  const int keys = start + n;  // keys visible to the chunk: the cached prefix and the chunk
  PrefillMaps maps;
  const uint64_t N = static_cast<uint64_t>(n), B = static_cast<uint64_t>(batch);
  const uint64_t L = static_cast<uint64_t>(max_len);
  const uint64_t qdims[4] = {kHeadDim, kNumHeads, N, B};
  const uint64_t qstr[3] = {kHeadDim * 2, kNumHeads * kHeadDim * 2, N * kNumHeads * kHeadDim * 2};
  const uint32_t qbox[4] = {kHeadDim, kGroup, 16, 1};
  // cache views end at the chunk's last key, so the tensor memory engine
  // zero-fills (never reads) cache rows past it
  const uint64_t cdims[4] = {kHeadDim, kNumKvHeads, static_cast<uint64_t>(keys), B};
  const uint64_t cstr[3] = {kHeadDim * 2, kNumKvHeads * kHeadDim * 2,
                            L * kNumKvHeads * kHeadDim * 2};
  const uint32_t kbox[4] = {kHeadDim, 1, 128, 1};
  const uint32_t kbox_band[4] = {kHeadDim, 1, 16, 1};  // 16-key blocks of the band kernel
  if (!make_tmap_bf16_4d(&maps.q, q, qdims, qstr, qbox) ||
      !make_tmap_bf16_4d(&maps.o, out, qdims, qstr, qbox) ||
      !make_tmap_bf16_4d(&maps.k, kcache, cdims, cstr, kbox) ||
      !make_tmap_bf16_4d(&maps.v, vcache, cdims, cstr, kbox) ||
      !make_tmap_bf16_4d(&maps.k_band, kcache, cdims, cstr, kbox_band) ||
      !make_tmap_bf16_4d(&maps.v_band, vcache, cdims, cstr, kbox_band))
    return GPTOSS_ATTN_ERR_TENSOR_MAP;

  PrefillArgs args;
  args.pos = pos;
  args.sinks = sinks;
  args.rope = table_of(dev, rope);
  args.err = err_word(dev, stream);
  args.out = out;
  args.lse = nullptr;
  args.batch = batch;
  args.seqlen = n;
  args.q_start = start;
  // A window covering every visible key is full causal.
  args.window = (window > 0 && window < keys) ? window : 0;
  args.n_qtiles = (n + 31) / 32;
  args.n_items = prefill_items(batch, n, args.window);
  args.grid = g_state[dev].num_sms;
  args.order_chunk = prefill_order_chunk(batch, keys, args.grid);
  // values into the cache, then the rotated keys, then the attention (which
  // may start during the key rotation and waits for it before reading keys)
  const size_t row = static_cast<size_t>(kNumKvHeads) * kHeadDim * 2;
  if (cudaMemcpy2DAsync(static_cast<uint8_t*>(vcache) + static_cast<size_t>(start) * row,
                        static_cast<size_t>(max_len) * row, v, static_cast<size_t>(n) * row,
                        static_cast<size_t>(n) * row, static_cast<size_t>(batch),
                        cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return GPTOSS_ATTN_ERR_LAUNCH;
  if (launch_rope_rows(k, pos, args.rope, kcache, batch, n, max_len, start, kNumKvHeads,
                       args.grid * 8, args.err, stream) != cudaSuccess)
    return GPTOSS_ATTN_ERR_LAUNCH;
  return launch_prefill(maps, args, stream) == cudaSuccess ? GPTOSS_ATTN_OK
                                                           : GPTOSS_ATTN_ERR_LAUNCH;
}

size_t gptoss_attn_decode_workspace_bytes(int batch, int max_len, int window) {
  if (batch < 1 || max_len < 1 || batch > 65535) return 0;
  int nsplit = 0, chunk = 0;
  decode_plan(batch, max_len, window, &nsplit, &chunk);
  return decode_workspace_bytes(batch, nsplit);
}

static int decode_impl(const void* q, const void* kcache, const void* vcache, const float* sinks,
                       const int32_t* len, int window, void* out, int batch, int max_len,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream, Rope rope) {
  if (!q || !kcache || !vcache || !sinks || !len || !out || !workspace)
    return GPTOSS_ATTN_ERR_NULL_PTR;
  if (batch < 1 || max_len < 1 || batch > 65535) return GPTOSS_ATTN_ERR_BAD_SHAPE;
  // the YaRN table covers positions below 131072
  if (rope == Rope::kYarn && max_len > kMaxPosition) return GPTOSS_ATTN_ERR_BAD_SHAPE;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(out) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(sinks) & 3u) ||
      (reinterpret_cast<uintptr_t>(len) & 3u))
    return GPTOSS_ATTN_ERR_BAD_ALIGN;
  int nsplit = 0, chunk = 0;
  decode_plan(batch, max_len, window, &nsplit, &chunk);
  const size_t need = decode_workspace_bytes(batch, nsplit);
  if (workspace_bytes < need) return GPTOSS_ATTN_ERR_SMALL_WORKSPACE;
  int dev = 0;
  int st = current_device(&dev);
  if (st == GPTOSS_ATTN_OK) st = ensure_state(dev, rope == Rope::kYarn ? Rope::kYarn : Rope::kNone);
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
  a.rope = rope == Rope::kYarn ? table_of(dev, rope) : nullptr;
  a.out = static_cast<uint16_t*>(out);
  const size_t rows = static_cast<size_t>(batch) * kNumHeads * nsplit;
  a.part_o = static_cast<float*>(workspace);
  a.part_ml = reinterpret_cast<float2*>(static_cast<char*>(workspace) + rows * kHeadDim * 4);
  a.err = err_word(dev, stream);
  a.batch = batch;
  a.max_len = max_len;
  a.window = window > 0 ? window : 0;
  a.nsplit = nsplit;
  a.chunk = chunk;
  return launch_decode(maps, a, stream) == cudaSuccess ? GPTOSS_ATTN_OK : GPTOSS_ATTN_ERR_LAUNCH;
}

int gptoss_attn_prefill(const void* q, const void* k, const void* v, const float* sinks,
                        const int32_t* pos, int window, void* out, int batch, int seqlen,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return prefill_impl(q, k, v, sinks, pos, window, out, batch, seqlen, workspace, workspace_bytes,
                      stream, Rope::kPlain, nullptr);
}

int gptoss_attn_prefill_lse(const void* q, const void* k, const void* v, const float* sinks,
                            const int32_t* pos, int window, void* out, float* lse, int batch,
                            int seqlen, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
  if (!lse) return GPTOSS_ATTN_ERR_NULL_PTR;
  return prefill_impl(q, k, v, sinks, pos, window, out, batch, seqlen, workspace, workspace_bytes,
                      stream, Rope::kPlain, lse);
}

int gptoss_attn_prefill_yarn(const void* q, const void* k, const void* v, const float* sinks,
                             const int32_t* pos, int window, void* out, int batch, int seqlen,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return prefill_impl(q, k, v, sinks, pos, window, out, batch, seqlen, workspace, workspace_bytes,
                      stream, Rope::kYarn, nullptr);
}

int gptoss_attn_prefill_chunk(const void* q, const void* k, const void* v, const float* sinks,
                              const int32_t* pos, int window, void* out, void* kcache,
                              void* vcache, int batch, int start, int n, int max_len,
                              cudaStream_t stream) {
  return prefill_chunk_impl(q, k, v, sinks, pos, window, out, kcache, vcache, batch, start, n,
                            max_len, stream, Rope::kPlain);
}

int gptoss_attn_prefill_chunk_yarn(const void* q, const void* k, const void* v,
                                   const float* sinks, const int32_t* pos, int window, void* out,
                                   void* kcache, void* vcache, int batch, int start, int n,
                                   int max_len, cudaStream_t stream) {
  return prefill_chunk_impl(q, k, v, sinks, pos, window, out, kcache, vcache, batch, start, n,
                            max_len, stream, Rope::kYarn);
}

int gptoss_attn_decode(const void* q, const void* kcache, const void* vcache, const float* sinks,
                       const int32_t* len, int window, void* out, int batch, int max_len,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return decode_impl(q, kcache, vcache, sinks, len, window, out, batch, max_len, workspace,
                     workspace_bytes, stream, Rope::kPlain);
}

int gptoss_attn_decode_yarn(const void* q, const void* kcache, const void* vcache,
                            const float* sinks, const int32_t* len, int window, void* out,
                            int batch, int max_len, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
  return decode_impl(q, kcache, vcache, sinks, len, window, out, batch, max_len, workspace,
                     workspace_bytes, stream, Rope::kYarn);
}

// Backward workspace: rotated q, rotated k, lse2 and D in [b][g][t][8] layout
// (each float array padded by one 128-row tile), then the fp32 sums of dK'
// and dV ([b][t][g][64] each).
static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
static void backward_layout(int batch, int seqlen, size_t off[7]) {
  const size_t BS = static_cast<size_t>(batch) * seqlen;
  off[0] = 0;
  off[1] = align256(BS * kNumHeads * kHeadDim * 2);
  off[2] = off[1] + align256(BS * kNumKvHeads * kHeadDim * 2);
  off[3] = off[2] + align256((BS * kNumHeads + 128) * 4);
  off[4] = off[3] + align256((BS * kNumHeads + 128) * 4);
  off[5] = off[4] + align256(BS * kNumKvHeads * kHeadDim * 4);
  off[6] = off[5] + align256(BS * kNumKvHeads * kHeadDim * 4);
}

size_t gptoss_attn_prefill_backward_workspace_bytes(int batch, int seqlen) {
  if (batch < 1 || seqlen < 1 || seqlen > kMaxPosition || batch > 65535) return 0;
  size_t off[7];
  backward_layout(batch, seqlen, off);
  return off[6];
}

int gptoss_attn_prefill_backward(const void* q, const void* k, const void* v, const float* sinks,
                                 const int32_t* pos, int window, const void* out, const float* lse,
                                 const void* dout, void* dq, void* dk, void* dv, float* dsinks,
                                 int batch, int seqlen, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
  if (!q || !k || !v || !sinks || !pos || !out || !lse || !dout || !dq || !dk || !dv ||
      !dsinks || !workspace)
    return GPTOSS_ATTN_ERR_NULL_PTR;
  if (batch < 1 || seqlen < 1 || seqlen > kMaxPosition || batch > 65535)
    return GPTOSS_ATTN_ERR_BAD_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(sinks) & 3u) || (reinterpret_cast<uintptr_t>(pos) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(dsinks) & 3u))
    return GPTOSS_ATTN_ERR_BAD_ALIGN;
  if (workspace_bytes < gptoss_attn_prefill_backward_workspace_bytes(batch, seqlen))
    return GPTOSS_ATTN_ERR_SMALL_WORKSPACE;
  int dev = 0;
  int st = current_device(&dev);
  if (st == GPTOSS_ATTN_OK) st = ensure_state(dev, Rope::kPlain);
  if (st != GPTOSS_ATTN_OK) return st;

  size_t off[7];
  backward_layout(batch, seqlen, off);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BackwardMaps maps;
  const uint64_t S = static_cast<uint64_t>(seqlen), B = static_cast<uint64_t>(batch);
  const uint64_t qdims[4] = {kHeadDim, kNumHeads, S, B};
  const uint64_t qstr[3] = {kHeadDim * 2, kNumHeads * kHeadDim * 2, S * kNumHeads * kHeadDim * 2};
  const uint32_t qbox[4] = {kHeadDim, kGroup, 16, 1};
  const uint64_t kdims[4] = {kHeadDim, kNumKvHeads, S, B};
  const uint64_t kstr[3] = {kHeadDim * 2, kNumKvHeads * kHeadDim * 2,
                            S * kNumKvHeads * kHeadDim * 2};
  const uint32_t kbox[4] = {kHeadDim, 1, 128, 1};
  const uint32_t qbox8[4] = {kHeadDim, kGroup, 8, 1};
  const uint32_t kbox64[4] = {kHeadDim, 1, 64, 1};
  if (!make_tmap_bf16_4d(&maps.q16, ws + off[0], qdims, qstr, qbox) ||
      !make_tmap_bf16_4d(&maps.dout16, dout, qdims, qstr, qbox) ||
      !make_tmap_bf16_4d(&maps.q8, ws + off[0], qdims, qstr, qbox8) ||
      !make_tmap_bf16_4d(&maps.dout8, dout, qdims, qstr, qbox8) ||
      !make_tmap_bf16_4d(&maps.k64, ws + off[1], kdims, kstr, kbox64) ||
      !make_tmap_bf16_4d(&maps.v64, v, kdims, kstr, kbox64) ||
      !make_tmap_bf16_4d(&maps.k128, ws + off[1], kdims, kstr, kbox) ||
      !make_tmap_bf16_4d(&maps.v128, v, kdims, kstr, kbox))
    return GPTOSS_ATTN_ERR_TENSOR_MAP;

  BackwardArgs a;
  a.pos = pos;
  a.sinks = sinks;
  a.rope = table_of(dev, Rope::kPlain);
  a.err = err_word(dev, stream);
  a.lse = lse;
  a.out = static_cast<const uint16_t*>(out);
  a.dout = static_cast<const uint16_t*>(dout);
  a.lse2 = reinterpret_cast<float*>(ws + off[2]);
  a.dd = reinterpret_cast<float*>(ws + off[3]);
  a.dsinks = dsinks;
  a.dq = static_cast<uint16_t*>(dq);
  a.dk = static_cast<uint16_t*>(dk);
  a.dv = static_cast<uint16_t*>(dv);
  a.dk32 = reinterpret_cast<float*>(ws + off[4]);
  a.dv32 = reinterpret_cast<float*>(ws + off[5]);
  a.batch = batch;
  a.seqlen = seqlen;
  a.window = (window > 0 && window < seqlen) ? window : 0;
  a.n_qt = backward_q_tiles(seqlen);
  const int sms = g_state[dev].num_sms;
  // dK/dV work in about four waves of two CTAs per SM
  backward_plan(&a, 8 * sms);
  // the per-row arrays' padding tile is read (and masked) by the last dK/dV steps
  const size_t rows = static_cast<size_t>(batch) * seqlen * kNumHeads;
  if (cudaMemsetAsync(dsinks, 0, kNumHeads * sizeof(float), stream) != cudaSuccess ||
      (a.kv_chunks > 1 &&
       cudaMemsetAsync(ws + off[4], 0, off[6] - off[4], stream) != cudaSuccess) ||
      cudaMemsetAsync(a.lse2 + rows, 0, 128 * sizeof(float), stream) != cudaSuccess ||
      cudaMemsetAsync(a.dd + rows, 0, 128 * sizeof(float), stream) != cudaSuccess ||
      launch_rope_rows(q, pos, a.rope, ws + off[0], batch, seqlen, seqlen, 0, kNumHeads, sms * 8,
                       a.err, stream) != cudaSuccess ||
      launch_rope_rows(k, pos, a.rope, ws + off[1], batch, seqlen, seqlen, 0, kNumKvHeads,
                       sms * 8, a.err, stream) != cudaSuccess)
    return GPTOSS_ATTN_ERR_LAUNCH;
  return launch_backward(maps, a, sms, stream) == cudaSuccess ? GPTOSS_ATTN_OK
                                                              : GPTOSS_ATTN_ERR_LAUNCH;
}

int gptoss_attn_debug_wait_timeout(unsigned timeout_us, cudaStream_t stream) {
  if (timeout_us == 0 || timeout_us > 2000000u) return GPTOSS_ATTN_ERR_BAD_SHAPE;
  int dev = 0;
  int st = current_device(&dev);
  if (st == GPTOSS_ATTN_OK) st = ensure_state(dev, Rope::kNone);
  if (st != GPTOSS_ATTN_OK) return st;
  return launch_wait_timeout(err_word(dev, stream), static_cast<uint64_t>(timeout_us) * 1000u,
                             stream) == cudaSuccess
             ? GPTOSS_ATTN_OK
             : GPTOSS_ATTN_ERR_LAUNCH;
}

int gptoss_attn_check(cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return GPTOSS_ATTN_ERR_NO_DEVICE;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GPTOSS_ATTN_ERR_LAUNCH;
  bool allocated = false;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    allocated = g_state[dev].err != nullptr;
  }
  if (!allocated) return GPTOSS_ATTN_OK;
  int* e = err_word(dev, stream);
  // Only this stream is waited on: the word is this stream's alone.
  int h = 0;
  if (cudaMemcpyAsync(&h, e, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemsetAsync(e, 0, sizeof(int), stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return GPTOSS_ATTN_ERR_LAUNCH;
  if (h & kErrTimeout) return GPTOSS_ATTN_ERR_DEVICE_TIMEOUT;
  if (h & kErrPosition) return GPTOSS_ATTN_ERR_BAD_POSITION;
  if (h & kErrLength) return GPTOSS_ATTN_ERR_BAD_LENGTH;
  return GPTOSS_ATTN_OK;
}

}  // extern "C"
