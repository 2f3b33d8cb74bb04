// Library-internal declarations shared by the host entry points and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace gqa {

constexpr int kNumHeads = 64;
constexpr int kNumKvHeads = 8;
constexpr int kGroup = kNumHeads / kNumKvHeads;  // query heads per key/value head
constexpr int kHeadDim = 64;
constexpr int kRopePairs = kHeadDim / 2;
constexpr int kMaxPosition = 131072;
constexpr double kRopeTheta = 150000.0;

// Device error word bits (set by kernels, read by gptoss_attn_check). After a
// timeout the kernels skip their work until the word is cleared.
constexpr int kErrTimeout = 1;
constexpr int kErrPosition = 2;
constexpr int kErrLength = 4;

// Pipeline waits give up after this long (a healthy wait lasts microseconds).
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

struct PrefillArgs {
  const int32_t* pos;   // [B][S]
  const float* sinks;   // [64]
  const float2* rope;   // [kMaxPosition][32] (cos, sin)
  int* err;             // device error word
  void* out;            // [B][S][64][64] bf16, the output (also reached through maps.o)
  float* lse;           // [B][S][64] natural-log softmax normaliser per row (sink
                        // included), written when not null; indexed like out
  int batch;
  int seqlen;           // query tokens per sequence (the rows of q, pos and out)
  int q_start;          // key index of query token 0: keys come from a cache
                        // whose rows [0, q_start) precede this call's tokens
  int window;           // <= 0: full causal
  int n_qtiles;         // ceil(seqlen / 32)
  int n_items;          // work items (prefill_items)
  int grid;             // persistent CTAs (the device's SM count)
  int order_chunk;      // 0: items by query tile (longest first), then group; C > 0:
                        // chunks of C query tiles (longest first), inside a chunk by
                        // (batch, group), so a wave reads few groups' keys and values
};

struct PrefillMaps {
  CUtensorMap q, k, v, o;   // q/o boxes (64, 8, 16, 1); k/v boxes (64, 1, 128, 1)
  CUtensorMap k_band, v_band;  // k/v boxes (64, 1, 16, 1): key blocks of the narrow-band kernel
};

// True when the narrow-band kernel (0 < window <= 128) serves the layer.
bool prefill_uses_band(int window);
// Query tokens per work item of the narrow-band kernel.
constexpr int kBandTokens = 16;
// Work items of one prefill launch.
int prefill_items(int batch, int seqlen, int window);
// Item order of the full-causal kernel for these sizes (PrefillArgs::order_chunk).
int prefill_order_chunk(int batch, int keys, int grid);

// Launches the prefill kernel; returns a cudaError_t.
cudaError_t launch_prefill(const PrefillMaps& maps, const PrefillArgs& args, cudaStream_t stream);
// Launches the narrow-band kernel on `grid` CTAs (called by launch_prefill).
cudaError_t launch_prefill_band(const PrefillMaps& maps, const PrefillArgs& args, int grid,
                                cudaStream_t stream);

// Diagnostic: a bounded wait on a barrier nothing arrives at (sets kErrTimeout).
cudaError_t launch_wait_timeout(int* err, uint64_t timeout_ns, cudaStream_t stream);

// Fills the rotary table [kMaxPosition][32] of (cos, sin); with `yarn` the
// YaRN frequencies and attention factor of the model.
cudaError_t launch_rope_table(float2* table, bool yarn, cudaStream_t stream);

// Rotates the rows of x [batch][n][heads][64] (bf16; heads = 8 for keys or 64
// for queries) by pos[batch][n] into x_rot laid out [batch][dst_len][heads][64],
// token t of each sequence going to token dst_start + t.
cudaError_t launch_rope_rows(const void* x, const int32_t* pos, const float2* table, void* x_rot,
                             int batch, int64_t n, int64_t dst_len, int64_t dst_start, int heads,
                             int grid_cap, int* err, cudaStream_t stream);

struct DecodeArgs {
  const uint16_t* q;       // [B][64][64] bf16, un-rotated
  const uint16_t* kcache;  // [B][L][8][64] bf16
  const uint16_t* vcache;  // [B][L][8][64] bf16
  const float* sinks;      // [64]
  const int32_t* len;      // [B]
  const float2* rope;      // rotary table rows for the query, or nullptr: plain RoPE
                           // evaluated in fp64 in the kernel
  uint16_t* out;           // [B][64][64] bf16
  float* part_o;           // [B][64][nsplit][64]
  float2* part_ml;         // [B][64][nsplit] (max in log2 units, sum)
  int* err;
  int batch;
  int max_len;
  int window;
  int nsplit;
  int chunk;               // keys per split
};

struct DecodeMaps {
  CUtensorMap k, v;
};

cudaError_t launch_decode(const DecodeMaps& maps, const DecodeArgs& args, cudaStream_t stream);

struct BackwardArgs {
  const int32_t* pos;      // [B][S]
  const float* sinks;      // [64]
  const float2* rope;      // rotary table
  int* err;
  const float* lse;        // [B][S][64] from the forward (natural log)
  const uint16_t* out;     // [B][S][64][64] bf16, the forward output
  const uint16_t* dout;    // [B][S][64][64] bf16
  float* lse2;             // workspace [B][8][S][8] (+ one tile of padding), log2 units
  float* dd;               // workspace [B][8][S][8] (+ padding): dO . out per row
  float* dsinks;           // [64], zeroed before the launch
  uint16_t* dq;            // [B][S][64][64] bf16
  uint16_t* dk;            // [B][S][8][64] bf16
  uint16_t* dv;            // [B][S][8][64] bf16
  float* dk32;             // workspace [B][S][8][64], zeroed: sums of dK' (rotated frame)
  float* dv32;             // workspace [B][S][8][64], zeroed: sums of dV
  int batch;
  int seqlen;
  int window;              // <= 0: full causal
  int n_qt;                // 16-token query tiles per sequence
  int kv_steps;            // 8-token query steps per dK/dV CTA (a key tile's steps are
                           // split over several CTAs whose partial sums are added)
  int kv_chunks;           // dK/dV CTAs per key tile (the most any tile needs)
};

struct BackwardMaps {
  CUtensorMap q16, dout16;  // rotated q and dO, boxes (64, 8, 16, 1): 128-row dQ tiles
  CUtensorMap q8, dout8;    // the same, boxes (64, 8, 8, 1): 64-row steps of dK/dV
  CUtensorMap k64, v64;     // rotated k and v, boxes (64, 1, 64, 1): steps of dQ
  CUtensorMap k128, v128;   // the same, boxes (64, 1, 128, 1): dK/dV tiles
};

int backward_q_tiles(int seqlen);
int backward_k_tiles(int seqlen);
// Splits the dK/dV work: sets args->kv_steps and args->kv_chunks so that about
// `target_ctas` CTAs of similar length cover every key tile's query steps.
void backward_plan(BackwardArgs* args, int target_ctas);
// Launches the preparation, dQ and dK/dV kernels (dsinks must be zeroed and
// the rotated q and k written to the workspace before).
cudaError_t launch_backward(const BackwardMaps& maps, const BackwardArgs& args, int num_sms,
                            cudaStream_t stream);

// Decode split planning shared by the workspace query and the launch.
void decode_plan(int batch, int max_len, int window, int* nsplit, int* chunk);
size_t decode_workspace_bytes(int batch, int nsplit);

}  // namespace gqa
