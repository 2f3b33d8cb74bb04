/*
 * gptoss_attn — gpt-oss-style causal grouped-query attention with learned
 * sinks, for NVIDIA B200 (sm_100a). C ABI of libgptoss_attn.so.
 *
 * The operation (gpt-oss pages):
 *   - 64 query heads share 8 key/value heads; query head h reads key/value
 *     head floor(h / 8) (inteligile "gpt-oss-120b" techniques map, row
 *     "Grouped-query attention"; llm-atlas gpt-oss-20b field table:
 *     num_attention_heads 64, num_key_value_heads 8, head_dim 64).
 *   - queries and keys are rotated by the half-split rotary embedding,
 *     theta = 150000, pair k = (element k, element k+32) turning by
 *     pos * theta^(-2k/64) (techniques map rows "Partial RoPE" and
 *     "Layers without positional encoding (NoPE)"; rope_theta in the
 *     llm-atlas field table).
 *   - scores are scaled by 1/sqrt(64); a per-head learned sink logit
 *     sigma_h (unscaled) joins the softmax denominator and carries no value
 *     (techniques map row "Learnable attention sink").
 *   - full-causal layers, or sliding-window causal layers in which query i
 *     sees keys i-W < j <= i (W = 128 in the model; techniques map rows
 *     "Sliding-window attention", "Interleaved sliding-window and global
 *     attention"; sliding_window in the llm-atlas field tables).
 *
 *   out[b,i,h,:] = sum_j p_j v[b,j,h/8,:],
 *   p_j = exp(s_j) / (exp(sigma_h) + sum_j' exp(s_j')),
 *   s_j = (R(pos_i) q[b,i,h]) . (R(pos_j) k[b,j,h/8]) / 8.
 *
 * Conventions for every entry point:
 *   - Tensors are bf16 (raw 16-bit patterns), row-major, contiguous,
 *     device memory owned by the caller. The library keeps no pointer
 *     after a call returns. Base pointers must be 16-byte aligned.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream).
 *   - The return value is GPTOSS_ATTN_OK (0) or a negative status code;
 *     no call aborts or prints. Argument errors are reported before any
 *     work is enqueued. Faults detected inside a kernel set the error word
 *     of the stream it was launched on, which gptoss_attn_check(stream)
 *     reports and clears. Each device keeps 64 such words, given to streams
 *     in order of first use; streams beyond the 64th share the last word.
 *   - Accumulation is fp32; the rotated q/k and the probabilities are
 *     rounded to bf16 for the tensor-core products; the output is rounded
 *     to bf16 once.
 */
#ifndef GPTOSS_ATTN_H
#define GPTOSS_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;

#define GPTOSS_ATTN_ABI_VERSION 1

#define GPTOSS_ATTN_NUM_HEADS 64
#define GPTOSS_ATTN_NUM_KV_HEADS 8
#define GPTOSS_ATTN_HEAD_DIM 64
#define GPTOSS_ATTN_MAX_POSITION 131072

enum gptoss_attn_status {
  GPTOSS_ATTN_OK = 0,
  GPTOSS_ATTN_ERR_NULL_PTR = -1,        /* a required pointer is NULL */
  GPTOSS_ATTN_ERR_BAD_SHAPE = -2,       /* batch, seqlen or max_len out of range */
  GPTOSS_ATTN_ERR_BAD_ALIGN = -3,       /* a tensor base pointer is not 16-byte aligned */
  GPTOSS_ATTN_ERR_SMALL_WORKSPACE = -4, /* workspace smaller than required */
  GPTOSS_ATTN_ERR_NO_DEVICE = -5,       /* no current device, or it is not sm_100 */
  GPTOSS_ATTN_ERR_LAUNCH = -6,          /* a CUDA call or kernel launch failed */
  GPTOSS_ATTN_ERR_TENSOR_MAP = -7,      /* the driver rejected a TMA tensor map */
  GPTOSS_ATTN_ERR_ALLOC = -8,           /* library-owned device memory could not be allocated */
  GPTOSS_ATTN_ERR_DEVICE_TIMEOUT = -9,  /* a kernel pipeline wait ran out (reported by check) */
  GPTOSS_ATTN_ERR_BAD_POSITION = -10,   /* a position was outside [0, 131072) (reported by check) */
  GPTOSS_ATTN_ERR_BAD_LENGTH = -11      /* a decode length was outside [0, max_len] (reported by check) */
};

/* ABI version of the loaded library (GPTOSS_ATTN_ABI_VERSION). */
int gptoss_attn_abi_version(void);

/* Static description of a status code; never NULL. */
const char* gptoss_attn_status_string(int status);

/*
 * Prepares the current device: builds the library-owned rotary table
 * (cos, sin of pos * theta^(-2k/64) for every pos < 131072 and k < 32,
 * evaluated in fp64 and stored as fp32, 33.5 MB) and a 4-byte device error
 * word. Idempotent and thread-safe. gptoss_attn_prefill() calls it on its
 * first use on a device; call it explicitly before capturing a CUDA graph,
 * since it allocates. The memory is released when the process exits.
 */
int gptoss_attn_init(void);

/*
 * Diagnostics: stores in *table the device address of the current device's
 * rotary table, fp32 pairs (cos, sin) laid out [131072][32], building it
 * first if needed. The table is read-only and owned by the library.
 */
int gptoss_attn_rope_table(const void** table);

/*
 * YaRN rotary scaling (techniques map row "YaRN RoPE scaling": rope_type yarn,
 * factor 32; initial_context_length 4096 in the llm-atlas field tables). The
 * pages leave the betas, the ramp and the attention factor out; this library
 * uses the transformers yarn initialisation the row names, with beta_fast 32,
 * beta_slow 1 and no truncation: pair k's frequency theta^(-2k/64) is blended
 * with theta^(-2k/64) / 32 by a weight linear in k, 0 up to the pair whose
 * wavelength fits 32 times into 4096 tokens (k ~ 8.09) and 1 from the pair
 * where it fits once (k ~ 17.40); cos and sin are scaled by the attention
 * factor 0.1 ln 32 + 1 (YaRN paper, Peng et al. 2023), so rotated queries and
 * keys both carry it and the logits grow by its square.
 *
 * gptoss_attn_init_yarn() builds the current device's YaRN table (another
 * 33.5 MB, same layout and evaluation as the plain one; allocates, call it
 * before capturing work that uses the _yarn entry points); the _yarn entry
 * points build it on first use. gptoss_attn_rope_table_yarn() returns its
 * address like gptoss_attn_rope_table().
 */
int gptoss_attn_init_yarn(void);
int gptoss_attn_rope_table_yarn(const void** table);

/*
 * Bytes of device workspace gptoss_attn_prefill() needs: room for the rotated
 * keys, batch * seqlen * 8 * 64 bf16 values. Returns 0 for invalid sizes.
 */
size_t gptoss_attn_prefill_workspace_bytes(int batch, int seqlen);

/*
 * Prefill: causal grouped-query attention over whole sequences.
 *   q      bf16 [batch][seqlen][64][64]   (token-major, as the projections emit)
 *   k, v   bf16 [batch][seqlen][8][64]
 *   sinks  fp32 [64] (device), the per-head sink logits sigma_h; -inf allowed
 *   pos    int32 [batch][seqlen] (device), rotary positions in [0, 131072);
 *          masking uses token indices, positions only drive the rotation
 *   window <= 0: full causal; W > 0: key j visible to query i iff i-W < j <= i
 *   out    bf16 [batch][seqlen][64][64]; must not overlap the inputs
 *   batch >= 1, 1 <= seqlen <= 131072 (batch * seqlen * 8 KB must fit the device)
 *   workspace, workspace_bytes: caller-owned device scratch of at least
 *          gptoss_attn_prefill_workspace_bytes(batch, seqlen) bytes, 16-byte
 *          aligned, not overlapping the other tensors; it receives the rotated
 *          keys (each key is rotated once per call, not once per query tile)
 *          and is garbage afterwards. Calls that overlap in time need
 *          separate workspaces.
 * Two kernels run on `stream`: the key rotation, then the attention, which
 * rotates the query rows itself; v is read as given.
 */
int gptoss_attn_prefill(const void* q, const void* k, const void* v, const float* sinks,
                        const int32_t* pos, int window, void* out, int batch, int seqlen,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * gptoss_attn_prefill() that also stores, for every query row, the natural
 * log of its softmax normaliser, sink included:
 *   lse[b][i][h] = ln(exp(sigma_h) + sum_j exp(s_j))   fp32 [batch][seqlen][64]
 * (4-byte aligned, caller-owned device memory). The backward pass
 * (gptoss_attn_prefill_backward) takes it instead of recomputing it.
 */
int gptoss_attn_prefill_lse(const void* q, const void* k, const void* v, const float* sinks,
                            const int32_t* pos, int window, void* out, float* lse, int batch,
                            int seqlen, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/*
 * Bytes of device workspace gptoss_attn_prefill_backward() needs: the rotated
 * queries and keys (bf16), two fp32 values per query row, and fp32 sums of the
 * key and value gradients (64 floats each per token and kv head), plus
 * alignment. Returns 0 for invalid sizes.
 */
size_t gptoss_attn_prefill_backward_workspace_bytes(int batch, int seqlen);

/*
 * Backward pass of gptoss_attn_prefill() (plain RoPE): given the upstream
 * gradient dout of out, the gradients of L = sum(dout * out) with respect to
 * q, k, v (the un-rotated inputs) and the sink logits. The pages print no
 * backward; these are the derivatives of the forward defined above (the sink
 * row of the techniques map makes the sink a softmax column with no value):
 *   D_i = dout_i . out_i,  dS_ij = p_ij (dout_i . v_j - D_i)
 *   dv_j = sum_i p_ij dout_i (over the 8 query heads of the group too)
 *   dq_i = R(pos_i)^T sum_j dS_ij R(pos_j) k_j / 8
 *   dk_j = R(pos_j)^T sum_i dS_ij R(pos_i) q_i / 8
 *   dsinks[h] = -sum_{b,i} exp(sigma_h - lse_i) D_i
 *   q, k, v, sinks, pos, window: the forward's inputs
 *   out    bf16 [batch][seqlen][64][64], the forward's output
 *   lse    fp32 [batch][seqlen][64], from gptoss_attn_prefill_lse()
 *   dout   bf16 [batch][seqlen][64][64]
 *   dq     bf16 [batch][seqlen][64][64];  dk, dv  bf16 [batch][seqlen][8][64]
 *   dsinks fp32 [64] (overwritten; accumulated with atomics, so the order of
 *          the fp32 additions varies from run to run; so does that of dk and
 *          dv, whose fp32 partial sums over chunks of queries are added in the
 *          workspace before the final rounding to bf16)
 *   workspace of gptoss_attn_prefill_backward_workspace_bytes() bytes.
 * Products run on the tensor cores in bf16 with fp32 accumulation: the
 * rotated q, k and the probabilities and dS are rounded to bf16 first. All
 * gradients are written whole (no accumulation into the caller's buffers).
 * Kernels on `stream`: the q and k rotations, a per-row preparation (D, the
 * sink gradient), the dq kernel, the dk/dv kernel.
 */
int gptoss_attn_prefill_backward(const void* q, const void* k, const void* v, const float* sinks,
                                 const int32_t* pos, int window, const void* out, const float* lse,
                                 const void* dout, void* dq, void* dk, void* dv, float* dsinks,
                                 int batch, int seqlen, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream);

/* gptoss_attn_prefill() with the YaRN rotation (see gptoss_attn_init_yarn). */
int gptoss_attn_prefill_yarn(const void* q, const void* k, const void* v, const float* sinks,
                             const int32_t* pos, int window, void* out, int batch, int seqlen,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Chunked prefill: the next n tokens of sequences whose first `start` tokens
 * are already in a key/value cache (a prompt prefilled in pieces, or several
 * new tokens at once against a cache). The same operation as
 * gptoss_attn_prefill() with query token i of the chunk at key index start+i:
 * it sees cache keys j <= start+i (and, for W > 0, j > start+i-W). The gpt-oss
 * pages name the cache (use_cache in the configuration table) but no chunked
 * step; this is the plainest joining of the prefill and decode operations.
 *   q       bf16 [batch][n][64][64], not rotated
 *   k, v    bf16 [batch][n][8][64], the chunk's keys (not rotated) and values
 *   sinks   fp32 [64]; pos int32 [batch][n], rotary positions of the chunk
 *   window  <= 0 full causal; W > 0 as above (W >= start+n is full causal)
 *   out     bf16 [batch][n][64][64]
 *   kcache, vcache  bf16 [batch][max_len][8][64]: rows [0, start) hold the
 *           cached keys (already rotated, as gptoss_attn_decode() expects) and
 *           values; the call writes the chunk's rotated keys to rows
 *           [start, start+n) of kcache and its values to the same rows of
 *           vcache, and reads no row at or past start+n
 *   0 <= start, 1 <= n, start + n <= max_len <= 131072, 1 <= batch <= 65535
 * No workspace. Kernels on `stream`: the value copy, the key rotation into the
 * cache, the attention. Calls on the same cache must be serialized.
 */
int gptoss_attn_prefill_chunk(const void* q, const void* k, const void* v, const float* sinks,
                              const int32_t* pos, int window, void* out, void* kcache,
                              void* vcache, int batch, int start, int n, int max_len,
                              cudaStream_t stream);

/* gptoss_attn_prefill_chunk() with the YaRN rotation: the cached keys must have
 * been rotated by YaRN too (by this call or gptoss_attn_prefill_yarn's layout). */
int gptoss_attn_prefill_chunk_yarn(const void* q, const void* k, const void* v,
                                   const float* sinks, const int32_t* pos, int window, void* out,
                                   void* kcache, void* vcache, int batch, int start, int n,
                                   int max_len, cudaStream_t stream);

/*
 * Bytes of device workspace gptoss_attn_decode() needs for these sizes.
 * Returns 0 for invalid sizes.
 */
size_t gptoss_attn_decode_workspace_bytes(int batch, int max_len, int window);

/*
 * Decode: one new query token per sequence against a key/value cache.
 *   q       bf16 [batch][64][64], not yet rotated; it is rotated here at
 *           position len[b]-1
 *   kcache  bf16 [batch][max_len][8][64], keys already rotated at their positions
 *   vcache  bf16 [batch][max_len][8][64]
 *   sinks   fp32 [64] (device)
 *   len     int32 [batch] (device), the number of cached tokens, the new one
 *           included; 0 <= len[b] <= max_len (len 0 gives a zero output)
 *   window  <= 0: keys [0, len); W > 0: keys [max(0, len-W), len)
 *   out     bf16 [batch][64][64]
 *   workspace, workspace_bytes: caller-owned device scratch of at least
 *           gptoss_attn_decode_workspace_bytes(batch, max_len, window) bytes,
 *           16-byte aligned; its contents need no initialisation and are
 *           garbage afterwards. Calls that overlap in time need separate
 *           workspaces.
 */
int gptoss_attn_decode(const void* q, const void* kcache, const void* vcache, const float* sinks,
                       const int32_t* len, int window, void* out, int batch, int max_len,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* gptoss_attn_decode() with the query rotated by YaRN at position len[b]-1;
 * the cache must hold YaRN-rotated keys. max_len <= 131072 (the table's
 * range), else GPTOSS_ATTN_ERR_BAD_SHAPE. Same workspace size. */
int gptoss_attn_decode_yarn(const void* q, const void* kcache, const void* vcache,
                            const float* sinks, const int32_t* len, int window, void* out,
                            int batch, int max_len, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/*
 * Allocation-free decode. The gpt-oss pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory while they
 * decode, such as serving engines that give all device memory to their own
 * pool up front and forbid later allocations, or latency-bound loops that
 * cannot pay for the synchronization an allocation implies.
 *
 * Same operation and arguments as gptoss_attn_decode() without the
 * workspace: the split partials live in a fixed array of
 * GPTOSS_ATTN_NOALLOC_SCRATCH_BYTES bytes that is part of the library's
 * device image, held on every GPU that loads the library until the process
 * exits. Sizes whose partials do not fit (batch * 64 heads * splits * 264
 * bytes, see gptoss_attn_decode_workspace_bytes()) are rejected with
 * GPTOSS_ATTN_ERR_SMALL_WORKSPACE before any work is enqueued. The call
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.
 * The looked-up address is cached per device ordinal for the life of the
 * process, which assumes the device's primary context throughout (no
 * cudaDeviceReset, no other driver context current during these calls).
 * Every call shares the array, and a call clears only its error word before
 * launching, so calls whose kernels overlap in time on the GPU race: issue
 * them on one stream or otherwise serialize them. Device-side conditions of
 * this path (a length outside [0, max_len], which is clamped; a pipeline
 * timeout) are not reported by gptoss_attn_check(), and this path keeps
 * running while the stream's error word of the other entry points holds a
 * timeout.
 */
#define GPTOSS_ATTN_NOALLOC_SCRATCH_BYTES (8u << 20)

int gptoss_attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                               const float* sinks, const int32_t* len, int window, void* out,
                               int batch, int max_len, cudaStream_t stream);

/*
 * Diagnostic, with no counterpart on the gpt-oss pages: exercises the failure
 * path every kernel pipeline wait uses. One thread waits, through the same
 * bounded wait, on a barrier that nothing arrives at; after timeout_us
 * microseconds (1 .. 2000000, else GPTOSS_ATTN_ERR_BAD_SHAPE) the wait gives
 * up, sets the timeout bit of `stream`'s error word and the kernel returns, so
 * the context stays usable. Until gptoss_attn_check(stream) clears the word,
 * prefill, decode and backward kernels launched on `stream` skip their work
 * (other streams are not affected); check then reports
 * GPTOSS_ATTN_ERR_DEVICE_TIMEOUT. Asynchronous on `stream`.
 */
int gptoss_attn_debug_wait_timeout(unsigned timeout_us, cudaStream_t stream);

/*
 * Synchronizes `stream`, then reads and clears its error word on the current
 * device (stream-ordered; no other stream is waited on). Returns
 * GPTOSS_ATTN_OK, GPTOSS_ATTN_ERR_DEVICE_TIMEOUT, GPTOSS_ATTN_ERR_BAD_POSITION,
 * GPTOSS_ATTN_ERR_BAD_LENGTH or GPTOSS_ATTN_ERR_LAUNCH (a CUDA error surfaced
 * by the synchronization). While a stream's word holds a timeout, kernels
 * launched on that stream skip their work.
 */
int gptoss_attn_check(cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTOSS_ATTN_H */
