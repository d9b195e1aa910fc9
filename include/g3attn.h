/*
 * g3attn -- attention of Gemma 3's 5:1 local/global decoder block on B200.
 *
 * One call computes one attention layer of the block:
 *   1. QK-norm: per token and head, q and k are divided by their RMS over
 *      head_dim (eps 1e-6) and multiplied by a per-feature gain (Gemma 3
 *      Technical Report, section 2 "Model Architecture"; eps and dim from the
 *      q_norm/k_norm lines of the printouts on "Gemma explained: what's new in
 *      Gemma 3").
 *   2. RoPE with the layer's own base and linear position interpolation:
 *      pairs (d, d + D/2) rotate by (p / interp) * base^(-2d/D) (Technical
 *      Report, section 2 "Long context": local base 10k, global base 1M,
 *      interpolation for the global layers).
 *   3. Masked softmax attention with scale 1/sqrt(D).  Key j is visible from
 *      query i iff (j <= i and (GLOBAL or i - j < window)) or i and j lie in
 *      the same image span (Technical Report, sections 1 and 2 "5:1
 *      interleaving"; "Gemma explained", section "Vision encoder and
 *      processing": bidirectional attention over image tokens).
 *   4. Grouped-query attention: query head h reads key/value head h / G,
 *      G = Hq / Hkv.
 *
 * Conventions for every entry point:
 *   - Tensor arguments are DEVICE pointers to contiguous row-major arrays
 *     owned by the caller.  bf16 tensors are raw IEEE bfloat16 (uint16).
 *     q, k, v, out, k_cache, v_cache must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous: G3_OK means the work was enqueued.
 *   - The library allocates no device memory and keeps no per-call state.
 *     Scratch lives in the caller's `workspace`, sized by the matching
 *     *_workspace_size() query; one workspace must not be shared by two
 *     calls that may run concurrently.
 *   - Argument errors are detected on the host before any launch and return
 *     G3_ERR_INVALID_ARG or G3_ERR_UNSUPPORTED; nothing is enqueued then.
 *     Errors that depend on device-resident values (image spans that are
 *     unsorted, overlapping or out of range; sequence lengths out of range)
 *     and bounded-wait timeouts inside the kernels are recorded in the
 *     workspace and reported by g3attn_check_device_error().  A kernel that
 *     meets such an error writes no output for the affected rows but never
 *     reads or writes out of bounds.
 *   - Launch failures return G3_ERR_CUDA; g3attn_last_error() gives detail.
 */
#ifndef G3ATTN_H
#define G3ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  G3_OK = 0,
  G3_ERR_INVALID_ARG = 1,  /* bad pointer, size, shape, or device-side value */
  G3_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim or group size    */
  G3_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small     */
  G3_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed           */
  G3_ERR_TIMEOUT = 5       /* a bounded wait inside a kernel gave up         */
} g3_status;

typedef enum { G3_LAYER_LOCAL = 0, G3_LAYER_GLOBAL = 1 } g3_layer_kind;

/* ------------------------------------------------------------------ prefill
 * Bytes of workspace g3attn_prefill needs for these sizes (0 if the sizes are
 * invalid).  The workspace must be 256-byte aligned.
 */
size_t g3attn_prefill_workspace_size(int32_t B, int32_t S, int32_t Hq, int32_t Hkv, int32_t D);

/*
 * Prefill: attention of all S query tokens of B sequences for one layer.
 *
 *   q          bf16 [B, S, Hq,  D]  raw query projections (before norm/RoPE)
 *   k, v       bf16 [B, S, Hkv, D]  raw key projections, value projections
 *   q_gamma    fp32 [D]             query norm gain (multiplier)
 *   k_gamma    fp32 [D]             key norm gain
 *   positions  int32 [B, S]         RoPE positions (the mask uses token index)
 *   layer_kind G3_LAYER_LOCAL (sliding window) or G3_LAYER_GLOBAL (causal)
 *   window     keys visible to a local query, itself included (>= 1); ignored
 *              for GLOBAL layers
 *   rope_base  > 0;  interp_factor > 0 (positions are divided by it)
 *   image_spans int32 [B, n_spans, 2] half-open [start, end) per sequence,
 *              sorted, disjoint, 0 <= start < end <= S; NULL iff n_spans == 0
 *   B, S, Hq, Hkv, D   S >= 1, Hq % Hkv == 0, D in {64, 128, 256}
 *   out        bf16 [B, S, Hq, D]
 *   lse        optional fp32 [B, Hq, S]: natural-log sum of exp of the scaled
 *              scores of each row (NULL to skip)
 *   k_cache, v_cache optional bf16 [B, Hkv, cache_capacity, D]: when given,
 *              the rotated keys and the values are also written there, for a
 *              later g3attn_decode.  GLOBAL: token t goes to slot t and
 *              cache_capacity >= S.  LOCAL: a ring of cache_capacity == window
 *              slots; token t goes to slot t % window and only the last
 *              min(S, window) tokens are written.  Both NULL to skip.  A
 *              filled cache is read by g3attn_decode, which rotates each new
 *              token by its index, so with a cache positions[b, t] must be t;
 *              any other position is recorded as G3_ERR_INVALID_ARG for
 *              g3attn_check_device_error() (the cache is still written).
 *   workspace  >= g3attn_prefill_workspace_size(B, S, Hq, Hkv, D) bytes
 */
g3_status g3attn_prefill(const void* q, const void* k, const void* v,
                         const float* q_gamma, const float* k_gamma,
                         const int32_t* positions,
                         g3_layer_kind layer_kind, int32_t window,
                         float rope_base, float interp_factor,
                         const int32_t* image_spans, int32_t n_spans,
                         int32_t B, int32_t S, int32_t Hq, int32_t Hkv, int32_t D,
                         void* out, float* lse,
                         void* k_cache, void* v_cache, int32_t cache_capacity,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------- chunked prefill
 * Bytes of workspace g3attn_prefill_chunk needs for these sizes (0 if the
 * sizes are invalid).  The workspace must be 256-byte aligned.
 */
size_t g3attn_prefill_chunk_workspace_size(int32_t B, int32_t C, int32_t Hq, int32_t Hkv, int32_t D,
                                           int32_t start, g3_layer_kind layer_kind, int32_t window);

/*
 * Chunked prefill: the next C tokens of B sequences whose first `start`
 * tokens are already in the KV cache.  The result equals rows start ..
 * start+C-1 of g3attn_prefill over all start + C tokens: the same local or
 * global mask of Gemma 3 (Technical Report, sections 1 and 2), with a long
 * prompt taken in pieces.
 *
 *   q, k, v    bf16 [B, C, Hq|Hkv, D]  raw projections of the chunk's tokens
 *   q_gamma, k_gamma, layer_kind, window, rope_base, interp_factor
 *              as for g3attn_prefill
 *   positions  int32 [B, C]  RoPE positions of the chunk's tokens: start + t
 *              for token t (the cached keys are rotated by their index, as
 *              decode expects); any other value is recorded as
 *              G3_ERR_INVALID_ARG for g3attn_check_device_error()
 *   k_cache, v_cache bf16 [B, Hkv, cache_capacity, D], required: rotated keys
 *              and values of tokens 0 .. start-1 as g3attn_prefill (with
 *              caches) or earlier chunks left them.  GLOBAL: token t in slot t,
 *              cache_capacity >= start + C.  LOCAL: a ring of cache_capacity ==
 *              window slots, token t in slot t % window, holding the last
 *              min(start, window) tokens.  The chunk's tokens are added the
 *              same way (the call reads the ring before it overwrites it).
 *   start      >= 0: tokens already cached; the same for every sequence
 *   image_spans int32 [B, n_spans, 2] half-open, in token indices of the whole
 *              sequence, sorted, disjoint, end <= start + C; no span may hold
 *              tokens on both sides of `start` or of start + C (an image never
 *              crosses a chunk boundary).  NULL iff n_spans == 0.  A violation
 *              found on the device is reported by g3attn_check_device_error().
 *   B, C, Hq, Hkv, D   C >= 1; as for g3attn_prefill otherwise
 *   out        bf16 [B, C, Hq, D];  lse optional fp32 [B, Hq, C]
 *   workspace  >= g3attn_prefill_chunk_workspace_size(...) bytes
 */
g3_status g3attn_prefill_chunk(const void* q, const void* k, const void* v,
                               const float* q_gamma, const float* k_gamma,
                               const int32_t* positions,
                               void* k_cache, void* v_cache, int32_t cache_capacity,
                               int32_t start,
                               g3_layer_kind layer_kind, int32_t window,
                               float rope_base, float interp_factor,
                               const int32_t* image_spans, int32_t n_spans,
                               int32_t B, int32_t C, int32_t Hq, int32_t Hkv, int32_t D,
                               void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------- prefill backward
 * Bytes of workspace g3attn_prefill_backward needs for these sizes (0 if the
 * sizes are invalid).  The workspace must be 256-byte aligned.
 */
size_t g3attn_prefill_backward_workspace_size(int32_t B, int32_t S, int32_t Hq, int32_t Hkv, int32_t D);

/*
 * Prefill backward: gradients of a loss through one g3attn_prefill call, with
 * respect to the raw q, k, v and both QK-norm gains, given dout = dLoss/dout.
 * The Gemma 3 Technical Report trains these layers (section 2.2, distillation;
 * section 2.3, quantization-aware training).  The chain rule runs through the
 * softmax over each row's visible set (the same mask as the forward call), the
 * grouped-query sharing of k and v, the RoPE rotation and the RMS norm.  The
 * rotated, normalised q and k are recomputed, not stored.
 *
 *   q, k, v, q_gamma, k_gamma, positions, layer_kind, window, rope_base,
 *   interp_factor, image_spans, n_spans, B, S, Hq, Hkv
 *              exactly as given to the forward g3attn_prefill call
 *   D          in {64, 128, 256} (G3_ERR_UNSUPPORTED otherwise)
 *   out        bf16 [B, S, Hq, D]  the forward call's output
 *   lse        fp32 [B, Hq, S]     the forward call's lse (required)
 *   dout       bf16 [B, S, Hq, D]  gradient of the loss with respect to out
 *   dq         bf16 [B, S, Hq,  D] gradient with respect to q (written)
 *   dk, dv     bf16 [B, S, Hkv, D] gradients with respect to k and v (written;
 *              summed over the Hq / Hkv query heads that share each kv head)
 *   dq_gamma, dk_gamma  fp32 [D] gradients of the two gains (written; summed
 *              over every token and head in a fixed order, so repeated calls
 *              give identical results)
 *   workspace  >= g3attn_prefill_backward_workspace_size(B, S, Hq, Hkv, D) bytes
 * All tensors are contiguous and 16-byte aligned; the caller owns every buffer.
 * Invalid arguments are rejected before any launch; a device-side wait that
 * times out is reported by g3attn_check_device_error().
 */
g3_status g3attn_prefill_backward(const void* q, const void* k, const void* v,
                                  const float* q_gamma, const float* k_gamma,
                                  const int32_t* positions,
                                  g3_layer_kind layer_kind, int32_t window,
                                  float rope_base, float interp_factor,
                                  const int32_t* image_spans, int32_t n_spans,
                                  int32_t B, int32_t S, int32_t Hq, int32_t Hkv, int32_t D,
                                  const void* out, const float* lse, const void* dout,
                                  void* dq, void* dk, void* dv, float* dq_gamma, float* dk_gamma,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* -------------------------------------------------------------- soft tokens
 * Image soft tokens of the multimodal projector ("Gemma explained: what's new
 * in Gemma 3", 27B printout: RMSNorm over the vision features with eps 1e-6,
 * and a 4x4 average pool with stride 4).  Each pool x pool block of an image's
 * patch grid (raster order) is averaged, then RMS-normalised over its F
 * features and multiplied by gamma.  An 896x896 image in 14x14 patches is a
 * 64x64 grid, i.e. 256 soft tokens.  The projection to the language model's
 * width (a trained matrix) is not part of this call.
 *
 *   patches   bf16 [B, grid_h * grid_w, F]   vision features, 16-byte aligned
 *   gamma     fp32 [F]                       gain (multiplier), 16-byte aligned
 *   grid_h, grid_w, pool   pool in {1, 2, 4}; grid_h and grid_w multiples of pool
 *   F         multiple of 8, 8 <= F <= 8192
 *   out       bf16 [B, (grid_h/pool) * (grid_w/pool), F], 16-byte aligned
 * No workspace; asynchronous on `stream`.
 */
g3_status g3attn_soft_tokens(const void* patches, const float* gamma, int32_t B, int32_t grid_h,
                             int32_t grid_w, int32_t F, int32_t pool, void* out, void* stream);

/* ------------------------------------------------------------------- decode
 * Bytes of workspace g3attn_decode needs (0 if the sizes are invalid).  The
 * figure for max_seq_len covers both layer kinds; a LOCAL layer needs only the
 * figure for min(max_seq_len, window), the most slots a query there can see.
 */
size_t g3attn_decode_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t D,
                                    int32_t max_seq_len);

/*
 * Decode: one new token per sequence, attending to its cached context.
 *
 *   q          bf16 [B, Hq, D]   raw query of the new token
 *   k_new, v_new bf16 [B, Hkv, D] raw key / value of the new token
 *   q_gamma, k_gamma fp32 [D]
 *   k_cache, v_cache bf16 [B, Hkv, cache_capacity, D]: rotated keys and values
 *              of earlier tokens.  GLOBAL: token t in slot t.  LOCAL: ring of
 *              cache_capacity == window slots, token t in slot t % window.
 *              The call first writes the new token's rotated key and its value
 *              into slot L-1 (GLOBAL) or (L-1) % window (LOCAL), then attends.
 *   seq_lens   int32 [B] on the device: tokens of each sequence including the
 *              new one (its position and index are L-1); 1 <= L <= max_seq_len,
 *              and L <= cache_capacity for GLOBAL layers
 *   max_seq_len host-side upper bound of seq_lens, used to size the launch
 *   out        bf16 [B, Hq, D]
 *   workspace  >= g3attn_decode_workspace_size(B, Hq, Hkv, D, n) bytes, n =
 *              max_seq_len (GLOBAL) or min(max_seq_len, window) (LOCAL)
 * A sequence whose length is out of range gets a zero output row, its cache is
 * left untouched, and G3_ERR_INVALID_ARG is recorded for
 * g3attn_check_device_error().
 */
g3_status g3attn_decode(const void* q, const void* k_new, const void* v_new,
                        const float* q_gamma, const float* k_gamma,
                        void* k_cache, void* v_cache, int32_t cache_capacity,
                        const int32_t* seq_lens, int32_t max_seq_len,
                        g3_layer_kind layer_kind, int32_t window,
                        float rope_base, float interp_factor,
                        int32_t B, int32_t Hq, int32_t Hkv, int32_t D,
                        void* out,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode without a caller workspace.  (The sources describe the model only;
 * this entry point has no counterpart there and exists for callers that
 * cannot allocate device memory: a plugin whose host framework owns all device
 * memory through its own pool, a serving loop that may not call cudaMalloc
 * because it can synchronise the device, a C caller with no allocator.)
 *
 * Same arguments and results as g3attn_decode, minus the workspace: the
 * scratch lives in a 16 MiB device array inside the library, which every GPU
 * that loads the library keeps until the process exits.  The call allocates
 * nothing.  Sizes whose scratch (the workspace g3attn_decode would need)
 * exceeds 16 MiB return G3_ERR_UNSUPPORTED with a message in g3attn_last_error().
 * All calls on a device share the array and it keeps the last call's
 * contents, so calls that may overlap on the GPU race and must be ordered by
 * the caller.  The first call on each device looks up the array's address;
 * make it before any stream capture starts.  Out-of-range sequence lengths
 * give zero output rows (their device-side status is not reported by this
 * variant).
 */
g3_status g3attn_decode_no_alloc(const void* q, const void* k_new, const void* v_new,
                                 const float* q_gamma, const float* k_gamma,
                                 void* k_cache, void* v_cache, int32_t cache_capacity,
                                 const int32_t* seq_lens, int32_t max_seq_len,
                                 g3_layer_kind layer_kind, int32_t window,
                                 float rope_base, float interp_factor,
                                 int32_t B, int32_t Hq, int32_t Hkv, int32_t D,
                                 void* out, void* stream);

/* ----------------------------------------------------------------- checking
 * Synchronises `stream`, then returns (and clears) the first device-side error
 * recorded in `workspace` by the last prefill/decode call that used it:
 * G3_OK, G3_ERR_INVALID_ARG (bad spans or sequence lengths) or G3_ERR_TIMEOUT.
 */
g3_status g3attn_check_device_error(void* workspace, void* stream);

/* Static text for a status code. */
const char* g3attn_status_string(g3_status status);

/* Detail of the last host-side error on the calling thread ("" if none). */
const char* g3attn_last_error(void);

/* ------------------------------------------------------------------ tracing
 * When enabled, every kernel the library launches is bracketed by a pair of
 * CUDA events on its own stream; g3attn_trace_collect() synchronises those
 * events and returns, per kernel name, the number of launches and their summed
 * device time since the last collect (which also resets the counts).
 */
typedef struct {
  char name[48];
  int64_t launches;
  double total_ms;
} g3_kernel_trace;

g3_status g3attn_trace_enable(int enable);
int32_t g3attn_trace_collect(g3_kernel_trace* out, int32_t max_entries);

#ifdef __cplusplus
}
#endif

#endif /* G3ATTN_H */
