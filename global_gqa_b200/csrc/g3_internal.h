// Internal interface between the host API (api.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace g3 {

constexpr int kTileRows = 128;       // query rows and key rows per attention tile
constexpr int kDecodeChunk = 512;    // cached tokens per decode split-KV block
constexpr size_t kHeaderBytes = 256; // workspace header: error word, site, spare

// Workspace header words (int32): [0] first device error (g3_status),
// [1] site tag of that error.
struct PrologueParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* q_gamma;
  const float* k_gamma;
  const int32_t* positions;
  const int32_t* spans;
  int n_spans;
  int B, S, Hq, Hkv;
  int kind;            // 0 local, 1 global
  int window;
  double rope_base;
  double interp;
  double inv_freq[128];  // base^(-2f/D), f < D/2 (D <= 256), computed on the host in double
  __nv_bfloat16* q_hat;  // [B,S,Hq,D]
  __nv_bfloat16* k_hat;  // [B,S,Hkv,D]
  int32_t* lo;           // [B,S] first visible key of each row
  int32_t* hi;           // [B,S] last visible key of each row
  float2* rope_table;    // optional output [B,S,D/2]: (cos, sin) of each rotation angle (NULL: not stored)
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  int cache_cap;
  // Chunked prefill: this call's tokens are start .. start+S-1 of a sequence
  // of `total` tokens; lo/hi count keys from token key_base; with fill_rows
  // every token's key and value go to row start + t - key_base of k_cache /
  // v_cache.  A whole prefill has start = key_base = 0, total = S, fill_rows 0.
  int start, key_base, total, fill_rows;
  int* err;
};

struct AttnParams {
  const int32_t* lo;
  const int32_t* hi;
  int kv_head_major;   // K/V tensor maps over [B, Hkv, rows, D] (a cache) instead of [B, S, Hkv, D]
  __nv_bfloat16* out;  // [B,S,Hq,D]
  float* lse;          // [B,Hq,S] or null
  int* err;
  int B, S, Hq, Hkv, G;
  int n_qtiles;
  int n_groups;        // G / heads_per_cta
  int heavy_by_head;   // causal layer: run the heavy query tiles kv head by kv head (see the kernel's work order)
  int light_qtiles;    // set by the launcher: query tiles per unit left in the all-units order at the end
  int withhold_cta;    // test-only build: this CTA's MMA thread skips its first "S ready" arrival (-1: none)
  float scale_log2;    // log2(e) / sqrt(D)
};

struct DecodeParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  const float* q_gamma;
  const float* k_gamma;
  __nv_bfloat16* k_cache;  // [B,Hkv,cap,D]
  __nv_bfloat16* v_cache;
  int cache_cap;
  const int32_t* seq_lens;
  int max_seq_len;
  int kind;
  int window;
  double rope_base;
  double interp;
  int B, Hq, Hkv, G;
  float scale_log2;
  int n_chunks;            // ceil(max visible slots / kDecodeChunk)
  float* q_hat;            // [B,Hq,D] fp32, pre-multiplied by scale_log2
  int32_t* n_slots;        // [B] visible cache slots (0 = invalid sequence)
  float* part_ml;          // [B,Hq,n_chunks,2]  (max, sum) in log2 units
  float* part_o;           // [B,Hq,n_chunks,D]
  __nv_bfloat16* out;      // [B,Hq,D]
  int* err;
};

// Launchers return the launch status; `name` receives a static kernel name
// for tracing.
cudaError_t launch_prefill_prologue(const PrologueParams& p, int D, cudaStream_t st);
// Clears a call's device-error word (err[0], err[1]) once the previous work in
// the stream has finished, as a kernel its dependents may launch behind.
cudaError_t launch_error_reset(int* err, cudaStream_t st);
// Chunked prefill on a local layer: copy the ring's history rows (tokens
// key_base .. key_base+hist-1, slot t % W) to rows 0..hist-1 of the [B, Hkv,
// rows, D] buffers ctx_k / ctx_v, or (write_back) the chunk's last min(C, W)
// tokens from rows hist + j back into the ring.
struct RingCopyParams {
  __nv_bfloat16* ring_k;
  __nv_bfloat16* ring_v;
  __nv_bfloat16* ctx_k;
  __nv_bfloat16* ctx_v;
  int B, Hkv, W, rows, hist, key_base, start, C;
};
cudaError_t launch_ring_gather(const RingCopyParams& p, int D, cudaStream_t st);
cudaError_t launch_ring_write_back(const RingCopyParams& p, int D, cudaStream_t st);
cudaError_t launch_prefill_attention(const AttnParams& p, int D, int heads_per_cta, const CUtensorMap& tm_q,
                                     const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_out,
                                     cudaStream_t st);
size_t prefill_attention_smem_bytes(int D, int heads_per_cta);

// Sets the calling thread's g3attn_last_error() text.
void set_last_error(const char* msg);

// Image soft tokens: pool x pool average of a grid_h x grid_w patch grid, then
// RMS norm over F features times gamma.
constexpr int kSoftTokenMaxThreads = 1024;
struct SoftTokenParams {
  const __nv_bfloat16* patches;  // [B, grid_h * grid_w, F]
  const float* gamma;            // [F]
  __nv_bfloat16* out;            // [B, (grid_h / pool) * (grid_w / pool), F]
  int B, grid_h, grid_w, F, pool;
};
cudaError_t launch_soft_tokens(const SoftTokenParams& p, cudaStream_t st);

// Prefill backward (gradients of one attention call).  Row data padded to
// whole 128-row tiles: lse2 [B, Hq, S_pad] = lse * log2 e (+inf on padding
// rows) and delta [B, Hq, S_pad] = dout . out (0 on padding rows); colmask
// [B, S_pad] of (lo, hi), never visible on padding rows; kvrange [B,
// n_kv_tiles] of the first and last query tile that sees each key tile.
struct BwdParams {
  const __nv_bfloat16* q;      // raw [B,S,Hq,D]
  const __nv_bfloat16* k;      // raw [B,S,Hkv,D]
  const float* q_gamma;
  const float* k_gamma;
  const __nv_bfloat16* out;    // forward output [B,S,Hq,D]
  const __nv_bfloat16* dout;   // [B,S,Hq,D]
  const float* lse;            // forward [B,Hq,S], natural log
  const __nv_bfloat16* q_hat;  // [B,S,Hq,D] normalised, rotated q (recomputed)
  const int32_t* lo;           // [B,S]
  const int32_t* hi;
  const float2* rope_table;    // [B,S,D/2] (cos, sin)
  float* lse2;
  float* delta;
  int2* colmask;
  int2* kvrange;
  float* dq_hat;               // [B,S,Hq,D] fp32, gradient w.r.t. the rotated, normalised q
  float* dk_hat;               // [B,S,Hkv,D] fp32
  __nv_bfloat16* dv;           // [B,S,Hkv,D]
  __nv_bfloat16* dq;           // [B,S,Hq,D]
  __nv_bfloat16* dk;           // [B,S,Hkv,D]
  float* gamma_part;           // [n_norm_blocks, 2, D] per-block gain gradients (q, k)
  float* dq_gamma;             // [D]
  float* dk_gamma;             // [D]
  int* err;
  int B, S, S_pad, Hq, Hkv, G;
  int n_qtiles, n_kvtiles;
  int n_norm_blocks;           // blocks of bwd_norm_rope (>= 2)
  int n_norm_q_blocks;         // the first ones take the query rows, the rest the key rows
  float scale_log2;            // log2(e) / sqrt(D)
  float inv_sqrt_d;
};
constexpr int kNormBwdMaxBlocks = 148 * 4;
cudaError_t launch_bwd_prep(const BwdParams& p, int D, cudaStream_t st);
cudaError_t launch_bwd_dkdv(const BwdParams& p, int D, const CUtensorMap& tm_q, const CUtensorMap& tm_do,
                            const CUtensorMap& tm_k, const CUtensorMap& tm_v, cudaStream_t st);
cudaError_t launch_bwd_dq(const BwdParams& p, int D, const CUtensorMap& tm_q, const CUtensorMap& tm_do,
                          const CUtensorMap& tm_k, const CUtensorMap& tm_v, cudaStream_t st);
cudaError_t launch_bwd_norm_rope(const BwdParams& p, int D, cudaStream_t st);
// Head dim 256 (backward256.cu): maps with 64-row boxes for the streamed
// sub-tiles, 128-row boxes for the resident tiles.
cudaError_t launch_bwd_dv256(const BwdParams& p, const CUtensorMap& tm_q64, const CUtensorMap& tm_do64,
                             const CUtensorMap& tm_k, cudaStream_t st);
cudaError_t launch_bwd_dk256(const BwdParams& p, const CUtensorMap& tm_q64, const CUtensorMap& tm_do64,
                             const CUtensorMap& tm_k, const CUtensorMap& tm_v, cudaStream_t st);
cudaError_t launch_bwd_dq256(const BwdParams& p, const CUtensorMap& tm_q, const CUtensorMap& tm_do,
                             const CUtensorMap& tm_k64, const CUtensorMap& tm_v64, cudaStream_t st);

cudaError_t launch_decode_prologue(const DecodeParams& p, int D, cudaStream_t st);
cudaError_t launch_decode_split(const DecodeParams& p, int D, int grid_chunks, cudaStream_t st);
cudaError_t launch_decode_combine(const DecodeParams& p, int D, cudaStream_t st);

}  // namespace g3
