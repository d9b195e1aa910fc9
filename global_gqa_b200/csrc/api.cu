// Host side of the C ABI declared in include/g3attn.h: argument validation,
// workspace carving, TMA descriptor encoding, kernel launches and tracing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "../../include/g3attn.h"
#include "g3_internal.h"

namespace {

thread_local std::string g_last_error;

g3_status fail(g3_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
g3_status fail(g3_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ tracing
// Events belong to the device that was current when they were created, and
// may only be recorded on that device's streams, so both the pending entries
// and the pool of reusable events carry their device.
struct TraceEntry {
  std::string name;
  int device;
  cudaEvent_t start, stop;
};
struct TraceState {
  std::mutex mu;
  std::atomic<bool> enabled{false};
  std::vector<TraceEntry> pending;
  std::vector<std::pair<int, cudaEvent_t>> pool;  // (device, event)
} g_trace;

// An event of device `dev` (the current device); the caller holds g_trace.mu.
cudaEvent_t trace_event(int dev) {
  for (size_t i = g_trace.pool.size(); i-- > 0;) {
    if (g_trace.pool[i].first == dev) {
      const cudaEvent_t e = g_trace.pool[i].second;
      g_trace.pool.erase(g_trace.pool.begin() + (std::ptrdiff_t)i);
      return e;
    }
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Runs `launch` bracketed by trace events when tracing is on.
template <class F>
cudaError_t traced(const char* name, cudaStream_t st, F&& launch) {
  if (!g_trace.enabled.load(std::memory_order_relaxed)) return launch();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return launch();
  std::lock_guard<std::mutex> lk(g_trace.mu);
  TraceEntry e{name, dev, trace_event(dev), trace_event(dev)};
  cudaEventRecord(e.start, st);
  cudaError_t r = launch();
  cudaEventRecord(e.stop, st);
  g_trace.pending.push_back(e);
  return r;
}

// ------------------------------------------------------------ TMA encoding
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B, S, H, D] bf16, boxes of 64 features x 1 head x 128 tokens x 1 sequence,
// 128-byte swizzle (matches the tcgen05 shared-memory descriptors).
bool make_bshd_map(CUtensorMap* map, const void* base, int B, int S, int H, int D, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)S * H * D * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 4-D tiled map over the first `rows` rows of a [B, H, capacity, D] bf16
// buffer (a KV cache): 64 x 128-row boxes, the same 128-byte-swizzled
// shared-memory tile as make_bshd_map.  Rows at or past `rows` read as zero,
// so a partly filled last tile never brings in stale cache contents.
bool make_bhsd_map(CUtensorMap* map, const void* base, int B, int H, int rows, int capacity, int D) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)capacity * D * 2, (cuuint64_t)H * capacity * D * 2};
  cuuint32_t box[4] = {64, 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------- workspace maps
struct PrefillWs {
  size_t lo, hi, table, q_hat, k_hat, total;
};
// The rotation table (cos, sin per token and frequency) is stored only for the
// backward pass, which re-applies the rotation to the gradients; the forward
// pass forms the angles in registers.
bool prefill_ws(int B, int S, int Hq, int Hkv, int D, PrefillWs* w, bool with_table = false) {
  if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || D < 1) return false;
  const size_t rows = (size_t)B * S;
  size_t off = g3::kHeaderBytes;
  w->lo = off;
  off = align_up(off + rows * 4, 1024);
  w->hi = off;
  off = align_up(off + rows * 4, 1024);
  w->table = off;
  if (with_table) off = align_up(off + rows * (D / 2) * 8, 1024);
  w->q_hat = off;
  off = align_up(off + rows * Hq * D * 2, 1024);
  w->k_hat = off;
  off = align_up(off + rows * Hkv * D * 2, 1024);
  w->total = off;
  return true;
}

// Chunked prefill: rows of history a local chunk reads from the ring.
int chunk_hist(int start, g3_layer_kind kind, int window) {
  return kind == G3_LAYER_LOCAL ? std::min(start, window - 1) : start;
}
struct ChunkWs {
  size_t lo, hi, q_hat, ctx_k, ctx_v, total;
  int rows;  // K/V rows of the local context buffers (history + chunk)
};
bool chunk_ws(int B, int C, int Hq, int Hkv, int D, int start, g3_layer_kind kind, int window, ChunkWs* w) {
  if (B < 1 || C < 1 || Hq < 1 || Hkv < 1 || D < 1 || start < 0) return false;
  if (kind == G3_LAYER_LOCAL && window < 1) return false;
  const size_t rows = (size_t)B * C;
  size_t off = g3::kHeaderBytes;
  w->lo = off;
  off = align_up(off + rows * 4, 1024);
  w->hi = off;
  off = align_up(off + rows * 4, 1024);
  w->q_hat = off;
  off = align_up(off + rows * Hq * D * 2, 1024);
  w->rows = 0;
  w->ctx_k = w->ctx_v = off;
  if (kind == G3_LAYER_LOCAL) {
    w->rows = chunk_hist(start, kind, window) + C;
    const size_t bytes = (size_t)B * Hkv * w->rows * D * 2;
    w->ctx_k = off;
    off = align_up(off + bytes, 1024);
    w->ctx_v = off;
    off = align_up(off + bytes, 1024);
  }
  w->total = off;
  return true;
}

struct DecodeWs {
  size_t q_hat, n_slots, part_ml, part_o, total;
  int n_chunks;
};
bool decode_ws(int B, int Hq, int Hkv, int D, int max_len, DecodeWs* w) {
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || max_len < 1) return false;
  w->n_chunks = (max_len + g3::kDecodeChunk - 1) / g3::kDecodeChunk;
  size_t off = g3::kHeaderBytes;
  w->q_hat = off;
  off = align_up(off + (size_t)B * Hq * D * 4, 256);
  w->n_slots = off;
  off = align_up(off + (size_t)B * 4, 256);
  w->part_ml = off;
  off = align_up(off + (size_t)B * Hq * w->n_chunks * 2 * 4, 256);
  w->part_o = off;
  off = align_up(off + (size_t)B * Hq * w->n_chunks * D * 4, 256);
  w->total = off;
  return true;
}

bool supported_d(int D) { return D == 64 || D == 128 || D == 256; }

// Prefill backward: the forward prologue's buffers, then the padded row data,
// the key-tile ranges, the fp32 gradients of the rotated q and k, and the
// per-block gain partials.
struct BwdWs {
  PrefillWs f;
  size_t lse2, delta, colmask, kvrange, dq_hat, dk_hat, gpart, total;
  int S_pad, n_kvtiles;
};
bool bwd_ws(int B, int S, int Hq, int Hkv, int D, BwdWs* w) {
  if (!prefill_ws(B, S, Hq, Hkv, D, &w->f, /*with_table=*/true)) return false;
  w->n_kvtiles = (S + g3::kTileRows - 1) / g3::kTileRows;
  w->S_pad = w->n_kvtiles * g3::kTileRows;
  size_t off = w->f.total;
  w->lse2 = off;
  off = align_up(off + (size_t)B * Hq * w->S_pad * 4, 1024);
  w->delta = off;
  off = align_up(off + (size_t)B * Hq * w->S_pad * 4, 1024);
  w->colmask = off;
  off = align_up(off + (size_t)B * w->S_pad * 8, 1024);
  w->kvrange = off;
  off = align_up(off + (size_t)B * w->n_kvtiles * 8, 1024);
  w->dq_hat = off;
  off = align_up(off + (size_t)B * S * Hq * D * 4, 1024);
  w->dk_hat = off;
  off = align_up(off + (size_t)B * S * Hkv * D * 4, 1024);
  w->gpart = off;
  off = align_up(off + (size_t)g3::kNormBwdMaxBlocks * 2 * D * 4, 1024);
  w->total = off;
  return true;
}

}  // namespace

void g3::set_last_error(const char* msg) { g_last_error = msg; }

#ifdef G3_FAULT_INJECT
// Test-only build (never the product library): the next prefill launch makes
// the MMA thread of CTA `cta` skip its first "S ready" arrival, so that the
// softmax warps' bounded wait runs out and the kernel reports G3_ERR_TIMEOUT.
namespace {
std::atomic<int> g_withhold_cta{-1};
}
extern "C" void g3attn_test_withhold_s_commit(int32_t cta) { g_withhold_cta.store(cta); }
static int take_withhold_cta() { return g_withhold_cta.exchange(-1); }
#else
static int take_withhold_cta() { return -1; }
#endif

extern "C" {

const char* g3attn_status_string(g3_status s) {
  switch (s) {
    case G3_OK: return "ok";
    case G3_ERR_INVALID_ARG: return "invalid argument";
    case G3_ERR_UNSUPPORTED: return "unsupported configuration";
    case G3_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case G3_ERR_CUDA: return "CUDA error";
    case G3_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

const char* g3attn_last_error(void) { return g_last_error.c_str(); }

size_t g3attn_prefill_workspace_size(int32_t B, int32_t S, int32_t Hq, int32_t Hkv, int32_t D) {
  PrefillWs w;
  if (!prefill_ws(B, S, Hq, Hkv, D, &w)) return 0;
  return w.total;
}

size_t g3attn_prefill_chunk_workspace_size(int32_t B, int32_t C, int32_t Hq, int32_t Hkv, int32_t D, int32_t start,
                                           g3_layer_kind layer_kind, int32_t window) {
  ChunkWs w;
  if (!chunk_ws(B, C, Hq, Hkv, D, start, layer_kind, window, &w)) return 0;
  return w.total;
}

size_t g3attn_prefill_backward_workspace_size(int32_t B, int32_t S, int32_t Hq, int32_t Hkv, int32_t D) {
  BwdWs w;
  if (!bwd_ws(B, S, Hq, Hkv, D, &w)) return 0;
  return w.total;
}

size_t g3attn_decode_workspace_size(int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t max_seq_len) {
  DecodeWs w;
  if (!decode_ws(B, Hq, Hkv, D, max_seq_len, &w)) return 0;
  return w.total;
}

g3_status g3attn_prefill(const void* q, const void* k, const void* v, const float* q_gamma, const float* k_gamma,
                         const int32_t* positions, g3_layer_kind layer_kind, int32_t window, float rope_base,
                         float interp_factor, const int32_t* image_spans, int32_t n_spans, int32_t B, int32_t S,
                         int32_t Hq, int32_t Hkv, int32_t D, void* out, float* lse, void* k_cache, void* v_cache,
                         int32_t cache_capacity, void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  if (!q || !k || !v || !q_gamma || !k_gamma || !positions || !out)
    return fail(G3_ERR_INVALID_ARG, "prefill: a required pointer is NULL");
  if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || D < 1)
    return fail(G3_ERR_INVALID_ARG, "prefill: sizes must be positive (B=%d S=%d Hq=%d Hkv=%d D=%d)", B, S, Hq, Hkv, D);
  if (Hq % Hkv != 0) return fail(G3_ERR_INVALID_ARG, "prefill: Hq %% Hkv != 0 (%d, %d)", Hq, Hkv);
  if (layer_kind != G3_LAYER_LOCAL && layer_kind != G3_LAYER_GLOBAL)
    return fail(G3_ERR_INVALID_ARG, "prefill: bad layer kind %d", (int)layer_kind);
  if (layer_kind == G3_LAYER_LOCAL && window < 1) return fail(G3_ERR_INVALID_ARG, "prefill: window < 1");
  if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return fail(G3_ERR_INVALID_ARG, "prefill: bad rope_base");
  if (!(interp_factor > 0.f) || !std::isfinite(interp_factor))
    return fail(G3_ERR_INVALID_ARG, "prefill: bad interp_factor");
  if (n_spans < 0 || (n_spans > 0 && image_spans == nullptr) || (n_spans == 0 && image_spans != nullptr))
    return fail(G3_ERR_INVALID_ARG, "prefill: image_spans must be NULL iff n_spans == 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(G3_ERR_INVALID_ARG, "prefill: q, k, v and out must be 16-byte aligned");
  if ((k_cache == nullptr) != (v_cache == nullptr))
    return fail(G3_ERR_INVALID_ARG, "prefill: give both caches or neither");
  if (k_cache != nullptr) {
    if (!aligned16(k_cache) || !aligned16(v_cache))
      return fail(G3_ERR_INVALID_ARG, "prefill: caches must be 16-byte aligned");
    if (layer_kind == G3_LAYER_GLOBAL && cache_capacity < S)
      return fail(G3_ERR_INVALID_ARG, "prefill: global cache capacity %d < S %d", cache_capacity, S);
    if (layer_kind == G3_LAYER_LOCAL && cache_capacity != window)
      return fail(G3_ERR_INVALID_ARG, "prefill: local ring capacity %d != window %d", cache_capacity, window);
  }
  if (!supported_d(D)) return fail(G3_ERR_UNSUPPORTED, "prefill: head_dim %d not built (64, 128, 256)", D);
  if ((size_t)B * S * Hq * D >= (1ull << 40)) return fail(G3_ERR_UNSUPPORTED, "prefill: problem too large");
  const int G = Hq / Hkv;
  // Heads per attention CTA.  Two heads of a kv group share each K/V tile
  // (one CTA per SM); sliding-window layers visit few tiles per query tile, so
  // there one-head CTAs, two per SM, hide each other's start and epilogue and
  // run faster.
  // (At D = 256 one head's S and O already take 384 of the 512 TMEM columns.)
  const int hpc = (G % 2 == 0 && layer_kind == G3_LAYER_GLOBAL && D <= 128) ? 2 : 1;
  const long long n_qtiles = (S + g3::kTileRows - 1) / g3::kTileRows;
  if (n_qtiles * B * Hkv * (G / hpc) > 0x7fffffffLL) return fail(G3_ERR_UNSUPPORTED, "prefill: grid too large");

  PrefillWs w;
  prefill_ws(B, S, Hq, Hkv, D, &w);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(G3_ERR_WORKSPACE, "prefill: workspace NULL or not 256-byte aligned");
  if (workspace_bytes < w.total)
    return fail(G3_ERR_WORKSPACE, "prefill: workspace %zu bytes < required %zu", workspace_bytes, w.total);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* err = reinterpret_cast<int*>(ws);

  g3::PrologueParams pp{};
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.v = static_cast<const __nv_bfloat16*>(v);
  pp.q_gamma = q_gamma;
  pp.k_gamma = k_gamma;
  pp.positions = positions;
  pp.spans = image_spans;
  pp.n_spans = n_spans;
  pp.B = B;
  pp.S = S;
  pp.Hq = Hq;
  pp.Hkv = Hkv;
  pp.kind = (int)layer_kind;
  pp.window = layer_kind == G3_LAYER_LOCAL ? window : S;
  pp.rope_base = rope_base;
  pp.interp = interp_factor;
  for (int f = 0; f < D / 2; ++f) pp.inv_freq[f] = std::pow((double)rope_base, -2.0 * f / D);
  pp.q_hat = reinterpret_cast<__nv_bfloat16*>(ws + w.q_hat);
  pp.k_hat = reinterpret_cast<__nv_bfloat16*>(ws + w.k_hat);
  pp.lo = reinterpret_cast<int32_t*>(ws + w.lo);
  pp.hi = reinterpret_cast<int32_t*>(ws + w.hi);
  pp.rope_table = nullptr;  // the forward pass needs no stored table
  pp.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  pp.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  pp.cache_cap = cache_capacity;
  pp.total = S;
  pp.err = err;

  CUtensorMap tq, tk, tv, to;
  if (!make_bshd_map(&tq, pp.q_hat, B, S, Hq, D) || !make_bshd_map(&tk, pp.k_hat, B, S, Hkv, D) ||
      !make_bshd_map(&tv, v, B, S, Hkv, D) ||
      !make_bshd_map(&to, out, B, S, Hq, D))
    return fail(G3_ERR_CUDA, "prefill: cuTensorMapEncodeTiled unavailable or failed");

  // Not traced: events around it would hold the prologue behind it.
  cudaError_t e = g3::launch_error_reset(err, st);
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill: %s", cudaGetErrorString(e));
  e = traced("prefill_prologue", st, [&] { return g3::launch_prefill_prologue(pp, D, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill prologue: %s", cudaGetErrorString(e));

  g3::AttnParams ap{};
  ap.lo = pp.lo;
  ap.hi = pp.hi;
  ap.out = static_cast<__nv_bfloat16*>(out);
  ap.lse = lse;
  ap.err = err;
  ap.B = B;
  ap.S = S;
  ap.Hq = Hq;
  ap.Hkv = Hkv;
  ap.G = G;
  ap.n_qtiles = (int)n_qtiles;
  ap.n_groups = G / hpc;
  ap.heavy_by_head = layer_kind == G3_LAYER_GLOBAL ? 1 : 0;
  ap.withhold_cta = take_withhold_cta();
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  e = traced("prefill_attention", st, [&] { return g3::launch_prefill_attention(ap, D, hpc, tq, tk, tv, to, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill attention: %s", cudaGetErrorString(e));
  return G3_OK;
}

g3_status g3attn_prefill_chunk(const void* q, const void* k, const void* v, const float* q_gamma,
                               const float* k_gamma, const int32_t* positions, void* k_cache, void* v_cache,
                               int32_t cache_capacity, int32_t start, g3_layer_kind layer_kind, int32_t window,
                               float rope_base, float interp_factor, const int32_t* image_spans, int32_t n_spans,
                               int32_t B, int32_t C, int32_t Hq, int32_t Hkv, int32_t D, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  if (!q || !k || !v || !q_gamma || !k_gamma || !positions || !k_cache || !v_cache || !out)
    return fail(G3_ERR_INVALID_ARG, "prefill_chunk: a required pointer is NULL");
  if (B < 1 || C < 1 || Hq < 1 || Hkv < 1 || D < 1 || start < 0)
    return fail(G3_ERR_INVALID_ARG, "prefill_chunk: sizes must be positive and start >= 0 (B=%d C=%d start=%d)", B, C,
                start);
  if (Hq % Hkv != 0) return fail(G3_ERR_INVALID_ARG, "prefill_chunk: Hq %% Hkv != 0 (%d, %d)", Hq, Hkv);
  if (layer_kind != G3_LAYER_LOCAL && layer_kind != G3_LAYER_GLOBAL)
    return fail(G3_ERR_INVALID_ARG, "prefill_chunk: bad layer kind %d", (int)layer_kind);
  if (layer_kind == G3_LAYER_LOCAL && (window < 1 || cache_capacity != window))
    return fail(G3_ERR_INVALID_ARG, "prefill_chunk: local layers need window >= 1 and cache_capacity == window");
  if (layer_kind == G3_LAYER_GLOBAL && (long long)cache_capacity < (long long)start + C)
    return fail(G3_ERR_INVALID_ARG, "prefill_chunk: global cache capacity %d < start + C = %lld", cache_capacity,
                (long long)start + C);
  if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return fail(G3_ERR_INVALID_ARG, "prefill_chunk: bad rope_base");
  if (!(interp_factor > 0.f) || !std::isfinite(interp_factor))
    return fail(G3_ERR_INVALID_ARG, "prefill_chunk: bad interp_factor");
  if (n_spans < 0 || (n_spans > 0 && image_spans == nullptr) || (n_spans == 0 && image_spans != nullptr))
    return fail(G3_ERR_INVALID_ARG, "prefill_chunk: image_spans must be NULL iff n_spans == 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(k_cache) ||
      !aligned16(v_cache))
    return fail(G3_ERR_INVALID_ARG, "prefill_chunk: q, k, v, out and the caches must be 16-byte aligned");
  if (!supported_d(D)) return fail(G3_ERR_UNSUPPORTED, "prefill_chunk: head_dim %d not built (64, 128, 256)", D);
  if ((long long)start + C > 0x7fffffffLL || (size_t)B * Hkv * cache_capacity * D >= (1ull << 40) ||
      (size_t)B * C * Hq * D >= (1ull << 40))
    return fail(G3_ERR_UNSUPPORTED, "prefill_chunk: problem too large");
  const int G = Hq / Hkv;
  const int hpc = (G % 2 == 0 && layer_kind == G3_LAYER_GLOBAL && D <= 128) ? 2 : 1;
  const long long n_qtiles = (C + g3::kTileRows - 1) / g3::kTileRows;
  if (n_qtiles * B * Hkv * (G / hpc) > 0x7fffffffLL) return fail(G3_ERR_UNSUPPORTED, "prefill_chunk: grid too large");

  ChunkWs w;
  chunk_ws(B, C, Hq, Hkv, D, start, layer_kind, window, &w);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(G3_ERR_WORKSPACE, "prefill_chunk: workspace NULL or not 256-byte aligned");
  if (workspace_bytes < w.total)
    return fail(G3_ERR_WORKSPACE, "prefill_chunk: workspace %zu bytes < required %zu", workspace_bytes, w.total);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* err = reinterpret_cast<int*>(ws);
  const bool local = layer_kind == G3_LAYER_LOCAL;
  // Keys the chunk can see, as rows of one [B, Hkv, rows, D] buffer: the cache
  // itself on a global layer (token t in row t); on a local layer a context
  // buffer holding the ring's last `hist` tokens and then the chunk.
  const int hist = chunk_hist(start, layer_kind, window);
  const int key_base = local ? start - hist : 0;
  __nv_bfloat16* keys = local ? reinterpret_cast<__nv_bfloat16*>(ws + w.ctx_k) : static_cast<__nv_bfloat16*>(k_cache);
  __nv_bfloat16* vals = local ? reinterpret_cast<__nv_bfloat16*>(ws + w.ctx_v) : static_cast<__nv_bfloat16*>(v_cache);
  const int rows = local ? w.rows : cache_capacity;  // row capacity of `keys` / `vals`
  const int visible = local ? hist + C : start + C;  // rows holding keys of tokens < start + C

  g3::PrologueParams pp{};
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.v = static_cast<const __nv_bfloat16*>(v);
  pp.q_gamma = q_gamma;
  pp.k_gamma = k_gamma;
  pp.positions = positions;
  pp.spans = image_spans;
  pp.n_spans = n_spans;
  pp.B = B;
  pp.S = C;
  pp.Hq = Hq;
  pp.Hkv = Hkv;
  pp.kind = (int)layer_kind;
  pp.window = local ? window : start + C;
  pp.rope_base = rope_base;
  pp.interp = interp_factor;
  for (int f = 0; f < D / 2; ++f) pp.inv_freq[f] = std::pow((double)rope_base, -2.0 * f / D);
  pp.q_hat = reinterpret_cast<__nv_bfloat16*>(ws + w.q_hat);
  pp.k_hat = nullptr;  // keys go straight to their rows in `keys`
  pp.lo = reinterpret_cast<int32_t*>(ws + w.lo);
  pp.hi = reinterpret_cast<int32_t*>(ws + w.hi);
  pp.rope_table = nullptr;  // the forward pass needs no stored table
  pp.k_cache = keys;
  pp.v_cache = vals;
  pp.cache_cap = rows;
  pp.start = start;
  pp.key_base = key_base;
  pp.total = start + C;
  pp.fill_rows = 1;
  pp.err = err;

  g3::RingCopyParams rp{};
  rp.ring_k = static_cast<__nv_bfloat16*>(k_cache);
  rp.ring_v = static_cast<__nv_bfloat16*>(v_cache);
  rp.ctx_k = keys;
  rp.ctx_v = vals;
  rp.B = B;
  rp.Hkv = Hkv;
  rp.W = local ? window : 1;
  rp.rows = rows;
  rp.hist = hist;
  rp.key_base = key_base;
  rp.start = start;
  rp.C = C;

  CUtensorMap tq, tk, tv, to;
  if (!make_bshd_map(&tq, pp.q_hat, B, C, Hq, D) || !make_bhsd_map(&tk, keys, B, Hkv, visible, rows, D) ||
      !make_bhsd_map(&tv, vals, B, Hkv, visible, rows, D) ||
      !make_bshd_map(&to, out, B, C, Hq, D))
    return fail(G3_ERR_CUDA, "prefill_chunk: cuTensorMapEncodeTiled unavailable or failed");

  // Not traced: events around it would hold the prologue behind it.
  cudaError_t e = g3::launch_error_reset(err, st);
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill_chunk: %s", cudaGetErrorString(e));
  if (local && hist > 0) {
    e = traced("prefill_ring_gather", st, [&] { return g3::launch_ring_gather(rp, D, st); });
    if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill_chunk gather: %s", cudaGetErrorString(e));
  }
  e = traced("prefill_prologue", st, [&] { return g3::launch_prefill_prologue(pp, D, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill_chunk prologue: %s", cudaGetErrorString(e));

  g3::AttnParams ap{};
  ap.lo = pp.lo;
  ap.hi = pp.hi;
  ap.kv_head_major = 1;
  ap.out = static_cast<__nv_bfloat16*>(out);
  ap.lse = lse;
  ap.err = err;
  ap.B = B;
  ap.S = C;
  ap.Hq = Hq;
  ap.Hkv = Hkv;
  ap.G = G;
  ap.n_qtiles = (int)n_qtiles;
  ap.n_groups = G / hpc;
  ap.heavy_by_head = 0;  // a chunk's query tiles carry near-equal work
  ap.withhold_cta = take_withhold_cta();
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  e = traced("prefill_attention", st, [&] { return g3::launch_prefill_attention(ap, D, hpc, tq, tk, tv, to, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill_chunk attention: %s", cudaGetErrorString(e));
  if (local) {
    e = traced("prefill_ring_write_back", st, [&] { return g3::launch_ring_write_back(rp, D, st); });
    if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill_chunk write-back: %s", cudaGetErrorString(e));
  }
  return G3_OK;
}

g3_status g3attn_prefill_backward(const void* q, const void* k, const void* v, const float* q_gamma,
                                  const float* k_gamma, const int32_t* positions, g3_layer_kind layer_kind,
                                  int32_t window, float rope_base, float interp_factor, const int32_t* image_spans,
                                  int32_t n_spans, int32_t B, int32_t S, int32_t Hq, int32_t Hkv, int32_t D,
                                  const void* out, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                  float* dq_gamma, float* dk_gamma, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  g_last_error.clear();
  if (!q || !k || !v || !q_gamma || !k_gamma || !positions || !out || !lse || !dout || !dq || !dk || !dv ||
      !dq_gamma || !dk_gamma)
    return fail(G3_ERR_INVALID_ARG, "prefill backward: a required pointer is NULL");
  if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || D < 1)
    return fail(G3_ERR_INVALID_ARG, "prefill backward: sizes must be positive (B=%d S=%d Hq=%d Hkv=%d D=%d)", B, S,
                Hq, Hkv, D);
  if (Hq % Hkv != 0) return fail(G3_ERR_INVALID_ARG, "prefill backward: Hq %% Hkv != 0 (%d, %d)", Hq, Hkv);
  if (layer_kind != G3_LAYER_LOCAL && layer_kind != G3_LAYER_GLOBAL)
    return fail(G3_ERR_INVALID_ARG, "prefill backward: bad layer kind %d", (int)layer_kind);
  if (layer_kind == G3_LAYER_LOCAL && window < 1) return fail(G3_ERR_INVALID_ARG, "prefill backward: window < 1");
  if (!(rope_base > 0.f) || !std::isfinite(rope_base))
    return fail(G3_ERR_INVALID_ARG, "prefill backward: bad rope_base");
  if (!(interp_factor > 0.f) || !std::isfinite(interp_factor))
    return fail(G3_ERR_INVALID_ARG, "prefill backward: bad interp_factor");
  if (n_spans < 0 || (n_spans > 0 && image_spans == nullptr) || (n_spans == 0 && image_spans != nullptr))
    return fail(G3_ERR_INVALID_ARG, "prefill backward: image_spans must be NULL iff n_spans == 0");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return fail(G3_ERR_INVALID_ARG, "prefill backward: bf16 tensors must be 16-byte aligned");
  if (!supported_d(D)) return fail(G3_ERR_UNSUPPORTED, "prefill backward: head_dim %d not built (64, 128, 256)", D);
  if ((size_t)B * S * Hq * D >= (1ull << 40)) return fail(G3_ERR_UNSUPPORTED, "prefill backward: problem too large");
  const int G = Hq / Hkv;
  const long long n_qtiles = (S + g3::kTileRows - 1) / g3::kTileRows;
  if (n_qtiles * B * Hq > 0x7fffffffLL) return fail(G3_ERR_UNSUPPORTED, "prefill backward: grid too large");

  BwdWs w;
  bwd_ws(B, S, Hq, Hkv, D, &w);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(G3_ERR_WORKSPACE, "prefill backward: workspace NULL or not 256-byte aligned");
  if (workspace_bytes < w.total)
    return fail(G3_ERR_WORKSPACE, "prefill backward: workspace %zu bytes < required %zu", workspace_bytes, w.total);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* err = reinterpret_cast<int*>(ws);

  // Forward prologue again: intervals, rotation table, normalised and rotated q and k.
  g3::PrologueParams pp{};
  pp.q = static_cast<const __nv_bfloat16*>(q);
  pp.k = static_cast<const __nv_bfloat16*>(k);
  pp.v = static_cast<const __nv_bfloat16*>(v);
  pp.q_gamma = q_gamma;
  pp.k_gamma = k_gamma;
  pp.positions = positions;
  pp.spans = image_spans;
  pp.n_spans = n_spans;
  pp.B = B;
  pp.S = S;
  pp.Hq = Hq;
  pp.Hkv = Hkv;
  pp.kind = (int)layer_kind;
  pp.window = layer_kind == G3_LAYER_LOCAL ? window : S;
  pp.rope_base = rope_base;
  pp.interp = interp_factor;
  for (int f = 0; f < D / 2; ++f) pp.inv_freq[f] = std::pow((double)rope_base, -2.0 * f / D);
  pp.q_hat = reinterpret_cast<__nv_bfloat16*>(ws + w.f.q_hat);
  pp.k_hat = reinterpret_cast<__nv_bfloat16*>(ws + w.f.k_hat);
  pp.lo = reinterpret_cast<int32_t*>(ws + w.f.lo);
  pp.hi = reinterpret_cast<int32_t*>(ws + w.f.hi);
  pp.rope_table = reinterpret_cast<float2*>(ws + w.f.table);
  pp.total = S;
  pp.err = err;

  g3::BwdParams bp{};
  bp.q = pp.q;
  bp.k = pp.k;
  bp.q_gamma = q_gamma;
  bp.k_gamma = k_gamma;
  bp.out = static_cast<const __nv_bfloat16*>(out);
  bp.dout = static_cast<const __nv_bfloat16*>(dout);
  bp.lse = lse;
  bp.q_hat = pp.q_hat;
  bp.lo = pp.lo;
  bp.hi = pp.hi;
  bp.rope_table = pp.rope_table;
  bp.lse2 = reinterpret_cast<float*>(ws + w.lse2);
  bp.delta = reinterpret_cast<float*>(ws + w.delta);
  bp.colmask = reinterpret_cast<int2*>(ws + w.colmask);
  bp.kvrange = reinterpret_cast<int2*>(ws + w.kvrange);
  bp.dq_hat = reinterpret_cast<float*>(ws + w.dq_hat);
  bp.dk_hat = reinterpret_cast<float*>(ws + w.dk_hat);
  bp.dv = static_cast<__nv_bfloat16*>(dv);
  bp.dq = static_cast<__nv_bfloat16*>(dq);
  bp.dk = static_cast<__nv_bfloat16*>(dk);
  bp.gamma_part = reinterpret_cast<float*>(ws + w.gpart);
  bp.dq_gamma = dq_gamma;
  bp.dk_gamma = dk_gamma;
  bp.err = err;
  bp.B = B;
  bp.S = S;
  bp.S_pad = w.S_pad;
  bp.Hq = Hq;
  bp.Hkv = Hkv;
  bp.G = G;
  bp.n_qtiles = (int)n_qtiles;
  bp.n_kvtiles = w.n_kvtiles;
  // Norm/RoPE backward blocks: query rows and key rows in proportion to Hq : Hkv.
  const long long norm_blocks = std::max<long long>(2, std::min<long long>(((long long)B * S + 7) / 8 * 2,
                                                                           g3::kNormBwdMaxBlocks));
  bp.n_norm_blocks = (int)norm_blocks;
  bp.n_norm_q_blocks =
      (int)std::min<long long>(norm_blocks - 1, std::max<long long>(1, norm_blocks * Hq / (Hq + Hkv)));
  bp.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  bp.inv_sqrt_d = (float)(1.0 / std::sqrt((double)D));

  CUtensorMap tq, tdo, tk, tv;
  if (!make_bshd_map(&tq, pp.q_hat, B, S, Hq, D) || !make_bshd_map(&tdo, dout, B, S, Hq, D) ||
      !make_bshd_map(&tk, pp.k_hat, B, S, Hkv, D) || !make_bshd_map(&tv, v, B, S, Hkv, D))
    return fail(G3_ERR_CUDA, "prefill backward: cuTensorMapEncodeTiled unavailable or failed");

  // Not traced: events around it would hold the prologue behind it.
  cudaError_t e = g3::launch_error_reset(err, st);
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill backward: %s", cudaGetErrorString(e));
  e = traced("prefill_prologue", st, [&] { return g3::launch_prefill_prologue(pp, D, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "prefill backward prologue: %s", cudaGetErrorString(e));
  e = traced("backward_prep", st, [&] { return g3::launch_bwd_prep(bp, D, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "backward prep: %s", cudaGetErrorString(e));
  if (D == 256) {
    // Head dim 256: 64-row sub-tiles on the streamed side, dV and dK from two kernels.
    CUtensorMap tq64, tdo64, tk64, tv64;
    if (!make_bshd_map(&tq64, pp.q_hat, B, S, Hq, D, 64) || !make_bshd_map(&tdo64, dout, B, S, Hq, D, 64) ||
        !make_bshd_map(&tk64, pp.k_hat, B, S, Hkv, D, 64) || !make_bshd_map(&tv64, v, B, S, Hkv, D, 64))
      return fail(G3_ERR_CUDA, "prefill backward: cuTensorMapEncodeTiled unavailable or failed");
    e = traced("backward_dv", st, [&] { return g3::launch_bwd_dv256(bp, tq64, tdo64, tk, st); });
    if (e != cudaSuccess) return fail(G3_ERR_CUDA, "backward dv: %s", cudaGetErrorString(e));
    e = traced("backward_dk", st, [&] { return g3::launch_bwd_dk256(bp, tq64, tdo64, tk, tv, st); });
    if (e != cudaSuccess) return fail(G3_ERR_CUDA, "backward dk: %s", cudaGetErrorString(e));
    e = traced("backward_dq", st, [&] { return g3::launch_bwd_dq256(bp, tq, tdo, tk64, tv64, st); });
    if (e != cudaSuccess) return fail(G3_ERR_CUDA, "backward dq: %s", cudaGetErrorString(e));
  } else {
    e = traced("backward_dkdv", st, [&] { return g3::launch_bwd_dkdv(bp, D, tq, tdo, tk, tv, st); });
    if (e != cudaSuccess) return fail(G3_ERR_CUDA, "backward dk/dv: %s", cudaGetErrorString(e));
    e = traced("backward_dq", st, [&] { return g3::launch_bwd_dq(bp, D, tq, tdo, tk, tv, st); });
    if (e != cudaSuccess) return fail(G3_ERR_CUDA, "backward dq: %s", cudaGetErrorString(e));
  }
  e = traced("backward_norm_rope", st, [&] { return g3::launch_bwd_norm_rope(bp, D, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "backward norm/rope: %s", cudaGetErrorString(e));
  return G3_OK;
}

g3_status g3attn_decode(const void* q, const void* k_new, const void* v_new, const float* q_gamma,
                        const float* k_gamma, void* k_cache, void* v_cache, int32_t cache_capacity,
                        const int32_t* seq_lens, int32_t max_seq_len, g3_layer_kind layer_kind, int32_t window,
                        float rope_base, float interp_factor, int32_t B, int32_t Hq, int32_t Hkv, int32_t D,
                        void* out, void* workspace, size_t workspace_bytes, void* stream) {
  g_last_error.clear();
  if (!q || !k_new || !v_new || !q_gamma || !k_gamma || !k_cache || !v_cache || !seq_lens || !out)
    return fail(G3_ERR_INVALID_ARG, "decode: a required pointer is NULL");
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || max_seq_len < 1 || cache_capacity < 1)
    return fail(G3_ERR_INVALID_ARG, "decode: sizes must be positive");
  if (Hq % Hkv != 0) return fail(G3_ERR_INVALID_ARG, "decode: Hq %% Hkv != 0 (%d, %d)", Hq, Hkv);
  if (layer_kind != G3_LAYER_LOCAL && layer_kind != G3_LAYER_GLOBAL)
    return fail(G3_ERR_INVALID_ARG, "decode: bad layer kind %d", (int)layer_kind);
  if (layer_kind == G3_LAYER_LOCAL && (window < 1 || cache_capacity != window))
    return fail(G3_ERR_INVALID_ARG, "decode: local layers need window >= 1 and cache_capacity == window");
  if (!(rope_base > 0.f) || !std::isfinite(rope_base)) return fail(G3_ERR_INVALID_ARG, "decode: bad rope_base");
  if (!(interp_factor > 0.f) || !std::isfinite(interp_factor))
    return fail(G3_ERR_INVALID_ARG, "decode: bad interp_factor");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(G3_ERR_INVALID_ARG, "decode: caches must be 16-byte aligned");
  if (!supported_d(D)) return fail(G3_ERR_UNSUPPORTED, "decode: head_dim %d not built (64, 128, 256)", D);
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4) return fail(G3_ERR_UNSUPPORTED, "decode: group size %d not built (1, 2, 4)", G);
  if ((size_t)B * Hkv * cache_capacity * D >= (1ull << 40)) return fail(G3_ERR_UNSUPPORTED, "decode: cache too large");

  // The split-KV partials are laid out for the slots a query can see: on a
  // local layer at most min(max_seq_len, window), however long the sequence.
  DecodeWs w;
  const int visible_max = layer_kind == G3_LAYER_LOCAL ? std::min(max_seq_len, window) : max_seq_len;
  decode_ws(B, Hq, Hkv, D, visible_max, &w);
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(G3_ERR_WORKSPACE, "decode: workspace NULL or not 256-byte aligned");
  if (workspace_bytes < w.total)
    return fail(G3_ERR_WORKSPACE, "decode: workspace %zu bytes < required %zu", workspace_bytes, w.total);

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  g3::DecodeParams dp{};
  dp.q = static_cast<const __nv_bfloat16*>(q);
  dp.k_new = static_cast<const __nv_bfloat16*>(k_new);
  dp.v_new = static_cast<const __nv_bfloat16*>(v_new);
  dp.q_gamma = q_gamma;
  dp.k_gamma = k_gamma;
  dp.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  dp.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  dp.cache_cap = cache_capacity;
  dp.seq_lens = seq_lens;
  dp.max_seq_len = max_seq_len;
  dp.kind = (int)layer_kind;
  dp.window = layer_kind == G3_LAYER_LOCAL ? window : cache_capacity;
  dp.rope_base = rope_base;
  dp.interp = interp_factor;
  dp.B = B;
  dp.Hq = Hq;
  dp.Hkv = Hkv;
  dp.G = G;
  dp.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  dp.n_chunks = w.n_chunks;
  dp.q_hat = reinterpret_cast<float*>(ws + w.q_hat);
  dp.n_slots = reinterpret_cast<int32_t*>(ws + w.n_slots);
  dp.part_ml = reinterpret_cast<float*>(ws + w.part_ml);
  dp.part_o = reinterpret_cast<float*>(ws + w.part_o);
  dp.out = static_cast<__nv_bfloat16*>(out);
  dp.err = reinterpret_cast<int*>(ws);

  // The split grid only needs to cover the slots a query can see.
  g3::DecodeParams split = dp;
  const int split_chunks = (visible_max + g3::kDecodeChunk - 1) / g3::kDecodeChunk;

  cudaError_t e = cudaMemsetAsync(dp.err, 0, 8, st);
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "decode: %s", cudaGetErrorString(e));
  e = traced("decode_prologue", st, [&] { return g3::launch_decode_prologue(dp, D, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "decode prologue: %s", cudaGetErrorString(e));
  e = traced("decode_split", st, [&] { return g3::launch_decode_split(split, D, split_chunks, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "decode split: %s", cudaGetErrorString(e));
  e = traced("decode_combine", st, [&] { return g3::launch_decode_combine(dp, D, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "decode combine: %s", cudaGetErrorString(e));
  return G3_OK;
}

g3_status g3attn_soft_tokens(const void* patches, const float* gamma, int32_t B, int32_t grid_h, int32_t grid_w,
                             int32_t F, int32_t pool, void* out, void* stream) {
  g_last_error.clear();
  if (!patches || !gamma || !out) return fail(G3_ERR_INVALID_ARG, "soft_tokens: a required pointer is NULL");
  if (B < 1 || grid_h < 1 || grid_w < 1 || F < 8 || pool < 1)
    return fail(G3_ERR_INVALID_ARG, "soft_tokens: sizes must be positive (B=%d grid %dx%d F=%d pool=%d)", B, grid_h,
                grid_w, F, pool);
  if (grid_h % pool != 0 || grid_w % pool != 0)
    return fail(G3_ERR_INVALID_ARG, "soft_tokens: grid %dx%d is not a multiple of pool %d", grid_h, grid_w, pool);
  if (!aligned16(patches) || !aligned16(gamma) || !aligned16(out))
    return fail(G3_ERR_INVALID_ARG, "soft_tokens: patches, gamma and out must be 16-byte aligned");
  if (F % 8 != 0 || F > 8 * g3::kSoftTokenMaxThreads)
    return fail(G3_ERR_UNSUPPORTED, "soft_tokens: F=%d not built (a multiple of 8 up to %d)", F,
                8 * g3::kSoftTokenMaxThreads);
  if (pool != 1 && pool != 2 && pool != 4) return fail(G3_ERR_UNSUPPORTED, "soft_tokens: pool %d not built (1, 2, 4)", pool);
  if ((long long)B * (grid_h / pool) * (grid_w / pool) > 0x7fffffffLL || (size_t)B * grid_h * grid_w * F >= (1ull << 40))
    return fail(G3_ERR_UNSUPPORTED, "soft_tokens: problem too large");
  g3::SoftTokenParams sp{};
  sp.patches = static_cast<const __nv_bfloat16*>(patches);
  sp.gamma = gamma;
  sp.out = static_cast<__nv_bfloat16*>(out);
  sp.B = B;
  sp.grid_h = grid_h;
  sp.grid_w = grid_w;
  sp.F = F;
  sp.pool = pool;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = traced("soft_tokens", st, [&] { return g3::launch_soft_tokens(sp, st); });
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "soft_tokens: %s", cudaGetErrorString(e));
  return G3_OK;
}

g3_status g3attn_check_device_error(void* workspace, void* stream) {
  if (workspace == nullptr) return fail(G3_ERR_WORKSPACE, "check: workspace is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int h[2] = {0, 0};
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(G3_ERR_CUDA, "check: %s", cudaGetErrorString(e));
  if (h[0] != 0) {
    const int zero[2] = {0, 0};
    cudaMemcpy(workspace, zero, sizeof(zero), cudaMemcpyHostToDevice);
    fail((g3_status)h[0], "device error %d at site %d", h[0], h[1]);
    return (g3_status)h[0];
  }
  return G3_OK;
}

g3_status g3attn_trace_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_trace.mu);
  g_trace.enabled.store(enable != 0, std::memory_order_relaxed);
  return G3_OK;
}

int32_t g3attn_trace_collect(g3_kernel_trace* out, int32_t max_entries) {
  std::lock_guard<std::mutex> lk(g_trace.mu);
  std::vector<g3_kernel_trace> agg;
  for (TraceEntry& t : g_trace.pending) {
    float ms = 0.f;
    cudaEventSynchronize(t.stop);
    cudaEventElapsedTime(&ms, t.start, t.stop);
    g3_kernel_trace* slot = nullptr;
    for (auto& a : agg)
      if (t.name == a.name) slot = &a;
    if (slot == nullptr) {
      agg.push_back(g3_kernel_trace{});
      slot = &agg.back();
      std::snprintf(slot->name, sizeof(slot->name), "%s", t.name.c_str());
    }
    slot->launches += 1;
    slot->total_ms += ms;
    g_trace.pool.emplace_back(t.device, t.start);
    g_trace.pool.emplace_back(t.device, t.stop);
  }
  g_trace.pending.clear();
  const int n = (int)agg.size() < max_entries ? (int)agg.size() : max_entries;
  for (int i = 0; i < n && out != nullptr; ++i) out[i] = agg[i];
  return n;
}

}  // extern "C"
