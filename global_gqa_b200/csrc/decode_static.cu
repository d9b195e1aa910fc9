// g3attn_decode_no_alloc: the decode step for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a device buffer for the workspace: a
// plugin whose host framework owns every byte of device memory through its own
// pool and forbids outside allocations, a real-time serving loop in which a
// cudaMalloc (which may synchronise the device) is not allowed, or a C caller
// with no allocator of its own at all.  This entry point runs the same three
// decode kernels as g3attn_decode, but their scratch (error header, rotated
// query, per-sequence slot counts and split-KV partials) lives in one
// file-scope device array owned by this library instead of a caller workspace.
//
// Costs and limits:
//   * every GPU that loads the library holds kStaticScratchBytes (16 MiB) of
//     device memory for this array until the process exits;
//   * sizes whose scratch would exceed the array are rejected with
//     G3_ERR_UNSUPPORTED (roughly B * Hq * ceil(n / 512) * (D + 2) * 4 bytes
//     plus a small header, n = max_seq_len on a global layer and
//     min(max_seq_len, window) on a local one; see
//     g3attn_decode_workspace_size);
//   * all calls on a device share the one array and it keeps the last call's
//     contents: calls that may overlap on the GPU (different streams without
//     ordering between them) race on it and must be serialised by the caller;
//   * the first call on each device looks up the array's device address; make
//     that first call before any stream capture begins.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/g3attn.h"
#include "g3_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per
// device, with that device current).
g3_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return G3_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[160];
      std::snprintf(msg, sizeof(msg), "decode_no_alloc: cudaGetSymbolAddress failed on device %d: %s", dev,
                    cudaGetErrorString(e));
      g3::set_last_error(msg);
      return G3_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return G3_OK;
}

}  // namespace

extern "C" g3_status g3attn_decode_no_alloc(const void* q, const void* k_new, const void* v_new,
                                            const float* q_gamma, const float* k_gamma, void* k_cache,
                                            void* v_cache, int32_t cache_capacity, const int32_t* seq_lens,
                                            int32_t max_seq_len, g3_layer_kind layer_kind, int32_t window,
                                            float rope_base, float interp_factor, int32_t B, int32_t Hq,
                                            int32_t Hkv, int32_t D, void* out, void* stream) {
  // Scratch as g3attn_decode lays it out: split-KV partials for the slots a
  // query can see (min(max_seq_len, window) on a local layer).
  const int32_t visible = (layer_kind == G3_LAYER_LOCAL && window >= 1 && window < max_seq_len) ? window : max_seq_len;
  const size_t need = g3attn_decode_workspace_size(B, Hq, Hkv, D, visible);
  if (need == 0) {
    // Invalid sizes: let the regular entry point report them (nothing runs).
    return g3attn_decode(q, k_new, v_new, q_gamma, k_gamma, k_cache, v_cache, cache_capacity, seq_lens,
                         max_seq_len, layer_kind, window, rope_base, interp_factor, B, Hq, Hkv, D, out, nullptr,
                         0, stream);
  }
  if (need > kStaticScratchBytes) {
    char msg[200];
    std::snprintf(msg, sizeof(msg),
                  "decode_no_alloc: these sizes need %zu bytes of scratch; the library's static array holds %zu",
                  need, kStaticScratchBytes);
    g3::set_last_error(msg);
    return G3_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const g3_status s = scratch_for_current_device(&scratch);
  if (s != G3_OK) return s;
  return g3attn_decode(q, k_new, v_new, q_gamma, k_gamma, k_cache, v_cache, cache_capacity, seq_lens,
                       max_seq_len, layer_kind, window, rope_base, interp_factor, B, Hq, Hkv, D, out, scratch,
                       kStaticScratchBytes, stream);
}
