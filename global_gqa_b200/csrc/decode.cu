// Decode path: one new token per sequence against its KV cache.
//
//   decode_prologue: QK-RMSNorm + RoPE of the new token's q and k at position
//                    L-1; the rotated key and the value go into cache slot L-1
//                    (global, linear cache) or (L-1) % W (local ring of W
//                    slots); q_hat is kept in fp32, pre-scaled to log2 units.
//   decode_split   : split-KV attention.  One block reads one chunk of up to
//                    kDecodeChunk cached rows of one (sequence, kv head) with
//                    coalesced 128-bit loads and serves all G query heads of the
//                    group from each load; it writes an fp32 partial softmax
//                    (max, sum, unnormalised output) per head.
//   decode_combine : merges the partials of each (sequence, head).
//
// Which slots are visible: a local layer's query sees its last W tokens
// (itself included), which are exactly the min(L, W) filled ring slots; a
// global layer's query sees all L tokens (Gemma 3 Technical Report, sections 1
// and 2).  Slot order inside the ring does not matter because each cached key
// already carries its own absolute rotation.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "g3_internal.h"
#include "sm100_ptx.cuh"

namespace g3 {

// ======================================================== decode prologue
constexpr int kDecPrologueThreads = 256;

template <int D>
__global__ void __launch_bounds__(kDecPrologueThreads) decode_prologue_kernel(DecodeParams p) {
  constexpr int H2 = D / 2;
  constexpr int PER = D / 64;
  __shared__ float s_cos[H2], s_sin[H2];
  __shared__ int s_valid;
  const int b = blockIdx.x;
  const int tid = threadIdx.x;
  const int L = p.seq_lens[b];
  if (tid == 0) {
    const bool valid = L >= 1 && L <= p.max_seq_len && (p.kind == 0 || L <= p.cache_cap);
    s_valid = valid ? 1 : 0;
    p.n_slots[b] = valid ? (p.kind == 1 ? L : min(L, p.window)) : 0;
    if (!valid) record_error(p.err, kErrInvalid, 200);
  }
  for (int f = tid; f < H2; f += blockDim.x) {
    const double inv_freq = exp(-2.0 * f / D * log(p.rope_base));
    const double theta = (double)(L - 1) / p.interp * inv_freq;
    double sd, cd;
    sincos(theta, &sd, &cd);
    s_cos[f] = (float)cd;
    s_sin[f] = (float)sd;
  }
  __syncthreads();
  if (!s_valid) return;

  const int warp = tid >> 5, lane = tid & 31;
  const int slot = (p.kind == 1) ? (L - 1) : ((L - 1) % p.window);
  for (int r = warp; r < p.Hq + p.Hkv; r += kDecPrologueThreads / 32) {
    const bool is_q = r < p.Hq;
    const int hh = is_q ? r : r - p.Hq;
    const __nv_bfloat16* src = is_q ? p.q + ((size_t)b * p.Hq + hh) * D : p.k_new + ((size_t)b * p.Hkv + hh) * D;
    const float* gam = is_q ? p.q_gamma : p.k_gamma;
    float x1[PER], x2[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      x1[e] = __bfloat162float(src[lane * PER + e]);
      x2[e] = __bfloat162float(src[H2 + lane * PER + e]);
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) ss += x1[e] * x1[e] + x2[e] * x2[e];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float rinv = rsqrtf(ss / (float)D + 1e-6f);
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int d = lane * PER + e;
      const float y1 = x1[e] * rinv * gam[d];
      const float y2 = x2[e] * rinv * gam[d + H2];
      const float o1 = y1 * s_cos[d] - y2 * s_sin[d];
      const float o2 = y1 * s_sin[d] + y2 * s_cos[d];
      if (is_q) {
        float* qd = p.q_hat + ((size_t)b * p.Hq + hh) * D;
        qd[d] = o1 * p.scale_log2;
        qd[d + H2] = o2 * p.scale_log2;
      } else {
        const size_t crow = ((size_t)b * p.Hkv + hh) * p.cache_cap + slot;
        const __nv_bfloat16* vsrc = p.v_new + ((size_t)b * p.Hkv + hh) * D;
        p.k_cache[crow * D + d] = __float2bfloat16_rn(o1);
        p.k_cache[crow * D + d + H2] = __float2bfloat16_rn(o2);
        p.v_cache[crow * D + d] = vsrc[d];
        p.v_cache[crow * D + d + H2] = vsrc[d + H2];
      }
    }
  }
}

// ============================================================ decode split
constexpr int kSplitThreads = 128;  // 4 warps
constexpr int kSplitUnroll = 4;     // load steps in flight per warp

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kSplitThreads) decode_split_kernel(DecodeParams p) {
  constexpr int LPT = D / 8;         // lanes per cached row (8 bf16 = 16 bytes each)
  constexpr int TPS = 32 / LPT;      // rows per warp-wide load
  constexpr int WARPS = kSplitThreads / 32;
  constexpr int ROWS_PER_WARP = kDecodeChunk / WARPS;
  __shared__ float s_m[WARPS][G], s_l[WARPS][G];
  __shared__ float s_o[WARPS][G][D];

  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int n = p.n_slots[b];
  const int c0 = chunk * kDecodeChunk;
  if (c0 >= n) return;
  const int c1 = min(c0 + kDecodeChunk, n);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane / LPT, li = lane % LPT;

  float q[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float* qs = p.q_hat + ((size_t)b * p.Hq + kvh * G + g) * D + li * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) q[g][i] = qs[i];
  }
  float m[G], l[G], o[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) o[g][i] = 0.f;
  }

  const size_t head_row0 = ((size_t)b * p.Hkv + kvh) * p.cache_cap;
  const uint4* kbase = reinterpret_cast<const uint4*>(p.k_cache + head_row0 * D) + li;
  const uint4* vbase = reinterpret_cast<const uint4*>(p.v_cache + head_row0 * D) + li;
  const int w0 = c0 + warp * ROWS_PER_WARP;
  const int w1 = min(w0 + ROWS_PER_WARP, c1);

  for (int tb = w0; tb < w1; tb += TPS * kSplitUnroll) {
    uint4 kx[kSplitUnroll], vx[kSplitUnroll];
    bool ok[kSplitUnroll];
#pragma unroll
    for (int u = 0; u < kSplitUnroll; ++u) {
      const int t = tb + u * TPS + sub;
      ok[u] = t < w1;
      kx[u] = ok[u] ? __ldg(kbase + (size_t)t * (D / 8)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kSplitUnroll; ++u) {
      const int t = tb + u * TPS + sub;
      vx[u] = ok[u] ? __ldg(vbase + (size_t)t * (D / 8)) : make_uint4(0, 0, 0, 0);
    }
    float s[kSplitUnroll][G];
#pragma unroll
    for (int u = 0; u < kSplitUnroll; ++u) {
      float kf[8];
      bf16x8_to_f32(kx[u], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) d = fmaf(q[g][i], kf[i], d);
#pragma unroll
        for (int off = LPT / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        s[u][g] = ok[u] ? d : -INFINITY;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = s[0][g];
#pragma unroll
      for (int u = 1; u < kSplitUnroll; ++u) mx = fmaxf(mx, s[u][g]);
      const float m_new = fmaxf(m[g], mx);
      if (m_new == -INFINITY) continue;
      const float alpha = ex2_approx(m[g] - m_new);
      l[g] *= alpha;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[g][i] *= alpha;
#pragma unroll
      for (int u = 0; u < kSplitUnroll; ++u) {
        const float pr = ex2_approx(s[u][g] - m_new);
        float vf[8];
        bf16x8_to_f32(vx[u], vf);
        l[g] += pr;
#pragma unroll
        for (int i = 0; i < 8; ++i) o[g][i] = fmaf(pr, vf[i], o[g][i]);
      }
      m[g] = m_new;
    }
  }

  // Merge the TPS row streams of the warp (lanes with equal li).
#pragma unroll
  for (int off = LPT; off < 32; off <<= 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[g], off);
      const float lo_ = __shfl_xor_sync(0xffffffffu, l[g], off);
      const float mn = fmaxf(m[g], mo);
      const float a = (mn == -INFINITY) ? 0.f : ex2_approx(m[g] - mn);
      const float bb = (mn == -INFINITY) ? 0.f : ex2_approx(mo - mn);
      l[g] = l[g] * a + lo_ * bb;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float oo = __shfl_xor_sync(0xffffffffu, o[g][i], off);
        o[g][i] = o[g][i] * a + oo * bb;
      }
      m[g] = mn;
    }
  }
  if (sub == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int i = 0; i < 8; ++i) s_o[warp][g][li * 8 + i] = o[g][i];
      if (li == 0) {
        s_m[warp][g] = m[g];
        s_l[warp][g] = l[g];
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kSplitThreads) {
    const int g = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, s_m[w][g]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float a = (s_m[w][g] == -INFINITY) ? 0.f : ex2_approx(s_m[w][g] - M);
      acc += a * s_o[w][g][d];
      lsum += a * s_l[w][g];
    }
    const size_t ph = ((size_t)b * p.Hq + kvh * G + g) * p.n_chunks + chunk;
    p.part_o[ph * D + d] = acc;
    if (d == 0) {
      p.part_ml[ph * 2] = M;
      p.part_ml[ph * 2 + 1] = lsum;
    }
  }
}

// ========================================================== decode combine
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  const int d = threadIdx.x;
  const int n = p.n_slots[b];
  __nv_bfloat16* dst = p.out + (size_t)bh * D + d;
  if (n <= 0) {
    *dst = __float2bfloat16_rn(0.f);
    return;
  }
  const int nc = (n + kDecodeChunk - 1) / kDecodeChunk;
  const float* ml = p.part_ml + (size_t)bh * p.n_chunks * 2;
  const float* po = p.part_o + (size_t)bh * p.n_chunks * D + d;
  float M = -INFINITY;
  for (int c = 0; c < nc; ++c) M = fmaxf(M, ml[2 * c]);
  float acc = 0.f, lsum = 0.f;
  for (int c = 0; c < nc; ++c) {
    const float a = ex2_approx(ml[2 * c] - M);
    acc = fmaf(a, po[(size_t)c * D], acc);
    lsum = fmaf(a, ml[2 * c + 1], lsum);
  }
  *dst = __float2bfloat16_rn(acc / lsum);
}

// ================================================================ launchers
cudaError_t launch_decode_prologue(const DecodeParams& p, int D, cudaStream_t st) {
  if (D == 128)
    decode_prologue_kernel<128><<<p.B, kDecPrologueThreads, 0, st>>>(p);
  else if (D == 64)
    decode_prologue_kernel<64><<<p.B, kDecPrologueThreads, 0, st>>>(p);
  else if (D == 256)
    decode_prologue_kernel<256><<<p.B, kDecPrologueThreads, 0, st>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_split_d(const DecodeParams& p, int grid_chunks, cudaStream_t st) {
  dim3 grid(grid_chunks, p.Hkv, p.B);
  switch (p.G) {
    case 1: decode_split_kernel<D, 1><<<grid, kSplitThreads, 0, st>>>(p); break;
    case 2: decode_split_kernel<D, 2><<<grid, kSplitThreads, 0, st>>>(p); break;
    case 4: decode_split_kernel<D, 4><<<grid, kSplitThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_split(const DecodeParams& p, int D, int grid_chunks, cudaStream_t st) {
  if (grid_chunks < 1 || grid_chunks > p.n_chunks) return cudaErrorInvalidValue;
  if (D == 128) return launch_split_d<128>(p, grid_chunks, st);
  if (D == 64) return launch_split_d<64>(p, grid_chunks, st);
  if (D == 256) return launch_split_d<256>(p, grid_chunks, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_combine(const DecodeParams& p, int D, cudaStream_t st) {
  if (D == 128)
    decode_combine_kernel<128><<<p.B * p.Hq, 128, 0, st>>>(p);
  else if (D == 64)
    decode_combine_kernel<64><<<p.B * p.Hq, 64, 0, st>>>(p);
  else if (D == 256)
    decode_combine_kernel<256><<<p.B * p.Hq, 256, 0, st>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace g3
