// Image soft tokens of Gemma 3's multimodal projector ("Gemma explained: what's
// new in Gemma 3", the 27B printout: an RMSNorm over the 1152 vision features,
// eps 1e-6, and a 4x4 average pool with stride 4): the grid_h x grid_w patch
// vectors of an image are averaged over pool x pool blocks (raster order), and
// every pooled vector is RMS-normalised and multiplied by its gain.  A 64x64
// patch grid (896x896 image, 14x14 patches) gives 256 tokens.
//
// Bandwidth-bound: one CTA per output token; thread t holds features 8t ..
// 8t+7, sums its pool^2 patches from 16-byte loads (all in flight), and the
// CTA reduces the sum of squares.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "g3_internal.h"
#include "sm100_ptx.cuh"

namespace g3 {

template <int POOL>
__global__ void __launch_bounds__(kSoftTokenMaxThreads) soft_tokens_kernel(SoftTokenParams p) {
  const int tpt = p.F / 8;  // threads holding features
  const int tw = p.grid_w / POOL, th = p.grid_h / POOL;
  const int tok = blockIdx.x;
  const int b = tok / (th * tw), r = tok % (th * tw), ty = r / tw, tx = r % tw;
  const int t = threadIdx.x;
  __shared__ float red[kSoftTokenMaxThreads / 32];

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  if (t < tpt) {
    uint4 u[POOL * POOL];
#pragma unroll
    for (int dy = 0; dy < POOL; ++dy)
#pragma unroll
      for (int dx = 0; dx < POOL; ++dx) {
        const size_t patch = (size_t)b * p.grid_h * p.grid_w + (size_t)(ty * POOL + dy) * p.grid_w + tx * POOL + dx;
        u[dy * POOL + dx] = __ldg(reinterpret_cast<const uint4*>(p.patches + patch * p.F) + t);
      }
#pragma unroll
    for (int i = 0; i < POOL * POOL; ++i) {
      const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += __uint_as_float(w[e] << 16);
        acc[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
      }
    }
    constexpr float inv = 1.0f / (POOL * POOL);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= inv;
  }
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) ss = fmaf(acc[e], acc[e], ss);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((t & 31) == 0) red[t >> 5] = ss;
  __syncthreads();
  if (t < 32) {
    float v = t < (int)(blockDim.x >> 5) ? red[t] : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (t == 0) red[0] = v;
  }
  __syncthreads();
  const float rinv = rsqrtf(red[0] / p.F + 1e-6f);
  if (t < tpt) {
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(p.gamma) + 2 * t);
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(p.gamma) + 2 * t + 1);
    const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_bf16x2(acc[2 * e] * rinv * g[2 * e], acc[2 * e + 1] * rinv * g[2 * e + 1]);
    reinterpret_cast<uint4*>(p.out + (size_t)tok * p.F)[t] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_soft_tokens(const SoftTokenParams& p, cudaStream_t st) {
  const long long tokens = (long long)p.B * (p.grid_h / p.pool) * (p.grid_w / p.pool);
  const int threads = ((p.F / 8 + 31) / 32) * 32;
  if (tokens < 1 || tokens > 0x7fffffffLL || threads > kSoftTokenMaxThreads) return cudaErrorInvalidValue;
  switch (p.pool) {
    case 1: soft_tokens_kernel<1><<<(unsigned)tokens, threads, 0, st>>>(p); break;
    case 2: soft_tokens_kernel<2><<<(unsigned)tokens, threads, 0, st>>>(p); break;
    case 4: soft_tokens_kernel<4><<<(unsigned)tokens, threads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace g3
