// Prefill prologue: QK-RMSNorm + RoPE of q and k, the per-row visible key
// interval, and the optional KV-cache fill, in one launch:
//
//   qk_norm_rope: bandwidth-bound pass over every (token, head) row of q and k.
//                 One warp per token: the warp forms the token's rotation
//                 angles and their cos/sin in double (each lane a few of the
//                 D/2 angles, then shuffles), which serve all of its Hq + Hkv
//                 rows; lane 0 writes the token's visible interval and, on
//                 token 0, validates the image spans.  Each lane holds 8
//                 features of each half of a row (16-byte accesses, rotation
//                 partners in the same lane), two row steps in flight per warp
//                 and 32 warps per SM; the gains are read from shared memory to
//                 keep registers free.  When a table is given (the backward
//                 pass reads it), the fp32 (cos, sin) of every angle is also
//                 stored as [B, S, D/2].
//
// Norm (Gemma 3 Technical Report, section 2; eps and dim from the q_norm /
// k_norm lines of "Gemma explained: what's new in Gemma 3"): x / sqrt(mean(x^2)
// + 1e-6) * gamma in fp32.  RoPE (Technical Report, section 2 "Long
// context"): pair (d, d + D/2) turns by theta = (p / interp) * base^(-2d/D);
// the rotation is done in fp32 and the result rounded to bf16.
//
// Visible interval of row i: the causal window [max(0, i-W+1), i] ([0, i] on a
// global layer) joined with the row's image span, which is contiguous because
// both contain i (Technical Report sections 1 and 2; "Gemma explained",
// section "Vision encoder and processing").
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <algorithm>
#include <cstdint>

#include "g3_internal.h"
#include "func_attr.cuh"
#include "sm100_ptx.cuh"

namespace g3 {

constexpr int kRowThreads = 256;  // 8 warps, one token each at a time
constexpr int kRowUnroll = 2;     // row steps in flight per warp (32 warps per SM)

__device__ __forceinline__ void unpack4_bf16(const uint2 u, float* f) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  f[0] = a.x;
  f[1] = a.y;
  f[2] = b.x;
  f[3] = b.y;
}

__device__ __forceinline__ uint2 pack4_bf16(const float* f) {
  return make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
}

template <int D>
__global__ void __launch_bounds__(kRowThreads, 4) qk_norm_rope_kernel(PrologueParams p) {
  constexpr int H2 = D / 2;
  constexpr int LPR = D / 16;    // lanes per row: each holds 8 features of each half
  constexpr int RPW = 32 / LPR;  // rows per warp step
  const int lane = threadIdx.x & 31;
  const int li = lane % LPR, sub = lane / LPR;
  const int d1 = li * 8;  // this lane: features d1..d1+7 and H2+d1..H2+d1+7 (rotation partners)
  const int heads = p.Hq + p.Hkv;
  const int n_tokens = p.B * p.S;
  const int warps_total = gridDim.x * (kRowThreads / 32);
  constexpr int FPL = (H2 + 31) / 32;  // rotation angles formed per lane (FPL divides 8)
  __shared__ __align__(16) float gam[2 * D];  // q gain, then k gain
  __shared__ double inv_freq_s[H2];
  // Launched as a programmatic dependent: nothing of the previous kernel's
  // (it may be producing q, k, v or the positions) is read before this.
  griddep_wait();
  for (int i = threadIdx.x; i < 2 * D; i += kRowThreads) gam[i] = i < D ? p.q_gamma[i] : p.k_gamma[i - D];
  for (int i = threadIdx.x; i < H2; i += kRowThreads) inv_freq_s[i] = p.inv_freq[i];
  __syncthreads();

  for (int bt = blockIdx.x * (kRowThreads / 32) + (threadIdx.x >> 5); bt < n_tokens; bt += warps_total) {
    // Angles (p / interp) * base^(-2f/D) and their cos/sin in double; lane L
    // forms f = FPL * L .. FPL * L + FPL - 1.
    float cl[FPL], sl[FPL];
    const double pos = (double)p.positions[bt] / p.interp;
#pragma unroll
    for (int i = 0; i < FPL; ++i) {
      const int f = FPL * lane + i;
      cl[i] = 1.f;
      sl[i] = 0.f;
      if (f < H2) {
        double sd, cd;
        sincos(pos * inv_freq_s[f], &sd, &cd);
        cl[i] = (float)cd;
        sl[i] = (float)sd;
        if (p.rope_table != nullptr) p.rope_table[(size_t)bt * H2 + f] = make_float2(cl[i], sl[i]);
      }
    }
    // This lane's features d1 + e (and their partners) use angle d1 + e, held by
    // lane (d1 + e) / FPL in slot e % FPL (d1 is a multiple of 8).
    float c[8], s[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      c[e] = __shfl_sync(0xffffffffu, cl[e % FPL], (d1 + e) / FPL);
      s[e] = __shfl_sync(0xffffffffu, sl[e % FPL], (d1 + e) / FPL);
    }
    if (lane == 0) {
      // Visible interval of token ta (whole-sequence index), as key rows from
      // key_base: the causal window (or [0, ta] on a global layer) joined with
      // the token's image span, which is contiguous because both contain ta.
      const int b = bt / p.S, t = bt % p.S;
      const int ta = p.start + t;
      int lo = (p.kind == 1) ? 0 : max(0, ta - p.window + 1);
      int hi = ta;
      const int32_t* sp = p.spans + (size_t)b * p.n_spans * 2;
      for (int k = 0; k < p.n_spans; ++k) {
        const int st = sp[2 * k], en = sp[2 * k + 1];
        if (st <= ta && ta < en) {
          lo = min(lo, max(st, 0));
          hi = max(hi, min(en, p.total) - 1);
          break;
        }
      }
      p.lo[bt] = lo - p.key_base;
      p.hi[bt] = hi - p.key_base;
      // A filled cache is read back by decode, which rotates each new token by
      // its index: keys cached here must have been rotated by theirs.
      if (p.k_cache != nullptr && p.positions[bt] != ta) record_error(p.err, kErrInvalid, 101);
      if (t == 0 && p.n_spans > 0) {
        // Sorted, disjoint, inside the sequence, and (chunked prefill) not
        // holding tokens on both sides of the chunk's first or last boundary.
        int prev_end = 0;
        bool ok = true;
        for (int k = 0; k < p.n_spans; ++k) {
          const int st = sp[2 * k], en = sp[2 * k + 1];
          ok = ok && st >= prev_end && st < en && en <= p.total;
          ok = ok && !(st < p.start && en > p.start) && !(st < p.total && en > p.total);
          prev_end = en;
        }
        if (!ok) record_error(p.err, kErrInvalid, 100);
      }
    }
    const __nv_bfloat16* qrow = p.q + (size_t)bt * p.Hq * D;
    const __nv_bfloat16* krow = p.k + (size_t)bt * p.Hkv * D;

    for (int h0 = 0; h0 < heads; h0 += RPW * kRowUnroll) {
      uint4 xa[kRowUnroll], xb[kRowUnroll];
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) {
        const int h = h0 + u * RPW + sub;
        if (h < heads) {
          const __nv_bfloat16* src = h < p.Hq ? qrow + h * D : krow + (h - p.Hq) * D;
          xa[u] = __ldg(reinterpret_cast<const uint4*>(src + d1));
          xb[u] = __ldg(reinterpret_cast<const uint4*>(src + H2 + d1));
        } else {
          xa[u] = xb[u] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int u = 0; u < kRowUnroll; ++u) {
        float x[16];
        unpack4_bf16(make_uint2(xa[u].x, xa[u].y), x);
        unpack4_bf16(make_uint2(xa[u].z, xa[u].w), x + 4);
        unpack4_bf16(make_uint2(xb[u].x, xb[u].y), x + 8);
        unpack4_bf16(make_uint2(xb[u].z, xb[u].w), x + 12);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const int h = h0 + u * RPW + sub;
        if (h >= heads) continue;
        const bool is_q = h < p.Hq;
        const float rinv = rsqrtf(ss * (1.0f / D) + 1e-6f);
        const float* gs = gam + (is_q ? 0 : D);
        float g[16];
        *reinterpret_cast<float4*>(g) = *reinterpret_cast<const float4*>(gs + d1);
        *reinterpret_cast<float4*>(g + 4) = *reinterpret_cast<const float4*>(gs + d1 + 4);
        *reinterpret_cast<float4*>(g + 8) = *reinterpret_cast<const float4*>(gs + H2 + d1);
        *reinterpret_cast<float4*>(g + 12) = *reinterpret_cast<const float4*>(gs + H2 + d1 + 4);
        float o[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float y1 = x[e] * rinv * g[e];
          const float y2 = x[8 + e] * rinv * g[8 + e];
          o[e] = y1 * c[e] - y2 * s[e];
          o[8 + e] = y1 * s[e] + y2 * c[e];
        }
        const uint2 a0 = pack4_bf16(o), a1 = pack4_bf16(o + 4), b0 = pack4_bf16(o + 8), b1 = pack4_bf16(o + 12);
        const uint4 lo8 = make_uint4(a0.x, a0.y, a1.x, a1.y), hi8 = make_uint4(b0.x, b0.y, b1.x, b1.y);
        if (is_q) {
          __nv_bfloat16* dst = p.q_hat + ((size_t)bt * p.Hq + h) * D;
          *reinterpret_cast<uint4*>(dst + d1) = lo8;
          *reinterpret_cast<uint4*>(dst + H2 + d1) = hi8;
        } else {
          const int kh = h - p.Hq;
          const size_t row = (size_t)bt * p.Hkv + kh;
          if (p.k_hat != nullptr) {
            __nv_bfloat16* dst = p.k_hat + row * D;
            *reinterpret_cast<uint4*>(dst + d1) = lo8;
            *reinterpret_cast<uint4*>(dst + H2 + d1) = hi8;
          }
          if (p.k_cache != nullptr) {
            const int b = bt / p.S, t = bt % p.S;
            const bool write =
                p.fill_rows || ((p.kind == 1) ? (t < p.cache_cap) : (t >= p.S - p.cache_cap));
            if (write) {
              const int slot = p.fill_rows ? p.start + t - p.key_base : (p.kind == 1) ? t : t % p.cache_cap;
              const size_t crow = ((size_t)b * p.Hkv + kh) * p.cache_cap + slot;
              *reinterpret_cast<uint4*>(p.k_cache + crow * D + d1) = lo8;
              *reinterpret_cast<uint4*>(p.k_cache + crow * D + H2 + d1) = hi8;
              const __nv_bfloat16* vsrc = p.v + row * D;
              *reinterpret_cast<uint4*>(p.v_cache + crow * D + d1) = __ldg(reinterpret_cast<const uint4*>(vsrc + d1));
              *reinterpret_cast<uint4*>(p.v_cache + crow * D + H2 + d1) =
                  __ldg(reinterpret_cast<const uint4*>(vsrc + H2 + d1));
            }
          }
        }
      }
    }
  }
}

// The call's device-error reset: lets its dependent (the prologue) launch at
// once, waits for the previous work in the stream (which may still record an
// error in this workspace), then clears the error word and its site.
__global__ void error_reset_kernel(int* err) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  griddep_wait();
  if (threadIdx.x == 0) {
    err[0] = 0;
    err[1] = 0;
  }
}

cudaError_t launch_error_reset(int* err, cudaStream_t st) {
  return launch_dependent(error_reset_kernel, dim3(1), dim3(32), 0, st, err);
}

cudaError_t launch_prefill_prologue(const PrologueParams& p, int D, cudaStream_t st) {
  const long long tokens = (long long)p.B * p.S;
  long long blocks = (tokens + (kRowThreads / 32) - 1) / (kRowThreads / 32);
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (D == 128) {
    return launch_dependent(qk_norm_rope_kernel<128>, dim3((unsigned)blocks), dim3(kRowThreads), 0, st, p);
  } else if (D == 64) {
    return launch_dependent(qk_norm_rope_kernel<64>, dim3((unsigned)blocks), dim3(kRowThreads), 0, st, p);
  } else if (D == 256) {
    return launch_dependent(qk_norm_rope_kernel<256>, dim3((unsigned)blocks), dim3(kRowThreads), 0, st, p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ======================================================= ring copies (local chunks)
// One thread per 16 bytes of a row; rows are (sequence, kv head, token).
constexpr int kRingThreads = 256;

template <int D, bool WRITE_BACK>
__global__ void __launch_bounds__(kRingThreads) ring_copy_kernel(RingCopyParams p) {
  constexpr int V16 = D / 8;  // 16-byte pieces per row
  const int n_tok = WRITE_BACK ? min(p.C, p.W) : p.hist;
  const size_t total = (size_t)p.B * p.Hkv * n_tok * V16;
  for (size_t i = (size_t)blockIdx.x * kRingThreads + threadIdx.x; i < total; i += (size_t)gridDim.x * kRingThreads) {
    const int v = (int)(i % V16);
    const size_t r = i / V16;
    const int j = (int)(r % n_tok);
    const size_t bh = r / n_tok;  // b * Hkv + kv head
    // Token of this row (whole-sequence index) and its ring slot / buffer row.
    const int tok = WRITE_BACK ? p.start + (p.C - n_tok) + j : p.key_base + j;
    const int ctx_row = tok - p.key_base;
    const size_t ring = (bh * p.W + (tok % p.W)) * V16 + v;
    const size_t ctx = (bh * p.rows + ctx_row) * V16 + v;
    uint4* rk = reinterpret_cast<uint4*>(p.ring_k);
    uint4* rv = reinterpret_cast<uint4*>(p.ring_v);
    uint4* ck = reinterpret_cast<uint4*>(p.ctx_k);
    uint4* cv = reinterpret_cast<uint4*>(p.ctx_v);
    if (WRITE_BACK) {
      rk[ring] = ck[ctx];
      rv[ring] = cv[ctx];
    } else {
      ck[ctx] = rk[ring];
      cv[ctx] = rv[ring];
    }
  }
}

template <bool WB>
static cudaError_t launch_ring_t(const RingCopyParams& p, int D, cudaStream_t st) {
  const long long n_tok = WB ? std::min(p.C, p.W) : p.hist;
  const long long work = (long long)p.B * p.Hkv * n_tok * (D / 8);
  if (work == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)std::min<long long>((work + kRingThreads - 1) / kRingThreads, 148 * 16);
  if (D == 128)
    ring_copy_kernel<128, WB><<<blocks, kRingThreads, 0, st>>>(p);
  else if (D == 64)
    ring_copy_kernel<64, WB><<<blocks, kRingThreads, 0, st>>>(p);
  else if (D == 256)
    ring_copy_kernel<256, WB><<<blocks, kRingThreads, 0, st>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_ring_gather(const RingCopyParams& p, int D, cudaStream_t st) { return launch_ring_t<false>(p, D, st); }
cudaError_t launch_ring_write_back(const RingCopyParams& p, int D, cudaStream_t st) {
  return launch_ring_t<true>(p, D, st);
}

}  // namespace g3
