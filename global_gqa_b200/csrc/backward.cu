// Prefill backward of one attention call of the Gemma 3 block on sm_100a:
// gradients of a loss with respect to the raw q, k, v and the two QK-norm
// gains, given dout = dLoss/dout and the forward's out and lse.
//
// The Gemma 3 Technical Report trains these layers (section 2.2 "Pre-training",
// distillation; section 2.3 "Quantization Aware Training"); the forward steps
// are QK-norm and RoPE (section 2 "Model Architecture", "Long context"), the
// 5:1 local/global mask with bidirectional image spans (sections 1 and 2;
// "Gemma explained: what's new in Gemma 3", section "Vision encoder and
// processing") and grouped-query attention.  Backward, per query head:
//
//   P_ij   = exp(q^_i . k^_j / sqrt(D) - lse_i)       (0 off the visible set)
//   delta_i = dout_i . out_i  (= sum_j P_ij dP_ij)
//   dP_ij  = dout_i . v_j,   dS_ij = P_ij (dP_ij - delta_i)
//   dv_j  += sum_i P_ij dout_i,  dk^_j += sum_i dS_ij q^_i / sqrt(D),
//   dq^_i  = sum_j dS_ij k^_j / sqrt(D)
//
// then the inverse rotation of RoPE and the RMSNorm chain rule.
//
// Launches:
//   bwd_prep      : delta and lse in log2 units per (row, head), padded to whole
//                   tiles; each row's visible interval; the range of query
//                   tiles that see each key tile.
//   bwd_dkdv      : one CTA per (sequence, kv head, 128-key tile), looping over
//                   every (query tile, query head of the group) that sees the
//                   tile: S^T = K Q^T and dP^T = V dO^T on the tensor cores,
//                   P^T and dS^T back into tensor memory as bf16, then
//                   dV += P^T dO and dK += dS^T Q with accumulators in tensor
//                   memory for the whole loop.
//   bwd_dq        : one CTA per (sequence, query head, 128-row query tile),
//                   looping over the key tiles it sees: S = Q K^T,
//                   dP = dO V^T, dS into tensor memory, dQ += dS K.
//   bwd_norm_rope : per (token, head) row, the inverse rotation and the
//                   RMSNorm chain rule; per-block partial gain gradients,
//                   then a fixed-order sum (deterministic).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "backward_common.cuh"
#include "func_attr.cuh"
#include "g3_internal.h"
#include "sm100_ptx.cuh"
#include "tmem_wide.cuh"

namespace g3 {

namespace {
constexpr int kPrepThreads = 256;
constexpr int kNormThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}
}  // namespace

// ================================================================ bwd_prep
// Rows of out and dout taken as chunks of consecutive tokens of one (sequence,
// head): LPR lanes per row, 16-byte loads, kPrepUnroll row steps in flight per
// warp.  Padding rows, the row intervals (colmask) and the key-tile ranges are
// grid-stride loops of their own.
constexpr int kPrepUnroll = 4;

template <int D>
__global__ void __launch_bounds__(kPrepThreads) bwd_prep_kernel(BwdParams p) {
  constexpr int LPR = D / 8;  // lanes per row, 8 features each
  constexpr int RPW = 32 / LPR;
  const long long gtid = (long long)blockIdx.x * kPrepThreads + threadIdx.x;
  const long long nthr = (long long)gridDim.x * kPrepThreads;

  // Query tiles that see key tile kt: rows i with hi_i >= j0 and lo_i <= j1.
  // Both ends are non-decreasing in i, so these rows are contiguous; row j0
  // itself is one of them.
  for (long long i = gtid; i < (long long)p.B * p.n_kvtiles; i += nthr) {
    const int b = (int)(i / p.n_kvtiles), kt = (int)(i % p.n_kvtiles);
    const int j0 = kt * kTileRows, j1 = min(j0 + kTileRows - 1, p.S - 1);
    const int32_t* lo = p.lo + (size_t)b * p.S;
    const int32_t* hi = p.hi + (size_t)b * p.S;
    int l = 0, r = j0;  // first i with hi_i >= j0 (hi_{j0} >= j0)
    while (l < r) {
      const int m = (l + r) >> 1;
      if (hi[m] >= j0) r = m; else l = m + 1;
    }
    const int i_min = l;
    l = j1;
    r = p.S - 1;  // last i with lo_i <= j1 (lo_{j1} <= j1)
    while (l < r) {
      const int m = (l + r + 1) >> 1;
      if (lo[m] <= j1) l = m; else r = m - 1;
    }
    p.kvrange[i] = make_int2(i_min / kTileRows, l / kTileRows);
  }
  // Row intervals padded to whole tiles (padding rows see nothing).
  for (long long i = gtid; i < (long long)p.B * p.S_pad; i += nthr) {
    const int b = (int)(i / p.S_pad), t = (int)(i % p.S_pad);
    const size_t src = (size_t)b * p.S + t;
    p.colmask[i] = t < p.S ? make_int2(p.lo[src], p.hi[src]) : make_int2(0x3fffffff, -1);
  }
  // Padding rows of lse2 / delta: P is exactly 0 there.
  const int pad = p.S_pad - p.S;
  for (long long i = gtid; i < (long long)p.B * p.Hq * pad; i += nthr) {
    const long long bh = i / pad;
    const size_t idx = (size_t)bh * p.S_pad + p.S + (int)(i % pad);
    p.lse2[idx] = INFINITY;
    p.delta[idx] = 0.f;
  }

  // Rows in (sequence, head, token) order, token fastest: lse reads and the
  // lse2 / delta writes are contiguous; each row of out / dout is 2D bytes.
  // A warp takes a chunk of RPW x kPrepUnroll consecutive tokens of one
  // (sequence, head).
  constexpr int kChunk = RPW * kPrepUnroll;
  const int lane = threadIdx.x & 31, li = lane % LPR, sub = lane / LPR;
  const int chunks_per_bh = (p.S + kChunk - 1) / kChunk;
  const long long n_chunks = (long long)p.B * p.Hq * chunks_per_bh;
  const long long warp_g = gtid >> 5, n_warps = nthr >> 5;
  for (long long c = warp_g; c < n_chunks; c += n_warps) {
    const int bh = (int)(c / chunks_per_bh);
    const int t0 = (int)(c - (long long)bh * chunks_per_bh) * kChunk;
    const int b = bh / p.Hq, h = bh - b * p.Hq;
    uint4 o[kPrepUnroll], g[kPrepUnroll];
    float l[kPrepUnroll];
#pragma unroll
    for (int u = 0; u < kPrepUnroll; ++u) {
      const int t = t0 + u * RPW + sub;
      if (t < p.S) {
        const size_t src = ((size_t)(b * p.S + t) * p.Hq + h) * D;
        o[u] = __ldg(reinterpret_cast<const uint4*>(p.out + src) + li);
        g[u] = __ldg(reinterpret_cast<const uint4*>(p.dout + src) + li);
        l[u] = li == 0 ? __ldg(p.lse + (size_t)bh * p.S + t) : 0.f;
      } else {
        o[u] = g[u] = make_uint4(0u, 0u, 0u, 0u);
        l[u] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kPrepUnroll; ++u) {
      float a[8], e8[8];
      bf16x8_to_f32(o[u], a);
      bf16x8_to_f32(g[u], e8);
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) d = fmaf(a[e], e8[e], d);
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      const int t = t0 + u * RPW + sub;
      if (li == 0 && t < p.S) {
        const size_t idx = (size_t)bh * p.S_pad + t;
        p.lse2[idx] = l[u] * kLog2e;
        p.delta[idx] = d;
      }
    }
  }
}

cudaError_t launch_bwd_prep(const BwdParams& p, int D, cudaStream_t st) {
  const long long rows = (long long)p.B * p.S * p.Hq;
  const int rpw = 32 / (D / 8);
  long long blocks = (rows + (long long)rpw * kPrepUnroll * 8 - 1) / ((long long)rpw * kPrepUnroll * 8);
  if (blocks > 148LL * 8) blocks = 148LL * 8;
  if (blocks < 1) blocks = 1;
  switch (D) {
    case 64: bwd_prep_kernel<64><<<(unsigned)blocks, kPrepThreads, 0, st>>>(p); break;
    case 128: bwd_prep_kernel<128><<<(unsigned)blocks, kPrepThreads, 0, st>>>(p); break;
    case 256: bwd_prep_kernel<256><<<(unsigned)blocks, kPrepThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// =========================================================== bwd_norm_rope
// One warp per token; lane li of a row holds features d1 .. d1+7 and
// D/2+d1 .. D/2+d1+7 (rotation partners together), as in the forward pass.
// The first n_norm_q_blocks blocks take the query rows, the others the key
// rows, so each lane accumulates the gradient of one gain only; kNormUnroll
// row steps are in flight per warp.
constexpr int kNormUnroll = 2;

template <int D>
__global__ void __launch_bounds__(kNormThreads, 2) bwd_norm_rope_kernel(BwdParams p) {
  constexpr int H2 = D / 2;
  constexpr int LPR = D / 16;
  constexpr int RPW = 32 / LPR;
  constexpr int NW = kNormThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int li = lane % LPR, sub = lane / LPR;
  const int d1 = li * 8;
  const bool is_q = (int)blockIdx.x < p.n_norm_q_blocks;
  const int blk = is_q ? (int)blockIdx.x : (int)blockIdx.x - p.n_norm_q_blocks;
  const int n_blk = is_q ? p.n_norm_q_blocks : p.n_norm_blocks - p.n_norm_q_blocks;
  const int heads = is_q ? p.Hq : p.Hkv;
  const __nv_bfloat16* xsrc = is_q ? p.q : p.k;
  const float* gsrc = is_q ? p.dq_hat : p.dk_hat;
  __nv_bfloat16* dst = is_q ? p.dq : p.dk;
  const int n_tokens = p.B * p.S;
  __shared__ __align__(16) float gam[D];
  __shared__ float red[NW][D];
  for (int i = threadIdx.x; i < D; i += kNormThreads) gam[i] = is_q ? p.q_gamma[i] : p.k_gamma[i];
  __syncthreads();
  float gv[16];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    gv[e] = gam[d1 + e];
    gv[8 + e] = gam[H2 + d1 + e];
  }

  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;

  for (int bt = blk * NW + warp; bt < n_tokens; bt += n_blk * NW) {
    const float4* tab = reinterpret_cast<const float4*>(p.rope_table + (size_t)bt * H2 + d1);
    float c[8], s[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = __ldg(tab + i);
      c[2 * i] = v.x;
      s[2 * i] = v.y;
      c[2 * i + 1] = v.z;
      s[2 * i + 1] = v.w;
    }
    for (int h0 = 0; h0 < heads; h0 += RPW * kNormUnroll) {
      uint4 xa[kNormUnroll], xb[kNormUnroll];
      float4 ga[kNormUnroll][2], gb[kNormUnroll][2];
#pragma unroll
      for (int u = 0; u < kNormUnroll; ++u) {
        const int h = h0 + u * RPW + sub;
        if (h < heads) {
          const size_t row = (size_t)bt * heads + h;
          xa[u] = __ldg(reinterpret_cast<const uint4*>(xsrc + row * D + d1));
          xb[u] = __ldg(reinterpret_cast<const uint4*>(xsrc + row * D + H2 + d1));
          ga[u][0] = __ldg(reinterpret_cast<const float4*>(gsrc + row * D + d1));
          ga[u][1] = __ldg(reinterpret_cast<const float4*>(gsrc + row * D + d1) + 1);
          gb[u][0] = __ldg(reinterpret_cast<const float4*>(gsrc + row * D + H2 + d1));
          gb[u][1] = __ldg(reinterpret_cast<const float4*>(gsrc + row * D + H2 + d1) + 1);
        } else {
          xa[u] = xb[u] = make_uint4(0u, 0u, 0u, 0u);
          ga[u][0] = ga[u][1] = gb[u][0] = gb[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < kNormUnroll; ++u) {
        const int h = h0 + u * RPW + sub;
        float x[16], g[16];
        bf16x8_to_f32(xa[u], x);
        bf16x8_to_f32(xb[u], x + 8);
        *reinterpret_cast<float4*>(g) = ga[u][0];
        *reinterpret_cast<float4*>(g + 4) = ga[u][1];
        *reinterpret_cast<float4*>(g + 8) = gb[u][0];
        *reinterpret_cast<float4*>(g + 12) = gb[u][1];
        // Inverse rotation: the gradient of y = R(theta) x is R(theta)^T dy.
        float gt[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          gt[e] = g[e] * c[e] + g[8 + e] * s[e];
          gt[8 + e] = g[8 + e] * c[e] - g[e] * s[e];
        }
        float ss = 0.f, inner = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          ss = fmaf(x[e], x[e], ss);
          inner = fmaf(gv[e] * gt[e], x[e], inner);
        }
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) {
          ss += __shfl_xor_sync(0xffffffffu, ss, off);
          inner += __shfl_xor_sync(0xffffffffu, inner, off);
        }
        if (h >= heads) continue;
        // y = x r gamma, r = (mean x^2 + eps)^(-1/2), as in the forward pass.
        const float r = rsqrtf(ss * (1.0f / D) + 1e-6f);
        const float t3 = r * r * r * inner * (1.0f / D);
        float dx[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          dx[e] = r * gv[e] * gt[e] - x[e] * t3;
          acc[e] = fmaf(gt[e] * r, x[e], acc[e]);
        }
        __nv_bfloat16* o = dst + ((size_t)bt * heads + h) * D;
        *reinterpret_cast<uint4*>(o + d1) = make_uint4(pack_bf16x2(dx[0], dx[1]), pack_bf16x2(dx[2], dx[3]),
                                                       pack_bf16x2(dx[4], dx[5]), pack_bf16x2(dx[6], dx[7]));
        *reinterpret_cast<uint4*>(o + H2 + d1) =
            make_uint4(pack_bf16x2(dx[8], dx[9]), pack_bf16x2(dx[10], dx[11]), pack_bf16x2(dx[12], dx[13]),
                       pack_bf16x2(dx[14], dx[15]));
      }
    }
  }
  // Gain: lanes with the same features (same li) combine, then the warps in a
  // fixed order; one partial row per block (the other gain's row is zero).
#pragma unroll
  for (int e = 0; e < 16; ++e) {
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
  }
  if (sub == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red[warp][d1 + e] = acc[e];
      red[warp][H2 + d1 + e] = acc[8 + e];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 2 * D; i += kNormThreads) {
    float sum = 0.f;
    if ((i < D) == is_q) {
#pragma unroll
      for (int w = 0; w < NW; ++w) sum += red[w][i % D];
    }
    p.gamma_part[(size_t)blockIdx.x * 2 * D + i] = sum;
  }
}

// Sum of the per-block partials: one CTA per 32 columns; warp w sums blocks
// w, w + 8, ... in eight interleaved partial sums (loads in flight), then the
// eight warps' sums are added in warp order.  The order is fixed, so repeated
// calls give identical results.
constexpr int kGammaWarps = 8;
__global__ void __launch_bounds__(kGammaWarps * 32) bwd_gamma_reduce_kernel(BwdParams p, int D) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i = blockIdx.x * 32 + lane;  // column of the [2, D] partial row
  __shared__ float part[kGammaWarps][32];
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
  if (i < 2 * D) {
    for (int blk0 = warp; blk0 < p.n_norm_blocks; blk0 += 8 * kGammaWarps) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int blk = blk0 + k * kGammaWarps;
        if (blk < p.n_norm_blocks) acc[k] += p.gamma_part[(size_t)blk * 2 * D + i];
      }
    }
  }
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) sum += acc[k];
  part[warp][lane] = sum;
  __syncthreads();
  if (warp == 0 && i < 2 * D) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kGammaWarps; ++w) tot += part[w][lane];
    if (i < D) p.dq_gamma[i] = tot;
    else p.dk_gamma[i - D] = tot;
  }
}

cudaError_t launch_bwd_norm_rope(const BwdParams& p, int D, cudaStream_t st) {
  if (p.n_norm_blocks < 2 || p.n_norm_blocks > kNormBwdMaxBlocks || p.n_norm_q_blocks < 1 ||
      p.n_norm_q_blocks >= p.n_norm_blocks)
    return cudaErrorInvalidValue;
  switch (D) {
    case 64: bwd_norm_rope_kernel<64><<<p.n_norm_blocks, kNormThreads, 0, st>>>(p); break;
    case 128: bwd_norm_rope_kernel<128><<<p.n_norm_blocks, kNormThreads, 0, st>>>(p); break;
    case 256: bwd_norm_rope_kernel<256><<<p.n_norm_blocks, kNormThreads, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bwd_gamma_reduce_kernel<<<(2 * D + 31) / 32, kGammaWarps * 32, 0, st>>>(p, D);
  return cudaGetLastError();
}

// ================================================================ bwd_dkdv
// The thread layout (backward_common.cuh) with 128-column tiles: each warp
// covers 16 rows x 64 columns; thread t holds columns 64h + 8k + 2(t%4) +
// {0,1}, k < 8, of its half h.

// The bf16 tile a column half packs (P^T, dS^T, dS) goes over the first 32 of
// its own 64 fp32 columns, so no warp overwrites columns another warp has yet
// to read: the 16-column (8 TMEM column) chunk kk of the 128 packed columns
// sits at TMEM column 8 kk + 32 (kk / 4).
__host__ __device__ constexpr uint32_t bf16_chunk_col(int kk) { return 8 * kk + 32 * (kk / 4); }

// Loads this thread's D/2 columns (half h) of a TMEM accumulator of D columns.
template <int D>
__device__ __forceinline__ void tmem_ld_half(uint32_t taddr, float* v) {
  if constexpr (D == 128) tmem_ld_16x256b_x8(taddr, v);
  else tmem_ld_16x256b_x4(taddr, v);
}

constexpr int kBwdMaxStages = 4;
struct BwdBarriers {
  uint64_t kv_full;
  uint64_t q_ready;  // bwd_dq: Q and dO are in tensor memory
  // A stage's tiles land on two barriers: full (Q and the side data, or K)
  // and full2 (dO, or V), so the first product waits for half of the stage.
  uint64_t full[kBwdMaxStages], full2[kBwdMaxStages], empty[kBwdMaxStages];
  uint64_t s_full, dp_full, p_full, ds_full, s_free, o_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
struct DkdvLayout {
  static constexpr int kStages = (D == 64) ? 3 : 2;
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kSide = 2 * 128 * 8;  // lse2, delta, then (lo, hi) of the stage's 128 query rows
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTile;
  static constexpr int kStage0 = kV + kTile;
  static constexpr int kStageBytes = 2 * kTile + kSide;  // Q, dO, side data
  static constexpr int kBar = kStage0 + kStages * kStageBytes;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

// TMEM columns: S^T (P^T as bf16 over it) at 0, dP^T (dS^T) at 128, dV at
// 256, dK at 256 + D.  Per item n the MMA thread issues dV(n) once P^T is
// stored, then S^T(n+1) (after the dV that read P^T), then dK(n) once dS^T
// is stored, then dP^T(n+1): the exponentials of item n+1 start while dK(n)
// and dP^T(n+1) run.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, BwdParams p) {
  using L = DkdvLayout<D>;
  constexpr int NS = L::kStages;
  static_assert(NS <= kBwdMaxStages && sizeof(BwdBarriers) <= L::kBytes - L::kBar, "barrier block");
  constexpr int KB = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + L::kBar);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Work item: key tiles in ascending order (on a global layer the first key
  // tiles are seen by the most query tiles).
  const int per_tile = p.B * p.Hkv;
  const int kt = (int)(blockIdx.x / per_tile);
  const int rem = (int)(blockIdx.x % per_tile);
  const int kvh = rem % p.Hkv, b = rem / p.Hkv;
  const int j0 = kt * kTileRows;
  const int2 qr = p.kvrange[(size_t)b * p.n_kvtiles + kt];
  // Items (query tile, query head of the group), query tiles in descending
  // order: the CTAs of neighbouring key tiles then stream the same query tiles
  // at the same time and share them in L2.
  const int n_items = (qr.y - qr.x + 1) * p.G;
  const int n_pre = min(n_items, NS);

  auto stage_ptr = [&](int s) { return smem + L::kStage0 + s * L::kStageBytes; };
  auto issue_stage = [&](int n) {
    const int s = n % NS;
    const int h = kvh * p.G + n % p.G;
    const int q0 = (qr.y - n / p.G) * kTileRows;
    uint8_t* st = stage_ptr(s);
    mbar_arrive_expect_tx(&bars->full[s], L::kTile + L::kSide);
    for (int kb = 0; kb < KB; ++kb) tma_load_4d(st + kb * kBwdSwizzleBlock, &tm_q, &bars->full[s], kb * 64, h, q0, b);
    const size_t rq = ((size_t)b * p.Hq + h) * p.S_pad + q0;
    bulk_load(st + 2 * L::kTile, p.lse2 + rq, 512, &bars->full[s]);
    bulk_load(st + 2 * L::kTile + 512, p.delta + rq, 512, &bars->full[s]);
    bulk_load(st + 2 * L::kTile + 1024, p.colmask + (size_t)b * p.S_pad + q0, 1024, &bars->full[s]);
    mbar_arrive_expect_tx(&bars->full2[s], L::kTile);
    for (int kb = 0; kb < KB; ++kb)
      tma_load_4d(st + L::kTile + kb * kBwdSwizzleBlock, &tm_do, &bars->full2[s], kb * 64, h, q0, b);
  };

  if (tid == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->full2[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_full, kBwdEwThreads);
    mbar_init(&bars->ds_full, kBwdEwThreads);
    mbar_init(&bars->s_free, kBwdEwThreads);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_do);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    mbar_arrive_expect_tx(&bars->kv_full, 2 * L::kTile);
    for (int kb = 0; kb < KB; ++kb) {
      tma_load_4d(smem + L::kK + kb * kBwdSwizzleBlock, &tm_k, &bars->kv_full, kb * 64, kvh, j0, b);
      tma_load_4d(smem + L::kV + kb * kBwdSwizzleBlock, &tm_v, &bars->kv_full, kb * 64, kvh, j0, b);
    }
    for (int n = 0; n < n_pre; ++n) issue_stage(n);
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last[kBwdMaxStages] = {-1, -1, -1, -1};
      for (int n = 0; n < n_pre; ++n) last[n] = 0;
      for (int n = n_pre; n < n_items; ++n) {
        const int s = n % NS;
        const uint32_t ph = (n / NS) & 1;
        if (!mbar_wait(&bars->empty[s], ph ^ 1, abort, p.err, 40)) break;
        issue_stage(n);
        last[s] = ph;
      }
      volatile int no_abort = 0;
      for (int s = 0; s < NS; ++s)
        if (last[s] >= 0) {
          mbar_wait(&bars->full[s], last[s], &no_abort, p.err, 41);
          mbar_wait(&bars->full2[s], last[s], &no_abort, p.err, 41);
        }
      mbar_wait(&bars->kv_full, 0, &no_abort, p.err, 41);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t k_addr = smem_u32(smem + L::kK), v_addr = smem_u32(smem + L::kV);
      // X^T = A B^T over the D features: A = K or V (rows = keys), B = Q or dO.
      auto issue_t = [&](uint32_t a_addr, uint32_t b_addr, uint32_t col) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kBwdSwizzleBlock + (kk % 4) * 32;
          mma_ss(tmem + col, smem_desc_sw128(a_addr + off, 16, 1024), smem_desc_sw128(b_addr + off, 16, 1024),
                 idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // acc += A B over the 128 query rows: A = P^T or dS^T from TMEM, B = dO or Q.
      auto issue_acc = [&](uint32_t a_col, uint32_t b_addr, uint32_t d_col, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + d_col, tmem + a_col + bf16_chunk_col(kk),
                 smem_desc_sw128(b_addr + kk * 2048, kBwdSwizzleBlock, 1024), idesc_o, (acc || kk > 0) ? 1u : 0u);
      };
      auto q_addr = [&](int s) { return smem_u32(stage_ptr(s)); };
      auto do_addr = [&](int s) { return smem_u32(stage_ptr(s) + L::kTile); };

      bool ok = mbar_wait(&bars->kv_full, 0, abort, p.err, 42);
      if (ok) ok = mbar_wait(&bars->full[0], 0, abort, p.err, 43);
      if (ok) {
        tc_fence_after();
        issue_t(k_addr, q_addr(0), 0);
        mma_commit(&bars->s_full);
      }
      if (ok) ok = mbar_wait(&bars->full2[0], 0, abort, p.err, 43);
      if (ok) {
        tc_fence_after();
        issue_t(v_addr, do_addr(0), 128);
        mma_commit(&bars->dp_full);
      }
      for (int n = 0; ok && n < n_items; ++n) {
        const int s = n % NS, s1 = (n + 1) % NS;
        if (!(ok = mbar_wait(&bars->p_full, n & 1, abort, p.err, 44))) break;
        tc_fence_after();
        issue_acc(0, do_addr(s), 256, n > 0);  // dV += P^T dO
        const bool more = n + 1 < n_items;
        if (more) {
          if (!(ok = mbar_wait(&bars->full[s1], ((n + 1) / NS) & 1, abort, p.err, 45))) break;
          tc_fence_after();
          issue_t(k_addr, q_addr(s1), 0);  // next S^T (after the dV that read P^T)
          mma_commit(&bars->s_full);
        }
        if (!(ok = mbar_wait(&bars->ds_full, n & 1, abort, p.err, 46))) break;
        tc_fence_after();
        issue_acc(128, q_addr(s), 256 + D, n > 0);  // dK += dS^T Q
        mma_commit(&bars->empty[s]);
        if (more) {
          if (!(ok = mbar_wait(&bars->full2[s1], ((n + 1) / NS) & 1, abort, p.err, 48))) break;
          tc_fence_after();
          issue_t(v_addr, do_addr(s1), 128);  // next dP^T (after the dK that read dS^T)
          mma_commit(&bars->dp_full);
        }
      }
      if (ok) mma_commit(&bars->o_full);
      mma_commit(&bars->drain);
      volatile int no_abort = 0;
      mbar_wait(&bars->drain, 0, &no_abort, p.err, 47);
    }
  } else {
    // ------------------------------------------------------ P^T and dS^T
    const int lane_base = bwd_lane_base(warp), ch = bwd_col_half(warp);
    const int m4 = lane & 3;
    const int ra = lane_base + (lane >> 2), rb = ra + 8;
    const int ja = j0 + ra, jb = j0 + rb;  // key index of each of this thread's rows
    const uint32_t t_lane = tmem + ((uint32_t)lane_base << 16);
    const float sc = p.scale_log2;
    bool ok = true;
    for (int n = 0; n < n_items; ++n) {
      const int s = n % NS;
      const int q0 = (qr.y - n / p.G) * kTileRows;
      const int q_last = min(q0 + kTileRows - 1, p.S - 1);
      // Side data of the stage, per pair of query columns c0 = 64h + 8k + 2 m4, c0 + 1.
      const float2* l2 = reinterpret_cast<const float2*>(stage_ptr(s) + 2 * L::kTile) + 32 * ch;
      const float2* dl = reinterpret_cast<const float2*>(stage_ptr(s) + 2 * L::kTile + 512) + 32 * ch;
      const int2* cm2 = reinterpret_cast<const int2*>(stage_ptr(s) + 2 * L::kTile + 1024);
      const int4* cm = reinterpret_cast<const int4*>(cm2) + 32 * ch;  // (lo, hi) of two columns per int4
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->full[s], (n / NS) & 1, abort, p.err, 50));
      if (!ok) break;
      // Every query row of the tile sees every key of this tile: no mask.
      const bool full = cm2[q_last - q0].x <= j0 && cm2[0].y >= j0 + kTileRows - 1;
      float2 lv[8];  // read while S^T is still being computed
#pragma unroll
      for (int k = 0; k < 8; ++k) lv[k] = l2[4 * k + m4];
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, n & 1, abort, p.err, 51));
      if (!ok) break;
      tc_fence_after();
      float pv[32];
      tmem_ld_16x256b_x8(t_lane + 64 * ch, pv);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float x0 = fmaf(pv[4 * k], sc, -lv[k].x), x1 = fmaf(pv[4 * k + 1], sc, -lv[k].y);
        float x2 = fmaf(pv[4 * k + 2], sc, -lv[k].x), x3 = fmaf(pv[4 * k + 3], sc, -lv[k].y);
        if (!full) {
          const int4 c = cm[4 * k + m4];  // (lo, hi) of the two query columns
          if (ja < c.x || ja > c.y) x0 = -INFINITY;
          if (ja < c.z || ja > c.w) x1 = -INFINITY;
          if (jb < c.x || jb > c.y) x2 = -INFINITY;
          if (jb < c.z || jb > c.w) x3 = -INFINITY;
        }
        pv[4 * k] = ex2_approx(x0);
        pv[4 * k + 1] = ex2_approx(x1);
        pv[4 * k + 2] = ex2_approx(x2);
        pv[4 * k + 3] = ex2_approx(x3);
        pk[2 * k] = pack_bf16x2(pv[4 * k], pv[4 * k + 1]);
        pk[2 * k + 1] = pack_bf16x2(pv[4 * k + 2], pv[4 * k + 3]);
      }
      tmem_st_16x128b_x8(t_lane + 64 * ch, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full);

#pragma unroll
      for (int k = 0; k < 8; ++k) lv[k] = dl[4 * k + m4];  // delta of the two columns
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, n & 1, abort, p.err, 52));
      if (!ok) break;
      tc_fence_after();
      float dp[32];
      tmem_ld_16x256b_x8(t_lane + 128 + 64 * ch, dp);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        pk[2 * k] = pack_bf16x2(pv[4 * k] * (dp[4 * k] - lv[k].x), pv[4 * k + 1] * (dp[4 * k + 1] - lv[k].y));
        pk[2 * k + 1] = pack_bf16x2(pv[4 * k + 2] * (dp[4 * k + 2] - lv[k].x), pv[4 * k + 3] * (dp[4 * k + 3] - lv[k].y));
      }
      tmem_st_16x128b_x8(t_lane + 128 + 64 * ch, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort, p.err, 53));
    if (ok) {
      tc_fence_after();
      constexpr int HC = D / 2;  // accumulator columns of this warp
      const bool va = ja < p.S, vb = jb < p.S;
      __nv_bfloat16* dva = p.dv + ((size_t)(b * p.S + ja) * p.Hkv + kvh) * D + HC * ch;
      __nv_bfloat16* dvb = p.dv + ((size_t)(b * p.S + jb) * p.Hkv + kvh) * D + HC * ch;
      float* dka = p.dk_hat + ((size_t)(b * p.S + ja) * p.Hkv + kvh) * D + HC * ch;
      float* dkb = p.dk_hat + ((size_t)(b * p.S + jb) * p.Hkv + kvh) * D + HC * ch;
      float o[HC / 2];
      tmem_ld_half<D>(t_lane + 256 + HC * ch, o);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < HC / 8; ++k) {
        const int col = 8 * k + 2 * m4;
        if (va) *reinterpret_cast<uint32_t*>(dva + col) = pack_bf16x2(o[4 * k], o[4 * k + 1]);
        if (vb) *reinterpret_cast<uint32_t*>(dvb + col) = pack_bf16x2(o[4 * k + 2], o[4 * k + 3]);
      }
      tmem_ld_half<D>(t_lane + 256 + D + HC * ch, o);
      tmem_wait_ld();
      const float is = p.inv_sqrt_d;
#pragma unroll
      for (int k = 0; k < HC / 8; ++k) {
        const int col = 8 * k + 2 * m4;
        if (va) *reinterpret_cast<float2*>(dka + col) = make_float2(o[4 * k] * is, o[4 * k + 1] * is);
        if (vb) *reinterpret_cast<float2*>(dkb + col) = make_float2(o[4 * k + 2] * is, o[4 * k + 3] * is);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
static cudaError_t launch_dkdv_t(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tdo,
                                 const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  using L = DkdvLayout<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  static std::atomic<uint64_t> configured{0};  // devices with the shared-memory limit raised
  const cudaError_t e = ensure_dynamic_smem(bwd_dkdv_kernel<D>, L::kAlloc, configured);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)p.n_kvtiles * p.B * p.Hkv;
  bwd_dkdv_kernel<D><<<grid, kBwdThreads, L::kAlloc, st>>>(tq, tdo, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv(const BwdParams& p, int D, const CUtensorMap& tq, const CUtensorMap& tdo,
                            const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  if (D == 128) return launch_dkdv_t<128>(p, tq, tdo, tk, tv, st);
  if (D == 64) return launch_dkdv_t<64>(p, tq, tdo, tk, tv, st);
  return cudaErrorInvalidValue;
}

// ================================================================== bwd_dq
template <int D>
struct DqLayout {
  static constexpr int kStages = (D == 64) ? 4 : 3;
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kStage0 = 0;
  static constexpr int kStageBytes = 2 * kTile;  // K, V
  static constexpr int kBar = kStage0 + kStages * kStageBytes;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

// TMEM columns: S at 0, dP (dS as bf16 over it) at 128, dQ at 256, and the
// CTA's Q and dO tiles as bf16 pairs at 384 and 384 + D/2: S = Q K^T and
// dP = dO V^T read their A operand from tensor memory, so shared memory holds
// only the K/V ring (three stages at D = 128).  Per key tile t the MMA thread
// issues S(t+1) as soon as the elementwise warps have read S(t), then
// dQ += dS(t) K(t), then dP(t+1), so the exponentials of tile t+1 overlap the
// tensor-core work of tile t.
constexpr int kDqQCol = 384;
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, BwdParams p) {
  using L = DqLayout<D>;
  constexpr int NS = L::kStages;
  static_assert(NS <= kBwdMaxStages && sizeof(BwdBarriers) <= L::kBytes - L::kBar, "barrier block");
  constexpr int KB = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + L::kBar);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Work item: heaviest (last) query tiles first.
  const int per_tile = p.B * p.Hq;
  const int qt = p.n_qtiles - 1 - (int)(blockIdx.x / per_tile);
  const int rem = (int)(blockIdx.x % per_tile);
  const int h = rem % p.Hq, b = rem / p.Hq;
  const int kvh = h / p.G;
  const int r0 = qt * kTileRows;
  const int r_last = min(r0 + kTileRows - 1, p.S - 1);
  const size_t rowbase = (size_t)b * p.S;
  const int lo_first = p.lo[rowbase + r0], hi_last = p.hi[rowbase + r_last];
  const int lo_last = p.lo[rowbase + r_last], hi_first = p.hi[rowbase + r0];
  const int t_begin = lo_first / kTileRows;
  const int n_tiles = max(hi_last / kTileRows, t_begin) - t_begin + 1;
  const int n_pre = min(n_tiles, NS);

  auto stage_ptr = [&](int s) { return smem + L::kStage0 + s * L::kStageBytes; };
  auto issue_stage = [&](int t) {
    const int s = t % NS;
    const int kv0 = (t_begin + t) * kTileRows;
    mbar_arrive_expect_tx(&bars->full[s], L::kTile);
    for (int kb = 0; kb < KB; ++kb)
      tma_load_4d(stage_ptr(s) + kb * kBwdSwizzleBlock, &tm_k, &bars->full[s], kb * 64, kvh, kv0, b);
    mbar_arrive_expect_tx(&bars->full2[s], L::kTile);
    for (int kb = 0; kb < KB; ++kb)
      tma_load_4d(stage_ptr(s) + L::kTile + kb * kBwdSwizzleBlock, &tm_v, &bars->full2[s], kb * 64, kvh, kv0, b);
  };

  // Q and dO into tensor memory: unit u (32 columns = 64 features of Q or
  // dO) is written by the elementwise warps with u = e >> 2, one row per
  // thread (the 32x32b shape), as the raw bf16 pairs of the row; rows past S
  // are zero.  The global loads start before the CTA-wide barrier.
  constexpr int kUnits = D / 32;
  const int q_unit = (warp - kBwdFirstWarp) >> 2;
  const bool q_writer = warp >= kBwdFirstWarp && q_unit < kUnits;
  const int q_row = (warp & 3) * 32 + lane;
  uint32_t qw[32];
  if (q_writer) {
    const int tensor = q_unit / (D / 64), cb = q_unit % (D / 64);
    if (r0 + q_row < p.S) {
      const __nv_bfloat16* src =
          (tensor == 0 ? p.q_hat : p.dout) + ((size_t)(b * p.S + r0 + q_row) * p.Hq + h) * D + cb * 64;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
        qw[4 * i] = v.x;
        qw[4 * i + 1] = v.y;
        qw[4 * i + 2] = v.z;
        qw[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) qw[i] = 0u;
    }
  }

  if (tid == 0) {
    mbar_init(&bars->q_ready, kBwdEwThreads);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->full2[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->p_full, kBwdEwThreads);
    mbar_init(&bars->ds_full, kBwdEwThreads);
    mbar_init(&bars->s_free, kBwdEwThreads);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    for (int t = 0; t < n_pre; ++t) issue_stage(t);
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last[kBwdMaxStages] = {-1, -1, -1, -1};
      for (int t = 0; t < n_pre; ++t) last[t] = 0;
      for (int t = n_pre; t < n_tiles; ++t) {
        const int s = t % NS;
        const uint32_t ph = (t / NS) & 1;
        if (!mbar_wait(&bars->empty[s], ph ^ 1, abort, p.err, 60)) break;
        issue_stage(t);
        last[s] = ph;
      }
      volatile int no_abort = 0;
      for (int s = 0; s < NS; ++s)
        if (last[s] >= 0) {
          mbar_wait(&bars->full[s], last[s], &no_abort, p.err, 61);
          mbar_wait(&bars->full2[s], last[s], &no_abort, p.err, 61);
        }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      constexpr uint32_t q_col = kDqQCol, do_col = kDqQCol + D / 2;
      // X = A B^T over the D features: A (Q or dO) from tensor memory, B (K or V) from shared memory.
      auto issue_x = [&](uint32_t a_col, uint32_t b_addr, uint32_t col) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kBwdSwizzleBlock + (kk % 4) * 32;
          mma_ts(tmem + col, tmem + a_col + kk * 8, smem_desc_sw128(b_addr + off, 16, 1024), idesc_s,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto k_addr = [&](int s) { return smem_u32(stage_ptr(s)); };
      auto v_addr = [&](int s) { return smem_u32(stage_ptr(s) + L::kTile); };

      bool ok = mbar_wait(&bars->q_ready, 0, abort, p.err, 62);
      if (ok) ok = mbar_wait(&bars->full[0], 0, abort, p.err, 63);
      if (ok) {
        tc_fence_after();
        issue_x(q_col, k_addr(0), 0);  // S = Q K^T
        mma_commit(&bars->s_full);
      }
      if (ok) ok = mbar_wait(&bars->full2[0], 0, abort, p.err, 63);
      if (ok) {
        tc_fence_after();
        issue_x(do_col, v_addr(0), 128);  // dP = dO V^T
        mma_commit(&bars->dp_full);
      }
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int s = t % NS, s1 = (t + 1) % NS;
        const bool more = t + 1 < n_tiles;
        if (more) {
          if (!(ok = mbar_wait(&bars->full[s1], ((t + 1) / NS) & 1, abort, p.err, 64))) break;
          if (!(ok = mbar_wait(&bars->s_free, t & 1, abort, p.err, 65))) break;
          tc_fence_after();
          issue_x(q_col, k_addr(s1), 0);
          mma_commit(&bars->s_full);
        }
        if (!(ok = mbar_wait(&bars->ds_full, t & 1, abort, p.err, 66))) break;
        tc_fence_after();
        // dQ += dS K: dS from TMEM (128 rows x 128 keys), K tile as [keys x D].
        const uint32_t kb_addr = k_addr(s);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + 256, tmem + 128 + bf16_chunk_col(kk),
                 smem_desc_sw128(kb_addr + kk * 2048, kBwdSwizzleBlock, 1024), idesc_o, (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars->empty[s]);
        if (more) {
          if (!(ok = mbar_wait(&bars->full2[s1], ((t + 1) / NS) & 1, abort, p.err, 68))) break;
          tc_fence_after();
          issue_x(do_col, v_addr(s1), 128);
          mma_commit(&bars->dp_full);
        }
      }
      if (ok) mma_commit(&bars->o_full);
      mma_commit(&bars->drain);
      volatile int no_abort = 0;
      mbar_wait(&bars->drain, 0, &no_abort, p.err, 67);
    }
  } else {
    // ------------------------------------------------------------ P and dS
    const int lane_base = bwd_lane_base(warp), ch = bwd_col_half(warp);
    const int m4 = lane & 3;
    const int ra = lane_base + (lane >> 2), rb = ra + 8;
    const bool valid_a = r0 + ra < p.S, valid_b = r0 + rb < p.S;
    const int lo_a = valid_a ? p.lo[rowbase + r0 + ra] : 1, hi_a = valid_a ? p.hi[rowbase + r0 + ra] : 0;
    const int lo_b = valid_b ? p.lo[rowbase + r0 + rb] : 1, hi_b = valid_b ? p.hi[rowbase + r0 + rb] : 0;
    const size_t rq = ((size_t)b * p.Hq + h) * p.S_pad + r0;  // padding rows: lse2 +inf, delta 0
    const float2 ria = make_float2(p.lse2[rq + ra], p.delta[rq + ra]);
    const float2 rib = make_float2(p.lse2[rq + rb], p.delta[rq + rb]);
    const uint32_t t_lane = tmem + ((uint32_t)lane_base << 16);
    const float sc = p.scale_log2;
    if (q_writer) {
      const int tensor = q_unit / (D / 64), cb = q_unit % (D / 64);
      tmem_st32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + kDqQCol + tensor * (D / 2) + cb * 32, qw);
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(&bars->q_ready);
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, t & 1, abort, p.err, 70));
      if (!ok) break;
      tc_fence_after();
      float pv[32];
      tmem_ld_16x256b_x8(t_lane + 64 * ch, pv);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_free);
      const int tile0 = (t_begin + t) * kTileRows;
      const bool full = tile0 >= lo_last && tile0 + kTileRows - 1 <= hi_first;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int col = tile0 + 64 * ch + 8 * k + 2 * m4;
        float x0 = fmaf(pv[4 * k], sc, -ria.x), x1 = fmaf(pv[4 * k + 1], sc, -ria.x);
        float x2 = fmaf(pv[4 * k + 2], sc, -rib.x), x3 = fmaf(pv[4 * k + 3], sc, -rib.x);
        if (!full) {
          if (col < lo_a || col > hi_a) x0 = -INFINITY;
          if (col + 1 < lo_a || col + 1 > hi_a) x1 = -INFINITY;
          if (col < lo_b || col > hi_b) x2 = -INFINITY;
          if (col + 1 < lo_b || col + 1 > hi_b) x3 = -INFINITY;
        }
        pv[4 * k] = ex2_approx(x0);
        pv[4 * k + 1] = ex2_approx(x1);
        pv[4 * k + 2] = ex2_approx(x2);
        pv[4 * k + 3] = ex2_approx(x3);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, t & 1, abort, p.err, 71));
      if (!ok) break;
      tc_fence_after();
      float dp[32];
      tmem_ld_16x256b_x8(t_lane + 128 + 64 * ch, dp);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        pk[2 * k] = pack_bf16x2(pv[4 * k] * (dp[4 * k] - ria.y), pv[4 * k + 1] * (dp[4 * k + 1] - ria.y));
        pk[2 * k + 1] = pack_bf16x2(pv[4 * k + 2] * (dp[4 * k + 2] - rib.y), pv[4 * k + 3] * (dp[4 * k + 3] - rib.y));
      }
      tmem_st_16x128b_x8(t_lane + 128 + 64 * ch, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort, p.err, 72));
    if (ok) {
      tc_fence_after();
      constexpr int HC = D / 2;
      float* dqa = p.dq_hat + ((size_t)(b * p.S + r0 + ra) * p.Hq + h) * D + HC * ch;
      float* dqb = p.dq_hat + ((size_t)(b * p.S + r0 + rb) * p.Hq + h) * D + HC * ch;
      float o[HC / 2];
      tmem_ld_half<D>(t_lane + 256 + HC * ch, o);
      tmem_wait_ld();
      const float is = p.inv_sqrt_d;
#pragma unroll
      for (int k = 0; k < HC / 8; ++k) {
        const int col = 8 * k + 2 * m4;
        if (valid_a) *reinterpret_cast<float2*>(dqa + col) = make_float2(o[4 * k] * is, o[4 * k + 1] * is);
        if (valid_b) *reinterpret_cast<float2*>(dqb + col) = make_float2(o[4 * k + 2] * is, o[4 * k + 3] * is);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
static cudaError_t launch_dq_t(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tdo,
                               const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  using L = DqLayout<D>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  static std::atomic<uint64_t> configured{0};  // devices with the shared-memory limit raised
  const cudaError_t e = ensure_dynamic_smem(bwd_dq_kernel<D>, L::kAlloc, configured);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)p.n_qtiles * p.B * p.Hq;
  bwd_dq_kernel<D><<<grid, kBwdThreads, L::kAlloc, st>>>(tq, tdo, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(const BwdParams& p, int D, const CUtensorMap& tq, const CUtensorMap& tdo,
                          const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  if (D == 128) return launch_dq_t<128>(p, tq, tdo, tk, tv, st);
  if (D == 64) return launch_dq_t<64>(p, tq, tdo, tk, tv, st);
  return cudaErrorInvalidValue;
}

}  // namespace g3
