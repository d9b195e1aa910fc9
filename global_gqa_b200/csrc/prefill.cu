// Prefill path of the Gemma 3 block attention on sm_100a.
//
//   prefill_prologue : QK-RMSNorm + RoPE of q and k (bf16 out), per-row visible
//                      key interval [lo, hi], optional KV-cache fill.
//   prefill_attention: warp-specialised flash attention.  TMA (no multicast)
//                      streams 128-row K/V tiles, one thread issues tcgen05.mma
//                      for S = Q K^T and O += P V with accumulators in tensor
//                      memory, and one warpgroup per query head of the GQA group
//                      runs the fp32 online softmax.  The KV tiles a query tile
//                      visits are exactly those its rows' visible intervals
//                      touch; tiles fully inside every row's interval skip the
//                      per-element mask.
//
// The visible set of row i is the single interval [lo_i, hi_i]: the causal
// window [max(0, i-W+1), i] (or [0, i] for a global layer) and the row's image
// span both contain i, so their union is contiguous, and both ends are
// non-decreasing in i (Gemma 3 Technical Report, sections 1 and 2; "Gemma
// explained", section "Vision encoder and processing").
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "g3_internal.h"
#include "sm100_ptx.cuh"

namespace g3 {

// ========================================================== prologue kernel
constexpr int kPrologueTokens = 4;     // tokens per block
constexpr int kPrologueThreads = 256;  // 8 warps

template <int D>
__global__ void __launch_bounds__(kPrologueThreads) prefill_prologue_kernel(PrologueParams p) {
  constexpr int H2 = D / 2;
  constexpr int PER = D / 64;  // elements per lane in each half of the head
  __shared__ float s_cos[kPrologueTokens][H2];
  __shared__ float s_sin[kPrologueTokens][H2];

  const int b = blockIdx.y;
  const int t0 = blockIdx.x * kPrologueTokens;
  const int tid = threadIdx.x;

  // Rotation angles in double: theta = (p / interp) * base^(-2f/D), then sin
  // and cos in double and rounded to fp32.
  for (int idx = tid; idx < kPrologueTokens * H2; idx += blockDim.x) {
    const int tt = idx / H2, f = idx % H2, t = t0 + tt;
    float c = 1.f, s = 0.f;
    if (t < p.S) {
      const double inv_freq = exp(-2.0 * f / D * log(p.rope_base));
      const double theta = (double)p.positions[(size_t)b * p.S + t] / p.interp * inv_freq;
      double sd, cd;
      sincos(theta, &sd, &cd);
      c = (float)cd;
      s = (float)sd;
    }
    s_cos[tt][f] = c;
    s_sin[tt][f] = s;
  }

  // Visible interval of each row of this block.
  if (tid < kPrologueTokens) {
    const int t = t0 + tid;
    if (t < p.S) {
      int lo = (p.kind == 1) ? 0 : max(0, t - p.window + 1);
      int hi = t;
      const int32_t* sp = p.spans + (size_t)b * p.n_spans * 2;
      for (int k = 0; k < p.n_spans; ++k) {
        const int st = sp[2 * k], en = sp[2 * k + 1];
        if (st <= t && t < en) {
          lo = min(lo, max(st, 0));
          hi = max(hi, min(en, p.S) - 1);
          break;
        }
      }
      p.lo[(size_t)b * p.S + t] = lo;
      p.hi[(size_t)b * p.S + t] = hi;
    }
  }
  // Span validation for this sequence (one thread of its first block).
  if (blockIdx.x == 0 && tid == 32 && p.n_spans > 0) {
    const int32_t* sp = p.spans + (size_t)b * p.n_spans * 2;
    int prev_end = 0;
    bool ok = true;
    for (int k = 0; k < p.n_spans; ++k) {
      const int st = sp[2 * k], en = sp[2 * k + 1];
      ok = ok && st >= prev_end && st < en && en <= p.S;
      prev_end = en;
    }
    if (!ok) record_error(p.err, kErrInvalid, 100);
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const int heads = p.Hq + p.Hkv;
  for (int r = warp; r < kPrologueTokens * heads; r += kPrologueThreads / 32) {
    const int tt = r / heads, h = r % heads, t = t0 + tt;
    if (t >= p.S) continue;
    const bool is_q = h < p.Hq;
    const int hh = is_q ? h : h - p.Hq;
    const int H = is_q ? p.Hq : p.Hkv;
    const size_t row = ((size_t)b * p.S + t) * H + hh;
    const __nv_bfloat16* src = (is_q ? p.q : p.k) + row * D;
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
    __nv_bfloat16* dst = (is_q ? p.q_hat : p.k_hat) + row * D;
    __nv_bfloat16 o1[PER], o2[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int d = lane * PER + e;
      const float y1 = x1[e] * rinv * gam[d];
      const float y2 = x2[e] * rinv * gam[d + H2];
      const float c = s_cos[tt][d], s = s_sin[tt][d];
      o1[e] = __float2bfloat16_rn(y1 * c - y2 * s);
      o2[e] = __float2bfloat16_rn(y1 * s + y2 * c);
      dst[d] = o1[e];
      dst[d + H2] = o2[e];
    }
    if (!is_q && p.k_cache != nullptr) {
      bool write;
      int slot;
      if (p.kind == 1) {
        write = t < p.cache_cap;
        slot = t;
      } else {
        write = t >= p.S - p.cache_cap;
        slot = t % p.cache_cap;
      }
      if (write) {
        const size_t crow = ((size_t)b * p.Hkv + hh) * p.cache_cap + slot;
        const __nv_bfloat16* vsrc = p.v + row * D;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          const int d = lane * PER + e;
          p.k_cache[crow * D + d] = o1[e];
          p.k_cache[crow * D + d + H2] = o2[e];
          p.v_cache[crow * D + d] = vsrc[d];
          p.v_cache[crow * D + d + H2] = vsrc[d + H2];
        }
      }
    }
  }
}

cudaError_t launch_prefill_prologue(const PrologueParams& p, int D, cudaStream_t st) {
  dim3 grid((p.S + kPrologueTokens - 1) / kPrologueTokens, p.B);
  if (D == 128) {
    prefill_prologue_kernel<128><<<grid, kPrologueThreads, 0, st>>>(p);
  } else if (D == 64) {
    prefill_prologue_kernel<64><<<grid, kPrologueThreads, 0, st>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ========================================================= attention kernel
// Warp roles (384 threads): warp 0 = TMA producer, warp 1 = MMA issuer and
// TMEM owner, warps 2-3 idle, warps 4-7 = softmax of head 0, warps 8-11 =
// softmax of head 1 (when two heads share the K/V tiles).
constexpr int kAttnThreads = 384;
constexpr int kSwizzleBlock = 128 * 64 * 2;  // 128 rows x 64 bf16 (one 128-byte swizzle column)

template <int D, int HPC>
struct AttnLayout {
  static constexpr int kStages = (D == 64) ? 3 : 2;
  static constexpr int kTile = 128 * D * 2;  // bytes of one 128-row tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + HPC * kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBar = kV + kStages * kTile;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr int kTmemCols = (HPC * (128 + D) <= 256) ? 256 : 512;
};

struct AttnBarriers {
  uint64_t q_full;
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2], p_full[2], o_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int D, int HPC>
__global__ void __launch_bounds__(kAttnThreads, 1)
    prefill_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, AttnParams p) {
  using L = AttnLayout<D, HPC>;
  constexpr int NS = L::kStages;
  constexpr int KB = D / 64;  // swizzle columns per tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnBarriers* bars = reinterpret_cast<AttnBarriers*>(smem + L::kBar);
  volatile int* abort = &bars->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item: heaviest (last) query tiles first
  const int per_tile = p.B * p.Hkv * p.n_groups;
  const int qt = p.n_qtiles - 1 - (int)(blockIdx.x / per_tile);
  int rem = (int)(blockIdx.x % per_tile);
  const int gp = rem % p.n_groups;
  rem /= p.n_groups;
  const int kvh = rem % p.Hkv;
  const int b = rem / p.Hkv;
  const int h0 = kvh * p.G + gp * HPC;
  const int r0 = qt * 128;
  const int r_last = min(r0 + 127, p.S - 1);

  const size_t rowbase = (size_t)b * p.S;
  const int lo_first = p.lo[rowbase + r0];
  const int hi_last = p.hi[rowbase + r_last];
  const int lo_last = p.lo[rowbase + r_last];  // largest lo of the tile's rows
  const int hi_first = p.hi[rowbase + r0];     // smallest hi of the tile's rows
  const int t_begin = lo_first / 128;
  const int n_tiles = max(hi_last / 128, t_begin) - t_begin + 1;

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int h = 0; h < HPC; ++h) {
      mbar_init(&bars->s_full[h], 1);
      mbar_init(&bars->p_full[h], 128);
      mbar_init(&bars->o_full[h], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, L::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      int last_k[3] = {-1, -1, -1}, last_v[3] = {-1, -1, -1};
      mbar_arrive_expect_tx(&bars->q_full, HPC * L::kTile);
      for (int h = 0; h < HPC; ++h)
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(smem + L::kQ + h * L::kTile + kb * kSwizzleBlock, &tm_q, &bars->q_full, kb * 64, h0 + h,
                      r0, b);
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % NS;
        const uint32_t ph = (t / NS) & 1;
        const int kv0 = (t_begin + t) * 128;
        if (!mbar_wait(&bars->k_empty[s], ph ^ 1, abort, p.err, 1)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], L::kTile);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(smem + L::kK + s * L::kTile + kb * kSwizzleBlock, &tm_k, &bars->k_full[s], kb * 64, kvh,
                      kv0, b);
        last_k[s] = ph;
        if (!mbar_wait(&bars->v_empty[s], ph ^ 1, abort, p.err, 2)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], L::kTile);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(smem + L::kV + s * L::kTile + kb * kSwizzleBlock, &tm_v, &bars->v_full[s], kb * 64, kvh,
                      kv0, b);
        last_v[s] = ph;
      }
      // Let every copy this thread started land before the block can exit.
      volatile int no_abort = 0;
      for (int s = 0; s < NS; ++s) {
        if (last_k[s] >= 0) mbar_wait(&bars->k_full[s], last_k[s], &no_abort, p.err, 3);
        if (last_v[s] >= 0) mbar_wait(&bars->v_full[s], last_v[s], &no_abort, p.err, 3);
      }
      mbar_wait(&bars->q_full, 0, &no_abort, p.err, 3);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      const uint32_t k_addr = smem_u32(smem + L::kK);
      const uint32_t v_addr = smem_u32(smem + L::kV);

      auto issue_s = [&](int h, int s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * kSwizzleBlock + (kk % 4) * 32;
          const uint64_t a = smem_desc_sw128(q_addr + h * L::kTile + off, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + s * L::kTile + off, 16, 1024);
          mma_ss(tmem + h * 128, a, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int h, int s, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = smem_desc_sw128(v_addr + s * L::kTile + kk * 2048, kSwizzleBlock, 1024);
          mma_ts(tmem + HPC * 128 + h * D, tmem + h * 128 + kk * 8, bd, idesc_o, (acc || kk > 0) ? 1u : 0u);
        }
      };

      bool ok = mbar_wait(&bars->q_full, 0, abort, p.err, 10);
      if (ok) tc_fence_after();
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int s = t % NS;
        const uint32_t ph = (t / NS) & 1;
        if (!(ok = mbar_wait(&bars->k_full[s], ph, abort, p.err, 11))) break;
        tc_fence_after();
        const int sp = (t + NS - 1) % NS;
        for (int h = 0; h < HPC && ok; ++h) {
          if (t > 0) {
            if (!(ok = mbar_wait(&bars->p_full[h], (t - 1) & 1, abort, p.err, 12))) break;
            if (h == 0 && !(ok = mbar_wait(&bars->v_full[sp], ((t - 1) / NS) & 1, abort, p.err, 13))) break;
            tc_fence_after();
            issue_pv(h, sp, t - 1 > 0);
          }
          issue_s(h, s);
          mma_commit(&bars->s_full[h]);
        }
        if (!ok) break;
        mma_commit(&bars->k_empty[s]);
        if (t > 0) mma_commit(&bars->v_empty[sp]);
      }
      if (ok) {
        const int t = n_tiles - 1;
        const int sl = t % NS;
        for (int h = 0; h < HPC && ok; ++h) {
          if (!(ok = mbar_wait(&bars->p_full[h], t & 1, abort, p.err, 14))) break;
          if (h == 0 && !(ok = mbar_wait(&bars->v_full[sl], (t / NS) & 1, abort, p.err, 15))) break;
          tc_fence_after();
          issue_pv(h, sl, t > 0);
          mma_commit(&bars->o_full[h]);
        }
        if (ok) mma_commit(&bars->v_empty[sl]);
      }
      // Every MMA this thread issued must finish before TMEM is released.
      mma_commit(&bars->drain);
      volatile int no_abort = 0;
      mbar_wait(&bars->drain, 0, &no_abort, p.err, 16);
    }
  } else if (warp >= 4 && warp < 4 + 4 * HPC) {
    // ------------------------------------------------------------- softmax
    const int h = (warp - 4) >> 2;
    const int lane_base = (warp & 3) * 32;
    const int row_in = lane_base + lane;
    const int row = r0 + row_in;
    const bool valid = row < p.S;
    const int lo_i = valid ? p.lo[rowbase + row] : 1;
    const int hi_i = valid ? p.hi[rowbase + row] : 0;
    const uint32_t t_lane = tmem + ((uint32_t)lane_base << 16);
    const uint32_t s_col = h * 128;
    const uint32_t o_col = HPC * 128 + h * D;
    const float sc = p.scale_log2;

    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[h], t & 1, abort, p.err, 20));
      if (!ok) break;
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(t_lane + s_col + c * 32, sv + c * 32);
      tmem_wait_ld();
      const int kv0 = (t_begin + t) * 128;
      const bool full = kv0 >= lo_last && kv0 + 127 <= hi_first;
      if (!full) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int j = kv0 + c;
          if (j < lo_i || j > hi_i) sv[c] = -INFINITY;
        }
      }
      float mx = sv[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, sv[c]);
      const float m_new = fmaxf(m_ref, mx * sc);
      const bool first = (m_ref == -INFINITY);
      const bool need = !first && (m_new > m_ref + 8.f);
      if (first) m_ref = m_new;
      if (__any_sync(0xffffffffu, need)) {
        float alpha = 1.f;
        if (!first) {
          alpha = ex2_approx(m_ref - m_new);
          m_ref = m_new;
        }
        l_sum *= alpha;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(t_lane + o_col + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(t_lane + o_col + c * 32, reinterpret_cast<uint32_t*>(o));
        }
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      float sum = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2_approx(fmaf(sv[2 * c], sc, -m_use));
        const float p1 = ex2_approx(fmaf(sv[2 * c + 1], sc, -m_use));
        sum += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l_sum += sum;
      tmem_st32(t_lane + s_col, pk);
      tmem_st32(t_lane + s_col + 32, pk + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[h]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full[h], 0, abort, p.err, 21));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_sum;
      const int hq = h0 + h;
      uint4* dst = reinterpret_cast<uint4*>(p.out + ((rowbase + row) * p.Hq + hq) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(t_lane + o_col + c * 32, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(o[2 * i] * inv_l, o[2 * i + 1] * inv_l);
        if (valid) {
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[c * 4 + i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (valid && p.lse != nullptr)
        p.lse[((size_t)b * p.Hq + hq) * p.S + row] = (m_ref + log2f(l_sum)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

size_t prefill_attention_smem_bytes(int D, int hpc) {
  if (D == 128) return hpc == 2 ? AttnLayout<128, 2>::kAlloc : AttnLayout<128, 1>::kAlloc;
  return hpc == 2 ? AttnLayout<64, 2>::kAlloc : AttnLayout<64, 1>::kAlloc;
}

template <int D, int HPC>
static cudaError_t launch_attn_t(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, cudaStream_t st) {
  using L = AttnLayout<D, HPC>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(prefill_attention_kernel<D, HPC>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)p.n_qtiles * p.B * p.Hkv * p.n_groups;
  prefill_attention_kernel<D, HPC><<<grid, kAttnThreads, L::kAlloc, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_prefill_attention(const AttnParams& p, int D, int hpc, const CUtensorMap& tq,
                                     const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  if (D == 128 && hpc == 2) return launch_attn_t<128, 2>(p, tq, tk, tv, st);
  if (D == 128 && hpc == 1) return launch_attn_t<128, 1>(p, tq, tk, tv, st);
  if (D == 64 && hpc == 2) return launch_attn_t<64, 2>(p, tq, tk, tv, st);
  if (D == 64 && hpc == 1) return launch_attn_t<64, 1>(p, tq, tk, tv, st);
  return cudaErrorInvalidValue;
}

}  // namespace g3
