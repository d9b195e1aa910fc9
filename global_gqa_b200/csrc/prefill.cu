// Prefill attention of the Gemma 3 block on sm_100a (the prologue that
// normalises and rotates q and k is in prologue.cu).
//
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

  // Producer / MMA warpgroup gives registers to the two softmax warpgroups
  // (128 x 56 + 256 x 224 = 384 x 168, the launch's register budget).  Each
  // role runs inside the branch that set its register count.
  if (warp < 4) {
    setmaxnreg_dec<56>();
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
   }
  } else {
    setmaxnreg_inc<224>();
   if (warp < 4 + 4 * HPC) {
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
      float mx0 = fmax3(sv[0], sv[1], sv[2]), mx1 = fmax3(sv[3], sv[4], sv[5]);
#pragma unroll
      for (int c = 6; c < 126; c += 4) {
        mx0 = fmax3(mx0, sv[c], sv[c + 1]);
        mx1 = fmax3(mx1, sv[c + 2], sv[c + 3]);
      }
      const float mx = fmax3(fmax3(mx0, mx1, sv[126]), sv[127], sv[127]);
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
      // Exponentials two at a time (one f16x2 exp-unit operation per pair),
      // scaling and sums as packed fp32x2 operations, two partial sum pairs.
      float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        float x0, x1, p0, p1;
        ffma2_bcast(sv[2 * c], sv[2 * c + 1], sc, -m_use, x0, x1);
        ex2_pair_f16(x0, x1, p0, p1);
        if (c & 1) {
          fadd2(sb0, sb1, p0, p1);
        } else {
          fadd2(sa0, sa1, p0, p1);
        }
        pk[c] = pack_bf16x2(p0, p1);
      }
      l_sum += (sa0 + sa1) + (sb0 + sb1);
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
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
