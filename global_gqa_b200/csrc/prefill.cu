// Prefill attention of the Gemma 3 block on sm_100a (the prologue that
// normalises and rotates q and k is in prologue.cu).
//
//   prefill_attention: warp-specialised flash attention.  TMA (no multicast)
//                      streams 128-row K/V tiles, one thread issues tcgen05.mma
//                      for S = Q K^T and O += P V with accumulators in tensor
//                      memory, and eight warps per query head of the GQA pair
//                      run the fp32 online softmax (four threads per row).  The KV tiles a query tile
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

#include "func_attr.cuh"
#include "g3_internal.h"
#include "sm100_ptx.cuh"
#include "tmem_wide.cuh"

namespace g3 {

// ========================================================= attention kernel
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer and TMEM owner, then
// eight softmax warps per query head (warps 4-11 and 12-19 when two heads share
// the K/V tiles, warps 2-9 for one head): two warps per TMEM lane quarter,
// each on 16 of its 32 rows.
template <int HPC>
struct AttnRoles {
  // Two heads: 640 threads, one CTA per SM.  One head: 320 threads (warp 0
  // producer, warp 1 MMA, warps 2-9 softmax) and two CTAs per SM, so one
  // CTA's start and epilogue overlap the other's main loop.
  static constexpr int kFirstSoftmaxWarp = (HPC == 2) ? 4 : 2;
  static constexpr int kThreads = (kFirstSoftmaxWarp + 8 * HPC) * 32;
  static constexpr int kMinBlocks = (HPC == 2) ? 1 : 2;
};
constexpr int kSwizzleBlock = 128 * 64 * 2;  // 128 rows x 64 bf16 (one 128-byte swizzle column)

template <int D, int HPC>
struct AttnLayout {
  // K/V ring depth; one-head CTAs keep two CTAs' shared memory within one SM.
  static constexpr int kStages = (HPC == 2) ? (D == 64 ? 3 : 2) : (D == 64 ? 2 : 1);
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
  uint64_t out_ready[2];  // a head's output tile is staged in shared memory
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int D, int HPC>
__global__ void __launch_bounds__(AttnRoles<HPC>::kThreads, AttnRoles<HPC>::kMinBlocks)
    prefill_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                             AttnParams p) {
  using L = AttnLayout<D, HPC>;
  constexpr int NS = L::kStages;
  constexpr int KB = D / 64;  // swizzle columns per tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnBarriers* bars = reinterpret_cast<AttnBarriers*>(smem + L::kBar);
  volatile int* abort = &bars->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- work item.  A unit is (sequence, kv head, head group).  The grid
  // first runs the heavy query tiles (index >= light_qtiles) unit by unit,
  // heaviest first within each unit: the CTAs resident at one time then share
  // one kv head's K/V in L2, which on long causal layers otherwise comes from
  // DRAM many times over.  It ends with the light tiles of all units,
  // heaviest first, interleaved over the units, so that the last heavy tile
  // starts while enough light work remains to cover it.  light_qtiles =
  // n_qtiles gives the plain heaviest-first order over all units.
  const int units = p.B * p.Hkv * p.n_groups;
  const int n_heavy = p.n_qtiles - p.light_qtiles;
  const int idx = (int)blockIdx.x;
  int qt, rem;
  if (idx < units * n_heavy) {
    rem = idx / n_heavy;
    qt = p.n_qtiles - 1 - idx % n_heavy;
  } else {
    const int j = idx - units * n_heavy;
    qt = p.light_qtiles - 1 - j / units;
    rem = j % units;
  }
  const int gp = rem % p.n_groups;
  rem /= p.n_groups;
  const int kvh = rem % p.Hkv;
  const int b = rem / p.Hkv;
  const int h0 = kvh * p.G + gp * HPC;
  const int r0 = qt * 128;
  const int r_last = min(r0 + 127, p.S - 1);

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
      mbar_init(&bars->p_full[h], 256);
      mbar_init(&bars->o_full[h], 1);
      mbar_init(&bars->out_ready[h], 8);  // softmax warps of the head
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, L::kTmemCols);

  // Everything above is independent of the prologue's results; launched as a
  // programmatic dependent of the prologue, the CTA waits only here for its
  // intervals and its rotated q and k.
  griddep_wait();
  const size_t rowbase = (size_t)b * p.S;
  const int lo_first = p.lo[rowbase + r0];
  const int hi_last = p.hi[rowbase + r_last];
  const int lo_last = p.lo[rowbase + r_last];  // largest lo of the tile's rows
  const int hi_first = p.hi[rowbase + r0];     // smallest hi of the tile's rows
  const int t_begin = lo_first / 128;
  const int n_tiles = max(hi_last / 128, t_begin) - t_begin + 1;
  const int n_pre = min(n_tiles, NS);  // K/V tiles loaded before the CTA-wide barrier

  if (tid == 0) {
    // Thread 0 is also the TMA producer: start the Q tiles and the first K/V
    // stages now, so their latency overlaps the CTA-wide barrier below (the
    // ring's empty barriers start released).
    mbar_arrive_expect_tx(&bars->q_full, HPC * L::kTile);
    for (int h = 0; h < HPC; ++h)
      for (int kb = 0; kb < KB; ++kb)
        tma_load_4d(smem + L::kQ + h * L::kTile + kb * kSwizzleBlock, &tm_q, &bars->q_full, kb * 64, h0 + h, r0, b);
    for (int t = 0; t < n_pre; ++t) {
      const int kv0 = (t_begin + t) * 128;
      const int c1 = p.kv_head_major ? kv0 : kvh, c2 = p.kv_head_major ? kvh : kv0;
      mbar_arrive_expect_tx(&bars->k_full[t], L::kTile);
      for (int kb = 0; kb < KB; ++kb)
        tma_load_4d(smem + L::kK + t * L::kTile + kb * kSwizzleBlock, &tm_k, &bars->k_full[t], kb * 64, c1, c2, b);
      mbar_arrive_expect_tx(&bars->v_full[t], L::kTile);
      for (int kb = 0; kb < KB; ++kb)
        tma_load_4d(smem + L::kV + t * L::kTile + kb * kSwizzleBlock, &tm_v, &bars->v_full[t], kb * 64, c1, c2, b);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  constexpr int SW0 = AttnRoles<HPC>::kFirstSoftmaxWarp;
  if (warp < SW0) {
   if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      // Tiles 0 .. n_pre-1 were started before the CTA-wide barrier.
      int last_k[3] = {-1, -1, -1}, last_v[3] = {-1, -1, -1};
      for (int t = 0; t < n_pre; ++t) last_k[t] = last_v[t] = 0;
      for (int t = n_pre; t < n_tiles; ++t) {
        const int s = t % NS;
        const uint32_t ph = (t / NS) & 1;
        const int kv0 = (t_begin + t) * 128;
        // Tile coordinates: [B, S, Hkv, D] maps take (head, row); [B, Hkv,
        // rows, D] maps over a cache take (row, head).
        const int c1 = p.kv_head_major ? kv0 : kvh, c2 = p.kv_head_major ? kvh : kv0;
        if (!mbar_wait(&bars->k_empty[s], ph ^ 1, abort, p.err, 1)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], L::kTile);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(smem + L::kK + s * L::kTile + kb * kSwizzleBlock, &tm_k, &bars->k_full[s], kb * 64, c1, c2, b);
        last_k[s] = ph;
        if (!mbar_wait(&bars->v_empty[s], ph ^ 1, abort, p.err, 2)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], L::kTile);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_4d(smem + L::kV + s * L::kTile + kb * kSwizzleBlock, &tm_v, &bars->v_full[s], kb * 64, c1, c2, b);
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
#ifdef G3_FAULT_INJECT
          if (!(t == 0 && h == 0 && (int)blockIdx.x == p.withhold_cta))
#endif
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
    const int h = (warp - SW0) >> 3;  // query head of the pair
    if (h < HPC) {
      // ----------------------------------------------------------- softmax
      // Warp (quarter q = warp % 4, half s) owns TMEM lanes 32q + 16s .. +15;
      // thread t holds rows ra = t/4 and rb = t/4 + 8 of that slice and, in
      // every 8-column chunk k, columns 8k + 2(t%4) and 8k + 2(t%4) + 1; the
      // four threads t%4 = 0..3 of a row combine their partials by shuffles.
      const int lane_base = (warp & 3) * 32 + (((warp - SW0) >> 2) & 1) * 16;
      const int m4 = lane & 3;
      const int ra = lane_base + (lane >> 2), rb = ra + 8;
      const bool valid_a = r0 + ra < p.S, valid_b = r0 + rb < p.S;
      const int lo_a = valid_a ? p.lo[rowbase + r0 + ra] : 1, hi_a = valid_a ? p.hi[rowbase + r0 + ra] : 0;
      const int lo_b = valid_b ? p.lo[rowbase + r0 + rb] : 1, hi_b = valid_b ? p.hi[rowbase + r0 + rb] : 0;
      const uint32_t t_lane = tmem + ((uint32_t)lane_base << 16);
      const uint32_t s_col = h * 128;
      const uint32_t o_col = HPC * 128 + h * D;
      const float sc = p.scale_log2;

      float mref_a = -INFINITY, mref_b = -INFINITY, l_a = 0.f, l_b = 0.f;
      bool ok = true;
      for (int t = 0; t < n_tiles; ++t) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[h], t & 1, abort, p.err, 20));
        if (!ok) break;
        tc_fence_after();
        float sv[64];
        tmem_ld_16x256b_x16(t_lane + s_col, sv);
        tmem_wait_ld();
        const int tile0 = (t_begin + t) * 128;
        const bool full = tile0 >= lo_last && tile0 + 127 <= hi_first;
        if (!full) {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int col = tile0 + 8 * k + 2 * m4;
            if (col < lo_a || col > hi_a) sv[4 * k] = -INFINITY;
            if (col + 1 < lo_a || col + 1 > hi_a) sv[4 * k + 1] = -INFINITY;
            if (col < lo_b || col > hi_b) sv[4 * k + 2] = -INFINITY;
            if (col + 1 < lo_b || col + 1 > hi_b) sv[4 * k + 3] = -INFINITY;
          }
        }
        float mxa = fmax3(sv[0], sv[1], sv[4]), mxb = fmax3(sv[2], sv[3], sv[6]);
        mxa = fmax3(mxa, sv[5], sv[8]);
        mxb = fmax3(mxb, sv[7], sv[10]);
#pragma unroll
        for (int k = 2; k < 16; ++k) {
          if (k > 2) {
            mxa = fmax3(mxa, sv[4 * k], sv[4 * k + 1]);
            mxb = fmax3(mxb, sv[4 * k + 2], sv[4 * k + 3]);
          } else {
            mxa = fmaxf(mxa, sv[9]);
            mxb = fmaxf(mxb, sv[11]);
          }
        }
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
        mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
        const float mna = fmaxf(mref_a, mxa * sc), mnb = fmaxf(mref_b, mxb * sc);
        const bool first_a = (mref_a == -INFINITY), first_b = (mref_b == -INFINITY);
        const bool need = (!first_a && mna > mref_a + 8.f) || (!first_b && mnb > mref_b + 8.f);
        if (first_a) mref_a = mna;
        if (first_b) mref_b = mnb;
        const bool rescale = __any_sync(0xffffffffu, need);
        float alpha_a = 1.f, alpha_b = 1.f;
        if (rescale) {
          if (!first_a) {
            alpha_a = ex2_approx(mref_a - mna);
            mref_a = mna;
          }
          if (!first_b) {
            alpha_b = ex2_approx(mref_b - mnb);
            mref_b = mnb;
          }
          l_a *= alpha_a;
          l_b *= alpha_b;
        }
        const float mua = (mref_a == -INFINITY) ? 0.f : mref_a;
        const float mub = (mref_b == -INFINITY) ? 0.f : mref_b;
        float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float x0, x1, x2, x3;
          ffma2_bcast(sv[4 * k], sv[4 * k + 1], sc, -mua, x0, x1);
          ffma2_bcast(sv[4 * k + 2], sv[4 * k + 3], sc, -mub, x2, x3);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
          fadd2(sa0, sa1, p0, p1);
          fadd2(sb0, sb1, p2, p3);
          pk[2 * k] = pack_bf16x2(p0, p1);
          pk[2 * k + 1] = pack_bf16x2(p2, p3);
        }
        l_a += sa0 + sa1;
        l_b += sb0 + sb1;
        // P (bf16 pairs) over the first 64 columns of this head's S region.
        tmem_st_16x128b_x16(t_lane + s_col, pk);
        if (rescale) {
          // O is idle here: the previous P·V has completed (it was issued
          // before this tile's S) and the next one waits for p_full.
          // (Rolled at head dim 256, where unrolling spills.)
#pragma unroll(D > 128 ? 1 : D / 64)
          for (int q = 0; q < D / 64; ++q) {
            float o[32];
            tmem_ld_16x256b_x8(t_lane + o_col + q * 64, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              o[4 * k] *= alpha_a;
              o[4 * k + 1] *= alpha_a;
              o[4 * k + 2] *= alpha_b;
              o[4 * k + 3] *= alpha_b;
            }
            tmem_st_16x256b_x8(t_lane + o_col + q * 64, reinterpret_cast<uint32_t*>(o));
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[h]);
      }
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full[h], 0, abort, p.err, 21));
      if (ok) {
        tc_fence_after();
        const float inv_a = 1.f / l_a, inv_b = 1.f / l_b;
        const int hq = h0 + h;
        // O / l in bf16 is staged in this head's Q tile (no MMA reads it any
        // more: every MMA completed before o_full) in the 128-byte-swizzled
        // layout of a TMA tile, then one thread stores the tile.  Rows past S
        // are clipped by the store.
        uint8_t* stage = smem + L::kQ + h * L::kTile;
        const int sw = ra & 7;  // rb = ra + 8 has the same swizzle phase
#pragma unroll(D > 128 ? 1 : D / 64)
        for (int q = 0; q < D / 64; ++q) {
          float o[32];
          tmem_ld_16x256b_x8(t_lane + o_col + q * 64, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint8_t* blk = stage + q * kSwizzleBlock + ((k ^ sw) * 16) + m4 * 4;
            *reinterpret_cast<uint32_t*>(blk + ra * 128) = pack_bf16x2(o[4 * k] * inv_a, o[4 * k + 1] * inv_a);
            *reinterpret_cast<uint32_t*>(blk + rb * 128) = pack_bf16x2(o[4 * k + 2] * inv_b, o[4 * k + 3] * inv_b);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->out_ready[h]);
        if (((warp - SW0) & 7) == 0 && lane == 0) {
          if (mbar_wait(&bars->out_ready[h], 0, abort, p.err, 22)) {
            for (int kb = 0; kb < KB; ++kb) tma_store_4d(&tm_out, stage + kb * kSwizzleBlock, kb * 64, hq, r0, b);
            bulk_commit_group();
            bulk_wait_group_read0();  // the staging tile must outlive the store's reads
          }
        }
        if (m4 == 0 && p.lse != nullptr) {
          const size_t lrow = ((size_t)b * p.Hq + hq) * p.S + r0;
          if (valid_a) p.lse[lrow + ra] = (mref_a + log2f(l_a)) * 0.69314718055994530942f;
          if (valid_b) p.lse[lrow + rb] = (mref_b + log2f(l_b)) * 0.69314718055994530942f;
        }
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
  if (D == 256) return AttnLayout<256, 1>::kAlloc;
  if (D == 128) return hpc == 2 ? AttnLayout<128, 2>::kAlloc : AttnLayout<128, 1>::kAlloc;
  return hpc == 2 ? AttnLayout<64, 2>::kAlloc : AttnLayout<64, 1>::kAlloc;
}

// Light query tiles per unit for the heavy-by-unit order of a causal layer,
// whose query tile t visits t + 1 key tiles.  The heaviest tile of the last
// unit starts with the light tiles of all units still to run; they hold
// units * T^2 / 2 tile visits, and covering its n_qtiles visits on each of the
// `resident` CTA slots needs T = sqrt(2 * n_qtiles * resident / units).
static int light_qtiles_for(int n_qtiles, long long units, int resident) {
  if (units <= 0 || resident <= 0) return n_qtiles;
  const double t = std::ceil(std::sqrt(2.0 * n_qtiles * (double)resident / (double)units));
  return t >= n_qtiles ? n_qtiles : (int)t;
}

// CTAs of `kernel` resident on the current device at once (SMs x CTAs per
// SM), cached per device; 0 when the runtime cannot say.
template <class Kernel>
static int resident_ctas(Kernel* kernel, int threads, size_t smem, std::atomic<int>* cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  const int r = sms * per_sm;
  if (dev >= 0 && dev < 64 && r > 0) cache[dev].store(r, std::memory_order_relaxed);
  return r;
}

template <int D, int HPC>
static cudaError_t launch_attn_t(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const CUtensorMap& to, cudaStream_t st) {
  using L = AttnLayout<D, HPC>;
  static_assert(L::kAlloc <= 232448, "shared memory budget");
  static std::atomic<uint64_t> configured{0};  // devices with the shared-memory limit raised
  static std::atomic<int> resident[64];        // per device; zero-initialised (static storage)
  const cudaError_t e = ensure_dynamic_smem(prefill_attention_kernel<D, HPC>, L::kAlloc, configured);
  if (e != cudaSuccess) return e;
  AttnParams q = p;
  q.light_qtiles = p.n_qtiles;
  if (p.heavy_by_head) {
    const int r = resident_ctas(prefill_attention_kernel<D, HPC>, AttnRoles<HPC>::kThreads, L::kAlloc, resident);
    q.light_qtiles = light_qtiles_for(p.n_qtiles, (long long)p.B * p.Hkv * p.n_groups, r);
  }
  const unsigned grid = (unsigned)p.n_qtiles * p.B * p.Hkv * p.n_groups;
  return launch_dependent(prefill_attention_kernel<D, HPC>, dim3(grid), dim3(AttnRoles<HPC>::kThreads), L::kAlloc,
                          st, tq, tk, tv, to, q);
}

cudaError_t launch_prefill_attention(const AttnParams& p, int D, int hpc, const CUtensorMap& tq,
                                     const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                                     cudaStream_t st) {
  if (D == 256 && hpc == 1) return launch_attn_t<256, 1>(p, tq, tk, tv, to, st);
  if (D == 128 && hpc == 2) return launch_attn_t<128, 2>(p, tq, tk, tv, to, st);
  if (D == 128 && hpc == 1) return launch_attn_t<128, 1>(p, tq, tk, tv, to, st);
  if (D == 64 && hpc == 2) return launch_attn_t<64, 2>(p, tq, tk, tv, to, st);
  if (D == 64 && hpc == 1) return launch_attn_t<64, 1>(p, tq, tk, tv, to, st);
  return cudaErrorInvalidValue;
}

}  // namespace g3
