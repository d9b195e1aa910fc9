// Prefill backward at head dim 256: the attention of the Gemma 3 1B model
// ("Gemma explained: what's new in Gemma 3", the 1B module printout: 4 query
// heads, 1 kv head, q_norm / k_norm over 256 features), trained like the
// larger models (Gemma 3 Technical Report, sections 2.2 and 2.3).  The
// gradients are those of backward.cu; only the tiling differs.
//
// At D = 256 a 128-row tile of q, k, v or dout is 64 KB of shared memory, and
// an accumulator of 128 rows takes 256 of the 512 tensor-memory columns.  So
// the tile that stays resident in a CTA keeps 128 rows while the streamed side
// moves in 64-row sub-tiles (the products S^T, dP^T, S, dP are 128 x 64), and
// dV and dK, which together would need all 512 columns before S^T and dP^T,
// come from two kernels:
//   bwd_dv256 : per (sequence, kv head, 128-key tile): K resident, (Q, dO)
//               sub-tiles of every query head of the group streamed through a
//               two-stage ring; S^T = K Q^T, P^T into tensor memory,
//               dV += P^T dO.
//   bwd_dk256 : the same CTAs with K and V resident, Q sub-tiles double- and
//               dO sub-tiles single-buffered: S^T and dP^T = V dO^T,
//               dS^T = P^T (dP^T - delta), dK += dS^T Q.
//   bwd_dq256 : per (sequence, query head, 128-row query tile): Q and dO
//               resident, K sub-tiles double- and V sub-tiles single-buffered:
//               S = Q K^T, dP = dO V^T, dQ += dS K.
// The packed bf16 tile of each accumulate product (P^T, dS^T, dS) has two
// buffers of its own, so the next S^T / dP^T (or S / dP) is issued as soon as
// the elementwise warps have read the current one.
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
constexpr int kD = 256;
constexpr int kKB = kD / 64;             // 128-byte swizzle columns per row
constexpr int kSub = 64;                 // rows of a streamed sub-tile
constexpr int kBlkRes = 128 * 128;       // one swizzle column of a 128-row tile (16 KB)
constexpr int kBlkSub = kSub * 128;      // one swizzle column of a 64-row sub-tile (8 KB)
constexpr int kTileRes = kKB * kBlkRes;  // 64 KB
constexpr int kTileSub = kKB * kBlkSub;  // 32 KB

// TMEM columns: the 128 x 64 product(s) at 0 (and 64), the packed bf16 tile
// of the accumulate product at 128 + 32 * buffer (at 64 + 32 * buffer in
// bwd_dv256, which has no dP^T), the 256-column accumulator at 256.
constexpr uint32_t kColAcc = 256;

struct Bwd256Barriers {
  uint64_t res_full;              // the resident tiles
  uint64_t full[2], empty[2];     // the double-buffered stream
  uint64_t full2, empty2;         // the single-buffered stream
  uint64_t s_full, s_free, dp_full, dp_free;
  uint64_t x_full[2], x_free[2];  // packed bf16 tile of the accumulate product
  uint64_t o_full, drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// X = A B^T over the 256 features, A a 128-row and B a 64-row tile (both
// K-major in shared memory): a 128 x 64 fp32 product at TMEM column `col`.
__device__ __forceinline__ void issue_x256(uint32_t tmem, uint32_t col, uint32_t a_addr, uint32_t b_addr) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, kSub, false, false);
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    const uint32_t off_a = (kk / 4) * kBlkRes + (kk % 4) * 32;
    const uint32_t off_b = (kk / 4) * kBlkSub + (kk % 4) * 32;
    mma_ss(tmem + col, smem_desc_sw128(a_addr + off_a, 16, 1024), smem_desc_sw128(b_addr + off_b, 16, 1024), idesc,
           kk > 0 ? 1u : 0u);
  }
}

// acc(128 x 256) += X B: X the packed bf16 128 x 64 tile at TMEM column
// `x_col`, B a 64-row sub-tile read MN-major (its rows are the reduction).
__device__ __forceinline__ void issue_acc256(uint32_t tmem, uint32_t x_col, uint32_t b_addr, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, kD, false, true);
#pragma unroll
  for (int kk = 0; kk < kSub / 16; ++kk)
    mma_ts(tmem + kColAcc, tmem + x_col + 8 * kk, smem_desc_sw128(b_addr + kk * 2048, kBlkSub, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

// The 256-column accumulator of this warp's 16 rows (its column half, two
// 64-column loads) to global memory: bf16, or fp32 scaled by `scale`.
template <bool kF32>
__device__ __forceinline__ void store_acc256(uint32_t t_lane, int ch, int m4, void* row_a, void* row_b, bool va,
                                             bool vb, float scale) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    float o[32];
    tmem_ld_16x256b_x8(t_lane + kColAcc + 128 * ch + 64 * c, o);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int col = 128 * ch + 64 * c + 8 * k + 2 * m4;
      if constexpr (kF32) {
        if (va) *reinterpret_cast<float2*>(static_cast<float*>(row_a) + col) = make_float2(o[4 * k] * scale, o[4 * k + 1] * scale);
        if (vb) *reinterpret_cast<float2*>(static_cast<float*>(row_b) + col) = make_float2(o[4 * k + 2] * scale, o[4 * k + 3] * scale);
      } else {
        if (va) *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(row_a) + col) = pack_bf16x2(o[4 * k], o[4 * k + 1]);
        if (vb) *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(row_b) + col) = pack_bf16x2(o[4 * k + 2], o[4 * k + 3]);
      }
    }
  }
}

// Work of the key-tile kernels: item n = (query head kvh*G + n%G, 64-row query
// sub-tile), the sub-tiles of the query tiles that see the key tile in
// descending order.
struct KeyTileWork {
  int b, kvh, j0, q_hi, n_items;
  __device__ KeyTileWork(const BwdParams& p) {
    const int per_tile = p.B * p.Hkv;
    const int kt = (int)(blockIdx.x / per_tile);
    const int rem = (int)(blockIdx.x % per_tile);
    kvh = rem % p.Hkv;
    b = rem / p.Hkv;
    j0 = kt * kTileRows;
    const int2 qr = p.kvrange[(size_t)b * p.n_kvtiles + kt];
    q_hi = 2 * qr.y + 1;
    n_items = 2 * (qr.y - qr.x + 1) * p.G;
  }
  __device__ int q0(int n, int G) const { return (q_hi - n / G) * kSub; }
  __device__ int head(int n, int G) const { return kvh * G + n % G; }
};

__device__ __forceinline__ void init_bwd256_barriers(Bwd256Barriers* bars) {
  mbar_init(&bars->res_full, 1);
  for (int s = 0; s < 2; ++s) {
    mbar_init(&bars->full[s], 1);
    mbar_init(&bars->empty[s], 1);
    mbar_init(&bars->x_full[s], kBwdEwThreads);
    mbar_init(&bars->x_free[s], 1);
  }
  mbar_init(&bars->full2, 1);
  mbar_init(&bars->empty2, 1);
  mbar_init(&bars->s_full, 1);
  mbar_init(&bars->s_free, kBwdEwThreads);
  mbar_init(&bars->dp_full, 1);
  mbar_init(&bars->dp_free, kBwdEwThreads);
  mbar_init(&bars->o_full, 1);
  mbar_init(&bars->drain, 1);
  bars->abort = 0;
  fence_mbar_init();
}
}  // namespace

// ================================================================ bwd_dv256
struct Dv256Layout {
  static constexpr int kK = 0;
  static constexpr int kStage0 = kTileRes;
  static constexpr int kSide = 2 * kTileSub;                // lse2 of the 64 rows, then their (lo, hi)
  static constexpr int kStageBytes = 2 * kTileSub + 1024;  // Q, dO, side data
  static constexpr int kBar = kStage0 + 2 * kStageBytes;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dv256_kernel(const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_do64,
                     const __grid_constant__ CUtensorMap tm_k, BwdParams p) {
  using L = Dv256Layout;
  static_assert(sizeof(Bwd256Barriers) <= L::kBytes - L::kBar, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Bwd256Barriers* bars = reinterpret_cast<Bwd256Barriers*>(smem + L::kBar);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const KeyTileWork w(p);
  const int n_items = w.n_items, n_pre = min(n_items, 2);
  auto stage_ptr = [&](int s) { return smem + L::kStage0 + s * L::kStageBytes; };
  auto issue_stage = [&](int n) {
    const int s = n & 1, h = w.head(n, p.G), q0 = w.q0(n, p.G);
    uint8_t* st = stage_ptr(s);
    mbar_arrive_expect_tx(&bars->full[s], 2 * kTileSub + 768);
    for (int kb = 0; kb < kKB; ++kb) {
      tma_load_4d(st + kb * kBlkSub, &tm_q64, &bars->full[s], kb * 64, h, q0, w.b);
      tma_load_4d(st + kTileSub + kb * kBlkSub, &tm_do64, &bars->full[s], kb * 64, h, q0, w.b);
    }
    bulk_load(st + L::kSide, p.lse2 + ((size_t)w.b * p.Hq + h) * p.S_pad + q0, 256, &bars->full[s]);
    bulk_load(st + L::kSide + 256, p.colmask + (size_t)w.b * p.S_pad + q0, 512, &bars->full[s]);
  };

  if (tid == 0) {
    init_bwd256_barriers(bars);
    prefetch_tensormap(&tm_q64);
    prefetch_tensormap(&tm_do64);
    prefetch_tensormap(&tm_k);
    mbar_arrive_expect_tx(&bars->res_full, kTileRes);
    for (int kb = 0; kb < kKB; ++kb)
      tma_load_4d(smem + L::kK + kb * kBlkRes, &tm_k, &bars->res_full, kb * 64, w.kvh, w.j0, w.b);
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
      int last[2] = {-1, -1};
      for (int n = 0; n < n_pre; ++n) last[n] = 0;
      for (int n = 2; n < n_items; ++n) {
        const int s = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        if (!mbar_wait(&bars->empty[s], ph ^ 1, abort, p.err, 80)) break;
        issue_stage(n);
        last[s] = ph;
      }
      volatile int no_abort = 0;
      mbar_wait(&bars->res_full, 0, &no_abort, p.err, 81);
      for (int s = 0; s < 2; ++s)
        if (last[s] >= 0) mbar_wait(&bars->full[s], last[s], &no_abort, p.err, 81);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t k_addr = smem_u32(smem + L::kK);
      auto q_addr = [&](int s) { return smem_u32(stage_ptr(s)); };
      auto do_addr = [&](int s) { return smem_u32(stage_ptr(s) + kTileSub); };
      bool ok = mbar_wait(&bars->res_full, 0, abort, p.err, 82);
      if (ok) ok = mbar_wait(&bars->full[0], 0, abort, p.err, 83);
      if (ok) {
        tc_fence_after();
        issue_x256(tmem, 0, k_addr, q_addr(0));  // S^T = K Q^T
        mma_commit(&bars->s_full);
      }
      for (int n = 0; ok && n < n_items; ++n) {
        const int s = n & 1;
        if (n + 1 < n_items) {
          if (!(ok = mbar_wait(&bars->full[s ^ 1], ((n + 1) >> 1) & 1, abort, p.err, 84))) break;
          if (!(ok = mbar_wait(&bars->s_free, n & 1, abort, p.err, 85))) break;
          tc_fence_after();
          issue_x256(tmem, 0, k_addr, q_addr(s ^ 1));
          mma_commit(&bars->s_full);
        }
        if (!(ok = mbar_wait(&bars->x_full[s], (n >> 1) & 1, abort, p.err, 86))) break;
        tc_fence_after();
        issue_acc256(tmem, 64 + 32 * s, do_addr(s), n > 0);  // dV += P^T dO
        mma_commit(&bars->empty[s]);
        mma_commit(&bars->x_free[s]);
      }
      if (ok) mma_commit(&bars->o_full);
      mma_commit(&bars->drain);
      volatile int no_abort = 0;
      mbar_wait(&bars->drain, 0, &no_abort, p.err, 87);
    }
  } else {
    // --------------------------------------------------------------- P^T
    const int lane_base = bwd_lane_base(warp), ch = bwd_col_half(warp);
    const int m4 = lane & 3;
    const int ra = lane_base + (lane >> 2), rb = ra + 8;
    const int ja = w.j0 + ra, jb = w.j0 + rb;  // key of each of this thread's rows
    const uint32_t t_lane = tmem + ((uint32_t)lane_base << 16);
    const float sc = p.scale_log2;
    bool ok = true;
    for (int n = 0; n < n_items; ++n) {
      const int s = n & 1, q0 = w.q0(n, p.G);
      // This thread's query columns: 32 ch + 8 k + 2 m4 + {0, 1}, k < 4.
      const float2* l2 = reinterpret_cast<const float2*>(stage_ptr(s) + L::kSide) + 16 * ch;
      const int2* cm2 = reinterpret_cast<const int2*>(stage_ptr(s) + L::kSide + 256);
      const int4* cm = reinterpret_cast<const int4*>(cm2) + 16 * ch;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->full[s], (n >> 1) & 1, abort, p.err, 88));
      if (!ok) break;
      const bool full = q0 + kSub - 1 < p.S && cm2[kSub - 1].x <= w.j0 && cm2[0].y >= w.j0 + kTileRows - 1;
      float2 lv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) lv[k] = l2[4 * k + m4];
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, n & 1, abort, p.err, 89));
      if (!ok) break;
      tc_fence_after();
      float pv[16];
      tmem_ld_16x256b_x4(t_lane + 32 * ch, pv);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_free);
      uint32_t pk[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float x0 = fmaf(pv[4 * k], sc, -lv[k].x), x1 = fmaf(pv[4 * k + 1], sc, -lv[k].y);
        float x2 = fmaf(pv[4 * k + 2], sc, -lv[k].x), x3 = fmaf(pv[4 * k + 3], sc, -lv[k].y);
        if (!full) {
          const int4 c = cm[4 * k + m4];  // (lo, hi) of the two query columns
          if (ja < c.x || ja > c.y) x0 = -INFINITY;
          if (ja < c.z || ja > c.w) x1 = -INFINITY;
          if (jb < c.x || jb > c.y) x2 = -INFINITY;
          if (jb < c.z || jb > c.w) x3 = -INFINITY;
        }
        pk[2 * k] = pack_bf16x2(ex2_approx(x0), ex2_approx(x1));
        pk[2 * k + 1] = pack_bf16x2(ex2_approx(x2), ex2_approx(x3));
      }
      if (n >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->x_free[s], ((n - 2) >> 1) & 1, abort, p.err, 90));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st_16x128b_x4(t_lane + 64 + 32 * s + 16 * ch, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->x_full[s]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort, p.err, 91));
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dva = p.dv + ((size_t)(w.b * p.S + ja) * p.Hkv + w.kvh) * kD;
      __nv_bfloat16* dvb = p.dv + ((size_t)(w.b * p.S + jb) * p.Hkv + w.kvh) * kD;
      store_acc256<false>(t_lane, ch, m4, dva, dvb, ja < p.S, jb < p.S, 1.f);
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

// ================================================================ bwd_dk256
struct Dk256Layout {
  static constexpr int kK = 0;
  static constexpr int kV = kTileRes;
  static constexpr int kQ0 = 2 * kTileRes;         // two Q sub-tile buffers
  static constexpr int kDo = kQ0 + 2 * kTileSub;   // one dO sub-tile buffer
  static constexpr int kSide0 = kDo + kTileSub;    // per Q buffer: lse2, then delta, of its 64 rows
  static constexpr int kBar = kSide0 + 2 * 512;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dk256_kernel(const __grid_constant__ CUtensorMap tm_q64, const __grid_constant__ CUtensorMap tm_do64,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, BwdParams p) {
  using L = Dk256Layout;
  static_assert(sizeof(Bwd256Barriers) <= L::kBytes - L::kBar, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Bwd256Barriers* bars = reinterpret_cast<Bwd256Barriers*>(smem + L::kBar);
  volatile int* abort = &bars->abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const KeyTileWork w(p);
  const int n_items = w.n_items;
  auto issue_q = [&](int n) {
    const int buf = n & 1, h = w.head(n, p.G), q0 = w.q0(n, p.G);
    uint8_t* dst = smem + L::kQ0 + buf * kTileSub;
    mbar_arrive_expect_tx(&bars->full[buf], kTileSub + 512);
    for (int kb = 0; kb < kKB; ++kb) tma_load_4d(dst + kb * kBlkSub, &tm_q64, &bars->full[buf], kb * 64, h, q0, w.b);
    const size_t rq = ((size_t)w.b * p.Hq + h) * p.S_pad + q0;
    bulk_load(smem + L::kSide0 + buf * 512, p.lse2 + rq, 256, &bars->full[buf]);
    bulk_load(smem + L::kSide0 + buf * 512 + 256, p.delta + rq, 256, &bars->full[buf]);
  };
  auto issue_do = [&](int n) {
    const int h = w.head(n, p.G), q0 = w.q0(n, p.G);
    mbar_arrive_expect_tx(&bars->full2, kTileSub);
    for (int kb = 0; kb < kKB; ++kb)
      tma_load_4d(smem + L::kDo + kb * kBlkSub, &tm_do64, &bars->full2, kb * 64, h, q0, w.b);
  };

  if (tid == 0) {
    init_bwd256_barriers(bars);
    prefetch_tensormap(&tm_q64);
    prefetch_tensormap(&tm_do64);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    mbar_arrive_expect_tx(&bars->res_full, 2 * kTileRes);
    for (int kb = 0; kb < kKB; ++kb) {
      tma_load_4d(smem + L::kK + kb * kBlkRes, &tm_k, &bars->res_full, kb * 64, w.kvh, w.j0, w.b);
      tma_load_4d(smem + L::kV + kb * kBlkRes, &tm_v, &bars->res_full, kb * 64, w.kvh, w.j0, w.b);
    }
    issue_q(0);
    if (n_items > 1) issue_q(1);
    issue_do(0);
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    // dO(n) once dP^T(n-1) has read the single dO buffer; Q(n+1) once dK(n-1)
    // has read the buffer it takes.
    if (lane == 0) {
      int last_q[2] = {0, n_items > 1 ? 0 : -1};
      int last_do = 0;
      for (int n = 1; n < n_items; ++n) {
        if (!mbar_wait(&bars->empty2, (n - 1) & 1, abort, p.err, 92)) break;
        issue_do(n);
        last_do = n & 1;
        if (n + 1 < n_items) {
          const int buf = (n + 1) & 1;
          const uint32_t ph = ((n + 1) >> 1) & 1;
          if (!mbar_wait(&bars->empty[buf], ph ^ 1, abort, p.err, 93)) break;
          issue_q(n + 1);
          last_q[buf] = ph;
        }
      }
      volatile int no_abort = 0;
      mbar_wait(&bars->res_full, 0, &no_abort, p.err, 94);
      mbar_wait(&bars->full2, last_do, &no_abort, p.err, 94);
      for (int s = 0; s < 2; ++s)
        if (last_q[s] >= 0) mbar_wait(&bars->full[s], last_q[s], &no_abort, p.err, 94);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t k_addr = smem_u32(smem + L::kK), v_addr = smem_u32(smem + L::kV);
      const uint32_t do_addr = smem_u32(smem + L::kDo);
      auto q_addr = [&](int buf) { return smem_u32(smem + L::kQ0 + buf * kTileSub); };
      bool ok = mbar_wait(&bars->res_full, 0, abort, p.err, 95);
      if (ok) ok = mbar_wait(&bars->full[0], 0, abort, p.err, 96);
      if (ok) {
        tc_fence_after();
        issue_x256(tmem, 0, k_addr, q_addr(0));  // S^T = K Q^T
        mma_commit(&bars->s_full);
      }
      if (ok) ok = mbar_wait(&bars->full2, 0, abort, p.err, 96);
      if (ok) {
        tc_fence_after();
        issue_x256(tmem, 64, v_addr, do_addr);  // dP^T = V dO^T
        mma_commit(&bars->dp_full);
        mma_commit(&bars->empty2);
      }
      for (int n = 0; ok && n < n_items; ++n) {
        const int buf = n & 1;
        if (n + 1 < n_items) {
          if (!(ok = mbar_wait(&bars->full[buf ^ 1], ((n + 1) >> 1) & 1, abort, p.err, 97))) break;
          if (!(ok = mbar_wait(&bars->s_free, n & 1, abort, p.err, 98))) break;
          tc_fence_after();
          issue_x256(tmem, 0, k_addr, q_addr(buf ^ 1));
          mma_commit(&bars->s_full);
          if (!(ok = mbar_wait(&bars->full2, (n + 1) & 1, abort, p.err, 99))) break;
          if (!(ok = mbar_wait(&bars->dp_free, n & 1, abort, p.err, 100))) break;
          tc_fence_after();
          issue_x256(tmem, 64, v_addr, do_addr);
          mma_commit(&bars->dp_full);
          mma_commit(&bars->empty2);
        }
        if (!(ok = mbar_wait(&bars->x_full[buf], (n >> 1) & 1, abort, p.err, 101))) break;
        tc_fence_after();
        issue_acc256(tmem, 128 + 32 * buf, q_addr(buf), n > 0);  // dK += dS^T Q
        mma_commit(&bars->empty[buf]);
        mma_commit(&bars->x_free[buf]);
      }
      if (ok) mma_commit(&bars->o_full);
      mma_commit(&bars->drain);
      volatile int no_abort = 0;
      mbar_wait(&bars->drain, 0, &no_abort, p.err, 102);
    }
  } else {
    // -------------------------------------------------------------- dS^T
    const int lane_base = bwd_lane_base(warp), ch = bwd_col_half(warp);
    const int m4 = lane & 3;
    const int ra = lane_base + (lane >> 2), rb = ra + 8;
    const int ja = w.j0 + ra, jb = w.j0 + rb;
    const uint32_t t_lane = tmem + ((uint32_t)lane_base << 16);
    const float sc = p.scale_log2;
    bool ok = true;
    for (int n = 0; n < n_items; ++n) {
      const int buf = n & 1, q0 = w.q0(n, p.G);
      // Row intervals of the query columns, read from global memory (L2): the
      // tile-wide test first, the per-column pairs only on edge tiles.
      const int2* cmg = p.colmask + (size_t)w.b * p.S_pad + q0;
      const bool full = q0 + kSub - 1 < p.S && cmg[kSub - 1].x <= w.j0 && cmg[0].y >= w.j0 + kTileRows - 1;
      const float2* l2 = reinterpret_cast<const float2*>(smem + L::kSide0 + buf * 512) + 16 * ch;
      const float2* dl = reinterpret_cast<const float2*>(smem + L::kSide0 + buf * 512 + 256) + 16 * ch;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->full[buf], (n >> 1) & 1, abort, p.err, 103));
      if (!ok) break;
      float2 lv[4], dv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        lv[k] = l2[4 * k + m4];
        dv[k] = dl[4 * k + m4];
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, n & 1, abort, p.err, 104));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, n & 1, abort, p.err, 105));
      if (!ok) break;
      tc_fence_after();
      float pv[16], dp[16];
      tmem_ld_16x256b_x4(t_lane + 32 * ch, pv);
      tmem_ld_16x256b_x4(t_lane + 64 + 32 * ch, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_free);
      mbar_arrive(&bars->dp_free);
      uint32_t pk[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float x0 = fmaf(pv[4 * k], sc, -lv[k].x), x1 = fmaf(pv[4 * k + 1], sc, -lv[k].y);
        float x2 = fmaf(pv[4 * k + 2], sc, -lv[k].x), x3 = fmaf(pv[4 * k + 3], sc, -lv[k].y);
        if (!full) {
          const int4 c = reinterpret_cast<const int4*>(cmg)[16 * ch + 4 * k + m4];
          if (ja < c.x || ja > c.y) x0 = -INFINITY;
          if (ja < c.z || ja > c.w) x1 = -INFINITY;
          if (jb < c.x || jb > c.y) x2 = -INFINITY;
          if (jb < c.z || jb > c.w) x3 = -INFINITY;
        }
        pk[2 * k] = pack_bf16x2(ex2_approx(x0) * (dp[4 * k] - dv[k].x), ex2_approx(x1) * (dp[4 * k + 1] - dv[k].y));
        pk[2 * k + 1] =
            pack_bf16x2(ex2_approx(x2) * (dp[4 * k + 2] - dv[k].x), ex2_approx(x3) * (dp[4 * k + 3] - dv[k].y));
      }
      if (n >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->x_free[buf], ((n - 2) >> 1) & 1, abort, p.err, 106));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st_16x128b_x4(t_lane + 128 + 32 * buf + 16 * ch, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->x_full[buf]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort, p.err, 107));
    if (ok) {
      tc_fence_after();
      float* dka = p.dk_hat + ((size_t)(w.b * p.S + ja) * p.Hkv + w.kvh) * kD;
      float* dkb = p.dk_hat + ((size_t)(w.b * p.S + jb) * p.Hkv + w.kvh) * kD;
      store_acc256<true>(t_lane, ch, m4, dka, dkb, ja < p.S, jb < p.S, p.inv_sqrt_d);
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

// ================================================================ bwd_dq256
struct Dq256Layout {
  static constexpr int kQ = 0;
  static constexpr int kDo = kTileRes;
  static constexpr int kK0 = 2 * kTileRes;       // two K sub-tile buffers
  static constexpr int kV = kK0 + 2 * kTileSub;  // one V sub-tile buffer
  static constexpr int kBar = kV + kTileSub;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k64, const __grid_constant__ CUtensorMap tm_v64,
                     BwdParams p) {
  using L = Dq256Layout;
  static_assert(sizeof(Bwd256Barriers) <= L::kBytes - L::kBar, "barrier block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  Bwd256Barriers* bars = reinterpret_cast<Bwd256Barriers*>(smem + L::kBar);
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
  const int t_begin = lo_first / kSub;
  const int n_tiles = max(hi_last / kSub, t_begin) - t_begin + 1;  // 64-key sub-tiles

  auto issue_k = [&](int t) {
    const int buf = t & 1;
    mbar_arrive_expect_tx(&bars->full[buf], kTileSub);
    for (int kb = 0; kb < kKB; ++kb)
      tma_load_4d(smem + L::kK0 + buf * kTileSub + kb * kBlkSub, &tm_k64, &bars->full[buf], kb * 64, kvh,
                  (t_begin + t) * kSub, b);
  };
  auto issue_v = [&](int t) {
    mbar_arrive_expect_tx(&bars->full2, kTileSub);
    for (int kb = 0; kb < kKB; ++kb)
      tma_load_4d(smem + L::kV + kb * kBlkSub, &tm_v64, &bars->full2, kb * 64, kvh, (t_begin + t) * kSub, b);
  };

  if (tid == 0) {
    init_bwd256_barriers(bars);
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_do);
    prefetch_tensormap(&tm_k64);
    prefetch_tensormap(&tm_v64);
    mbar_arrive_expect_tx(&bars->res_full, 2 * kTileRes);
    for (int kb = 0; kb < kKB; ++kb) {
      tma_load_4d(smem + L::kQ + kb * kBlkRes, &tm_q, &bars->res_full, kb * 64, h, r0, b);
      tma_load_4d(smem + L::kDo + kb * kBlkRes, &tm_do, &bars->res_full, kb * 64, h, r0, b);
    }
    issue_k(0);
    if (n_tiles > 1) issue_k(1);
    issue_v(0);
  }
  if (warp == 1) tmem_alloc(&bars->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    // V(t) once dP(t-1) has read the single V buffer; K(t+1) once dQ(t-1)
    // has read the buffer it takes.
    if (lane == 0) {
      int last_k[2] = {0, n_tiles > 1 ? 0 : -1};
      int last_v = 0;
      for (int t = 1; t < n_tiles; ++t) {
        if (!mbar_wait(&bars->empty2, (t - 1) & 1, abort, p.err, 108)) break;
        issue_v(t);
        last_v = t & 1;
        if (t + 1 < n_tiles) {
          const int buf = (t + 1) & 1;
          const uint32_t ph = ((t + 1) >> 1) & 1;
          if (!mbar_wait(&bars->empty[buf], ph ^ 1, abort, p.err, 109)) break;
          issue_k(t + 1);
          last_k[buf] = ph;
        }
      }
      volatile int no_abort = 0;
      mbar_wait(&bars->res_full, 0, &no_abort, p.err, 110);
      mbar_wait(&bars->full2, last_v, &no_abort, p.err, 110);
      for (int s = 0; s < 2; ++s)
        if (last_k[s] >= 0) mbar_wait(&bars->full[s], last_k[s], &no_abort, p.err, 110);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(smem + L::kQ), do_addr = smem_u32(smem + L::kDo);
      const uint32_t v_addr = smem_u32(smem + L::kV);
      auto k_addr = [&](int buf) { return smem_u32(smem + L::kK0 + buf * kTileSub); };
      bool ok = mbar_wait(&bars->res_full, 0, abort, p.err, 111);
      if (ok) ok = mbar_wait(&bars->full[0], 0, abort, p.err, 112);
      if (ok) {
        tc_fence_after();
        issue_x256(tmem, 0, q_addr, k_addr(0));  // S = Q K^T
        mma_commit(&bars->s_full);
      }
      if (ok) ok = mbar_wait(&bars->full2, 0, abort, p.err, 112);
      if (ok) {
        tc_fence_after();
        issue_x256(tmem, 64, do_addr, v_addr);  // dP = dO V^T
        mma_commit(&bars->dp_full);
        mma_commit(&bars->empty2);
      }
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < n_tiles) {
          if (!(ok = mbar_wait(&bars->full[buf ^ 1], ((t + 1) >> 1) & 1, abort, p.err, 113))) break;
          if (!(ok = mbar_wait(&bars->s_free, t & 1, abort, p.err, 114))) break;
          tc_fence_after();
          issue_x256(tmem, 0, q_addr, k_addr(buf ^ 1));
          mma_commit(&bars->s_full);
          if (!(ok = mbar_wait(&bars->full2, (t + 1) & 1, abort, p.err, 115))) break;
          if (!(ok = mbar_wait(&bars->dp_free, t & 1, abort, p.err, 116))) break;
          tc_fence_after();
          issue_x256(tmem, 64, do_addr, v_addr);
          mma_commit(&bars->dp_full);
          mma_commit(&bars->empty2);
        }
        if (!(ok = mbar_wait(&bars->x_full[buf], (t >> 1) & 1, abort, p.err, 117))) break;
        tc_fence_after();
        issue_acc256(tmem, 128 + 32 * buf, k_addr(buf), t > 0);  // dQ += dS K
        mma_commit(&bars->empty[buf]);
        mma_commit(&bars->x_free[buf]);
      }
      if (ok) mma_commit(&bars->o_full);
      mma_commit(&bars->drain);
      volatile int no_abort = 0;
      mbar_wait(&bars->drain, 0, &no_abort, p.err, 118);
    }
  } else {
    // ---------------------------------------------------------------- dS
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
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int buf = t & 1;
      const int kv0 = (t_begin + t) * kSub;
      const bool full = kv0 >= lo_last && kv0 + kSub - 1 <= hi_first;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full, t & 1, abort, p.err, 119));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->dp_full, t & 1, abort, p.err, 120));
      if (!ok) break;
      tc_fence_after();
      float pv[16], dp[16];
      tmem_ld_16x256b_x4(t_lane + 32 * ch, pv);
      tmem_ld_16x256b_x4(t_lane + 64 + 32 * ch, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->s_free);
      mbar_arrive(&bars->dp_free);
      uint32_t pk[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int col = kv0 + 32 * ch + 8 * k + 2 * m4;
        float x0 = fmaf(pv[4 * k], sc, -ria.x), x1 = fmaf(pv[4 * k + 1], sc, -ria.x);
        float x2 = fmaf(pv[4 * k + 2], sc, -rib.x), x3 = fmaf(pv[4 * k + 3], sc, -rib.x);
        if (!full) {
          if (col < lo_a || col > hi_a) x0 = -INFINITY;
          if (col + 1 < lo_a || col + 1 > hi_a) x1 = -INFINITY;
          if (col < lo_b || col > hi_b) x2 = -INFINITY;
          if (col + 1 < lo_b || col + 1 > hi_b) x3 = -INFINITY;
        }
        pk[2 * k] = pack_bf16x2(ex2_approx(x0) * (dp[4 * k] - ria.y), ex2_approx(x1) * (dp[4 * k + 1] - ria.y));
        pk[2 * k + 1] = pack_bf16x2(ex2_approx(x2) * (dp[4 * k + 2] - rib.y), ex2_approx(x3) * (dp[4 * k + 3] - rib.y));
      }
      if (t >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars->x_free[buf], ((t - 2) >> 1) & 1, abort, p.err, 121));
        if (!ok) break;
        tc_fence_after();
      }
      tmem_st_16x128b_x4(t_lane + 128 + 32 * buf + 16 * ch, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->x_full[buf]);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort, p.err, 122));
    if (ok) {
      tc_fence_after();
      float* dqa = p.dq_hat + ((size_t)(b * p.S + r0 + ra) * p.Hq + h) * kD;
      float* dqb = p.dq_hat + ((size_t)(b * p.S + r0 + rb) * p.Hq + h) * kD;
      store_acc256<true>(t_lane, ch, m4, dqa, dqb, valid_a, valid_b, p.inv_sqrt_d);
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

// ================================================================ launchers
template <class Kernel, class... Args>
static cudaError_t launch_256(Kernel* kernel, int alloc, std::atomic<uint64_t>& configured, unsigned grid,
                              cudaStream_t st, const Args&... args) {
  const cudaError_t e = ensure_dynamic_smem(kernel, alloc, configured);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kBwdThreads, alloc, st>>>(args...);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dv256(const BwdParams& p, const CUtensorMap& tq64, const CUtensorMap& tdo64,
                             const CUtensorMap& tk, cudaStream_t st) {
  static_assert(Dv256Layout::kAlloc <= 232448, "shared memory budget");
  static std::atomic<uint64_t> configured{0};
  return launch_256(bwd_dv256_kernel, Dv256Layout::kAlloc, configured, (unsigned)p.n_kvtiles * p.B * p.Hkv, st,
                    tq64, tdo64, tk, p);
}

cudaError_t launch_bwd_dk256(const BwdParams& p, const CUtensorMap& tq64, const CUtensorMap& tdo64,
                             const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t st) {
  static_assert(Dk256Layout::kAlloc <= 232448, "shared memory budget");
  static std::atomic<uint64_t> configured{0};
  return launch_256(bwd_dk256_kernel, Dk256Layout::kAlloc, configured, (unsigned)p.n_kvtiles * p.B * p.Hkv, st,
                    tq64, tdo64, tk, tv, p);
}

cudaError_t launch_bwd_dq256(const BwdParams& p, const CUtensorMap& tq, const CUtensorMap& tdo,
                             const CUtensorMap& tk64, const CUtensorMap& tv64, cudaStream_t st) {
  static_assert(Dq256Layout::kAlloc <= 232448, "shared memory budget");
  static std::atomic<uint64_t> configured{0};
  return launch_256(bwd_dq256_kernel, Dq256Layout::kAlloc, configured, (unsigned)p.n_qtiles * p.B * p.Hq, st, tq,
                    tdo, tk64, tv64, p);
}

}  // namespace g3
