// Warp roles and thread layout shared by the tensor-core kernels of the
// prefill backward (backward.cu: head dims 64 and 128; backward256.cu: head
// dim 256).
#pragma once

#include <cstdint>

namespace g3 {

// Warp 0 TMA producer, warp 1 tensor-memory owner and tcgen05.mma issuer,
// warps 2-17 the elementwise work.  The elementwise step needs no row
// reduction (lse and delta are known), so the columns of a tile are split
// between two warps: four warps per TMEM lane quarter, each on 16 rows and
// one column half; thread t holds rows t/4 and t/4+8 of its slice.
constexpr int kBwdEwWarps = 16;
constexpr int kBwdThreads = (2 + kBwdEwWarps) * 32;
constexpr int kBwdEwThreads = kBwdEwWarps * 32;
constexpr int kBwdFirstWarp = 2;

// Elementwise warp e = warp - 2: TMEM lane quarter warp % 4 (hardware rule),
// 16-row half (e >> 2) & 1, column half e >> 3.
__device__ __forceinline__ int bwd_lane_base(int warp) {
  return (warp & 3) * 32 + (((warp - kBwdFirstWarp) >> 2) & 1) * 16;
}
__device__ __forceinline__ int bwd_col_half(int warp) { return (warp - kBwdFirstWarp) >> 3; }

constexpr int kBwdSwizzleBlock = 128 * 64 * 2;  // 128 rows x 64 bf16 (one 128-byte swizzle column)

}  // namespace g3
