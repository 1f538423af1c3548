// philox.cuh -- Philox4x64-10 on the device.
//
// Counter-based generator of Salmon, Moraes, Dror and Shaw, "Parallel random
// numbers: as easy as 1, 2, 3" (SC'11): ten rounds of the Philox bijection on
// four 64-bit words, the two-word key advanced by the Weyl constants between
// rounds.  The Random Attention article ("Random Attention：不判断重要性，只随机
// 保留") needs one random draw per (head, position) and round; a counter-based
// generator gives it with no state: counter = (position, head, layer,
// request), key = (seed, round).
#pragma once
#include <stdint.h>

namespace kvc {

__device__ __forceinline__ uint32_t philox4x64_10_word0_hi32(uint64_t x0, uint64_t x1,
                                                             uint64_t x2, uint64_t x3,
                                                             uint64_t k0, uint64_t k1) {
  constexpr uint64_t kM0 = 0xD2E7470EE14C6C93ULL, kM1 = 0xCA5A826395121157ULL;
  constexpr uint64_t kW0 = 0x9E3779B97F4A7C15ULL, kW1 = 0xBB67AE8584CAA73BULL;
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    if (i > 0) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint64_t p0hi = __umul64hi(kM0, x0), p0lo = kM0 * x0;
    const uint64_t p1hi = __umul64hi(kM1, x2), p1lo = kM1 * x2;
    const uint64_t n0 = p1hi ^ x1 ^ k0;
    const uint64_t n2 = p0hi ^ x3 ^ k1;
    x0 = n0;
    x1 = p1lo;
    x2 = n2;
    x3 = p0lo;
  }
  return static_cast<uint32_t>(x0 >> 32);
}

}  // namespace kvc
