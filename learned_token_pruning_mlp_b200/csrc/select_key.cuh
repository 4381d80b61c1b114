// select_key.cuh -- the order key of the top-K selector, shared by the selector and
// by the gate epilogue that histograms it (the two must agree bit for bit).
#pragma once
#include <cstdint>

namespace tg {

// Order key: larger key = earlier in (score desc, NaN last).  0 marks a question
// token (never competes), 1 is NaN, every number maps to >= 0x007FFFFF; -0.0 ranks
// with +0.0.
__device__ __forceinline__ uint32_t order_key(float f, bool doc) {
  if (!doc) return 0u;
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7FFFFFFFu) > 0x7F800000u) return 1u;  // NaN
  if (b == 0x80000000u) b = 0u;                      // -0.0 ranks with +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

}  // namespace tg
