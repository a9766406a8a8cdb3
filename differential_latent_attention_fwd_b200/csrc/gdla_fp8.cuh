// MXFP8 latent-cache rows: the report's low-precision storage format (paperglide.net summary,
// the low-precision paragraph and the Figure 3 caption: MXFP8, i.e. blocks of 32 values that
// share one power-of-two scale, each value in FP8 E4M3).  A latent row (576 values: normalised
// c^KV | rotated k^R) is stored in 608 bytes:
//   bytes   0 .. 575  E4M3 codes of the values v / 2^k(block)      (block b = values 32 b .. 32 b + 31)
//   bytes 576 .. 593  one byte per block: k + 127                  (scale 2^k)
//   bytes 594 .. 607  zero
// k is the smallest integer with max|v| <= 448 2^k over the block (clamped to [-127, 127]; an
// all-zero block takes -127), so nothing is clipped; the values are rounded to the nearest E4M3
// value, ties to even.  The values quantized are the bf16 latent values (what a bf16 cache
// would hold), so the stored bytes are a function of those bf16 numbers alone.
#pragma once
#include "gdla_common.cuh"

namespace gdla {

constexpr int FP8_ROW_BYTES = 608;
constexpr int FP8_ROW_VALUES = 576;
constexpr int FP8_SCALE_OFF = 576;

// Smallest k with amax <= 448 * 2^k: with amax = f 2^e (f in [0.5, 1)), 448 2^(e - 9) = 0.875 2^e.
__device__ __forceinline__ int mx_block_exp(float amax) {
  if (!(amax > 0.f)) return -127;
  int e;
  const float f = frexpf(amax, &e);
  const int k = e - 9 + (f > 0.875f ? 1 : 0);
  return k < -127 ? -127 : (k > 127 ? 127 : k);
}

// Two values (already divided by the block scale) -> two E4M3 codes, lo in the low byte.
__device__ __forceinline__ uint16_t e4m3x2_from(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// Two E4M3 codes (lo in the low byte) -> f16x2 (exact).
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint16_t v) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(v));
  return d;
}

// 2^k as a float for k in [-127, 127] (2^-127 is subnormal, exact).
__device__ __forceinline__ float exp2i(int k) { return ldexpf(1.0f, k); }

}  // namespace gdla
