// grad_quant.cuh -- the backward pass's quantizer arithmetic: E5M2 gradient
// codes by the per-32 MX rule with E5M2's largest finite value, rounded to
// nearest even or stochastically with counter-based (Philox4x64-10) draws.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

#include "mx_quant.cuh"

namespace bq {

// Gradient form (E5M2 codes): the same rule with E5M2's largest finite value
// 57344 in place of 448 (fp32(1/57344) = fp32(1/448) * 2^-7), rounding to
// nearest even or stochastically between the two neighbouring E5M2 values.
__device__ __forceinline__ int mx_exponent_e5m2(uint32_t amax_bits) {
  const float amax = fmaxf(__uint_as_float(amax_bits << 16), 1e-4f);
  const float t = __fmul_rn(amax, __uint_as_float(0x37924925u));  // fp32(1/57344)
  const uint32_t tb = __float_as_uint(t);
  return static_cast<int>((tb >> 23) & 0xFFu) - 127 + ((tb & 0x7FFFFFu) != 0u ? 1 : 0);
}

__device__ __forceinline__ uint32_t e5m2x2(float a, float b) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E5M2));
}

// Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC 2011), counter (c0, 0, 0, 0), key (k0, 0): ten rounds
// of two 64 x 64 -> 128-bit products, the key bumped by the Weyl constants
// between rounds.
struct Philox4 {
  uint64_t w[4];
};

__device__ __forceinline__ Philox4 philox4x64_10(uint64_t c0, uint64_t k0) {
  uint64_t x0 = c0, x1 = 0, x2 = 0, x3 = 0, k1 = 0;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B97F4A7C15ull;
      k1 += 0xBB67AE8584CAA73Bull;
    }
    const uint64_t a = 0xD2E7470EE14C6C93ull * x0, ah = __umul64hi(0xD2E7470EE14C6C93ull, x0);
    const uint64_t b = 0xCA5A826395121157ull * x2, bh = __umul64hi(0xCA5A826395121157ull, x2);
    x0 = bh ^ x1 ^ k0;
    x1 = b;
    x2 = ah ^ x3 ^ k1;
    x3 = a;
  }
  return Philox4{{x0, x1, x2, x3}};
}

// Stochastic E5M2 rounding of y (|y| <= 57344) with the element's Philox
// word: lo and hi are the E5M2 magnitudes around |y| -- truncation to two
// mantissa bits for |y| >= 2^-14, the 2^-16 grid below -- and the result is
// hi when u < (|y| - lo) / (hi - lo), u = (word >> 11) * 2^-53 the draw, with
// y's sign; returns the code byte.  |y| - lo is exact (lo truncates |y| on its
// own grid) and hi - lo is a power of two, so the fraction d is exact in fp32;
// u < d is decided exactly in integers as (word >> 11) < ceil(d * 2^53).
__device__ __forceinline__ uint32_t e5m2_sr(float y, uint64_t word) {
  const float a = fabsf(y);
  float lo, step, inv_step;
  if (a >= 0x1.0p-14f) {
    const uint32_t eb = __float_as_uint(a) & 0x7F800000u;  // 2^exp of |y|
    lo = __uint_as_float(__float_as_uint(a) & ~((1u << 21) - 1u));
    step = __uint_as_float(eb - (2u << 23));                     // 2^(exp - 2)
    inv_step = __uint_as_float((254u << 23) - eb + (2u << 23));  // 2^(2 - exp)
  } else {
    lo = floorf(a * 65536.0f) * 0x1.0p-16f;
    step = 0x1.0p-16f;
    inv_step = 65536.0f;
  }
  const float d = __fmul_rn(a - lo, inv_step);                     // in [0, 1), exact
  const uint64_t thr = __float2ull_rz(ceilf(__fmul_rn(d, 0x1.0p53f)));  // exact integer
  const float m = ((word >> 11) < thr) ? lo + step : lo;               // an E5M2 value
  return e5m2x2(copysignf(m, y), 0.0f) & 0xFFu;
}

}  // namespace bq
