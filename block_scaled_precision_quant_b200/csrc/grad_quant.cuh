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
// Capped at 113 (the largest bf16 gives 113, byte 240) as mx_exponent is.
__device__ __forceinline__ int mx_exponent_e5m2(uint32_t amax_bits) {
  const float amax = fmaxf(__uint_as_float(amax_bits << 16), 1e-4f);
  const float t = __fmul_rn(amax, __uint_as_float(0x37924925u));  // fp32(1/57344)
  const uint32_t tb = __float_as_uint(t);
  const int e = static_cast<int>((tb >> 23) & 0xFFu) - 127 + ((tb & 0x7FFFFFu) != 0u ? 1 : 0);
  return min(e, 113);
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

// The draw of element j (0..7) of a Philox block: the 32-bit half (j % 2, low
// half first) of word j / 2.  A block at counter i / 8 serves elements i with
// the same i / 8.
__device__ __forceinline__ uint32_t philox_draw(const Philox4 &r, int j) {
  const uint64_t w = r.w[(j >> 1) & 3];
  return (j & 1) ? static_cast<uint32_t>(w >> 32) : static_cast<uint32_t>(w);
}

// Stochastic E5M2 rounding of y (|y| <= 57344) with the element's 32-bit
// draw: lo and hi are the E5M2 magnitudes around |y| and the result is hi when
// u < (|y| - lo) / (hi - lo), u = draw * 2^-32, with y's sign; returns the code
// byte.
//   |y| >= 2^-14 (E5M2 normal): lo is |y| truncated to two mantissa bits, its
//     code (exponent rebiased from 127 to 15, two mantissa bits) is read off
//     the fp32 bits, and the fraction is k / 2^21 with k the 21 dropped
//     mantissa bits, so u < d exactly when (draw >> 11) < k.
//   |y| < 2^-14 (E5M2 subnormal, step 2^-16): t = |y| 2^16 is exact, lo = floor
//     t, the fraction t - lo is exact in fp32 and compared with the draw
//     exactly as draw < ceil(frac 2^32).
__device__ __forceinline__ uint32_t e5m2_sr(float y, uint32_t draw) {
  const uint32_t bits = __float_as_uint(y);
  const uint32_t sign = (bits >> 24) & 0x80u;
  const uint32_t mag = bits & 0x7FFFFFFFu;
  uint32_t code;
  if (mag >= 0x38800000u) {  // 2^-14
    const uint32_t k = mag & 0x1FFFFFu;
    code = (mag >> 21) - (112u << 2) + ((draw >> 11) < k ? 1u : 0u);
  } else {
    const float t = __fmul_rn(__uint_as_float(mag), 65536.0f);
    const float lo = floorf(t);
    const float frac = t - lo;
    const uint64_t thr = __float2ull_rz(ceilf(__fmul_rn(frac, 0x1.0p32f)));
    code = static_cast<uint32_t>(lo) + (static_cast<uint64_t>(draw) < thr ? 1u : 0u);
  }
  return sign | code;
}

}  // namespace bq
