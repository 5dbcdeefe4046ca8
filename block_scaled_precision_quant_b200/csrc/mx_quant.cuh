// mx_quant.cuh -- the per-32 MX quantizer's arithmetic, shared by the
// activation quantizer kernel and the GEMM epilogue that emits its output in
// the same format.
//
// The quantizer ("formats.py" page: act_scale, act_quant, _log2_ceil_pow2):
//   amax = max(max|x|, fp32(1e-4));  t = fp32(amax * fp32(1/448))
//   e    = ceil(log2 t) from t's exponent bits;  scale byte = e + 127
//   q    = E4M3 round-to-nearest-even of clamp(x / 2^e, -448, 448)
// x / 2^e is computed as x * 2^-e: 2^-e is an exact binary32 power of two for
// every e the rule can produce (-22 .. 120), so the correctly rounded product
// equals the correctly rounded quotient.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace bq {

// Byte offset of scale (row r, column c) in an MMA-layout buffer with
// `katoms` = ceil(G / 4) atoms per 128-row band.
__host__ __device__ __forceinline__ int64_t sf_mma_offset(int64_t r, int64_t c, int64_t katoms) {
  return ((r >> 7) * katoms + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// The value of a non-negative finite E4M3 byte.
__device__ __forceinline__ float e4m3_value(uint32_t byte) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(byte), __NV_E4M3);
  return __half2float(__half(h));
}

// The smallest positive E4M3 value >= t (t >= 0): the nearest one, moved up
// one code when below t; at least 2^-9 (byte 1), at most 448 (byte 0x7E).
__device__ __forceinline__ uint32_t e4m3_ceil(float t) {
  uint32_t b = e4m3x2(t, 0.0f) & 0xFFu;  // nearest, saturating at 448
  if (b < 0x7Eu && e4m3_value(b) < t) ++b;
  return b < 1u ? 1u : b;
}

// Per-halfword unsigned maximum of two words of 16-bit pairs.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Largest magnitude bits (15 bits, sign dropped) of the bf16 pairs in w: an
// integer max is order-preserving for non-negative floats, taken on both
// halves of each word at once.  `bad` collects non-finite inputs: a value has
// an all-ones exponent exactly when its magnitude bits are >= 0x7F80, so the
// largest magnitude tells whether any of them has.
template <int NW>
__device__ __forceinline__ uint32_t bf16_amax_bits(const uint32_t (&w)[NW], uint32_t &bad) {
  uint32_t m = w[0] & 0x7FFF7FFFu;
#pragma unroll
  for (int i = 1; i < NW; ++i) m = max_u16x2(m, w[i] & 0x7FFF7FFFu);
  const uint32_t mx = max(m & 0xFFFFu, m >> 16);
  bad |= mx >= 0x7F80u ? 1u : 0u;
  return mx;
}

// Scale exponent e of a group from its amax bits.  Finite bf16 input gives
// e <= 120 (amax = the largest bf16, byte 247); a group holding an Inf would
// give 128 (byte 255, the NaN scale), so e is capped at 120: such a group,
// which every caller reports as non-finite, still gets a valid scale byte
// (its Inf codes saturate to +-448, a NaN input stays a NaN code), and a GEMM
// that consumes it never meets the NaN scale.
__device__ __forceinline__ int mx_exponent(uint32_t amax_bits) {
  const float amax = fmaxf(__uint_as_float(amax_bits << 16), 1e-4f);
  const float t = __fmul_rn(amax, __uint_as_float(0x3B124925u));  // fp32(1/448)
  const uint32_t tb = __float_as_uint(t);
  const int e = static_cast<int>((tb >> 23) & 0xFFu) - 127 + ((tb & 0x7FFFFFu) != 0u ? 1 : 0);
  return min(e, 120);
}

// E4M3 codes of the 2 * NW bf16 values in w (element 2i in the low half of
// word i) scaled by 2^-e, four codes per output word.  The clamp to +-448 is
// the conversion's saturation: a finite value above 448 (below 464 it rounds
// to 448 anyway) becomes 448 with its sign, which is what clamping first and
// rounding gives.
template <int NW>
__device__ __forceinline__ void mx_encode(const uint32_t (&w)[NW], int e,
                                          uint32_t (&codes)[NW / 2]) {
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e
#pragma unroll
  for (int i = 0; i < NW / 2; ++i) {
    float f[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t word = w[2 * i + j];
      f[2 * j] = __fmul_rn(__uint_as_float(word << 16), inv);
      f[2 * j + 1] = __fmul_rn(__uint_as_float(word & 0xFFFF0000u), inv);
    }
    codes[i] = e4m3x4(f[0], f[1], f[2], f[3]);
  }
}

// MXFP4 form of the quantizer (E2M1 codes): the same rule with the E2M1
// maximum 6 in place of 448,
//   t = fp32(amax * fp32(1/6)),  e = ceil(log2 t),  q = E2M1_RNE(clamp(x / 2^e, -6, 6)),
// codes packed two per byte with the even element in the low nibble.
// Capped at 126 (the largest bf16 gives 126, byte 253) for the same reason
// as mx_exponent.
__device__ __forceinline__ int mx_exponent_fp4(uint32_t amax_bits) {
  const float amax = fmaxf(__uint_as_float(amax_bits << 16), 1e-4f);
  const float t = __fmul_rn(amax, __uint_as_float(0x3E2AAAABu));  // fp32(1/6)
  const uint32_t tb = __float_as_uint(t);
  const int e = static_cast<int>((tb >> 23) & 0xFFu) - 127 + ((tb & 0x7FFFFFu) != 0u ? 1 : 0);
  return min(e, 126);
}

// One byte of two E2M1 codes for the bf16 pair in `word` (element 2i in the
// low half) scaled by inv = 2^-e: round to nearest even with saturation at
// +-6 (the clamp), then each code's sign bit set from its input, so that
// negative values that round to zero keep their sign (-0, code 8).
__device__ __forceinline__ uint32_t e2m1x2_byte(uint32_t word, float inv) {
  const float lo = __fmul_rn(__uint_as_float(word << 16), inv);
  const float hi = __fmul_rn(__uint_as_float(word & 0xFFFF0000u), inv);
  const uint32_t b = static_cast<uint32_t>(
      __nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest));
  return (b & 0xFFu) | ((word >> 12) & 0x8u) | ((word >> 24) & 0x80u);
}

// Packed E2M1 bytes of the 2 * NW bf16 values in w, four bytes per word.
template <int NW>
__device__ __forceinline__ void mx_encode_fp4(const uint32_t (&w)[NW], int e,
                                              uint32_t (&packed)[NW / 4]) {
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e
#pragma unroll
  for (int i = 0; i < NW / 4; ++i)
    packed[i] = e2m1x2_byte(w[4 * i], inv) | (e2m1x2_byte(w[4 * i + 1], inv) << 8) |
                (e2m1x2_byte(w[4 * i + 2], inv) << 16) | (e2m1x2_byte(w[4 * i + 3], inv) << 24);
}

}  // namespace bq
