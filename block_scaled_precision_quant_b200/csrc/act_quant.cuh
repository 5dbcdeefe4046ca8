// act_quant.cuh -- per-32 MX activation quantization and the scale-factor
// layout kernels (prepack / unpack) for sm_100a.
//
// Quantizer ("formats.py" page: act_scale, act_quant, _log2_ceil_pow2 and the
// module docstring "act_qdq reproduces ..."), for each 32 consecutive
// elements of a row:
//   amax = max(max|x|, fp32(1e-4));  t = fp32(amax * fp32(1/448))
//   e    = ceil(log2 t) from t's exponent bits;  scale byte = e + 127
//   q    = E4M3 round-to-nearest-even of clamp(x / 2^e, -448, 448)
// x / 2^e is computed as x * 2^-e: 2^-e is an exact binary32 power of two for
// every e the rule can produce (-22 .. 120), so the correctly rounded product
// equals the correctly rounded quotient.
//
// Work split: one warp per 512 consecutive elements of one row (16 groups);
// a thread owns half a group (16 bf16 = two 16-byte loads), the two halves
// meet through one shuffle.  The scale bytes of 4 consecutive groups are
// gathered by shuffles into one 32-bit store in the MMA scale layout.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "bq_ptx.cuh"

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

// grid: x*8 + warp = row, y = chunk of 16 groups within the row.  Rows in
// [M, rows_pad) only write padding scale bytes (127).
__global__ void __launch_bounds__(256) act_quant_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t M, int64_t K, int64_t ldx, int64_t rows_pad,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf_mma, uint8_t *__restrict__ sf_row,
    int *__restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows_pad) return;
  const int64_t G = K >> 5;            // groups per row
  const int64_t katoms = (G + 3) >> 2;
  const int64_t g = static_cast<int64_t>(blockIdx.y) * 16 + (lane >> 1);  // this lane's group
  const int half = lane & 1;

  // Every lane runs the shuffles below (full-warp masks); lanes without data
  // (past the row's last group, or padding rows) carry zeros through them.
  const bool active = row < M && g < G;
  const int64_t col = g * 32 + half * 16;
  uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  // Programmatic dependent launch: x may come from the kernel before this one;
  // the kernel after this one (the GEMM) may begin its prologue now.
  griddep_wait();
  griddep_launch_dependents();
  if (active) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + row * ldx + col);
    const uint4 v0 = __ldg(src);
    const uint4 v1 = __ldg(src + 1);
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  }
  // amax over |x| as an integer max of the magnitude bits (order-preserving
  // for non-negative floats); non-finite detection from the exponent bits.
  uint32_t mx = 0, bad = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = w[i] & 0x7FFFu, hi = (w[i] >> 16) & 0x7FFFu;
    mx = max(mx, max(lo, hi));
    bad |= ((lo & 0x7F80u) == 0x7F80u) | ((hi & 0x7F80u) == 0x7F80u);
  }
  mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  uint32_t sbyte = 127;
  if (active) {
    if (bad && status) atomicOr(status, 1);
    const float amax = fmaxf(__uint_as_float(mx << 16), 1e-4f);
    const float t = __fmul_rn(amax, __uint_as_float(0x3B124925u));  // fp32(1/448)
    const uint32_t tb = __float_as_uint(t);
    const int e = static_cast<int>((tb >> 23) & 0xFFu) - 127 + ((tb & 0x7FFFFFu) != 0u ? 1 : 0);
    sbyte = static_cast<uint32_t>(e + 127);
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e
    float f[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      f[2 * i] = fminf(fmaxf(__fmul_rn(__uint_as_float(w[i] << 16), inv), -448.0f), 448.0f);
      f[2 * i + 1] =
          fminf(fmaxf(__fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv), -448.0f), 448.0f);
    }
    uint4 out;
    out.x = e4m3x4(f[0], f[1], f[2], f[3]);
    out.y = e4m3x4(f[4], f[5], f[6], f[7]);
    out.z = e4m3x4(f[8], f[9], f[10], f[11]);
    out.w = e4m3x4(f[12], f[13], f[14], f[15]);
    *reinterpret_cast<uint4 *>(q + row * K + col) = out;
    if (sf_row && half == 0) sf_row[row * G + g] = static_cast<uint8_t>(sbyte);
  }
  // Gather the bytes of groups 4j..4j+3 of this chunk (lanes 8j, 8j+2, 8j+4,
  // 8j+6) and store them as one word; groups past G (column padding) and rows
  // past M (row padding) keep 127.
  const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 2);
  const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 4);
  const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 6);
  if ((lane & 7) == 0) {
    const int64_t g4 = g;  // multiple of 4
    if (g4 < katoms * 4) {
      const uint32_t word = sbyte | (b1 << 8) | (b2 << 16) | (b3 << 24);
      *reinterpret_cast<uint32_t *>(sf_mma + sf_mma_offset(row, g4, katoms)) = word;
    }
  }
}

// Row-major scales (ROW32: [N, G]; BLK32x32: [ceil(N/32), G] repeated over
// the 32 rows of each block) -> MMA layout with 127 padding.  One thread per
// output 32-bit word (4 scale columns of one row).  Flags 255 bytes in
// flags bit 0.
__global__ void pack_scales_kernel(const uint8_t *__restrict__ src, int kind, int64_t N, int64_t G,
                                   int64_t rows_pad, uint8_t *__restrict__ dst,
                                   int *__restrict__ flags) {
  const int64_t katoms = (G + 3) >> 2;
  const int64_t words = rows_pad * katoms;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < words;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / katoms;
    const int64_t c0 = (i - r * katoms) * 4;
    uint32_t word = 0;
    bool nan = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t b = 127;
      const int64_t c = c0 + j;
      if (r < N && c < G) {
        b = (kind == 0) ? src[r * G + c] : src[(r >> 5) * G + c];
        nan |= (b == 255u);
      }
      word |= b << (8 * j);
    }
    if (nan) atomicOr(flags, 1);
    *reinterpret_cast<uint32_t *>(dst + sf_mma_offset(r, c0, katoms)) = word;
  }
}

// Flags E4M3 NaN codes (0x7F / 0xFF) in flags bit 1.  n bytes, 16-byte aligned.
__global__ void scan_e4m3_nan_kernel(const uint8_t *__restrict__ codes, int64_t n,
                                     int *__restrict__ flags) {
  bool nan = false;
  const int64_t nv = n >> 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nv;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(codes) + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 16; ++j) nan |= ((w[j >> 2] >> (8 * (j & 3))) & 0x7Fu) == 0x7Fu;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t i = nv << 4; i < n; ++i) nan |= ((codes[i] & 0x7F) == 0x7F);
  }
  if (nan) atomicOr(flags, 2);
}

__global__ void unpack_scales_kernel(const uint8_t *__restrict__ src, int64_t rows, int64_t G,
                                     uint8_t *__restrict__ dst) {
  const int64_t katoms = (G + 3) >> 2;
  const int64_t total = rows * G;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / G, c = i - (i / G) * G;
    dst[i] = src[sf_mma_offset(r, c, katoms)];
  }
}

}  // namespace bq
