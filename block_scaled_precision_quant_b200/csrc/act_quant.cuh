// act_quant.cuh -- per-32 MX activation quantization and the scale-factor
// layout kernels (prepack / unpack) for sm_100a.
//
// Quantizer ("formats.py" page: act_scale, act_quant, _log2_ceil_pow2 and the
// module docstring "act_qdq reproduces ..."), per 32 consecutive elements of
// a row; the arithmetic is in mx_quant.cuh.
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
#include "mx_quant.cuh"

namespace bq {

// grid: x*8 + warp = row, y = chunk of 16 groups within the row.  Rows in
// [M, rows_pad) only write padding scale bytes (127).  FP4: E2M1 codes
// (packed [M, K/2], the per-32 rule with 6 in place of 448) instead of E4M3.
template <bool FP4>
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
  // amax of the two half-groups met through one shuffle
  uint32_t bad = 0;
  uint32_t mx = bf16_amax_bits(w, bad);
  mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  uint32_t sbyte = 127;
  if (active) {
    if (bad && status) atomicOr(status, 1);
    const int e = FP4 ? mx_exponent_fp4(mx) : mx_exponent(mx);
    sbyte = static_cast<uint32_t>(e + 127);
    if constexpr (FP4) {
      uint32_t c[2];
      mx_encode_fp4(w, e, c);
      *reinterpret_cast<uint2 *>(q + row * (K >> 1) + (col >> 1)) = make_uint2(c[0], c[1]);
    } else {
      uint32_t c[4];
      mx_encode(w, e, c);
      *reinterpret_cast<uint4 *>(q + row * K + col) = make_uint4(c[0], c[1], c[2], c[3]);
    }
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
