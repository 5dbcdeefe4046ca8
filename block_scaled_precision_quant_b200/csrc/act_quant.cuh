// act_quant.cuh -- per-32 MX activation quantization and the scale-factor
// layout kernels (prepack / unpack) for sm_100a.
//
// Quantizer ("formats.py" page: act_scale, act_quant, _log2_ceil_pow2 and the
// module docstring's description of act_qdq), per 32 consecutive elements of
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
#include "grad_quant.cuh"
#include "mx_quant.cuh"

namespace bq {

// Code formats of the quantizers.
enum QuantFmt : int { kQE4M3 = 0, kQFP4 = 1, kQE5M2 = 2 };

// E5M2 codes of 16 bf16 values (8 words, element 2i in the low half of word
// i) scaled by 2^-e; SR: stochastic rounding with the draws of elements
// idx0 .. idx0 + 15 (idx0 a multiple of 8: two Philox blocks) under `seed`.
template <bool SR>
__device__ __forceinline__ void e5m2_encode16(const uint32_t (&w)[8], int e, uint64_t seed,
                                              uint64_t idx0, uint32_t (&codes)[4]) {
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e
  Philox4 r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float f[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t word = w[2 * i + j];
      f[2 * j] = fminf(fmaxf(__fmul_rn(__uint_as_float(word << 16), inv), -57344.0f), 57344.0f);
      f[2 * j + 1] =
          fminf(fmaxf(__fmul_rn(__uint_as_float(word & 0xFFFF0000u), inv), -57344.0f), 57344.0f);
    }
    if constexpr (SR) {
      if (i % 2 == 0) r = philox4x64_10((idx0 >> 3) + (i >> 1), seed);
      const int j0 = (4 * i) & 7;
      codes[i] = e5m2_sr(f[0], philox_draw(r, j0)) | (e5m2_sr(f[1], philox_draw(r, j0 + 1)) << 8) |
                 (e5m2_sr(f[2], philox_draw(r, j0 + 2)) << 16) |
                 (e5m2_sr(f[3], philox_draw(r, j0 + 3)) << 24);
    } else {
      codes[i] = e5m2x2(f[0], f[1]) | (e5m2x2(f[2], f[3]) << 16);
    }
  }
}

// One warp's share of one row in act_quant_kernel: lane 2i + h holds half h
// (16 bf16 values, 8 words) of group g = chunk * 16 + i; `active` is false for
// padding rows and for groups past the row's end, whose lanes carry zeros
// through the full-warp shuffles.
template <int FMT, bool SR>
__device__ __forceinline__ void act_quant_row_part(const uint32_t (&w)[8], int64_t row, bool active,
                                                   int lane, int64_t g, int64_t col, int64_t K,
                                                   int64_t G, int64_t katoms,
                                                   uint8_t *__restrict__ q,
                                                   uint8_t *__restrict__ sf_mma,
                                                   uint8_t *__restrict__ sf_row,
                                                   int *__restrict__ status, uint64_t seed) {
  const int half = lane & 1;
  // amax of the two half-groups met through one shuffle
  uint32_t bad = 0;
  uint32_t mx = bf16_amax_bits(w, bad);
  mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
  uint32_t sbyte = 127;
  if (active) {
    if (bad && status) atomicOr(status, 1);
    const int e = FMT == kQFP4    ? mx_exponent_fp4(mx)
                  : FMT == kQE5M2 ? mx_exponent_e5m2(mx)
                                  : mx_exponent(mx);
    sbyte = static_cast<uint32_t>(e + 127);
    if constexpr (FMT == kQE5M2) {
      uint32_t c[4];
      e5m2_encode16<SR>(w, e, seed, static_cast<uint64_t>(row * K + col), c);
      *reinterpret_cast<uint4 *>(q + row * K + col) = make_uint4(c[0], c[1], c[2], c[3]);
    } else if constexpr (FMT == kQFP4) {
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

// grid: x = band of 8 * R rows (warp w takes rows band * 8R + w + 8r, r < R),
// y = chunk of 16 groups within the row; rows_pad is a multiple of 8 * R.
// Each warp loads all R rows' data before quantizing any of them, so a thread
// has R x 32 bytes in flight.  Rows in [M, rows_pad) only write padding scale
// bytes (127).  FMT: E4M3 codes; FP4: E2M1 codes (packed [M, K/2], the per-32
// rule with 6 in place of 448); E5M2: gradient codes (the rule with 57344), SR
// with stochastic rounding (the draw of element (row, col) is index
// row * K + col under `seed`).
template <int FMT, bool SR = false, int R = 1>
__global__ void __launch_bounds__(256) act_quant_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t M, int64_t K, int64_t ldx, int64_t rows_pad,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf_mma, uint8_t *__restrict__ sf_row,
    int *__restrict__ status, uint64_t seed) {
  static_assert(!SR || FMT == kQE5M2, "stochastic rounding is for E5M2 gradients");
  const int lane = threadIdx.x & 31;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * (8 * R) + (threadIdx.x >> 5);
  const int64_t G = K >> 5;            // groups per row
  const int64_t katoms = (G + 3) >> 2;
  const int64_t g = static_cast<int64_t>(blockIdx.y) * 16 + (lane >> 1);  // this lane's group
  const int64_t col = g * 32 + (lane & 1) * 16;

  uint32_t w[R][8];
  // Programmatic dependent launch: x may come from the kernel before this one;
  // the kernel after this one (the GEMM) may begin its prologue now.
  griddep_wait();
  griddep_launch_dependents();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t row = row0 + 8 * r;
#pragma unroll
    for (int i = 0; i < 8; ++i) w[r][i] = 0u;
    if (row < M && g < G) {
      const uint4 *src = reinterpret_cast<const uint4 *>(x + row * ldx + col);
      const uint4 v0 = __ldg(src);
      const uint4 v1 = __ldg(src + 1);
      w[r][0] = v0.x; w[r][1] = v0.y; w[r][2] = v0.z; w[r][3] = v0.w;
      w[r][4] = v1.x; w[r][5] = v1.y; w[r][6] = v1.z; w[r][7] = v1.w;
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t row = row0 + 8 * r;  // warp-uniform
    if (row >= rows_pad) break;
    act_quant_row_part<FMT, SR>(w[r], row, row < M && g < G, lane, g, col, K, G, katoms, q,
                                sf_mma, sf_row, status, seed);
  }
}

// NVFP4 quantization: every value first fp32(x * g) (g the per-tensor scale),
// then per 16 consecutive values of a row an E4M3 scale s = the smallest E4M3
// value >= fp32(amax * fp32(1/6)) (2^-9 at least, 448 at most) and E2M1 codes
// of fp32(x / s), round to nearest even with the sign kept, packed two per
// byte (even element low).  Scales go to the MMA layout of 16-input groups
// (an atom covers 64 inputs); padding bytes are 0x38 (1.0: 127 would be an
// E4M3 NaN).  Work split as act_quant_kernel: a lane owns one group of 16.
// grid: x*8 + warp = row, y = chunk of 32 groups within the row.
__global__ void __launch_bounds__(256) nvfp4_quant_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t M, int64_t K, int64_t ldx, int64_t rows_pad,
    float gs, uint8_t *__restrict__ q, uint8_t *__restrict__ sf_mma,
    uint8_t *__restrict__ sf_row, int *__restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows_pad) return;
  const int64_t G = K >> 4;  // 16-input groups per row
  const int64_t katoms = (G + 3) >> 2;
  const int64_t grp = static_cast<int64_t>(blockIdx.y) * 32 + lane;
  const bool active = row < M && grp < G;
  const int64_t col = grp * 16;
  uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  griddep_wait();
  griddep_launch_dependents();
  if (active) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + row * ldx + col);
    const uint4 v0 = __ldg(src);
    const uint4 v1 = __ldg(src + 1);
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
  }
  uint32_t bad = 0;
  const uint32_t mx = bf16_amax_bits(w, bad);
  uint32_t sbyte = 0x38u;
  if (active) {
    if (bad && status) atomicOr(status, 1);
    // max |x g| = fp32(max|x| g): rounding is monotonic
    const float amax = __fmul_rn(__uint_as_float(mx << 16), gs);
    const float t = __fmul_rn(amax, __uint_as_float(0x3E2AAAABu));  // fp32(1/6)
    sbyte = e4m3_ceil(t);
    const float s = e4m3_value(sbyte);
    uint32_t packed[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t v = w[4 * h + j];
        const float lo = __fdiv_rn(__fmul_rn(__uint_as_float(v << 16), gs), s);
        const float hi = __fdiv_rn(__fmul_rn(__uint_as_float(v & 0xFFFF0000u), gs), s);
        const uint32_t b = static_cast<uint32_t>(
            __nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest));
        // each code's sign from its input (and g > 0), so -0 keeps its sign
        word |= ((b & 0xFFu) | ((v >> 12) & 0x8u) | ((v >> 24) & 0x80u)) << (8 * j);
      }
      packed[h] = word;
    }
    *reinterpret_cast<uint2 *>(q + row * (K >> 1) + (col >> 1)) = make_uint2(packed[0], packed[1]);
    if (sf_row) sf_row[row * G + grp] = static_cast<uint8_t>(sbyte);
  }
  // groups 4j..4j+3 are lanes 4j..4j+3: one word per four lanes
  const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 1);
  const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 2);
  const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 3);
  if ((lane & 3) == 0 && grp < katoms * 4) {
    const uint32_t word = sbyte | (b1 << 8) | (b2 << 16) | (b3 << 24);
    *reinterpret_cast<uint32_t *>(sf_mma + sf_mma_offset(row, grp, katoms)) = word;
  }
}

// Transposed quantization (the operands of the weight gradient, and the
// weight operand of the input gradient): x bf16 [R, ldx] with C columns used,
// quantized along R -- per 32 consecutive rows of one column -- and written
// transposed: codes [C, R] (row pitch R) and scales in the MMA layout of a
// [C, R] operand.  FMT kQE4M3 (the act_quant rule) or kQE5M2 (the gradient
// rule; SR: the draw of element (r, c) is index r * C + c under `seed`).
//
// A warp owns 32 rows x 64 columns: lane l loads row r0 + l (64 values, 8 x
// 16 B).  The column maxima over the 32 rows come from a reduce-scatter of
// the packed 16-bit magnitudes (two columns per word, recursive halving: 31
// shuffles) that leaves lane l with columns 2l and 2l + 1; that lane forms
// their scale exponents and stores their scale bytes, and 32 shuffles hand
// every lane all 64 exponents.  Each lane encodes its 64 values, the codes
// turn around through 2 KB of shared memory per warp and leave as 32-byte
// pieces of the output rows.
// grid.x = row group (32 rows), grid.y * 8 + warp = column tile (64 columns).
// Tiles past C or past R/32 write padding scales (127) only.
template <int FMT, bool SR>
__global__ void __launch_bounds__(256) quant_t_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t R, int64_t C, int64_t ldx, int64_t col_tiles,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf_mma, int *__restrict__ status,
    uint64_t seed) {
  static_assert(FMT == kQE4M3 || FMT == kQE5M2, "E4M3 or E5M2 codes");
  static_assert(!SR || FMT == kQE5M2, "stochastic rounding is for E5M2 gradients");
  __shared__ __align__(16) uint8_t stage[8][64 * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ct = static_cast<int64_t>(blockIdx.y) * 8 + warp;
  if (ct >= col_tiles) return;  // whole warps leave; only warp-level sync below
  const int64_t c0 = ct * 64;
  const int64_t g = blockIdx.x;
  const int64_t r0 = g * 32;
  const int64_t G = R >> 5;
  const int64_t katoms = (G + 3) >> 2;
  const bool rows_ok = g < G;
  griddep_wait();
  griddep_launch_dependents();

  uint32_t w[32];  // columns 2i (low half) and 2i + 1 (high half) of row r0 + lane
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    uint4 t = make_uint4(0u, 0u, 0u, 0u);
    const int64_t c = c0 + v * 8;
    if (rows_ok && c < C)
      t = __ldg(reinterpret_cast<const uint4 *>(x + (r0 + lane) * ldx + c));
    w[4 * v] = t.x;
    w[4 * v + 1] = t.y;
    w[4 * v + 2] = t.z;
    w[4 * v + 3] = t.w;
  }
  // reduce-scatter of the column maxima: after the step of distance k the
  // lane keeps k words (the upper half when lane bit k is set)
  uint32_t m[32];
  uint32_t bad = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    m[i] = w[i] & 0x7FFF7FFFu;
    bad |= ((m[i] & 0x7F80u) == 0x7F80u) | ((m[i] & 0x7F800000u) == 0x7F800000u);
  }
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const uint32_t send = up ? m[i] : m[i + k];
      const uint32_t keep = up ? m[i + k] : m[i];
      m[i] = __vmaxu2(keep, __shfl_xor_sync(0xFFFFFFFFu, send, k));
    }
  }
  if (bad && status && rows_ok) atomicOr(status, 1);
  // lane l: columns 2l, 2l + 1 -> scale bytes (padding 127), packed pair
  uint32_t pe;
  {
    const uint32_t a0 = m[0] & 0xFFFFu, a1 = m[0] >> 16;
    const int e0 = FMT == kQE5M2 ? mx_exponent_e5m2(a0) : mx_exponent(a0);
    const int e1 = FMT == kQE5M2 ? mx_exponent_e5m2(a1) : mx_exponent(a1);
    pe = static_cast<uint32_t>(e0 + 127) | (static_cast<uint32_t>(e1 + 127) << 8);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t c = c0 + 2 * lane + h;
      const uint32_t b = (rows_ok && c < C) ? ((pe >> (8 * h)) & 0xFFu) : 127u;
      sf_mma[sf_mma_offset(c, g, katoms)] = static_cast<uint8_t>(b);
    }
  }

  uint8_t *st = stage[warp];
  const int64_t row = r0 + lane;
  Philox4 rnd;  // SR: the draws of the current 8 columns
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t p = __shfl_sync(0xFFFFFFFFu, pe, i);  // scale bytes of columns 2i, 2i + 1
    const float inv0 = __uint_as_float((254u - (p & 0xFFu)) << 23);  // 2^-e
    const float inv1 = __uint_as_float((254u - (p >> 8)) << 23);
    // |x| / 2^e never exceeds the format's largest value for bf16 input; the
    // satfinite conversions would clamp it anyway
    const float f0 = __fmul_rn(__uint_as_float(w[i] << 16), inv0);
    const float f1 = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv1);
    uint32_t b0, b1;
    if constexpr (SR) {
      // draws of columns c0 + 2i, c0 + 2i + 1: one Philox block serves 8
      // columns (row * C + c0 is a multiple of 8: C % 8 == 0, c0 % 64 == 0)
      if (i % 4 == 0)
        rnd = philox4x64_10(static_cast<uint64_t>(row * C + c0 + 2 * i) >> 3, seed);
      b0 = e5m2_sr(fminf(fmaxf(f0, -57344.0f), 57344.0f), philox_draw(rnd, (2 * i) & 7));
      b1 = e5m2_sr(fminf(fmaxf(f1, -57344.0f), 57344.0f), philox_draw(rnd, ((2 * i) & 7) + 1));
    } else if constexpr (FMT == kQE5M2) {
      const uint32_t pk = e5m2x2(f0, f1);
      b0 = pk & 0xFFu;
      b1 = pk >> 8;
    } else {
      const uint32_t pk = e4m3x4(f0, f1, 0.0f, 0.0f);
      b0 = pk & 0xFFu;
      b1 = (pk >> 8) & 0xFFu;
    }
    st[(2 * i) * 32 + lane] = static_cast<uint8_t>(b0);
    st[(2 * i + 1) * 32 + lane] = static_cast<uint8_t>(b1);
  }
  __syncwarp();
  if (rows_ok) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 2 * lane + h;
      if (c0 + j < C) {
        const uint4 *src = reinterpret_cast<const uint4 *>(st + j * 32);
        uint4 *dst = reinterpret_cast<uint4 *>(q + (c0 + j) * R + r0);
        dst[0] = src[0];
        dst[1] = src[1];
      }
    }
  }
}

// Transposed quantization with round to nearest even (E4M3, or E5M2 without
// stochastic rounding): a warp owns 32 rows x 64 columns and lane l the two
// columns c0 + 2l, c0 + 2l + 1 -- one 4-byte load per row, so every warp load
// is one 128-byte row segment.  A lane's two columns are whole groups: their
// maxima, scales and codes need no other lane, and each output row (one
// column, 32 codes) leaves from its lane as two 16-byte stores.
// grid.x = row group (32 rows), grid.y * 8 + warp = column tile (64 columns).
template <int FMT>
__global__ void __launch_bounds__(256) quant_t_rne_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t R, int64_t C, int64_t ldx, int64_t col_tiles,
    uint8_t *__restrict__ q, uint8_t *__restrict__ sf_mma, int *__restrict__ status) {
  static_assert(FMT == kQE4M3 || FMT == kQE5M2, "E4M3 or E5M2 codes");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ct = static_cast<int64_t>(blockIdx.y) * 8 + warp;
  if (ct >= col_tiles) return;
  const int64_t c = ct * 64 + 2 * lane;  // this lane's first column
  const int64_t g = blockIdx.x;
  const int64_t r0 = g * 32;
  const int64_t G = R >> 5;
  const int64_t katoms = (G + 3) >> 2;
  const bool ok = g < G && c < C;  // C % 8 == 0: both columns or neither
  griddep_wait();
  griddep_launch_dependents();

  uint32_t w[32];  // row r0 + r: column c (low half), c + 1 (high half)
#pragma unroll
  for (int r = 0; r < 32; ++r)
    w[r] = ok ? __ldg(reinterpret_cast<const unsigned int *>(x + (r0 + r) * ldx + c)) : 0u;
  uint32_t m = 0;
#pragma unroll
  for (int r = 0; r < 32; ++r) m = __vmaxu2(m, w[r] & 0x7FFF7FFFu);
  const uint32_t a0 = m & 0xFFFFu, a1 = m >> 16;
  if (ok && (a0 >= 0x7F80u || a1 >= 0x7F80u) && status) atomicOr(status, 1);
  const int e0 = FMT == kQE5M2 ? mx_exponent_e5m2(a0) : mx_exponent(a0);
  const int e1 = FMT == kQE5M2 ? mx_exponent_e5m2(a1) : mx_exponent(a1);
  sf_mma[sf_mma_offset(c, g, katoms)] = static_cast<uint8_t>(ok ? e0 + 127 : 127);
  sf_mma[sf_mma_offset(c + 1, g, katoms)] = static_cast<uint8_t>(ok ? e1 + 127 : 127);
  if (!ok) return;
  const float inv0 = __uint_as_float(static_cast<uint32_t>(127 - e0) << 23);  // 2^-e
  const float inv1 = __uint_as_float(static_cast<uint32_t>(127 - e1) << 23);
  uint32_t out0[8], out1[8];  // the codes of columns c and c + 1, rows r0 .. r0 + 31
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t p[4];  // rows 4j .. 4j + 3: byte 0 column c, byte 1 column c + 1
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t v = w[4 * j + t];
      const float f0 = __fmul_rn(__uint_as_float(v << 16), inv0);
      const float f1 = __fmul_rn(__uint_as_float(v & 0xFFFF0000u), inv1);
      p[t] = FMT == kQE5M2 ? e5m2x2(f0, f1) : e4m3x2(f0, f1);
    }
    const uint32_t lo = __byte_perm(p[0], p[1], 0x5140), hi = __byte_perm(p[2], p[3], 0x5140);
    out0[j] = __byte_perm(lo, hi, 0x5410);
    out1[j] = __byte_perm(lo, hi, 0x7632);
  }
  uint4 *d0 = reinterpret_cast<uint4 *>(q + c * R + r0);
  uint4 *d1 = reinterpret_cast<uint4 *>(q + (c + 1) * R + r0);
  d0[0] = make_uint4(out0[0], out0[1], out0[2], out0[3]);
  d0[1] = make_uint4(out0[4], out0[5], out0[6], out0[7]);
  d1[0] = make_uint4(out1[0], out1[1], out1[2], out1[3]);
  d1[1] = make_uint4(out1[4], out1[5], out1[6], out1[7]);
}

// Both quantizations of a gradient in one pass (the output gradient dY feeds
// dX = dY W, contracting over its columns, and dW = dY^T x, contracting over
// its rows): g bf16 [R, ldg] (C columns) -> E5M2 codes q_row [R, C] with
// scales along C (bq_grad_quant) and q_t [C, R] with scales along R
// (bq_quant_transposed), each element's stochastic draw (index r * C + c
// under `seed`) drawn once and used by both.  R % 32 == 0, C % 32 == 0.
// The warp tile, the column reduce-scatter and the transposed store are those
// of quant_t_kernel; a lane's 64 values of one row are two row groups whose
// maxima need no shuffles, and its 64 row codes leave as four 16-byte stores.
template <bool SR>
__global__ void __launch_bounds__(256, 3) grad_quant_dual_kernel(
    const __nv_bfloat16 *__restrict__ x, int64_t R, int64_t C, int64_t ldx, int64_t col_tiles,
    int64_t row_tiles, uint8_t *__restrict__ q_row, uint8_t *__restrict__ sf_row,
    uint8_t *__restrict__ q_t, uint8_t *__restrict__ sf_t, int *__restrict__ status,
    uint64_t seed) {
  __shared__ __align__(16) uint8_t stage[8][64 * 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ct = static_cast<int64_t>(blockIdx.y) * 8 + warp;
  if (ct >= col_tiles) return;  // whole warps leave; only warp-level sync below
  const int64_t c0 = ct * 64;
  const int64_t g = blockIdx.x;  // 32-row group
  const int64_t r0 = g * 32;
  const int64_t G_t = R >> 5, G_r = C >> 5;  // groups per row of q_t, of q_row
  const int64_t katoms_t = (G_t + 3) >> 2, katoms_r = (G_r + 3) >> 2;
  const bool rows_ok = g < G_t;
  griddep_wait();
  griddep_launch_dependents();

  uint32_t w[32];
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    uint4 t = make_uint4(0u, 0u, 0u, 0u);
    const int64_t c = c0 + v * 8;
    if (rows_ok && c < C)
      t = __ldg(reinterpret_cast<const uint4 *>(x + (r0 + lane) * ldx + c));
    w[4 * v] = t.x;
    w[4 * v + 1] = t.y;
    w[4 * v + 2] = t.z;
    w[4 * v + 3] = t.w;
  }
  uint32_t m[32];
  uint32_t rmax[2] = {0u, 0u};  // this row's two 32-column groups
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    m[i] = w[i] & 0x7FFF7FFFu;
    rmax[i / 16] = max(rmax[i / 16], max(m[i] & 0xFFFFu, m[i] >> 16));
  }
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const uint32_t send = up ? m[i] : m[i + k];
      const uint32_t keep = up ? m[i + k] : m[i];
      m[i] = __vmaxu2(keep, __shfl_xor_sync(0xFFFFFFFFu, send, k));
    }
  }
  // lane l: transposed scales of columns 2l, 2l + 1
  uint32_t pe;
  {
    const uint32_t a0 = m[0] & 0xFFFFu, a1 = m[0] >> 16;
    if ((a0 >= 0x7F80u || a1 >= 0x7F80u) && status && rows_ok) atomicOr(status, 1);
    pe = static_cast<uint32_t>(mx_exponent_e5m2(a0) + 127) |
         (static_cast<uint32_t>(mx_exponent_e5m2(a1) + 127) << 8);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t c = c0 + 2 * lane + h;
      const uint32_t b = (rows_ok && c < C) ? ((pe >> (8 * h)) & 0xFFu) : 127u;
      sf_t[sf_mma_offset(c, g, katoms_t)] = static_cast<uint8_t>(b);
    }
  }
  // this row's scales; the row-wise buffer's padding rows and groups are
  // written by the tiles that cover them
  const int64_t row = r0 + lane;
  const int er0 = mx_exponent_e5m2(rmax[0]), er1 = mx_exponent_e5m2(rmax[1]);
  {
    const int64_t rows_pad_r = (R + 127) / 128 * 128;
    const int64_t gc = c0 >> 5;  // first row group of this tile's columns
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const bool valid = rows_ok && c0 + 32 * h < C;
      if (row < rows_pad_r && gc + h < katoms_r * 4)
        sf_row[sf_mma_offset(row, gc + h, katoms_r)] =
            static_cast<uint8_t>(valid ? (h ? er1 : er0) + 127 : 127);
    }
  }
  const float rinv0 = __uint_as_float(static_cast<uint32_t>(127 - er0) << 23);
  const float rinv1 = __uint_as_float(static_cast<uint32_t>(127 - er1) << 23);

  uint8_t *st = stage[warp];
  Philox4 rnd;
  uint32_t rowc[16];  // this row's 64 codes, four per word
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t p = __shfl_sync(0xFFFFFFFFu, pe, i);
    const float inv0 = __uint_as_float((254u - (p & 0xFFu)) << 23);
    const float inv1 = __uint_as_float((254u - (p >> 8)) << 23);
    const float rinv = i < 16 ? rinv0 : rinv1;
    const float x0 = __uint_as_float(w[i] << 16), x1 = __uint_as_float(w[i] & 0xFFFF0000u);
    const float t0 = __fmul_rn(x0, inv0), t1 = __fmul_rn(x1, inv1);  // transposed scaling
    const float r0f = __fmul_rn(x0, rinv), r1f = __fmul_rn(x1, rinv);  // row-wise scaling
    uint32_t bt0, bt1, br0, br1;
    if constexpr (SR) {
      if (i % 4 == 0)
        rnd = philox4x64_10(static_cast<uint64_t>(row * C + c0 + 2 * i) >> 3, seed);
      const uint32_t u0 = philox_draw(rnd, (2 * i) & 7), u1 = philox_draw(rnd, ((2 * i) & 7) + 1);
      bt0 = e5m2_sr(fminf(fmaxf(t0, -57344.0f), 57344.0f), u0);
      bt1 = e5m2_sr(fminf(fmaxf(t1, -57344.0f), 57344.0f), u1);
      br0 = e5m2_sr(fminf(fmaxf(r0f, -57344.0f), 57344.0f), u0);
      br1 = e5m2_sr(fminf(fmaxf(r1f, -57344.0f), 57344.0f), u1);
    } else {
      const uint32_t pt = e5m2x2(t0, t1), pr = e5m2x2(r0f, r1f);
      bt0 = pt & 0xFFu;
      bt1 = pt >> 8;
      br0 = pr & 0xFFu;
      br1 = pr >> 8;
    }
    st[(2 * i) * 32 + lane] = static_cast<uint8_t>(bt0);
    st[(2 * i + 1) * 32 + lane] = static_cast<uint8_t>(bt1);
    const uint32_t pair = br0 | (br1 << 8);
    if (i % 2 == 0)
      rowc[i / 2] = pair;
    else
      rowc[i / 2] |= pair << 16;
  }
  if (rows_ok) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      if (c0 + 16 * v < C)
        *reinterpret_cast<uint4 *>(q_row + row * C + c0 + 16 * v) =
            make_uint4(rowc[4 * v], rowc[4 * v + 1], rowc[4 * v + 2], rowc[4 * v + 3]);
    }
  }
  __syncwarp();
  if (rows_ok) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 2 * lane + h;
      if (c0 + j < C) {
        const uint4 *src = reinterpret_cast<const uint4 *>(st + j * 32);
        uint4 *dst = reinterpret_cast<uint4 *>(q_t + (c0 + j) * R + r0);
        dst[0] = src[0];
        dst[1] = src[1];
      }
    }
  }
  (void)row_tiles;
}

// Row-major scales (ROW32: [N, G]; BLK32x32: [ceil(N/32), G] repeated over
// the 32 rows of each block; ROW16_E4M3: [N, G] E4M3 bytes of 16-input
// groups) -> MMA layout with 127 padding (0x38 for E4M3).  One thread per
// output 32-bit word (4 scale columns of one row).  Flags NaN scale bytes
// (E8M0 255, E4M3 0x7F / 0xFF) in flags bit 0.
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
      // kind 2 (ROW16_E4M3): E4M3 bytes, NaN 0x7F / 0xFF, padding 1.0 (0x38)
      uint32_t b = kind == 2 ? 0x38u : 127u;
      const int64_t c = c0 + j;
      if (r < N && c < G) {
        b = (kind == 1) ? src[(r >> 5) * G + c] : src[r * G + c];
        nan |= kind == 2 ? ((b & 0x7Fu) == 0x7Fu) : (b == 255u);
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
