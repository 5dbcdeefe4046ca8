// gemm_bs.cuh -- block-scaled (MX) GEMM for sm_100a on the 5th-generation
// tensor cores.
//
// Computes, per problem of a batch, y = bf16_RNE(act(alpha * A B^T + bias) + residual)
// where A holds E4M3 activation codes with one E8M0 scale per 32 inputs of a
// row, and B holds E2M1 (MXFP4) or E4M3 weight codes with one E8M0 scale per
// 32 inputs of a row (32x32 FP8 block scales are expanded per row by the
// prepack).  The decoded operands are code * 2^(scale - 127) ("formats.py"
// page, docstring "Formats"; decode_fp4, decode_fp8_block), multiplied exactly
// and accumulated in fp32 by tcgen05.mma kind::mxf8f6f4 with block scaling.
// The same kernel also runs E5M2 gradient operands (kind::mxf8f6f4 format 1),
// packed E2M1 x E2M1 (kind::mxf4, A4 == 1) and NVFP4 with E4M3 scales per 16
// inputs (kind::mxf4nvf4, A4 == 2).  The epilogue can emit MXFP8 codes and
// scales of y instead of bf16 (GemmArgs::q_out), and decode tiles can quantize
// their bf16 activation rows in the producer themselves (FUSEQ).
//
// Structure (one persistent CTA per SM, warp-specialized; 9 warps, 13 for
// unsplit wide tiles):
//   warps 0, 6, 7, 8   TMA copy threads: the weight tile, the activation tile,
//            the weight scales and the activation scales of each stage
//            (operands 128B-swizzled, scales as 512-byte atoms) into a
//            STAGES-deep shared-memory ring; every thread arrives on the
//            stage's mbarrier with its own transaction bytes;
//   warp 1   TMEM allocator and MMA issuer: per stage, tcgen05.cp copies the
//            scale atoms into TMEM, then the stage's MMAs consume it;
//            tcgen05.commit releases the stage and, after the last k-block of
//            a tile, signals the accumulator (ACC buffers) as full;
//   warps 2-5 (and 9-12) epilogue: tcgen05.ld of the fp32 accumulator (one
//            TMEM lane quadrant per warp), alpha / bias / GELU / residual in
//            fp32, one bf16 rounding, a swizzled shared-memory staging tile
//            written out by TMA stores (residual tiles arrive by TMA into the
//            same slots).  Split-K runs either through an fp32 workspace (the
//            last slice to arrive, by atomic ticket, sums all slices in slice
//            order, so the result does not depend on arrival order) or across
//            a thread-block cluster whose CTAs reduce their slices through
//            distributed shared memory in a fixed order.
//
// "P" is the operand on the MMA's 128-row side and "Q" the one on its BN-row
// side.  Normally P = activations and Q = weights (y[p][q]); with SWAP the
// weights go on the 128-row side and a short activation matrix (decode
// shapes) on the BN side, and the epilogue writes the transpose (y[q][p]).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "bq_ptx.cuh"
#include "mx_quant.cuh"

namespace bq {

constexpr int kBlockP = 128;  // MMA M
constexpr int kBlockK = 128;  // inputs per stage: 128 one-byte codes = one 128B-swizzle row
constexpr int kMmaK = 32;     // inputs per tcgen05.mma (one scale per row per MMA)
constexpr int kSfAtom = 512;  // bytes of one 128-row x 4-column scale atom
constexpr int kYChunkBytes = kBlockP * 32 * 2;  // a 128-row x 32-column bf16 staging tile
// Warp roles: 0 weight-operand copies (and barrier set-up), 1 TMEM
// allocation and MMA issue, 2-5 epilogue (one TMEM lane quadrant each),
// 6 activation-operand copies, 7 weight-scale copies, 8 activation-scale
// copies.  A thread issues about one copy per ~700 SM cycles whatever its
// size, while an SM serves several issuing threads at once: four copy
// threads, each arriving on every stage barrier with its own bytes.
constexpr int kNumThreads = 288;
constexpr int kActWarp = 6;
constexpr int kWsfWarp = 7;
constexpr int kAsfWarp = 8;
constexpr int kCopyThreads = 4;
// Unsplit wide tiles (activation rows on the TMEM lanes) add a second group
// of four epilogue warps (9-12, one per TMEM lane quadrant): the two groups
// take alternate 32-column chunks of the accumulator, so an epilogue with a
// heavy activation (erf-GELU) or one accumulator (128 x 256 tiles) takes
// half the time next to the mainloop.
constexpr int kWideThreads = kNumThreads + 128;
constexpr int kEpi2FirstThread = (kAsfWarp + 1) * 32;  // first thread of the second group

// tcgen05 operand formats (instruction descriptor fields a_format / b_format):
// kind::mxf8f6f4 codes E4M3 0, E5M2 1 and E2M1 5 (one byte slot per FP4 code in
// shared memory); kind::mxf4 code E2M1 1 (two codes per byte).
constexpr uint32_t kFmtE4M3 = 0;
constexpr uint32_t kFmtE5M2 = 1;
constexpr uint32_t kFmtE2M1 = 5;
constexpr uint32_t kFmtMxf4E2M1 = 1;

struct GemmArgs {
  int M, N, K;     // one problem: y[M, N] = A[M, K] B[N, K]^T
  uint32_t fmt_p, fmt_q;  // kind::mxf8f6f4 operand formats of the P and Q sides
  int batch;       // number of problems
  int kt_total;    // ceil(K / 128)
  int splits;      // K slices per output tile (1 = no split)
  int kt_per_split;
  int tiles_p, tiles_q;
  int raster_group;
  int sf_katoms;   // scale atoms along K = ceil(K / 128)
  int sf_q_rowatoms;  // 128-row scale bands of the Q-side operand = ceil(rows_q / 128)
  int split_lg;       // log2(splits) for cluster split-K
  // Rows of the Q-side copy box (<= BN): when one Q tile covers all of a
  // short operand, the box stops at the operand's last row rounded up to 8;
  // the tile rows past it are never loaded and only feed output columns that
  // are not stored.  A KC-chunk box lands as KC consecutive blocks of
  // q_box_rows x 128 bytes.
  int q_box_rows;
  // scale buffers (MMA layout) of the P- and Q-side operands, batch strides in bytes
  const uint8_t *sf_p;
  const uint8_t *sf_q;
  int64_t sf_p_bstride, sf_q_bstride;
  int p_batched, q_batched;  // operand tensor maps carry a batch dimension
  // output and epilogue
  __nv_bfloat16 *y;
  int64_t ldy, y_bstride;  // elements
  const __nv_bfloat16 *bias;
  const __nv_bfloat16 *res;
  int64_t ldres, res_bstride;  // elements
  float alpha;
  int act;
  // optional quantized output (codes [M][ldy] u8, batch stride y_bstride
  // bytes; scales in the MMA layout, batch stride sf_out_bstride bytes)
  uint8_t *q_out;
  uint8_t *sf_out;
  int64_t sf_out_bstride;
  // fused activation quantization (swap-AB decode tiles): bf16 activations x
  // [M, ldx]; optionally their codes [M, K] and MMA-layout scales are also
  // stored (by the CTAs of the first weight tile), non-finite input reported
  const __nv_bfloat16 *x;
  int64_t ldx;
  uint8_t *a_q_out;
  uint8_t *a_sf_out;
  int *status;
  // split-K workspace: fp32 partials [units][128][BN] and per-tile tickets
  float *ws_partial;
  int *ws_ticket;
  int *err;
};

// How the K slices of an output tile are combined (a compile-time property of
// each kernel instance, so an instance carries only the code it runs).
enum SplitMode : int { kSplitNone = 0, kSplitWorkspace = 1, kSplitCluster = 2 };

// Shared-memory layout of one kernel instance.  A stage holds KC chunks of
// 128 bytes of K per row (each chunk a 128B-swizzled K-major tile per
// operand: 128 K of one-byte codes, or 256 K of packed E2M1 codes) and the
// chunks' scale-factor atoms (APC atoms of 128 K per chunk and 128-row band);
// more bytes behind one stage barrier means fewer barrier round trips per
// byte, which is what bounds a CTA's copy rate.
template <int BN, int STAGES, int ACC, bool CSPLIT = false, int KC = 1, bool OUT_STAGE = false,
          bool LANDING = false, bool YSTAGE = false, int APC = 1>
struct GemmSmem {
  static constexpr int kSfqAtoms = BN > 128 ? BN / 128 : 1;  // 128-row bands, Q side
  static constexpr int kSfqCols = 4 * kSfqAtoms;
  static constexpr int kSfColsChunk = APC * (4 + kSfqCols);  // TMEM scale columns per chunk
  static constexpr int kSfCols = KC * kSfColsChunk;          // TMEM scale columns per stage
  static constexpr int kChunkP = kBlockP * kBlockK;  // bytes of one 128-K chunk, P side
  static constexpr int kChunkQ = BN * kBlockK;       // Q side
  static constexpr int kBytesP = KC * kChunkP;
  static constexpr int kBytesQ = KC * kChunkQ;
  static constexpr int kSfpBytes = KC * APC * kSfAtom;              // per stage
  static constexpr int kSfqBytes = KC * APC * kSfqAtoms * kSfAtom;  // per stage
  static constexpr int kOffQ = STAGES * kBytesP;
  // wide tiles: two 128x32 bf16 staging tiles for the TMA-store epilogue
  // (1024-byte aligned: the 64-byte swizzle follows address bits)
  static constexpr int kOffYStage = kOffQ + STAGES * kBytesQ;
  static constexpr int kBytesYStage = YSTAGE ? 2 * kYChunkBytes : 0;
  static constexpr int kOffSfp = kOffYStage + kBytesYStage;
  static constexpr int kOffSfq = kOffSfp + STAGES * kSfpBytes;
  // cluster split-K: receive buffer [S slices][128/S rows][BN + 4] fp32 (the
  // +4 pad keeps float4 row accesses free of bank conflicts)
  static constexpr int kRecvStride = BN + 4;
  static constexpr int kOffPart = kOffSfq + STAGES * kSfqBytes;
  static constexpr int kBytesPart = CSPLIT ? kBlockP * kRecvStride * 4 : 0;
  // swap-AB output staging: the bf16 tile [BN rows m][128 columns n]
  static constexpr int kOffOut = kOffPart + kBytesPart;
  static constexpr int kBytesOut = OUT_STAGE ? BN * kBlockP * 2 : 0;
  // swap-AB workspace split: this slice's fp32 partial tile [BN m][128 n],
  // then the landing area for the other slices' partial tiles ([slice][m][128
  // n], as many slices per pass as fit)
  static constexpr int kOffAcc = kOffOut + kBytesOut;
  static constexpr int kBytesAcc = LANDING ? BN * kBlockP * 4 : 0;
  static constexpr int kOffLand = kOffAcc + kBytesAcc;
  static constexpr int kBytesLand = LANDING ? 64 * 1024 : 0;
  static constexpr int kOffBiasS = kOffLand + kBytesLand;  // the tile's 128 biases (fp32)
  static constexpr int kBytesBiasS = LANDING ? kBlockP * 4 : 0;
  static constexpr int kOffBar = kOffBiasS + kBytesBiasS;
  static constexpr int kNumBars =
      2 * STAGES + 2 * ACC + 1 + (CSPLIT ? 2 : 0) + (LANDING ? 1 : 0) + (YSTAGE ? 2 : 0);
  static constexpr int kRbarIndex = kNumBars - 2;  // residual staging barriers (YSTAGE)
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static constexpr int kStages = STAGES;
  static constexpr int kTmemUsed = ACC * BN + STAGES * kSfCols;
  static constexpr int kTmemCols = kTmemUsed <= 32    ? 32
                                   : kTmemUsed <= 64  ? 64
                                   : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256
                                                      : 512;
  static_assert(kTmemUsed <= 512, "TMEM budget");
  static_assert(kBytes <= 232448, "shared memory budget");
};

// The layout a kernel instance uses: unsplit swap-AB tiles stage their bf16
// output in shared memory for row-contiguous stores; swap-AB workspace splits
// gather the slices' partial tiles in shared memory.
template <int BN, int STAGES, int ACC, bool SWAP, int MODE, int KC, int APC = 1>
using KernelSmem = GemmSmem<BN, STAGES, ACC, MODE == kSplitCluster, KC,
                            SWAP && MODE == kSplitNone, SWAP && MODE == kSplitWorkspace,
                            !SWAP && MODE == kSplitNone, APC>;

__device__ __forceinline__ uint32_t make_idesc(uint32_t fmt_p, uint32_t fmt_q, int bn, int sf_id) {
  uint32_t d = 0;
  d |= static_cast<uint32_t>(sf_id & 3) << 4;    // scale-factor id of B (Q side)
  d |= fmt_p << 7;                               // A format
  d |= fmt_q << 10;                              // B format
  d |= static_cast<uint32_t>(bn >> 3) << 17;     // N / 8
  d |= 1u << 23;                                 // scale format: UE8M0
  d |= static_cast<uint32_t>(kBlockP >> 4) << 24;  // M / 16
  d |= static_cast<uint32_t>(sf_id & 3) << 29;   // scale-factor id of A (P side)
  return d;
}

// Work unit -> (batch, P tile, Q tile, K slice) with grouped rasterization
// over P tiles, and the unit's K-block range (slices dealt out evenly, never
// empty while splits <= K blocks).  32-bit arithmetic throughout.
struct UnitPos {
  int b, tp, tq, split, tile, kt0, kt1;
};

__device__ __forceinline__ UnitPos unit_pos(const GemmArgs &a, int unit) {
  UnitPos u;
  u.split = unit % a.splits;
  u.tile = unit / a.splits;
  const int per_batch = a.tiles_p * a.tiles_q;
  u.b = u.tile / per_batch;
  const int idx = u.tile - u.b * per_batch;
  const int group = a.raster_group * a.tiles_q;
  const int g = idx / group;
  const int first_p = g * a.raster_group;
  const int gp = min(a.raster_group, a.tiles_p - first_p);
  const int r = idx - g * group;
  u.tp = first_p + r % gp;
  u.tq = r / gp;
  u.kt0 = (u.split * a.kt_total) / a.splits;
  u.kt1 = ((u.split + 1) * a.kt_total) / a.splits;
  return u;
}

// erf-form GELU, 0.5 t (1 + erf(t / sqrt 2)), inline: an out-of-line call
// per element costs the unrolled epilogue its registers at every call.
// erf is the rational-exponential approximation of Abramowitz and Stegun,
// Handbook of Mathematical Functions, formula 7.1.26 (after Hastings):
//   erf(x) = 1 - (a1 u + a2 u^2 + a3 u^3 + a4 u^4 + a5 u^5) exp(-x^2),
//   u = 1 / (1 + p x), x >= 0, odd in x, absolute error <= 1.5e-7,
// evaluated with the fast division and exponential (relative errors near
// 2^-22): one branch-free formula, so the epilogue's values interleave.  The
// GELU's error is then below 1e-7 |t|, far inside the GEMM's tolerance
// (2^-20 |alpha| sum |a b| + |bias| >= 1e-6 |t|) and half a bf16 ulp of large
// outputs.  Callers branch on the activation once per group of values, so
// code without GELU never runs through it.
__device__ __forceinline__ float gelu_erf(float t) {
  const float x = fabsf(t) * 0.70710678118654752f;
  const float u = __fdividef(1.0f, fmaf(0.3275911f, x, 1.0f));
  float poly = fmaf(u, 1.061405429f, -1.453152027f);
  poly = fmaf(u, poly, 1.421413741f);
  poly = fmaf(u, poly, -0.284496736f);
  poly = fmaf(u, poly, 0.254829592f);
  poly *= u;
  const float erfc_x = poly * __expf(-x * x);  // 1 - erf(x)
  // 1 + erf(t / sqrt 2): 2 - erfc for t >= 0, erfc for t < 0 (odd erf)
  const float one_plus = t >= 0.0f ? 2.0f - erfc_x : erfc_x;
  return 0.5f * t * one_plus;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
  return __uint_as_float(h << 16);
}

// Epilogue math for one output element (fp32, single final rounding by caller).
__device__ __forceinline__ float epi_value(const GemmArgs &a, float acc, float bias, float res) {
  float t = a.alpha * acc + bias;
  if (a.act == 1) t = gelu_erf(t);
  return t + res;
}

// Writes 32 accumulator values of one TMEM lane: row `prow` of the P side,
// columns q0 .. q0+31 of the Q side, batch b.  Swap-AB: `bias_swap` is the
// bias of output column prow, fetched by the caller.
template <bool SWAP>
__device__ __forceinline__ void emit32(const GemmArgs &a, int b, int prow, int q0,
                                       const float (&f)[32], float bias_swap) {
  if constexpr (!SWAP) {
    const int m = prow;
    if (m >= a.M) return;
    __nv_bfloat16 *yrow = a.y + b * a.y_bstride + static_cast<int64_t>(m) * a.ldy;
    const __nv_bfloat16 *rrow =
        a.res ? a.res + b * a.res_bstride + static_cast<int64_t>(m) * a.ldres : nullptr;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int n = q0 + 8 * g;
      if (n >= a.N) break;
      float bias8[8], res8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) bias8[j] = res8[j] = 0.0f;
      if (a.bias) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.bias + n));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bias8[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFF);
          bias8[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
        }
      }
      if (rrow) {
        const uint4 v = *reinterpret_cast<const uint4 *>(rrow + n);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          res8[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFF);
          res8[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
        }
      }
      float t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = a.alpha * f[8 * g + j] + bias8[j];
      if (a.act == 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = gelu_erf(t[j]);
      }
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(t[2 * j] + res8[2 * j],
                                                        t[2 * j + 1] + res8[2 * j + 1]);
        o[j] = *reinterpret_cast<const uint32_t *>(&p2);
      }
      *reinterpret_cast<uint4 *>(yrow + n) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    // Thread = output column n, its 32 values = rows m = q0 .. q0+31: one
    // bf16 per row; across the warp each row's store is 64 contiguous bytes.
    const int n = prow;
    if (n >= a.N || q0 >= a.M) return;
    const float bias = bias_swap;
    const int cnt = min(32, a.M - q0);
    __nv_bfloat16 *yp = a.y + b * a.y_bstride + static_cast<int64_t>(q0) * a.ldy + n;
    const int ldy = static_cast<int>(a.ldy);
    if (a.res == nullptr && a.act == 0) {
      const float alpha = a.alpha;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < cnt) yp[j * ldy] = __float2bfloat16_rn(alpha * f[j] + bias);
    } else {
      const __nv_bfloat16 *rp =
          a.res ? a.res + b * a.res_bstride + static_cast<int64_t>(q0) * a.ldres + n : nullptr;
      const int ldr = static_cast<int>(a.ldres);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < cnt) {
          const float res = rp ? __bfloat162float(rp[j * ldr]) : 0.0f;
          yp[j * ldy] = __float2bfloat16_rn(epi_value(a, f[j], bias, res));
        }
    }
  }
}

__device__ __forceinline__ void epi_bar_sync(int group = 0) {
  __syncwarp();
  // the 4 warps of epilogue group `group` (named barriers 1 and 2)
  asm volatile("barrier.sync %0, 128;" ::"r"(1 + group) : "memory");
}

// Quantized output of one 32-group: row m, columns q0 .. q0+31, the bf16
// outputs packed in o (column 2i in the low half of word i) -- the same codes
// and scale byte bq_act_quant gives for them.  Rows in [M, rows padded to
// 128) get the padding scale 127, and the row's last group also writes the
// padding columns of its scale atom.
__device__ __forceinline__ void quant_out_row32(const GemmArgs &a, int b, int m, int q0,
                                                const uint32_t (&o)[16]) {
  const int64_t groups = a.N >> 5;
  const int64_t katoms = (groups + 3) >> 2;
  const int64_t rows_pad = (static_cast<int64_t>(a.M) + 127) / 128 * 128;
  if (m >= rows_pad) return;
  uint8_t *sfo = a.sf_out + b * a.sf_out_bstride;
  const int g = q0 >> 5;
  if (m < a.M) {
    uint32_t bad = 0;
    const int e = mx_exponent(bf16_amax_bits(o, bad));
    uint32_t codes[8];
    mx_encode(o, e, codes);
    uint4 *qd = reinterpret_cast<uint4 *>(a.q_out + b * a.y_bstride +
                                          static_cast<int64_t>(m) * a.ldy + q0);
    qd[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    qd[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
    sfo[sf_mma_offset(m, g, katoms)] = static_cast<uint8_t>(e + 127);
    if (bad) atomicOr(a.err, BQ_DEV_ERR_NONFINITE);  // NaN or Inf among the outputs
  } else {
    sfo[sf_mma_offset(m, g, katoms)] = 127;
  }
  if (g == groups - 1)
    for (int64_t cc = groups; cc < katoms * 4; ++cc) sfo[sf_mma_offset(m, cc, katoms)] = 127;
}

// Swap-AB tile output through the staged bf16 tile, with the quantized
// output: rows m of the tile go out as 16-byte vectors of y (when y is
// written) and as 8-byte vectors of codes; the 4 lanes covering one 32-group
// of a row meet through two shuffles for its amax.  The loop is warp-uniform
// (every lane takes part in the shuffles).  The tile of the last activation
// rows writes the padding rows' scale bytes, the tile of the last column
// group the padding columns.
template <int BN>
__device__ __forceinline__ void copy_out_swap_q(const GemmArgs &a, const UnitPos &u, int epi_tid,
                                                const __nv_bfloat16 *stage) {
  const int n0 = u.tp * kBlockP;
  const int m0 = u.tq * BN;
  const int rows = min(BN, a.M - m0);
  const int nvec = min(kBlockP / 8, (a.N - n0) / 8);  // a multiple of 4 (N % 32 == 0)
  const int64_t groups = a.N >> 5;
  const int64_t katoms = (groups + 3) >> 2;
  uint8_t *sfo = a.sf_out + u.b * a.sf_out_bstride;
  const int lane = epi_tid & 31;
  for (int base = epi_tid & ~31; base < rows * 16; base += 128) {
    const int i = base + lane;
    const int r = i >> 4, v = i & 15;
    const bool ok = i < rows * 16 && v < nvec;
    const uint4 val =
        ok ? *reinterpret_cast<const uint4 *>(stage + r * kBlockP + v * 8) : make_uint4(0, 0, 0, 0);
    const int m = m0 + r;
    const int n = n0 + v * 8;
    if (ok && a.y)
      *reinterpret_cast<uint4 *>(a.y + u.b * a.y_bstride + static_cast<int64_t>(m) * a.ldy + n) =
          val;
    const uint32_t w[4] = {val.x, val.y, val.z, val.w};
    uint32_t bad = 0;
    uint32_t mx = bf16_amax_bits(w, bad);
    mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
    mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
    if (ok) {
      const int e = mx_exponent(mx);
      uint32_t codes[2];
      mx_encode(w, e, codes);
      *reinterpret_cast<uint2 *>(a.q_out + u.b * a.y_bstride + static_cast<int64_t>(m) * a.ldy +
                                 n) = make_uint2(codes[0], codes[1]);
      if ((v & 3) == 0) sfo[sf_mma_offset(m, n >> 5, katoms)] = static_cast<uint8_t>(e + 127);
      if (bad) atomicOr(a.err, BQ_DEV_ERR_NONFINITE);  // NaN or Inf among the outputs
    }
  }
  // padding scale bytes
  const int64_t g0 = n0 >> 5;
  const int64_t g1 = g0 + nvec / 4;  // this tile's groups [g0, g1)
  const int64_t gend = g1 == groups ? katoms * 4 : g1;
  if (u.tq == a.tiles_q - 1) {  // rows [M, 128-row padding) of this tile's columns
    const int64_t rows_pad = (static_cast<int64_t>(a.M) + 127) / 128 * 128;
    const int64_t nc = gend - g0;
    for (int64_t idx = epi_tid; idx < (rows_pad - a.M) * nc; idx += 128)
      sfo[sf_mma_offset(a.M + idx / nc, g0 + idx % nc, katoms)] = 127;
  }
  if (gend > g1) {  // padding columns of this tile's real rows
    const int64_t nc = gend - g1;
    for (int64_t idx = epi_tid; idx < rows * nc; idx += 128)
      sfo[sf_mma_offset(m0 + idx / nc, g1 + idx % nc, katoms)] = 127;
  }
}

// Wide-tile epilogue (activation rows on the TMEM lanes): rows m0 .. m0+127
// (this thread owns m0 + row) and columns n0 .. n0+NCOLS-1, in chunks of 32
// columns: TMEM -> registers -> alpha, bias, GELU, residual in fp32 -> one
// bf16 rounding -> a 128x32 bf16 staging tile in shared memory (the 64-byte
// swizzle, so each warp store is conflict-free) -> one TMA store per chunk,
// double-buffered.  Stores clip rows past M and columns past N.  With a
// residual, its chunk arrives by a TMA load into the same staging slot (two
// chunks ahead, on the slot's barrier in `rbar`); each thread reads its row
// there and writes its outputs over it.  `rphase` carries the two slots'
// barrier parities (bits 0 and 1) from call to call.
template <int NCOLS>
__device__ __forceinline__ void epilogue_rows_tma(const GemmArgs &a, const CUtensorMap *tm_y,
                                                  const CUtensorMap *tm_res, uint64_t *rbar,
                                                  uint32_t &rphase, uint32_t t_row, int b, int m0,
                                                  int n0, int row, int epi_tid, uint8_t *ystage,
                                                  volatile int *abort_flag) {
  const int m = m0 + row;
  const bool res = a.res != nullptr;
  const int nch = min(NCOLS / 32, (a.N - n0 + 31) / 32);
  auto load_res = [&](int c) {  // one thread: residual chunk c into slot c & 1
    const int slot = c & 1;
    mbar_arrive_expect_tx(&rbar[slot], static_cast<uint32_t>(kYChunkBytes));
    if (a.batch > 1 && a.res_bstride != 0)  // else one residual serves every problem
      tma_load_3d(ystage + slot * kYChunkBytes, tm_res, &rbar[slot], n0 + c * 32, m0, b);
    else
      tma_load_2d(ystage + slot * kYChunkBytes, tm_res, &rbar[slot], n0 + c * 32, m0);
  };
  if (res && epi_tid == 0) {
    bulk_wait_group_read<0>();  // earlier stores have read both slots
    load_res(0);
    if (nch > 1) load_res(1);
  }
#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
    const int q0 = n0 + c * 32;
    uint32_t v[32];
    __syncwarp();
    tmem_ld_32x32b_x32(t_row + c * 32, v);
    tmem_ld_wait();
    uint8_t *buf = ystage + (c & 1) * kYChunkBytes;
    uint4 rv[4];
    if (res) {
      const uint32_t bit = 1u << (c & 1);
      if (!mbar_wait(&rbar[c & 1], (rphase & bit) ? 1u : 0u, a.err, abort_flag, kWaitEpiFull))
        return;
      rphase ^= bit;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        rv[j] = *reinterpret_cast<const uint4 *>(buf + row * 64 + ((j ^ ((row >> 1) & 3)) << 4));
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) rv[j] = make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t o[16];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float bias8[8];
      if (a.bias && q0 + 8 * g < a.N) {
        const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(a.bias + q0 + 8 * g));
        const uint32_t w[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bias8[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFF);
          bias8[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) bias8[j] = 0.0f;
      }
      float t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = a.alpha * __uint_as_float(v[8 * g + j]) + bias8[j];
      if (a.act == 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = gelu_erf(t[j]);
      }
      const uint32_t rw[4] = {rv[g].x, rv[g].y, rv[g].z, rv[g].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 p2 =
            __floats2bfloat162_rn(t[2 * j] + bf16_bits_to_f32(rw[j] & 0xFFFF),
                                  t[2 * j + 1] + bf16_bits_to_f32(rw[j] >> 16));
        o[4 * g + j] = *reinterpret_cast<const uint32_t *>(&p2);
      }
    }
    if (a.q_out) quant_out_row32(a, b, m, q0, o);
    if (a.y) {  // uniform
      if (!res) {
        if (epi_tid == 0) bulk_wait_group_read<1>();  // the store two chunks back has read buf
        epi_bar_sync();
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(buf + row * 64 + ((j ^ ((row >> 1) & 3)) << 4)) =
            make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
      fence_proxy_async_smem();
      epi_bar_sync();
      if (epi_tid == 0) {
        if (a.batch > 1)
          tma_store_3d(tm_y, buf, q0, m0, b);
        else
          tma_store_2d(tm_y, buf, q0, m0);
        bulk_commit_group();
      }
    } else if (res) {
      epi_bar_sync();  // every thread has read its residual from the slot
    }
    if (res && epi_tid == 0 && c + 2 < nch) {
      bulk_wait_group_read<0>();  // this chunk's store has read the slot
      load_res(c + 2);
    }
  }
}

// The same with two epilogue groups (unsplit wide tiles of gemm_bs_kernel):
// group g takes chunks g, g + 2, ... of the accumulator row and staging slot
// g; its first thread waits for the group's previous TMA store to have read
// the slot before the slot is refilled (with the next chunk's residual, by a
// TMA load on rbar[g], or with outputs).  `rphase` bit g carries the slot
// barrier's parity.
template <int NCOLS>
__device__ __forceinline__ void epilogue_rows_tma_g2(const GemmArgs &a, const CUtensorMap *tm_y,
                                                     const CUtensorMap *tm_res, uint64_t *rbar,
                                                     uint32_t &rphase, uint32_t t_row, int b,
                                                     int m0, int n0, int row, int epi_tid,
                                                     int group, uint8_t *ystage,
                                                     volatile int *abort_flag) {
  const int m = m0 + row;
  const bool res = a.res != nullptr;
  const int nch = min(NCOLS / 32, (a.N - n0 + 31) / 32);
  uint8_t *buf = ystage + group * kYChunkBytes;
  const bool batched_res = a.batch > 1 && a.res_bstride != 0;
#pragma unroll 1
  for (int c = group; c < nch; c += 2) {
    const int q0 = n0 + c * 32;
    if (epi_tid == 0) {
      bulk_wait_group_read<0>();  // the group's previous store has read the slot
      if (res) {
        mbar_arrive_expect_tx(&rbar[group], static_cast<uint32_t>(kYChunkBytes));
        if (batched_res)
          tma_load_3d(buf, tm_res, &rbar[group], q0, m0, b);
        else
          tma_load_2d(buf, tm_res, &rbar[group], q0, m0);
      }
    }
    uint32_t v[32];
    __syncwarp();
    tmem_ld_32x32b_x32(t_row + c * 32, v);
    tmem_ld_wait();
    uint4 rv[4];
    if (res) {
      if (!mbar_wait(&rbar[group], (rphase >> group) & 1u, a.err, abort_flag, kWaitEpiFull))
        return;
      rphase ^= 1u << group;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        rv[j] = *reinterpret_cast<const uint4 *>(buf + row * 64 + ((j ^ ((row >> 1) & 3)) << 4));
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) rv[j] = make_uint4(0u, 0u, 0u, 0u);
      if (a.y) epi_bar_sync(group);  // the slot is free
    }
    uint32_t o[16];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float bias8[8];
      if (a.bias && q0 + 8 * g < a.N) {
        const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(a.bias + q0 + 8 * g));
        const uint32_t w[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bias8[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFF);
          bias8[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) bias8[j] = 0.0f;
      }
      float t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = a.alpha * __uint_as_float(v[8 * g + j]) + bias8[j];
      if (a.act == 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = gelu_erf(t[j]);
      }
      const uint32_t rw[4] = {rv[g].x, rv[g].y, rv[g].z, rv[g].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 p2 =
            __floats2bfloat162_rn(t[2 * j] + bf16_bits_to_f32(rw[j] & 0xFFFF),
                                  t[2 * j + 1] + bf16_bits_to_f32(rw[j] >> 16));
        o[4 * g + j] = *reinterpret_cast<const uint32_t *>(&p2);
      }
    }
    if (a.q_out) quant_out_row32(a, b, m, q0, o);
    if (a.y) {  // uniform
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(buf + row * 64 + ((j ^ ((row >> 1) & 3)) << 4)) =
            make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
      fence_proxy_async_smem();
      epi_bar_sync(group);
      if (epi_tid == 0) {
        if (a.batch > 1)
          tma_store_3d(tm_y, buf, q0, m0, b);
        else
          tma_store_2d(tm_y, buf, q0, m0);
        bulk_commit_group();
      }
    } else if (res) {
      epi_bar_sync(group);  // every row has read its residual before the next load
    }
  }
}

// The two-group epilogue without a residual, accumulator released first: each
// thread reads its row's chunks of the group (NCOLS / 64 of them) from TMEM and
// turns them into final bf16 values in registers, then the group's warps
// release the accumulator (`tempty`) and only afterwards stage and store the
// chunks.  The accumulator is then busy only for the TMEM reads, so with one
// accumulator per CTA the next tile's MMAs start while this tile's output is
// still being written.  (With a residual the final value needs the residual
// tile, which is brought in chunk by chunk through the staging slot:
// epilogue_rows_tma_g2 keeps the accumulator until the last chunk.)
template <int NCOLS>
__device__ __forceinline__ void epilogue_rows_drain_g2(const GemmArgs &a, const CUtensorMap *tm_y,
                                                       uint32_t t_row, int b, int m0, int n0,
                                                       int row, int epi_tid, int group,
                                                       uint8_t *ystage, uint64_t *tempty_bar) {
  constexpr int kPer = NCOLS / 64;  // chunks of 32 columns per group
  const int m = m0 + row;
  const int nch = min(NCOLS / 32, (a.N - n0 + 31) / 32);
  uint8_t *buf = ystage + group * kYChunkBytes;
  uint32_t o[kPer][16];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = group + 2 * i;
    if (c >= nch) break;  // uniform
    const int q0 = n0 + c * 32;
    uint32_t v[32];
    __syncwarp();
    tmem_ld_32x32b_x32(t_row + c * 32, v);
    tmem_ld_wait();
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float bias8[8];
      if (a.bias && q0 + 8 * g < a.N) {
        const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(a.bias + q0 + 8 * g));
        const uint32_t w[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          bias8[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFF);
          bias8[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) bias8[j] = 0.0f;
      }
      float t[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) t[j] = a.alpha * __uint_as_float(v[8 * g + j]) + bias8[j];
      if (a.act == 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = gelu_erf(t[j]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(t[2 * j], t[2 * j + 1]);
        o[i][4 * g + j] = *reinterpret_cast<const uint32_t *>(&p2);
      }
    }
  }
  tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(tempty_bar);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = group + 2 * i;
    if (c >= nch) break;  // uniform
    const int q0 = n0 + c * 32;
    if (a.q_out) quant_out_row32(a, b, m, q0, o[i]);
    if (a.y) {  // uniform
      if (epi_tid == 0) bulk_wait_group_read<0>();  // the group's previous store has read the slot
      epi_bar_sync(group);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4 *>(buf + row * 64 + ((j ^ ((row >> 1) & 3)) << 4)) =
            make_uint4(o[i][4 * j], o[i][4 * j + 1], o[i][4 * j + 2], o[i][4 * j + 3]);
      fence_proxy_async_smem();
      epi_bar_sync(group);
      if (epi_tid == 0) {
        if (a.batch > 1)
          tma_store_3d(tm_y, buf, q0, m0, b);
        else
          tma_store_2d(tm_y, buf, q0, m0);
        bulk_commit_group();
      }
    }
  }
}

// Swap-AB epilogue, first half: the 32 values of output column n = prow
// (rows m = q0 .. q0+31, tile columns c0 .. c0+31) become final bf16 values
// in the staging tile stage[c][n - n0].  Across a warp each row is written as
// 64 contiguous bytes.  The epilogue runs once per tile, so its code is
// fetched cold: the bias-only case gets a short straight-line body.
__device__ __forceinline__ void stage32_swap(const GemmArgs &a, int b, int prow, int nl, int q0,
                                             int c0, const float (&f)[32], float bias,
                                             __nv_bfloat16 *stage) {
  __nv_bfloat16 *dst = stage + c0 * kBlockP + nl;
  if (a.res == nullptr && a.act == 0) {
    const float alpha = a.alpha;
#pragma unroll
    for (int j = 0; j < 32; ++j) dst[j * kBlockP] = __float2bfloat16_rn(alpha * f[j] + bias);
    return;
  }
  const __nv_bfloat16 *rcol =
      a.res ? a.res + b * a.res_bstride + static_cast<int64_t>(q0) * a.ldres + prow : nullptr;
#pragma unroll 1
  for (int j = 0; j < 32; j += 8) {
    float r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      r[i] = (rcol && q0 + j + i < a.M)
                 ? __bfloat162float(rcol[static_cast<int64_t>(j + i) * a.ldres])
                 : 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // f is indexed by a loop counter here; select the 8 values with a
      // switch-free form the compiler keeps in registers.
      float v = 0.0f;
#pragma unroll
      for (int t = 0; t < 32; t += 8)
        if (t == j) v = f[t + i];
      dst[(j + i) * kBlockP] = __float2bfloat16_rn(epi_value(a, v, bias, r[i]));
    }
  }
}

// Final value of output y[m][n] (swap-AB element), general epilogue.
__device__ __forceinline__ float swap_value(const GemmArgs &a, int b, int m, int n, float acc,
                                            float bias) {
  const float r =
      a.res ? __bfloat162float(a.res[b * a.res_bstride + static_cast<int64_t>(m) * a.ldres + n])
            : 0.0f;
  return epi_value(a, acc, bias, r);
}

// Swap-AB epilogue, second half: the staged tile goes out as 16-byte vectors,
// each row m of the tile as 256 contiguous bytes of y (N % 8 == 0 keeps every
// vector wholly inside or outside the output).
template <int BN>
__device__ __forceinline__ void copy_out_swap(const GemmArgs &a, const UnitPos &u, int epi_tid,
                                              const __nv_bfloat16 *stage) {
  const int n0 = u.tp * kBlockP;
  const int m0 = u.tq * BN;
  const int rows = min(BN, a.M - m0);
  const int nvec = min(kBlockP / 8, (a.N - n0) / 8);
  __nv_bfloat16 *ybase = a.y + u.b * a.y_bstride + static_cast<int64_t>(m0) * a.ldy + n0;
#pragma unroll 2
  for (int i = epi_tid; i < rows * (kBlockP / 8); i += 128) {
    const int r = i / (kBlockP / 8);
    const int v = i % (kBlockP / 8);
    if (v < nvec)
      *reinterpret_cast<uint4 *>(ybase + static_cast<int64_t>(r) * a.ldy + v * 8) =
          *reinterpret_cast<const uint4 *>(stage + r * kBlockP + v * 8);
  }
}

// Scale atoms (128 K each) of the stage chunks [kt, kt + nvalid) that exist:
// with packed E2M1 operands a chunk spans APC = 2 atoms and the last chunk of
// K may hold only the first.
template <int APC>
__device__ __forceinline__ int stage_atoms(const GemmArgs &a, int kt, int nvalid) {
  return min(nvalid * APC, a.sf_katoms - kt * APC);
}

// Loads one part of one stage (KC chunks of 128 bytes of K starting at chunk
// kt, of which `nvalid` belong to the unit): the operand tile or the scale
// atoms of the P side or the Q side.  KC == 1 uses 2-D (3-D batched) maps
// with the K offset in bytes; KC > 1 uses maps that view K as (128 bytes,
// chunks), so one copy brings all chunks.  Scale atoms of one 128-row band
// are contiguous along K, so one bulk copy per band brings a stage's atoms.
template <int BN, class L, int KC, int APC = 1>
__device__ __forceinline__ void issue_part(const GemmArgs &a, const CUtensorMap *tm_p,
                                           const CUtensorMap *tm_q, uint8_t *smem,
                                           uint64_t *full, int st, int kt, int nvalid,
                                           const UnitPos &u, bool p_side, bool scales) {
  if (p_side) {
    if (scales) {
      const uint8_t *sfp = a.sf_p + u.b * a.sf_p_bstride +
                           (static_cast<int64_t>(u.tp) * a.sf_katoms + kt * APC) * kSfAtom;
      bulk_load(smem + L::kOffSfp + st * L::kSfpBytes, sfp,
                stage_atoms<APC>(a, kt, nvalid) * kSfAtom, &full[st]);
      return;
    }
    uint8_t *dst = smem + st * L::kBytesP;
    const int row = u.tp * kBlockP;
    if constexpr (KC == 1) {
      if (a.p_batched)
        tma_load_3d(dst, tm_p, &full[st], kt * kBlockK, row, u.b);
      else
        tma_load_2d(dst, tm_p, &full[st], kt * kBlockK, row);
    } else {
      if (a.p_batched)
        tma_load_4d(dst, tm_p, &full[st], 0, row, kt, u.b);
      else
        tma_load_3d(dst, tm_p, &full[st], 0, row, kt);
    }
  } else {
    const int q_row0 = u.tq * BN;
    if (scales) {
#pragma unroll
      for (int j = 0; j < L::kSfqAtoms; ++j) {
        // A band past the operand's last row would be outside the scale
        // buffer; those rows are never stored, so any finite scale band
        // serves -- reuse the last one.
        const int band = min(q_row0 / 128 + j, a.sf_q_rowatoms - 1);
        const uint8_t *sfq = a.sf_q + u.b * a.sf_q_bstride +
                             (static_cast<int64_t>(band) * a.sf_katoms + kt * APC) * kSfAtom;
        bulk_load(smem + L::kOffSfq + st * L::kSfqBytes + j * KC * APC * kSfAtom, sfq,
                  stage_atoms<APC>(a, kt, nvalid) * kSfAtom, &full[st]);
      }
      return;
    }
    uint8_t *dst = smem + L::kOffQ + st * L::kBytesQ;
    if constexpr (KC == 1) {
      if (a.q_batched)
        tma_load_3d(dst, tm_q, &full[st], kt * kBlockK, q_row0, u.b);
      else
        tma_load_2d(dst, tm_q, &full[st], kt * kBlockK, q_row0);
    } else {
      if (a.q_batched)
        tma_load_4d(dst, tm_q, &full[st], 0, q_row0, kt, u.b);
      else
        tma_load_3d(dst, tm_q, &full[st], 0, q_row0, kt);
    }
  }
}

// Cluster split-K, second half: this CTA owns rows [split * R, (split+1) * R)
// (R = 128 / S) of the output tile and has received every slice's fp32
// partial of those rows in its receive buffer.  A thread owns one row (the
// same for every column group it handles), sums the S slices in slice order
// and writes 4 columns (activation rows m) per group; `bias` is that row's
// bias, fetched by the caller.
template <int BN, int LG>
__device__ __forceinline__ void cluster_reduce_local(const GemmArgs &a, const UnitPos &u,
                                                     int epi_tid, const float *recv,
                                                     float bias) {
  constexpr int S = 1 << LG;
  constexpr int R = kBlockP >> LG;
  constexpr int kStride = BN + 4;
  constexpr int kIters = R * (BN / 4) / 128;
  static_assert(kIters >= 1 && R * (BN / 4) % 128 == 0, "slice shape");
  const int rl = epi_tid % R;
  const int n = u.tp * kBlockP + u.split * R + rl;
  if (n >= a.N) return;
#pragma unroll
  for (int i = 0; i < kIters; ++i) {
    const int c4 = (epi_tid + 128 * i) / R;
    if (u.tq * BN + c4 * 4 >= a.M) continue;  // columns past M were not pushed
    float4 acc = *reinterpret_cast<const float4 *>(recv + rl * kStride + c4 * 4);
#pragma unroll
    for (int s = 1; s < S; ++s) {
      const float4 v = *reinterpret_cast<const float4 *>(recv + (s * R + rl) * kStride + c4 * 4);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
    const int m0 = u.tq * BN + c4 * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + j;
      if (m < a.M) {
        const float res =
            a.res ? __bfloat162float(a.res[u.b * a.res_bstride + static_cast<int64_t>(m) * a.ldres + n])
                  : 0.0f;
        a.y[u.b * a.y_bstride + static_cast<int64_t>(m) * a.ldy + n] =
            __float2bfloat16_rn(epi_value(a, vals[j], bias, res));
      }
    }
  }
}

// Fused activation quantizer (swap-AB tiles whose activation tile holds all M
// rows): for each stage of the unit the epilogue warps read the stage's bf16
// inputs, apply the activation quantizer per 32-group (the same arithmetic as
// bq_act_quant) and write the E4M3 codes straight into the stage in the
// layout a TMA copy with the 128-byte swizzle would give (row r at r * 128,
// 16-byte unit j at j ^ (r % 8)) and the scale bytes into the stage's scale
// atom; then each warp arrives on the stage barrier.  Up to kFusedGroups
// groups per thread are loaded before any is quantized (a 41-row, 512-K stage
// in one round trip).  The CTAs of the first weight tile
// also store the codes and scales to global memory when asked.
constexpr int kFusedGroups = 3;

template <class L, int KC>
__device__ __forceinline__ bool fused_quant_unit(const GemmArgs &a, const UnitPos &u,
                                                 uint8_t *smem, uint64_t *full, uint64_t *empty,
                                                 int &stage, uint32_t &phase, int epi_tid,
                                                 int lane, volatile int *abort_flag) {
  const int M = a.M;
  const bool store_out = u.tp == 0 && a.a_q_out != nullptr;
  const int64_t katoms = (static_cast<int64_t>(a.K) / 32 + 3) / 4;
  const int q_chunk = a.q_box_rows * kBlockK;
  for (int kt = u.kt0; kt < u.kt1; kt += KC) {
    if (!mbar_wait(&empty[stage], phase ^ 1, a.err, abort_flag, kWaitProdEmpty)) return false;
    const int nv = min(KC, u.kt1 - kt);
    const int gpr = nv * 4;  // 32-groups per row in this stage
    const int total = M * gpr;
    uint8_t *sq = smem + L::kOffQ + stage * L::kBytesQ;
    uint8_t *ssf = smem + L::kOffSfq + stage * L::kSfqBytes;
#pragma unroll 1
    for (int base = 0; base < total; base += 128 * kFusedGroups) {
      uint32_t w[kFusedGroups][16];
      int row[kFusedGroups], gk[kFusedGroups];
#pragma unroll
      for (int j = 0; j < kFusedGroups; ++j) {
        const int idx = base + epi_tid + 128 * j;
        row[j] = idx / gpr;
        gk[j] = idx - row[j] * gpr;
        if (idx < total) {
          const uint4 *src = reinterpret_cast<const uint4 *>(
              a.x + static_cast<int64_t>(row[j]) * a.ldx + kt * kBlockK + gk[j] * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 t = __ldg(src + v);
            w[j][4 * v] = t.x;
            w[j][4 * v + 1] = t.y;
            w[j][4 * v + 2] = t.z;
            w[j][4 * v + 3] = t.w;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kFusedGroups; ++j) {
        if (base + epi_tid + 128 * j >= total) break;
        uint32_t bad = 0;
        const int e = mx_exponent(bf16_amax_bits(w[j], bad));
        uint32_t codes[8];
        mx_encode(w[j], e, codes);
        const int r = row[j];
        const int c = gk[j] >> 2;  // chunk of the stage
        const int u0 = (gk[j] & 3) * 2;
        uint8_t *rowp = sq + c * q_chunk + r * kBlockK;
        *reinterpret_cast<uint4 *>(rowp + ((u0 ^ (r & 7)) << 4)) =
            make_uint4(codes[0], codes[1], codes[2], codes[3]);
        *reinterpret_cast<uint4 *>(rowp + (((u0 + 1) ^ (r & 7)) << 4)) =
            make_uint4(codes[4], codes[5], codes[6], codes[7]);
        ssf[c * kSfAtom + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (gk[j] & 3)] =
            static_cast<uint8_t>(e + 127);
        if (store_out) {
          const int64_t col = static_cast<int64_t>(kt) * kBlockK + gk[j] * 32;
          uint4 *qd = reinterpret_cast<uint4 *>(a.a_q_out + static_cast<int64_t>(r) * a.K + col);
          qd[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
          qd[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
          a.a_sf_out[sf_mma_offset(r, col >> 5, katoms)] = static_cast<uint8_t>(e + 127);
          if (bad && a.status) atomicOr(a.status, 1);
        }
      }
    }
    fence_proxy_async_smem();  // the MMA reads the stage through the async proxy
    __syncwarp();
    if (lane == 0) mbar_arrive(&full[stage]);
    if (++stage == L::kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
  if (store_out) {  // padding rows of the stored scales (K % 128 == 0: no padding columns)
    const int64_t rows_pad = (static_cast<int64_t>(M) + 127) / 128 * 128;
    const int64_t c0 = static_cast<int64_t>(u.kt0) * 4, c1 = static_cast<int64_t>(u.kt1) * 4;
    for (int64_t idx = epi_tid; idx < (rows_pad - M) * (c1 - c0); idx += 128)
      a.a_sf_out[sf_mma_offset(M + idx / (c1 - c0), c0 + idx % (c1 - c0), katoms)] = 127;
  }
  return true;
}

template <int BN, int STAGES, int ACC, bool SWAP, bool P_FP4, bool Q_FP4, int MODE, int KC,
          bool FUSEQ = false, int A4 = 0>
__global__ void __launch_bounds__((!SWAP && MODE == kSplitNone) ? kWideThreads : kNumThreads,
                                  (MODE == kSplitCluster && KC == 1) ? 2 : 1)
    gemm_bs_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_y,
                   const __grid_constant__ CUtensorMap tm_res, const GemmArgs a) {
  constexpr bool CSPLIT = MODE == kSplitCluster;
  static_assert(!CSPLIT || SWAP, "cluster split-K is built for the swap-AB (decode) tiles");
  static_assert(!CSPLIT || ACC == 1, "cluster split-K uses one accumulator");
  // A4: both operands packed E2M1 (K = 64 per MMA); a 128-byte chunk is 256 K.
  //   A4 == 1: MXFP4, E8M0 scales per 32 (kind::mxf4): two scale atoms a chunk;
  //   A4 == 2: NVFP4, E4M3 scales per 16 (kind::mxf4nvf4): four atoms a chunk.
  static_assert(!A4 || (!P_FP4 && !Q_FP4 && !FUSEQ), "A4 operands are plain packed bytes");
  constexpr int APC = A4 == 2 ? 4 : (A4 ? 2 : 1);
  using L = KernelSmem<BN, STAGES, ACC, SWAP, MODE, KC, APC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *s_p = smem;
  uint8_t *s_q = smem + L::kOffQ;
  uint8_t *s_sfp = smem + L::kOffSfp;
  uint8_t *s_sfq = smem + L::kOffSfq;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + ACC;
  uint64_t *drain = tempty + ACC;
  uint64_t *peer_ready = drain + 1;  // CSPLIT: every slice's rows for this CTA have arrived
  uint64_t *peer_free = drain + 2;   // CSPLIT: every owner has consumed the previous tile
  uint64_t *land_bar = drain + 1;    // workspace split: a pass of partial tiles has landed
  float *recv = reinterpret_cast<float *>(smem + L::kOffPart);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
  int *last_flag = reinterpret_cast<int *>(smem + L::kOffMisc + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int total_units = a.batch * a.tiles_p * a.tiles_q * a.splits;
  // Transaction bytes one producer expects for its half of a stage with `nv`
  // chunks inside the unit.  The operand copies always move whole boxes
  // (chunks past the tensor are zero filled); a 4-bit operand lands in shared
  // memory with one byte-slot per code but counts its packed size (half the
  // footprint).  Scale atoms are copied for the unit's chunks only.
  const int q_box_bytes = KC * a.q_box_rows * kBlockK;
  auto tx_part = [q_box_bytes, &a](int kt, int nv, bool p_side, bool scales) -> uint32_t {
    if (scales)
      return static_cast<uint32_t>(stage_atoms<APC>(a, kt, nv) * (p_side ? 1 : L::kSfqAtoms) *
                                   kSfAtom);
    return p_side ? static_cast<uint32_t>(P_FP4 ? L::kBytesP / 2 : L::kBytesP)
                  : static_cast<uint32_t>(Q_FP4 ? q_box_bytes / 2 : q_box_bytes);
  };

  // Thread 0 (the weight-operand copier) sets up the barriers and at once issues
  // the weight tiles of the first unit's first stages: the weights do not depend on
  // the kernel before this one in the stream, and these copies then overlap
  // the TMEM allocation, the cluster barrier and (under programmatic dependent
  // launch) the tail of that kernel.
  int pre_n = 0;
  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      // one arrival per copy thread; with fused activation quantization the
      // two weight copiers and the four quantizing warps
      mbar_init(&full[st], FUSEQ ? 6 : kCopyThreads);
      mbar_init(&empty[st], 1);
    }
    for (int st = 0; st < ACC; ++st) {
      mbar_init(&tfull[st], 1);
      // one arrival per epilogue warp (two groups on unsplit wide tiles)
      mbar_init(&tempty[st], (!SWAP && MODE == kSplitNone) ? 8 : 4);
    }
    mbar_init(drain, 1);
    if constexpr (CSPLIT) {
      // one arrival: this CTA's own expect_tx for the rows its peers send
      mbar_init(peer_ready, 1);
      mbar_init(peer_free, a.splits);
    }
    if constexpr (L::kBytesLand > 0) mbar_init(land_bar, 1);
    if constexpr (L::kBytesYStage > 0) {
      mbar_init(full + L::kRbarIndex, 1);
      mbar_init(full + L::kRbarIndex + 1, 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_p);
    tma_prefetch_desc(&tm_q);
    if (static_cast<int>(blockIdx.x) < total_units) {
      const UnitPos u = unit_pos(a, blockIdx.x);
      pre_n = min(STAGES, (u.kt1 - u.kt0 + KC - 1) / KC);
      for (int j = 0; j < pre_n; ++j) {
        const int kt = u.kt0 + j * KC;
        const int nv = min(KC, u.kt1 - kt);
        mbar_arrive_expect_tx(&full[j], tx_part(kt, nv, SWAP, false));
        issue_part<BN, L, KC, APC>(a, &tm_p, &tm_q, smem, full, j, kt, nv, u, SWAP, false);
      }
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, L::kTmemCols);
  tc_fence_before();
  __syncthreads();
  // Peers store into this CTA's receive buffer and arrive on its barriers:
  // every CTA of the cluster must have initialised its barriers first.
  if constexpr (CSPLIT) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || (warp >= kActWarp && warp <= kAsfWarp)) {
    // ----------------------------------------------------------- producers --
    // All four walk the same stage ring; each arrives once per stage with the
    // bytes of its own part.  The weight copies never wait for the preceding
    // kernel; the activation copies do, and once every CTA's activation-operand
    // thread is past that wait the next kernel in the stream may launch (it,
    // in turn, waits for this grid before reading its outputs).
    const bool weights = warp == 0 || warp == kWsfWarp;
    if (lane == 0 && (weights || !FUSEQ)) {
      const bool scales = warp == kWsfWarp || warp == kAsfWarp;
      const bool p_side = weights == SWAP;
      if (!weights) {
        griddep_wait();
        if (!scales) griddep_launch_dependents();
      }
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool first = true;
      for (int unit = blockIdx.x; unit < total_units && ok; unit += gridDim.x) {
        const UnitPos u = unit_pos(a, unit);
        int kt = u.kt0;
        if (first && warp == 0) {  // stages whose weight tile went out before the barrier
          kt += pre_n * KC;
          stage = pre_n % STAGES;
          phase = pre_n == STAGES ? 1u : 0u;
        }
        first = false;
        for (; kt < u.kt1; kt += KC) {
          if (!mbar_wait(&empty[stage], phase ^ 1, a.err, abort_flag, kWaitProdEmpty)) {
            ok = false;
            break;
          }
          const int nv = min(KC, u.kt1 - kt);
          mbar_arrive_expect_tx(&full[stage], tx_part(kt, nv, p_side, scales));
          issue_part<BN, L, KC, APC>(a, &tm_p, &tm_q, smem, full, stage, kt, nv, u, p_side,
                                     scales);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // After an abort, give copies already issued time to land before the
      // CTA (and its shared memory) goes away.
      if (!ok) sleep_ns(200000);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < total_units && ok; unit += gridDim.x) {
        const UnitPos u = unit_pos(a, unit);
        const uint32_t sfq_row_off = static_cast<uint32_t>((u.tq * BN) % 128) / 32;
        const uint32_t q_chunk = static_cast<uint32_t>(a.q_box_rows * kBlockK);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, a.err, abort_flag, kWaitMmaTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kt = u.kt0; kt < u.kt1; kt += KC) {
          if (!mbar_wait(&full[stage], phase, a.err, abort_flag, kWaitMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nv = min(KC, u.kt1 - kt);  // chunks of this stage inside the unit
          const uint32_t sf_stage = tmem_base + ACC * BN + stage * L::kSfCols;
          const uint32_t pa0 = smem_u32(s_p + stage * L::kBytesP);
          const uint32_t qa0 = smem_u32(s_q + stage * L::kBytesQ);
          const uint32_t sfp0 = smem_u32(s_sfp + stage * L::kSfpBytes);
          const uint32_t sfq0 = smem_u32(s_sfq + stage * L::kSfqBytes);
#pragma unroll 1
          for (int c = 0; c < nv; ++c) {
            // TMEM scale columns of a chunk: the P side's APC atoms (4 columns
            // each), then per atom the Q side's kSfqAtoms bands.
            const uint32_t sf_t = sf_stage + c * L::kSfColsChunk;
            const uint32_t sfq_t = sf_t + 4 * APC;
            const int na = stage_atoms<APC>(a, kt + c, 1);
            for (int t = 0; t < na; ++t) {
              tc_cp_sf(sf_t + 4 * t, desc_sf_32x128b(sfp0 + (c * APC + t) * kSfAtom));
#pragma unroll
              for (int j = 0; j < L::kSfqAtoms; ++j)
                tc_cp_sf(sfq_t + 4 * (t * L::kSfqAtoms + j),
                         desc_sf_32x128b(sfq0 + (j * KC * APC + c * APC + t) * kSfAtom));
            }
            const uint32_t pa = pa0 + c * L::kChunkP;
            const uint32_t qa = qa0 + c * q_chunk;
#pragma unroll
            for (int ks = 0; ks < kBlockK / kMmaK; ++ks) {
              const uint32_t acc_in = (kt > u.kt0 || c > 0 || ks > 0) ? 1u : 0u;
              if constexpr (A4 == 2) {
                // 64 K per MMA: atom ks, its four scale bytes (16 K each, E4M3)
                if (ks < na) {
                  const uint32_t idesc =
                      make_idesc(kFmtMxf4E2M1, kFmtMxf4E2M1, BN, 0) & ~(1u << 23);  // UE4M3
                  tc_mma_nvf4(d_tmem, desc_kmajor_sw128(pa + ks * kMmaK),
                              desc_kmajor_sw128(qa + ks * kMmaK), idesc, sf_t + 4 * ks,
                              sfq_t + 4 * ks * L::kSfqAtoms + sfq_row_off, acc_in);
                }
              } else if constexpr (A4) {
                // 64 K per MMA: atom ks / 2, scale bytes 2 (ks % 2) and 2 (ks % 2) + 1
                const int t = ks >> 1;
                if (t < na) {
                  const uint32_t idesc =
                      make_idesc(kFmtMxf4E2M1, kFmtMxf4E2M1, BN, (ks & 1) * 2);
                  tc_mma_mxf4(d_tmem, desc_kmajor_sw128(pa + ks * kMmaK),
                              desc_kmajor_sw128(qa + ks * kMmaK), idesc, sf_t + 4 * t,
                              sfq_t + 4 * t * L::kSfqAtoms + sfq_row_off, acc_in);
                }
              } else {
                const uint32_t idesc = make_idesc(a.fmt_p, a.fmt_q, BN, ks);
                tc_mma_mxf8f6f4(d_tmem, desc_kmajor_sw128(pa + ks * kMmaK),
                                desc_kmajor_sw128(qa + ks * kMmaK), idesc, sf_t, sfq_t + sfq_row_off,
                                acc_in);
              }
            }
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        if (++acc == ACC) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // Wait until every MMA this thread issued has completed before the
      // TMEM is released (bounded; after an abort also give them time).
      tc_commit(drain);
      if (!mbar_wait_timed(drain, 0, a.err, kWaitDrain)) sleep_ns(200000);
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int quad = warp % 4;  // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    // epilogue group 0: warps 2-5; group 1 (unsplit wide tiles): warps 9-12
    const int egroup = warp > kAsfWarp ? 1 : 0;
    const int epi_tid = threadIdx.x - (egroup ? kEpi2FirstThread : 64);  // 0..127
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t ready_phase = 0, free_phase = 0, land_phase = 0;
    bool free_pending = false;  // CSPLIT: owners may still be reading the previous tile
    // The bias and residual (and the fused path's activations) may come from
    // the preceding kernel.
    griddep_wait();
    int qstage = 0;
    uint32_t qphase = 0;
    uint32_t rphase = 0;  // residual staging barrier parities
    if constexpr (FUSEQ) {
      if (epi_tid == 0) griddep_launch_dependents();
    }
    for (int unit = blockIdx.x; unit < total_units; unit += gridDim.x) {
      const UnitPos u = unit_pos(a, unit);
      if constexpr (FUSEQ) {
        if (!fused_quant_unit<L, KC>(a, u, smem, full, empty, qstage, qphase, epi_tid, lane,
                                     abort_flag))
          break;
      }
      const int prow = u.tp * kBlockP + row;
      // Swap-AB: the output column (bias index) of this thread's row is known
      // before the accumulator is; fetch its bias while the mainloop runs.
      float bias_n = 0.0f;
      if constexpr (SWAP) {
        const int n = CSPLIT ? u.tp * kBlockP + u.split * (kBlockP >> a.split_lg) +
                                   (epi_tid & ((kBlockP >> a.split_lg) - 1))
                             : prow;
        if (a.bias && n < a.N) bias_n = __bfloat162float(a.bias[n]);
        if constexpr (L::kBytesBiasS > 0)
          reinterpret_cast<float *>(smem + L::kOffBiasS)[row] = bias_n;
      }
      __syncwarp();
      if (!mbar_wait(&tfull[acc], acc_phase, a.err, abort_flag, kWaitEpiFull)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * BN + (static_cast<uint32_t>(quad * 32) << 16);
      if constexpr (MODE == kSplitCluster) {
        // Cluster split-K: the S CTAs of this cluster hold the S K-slices of
        // one output tile.  Every CTA sends each row of its fp32 partial
        // straight from TMEM registers to the CTA that owns that row: rows it
        // owns itself go to its own receive buffer by plain stores, the others
        // by asynchronous DSMEM stores that complete transaction bytes on the
        // owner's peer_ready barrier (armed by the owner with the bytes its
        // S - 1 peers send), so no release fence or remote arrive is needed.
        // Then each CTA finishes its own 128/S rows from local shared memory.
        const int lg = a.split_lg;
        const int S = 1 << lg;
        if (free_pending) {  // the owners' receive buffers are free again
          if (!mbar_wait_cluster(peer_free, free_phase, a.err, abort_flag, kWaitPeerDone)) break;
          free_phase ^= 1;
          free_pending = false;
        }
        const int R = kBlockP >> lg;
        // only the tile's activation columns that exist are sent (a 41-row
        // operand fills 41 of 64), in 16-byte pieces: ceil(mvalid / 4) per row
        const int mvalid = min(BN, a.M - u.tq * BN);
        const int pieces = (mvalid + 3) >> 2;
        if (epi_tid == 0)
          mbar_arrive_expect_tx(peer_ready, static_cast<uint32_t>((S - 1) * R * pieces * 16));
        const uint32_t owner = static_cast<uint32_t>(row >> (7 - lg));
        const bool mine = owner == static_cast<uint32_t>(u.split);  // cluster rank == slice
        const uint32_t slot =
            static_cast<uint32_t>((u.split * R + (row & (R - 1))) * L::kRecvStride * 4);
        const uint32_t dst = mapa_shared(smem_u32(recv), owner) + slot;
        const uint32_t dbar = mapa_shared(smem_u32(peer_ready), owner);
        float *local = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(recv) + slot);
#pragma unroll 1
        for (int c = 0; c < BN / 32 && c * 32 < mvalid; ++c) {  // warp-uniform
          uint32_t v[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (c * 32 + 4 * q < mvalid) {
              if (mine)
                *reinterpret_cast<uint4 *>(local + c * 32 + 4 * q) =
                    make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
              else
                st_async_u4(dst + static_cast<uint32_t>((c * 32 + 4 * q) * 4), v[4 * q],
                            v[4 * q + 1], v[4 * q + 2], v[4 * q + 3], dbar);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        epi_bar_sync();  // this CTA's own rows are in its receive buffer
        if (!mbar_wait_cluster(peer_ready, ready_phase, a.err, abort_flag, kWaitPeerReady)) break;
        ready_phase ^= 1;
        switch (lg) {
          case 1: cluster_reduce_local<BN, 1>(a, u, epi_tid, recv, bias_n); break;
          case 2: cluster_reduce_local<BN, 2>(a, u, epi_tid, recv, bias_n); break;
          default: cluster_reduce_local<BN, 3>(a, u, epi_tid, recv, bias_n); break;
        }
        if (unit + static_cast<int>(gridDim.x) < total_units) {
          // another tile follows: release this CTA's receive buffer to the pushers
          epi_bar_sync();
          if (epi_tid == 0) {
            fence_acq_rel_cluster();
            const uint32_t fb = smem_u32(peer_free);
            for (int r = 0; r < S; ++r)
              mbar_arrive_cluster(mapa_shared(fb, static_cast<uint32_t>(r)));
          }
          free_pending = true;
        }
      } else if constexpr (MODE == kSplitNone && SWAP) {
        // Stage the tile as bf16, release the accumulator, then write the
        // tile row by row.
        __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(smem + L::kOffOut);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int q0 = u.tq * BN + c * 32;
          if (q0 >= a.M) break;  // warp-uniform: the remaining columns are all past M
          uint32_t v[32];
          __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the stores
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
          if (prow < a.N) stage32_swap(a, u.b, prow, row, q0, c * 32, f, bias_n, stage);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        epi_bar_sync();
        if (a.q_out)
          copy_out_swap_q<BN>(a, u, epi_tid, stage);
        else
          copy_out_swap<BN>(a, u, epi_tid, stage);
        if (unit + static_cast<int>(gridDim.x) < total_units) epi_bar_sync();  // staging free
      } else if constexpr (MODE == kSplitNone) {
        if (a.res == nullptr) {
          epilogue_rows_drain_g2<BN>(a, &tm_y, t_row, u.b, u.tp * kBlockP, u.tq * BN, row,
                                     epi_tid, egroup, smem + L::kOffYStage, &tempty[acc]);
        } else {
          epilogue_rows_tma_g2<BN>(a, &tm_y, &tm_res, full + L::kRbarIndex, rphase, t_row, u.b,
                                   u.tp * kBlockP, u.tq * BN, row, epi_tid, egroup,
                                   smem + L::kOffYStage, abort_flag);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
      } else if constexpr (MODE == kSplitWorkspace && SWAP) {
        // Split-K, swap-AB: publish this slice's fp32 partial (valid rows m
        // only, stored [m][n] so a warp writes 128 contiguous bytes per m) and
        // take a ticket.  The last slice of the tile to arrive sums all slices
        // in slice order -- its own straight from TMEM -- and writes the tile
        // through the staging buffer.
        const int mt = min(BN, a.M - u.tq * BN);  // valid tile rows m
        const int64_t slice_floats = static_cast<int64_t>(BN) * kBlockP;
        const float *tile_ws = a.ws_partial + static_cast<int64_t>(u.tile) * a.splits * slice_floats;
        float *mine = a.ws_partial + static_cast<int64_t>(unit) * slice_floats + row;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          const int q0 = c * 32;
          if (q0 >= mt) break;  // warp-uniform
          uint32_t v[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (q0 + j < mt) __stcg(mine + (q0 + j) * kBlockP, __uint_as_float(v[j]));
        }
        // the last slice's bulk copies (async proxy) read these partials
        fence_proxy_async_global();
        epi_bar_sync();  // every partial store of this CTA is issued
        if (epi_tid == 0) {
          __threadfence();  // ... and visible device-wide before the ticket
          const int prev = atomicAdd(&a.ws_ticket[u.tile], 1);
          const int last = prev == a.splits - 1;
          if (last) {
            a.ws_ticket[u.tile] = 0;  // ready for the next call
            __threadfence();          // the other slices' partials are visible from here
          }
          *last_flag = last;
        }
        epi_bar_sync();
        if (*last_flag) {
          // The other slices' partial tiles arrive by bulk copies (one per
          // slice, as many per pass as the landing area holds) while this
          // slice's own partial goes from TMEM into shared memory in the same
          // [m][n] layout.  Then every thread sums float4 groups of the tile
          // (up to BN/4 of them, all loads independent) in slice order and
          // writes them, 4 outputs of one row m per store.
          float *land = reinterpret_cast<float *>(smem + L::kOffLand);
          float *own = reinterpret_cast<float *>(smem + L::kOffAcc);
          const int tile_floats = mt * kBlockP;
          const int groups = mt * (kBlockP / 4);  // float4 groups of the tile
          const int cap = L::kBytesLand / (tile_floats * 4);  // >= 2 (mt <= 64)
          float4 r[BN / 4];
#pragma unroll
          for (int i = 0; i < BN / 4; ++i) r[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          bool ok = true, dumped = false;
#pragma unroll 1
          for (int s0 = 0; s0 < a.splits && ok;) {
            // slices [s0, s1) of this pass hold `n` landed (other) slices
            int s1 = s0, n = 0;
            while (s1 < a.splits && (n < cap || s1 == u.split)) {
              if (s1 != u.split) ++n;
              ++s1;
            }
            if (n > 0 && epi_tid == 0) {
              // the other slices' generic stores, acquired through the
              // ticket, are read next by bulk copies (async proxy)
              fence_proxy_async_global();
              mbar_arrive_expect_tx(land_bar, static_cast<uint32_t>(n * tile_floats * 4));
              int slot = 0;
              for (int sl = s0; sl < s1; ++sl)
                if (sl != u.split)
                  bulk_load(land + (slot++) * tile_floats, tile_ws + sl * slice_floats,
                            static_cast<uint32_t>(tile_floats * 4), land_bar);
            }
            if (!dumped) {
#pragma unroll 1
              for (int c = 0; c < BN / 32; ++c) {
                if (c * 32 >= mt) break;  // warp-uniform
                uint32_t v[32];
                __syncwarp();
                tmem_ld_32x32b_x32(t_row + c * 32, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (c * 32 + j < mt) own[(c * 32 + j) * kBlockP + row] = __uint_as_float(v[j]);
              }
              dumped = true;
            }
            epi_bar_sync();  // the own tile (and the biases) are in shared memory
            if (n > 0) {
              ok = mbar_wait(land_bar, land_phase, a.err, abort_flag, kWaitLanding);
              land_phase ^= 1;
            }
            int slot = 0;
#pragma unroll 1
            for (int sl = s0; sl < s1 && ok; ++sl) {
              const float4 *src = reinterpret_cast<const float4 *>(
                  sl == u.split ? own : land + (slot++) * tile_floats);
#pragma unroll
              for (int i = 0; i < BN / 4; ++i) {
                const int g = epi_tid + 128 * i;
                if (g < groups) {
                  const float4 w = src[g];
                  r[i].x += w.x;
                  r[i].y += w.y;
                  r[i].z += w.z;
                  r[i].w += w.w;
                }
              }
            }
            epi_bar_sync();  // the landing area is free for the next pass
            s0 = s1;
          }
          const float *bias_s = reinterpret_cast<const float *>(smem + L::kOffBiasS);
          const bool lean = a.res == nullptr && a.act == 0;
#pragma unroll
          for (int i = 0; i < BN / 4; ++i) {
            const int g = epi_tid + 128 * i;
            const int m = g / (kBlockP / 4);
            const int nl = (g % (kBlockP / 4)) * 4;
            const int n = u.tp * kBlockP + nl;
            if (g < groups && n < a.N) {
              const float vals[4] = {r[i].x, r[i].y, r[i].z, r[i].w};
              float o[4];
#pragma unroll
              for (int j = 0; j < 4; ++j)
                o[j] = lean ? a.alpha * vals[j] + bias_s[nl + j]
                            : swap_value(a, u.b, u.tq * BN + m, n + j, vals[j], bias_s[nl + j]);
              const __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]);
              const __nv_bfloat162 hi = __floats2bfloat162_rn(o[2], o[3]);
              uint2 pk;
              pk.x = *reinterpret_cast<const uint32_t *>(&lo);
              pk.y = *reinterpret_cast<const uint32_t *>(&hi);
              *reinterpret_cast<uint2 *>(a.y + u.b * a.y_bstride +
                                         static_cast<int64_t>(u.tq * BN + m) * a.ldy + n) = pk;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        epi_bar_sync();  // last_flag and the shared tiles are free again
      } else {
        static_assert(MODE == kSplitWorkspace, "split mode");
        // Split-K: publish this slice's partial tile, then the last slice to
        // arrive reduces all slices in slice order.
        float *mine = a.ws_partial + (static_cast<int64_t>(unit) * kBlockP + row) * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(mine + c * 32 + j) =
                make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                            __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        __threadfence();
        epi_bar_sync();
        if (epi_tid == 0) {
          const int prev = atomicAdd(&a.ws_ticket[u.tile], 1);
          *last_flag = (prev == a.splits - 1);
        }
        epi_bar_sync();
        if (*last_flag) {
          __threadfence();
          const float *base =
              a.ws_partial + (static_cast<int64_t>(u.tile) * a.splits * kBlockP + row) * BN;
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            float f[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = 0.0f;
            for (int sl = 0; sl < a.splits; ++sl) {
              const float *src = base + static_cast<int64_t>(sl) * kBlockP * BN + c * 32;
              float4 w[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) w[j] = __ldcg(reinterpret_cast<const float4 *>(src) + j);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                f[4 * j] += w[j].x;
                f[4 * j + 1] += w[j].y;
                f[4 * j + 2] += w[j].z;
                f[4 * j + 3] += w[j].w;
              }
            }
            emit32<SWAP>(a, u.b, prow, u.tq * BN + c * 32, f, bias_n);
          }
          if (epi_tid == 0) a.ws_ticket[u.tile] = 0;  // ready for the next call
        }
        epi_bar_sync();
      }
      if (++acc == ACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  // The epilogue's last TMA stores must be done before the CTA retires.
  if constexpr (L::kBytesYStage > 0)
    if (threadIdx.x == 64 || threadIdx.x == kEpi2FirstThread) bulk_wait_group_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace bq
