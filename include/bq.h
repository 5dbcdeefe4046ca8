/*
 * bq.h -- C ABI of libbq: MX (per-32, E8M0-scaled) activation quantization and
 * block-scaled GEMMs for NVIDIA B200 (sm_100a).
 *
 * What the calls compute is defined on the "formats.py" page
 * (dsv41-sampled-drafting, code/offload/dspark/native/formats.py): the
 * activation quantizer (act_scale / act_quant and the module docstring's
 * description of act_qdq) and the exact decoders of the weight formats (module
 * docstring "Formats", decode_fp4, decode_fp8_block).  The fused bias /
 * residual / GELU epilogue follows the FlashRT "fp4-gemm" page ("Available
 * Functions": nvfp4_gemm_bias_bf16, ..._bias_residual_bf16, ..._bias_gelu_bf16)
 * and the AstrAI commit log (bias added in fp32 before the single bf16
 * rounding; batch strides with stride 0 broadcasting a size-1 batch).
 *
 * Conventions for every call:
 *   - All data pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or synchronizes on the data path.
 *   - Every call is asynchronous on the caller's stream (NULL = the legacy
 *     default stream); the return value only reports argument checks and
 *     launch errors.  Exceptions, which synchronize the stream, are named.
 *   - Sizes are 64-bit.  M or N equal to 0 returns BQ_OK without a launch.
 *   - Argument faults are detected on the host before any launch; nothing is
 *     launched when a call returns an error.
 *   - The current device must be compute capability 10.0 (B200), else
 *     BQ_ERR_ARCH.
 *
 * Layouts:
 *   - bf16 activations x [M, K] row-major with row stride ldx elements.
 *   - E4M3 codes (activations, FP8 weights) [rows, K] row-major, 1 byte each.
 *   - MXFP4 weights [N, K/2] bytes; byte j of a row holds input 2j in the
 *     low nibble and 2j+1 in the high nibble.
 *   - bf16 output y [M, N] row-major, y = A * B^T.
 *   - Scale factors in "MMA layout" (the layout the GEMM consumes): for a
 *     matrix of R rows and K inputs the G = K/32 scale bytes of each row are
 *     stored in 512-byte atoms of 128 rows x 4 scale columns.  The atom of
 *     (row r, column c) is (r / 128) * ceil(G / 4) + c / 4 and the byte inside
 *     it is (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4).  Rows are padded to a
 *     multiple of 128 and columns to a multiple of 4; the producers write the
 *     padding bytes as 127 (2^0).  Size: bq_sf_bytes(R, K).
 */
#ifndef BQ_H
#define BQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *bq_stream_t;

/* ---- status codes ---------------------------------------------------- */
enum {
  BQ_OK = 0,
  BQ_ERR_NULL = 1,        /* a required pointer is NULL */
  BQ_ERR_SHAPE = 2,       /* size out of range or not a multiple the call needs */
  BQ_ERR_ALIGN = 3,       /* base address or row stride breaks the 16-byte (FP4: 32-byte) rule */
  BQ_ERR_NAN_SCALE = 4,   /* an E8M0 scale byte is 255 (NaN) -- prepack only */
  BQ_ERR_NAN_CODE = 5,    /* an E4M3 weight code is 0x7F or 0xFF (NaN) -- prepack only */
  BQ_ERR_ARCH = 6,        /* current device is not compute capability 10.0 */
  BQ_ERR_WORKSPACE = 7,   /* workspace NULL or smaller than bq_gemm_workspace_bytes() */
  BQ_ERR_CUDA = 8,        /* a CUDA runtime call or kernel launch failed */
  BQ_ERR_TIMEOUT = 9,     /* a kernel gave up waiting on one of its own barriers */
  BQ_ERR_NONFINITE = 10,  /* a NaN or Inf input (act_quant) or quantized output (GEMM) */
  BQ_ERR_INVALID = 11     /* an enum argument is out of range */
};

/* Human-readable name of a status code (static string, never NULL). */
const char *bq_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
int bq_version(void);

/* Bytes of an MMA-layout scale buffer for `rows` rows and `K` inputs
 * (K % 32 == 0): ceil(rows / 128) * ceil(K / 128) * 512.  0 for bad sizes. */
size_t bq_sf_bytes(int64_t rows, int64_t K);

/* Bytes of an MMA-layout buffer of NVFP4 scales (one E4M3 byte per 16 inputs,
 * K % 16 == 0): ceil(rows / 128) * ceil(K / 64) * 512 (an atom holds 4 groups
 * of 16).  0 for bad sizes. */
size_t bq_sf_bytes_nvfp4(int64_t rows, int64_t K);

/* ---- activation quantization ------------------------------------------ */

/* bq_act_quant -- per-32 MX quantization of bf16 activations
 * ("formats.py" page: act_scale, act_quant; the module docstring on act_qdq).
 *
 * For every 32 consecutive elements of a row: amax = max(max|x|, 1e-4) in
 * fp32; t = fp32(amax * fp32(1/448)); e = ceil(log2 t) from t's exponent bits;
 * scale byte = e + 127 (E8M0); q = E4M3 round-to-nearest-even of
 * clamp(x / 2^e, -448, 448).  Bit-exact with that definition for finite input.
 *
 *   x_bf16      [M, K] bf16, row stride ldx elements (ldx >= K, ldx % 8 == 0,
 *               base 16-byte aligned)
 *   M, K        M >= 0; K > 0 and K % 32 == 0
 *   q_e4m3      out [M, K] E4M3 codes, row stride K, 16-byte aligned
 *   sf_mma      out bq_sf_bytes(M, K) bytes, MMA layout, padding written as 127
 *   sf_rowmajor optional out [M, K/32] scale bytes row-major (NULL to skip)
 *   d_status    optional device int; the kernel ORs in 1 when it meets a NaN
 *               or Inf input (whose outputs are then unspecified).  The caller
 *               zeroes it.  NULL to skip the check.
 * Errors: BQ_ERR_NULL, BQ_ERR_SHAPE, BQ_ERR_ALIGN, BQ_ERR_ARCH, BQ_ERR_CUDA. */
int bq_act_quant(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, void *q_e4m3,
                 void *sf_mma, void *sf_rowmajor, int *d_status, bq_stream_t stream);

/* bq_act_quant_mxfp4 -- per-32 MXFP4 quantization of bf16 activations, for the
 * FP4 x FP4 GEMM (the A4W4 kernels of the "fp4-gemm" page, README "Available
 * Functions" and "Tensor Contract": packed E2M1 activations with block
 * scales).  The pages define the per-32 rule for E4M3 codes (bq_act_quant);
 * for E2M1 codes the same rule takes the format's largest value 6 in place of
 * 448: t = fp32(amax * fp32(1/6)), e = ceil(log2 t), scale byte = e + 127,
 * q = E2M1 round-to-nearest-even of clamp(x / 2^e, -6, 6), the sign kept
 * (negative values that round to zero give code 8, -0).  Two codes per byte,
 * the even element in the low nibble (the pages' MXFP4 weight layout).
 *   q_fp4  out [M, K/2] packed E2M1 codes, row stride K/2 bytes, 16-byte aligned
 *   all other arguments and errors as bq_act_quant. */
int bq_act_quant_mxfp4(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, void *q_fp4,
                       void *sf_mma, void *sf_rowmajor, int *d_status, bq_stream_t stream);

/* bq_act_quant_nvfp4 -- NVFP4 quantization of bf16 activations for the NVFP4
 * A4W4 GEMM (the "fp4-gemm" page, README: NVFP4 A4W4 kernels, E2M1 codes with
 * CUTLASS-layout scale buffers).  The pages give no quantization rule; this
 * one: every value is first fp32(x * g), g > 0 the caller's per-tensor scale;
 * per 16 consecutive values of a row the scale is s = the smallest E4M3 value
 * >= fp32(amax * fp32(1/6)) (2^-9 at least, 448 at most: the round-up
 * counterpart of bq_act_quant's rule, so no value clips unless amax g > 2688)
 * and q = E2M1 round-to-nearest-even of fp32(x g / s), sign kept.  A GEMM of
 * two such operands returns alpha * sum(q_a s_a q_b s_b); alpha = 1 / (g_a g_b)
 * in the epilogue gives the product of the unscaled tensors.
 *   q_fp4   out [M, K/2] packed E2M1 (even element low), 16-byte aligned
 *   sf_mma  out bq_sf_bytes_nvfp4(M, K): MMA layout of 16-input groups,
 *           padding bytes 0x38 (1.0)
 *   sf_rowmajor optional out [M, K/16]; K % 32 == 0; other arguments as
 *   bq_act_quant.  Errors: as bq_act_quant, BQ_ERR_INVALID for g <= 0 or not
 *   finite. */
int bq_act_quant_nvfp4(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, float g,
                       void *q_fp4, void *sf_mma, void *sf_rowmajor, int *d_status,
                       bq_stream_t stream);

/* ---- backward-pass quantizers ------------------------------------------- */

enum { BQ_ROUND_NEAREST = 0, BQ_ROUND_STOCHASTIC = 1 };
enum { BQ_FMT_E4M3 = 0, BQ_FMT_E5M2 = 1 };

/* bq_grad_quant -- per-32 E5M2 quantization of bf16 gradients along the last
 * dimension (the "hip_quant" README on the pages: E5M2 for backward gradients,
 * "Stochastic E5M2 Backward Gradients", "Block-wise FP8 Scaling"), with the
 * scale rule of bq_act_quant taking E5M2's largest finite value 57344 in place
 * of 448: t = fp32(max(amax, 1e-4) * fp32(1/57344)), e = ceil(log2 t), scale
 * byte e + 127, q = E5M2 of clamp(g / 2^e, -57344, 57344).
 *   rounding BQ_ROUND_NEAREST: round to nearest even (saturating), sign kept.
 *   rounding BQ_ROUND_STOCHASTIC: between the two neighbouring E5M2 values of
 *            |g / 2^e| (lo, hi; the 2^-16 grid below 2^-14), hi when
 *            u < (|v| - lo) / (hi - lo), u the element's draw times 2^-32: the
 *            32-bit half (i mod 2, low half first) of word (i / 2) mod 4 of
 *            Philox4x64-10 at counter (i / 8, 0, 0, 0) under key (seed, 0),
 *            i = row * K + column, so the draws are a stateless function of
 *            (seed, element index).
 *   g_bf16 [M, K] (row stride ldg), q_e5m2 out [M, K], sf_mma out
 *   bq_sf_bytes(M, K) (MMA layout), sf_rowmajor / d_status as bq_act_quant.
 * Errors: as bq_act_quant, BQ_ERR_INVALID for a bad rounding mode. */
int bq_grad_quant(const void *g_bf16, int64_t M, int64_t K, int64_t ldg, void *q_e5m2,
                  void *sf_mma, void *sf_rowmajor, int *d_status, int rounding, uint64_t seed,
                  bq_stream_t stream);

/* bq_quant_transposed -- quantization along the FIRST dimension, written
 * transposed (the operands of the weight gradient dW = dY^T X contract over
 * the token dimension, and the input gradient dX = dY W over the output
 * dimension: "quantize_e5m2_transpose" on the "hip_quant" README page).
 * x [R, C] bf16 (row stride ldx >= C, ldx % 8 == 0, C % 8 == 0, R % 32 == 0) is
 * quantized per 32 consecutive rows of each column by the bq_act_quant rule
 * (fmt BQ_FMT_E4M3) or the bq_grad_quant rule (fmt BQ_FMT_E5M2; stochastic
 * rounding draws with i = r * C + c, the element's index in x), and stored as
 *   q_t     out [C, R] codes (row pitch R), 16-byte aligned
 *   sf_mma  out bq_sf_bytes(C, R): the MMA-layout scales of the [C, R] operand
 * so that (q_t, sf_mma) is an operand of the GEMMs with C rows and K = R.
 * Errors: BQ_ERR_NULL, BQ_ERR_SHAPE, BQ_ERR_ALIGN, BQ_ERR_INVALID (fmt,
 * rounding, or stochastic E4M3), BQ_ERR_ARCH, BQ_ERR_CUDA. */
int bq_quant_transposed(const void *x_bf16, int64_t R, int64_t C, int64_t ldx, int fmt,
                        int rounding, uint64_t seed, void *q_t, void *sf_mma, int *d_status,
                        bq_stream_t stream);

/* bq_grad_quant_dual -- both quantizations of an output gradient g [R, C] in
 * one pass: q_row [R, C] with scales along C (exactly bq_grad_quant) and q_t
 * [C, R] with scales along R (exactly bq_quant_transposed with BQ_FMT_E5M2),
 * reading g once and drawing each element's stochastic draw (index r * C + c
 * under `seed`) once for both.  R % 32 == 0, C % 32 == 0, ldg >= C,
 * ldg % 8 == 0; sf_row: bq_sf_bytes(R, C), sf_t: bq_sf_bytes(C, R); q_row and
 * q_t 16-byte aligned.  Errors as bq_grad_quant. */
int bq_grad_quant_dual(const void *g_bf16, int64_t R, int64_t C, int64_t ldg, int rounding,
                       uint64_t seed, void *q_row, void *sf_row, void *q_t, void *sf_t,
                       int *d_status, bq_stream_t stream);

/* ---- weight scale prepack (off the hot path) --------------------------- */

enum {
  BQ_SF_ROW32 = 0,    /* scales [N, K/32]: one per 32 inputs of a row (MXFP4, MXFP8) */
  BQ_SF_BLK32x32 = 1, /* scales [ceil(N/32), ceil(K/32)]: one per 32x32 block (FP8 weights) */
  BQ_SF_ROW16_E4M3 = 2 /* NVFP4: E4M3 scales [N, K/16], one per 16 inputs of a row; output
                          bq_sf_bytes_nvfp4(N, K) bytes, padding 0x38; 0x7F/0xFF refused */
};

/* bq_pack_weight_scales -- E8M0 weight scales to MMA layout
 * ("formats.py" page, docstring "Formats": FP4 scales [out, in/32], FP8 scales
 * [ceil(out/32), ceil(in/32)]; decode_fp8_block repeats a block's scale over
 * its 32 rows and 32 inputs).  A 32x32 block scale is written to each of its
 * 32 rows.  Scans the scales for 255 (NaN) and, when e4m3_codes ([N, K]) is
 * given, the codes for 0x7F/0xFF.  SYNCHRONIZES `stream` to report those.
 *   sf_mma: out, bq_sf_bytes(N, K) bytes.  K % 32 == 0.
 * Errors: BQ_ERR_NAN_SCALE, BQ_ERR_NAN_CODE (sf_mma content then unspecified),
 *         BQ_ERR_NULL, BQ_ERR_SHAPE, BQ_ERR_INVALID, BQ_ERR_ARCH, BQ_ERR_CUDA. */
int bq_pack_weight_scales(const void *scales_u8, int kind, int64_t N, int64_t K, void *sf_mma,
                          const void *e4m3_codes, bq_stream_t stream);

/* bq_unpack_scales -- MMA layout back to row-major [rows, K/32] bytes (for
 * tests and inspection). */
int bq_unpack_scales(const void *sf_mma, int64_t rows, int64_t K, void *rowmajor,
                     bq_stream_t stream);

/* ---- block-scaled GEMM -------------------------------------------------- */

/* Operands of every GEMM call:
 *   a_q   [M, K] E4M3 activation codes (from bq_act_quant), 16-byte aligned
 *   a_sf  MMA-layout scales of A (from bq_act_quant), bq_sf_bytes(M, K)
 *   b     weights, 16-byte aligned (MXFP4: 32-byte aligned):
 *           mxfp4:    [N, K/2] packed E2M1, requires K % 128 == 0 (BQ_ERR_SHAPE
 *                     otherwise).  The "formats.py" page ("Formats") only asks
 *                     for K % 32 == 0; the narrower rule is this library's: the
 *                     tensor-memory-access type that spreads 4-bit codes to the
 *                     byte slots the MMA reads moves whole 128-code rows, and a
 *                     tail shorter than 128 codes would need a read past the end
 *                     of the weight buffer.  Pad K of both operands to a multiple
 *                     of 128 with zero codes (and any finite scale) to use other
 *                     sizes.
 *           fp8blk32: [N, K] E4M3 (32x32 block scales, packed by
 *                     bq_pack_weight_scales(BQ_SF_BLK32x32))
 *           mxfp8:    [N, K] E4M3 (per-32 row scales, from bq_act_quant or
 *                     bq_pack_weight_scales(BQ_SF_ROW32))
 *   b_sf  MMA-layout scales of B, bq_sf_bytes(N, K)
 *   y     [M, N] bf16 out, N % 8 == 0, 16-byte aligned
 * y[m, n] = bf16_RNE(sum_k a[m,k] b[n,k]) with a, b the decoded operands
 * (code * 2^(scale-127)) and fp32 accumulation.
 * Errors: BQ_ERR_NULL, BQ_ERR_SHAPE, BQ_ERR_ALIGN, BQ_ERR_ARCH, BQ_ERR_CUDA.
 * No data is scanned on this path: NaN scales or codes give NaN outputs.
 * Launch order: the GEMM kernels (and bq_act_quant) use programmatic dependent
 * launch -- a GEMM may start while the kernel just before it in the stream is
 * still running.  It waits for that kernel before reading the activations,
 * scales, bias or residual and before writing y, but it may read the weight
 * operand b and b_sf early: they must not be written by the kernel issued
 * immediately before the GEMM on the same stream (anything older has finished).
 * Once all its thread blocks are past that wait, a GEMM lets the next kernel
 * of the stream launch if that kernel was launched programmatically (as this
 * library's are); such a kernel waits for the GEMM before touching its output. */
int bq_gemm_mxfp8_mxfp4(const void *a_q, const void *a_sf, const void *b_fp4, const void *b_sf,
                        int64_t M, int64_t N, int64_t K, void *y_bf16, bq_stream_t stream);
int bq_gemm_mxfp8_fp8blk32(const void *a_q, const void *a_sf, const void *b_e4m3,
                           const void *b_sf, int64_t M, int64_t N, int64_t K, void *y_bf16,
                           bq_stream_t stream);
int bq_gemm_mxfp8_mxfp8(const void *a_q, const void *a_sf, const void *b_e4m3, const void *b_sf,
                        int64_t M, int64_t N, int64_t K, void *y_bf16, bq_stream_t stream);

/* bq_gemm_mxfp4_mxfp4 -- the FP4 x FP4 (A4W4) product ("fp4-gemm" page,
 * README "Available Functions": the bf16-output A4W4 GEMM; "Tensor
 * Contract": a_packed [M, K/2], b_packed [N, K/2], scale buffers in the MMA
 * layout, bf16 [M, N] out) with E8M0 scales per 32 inputs on both sides
 * (MXFP4), on tcgen05.mma kind::mxf4:
 *   a_fp4  [M, K/2] packed E2M1 activation codes (bq_act_quant_mxfp4), 16-byte aligned
 *   a_sf   MMA-layout scales of A (bq_act_quant_mxfp4), bq_sf_bytes(M, K)
 *   b_fp4  [N, K/2] packed E2M1 weight codes, low nibble = even input, 16-byte aligned
 *   b_sf   bq_pack_weight_scales(BQ_SF_ROW32) of the [N, K/32] weight scales
 * K % 128 == 0; everything else (y, errors, stream order) as the GEMMs above.
 * The pages' A4W4 kernels use NVFP4 (E4M3 scales per 16 inputs); that scale
 * format is not implemented here. */
int bq_gemm_mxfp4_mxfp4(const void *a_fp4, const void *a_sf, const void *b_fp4, const void *b_sf,
                        int64_t M, int64_t N, int64_t K, void *y_bf16, bq_stream_t stream);

/* bq_gemm_nvfp4_nvfp4 -- the NVFP4 A4W4 product ("fp4-gemm" page, README
 * "Available Functions": the bf16-output NVFP4 GEMM with alpha) on
 * tcgen05.mma kind::mxf4nvf4 (scale_vec::4X, UE4M3 scales): a_fp4 / b_fp4
 * packed E2M1 [M, K/2] / [N, K/2], a_sf from bq_act_quant_nvfp4, b_sf from
 * bq_pack_weight_scales(BQ_SF_ROW16_E4M3).  K % 128 == 0.  Schedules: wide
 * tiles (128 x 128, 128 x 256) and unsplit swap-AB decode tiles, one 256-K
 * chunk per stage; a K split, pair tiles or more chunks per stage are
 * refused (BQ_ERR_INVALID).  Everything else as the other GEMMs. */
int bq_gemm_nvfp4_nvfp4(const void *a_fp4, const void *a_sf, const void *b_fp4, const void *b_sf,
                        int64_t M, int64_t N, int64_t K, void *y_bf16, bq_stream_t stream);

/* bq_gemm_e5m2_mxfp8 -- the backward products: A holds E5M2 gradient codes
 * with E8M0 scales per 32 along K (bq_grad_quant, or bq_quant_transposed with
 * BQ_FMT_E5M2), B E4M3 codes with per-32 scales along K (bq_act_quant /
 * bq_quant_transposed with BQ_FMT_E4M3), y = A B^T in bf16 (fp32 accumulate,
 * kind::mxf8f6f4 with an E5M2 A operand).  dX = bq_gemm_e5m2_mxfp8(dY_q,
 * W^T_q) with W^T quantized along the output dimension; dW =
 * bq_gemm_e5m2_mxfp8(dY^T_q, X^T_q), both transposed along the token
 * dimension.  Operand layouts, alignment, errors and stream order as the other
 * GEMMs: B is read early, so quantize both B operands (W^T, X^T) before dY. */
int bq_gemm_e5m2_mxfp8(const void *a_e5m2, const void *a_sf, const void *b_e4m3, const void *b_sf,
                       int64_t M, int64_t N, int64_t K, void *y_bf16, bq_stream_t stream);

enum { BQ_ACT_NONE = 0, BQ_ACT_GELU = 1 };

/* Fused epilogue, applied in fp32 with one bf16 rounding at the end:
 *   y = bf16_RNE( act(alpha * acc + bias[n]) + residual[m, n] )
 * act: BQ_ACT_NONE or BQ_ACT_GELU (erf form 0.5 t (1 + erf(t / sqrt 2))).
 * bias: [N] bf16 or NULL.  residual: [M, ld_residual] bf16 or NULL
 * (ld_residual % 8 == 0, 16-byte aligned).
 *
 * Quantized output (optional, q_out and sf_out both set or both NULL): the
 * epilogue also applies bq_act_quant to y along N -- per 32 consecutive
 * outputs of a row, the same amax, E8M0 scale and E4M3 codes as bq_act_quant
 * on the bf16 y -- and writes q_out [M, N] u8 (E4M3 codes, row-major) and
 * sf_out (bq_sf_bytes(M, N) bytes, the MMA scale layout with 127 padding), so
 * the output feeds another GEMM as its activation operand directly.  The
 * "fp4-gemm" page (README, "Available Functions" and "Tensor Contract": the
 * bias+GELU epilogue that emits packed FP4 plus its scale layout for the
 * following projection) describes this epilogue for NVFP4; here it is the
 * MXFP8 form of the activation quantizer above.  Needs N % 32 == 0,
 * q_out 16-byte aligned, sf_out 4-byte aligned; y may then be NULL (no bf16
 * output written).  Batched calls step q_out by stride_y / 2 bytes and sf_out
 * by bq_sf_bytes(M, N).  Schedules that split K are not available with it
 * (an explicit split is refused with BQ_ERR_INVALID; the automatic schedule
 * does not split). */
typedef struct {
  const void *bias;
  const void *residual;
  int64_t ld_residual;
  float alpha;
  int act;
  void *q_out;
  void *sf_out;
} bq_epilogue;

/* Batched GEMM: `count` independent problems.  Strides are in BYTES between
 * consecutive problems; a stride of 0 broadcasts that operand (e.g. one weight
 * shared by all problems).  stride_a_sf / stride_b_sf step the MMA-layout
 * scale buffers and must be multiples of 16.  Bias is shared by all problems. */
typedef struct {
  int64_t count;
  int64_t stride_a, stride_a_sf;
  int64_t stride_b, stride_b_sf;
  int64_t stride_y, stride_res;
} bq_batch;

/* Optional schedule override (tests and sweeps); NULL = built-in dispatch.
 * block_n:    0 (auto); 128 or 256 weight rows per CTA tile, or with swap_ab 32
 *             or 64 activation rows per CTA tile.
 * split_k:    0 (auto) or 1..16 slices of K.
 * swap_ab:    -1 (auto), 0, or 1 (weights on the 128-row MMA side, for M <= 64).
 * split_mode: how K slices are combined, always in slice order:
 *             BQ_SPLIT_AUTO      cluster when possible, else workspace;
 *             BQ_SPLIT_WORKSPACE fp32 partials in the caller's workspace, the
 *                                last slice to finish reduces (needs workspace);
 *             BQ_SPLIT_CLUSTER   the slices of a tile form a thread-block cluster
 *                                and reduce through distributed shared memory
 *                                (swap_ab tiles, split_k a power of two <= 8;
 *                                no workspace). */
enum { BQ_SPLIT_AUTO = 0, BQ_SPLIT_WORKSPACE = 1, BQ_SPLIT_CLUSTER = 2 };
typedef struct {
  int block_n;
  int split_k;
  int swap_ab;
  int split_mode;
  int k_chunks; /* 128-K chunks per pipeline stage: 0 (auto), 1, 2 or (swap_ab) 4;
                   more than 1 needs K % 128 == 0 and no workspace split */
  int cta_pair; /* 0 (auto), 1 single-SM tiles, 2 256x256 tiles on pairs of SMs (a
                   2-CTA cluster sharing each MMA; wide tiles, no split, k_chunks <= 2) */
} bq_gemm_config;

/* Workspace bytes the *_epilogue calls need for a problem (0 when the chosen
 * schedule needs none).  weight_kind: 0 mxfp4, 1 fp8blk32, 2 mxfp8, 3 mxfp4 weights
 * with MXFP4 activations (bq_gemm_mxfp4_mxfp4*), 4 E5M2 x MXFP8 (bq_gemm_e5m2_mxfp8*),
 * 5 NVFP4 x NVFP4 (bq_gemm_nvfp4_nvfp4*). */
size_t bq_gemm_workspace_bytes(int weight_kind, int64_t M, int64_t N, int64_t K, int64_t batch,
                               const bq_gemm_config *cfg);

/* The schedule the built-in dispatch picks for a problem of weight_kind (as
 * for bq_gemm_workspace_bytes) on a device with `num_sms` SMs, with `cfg`
 * (NULL = all auto) as a *_epilogue call would get it: every field of *out
 * resolved (block_n, split_k >= 1, swap_ab 0/1,
 * split_mode BQ_SPLIT_WORKSPACE or BQ_SPLIT_CLUSTER when split_k > 1, else
 * BQ_SPLIT_AUTO, k_chunks >= 1, cta_pair 1 or 2).  Host-only: touches no
 * device.  Calls that ask for a quantized output run unsplit.  Returns
 * BQ_ERR_NULL (out NULL), BQ_ERR_SHAPE (sizes out of range, num_sms < 1) or
 * BQ_ERR_INVALID (weight_kind or cfg not schedulable, the status the GEMM call
 * returns). */
int bq_gemm_plan(int weight_kind, int64_t M, int64_t N, int64_t K, int64_t batch,
                 const bq_gemm_config *cfg, int num_sms, bq_gemm_config *out);

/* GEMM + fused epilogue (+ optional batch).  epi NULL = plain (alpha 1, no
 * bias, residual or activation).  batch NULL = one problem.  workspace: device
 * memory of at least bq_gemm_workspace_bytes(...) bytes (may be NULL when that
 * is 0), 16-byte aligned.  Its first 64 KiB hold per-tile counters that must be
 * zero before the first use (e.g. a zero-filled allocation); every call that
 * completes leaves them zero again, so one workspace serves any sequence of
 * problems.  Calls that share one workspace must not overlap on the GPU.  A
 * split-K schedule is limited to 16384 output tiles (else BQ_ERR_SHAPE). */
int bq_gemm_mxfp8_mxfp4_epilogue(const void *a_q, const void *a_sf, const void *b_fp4,
                                 const void *b_sf, int64_t M, int64_t N, int64_t K, void *y_bf16,
                                 const bq_epilogue *epi, const bq_batch *batch, void *workspace,
                                 size_t workspace_bytes, const bq_gemm_config *cfg,
                                 bq_stream_t stream);
int bq_gemm_mxfp8_fp8blk32_epilogue(const void *a_q, const void *a_sf, const void *b_e4m3,
                                    const void *b_sf, int64_t M, int64_t N, int64_t K,
                                    void *y_bf16, const bq_epilogue *epi, const bq_batch *batch,
                                    void *workspace, size_t workspace_bytes,
                                    const bq_gemm_config *cfg, bq_stream_t stream);
int bq_gemm_mxfp8_mxfp8_epilogue(const void *a_q, const void *a_sf, const void *b_e4m3,
                                 const void *b_sf, int64_t M, int64_t N, int64_t K, void *y_bf16,
                                 const bq_epilogue *epi, const bq_batch *batch, void *workspace,
                                 size_t workspace_bytes, const bq_gemm_config *cfg,
                                 bq_stream_t stream);
/* NVFP4 x NVFP4 with the same epilogue (alpha = 1 / (g_a g_b) undoes the
 * per-tensor scales), batch and schedule options within the limits above. */
int bq_gemm_nvfp4_nvfp4_epilogue(const void *a_fp4, const void *a_sf, const void *b_fp4,
                                 const void *b_sf, int64_t M, int64_t N, int64_t K, void *y_bf16,
                                 const bq_epilogue *epi, const bq_batch *batch, void *workspace,
                                 size_t workspace_bytes, const bq_gemm_config *cfg,
                                 bq_stream_t stream);
/* E5M2 x MXFP8 (bq_gemm_e5m2_mxfp8) with the same options. */
int bq_gemm_e5m2_mxfp8_epilogue(const void *a_e5m2, const void *a_sf, const void *b_e4m3,
                                const void *b_sf, int64_t M, int64_t N, int64_t K, void *y_bf16,
                                const bq_epilogue *epi, const bq_batch *batch, void *workspace,
                                size_t workspace_bytes, const bq_gemm_config *cfg,
                                bq_stream_t stream);
/* A4W4 (bq_gemm_mxfp4_mxfp4) with the same epilogue, batch, workspace and
 * schedule options. */
int bq_gemm_mxfp4_mxfp4_epilogue(const void *a_fp4, const void *a_sf, const void *b_fp4,
                                 const void *b_sf, int64_t M, int64_t N, int64_t K, void *y_bf16,
                                 const bq_epilogue *epi, const bq_batch *batch, void *workspace,
                                 size_t workspace_bytes, const bq_gemm_config *cfg,
                                 bq_stream_t stream);

/* ---- activation quantization fused into the decode GEMM -------------------
 *
 * bq_gemm_bf16act_epilogue -- bq_act_quant followed by the *_epilogue GEMM of
 * weight_kind (0 mxfp4, 1 fp8blk32, 2 mxfp8) in one launch, for decode-shaped
 * problems: the GEMM's CTAs quantize the bf16 activations x [M, ldx] per
 * 32-group (the bq_act_quant arithmetic) straight into their shared-memory
 * operand stages, so neither the separate launch nor the codes' round trip
 * through memory is on the path.  The results equal bq_act_quant + the
 * epilogue GEMM bit for bit.  a_q_out [M, K] u8 and a_sf_out
 * (bq_sf_bytes(M, K) bytes, MMA layout) optionally receive the activation
 * codes and scales as bq_act_quant writes them; d_status (nullable) gets bit 0
 * set for a non-finite input, as with bq_act_quant.  When the problem's K
 * loop is long enough for a split schedule to win (the 6144-deep decode
 * projection), the call runs bq_act_quant into a_q_out / a_sf_out and the
 * split GEMM instead (two launches; the buffers are then required,
 * BQ_ERR_NULL without them); with a quantized output it always fuses.
 * Scope: 1 <= M <= 64,
 * K % 128 == 0, one problem (no batch), ldx % 8 == 0, x 16-byte aligned; the
 * epilogue options of bq_epilogue apply (quantized output included).  The
 * "fp4-gemm" page ("Minimal Usage") produces the packed activations and their
 * scale layout from bf16 with a separate producer call before the GEMM; here
 * that producer runs inside the GEMM.  Errors as the *_epilogue calls,
 * BQ_ERR_SHAPE outside the scope.
 * Measured on B200 it is slower than the two calls for the decode shapes
 * (every CTA of the GEMM quantizes the whole activation block, and its
 * ordinary loads are throttled while shared memory holds the operand ring):
 * it is provided for callers that want one launch per layer. */
int bq_gemm_bf16act_epilogue(int weight_kind, const void *x_bf16, int64_t ldx, const void *b,
                             const void *b_sf, int64_t M, int64_t N, int64_t K, void *y_bf16,
                             const bq_epilogue *epi, void *a_q_out, void *a_sf_out, int *d_status,
                             bq_stream_t stream);

/* ---- allocation-free GEMM -------------------------------------------------
 *
 * No counterpart on the pages: this is a library convenience.
 *
 * bq_gemm_mxfp8_mxfp4_epilogue_noalloc -- the same computation, arguments and
 * errors as bq_gemm_mxfp8_mxfp4_epilogue, for callers that cannot allocate
 * device memory (for example a plugin inside another runtime that is given only
 * its input and output buffers, or a serving loop whose memory is fixed at
 * start-up).  Instead of a caller-provided workspace, the K-split schedule uses
 * scratch memory the library owns: one array of bq_noalloc_scratch_bytes()
 * bytes (8 MiB) in global memory on every device that loads the library, held
 * until the process exits.  The call allocates nothing (no cudaMalloc or
 * allocating library routine).
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture.
 *   - Every call clears the counters it needs on its stream before the kernel;
 *     all calls share the one array, so calls that overlap on the GPU (other
 *     streams, other host threads) race -- serialize them.
 *   - A problem whose schedule needs more scratch than the array holds returns
 *     BQ_ERR_WORKSPACE without launching (use the workspace variant instead). */
int bq_gemm_mxfp8_mxfp4_epilogue_noalloc(const void *a_q, const void *a_sf, const void *b_fp4,
                                         const void *b_sf, int64_t M, int64_t N, int64_t K,
                                         void *y_bf16, const bq_epilogue *epi,
                                         const bq_batch *batch, const bq_gemm_config *cfg,
                                         bq_stream_t stream);

/* Size in bytes of the library-owned scratch array used by the _noalloc call. */
size_t bq_noalloc_scratch_bytes(void);

/* ---- diagnostics -------------------------------------------------------- */

/* Reads and clears the library's device error word on the current device.
 * SYNCHRONIZES `stream`.  Returns BQ_OK; BQ_ERR_TIMEOUT when a kernel gave up
 * on a barrier wait since the last call (its outputs are then invalid); else
 * BQ_ERR_NONFINITE when a GEMM's quantized-output epilogue met a NaN or Inf
 * output (those groups' scale bytes stay valid, their codes are unspecified). */
int bq_device_status(bq_stream_t stream);

/* bq_device_status, also returning the raw error word in *detail (may be
 * NULL): 0, or bit 0 (a wait gave up) with bits 8..15 naming the site of the
 * first wait that gave up (1 producer/free stage, 2 MMA/free accumulator,
 * 3 MMA/loaded stage, 4 epilogue/finished accumulator, 5 teardown drain,
 * 6/7 cluster split exchange, 8 workspace split landing, 9 the self-test
 * below), and bit 1 (non-finite quantized output).  SYNCHRONIZES. */
int bq_device_status_detail(bq_stream_t stream, int *detail);

/* Watchdog self-test (the hip_quant README's memory-safety guards on the
 * pages, restated for this library's waits): launches one thread that waits,
 * with the bounded wait every kernel here uses, on a barrier nothing ever
 * completes.  The wait gives up after limit_us microseconds (1 .. 1000000),
 * records the timeout in the device error word and the kernel returns: the
 * next bq_device_status call reports BQ_ERR_TIMEOUT (site 9) and clears it,
 * and the context stays usable.  Errors: BQ_ERR_SHAPE (limit out of range),
 * BQ_ERR_ARCH, BQ_ERR_CUDA. */
int bq_selftest_wait_timeout(int64_t limit_us, bq_stream_t stream);

/* Test hook for the architecture check (the hip_quant README's guards on the
 * pages): every entry point that checks the device compares (major, minor)
 * instead of the probed compute capability, so a value other than 10.0 makes
 * them return BQ_ERR_ARCH before launching anything.  It can only refuse: a
 * device that is not 10.0 is refused whatever the override.  Negative values
 * restore the probe.  Host-only; not thread-safe against concurrent calls.
 * Errors: BQ_ERR_INVALID (major > 99 or minor > 9). */
int bq_debug_override_compute_capability(int major, int minor);

/* Writes a one-line report of the current device (name, compute capability,
 * SM count, L2 size, clocks) into buf (always NUL-terminated). */
int bq_device_report(char *buf, size_t n);

#ifdef __cplusplus
}
#endif

#endif /* BQ_H */
