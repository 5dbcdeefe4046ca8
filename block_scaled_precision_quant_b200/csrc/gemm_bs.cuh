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
//
// Structure (one persistent CTA per SM, warp-specialized, 6 warps):
//   warp 0   TMA producer: operand tiles (128B swizzle) and the 512-byte
//            scale-factor atoms into a STAGES-deep shared-memory ring, each
//            stage signalled on an mbarrier with a transaction count;
//   warp 1   TMEM allocator and MMA issuer: per stage, tcgen05.cp copies the
//            scale atoms into TMEM, then 4 MMAs of K = 32 each consume the
//            stage; tcgen05.commit releases the stage and, after the last
//            k-block of a tile, signals the accumulator as full;
//   warps 2-5 epilogue: tcgen05.ld of the fp32 accumulator (one TMEM lane
//            quadrant per warp), alpha / bias / GELU / residual in fp32, one
//            bf16 rounding, vector stores.  With split-K every slice writes
//            fp32 partials to the workspace and the last slice to arrive
//            (atomic ticket) sums all slices in slice order -- the result does
//            not depend on which slice arrives last -- and runs the epilogue.
//
// "P" is the operand on the MMA's 128-row side and "Q" the one on its BN-row
// side.  Normally P = activations and Q = weights (y[p][q]); with SWAP the
// weights go on the 128-row side and a short activation matrix (decode
// shapes) on the BN side, and the epilogue writes the transpose (y[q][p]).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "bq_ptx.cuh"

namespace bq {

constexpr int kBlockP = 128;  // MMA M
constexpr int kBlockK = 128;  // inputs per stage: 128 one-byte codes = one 128B-swizzle row
constexpr int kMmaK = 32;     // inputs per tcgen05.mma (one scale per row per MMA)
constexpr int kSfAtom = 512;  // bytes of one 128-row x 4-column scale atom
constexpr int kNumThreads = 192;

// tcgen05 operand formats (instruction descriptor fields a_format / b_format).
constexpr uint32_t kFmtE4M3 = 0;
constexpr uint32_t kFmtE2M1 = 5;

struct GemmArgs {
  int M, N, K;     // one problem: y[M, N] = A[M, K] B[N, K]^T
  int batch;       // number of problems
  int kt_total;    // ceil(K / 128)
  int splits;      // K slices per output tile (1 = no split)
  int kt_per_split;
  int tiles_p, tiles_q;
  int raster_group;
  int sf_katoms;   // scale atoms along K = ceil(K / 128)
  int sf_q_rowatoms;  // 128-row scale bands of the Q-side operand = ceil(rows_q / 128)
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
  // split-K workspace: fp32 partials [units][128][BN] and per-tile tickets
  float *ws_partial;
  int *ws_ticket;
  int *err;
};

template <int BN, int STAGES, int ACC>
struct GemmSmem {
  static constexpr int kSfqAtoms = BN > 128 ? BN / 128 : 1;
  static constexpr int kSfqCols = 4 * kSfqAtoms;
  static constexpr int kSfCols = 4 + kSfqCols;  // TMEM columns of scales per stage
  static constexpr int kBytesP = kBlockP * kBlockK;
  static constexpr int kBytesQ = BN * kBlockK;
  static constexpr int kOffQ = STAGES * kBytesP;
  static constexpr int kOffSfp = kOffQ + STAGES * kBytesQ;
  static constexpr int kOffSfq = kOffSfp + STAGES * kSfAtom;
  static constexpr int kOffBar = kOffSfq + STAGES * kSfqAtoms * kSfAtom;
  static constexpr int kNumBars = 2 * STAGES + 2 * ACC + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static constexpr int kTmemUsed = ACC * BN + STAGES * kSfCols;
  static constexpr int kTmemCols = kTmemUsed <= 32    ? 32
                                   : kTmemUsed <= 64  ? 64
                                   : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256
                                                      : 512;
  static_assert(kTmemUsed <= 512, "TMEM budget");
  static_assert(kBytes <= 232448, "shared memory budget");
};

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

__device__ __forceinline__ void decode_unit(const GemmArgs &a, int unit, int &b, int &tp, int &tq,
                                            int &split, int &tile) {
  split = unit % a.splits;
  tile = unit / a.splits;
  const int per_batch = a.tiles_p * a.tiles_q;
  b = tile / per_batch;
  const int idx = tile - b * per_batch;
  const int group = a.raster_group * a.tiles_q;
  const int g = idx / group;
  const int first_p = g * a.raster_group;
  const int gp = min(a.raster_group, a.tiles_p - first_p);
  const int r = idx - g * group;
  tp = first_p + r % gp;
  tq = r / gp;
}

__device__ __forceinline__ float gelu_erf(float t) {
  return 0.5f * t * (1.0f + erff(t * 0.70710678118654752f));
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
// columns q0 .. q0+31 of the Q side, batch b.
template <bool SWAP>
__device__ __forceinline__ void emit32(const GemmArgs &a, int b, int prow, int q0,
                                       const float (&f)[32]) {
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
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = epi_value(a, f[8 * g + 2 * j], bias8[2 * j], res8[2 * j]);
        const float hi = epi_value(a, f[8 * g + 2 * j + 1], bias8[2 * j + 1], res8[2 * j + 1]);
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(lo, hi);
        o[j] = *reinterpret_cast<const uint32_t *>(&p2);
      }
      *reinterpret_cast<uint4 *>(yrow + n) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    const int n = prow;
    if (n >= a.N) return;
    const float bias = a.bias ? __bfloat162float(a.bias[n]) : 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int m = q0 + j;
      if (m >= a.M) break;
      const float res =
          a.res ? __bfloat162float(a.res[b * a.res_bstride + static_cast<int64_t>(m) * a.ldres + n])
                : 0.0f;
      a.y[b * a.y_bstride + static_cast<int64_t>(m) * a.ldy + n] =
          __float2bfloat16_rn(epi_value(a, f[j], bias, res));
    }
  }
}

template <int BN, int STAGES, int ACC, bool SWAP, bool P_FP4, bool Q_FP4>
__global__ void __launch_bounds__(kNumThreads, 1)
    gemm_bs_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q,
                   const GemmArgs a) {
  using L = GemmSmem<BN, STAGES, ACC>;
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
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
  int *last_flag = reinterpret_cast<int *>(smem + L::kOffMisc + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < ACC; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_p);
    tma_prefetch_desc(&tm_q);
  }
  if (warp == 1) tmem_alloc(tmem_slot, L::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total_units = a.batch * a.tiles_p * a.tiles_q * a.splits;
  // Transaction bytes of one stage.  A 4-bit operand lands in shared memory
  // with one byte-slot per code, but the transaction count is the packed size
  // (half the footprint).
  constexpr uint32_t kTxBytes = (P_FP4 ? L::kBytesP / 2 : L::kBytesP) +
                                (Q_FP4 ? L::kBytesQ / 2 : L::kBytesQ) + kSfAtom +
                                L::kSfqAtoms * kSfAtom;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < total_units && ok; unit += gridDim.x) {
        int b, tp, tq, split, tile;
        decode_unit(a, unit, b, tp, tq, split, tile);
        const int kt0 = split * a.kt_per_split;
        const int kt1 = min(a.kt_total, kt0 + a.kt_per_split);
        const int q_row0 = tq * BN;
        const uint8_t *sfp = a.sf_p + b * a.sf_p_bstride +
                             static_cast<int64_t>(tp) * a.sf_katoms * kSfAtom;
        const uint8_t *sfq = a.sf_q + b * a.sf_q_bstride +
                             static_cast<int64_t>(q_row0 / 128) * a.sf_katoms * kSfAtom;
        for (int kt = kt0; kt < kt1; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, a.err, abort_flag, kWaitProdEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kTxBytes);
          const int kx = kt * kBlockK;
          if (a.p_batched)
            tma_load_3d(s_p + stage * L::kBytesP, &tm_p, &full[stage], kx, tp * kBlockP, b);
          else
            tma_load_2d(s_p + stage * L::kBytesP, &tm_p, &full[stage], kx, tp * kBlockP);
          if (a.q_batched)
            tma_load_3d(s_q + stage * L::kBytesQ, &tm_q, &full[stage], kx, q_row0, b);
          else
            tma_load_2d(s_q + stage * L::kBytesQ, &tm_q, &full[stage], kx, q_row0);
          bulk_load(s_sfp + stage * kSfAtom, sfp + kt * kSfAtom, kSfAtom, &full[stage]);
#pragma unroll
          for (int j = 0; j < L::kSfqAtoms; ++j) {
            // A band past the operand's last row would be outside the scale
            // buffer; those rows are zero-filled by TMA, so any finite scale
            // band serves -- reuse the last one.
            const int band = min(q_row0 / 128 + j, a.sf_q_rowatoms - 1) - q_row0 / 128;
            bulk_load(s_sfq + (stage * L::kSfqAtoms + j) * kSfAtom,
                      sfq + (static_cast<int64_t>(band) * a.sf_katoms + kt) * kSfAtom, kSfAtom,
                      &full[stage]);
          }
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
        int b, tp, tq, split, tile;
        decode_unit(a, unit, b, tp, tq, split, tile);
        const int kt0 = split * a.kt_per_split;
        const int kt1 = min(a.kt_total, kt0 + a.kt_per_split);
        const uint32_t sfq_row_off = static_cast<uint32_t>((tq * BN) % 128) / 32;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, a.err, abort_flag, kWaitMmaTmemEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kt = kt0; kt < kt1; ++kt) {
          if (!mbar_wait(&full[stage], phase, a.err, abort_flag, kWaitMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf_t = tmem_base + ACC * BN + stage * L::kSfCols;
          tc_cp_sf(sf_t, desc_sf_32x128b(smem_u32(s_sfp + stage * kSfAtom)));
#pragma unroll
          for (int j = 0; j < L::kSfqAtoms; ++j)
            tc_cp_sf(sf_t + 4 + 4 * j,
                     desc_sf_32x128b(smem_u32(s_sfq + (stage * L::kSfqAtoms + j) * kSfAtom)));
          const uint32_t pa = smem_u32(s_p + stage * L::kBytesP);
          const uint32_t qa = smem_u32(s_q + stage * L::kBytesQ);
#pragma unroll
          for (int ks = 0; ks < kBlockK / kMmaK; ++ks) {
            const uint32_t idesc = make_idesc(P_FP4 ? kFmtE2M1 : kFmtE4M3,
                                              Q_FP4 ? kFmtE2M1 : kFmtE4M3, BN, ks);
            tc_mma_mxf8f6f4(d_tmem, desc_kmajor_sw128(pa + ks * kMmaK),
                            desc_kmajor_sw128(qa + ks * kMmaK), idesc, sf_t,
                            sf_t + 4 + sfq_row_off, (kt > kt0 || ks > 0) ? 1u : 0u);
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
    const int epi_tid = threadIdx.x - 64;  // 0..127
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int unit = blockIdx.x; unit < total_units; unit += gridDim.x) {
      int b, tp, tq, split, tile;
      decode_unit(a, unit, b, tp, tq, split, tile);
      __syncwarp();
      if (!mbar_wait(&tfull[acc], acc_phase, a.err, abort_flag, kWaitEpiFull)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * BN + (static_cast<uint32_t>(quad * 32) << 16);
      const int prow = tp * kBlockP + row;
      if (a.splits == 1) {
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the stores
          tmem_ld_32x32b_x32(t_row + c * 32, v);
          tmem_ld_wait();
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(v[j]);
          emit32<SWAP>(a, b, prow, tq * BN + c * 32, f);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      } else {
        // Split-K: publish this slice's partial tile, then the last slice to
        // arrive reduces all slices in slice order.
        float *mine = a.ws_partial + (static_cast<int64_t>(unit) * kBlockP + row) * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[32];
          __syncwarp();  // tcgen05.ld is warp-collective: reconverge after the stores
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
        __syncwarp();
        asm volatile("barrier.sync 1, 128;" ::: "memory");
        if (epi_tid == 0) {
          const int prev = atomicAdd(&a.ws_ticket[tile], 1);
          *last_flag = (prev == a.splits - 1);
        }
        __syncwarp();
        asm volatile("barrier.sync 1, 128;" ::: "memory");
        if (*last_flag) {
          __threadfence();
          const float *base =
              a.ws_partial + (static_cast<int64_t>(tile) * a.splits * kBlockP + row) * BN;
#pragma unroll 1
          for (int c = 0; c < BN / 32; ++c) {
            float f[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) f[j] = 0.0f;
            for (int s = 0; s < a.splits; ++s) {
              const float *src = base + static_cast<int64_t>(s) * kBlockP * BN + c * 32;
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + j));
                f[j] += v.x;
                f[j + 1] += v.y;
                f[j + 2] += v.z;
                f[j + 3] += v.w;
              }
            }
            emit32<SWAP>(a, b, prow, tq * BN + c * 32, f);
          }
          if (epi_tid == 0) a.ws_ticket[tile] = 0;  // ready for the next call
        }
        __syncwarp();
        asm volatile("barrier.sync 1, 128;" ::: "memory");
      }
      if (++acc == ACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace bq
