// Block-scaled GEMM on CTA pairs: one 256x256 output tile per pair of SMs
// (a thread-block cluster of 2), computed by tcgen05 MMAs of the cta_group::2
// form with M = 256.
//
// Same computation as gemm_bs_kernel (y = bf16(act(alpha * A B^T + bias) +
// residual) with fp32 accumulation in TMEM and per-32 E8M0 block scales): the
// operand formats, scale layout and epilogue are the ones the single-SM kernel
// uses.  What differs is how the tile is shared:
//   * each CTA of the pair loads its own 128 activation rows (operand A) and
//     its half of the tile's 256 weight rows (operand B), plus the scale atoms
//     of its A rows and of all 256 B rows;
//   * the leader (cluster rank 0) issues every MMA and scale copy once for
//     the pair; both CTAs' TMEM hold their own 128 accumulator rows;
//   * every copy of both CTAs completes on the leader's stage barrier, the
//     leader's commits arrive on both CTAs' barriers, and both epilogues
//     report back to the leader before it reuses the accumulator.
// Per 128-K block an SM then moves 32 KB into shared memory and its tensor
// core reads 32 KB (own A + own half of B, shared with the peer), where a
// single-SM 128x256 tile moves 48 KB and reads 48 KB for the same MMA work.
// Measured on the 8192^3 MXFP8 problem the copies are not what limits either
// kernel, and this one is the slower: it holds one accumulator per CTA whose
// four epilogue warps drain it chunk by chunk while the next tile's MMAs
// wait, and even with no copies at all its mainloop runs well below the MMA
// rate.  The built-in dispatch therefore runs it only on request.
#pragma once

#include "gemm_bs.cuh"

namespace bq {

constexpr int kPairN = 256;  // B rows (output columns) of a pair tile

// Shared-memory layout of one CTA of a pair: STAGES stages of KC chunks,
// each chunk with APC scale atoms per 128-row band (2 for packed E2M1
// operands, whose 128-byte chunk is 256 K).
template <int STAGES, int KC, int APC = 1>
struct PairSmem {
  static constexpr int kChunkA = kBlockP * kBlockK;        // own 128 rows
  static constexpr int kChunkB = (kPairN / 2) * kBlockK;   // own 128 of the 256 B rows
  static constexpr int kBytesA = KC * kChunkA;
  static constexpr int kBytesB = KC * kChunkB;
  static constexpr int kSfbAtoms = kPairN / 128;           // scale bands of all 256 B rows
  static constexpr int kSfaBytes = KC * APC * kSfAtom;
  static constexpr int kSfbBytes = KC * APC * kSfbAtoms * kSfAtom;
  static constexpr int kSfColsChunk = APC * (4 + 4 * kSfbAtoms);  // TMEM scale columns per chunk
  static constexpr int kSfCols = KC * kSfColsChunk;
  static constexpr int kOffB = STAGES * kBytesA;
  static constexpr int kOffYStage = kOffB + STAGES * kBytesB;  // 1024-aligned
  static constexpr int kOffSfa = kOffYStage + 2 * kYChunkBytes;
  static constexpr int kOffSfb = kOffSfa + STAGES * kSfaBytes;
  static constexpr int kOffBar = kOffSfb + STAGES * kSfbBytes;
  // full, empty, tfull, tempty, drain, two residual staging barriers
  static constexpr int kNumBars = 2 * STAGES + 5;
  static constexpr int kRbarIndex = 2 * STAGES + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64 + 1024;      // + alignment slack
  static constexpr int kTmemUsed = kPairN + STAGES * kSfCols;
  static constexpr int kTmemCols = kTmemUsed <= 256 ? 256 : 512;
  static_assert(kTmemUsed <= 512, "TMEM budget");
  static_assert(kBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ uint32_t make_idesc_m(uint32_t fmt_a, uint32_t fmt_b, int m, int n,
                                                 int sf_id) {
  uint32_t d = 0;
  d |= static_cast<uint32_t>(sf_id & 3) << 4;  // scale-factor id of B
  d |= fmt_a << 7;
  d |= fmt_b << 10;
  d |= static_cast<uint32_t>(n >> 3) << 17;    // N / 8
  d |= 1u << 23;                               // scale format: UE8M0
  d |= static_cast<uint32_t>(m >> 4) << 24;    // M / 16
  d |= static_cast<uint32_t>(sf_id & 3) << 29; // scale-factor id of A
  return d;
}

// Loads one part of a stage into this CTA's shared memory, completing on the
// leader's stage barrier `bar`: the A tile (own 128 activation rows), the B
// tile (own 128 weight rows), the A scale atoms (own band) or the B scale
// atoms (both bands).  Operand maps view K as (128 bytes, chunks) when KC > 1;
// scale maps view a scale buffer as (128 words, K atoms, 128-row bands), a
// box KC * APC atoms long.
template <class L, int KC, int APC = 1>
__device__ __forceinline__ void pair_issue(const GemmArgs &a, const CUtensorMap *tm_a,
                                           const CUtensorMap *tm_b, const CUtensorMap *tm_sfa,
                                           const CUtensorMap *tm_sfb, uint8_t *smem, int st,
                                           uint32_t bar, int kt, const UnitPos &u, uint32_t rank,
                                           bool weights, bool scales) {
  const int band_a = 2 * u.tp + static_cast<int>(rank);  // 128-row band of this CTA's A rows
  if (!weights) {
    if (scales) {
      uint8_t *dst = smem + L::kOffSfa + st * L::kSfaBytes;
      if (a.p_batched)
        tma2_load_4d(dst, tm_sfa, bar, 0, kt * APC, band_a, u.b);
      else
        tma2_load_3d(dst, tm_sfa, bar, 0, kt * APC, band_a);
      return;
    }
    uint8_t *dst = smem + st * L::kBytesA;
    const int row = band_a * kBlockP;
    if constexpr (KC == 1) {
      if (a.p_batched)
        tma2_load_3d(dst, tm_a, bar, kt * kBlockK, row, u.b);
      else
        tma2_load_2d(dst, tm_a, bar, kt * kBlockK, row);
    } else {
      if (a.p_batched)
        tma2_load_4d(dst, tm_a, bar, 0, row, kt, u.b);
      else
        tma2_load_3d(dst, tm_a, bar, 0, row, kt);
    }
    return;
  }
  if (scales) {
    uint8_t *dst = smem + L::kOffSfb + st * L::kSfbBytes;
    if (a.q_batched)
      tma2_load_4d(dst, tm_sfb, bar, 0, kt * APC, 2 * u.tq, u.b);
    else
      tma2_load_3d(dst, tm_sfb, bar, 0, kt * APC, 2 * u.tq);
    return;
  }
  uint8_t *dst = smem + L::kOffB + st * L::kBytesB;
  const int row = u.tq * kPairN + static_cast<int>(rank) * (kPairN / 2);
  if constexpr (KC == 1) {
    if (a.q_batched)
      tma2_load_3d(dst, tm_b, bar, kt * kBlockK, row, u.b);
    else
      tma2_load_2d(dst, tm_b, bar, kt * kBlockK, row);
  } else {
    if (a.q_batched)
      tma2_load_4d(dst, tm_b, bar, 0, row, kt, u.b);
    else
      tma2_load_3d(dst, tm_b, bar, 0, row, kt);
  }
}

template <int STAGES, int KC, bool Q_FP4, bool A4 = false>
__global__ void __launch_bounds__(kNumThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_sfa,
                     const __grid_constant__ CUtensorMap tm_sfb,
                     const __grid_constant__ CUtensorMap tm_y,
                     const __grid_constant__ CUtensorMap tm_res, const GemmArgs a) {
  // A4: both operands packed E2M1 (kind::mxf4, K = 64 per MMA, two scale
  // atoms per 128-byte chunk), as in gemm_bs_kernel.
  static_assert(!A4 || !Q_FP4, "A4 operands are plain packed bytes");
  constexpr int APC = A4 ? 2 : 1;
  using L = PairSmem<STAGES, KC, APC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 1;
  uint64_t *drain = tempty + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0: leader, 1: peer
  const int pair = blockIdx.x / 2;
  const int num_pairs = gridDim.x / 2;
  const int total_units = a.batch * a.tiles_p * a.tiles_q;
  // Bytes one CTA's part of a stage moves (the leader expects both CTAs').
  auto part_bytes = [](bool weights, bool scales) -> uint32_t {
    if (scales) return weights ? L::kSfbBytes : L::kSfaBytes;
    return weights ? (Q_FP4 ? L::kBytesB / 2 : L::kBytesB) : L::kBytesA;
  };

  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(&full[st], kCopyThreads);  // the leader's copy threads (bytes of both CTAs)
      mbar_init(&empty[st], 1);            // the leader's commit
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 8);  // every epilogue warp of both CTAs
    mbar_init(drain, 1);
    mbar_init(full + L::kRbarIndex, 1);
    mbar_init(full + L::kRbarIndex + 1, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_sfa);
    tma_prefetch_desc(&tm_sfb);
  }
  if (warp == 1) tmem_alloc2(tmem_slot, L::kTmemCols);
  tc_fence_before();
  __syncthreads();
  // Copies of both CTAs complete on the leader's barriers and the leader's
  // commits arrive on the peer's: every barrier of the pair is initialised
  // (and the TMEM allocated) before anything crosses.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tempty_lead = mapa_shared(smem_u32(tempty), 0);

  if (warp == 0 || warp >= kActWarp) {
    // ---------------------------------------------------------- copy threads --
    if (lane == 0) {
      const bool weights = warp == 0 || warp == kWsfWarp;
      const bool scales = warp == kWsfWarp || warp == kAsfWarp;
      if (!weights) {
        griddep_wait();
        if (!scales) griddep_launch_dependents();
      }
      const uint32_t tx = 2 * part_bytes(weights, scales);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int unit = pair; unit < total_units && ok; unit += num_pairs) {
        const UnitPos u = unit_pos(a, unit);
        for (int kt = 0; kt < a.kt_total; kt += KC) {
          // the leader's commit frees this CTA's stage (a cross-CTA arrival)
          if (!mbar_wait_cluster(&empty[stage], phase ^ 1, a.err, abort_flag, kWaitProdEmpty)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], tx);
          pair_issue<L, KC, APC>(a, &tm_a, &tm_b, &tm_sfa, &tm_sfb, smem, stage,
                            mapa_shared(smem_u32(&full[stage]), 0), kt, u, rank, weights, scales);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) sleep_ns(200000);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issue (leader only) --
    if (rank == 0 && lane == 0) {
      const uint32_t a0 = smem_u32(smem);
      const uint32_t b0 = smem_u32(smem + L::kOffB);
      const uint32_t sfa0 = smem_u32(smem + L::kOffSfa);
      const uint32_t sfb0 = smem_u32(smem + L::kOffSfb);
      const uint32_t fmt_a = a.fmt_p, fmt_b = a.fmt_q;
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int unit = pair; unit < total_units && ok; unit += num_pairs) {
        if (!mbar_wait_cluster(tempty, acc_phase ^ 1, a.err, abort_flag, kWaitMmaTmemEmpty)) break;
        tc_fence_after();
        for (int kt = 0; kt < a.kt_total; kt += KC) {
          if (!mbar_wait_cluster(&full[stage], phase, a.err, abort_flag, kWaitMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nv = min(KC, a.kt_total - kt);
          const uint32_t sf_stage = tmem_base + kPairN + stage * L::kSfCols;
#pragma unroll 1
          for (int c = 0; c < nv; ++c) {
            // scale columns of a chunk: A's APC atoms, then per atom B's two bands
            const uint32_t sf_t = sf_stage + c * L::kSfColsChunk;
            const uint32_t sfb_t = sf_t + 4 * APC;
            const int na = min(APC, a.sf_katoms - (kt + c) * APC);
            for (int t = 0; t < na; ++t) {
              tc_cp_sf2(sf_t + 4 * t,
                        desc_sf_32x128b(sfa0 + stage * L::kSfaBytes + (c * APC + t) * kSfAtom));
#pragma unroll
              for (int j = 0; j < L::kSfbAtoms; ++j)
                tc_cp_sf2(sfb_t + 4 * (t * L::kSfbAtoms + j),
                          desc_sf_32x128b(sfb0 + stage * L::kSfbBytes +
                                          (j * KC * APC + c * APC + t) * kSfAtom));
            }
            const uint32_t pa = a0 + stage * L::kBytesA + c * L::kChunkA;
            const uint32_t pb = b0 + stage * L::kBytesB + c * L::kChunkB;
#pragma unroll
            for (int ks = 0; ks < kBlockK / kMmaK; ++ks) {
              const uint32_t acc_in = (kt > 0 || c > 0 || ks > 0) ? 1u : 0u;
              if constexpr (A4) {
                const int t = ks >> 1;  // atom of this K = 64 step
                if (t < na)
                  tc_mma2_mxf4(tmem_base, desc_kmajor_sw128(pa + ks * kMmaK),
                               desc_kmajor_sw128(pb + ks * kMmaK),
                               make_idesc_m(kFmtMxf4E2M1, kFmtMxf4E2M1, 2 * kBlockP, kPairN,
                                            (ks & 1) * 2),
                               sf_t + 4 * t, sfb_t + 4 * t * L::kSfbAtoms, acc_in);
              } else {
                tc_mma2_mxf8f6f4(tmem_base, desc_kmajor_sw128(pa + ks * kMmaK),
                                 desc_kmajor_sw128(pb + ks * kMmaK),
                                 make_idesc_m(fmt_a, fmt_b, 2 * kBlockP, kPairN, ks), sf_t,
                                 sfb_t, acc_in);
              }
            }
          }
          tc_commit2(mapa_shared(smem_u32(&empty[stage]), 0));
          tc_commit2(mapa_shared(smem_u32(&empty[stage]), 1));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit2(mapa_shared(smem_u32(tfull), 0));
        tc_commit2(mapa_shared(smem_u32(tfull), 1));
        acc_phase ^= 1;
      }
      tc_commit2(mapa_shared(smem_u32(drain), 0));
      if (!mbar_wait_timed(drain, 0, a.err, kWaitDrain)) sleep_ns(200000);
    }
  } else {
    // ---------------------------------------------------- epilogue (both CTAs) --
    const int quad = warp % 4;
    const int row = quad * 32 + lane;
    const int epi_tid = threadIdx.x - 64;
    uint32_t acc_phase = 0;
    uint32_t rphase = 0;  // residual staging barrier parities
    griddep_wait();  // the bias and residual may come from the preceding kernel
    for (int unit = pair; unit < total_units; unit += num_pairs) {
      const UnitPos u = unit_pos(a, unit);
      __syncwarp();
      if (!mbar_wait_cluster(tfull, acc_phase, a.err, abort_flag, kWaitEpiFull)) break;
      acc_phase ^= 1;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      epilogue_rows_tma<kPairN>(a, &tm_y, &tm_res, full + L::kRbarIndex, rphase, t_row, u.b,
                                (2 * u.tp + static_cast<int>(rank)) * kBlockP, u.tq * kPairN,
                                row, epi_tid, smem + L::kOffYStage, abort_flag);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_lead);
    }
  }

  // Teardown: the leader has drained its MMAs; nothing may still be arriving
  // on either CTA's barriers or reading its TMEM when the pair frees it, and
  // the epilogue's last TMA stores are done.
  if (threadIdx.x == 64) bulk_wait_group_all();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem_base, L::kTmemCols);
  }
}

}  // namespace bq
