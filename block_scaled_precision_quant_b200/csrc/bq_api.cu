// bq_api.cu -- host side of libbq: argument checks, tensor maps, schedule
// choice and kernel launches behind the C ABI declared in include/bq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cmath>
#include <cstring>
#include <mutex>

#include "act_quant.cuh"
#include "bq.h"
#include "gemm_bs.cuh"
#include "gemm_pair.cuh"

namespace {

// ------------------------------------------------------------ device state --

// Error word the GEMM kernels write when a barrier wait gives up, and the
// flag word of the prepack scans.  One copy per device (module globals).
__device__ int g_dev_error;
__device__ int g_pack_flags;

constexpr int kMaxDevices = 64;

struct DevInfo {
  bool ready = false;
  bool arch_ok = false;
  int num_sms = 0;
  int* err_ptr = nullptr;
  int* flags_ptr = nullptr;
};

std::mutex g_mu;
DevInfo g_dev[kMaxDevices];

// Compute capability the arch check compares instead of the probed one
// (major * 10 + minor; -1 = the probe's): set by bq_debug_override_compute_capability.
std::atomic<int> g_cc_override{-1};

// Returns BQ_OK and fills `info` for the current device, BQ_ERR_ARCH if it is
// not compute capability 10.0.
int current_device(DevInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BQ_ERR_CUDA;
    d.arch_ok = (major == 10 && minor == 0);
    if (d.arch_ok) {
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err_ptr), g_dev_error) != cudaSuccess ||
          cudaGetSymbolAddress(reinterpret_cast<void**>(&d.flags_ptr), g_pack_flags) !=
              cudaSuccess)
        return BQ_ERR_CUDA;
    }
    d.ready = true;
  }
  *info = &d;
  const int ov = g_cc_override.load();
  return (d.arch_ok && (ov < 0 || ov == 100)) ? BQ_OK : BQ_ERR_ARCH;
}

// Watchdog self-test: one thread waits, with the bounded wait every kernel of
// the library uses, on a shared-memory barrier that nothing ever arrives on,
// so the wait runs out after limit_ns, records the timeout (site
// kWaitSelftest) in the error word and returns.
__global__ void wait_selftest_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    bq::mbar_init(&bar, 1);
    abort_flag = 0;
    bq::fence_mbar_init();
    bq::mbar_wait(&bar, 0, err, &abort_flag, bq::kWaitSelftest, limit_ns);
  }
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline int launch_status() {
  return cudaGetLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

// ------------------------------------------------------------- tensor maps --

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encoder() {
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? BQ_OK : BQ_ERR_CUDA;
}

// K-major operand: `rows` rows of K codes (row stride `row_bytes`), optional
// batch dimension (count, stride in bytes), box of 128 codes x box_rows rows,
// 128B swizzle, zero fill outside the tensor.  fp4 selects the 4-bit type that
// TMA expands to one byte-slot per code in shared memory (8 data bytes then 8
// padding bytes per 16 codes), the operand layout kind::mxf8f6f4 reads.
// With kc > 1 (K % 128 == 0) K is viewed as (128 codes, K/128 chunks) so one
// box of {128, box_rows, kc} brings kc consecutive 128-K chunks, each landing
// as its own 128B-swizzled [box_rows][128 B] tile.
int make_operand_map(CUtensorMap* m, const void* base, bool fp4, int64_t K, int64_t rows,
                     int64_t row_bytes, int64_t batch, int64_t batch_bytes, int box_rows,
                     int kc) {
  cuuint64_t dims[4];
  cuuint64_t strides[3];
  cuuint32_t box[4];
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  cuuint32_t rank;
  if (kc <= 1) {
    dims[0] = static_cast<cuuint64_t>(K);
    dims[1] = static_cast<cuuint64_t>(rows);
    dims[2] = static_cast<cuuint64_t>(batch);
    strides[0] = static_cast<cuuint64_t>(row_bytes);
    strides[1] = static_cast<cuuint64_t>(batch_bytes);
    box[0] = 128u;
    box[1] = static_cast<cuuint32_t>(box_rows);
    box[2] = 1u;
    rank = batch > 1 ? 3 : 2;
  } else {
    dims[0] = 128;
    dims[1] = static_cast<cuuint64_t>(rows);
    dims[2] = static_cast<cuuint64_t>(K / 128);
    dims[3] = static_cast<cuuint64_t>(batch);
    strides[0] = static_cast<cuuint64_t>(row_bytes);
    strides[1] = fp4 ? 64u : 128u;  // bytes per 128-code chunk
    strides[2] = static_cast<cuuint64_t>(batch_bytes);
    box[0] = 128u;
    box[1] = static_cast<cuuint32_t>(box_rows);
    box[2] = static_cast<cuuint32_t>(kc);
    box[3] = 1u;
    rank = batch > 1 ? 4 : 3;
  }
  CUresult r = g_encode(m,
                        fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                        rank, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BQ_OK : BQ_ERR_ALIGN;
}

// A scale buffer (MMA layout: 128-row bands of K-block atoms, 512 bytes each)
// viewed as (128 words, K blocks, bands[, batch]); a box is `kc` consecutive
// atoms of `bands_box` bands.
int make_scale_map(CUtensorMap* m, const void* base, int64_t rows, int64_t K, int64_t batch,
                   int64_t batch_bytes, int kc, int bands_box) {
  const int64_t katoms = (K + 127) / 128;
  const int64_t bands = (rows + 127) / 128;
  cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(katoms), static_cast<cuuint64_t>(bands),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {512, static_cast<cuuint64_t>(katoms * 512),
                           static_cast<cuuint64_t>(batch_bytes)};
  cuuint32_t box[4] = {128u, static_cast<cuuint32_t>(kc), static_cast<cuuint32_t>(bands_box), 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, batch > 1 ? 4 : 3,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BQ_OK : BQ_ERR_ALIGN;
}

// A bf16 [batch][M][ld] matrix of N used columns (the output y, or the
// residual) as (N, M[, batch]); box 32 x 128 with the 64-byte swizzle of the
// epilogue's staging tile.
int make_y_map(CUtensorMap* m, const void* y, int64_t M, int64_t N, int64_t ld, int64_t batch,
               int64_t batch_bytes) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * 2), static_cast<cuuint64_t>(batch_bytes)};
  cuuint32_t box[3] = {32u, 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, batch > 1 ? 3 : 2,
                        const_cast<void*>(y), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BQ_OK : BQ_ERR_ALIGN;
}

// ---------------------------------------------------------------- schedule --

// kA4W4: MXFP4 weights with MXFP4 (packed E2M1) activations, kind::mxf4.
// kGrad: E5M2 gradient codes on the activation side, an E4M3 operand with
// per-32 scales (MXFP8) on the weight side (the backward GEMMs).
// kNv4: NVFP4 x NVFP4 (E4M3 scales per 16), kind::mxf4nvf4.
enum WeightKind { kMxfp4 = 0, kFp8Blk32 = 1, kMxfp8 = 2, kA4W4 = 3, kGrad = 4, kNv4 = 5 };

struct Plan {
  bool swap = false;
  bool pair = false;     // 256x256 tiles on CTA pairs (cta_group::2 MMA)
  int kc = 1;            // 128-K chunks per pipeline stage
  bool cluster = false;  // K slices reduced through DSMEM inside a thread-block cluster
  int bn = 256;
  int splits = 1;
  int kt_total = 0;
  int kt_per_split = 0;
  int tiles_p = 0, tiles_q = 0;
  int64_t units = 0;
  size_t ws_partial = 0, ws_ticket = 0;
};

int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

constexpr int64_t kMaxSplitTiles = 16384;                       // output tiles of a split-K call
constexpr size_t kTicketRegion = kMaxSplitTiles * sizeof(int);  // 64 KiB
constexpr int kMaxClusterSplit = 8;                             // portable cluster size

int make_plan(int64_t M, int64_t N, int64_t K, int64_t batch, const bq_gemm_config* cfg,
              int num_sms, Plan* p) {
  const int req_bn = cfg ? cfg->block_n : 0;
  const int req_split = cfg ? cfg->split_k : 0;
  const int req_swap = cfg ? cfg->swap_ab : -1;
  const int req_mode = cfg ? cfg->split_mode : BQ_SPLIT_AUTO;
  if (req_bn != 0 && req_bn != 32 && req_bn != 64 && req_bn != 128 && req_bn != 256)
    return BQ_ERR_INVALID;
  if (req_split < 0 || req_split > 16 || req_swap < -1 || req_swap > 1) return BQ_ERR_INVALID;
  if (req_mode < BQ_SPLIT_AUTO || req_mode > BQ_SPLIT_CLUSTER) return BQ_ERR_INVALID;
  const int req_kc = cfg ? cfg->k_chunks : 0;
  if (req_kc < 0 || req_kc > 4 || req_kc == 3) return BQ_ERR_INVALID;
  const int req_pair = cfg ? cfg->cta_pair : 0;
  if (req_pair < 0 || req_pair > 2) return BQ_ERR_INVALID;
  p->kt_total = ceil_div(K, 128);
  p->swap = req_swap == 1 || (req_swap == -1 && M <= 64);
  if (p->swap) {
    if (M > 64) return BQ_ERR_INVALID;
    p->bn = req_bn ? req_bn : (M <= 32 ? 32 : 64);
    if (p->bn != 32 && p->bn != 64) return BQ_ERR_INVALID;
    p->tiles_p = ceil_div(N, 128);
    p->tiles_q = ceil_div(M, p->bn);
  } else {
    p->tiles_p = ceil_div(M, 128);
    if (req_bn) {
      p->bn = req_bn;
    } else {
      // Wave model fitted to the schedule sweeps (in units of one 128x256
      // K-block step): a 128x128 tile takes 0.61 of that per K block, and a
      // 128x256 tile, whose single TMEM accumulator leaves its epilogue
      // unoverlapped, pays ~7 units of epilogue per tile; 128x128 tiles keep
      // two accumulators and expose only the last epilogue.  Pick the width
      // whose tiles per SM finish first.  Tiles per SM are counted
      // fractionally: a partial last wave runs on fewer SMs, which under the
      // power cap clock higher, and the sweeps fit that better than whole
      // waves.
      const double t256 = static_cast<double>(batch * p->tiles_p * ceil_div(N, 256));
      const double t128 = static_cast<double>(batch * p->tiles_p * ceil_div(N, 128));
      const double kt = static_cast<double>(ceil_div(K, 128));
      const double c256 = t256 / num_sms * (kt + 7.0);
      const double c128 = t128 / num_sms * kt * 0.61 + 3.5;
      p->bn = (N > 128 && c256 <= c128) ? 256 : 128;
    }
    if (p->bn != 128 && p->bn != 256) return BQ_ERR_INVALID;
    p->tiles_q = ceil_div(N, p->bn);
  }
  const int64_t tiles = batch * p->tiles_p * p->tiles_q;
  int splits = req_split;
  const bool use_ws = req_mode == BQ_SPLIT_WORKSPACE;
  if (splits == 0) {
    splits = 1;
    // Decode tiles (sweeps): a cluster split pays ~2 us of exchange (the
    // slices' fp32 rows through DSMEM, ~1 us for the last of them to land,
    // the owners' reduce), so it wins only where it cuts a long per-tile
    // mainloop.  With a long K loop (>= 24 K blocks) a power-of-two cluster
    // split wins: spread it while the grid stays within one CTA per SM.
    // With 12..23 K blocks it wins only when the slices fill nearly every
    // SM (41x4608x1536: 36 tiles x 4 slices on 148 SMs, 6.8 against 7.0 us
    // unsplit; 48 tiles x 2 slices lose, 7.7 against 7.1 us).
    if (p->swap && req_mode != BQ_SPLIT_WORKSPACE && p->kt_total >= 24) {
      while (splits * 2 <= kMaxClusterSplit && tiles * splits * 2 <= num_sms &&
             p->kt_total / (splits * 2) >= 4)
        splits *= 2;
    } else if (p->swap && req_mode != BQ_SPLIT_WORKSPACE && p->kt_total >= 12) {
      int s = 1;
      while (s * 2 <= kMaxClusterSplit && tiles * s * 2 <= num_sms && p->kt_total / (s * 2) >= 3)
        s *= 2;
      if (s > 1 && tiles * s * 10 >= num_sms * 9) splits = s;
    }
  }
  if (splits > p->kt_total) splits = p->kt_total;
  const bool pow2 = (splits & (splits - 1)) == 0;
  p->cluster = p->swap && splits > 1 && pow2 && splits <= kMaxClusterSplit && !use_ws;
  if (req_mode == BQ_SPLIT_CLUSTER && splits > 1 && !p->cluster) return BQ_ERR_INVALID;
  // 256x256 pair tiles run on request only: since the single-SM 128x256 tile
  // has two epilogue groups its epilogue no longer stalls the next tile, and
  // it matches or beats the pair tile in every sweep (8192^3 MXFP8: 494 us
  // against 536 us in one run; 4096x1536x6144: 50.7 against 55.6 us).
  const bool auto_pair = false;
  if (req_pair == 2 || auto_pair) {  // 256x256 tiles on CTA pairs: wide tiles, no split
    if (p->swap || splits != 1 || (req_bn != 0 && req_bn != 256)) return BQ_ERR_INVALID;
    if (req_kc > 2 || (req_kc == 2 && K % 128 != 0)) return BQ_ERR_INVALID;
    p->pair = true;
    p->bn = 256;
    p->tiles_p = ceil_div(M, 256);
    p->tiles_q = ceil_div(N, 256);
    p->splits = 1;
    p->kt_per_split = p->kt_total;
    p->units = batch * p->tiles_p * p->tiles_q;
    if (p->units > 0x7FFFFFFF) return BQ_ERR_SHAPE;
    p->kc = req_kc ? req_kc : (K % 128 == 0 ? 2 : 1);
    return BQ_OK;
  }
  // K blocks are dealt out evenly: slice s covers [s*KT/S, (s+1)*KT/S), never empty.
  p->splits = splits;
  p->kt_per_split = ceil_div(p->kt_total, splits);
  p->units = tiles * p->splits;
  if (p->units > 0x7FFFFFFF) return BQ_ERR_SHAPE;
  // Chunks per stage: several 128-K chunks behind one barrier need whole
  // chunks (K % 128 == 0); the swap-AB tiles take 4, the wide tiles 2.
  const int kc_max = p->swap ? 4 : 2;
  if (req_kc > 1 && (K % 128 != 0 || req_kc > kc_max)) return BQ_ERR_INVALID;
  if (req_kc > 1 && p->splits > 1 && !p->cluster) return BQ_ERR_INVALID;
  // Sweeps: 4 chunks for unsplit swap tiles, 1 for cluster slices (two CTAs
  // per SM), 2 for 128-wide tiles, 1 for 256-wide tiles.
  int kc_auto = 1;
  if (K % 128 == 0) {
    if (p->swap)
      kc_auto = p->splits == 1 ? 4 : 1;
    else
      kc_auto = (p->bn == 128 && p->splits == 1) ? 2 : 1;
  }
  p->kc = req_kc ? req_kc : kc_auto;
  if (p->splits > 1 && !p->cluster) {
    if (tiles > kMaxSplitTiles) return BQ_ERR_SHAPE;
    p->ws_partial = static_cast<size_t>(p->units) * 128 * p->bn * sizeof(float);
    p->ws_ticket = static_cast<size_t>(tiles) * sizeof(int);
  }
  return BQ_OK;
}

// Split-K workspace: a fixed region of per-tile tickets at the start (the
// same bytes for every problem, so a call never finds another call's partial
// sums where it expects zeroed tickets), then the fp32 partial tiles.
size_t plan_ws_bytes(const Plan& p) {
  if (p.splits <= 1 || p.cluster) return 0;
  return kTicketRegion + p.ws_partial;
}

// The plan a call runs; one that needs more workspace than given is refused.
// The plan of a call of weight kind wk.  Packed E2M1 operands on both sides
// (A4W4) have K/2 bytes per row, so their schedule counts chunks of 256 K;
// they move half the shared-memory bytes per MMA, so pair tiles do not pay
// (sweep, 8192^3: 367 us against 347 us for 128x256 tiles) and are used only
// on request, and wide tiles take 2 chunks per stage (347 vs 354 us).
int plan_kind(WeightKind wk, int64_t M, int64_t N, int64_t K, int64_t batch,
              const bq_gemm_config* cfg, int num_sms, Plan* p) {
  if (wk == kNv4) {
    // NVFP4 stages carry four scale atoms per chunk: one chunk per stage,
    // unsplit, single-SM tiles
    bq_gemm_config c = cfg ? *cfg : bq_gemm_config{0, 0, -1, BQ_SPLIT_AUTO, 0, 0};
    if (c.cta_pair == 2 || c.split_k > 1 || c.k_chunks > 1) return BQ_ERR_INVALID;
    c.cta_pair = 1;
    c.split_k = 1;
    c.k_chunks = 1;
    return make_plan(M, N, K / 2, batch, &c, num_sms, p);
  }
  if (wk != kA4W4) return make_plan(M, N, K, batch, cfg, num_sms, p);
  const int64_t Kb = K / 2;
  bq_gemm_config c = cfg ? *cfg : bq_gemm_config{0, 0, -1, BQ_SPLIT_AUTO, 0, 0};
  if (c.cta_pair == 0) c.cta_pair = 1;
  int st = make_plan(M, N, Kb, batch, &c, num_sms, p);
  if (st == BQ_OK && c.k_chunks == 0 && !p->swap && !p->pair && p->splits == 1 && p->kc == 1 &&
      Kb % 128 == 0) {
    c.k_chunks = 2;
    st = make_plan(M, N, Kb, batch, &c, num_sms, p);
  }
  return st;
}

int plan_for_call(WeightKind wk, int64_t M, int64_t N, int64_t K, int64_t batch,
                  const bq_gemm_config* cfg, int num_sms, const void* ws, size_t ws_bytes,
                  Plan* p) {
  const int st = plan_kind(wk, M, N, K, batch, cfg, num_sms, p);
  if (st != BQ_OK) return st;
  const size_t need = plan_ws_bytes(*p);
  return (need == 0 || (ws && ws_bytes >= need)) ? BQ_OK : BQ_ERR_WORKSPACE;
}

// --------------------------------------------------------------- launches --

template <int BN, int STAGES, int ACC, bool SWAP, bool P_FP4, bool Q_FP4, int MODE, int KC,
          bool FUSEQ = false, int A4 = 0>
int launch_gemm(const CUtensorMap& tp, const CUtensorMap& tq, const CUtensorMap& ty,
                const CUtensorMap& tr, const bq::GemmArgs& args,
                int64_t units, int num_sms, cudaStream_t stream) {
  constexpr bool CSPLIT = MODE == bq::kSplitCluster;
  using L = bq::KernelSmem<BN, STAGES, ACC, SWAP, MODE, KC, A4 == 2 ? 4 : (A4 ? 2 : 1)>;
  // unsplit wide tiles run a second group of epilogue warps
  constexpr int kThreads = (!SWAP && MODE == bq::kSplitNone) ? bq::kWideThreads : bq::kNumThreads;
  auto kern = bq::gemm_bs_kernel<BN, STAGES, ACC, SWAP, P_FP4, Q_FP4, MODE, KC, FUSEQ, A4>;
  static bool attr_set[kMaxDevices] = {};
  static int per_sm_cache[kMaxDevices] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return BQ_ERR_CUDA;
    int per_sm = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, L::kBytes);
    if (per_sm < 1) per_sm = 1;
    // Co-resident CTAs share the SM's 512 TMEM columns.
    const int tmem_fit = 512 / L::kTmemCols;
    if (per_sm > tmem_fit) per_sm = tmem_fit;
    per_sm_cache[dev] = per_sm;
    attr_set[dev] = true;
  }
  const int per_sm = per_sm_cache[dev];
  const int S = CSPLIT ? args.splits : 1;
  int64_t grid = static_cast<int64_t>(num_sms) * per_sm / S * S;
  if (grid < S) grid = S;
  if (grid > units) grid = units;  // units is a multiple of S
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(grid));
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = L::kBytes;
  lc.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  // May start while the preceding kernel (the activation quantizer) finishes:
  // prologue and weight loads overlap it; griddepcontrol.wait guards the rest.
  // The kernel in turn releases its own dependents once every CTA is past that
  // wait, so the next programmatic launch overlaps this one's mainloop.
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (CSPLIT) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(S);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  lc.attrs = attr;
  lc.numAttrs = na;
  if (cudaLaunchKernelEx(&lc, kern, tp, tq, ty, tr, args) != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return launch_status();
}

template <int BN, int STAGES, int ACC, bool SWAP, int MODE, int KC, bool FUSEQ = false,
          int A4 = 0>
int launch_kind(bool w_fp4, const CUtensorMap& tp, const CUtensorMap& tq, const CUtensorMap& ty,
                const CUtensorMap& tr, const bq::GemmArgs& args, int64_t u, int num_sms,
                cudaStream_t st) {
  if constexpr (A4 != 0)  // packed E2M1 on both sides: plain byte operands
    return launch_gemm<BN, STAGES, ACC, SWAP, false, false, MODE, KC, false, A4>(
        tp, tq, ty, tr, args, u, num_sms, st);
  // FP4 weights sit on the P side with SWAP, on the Q side otherwise.
  if (w_fp4)
    return launch_gemm<BN, STAGES, ACC, SWAP, SWAP, !SWAP, MODE, KC, FUSEQ>(tp, tq, ty, tr, args, u,
                                                                           num_sms, st);
  return launch_gemm<BN, STAGES, ACC, SWAP, false, false, MODE, KC, FUSEQ>(tp, tq, ty, tr, args, u,
                                                                           num_sms, st);
}

template <int STAGES, int KC, bool Q_FP4, bool A4 = false>
int launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa,
                const CUtensorMap& tsb, const CUtensorMap& ty, const CUtensorMap& tr,
                const bq::GemmArgs& args,
                int64_t units, int num_sms, cudaStream_t stream) {
  using L = bq::PairSmem<STAGES, KC, A4 ? 2 : 1>;
  auto kern = bq::gemm_pair_kernel<STAGES, KC, Q_FP4, A4>;
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return BQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  // One CTA per SM (shared memory and TMEM), so at most num_sms / 2 pairs.
  int64_t pairs = num_sms / 2;
  if (pairs > units) pairs = units;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  lc.blockDim = dim3(bq::kNumThreads);
  lc.dynamicSmemBytes = L::kBytes;
  lc.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 2;
  if (cudaLaunchKernelEx(&lc, kern, ta, tb, tsa, tsb, ty, tr, args) != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return launch_status();
}

// Dispatch on (swap, bn, chunks per stage, split mode, weight format) to the
// compiled instances.  Stage counts fill ~200 KB of shared memory.
template <int A4>
int run_gemm(const Plan& pl, bool w_fp4, const CUtensorMap& tp, const CUtensorMap& tq,
             const CUtensorMap& ty, const CUtensorMap& tr, const bq::GemmArgs& a, int ns,
             cudaStream_t st) {
  const int64_t u = pl.units;
  constexpr int kNone = bq::kSplitNone, kWs = bq::kSplitWorkspace, kCl = bq::kSplitCluster;
  const bool b32 = pl.bn == 32;
  if (!pl.swap) {
    if (pl.bn == 256) {
      if (pl.splits > 1) return launch_kind<256, 4, 1, false, kWs, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
      return pl.kc == 2 ? launch_kind<256, 2, 1, false, kNone, 2, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st)
                        : launch_kind<256, 4, 1, false, kNone, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
    }
    if (pl.splits > 1) return launch_kind<128, 6, 2, false, kWs, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
    return pl.kc == 2 ? launch_kind<128, 3, 2, false, kNone, 2, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st)
                      : launch_kind<128, 6, 2, false, kNone, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
  }
  if constexpr (!A4) {
    if (a.x) {  // fused activation quantization: unsplit 4-chunk swap tiles
      return b32 ? launch_kind<32, 2, 1, true, kNone, 4, true>(w_fp4, tp, tq, ty, tr, a, u, ns, st)
                 : launch_kind<64, 2, 1, true, kNone, 4, true>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
    }
  }
  if (pl.cluster) {
    if (pl.kc == 4)
      return b32 ? launch_kind<32, 1, 1, true, kCl, 4, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st)
                 : launch_kind<64, 1, 1, true, kCl, 4, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
    return b32 ? launch_kind<32, 3, 1, true, kCl, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st)
               : launch_kind<64, 3, 1, true, kCl, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
  }
  if (pl.splits > 1)
    return b32 ? launch_kind<32, 4, 1, true, kWs, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st)
               : launch_kind<64, 4, 1, true, kWs, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
  if (pl.kc == 4)
    return b32 ? launch_kind<32, 2, 1, true, kNone, 4, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st)
               : launch_kind<64, 2, 1, true, kNone, 4, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
  return b32 ? launch_kind<32, 8, 1, true, kNone, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st)
             : launch_kind<64, 8, 1, true, kNone, 1, false, A4>(w_fp4, tp, tq, ty, tr, a, u, ns, st);
}

// NVFP4 x NVFP4: one chunk per stage (four scale atoms each), unsplit.
int run_gemm_nv(const Plan& pl, const CUtensorMap& tp, const CUtensorMap& tq,
                const CUtensorMap& ty, const CUtensorMap& tr, const bq::GemmArgs& a, int ns,
                cudaStream_t st) {
  const int64_t u = pl.units;
  constexpr int kNone = bq::kSplitNone;
  if (!pl.swap)
    return pl.bn == 256
               ? launch_kind<256, 3, 1, false, kNone, 1, false, 2>(false, tp, tq, ty, tr, a, u,
                                                                   ns, st)
               : launch_kind<128, 5, 2, false, kNone, 1, false, 2>(false, tp, tq, ty, tr, a, u,
                                                                   ns, st);
  return pl.bn == 32
             ? launch_kind<32, 6, 1, true, kNone, 1, false, 2>(false, tp, tq, ty, tr, a, u, ns, st)
             : launch_kind<64, 6, 1, true, kNone, 1, false, 2>(false, tp, tq, ty, tr, a, u, ns, st);
}

// Activations given as bf16 and quantized inside the GEMM (decode tiles).
struct FusedAct {
  const void* x;
  int64_t ldx;
  void* a_q_out;   // nullable
  void* a_sf_out;  // nullable (set together with a_q_out)
  int* status;     // nullable
};

int gemm_entry(WeightKind wk, const void* a_q, const void* a_sf, const void* b, const void* b_sf,
               int64_t M, int64_t N, int64_t K, void* y, const bq_epilogue* epi,
               const bq_batch* batch, void* ws, size_t ws_bytes, const bq_gemm_config* cfg,
               bq_stream_t stream, const FusedAct* fused = nullptr, bool clear_tickets = false) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  if (M < 0 || N < 0 || K <= 0 || K % 32 != 0) return BQ_ERR_SHAPE;
  const int64_t count = batch ? batch->count : 1;
  if (count < 0) return BQ_ERR_SHAPE;
  if (M == 0 || N == 0 || count == 0) return BQ_OK;
  void* q_out = epi ? epi->q_out : nullptr;
  void* sf_out = epi ? epi->sf_out : nullptr;
  if ((q_out || sf_out) && N % 32 != 0) return BQ_ERR_SHAPE;
  if ((q_out != nullptr) != (sf_out != nullptr)) return BQ_ERR_NULL;
  if ((!fused && (!a_q || !a_sf)) || !b || !b_sf || (!y && !q_out)) return BQ_ERR_NULL;
  if (fused) {
    // one activation tile of all M rows, whole 128-K chunks, one problem
    if (M > 64 || K % 128 != 0 || (batch && batch->count > 1)) return BQ_ERR_SHAPE;
    if (!fused->x) return BQ_ERR_NULL;
    if (fused->ldx < K || fused->ldx % 8 != 0 || !aligned(fused->x, 16)) return BQ_ERR_ALIGN;
    if ((fused->a_q_out != nullptr) != (fused->a_sf_out != nullptr)) return BQ_ERR_NULL;
    if (fused->a_q_out && (!aligned(fused->a_q_out, 16) || !aligned(fused->a_sf_out, 4)))
      return BQ_ERR_ALIGN;
  }
  if (q_out && (!aligned(q_out, 16) || !aligned(sf_out, 4))) return BQ_ERR_ALIGN;
  const bool w_fp4 = wk == kMxfp4;
  const bool a4 = wk == kA4W4 || wk == kNv4;  // packed E2M1 activations and weights
  if (a4 && fused) return BQ_ERR_INVALID;  // the fused quantizer emits E4M3 codes
  // Bytes of K per operand row: packed E2M1 rows hold two codes per byte.
  const int64_t Kb = a4 ? K / 2 : K;
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF || count > 65535) return BQ_ERR_SHAPE;
  if (N % 8 != 0) return BQ_ERR_SHAPE;
  if ((w_fp4 || a4) && K % 128 != 0) return BQ_ERR_SHAPE;
  if ((!fused && (!aligned(a_q, 16) || !aligned(a_sf, 16))) || !aligned(b_sf, 16) ||
      (y && !aligned(y, 16)) || !aligned(b, w_fp4 ? 32 : 16))
    return BQ_ERR_ALIGN;
  const void* bias = epi ? epi->bias : nullptr;
  const void* res = epi ? epi->residual : nullptr;
  const int64_t ldres = epi ? epi->ld_residual : 0;
  if (epi && epi->act != BQ_ACT_NONE && epi->act != BQ_ACT_GELU) return BQ_ERR_INVALID;
  if (bias && !aligned(bias, 16)) return BQ_ERR_ALIGN;
  if (res && (!aligned(res, 16) || ldres % 8 != 0 || ldres < N)) return BQ_ERR_ALIGN;
  int64_t sa = 0, ssa = 0, sb = 0, ssb = 0, sy = 0, sr = 0;
  if (batch && count > 1) {
    sa = batch->stride_a;
    ssa = batch->stride_a_sf;
    sb = batch->stride_b;
    ssb = batch->stride_b_sf;
    sy = batch->stride_y;
    sr = batch->stride_res;
    if (sa < 0 || ssa < 0 || sb < 0 || ssb < 0 || sy < 0 || sr < 0) return BQ_ERR_SHAPE;
    if (sa % 16 || ssa % 16 || ssb % 16 || sy % 16 || sr % 16 || sb % (w_fp4 ? 32 : 16))
      return BQ_ERR_ALIGN;
    if (sy == 0) return BQ_ERR_SHAPE;  // problems would overwrite each other
  }
  // The quantized output is written by epilogues that finish a tile in one
  // CTA: no K split (an explicit one is refused).
  bq_gemm_config cfg_q = cfg ? *cfg : bq_gemm_config{0, 0, -1, BQ_SPLIT_AUTO, 0, 0};
  if (q_out) {
    if (cfg_q.split_k > 1) return BQ_ERR_INVALID;
    cfg_q.split_k = 1;
    cfg = &cfg_q;
  }
  if (fused) {  // its one schedule: swap-AB, unsplit, 4 chunks per stage
    cfg_q = bq_gemm_config{0, 1, 1, BQ_SPLIT_AUTO, 4, 1};
    cfg = &cfg_q;
  }
  Plan pl;
  st = plan_for_call(wk, M, N, K, count, cfg, dev->num_sms, ws, ws_bytes, &pl);
  if (st != BQ_OK) return st;
  const size_t need = plan_ws_bytes(pl);
  if (need > 0 && !aligned(ws, 16)) return BQ_ERR_WORKSPACE;
  if (get_encoder() != BQ_OK) return BQ_ERR_CUDA;

  // Tensor maps: activations A [M, K] (row stride K), weights B [N, K] or [N, K/2].
  CUtensorMap map_a, map_b;
  // Swap-AB with every activation row in one tile: the box ends at the last
  // row (rounded up to 8), which copies far faster than a box whose trailing
  // rows all fall outside the tensor.
  const int a_box =
      pl.swap ? (pl.tiles_q == 1 ? static_cast<int>(std::min<int64_t>(pl.bn, (M + 7) / 8 * 8))
                                 : pl.bn)
              : 128;
  const int b_box = (pl.swap || pl.pair) ? 128 : pl.bn;  // a pair CTA loads 128 of 256 rows
  const bool a_batched = count > 1 && sa != 0;
  const bool b_batched = count > 1 && sb != 0;
  if (fused) {
    st = BQ_OK;  // no activation copies: map_a is set to a placeholder below
  } else {
    st = make_operand_map(&map_a, a_q, false, Kb, M, Kb, a_batched ? count : 1, sa, a_box,
                          pl.kc);
    if (st != BQ_OK) return st;
  }
  st = make_operand_map(&map_b, b, w_fp4, Kb, N, w_fp4 ? K / 2 : Kb, b_batched ? count : 1, sb,
                        b_box, pl.kc);
  if (st != BQ_OK) return st;
  if (fused) map_a = map_b;
  // Output y [batch][M][N] bf16 for the wide tiles' TMA-store epilogue: 128-row
  // x 32-column boxes with the 64-byte swizzle.
  CUtensorMap map_y = map_a;  // placeholder when no bf16 output is written
  if (y) {
    st = make_y_map(&map_y, y, M, N, N, count, sy);
    if (st != BQ_OK) return st;
  }
  // The residual, loaded by the same tiles into the staging buffer; a zero
  // batch stride (one residual for every problem) makes it a 2-D map.
  CUtensorMap map_res = map_y;  // placeholder without a residual
  if (res) {
    st = make_y_map(&map_res, res, M, N, ldres, count > 1 && sr != 0 ? count : 1, sr);
    if (st != BQ_OK) return st;
  }

  bq::GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.M = static_cast<int>(M);
  {
    const uint32_t f_act = wk == kGrad ? bq::kFmtE5M2 : bq::kFmtE4M3;
    const uint32_t f_w = w_fp4 ? bq::kFmtE2M1 : bq::kFmtE4M3;
    g.fmt_p = pl.swap ? f_w : f_act;
    g.fmt_q = pl.swap ? f_act : f_w;
  }
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.batch = static_cast<int>(count);
  g.kt_total = pl.kt_total;
  g.splits = pl.splits;
  g.kt_per_split = pl.kt_per_split;
  g.tiles_p = pl.tiles_p;
  g.tiles_q = pl.tiles_q;
  g.raster_group = 8;
  g.sf_katoms = ceil_div(K, wk == kNv4 ? 64 : 128);  // scale atoms: 4 groups of 16 or 32
  g.sf_q_rowatoms = ceil_div(pl.swap ? M : N, 128);
  // the fused quantizer lays the activation tile out with chunks BN rows apart
  g.q_box_rows = fused ? pl.bn : (pl.swap ? a_box : b_box);
  g.split_lg = 0;
  while ((1 << g.split_lg) < pl.splits) ++g.split_lg;
  const uint8_t* sfa = static_cast<const uint8_t*>(a_sf);
  const uint8_t* sfb = static_cast<const uint8_t*>(b_sf);
  g.sf_p = pl.swap ? sfb : sfa;
  g.sf_q = pl.swap ? sfa : sfb;
  g.sf_p_bstride = pl.swap ? ssb : ssa;
  g.sf_q_bstride = pl.swap ? ssa : ssb;
  g.p_batched = pl.swap ? b_batched : a_batched;
  g.q_batched = pl.swap ? a_batched : b_batched;
  g.y = static_cast<__nv_bfloat16*>(y);
  g.ldy = N;
  g.y_bstride = sy / 2;
  g.bias = static_cast<const __nv_bfloat16*>(bias);
  g.res = static_cast<const __nv_bfloat16*>(res);
  g.ldres = ldres;
  g.res_bstride = sr / 2;
  g.alpha = epi ? epi->alpha : 1.0f;
  g.act = epi ? epi->act : BQ_ACT_NONE;
  if (fused) {
    g.x = static_cast<const __nv_bfloat16*>(fused->x);
    g.ldx = fused->ldx;
    g.a_q_out = static_cast<uint8_t*>(fused->a_q_out);
    g.a_sf_out = static_cast<uint8_t*>(fused->a_sf_out);
    g.status = fused->status;
  }
  g.q_out = static_cast<uint8_t*>(q_out);
  g.sf_out = static_cast<uint8_t*>(sf_out);
  g.sf_out_bstride = static_cast<int64_t>(bq_sf_bytes(M, N));
  if (pl.splits > 1 && !pl.cluster) {
    g.ws_ticket = static_cast<int*>(ws);
    g.ws_partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kTicketRegion);
  }
  g.err = dev->err_ptr;
  // A workspace that may hold another call's leftovers (the allocation-free
  // entry's scratch): its ticket counters are zeroed on the stream only now,
  // after every argument check, right before the kernel that reads them.
  if (clear_tickets && pl.splits > 1 && !pl.cluster &&
      cudaMemsetAsync(ws, 0, pl.ws_ticket, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BQ_ERR_CUDA;
  if (pl.pair) {
    CUtensorMap map_sfa, map_sfb;
    // a stage's scale box: its chunks' atoms (two per chunk for packed E2M1)
    const int sf_box = pl.kc * (a4 ? 2 : 1);
    st = make_scale_map(&map_sfa, a_sf, M, K, a_batched ? count : 1, ssa, sf_box, 1);
    if (st != BQ_OK) return st;
    st = make_scale_map(&map_sfb, b_sf, N, K, b_batched ? count : 1, ssb, sf_box, 2);
    if (st != BQ_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t u = pl.units;
    const int ns = dev->num_sms;
    if (a4)  // the packed stages hold the scale atoms of 256 K per chunk: fewer fit
      return pl.kc == 2
                 ? launch_pair<2, 2, false, true>(map_a, map_b, map_sfa, map_sfb, map_y, map_res,
                                                  g, u, ns, s)
                 : launch_pair<5, 1, false, true>(map_a, map_b, map_sfa, map_sfb, map_y, map_res,
                                                  g, u, ns, s);
    if (pl.kc == 2)
      return w_fp4 ? launch_pair<3, 2, true>(map_a, map_b, map_sfa, map_sfb, map_y, map_res, g, u, ns, s)
                   : launch_pair<3, 2, false>(map_a, map_b, map_sfa, map_sfb, map_y, map_res, g, u, ns, s);
    return w_fp4 ? launch_pair<6, 1, true>(map_a, map_b, map_sfa, map_sfb, map_y, map_res, g, u, ns, s)
                 : launch_pair<6, 1, false>(map_a, map_b, map_sfa, map_sfb, map_y, map_res, g, u, ns, s);
  }
  const CUtensorMap& tp = pl.swap ? map_b : map_a;
  const CUtensorMap& tq = pl.swap ? map_a : map_b;
  if (wk == kNv4)
    return run_gemm_nv(pl, tp, tq, map_y, map_res, g, dev->num_sms,
                       reinterpret_cast<cudaStream_t>(stream));
  if (a4)
    return run_gemm<1>(pl, false, tp, tq, map_y, map_res, g, dev->num_sms,
                       reinterpret_cast<cudaStream_t>(stream));
  return run_gemm<0>(pl, w_fp4, tp, tq, map_y, map_res, g, dev->num_sms,
                     reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

// ================================================================== C ABI ==

extern "C" {

const char* bq_status_string(int status) {
  switch (status) {
    case BQ_OK: return "BQ_OK";
    case BQ_ERR_NULL: return "BQ_ERR_NULL: a required pointer is NULL";
    case BQ_ERR_SHAPE: return "BQ_ERR_SHAPE: size out of range or not a required multiple";
    case BQ_ERR_ALIGN: return "BQ_ERR_ALIGN: address or stride breaks the alignment rule";
    case BQ_ERR_NAN_SCALE: return "BQ_ERR_NAN_SCALE: E8M0 scale byte 255 (NaN)";
    case BQ_ERR_NAN_CODE: return "BQ_ERR_NAN_CODE: E4M3 weight code 0x7F/0xFF (NaN)";
    case BQ_ERR_ARCH: return "BQ_ERR_ARCH: device is not compute capability 10.0";
    case BQ_ERR_WORKSPACE: return "BQ_ERR_WORKSPACE: workspace missing or too small";
    case BQ_ERR_CUDA: return "BQ_ERR_CUDA: CUDA call or launch failed";
    case BQ_ERR_TIMEOUT: return "BQ_ERR_TIMEOUT: a kernel gave up waiting on a barrier";
    case BQ_ERR_NONFINITE: return "BQ_ERR_NONFINITE: NaN or Inf activation";
    case BQ_ERR_INVALID: return "BQ_ERR_INVALID: enum or option out of range";
    default: return "BQ_ERR_UNKNOWN";
  }
}

int bq_version(void) { return 100; }

size_t bq_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 32 != 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((K + 127) / 128) * 512;
}

size_t bq_sf_bytes_nvfp4(int64_t rows, int64_t K) {
  if (rows < 0 || K <= 0 || K % 16 != 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((K + 63) / 64) * 512;
}

}  // extern "C"

namespace {

// Launch of the per-32 quantizer along rows: fmt bq::kQE4M3 / kQFP4 /
// kQE5M2, sr stochastic rounding (E5M2 only) under `seed`.
// Rows per warp of act_quant_kernel on large operands (rows_pad is a multiple
// of 128, so of 8 * kAqRows).
constexpr int kAqRows = 2;

int act_quant_launch(int fmt, bool sr, uint64_t seed, const void* x_bf16, int64_t M, int64_t K,
                     int64_t ldx, void* q_out, void* sf_mma, void* sf_rowmajor, int* d_status,
                     bq_stream_t stream) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  if (M < 0 || K <= 0 || K % 32 != 0 || ldx < K) return BQ_ERR_SHAPE;
  if (M == 0) return BQ_OK;
  if (!x_bf16 || !q_out || !sf_mma) return BQ_ERR_NULL;
  if (!aligned(x_bf16, 16) || ldx % 8 != 0 || !aligned(q_out, 16) || !aligned(sf_mma, 4))
    return BQ_ERR_ALIGN;
  const int64_t rows_pad = (M + 127) / 128 * 128;
  const int64_t chunks = (K / 32 + 15) / 16;
  if (rows_pad / 8 > 0x7FFFFFFF || chunks > 65535) return BQ_ERR_SHAPE;
  // Grids of >= 6144 one-row blocks (about five waves of resident blocks):
  // each warp takes kAqRows rows, their loads all in flight before any is
  // quantized, and half as many blocks come and go (8192 x 8192: 47.9 ->
  // 45.1 us).  Smaller grids keep one row per warp: there the longer per-warp
  // path costs more than it saves (1024 x 4096: 4.6 -> 6.1 us).  Stochastic
  // rounding is bound by its Philox arithmetic and keeps one row.
  const int rows_per_warp = (!sr && (rows_pad / 8) * chunks >= 6144) ? kAqRows : 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(rows_pad / (8 * rows_per_warp)),
                    static_cast<unsigned>(chunks));
  lc.blockDim = dim3(256);
  lc.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  const bool multi = rows_per_warp > 1;
  auto kern = fmt == bq::kQFP4
                  ? (multi ? bq::act_quant_kernel<bq::kQFP4, false, kAqRows>
                           : bq::act_quant_kernel<bq::kQFP4>)
              : fmt == bq::kQE5M2
                  ? (sr ? bq::act_quant_kernel<bq::kQE5M2, true>
                        : multi ? bq::act_quant_kernel<bq::kQE5M2, false, kAqRows>
                                : bq::act_quant_kernel<bq::kQE5M2>)
                  : (multi ? bq::act_quant_kernel<bq::kQE4M3, false, kAqRows>
                           : bq::act_quant_kernel<bq::kQE4M3>);
  if (cudaLaunchKernelEx(&lc, kern, static_cast<const __nv_bfloat16*>(x_bf16), M, K, ldx,
                         rows_pad, static_cast<uint8_t*>(q_out), static_cast<uint8_t*>(sf_mma),
                         static_cast<uint8_t*>(sf_rowmajor), d_status, seed) != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return launch_status();
}

// Launch of the transposed quantizer: x [R, ldx] (C columns) along R into
// codes [C, R] and the MMA-layout scales of a [C, R] operand.
int quant_t_launch(int fmt, bool sr, uint64_t seed, const void* x_bf16, int64_t R, int64_t C,
                   int64_t ldx, void* q_t, void* sf_mma, int* d_status, bq_stream_t stream) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  if (R <= 0 || R % 32 != 0 || C < 0 || C % 8 != 0 || ldx < C) return BQ_ERR_SHAPE;
  if (C == 0) return BQ_OK;
  if (!x_bf16 || !q_t || !sf_mma) return BQ_ERR_NULL;
  if (!aligned(x_bf16, 16) || ldx % 8 != 0 || !aligned(q_t, 16)) return BQ_ERR_ALIGN;
  const int64_t rows_pad = (C + 127) / 128 * 128;  // rows of the transposed operand
  const int64_t col_tiles = rows_pad / 64;
  const int64_t groups_pad = (R / 32 + 3) / 4 * 4;
  if (groups_pad > 0x7FFFFFFF || (col_tiles + 7) / 8 > 65535) return BQ_ERR_SHAPE;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(groups_pad), static_cast<unsigned>((col_tiles + 7) / 8));
  lc.blockDim = dim3(256);
  lc.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  cudaError_t e;
  if (sr) {  // stochastic: the row-per-lane kernel, one Philox block per 4 columns
    e = cudaLaunchKernelEx(&lc, bq::quant_t_kernel<bq::kQE5M2, true>,
                           static_cast<const __nv_bfloat16*>(x_bf16), R, C, ldx, col_tiles,
                           static_cast<uint8_t*>(q_t), static_cast<uint8_t*>(sf_mma), d_status,
                           seed);
  } else {
    auto kern = fmt == bq::kQE5M2 ? bq::quant_t_rne_kernel<bq::kQE5M2>
                                  : bq::quant_t_rne_kernel<bq::kQE4M3>;
    e = cudaLaunchKernelEx(&lc, kern, static_cast<const __nv_bfloat16*>(x_bf16), R, C, ldx,
                           col_tiles, static_cast<uint8_t*>(q_t), static_cast<uint8_t*>(sf_mma),
                           d_status);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return launch_status();
}

// Launch of the fused row-wise + transposed gradient quantizer.
int grad_dual_launch(bool sr, uint64_t seed, const void* g_bf16, int64_t R, int64_t C,
                     int64_t ldg, void* q_row, void* sf_row, void* q_t, void* sf_t,
                     int* d_status, bq_stream_t stream) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  if (R < 0 || R % 32 != 0 || C <= 0 || C % 32 != 0 || ldg < C) return BQ_ERR_SHAPE;
  if (R == 0) return BQ_OK;
  if (!g_bf16 || !q_row || !sf_row || !q_t || !sf_t) return BQ_ERR_NULL;
  if (!aligned(g_bf16, 16) || ldg % 8 != 0 || !aligned(q_row, 16) || !aligned(q_t, 16))
    return BQ_ERR_ALIGN;
  const int64_t col_tiles = (C + 127) / 128 * 128 / 64;
  const int64_t groups_pad = (R / 32 + 3) / 4 * 4;
  if (groups_pad > 0x7FFFFFFF || (col_tiles + 7) / 8 > 65535) return BQ_ERR_SHAPE;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(groups_pad), static_cast<unsigned>((col_tiles + 7) / 8));
  lc.blockDim = dim3(256);
  lc.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  auto kern = sr ? bq::grad_quant_dual_kernel<true> : bq::grad_quant_dual_kernel<false>;
  if (cudaLaunchKernelEx(&lc, kern, static_cast<const __nv_bfloat16*>(g_bf16), R, C, ldg,
                         col_tiles, groups_pad, static_cast<uint8_t*>(q_row),
                         static_cast<uint8_t*>(sf_row), static_cast<uint8_t*>(q_t),
                         static_cast<uint8_t*>(sf_t), d_status, seed) != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace

extern "C" {

int bq_act_quant(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, void* q_e4m3,
                 void* sf_mma, void* sf_rowmajor, int* d_status, bq_stream_t stream) {
  return act_quant_launch(bq::kQE4M3, false, 0, x_bf16, M, K, ldx, q_e4m3, sf_mma, sf_rowmajor,
                          d_status, stream);
}

int bq_act_quant_mxfp4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, void* q_fp4,
                       void* sf_mma, void* sf_rowmajor, int* d_status, bq_stream_t stream) {
  return act_quant_launch(bq::kQFP4, false, 0, x_bf16, M, K, ldx, q_fp4, sf_mma, sf_rowmajor,
                          d_status, stream);
}

int bq_act_quant_nvfp4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, float g,
                       void* q_fp4, void* sf_mma, void* sf_rowmajor, int* d_status,
                       bq_stream_t stream) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  if (M < 0 || K <= 0 || K % 32 != 0 || ldx < K) return BQ_ERR_SHAPE;
  if (!(g > 0.0f) || !std::isfinite(g)) return BQ_ERR_INVALID;
  if (M == 0) return BQ_OK;
  if (!x_bf16 || !q_fp4 || !sf_mma) return BQ_ERR_NULL;
  if (!aligned(x_bf16, 16) || ldx % 8 != 0 || !aligned(q_fp4, 16) || !aligned(sf_mma, 4))
    return BQ_ERR_ALIGN;
  const int64_t rows_pad = (M + 127) / 128 * 128;
  const int64_t chunks = (K / 16 + 31) / 32;
  if (rows_pad / 8 > 0x7FFFFFFF || chunks > 65535) return BQ_ERR_SHAPE;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(rows_pad / 8), static_cast<unsigned>(chunks));
  lc.blockDim = dim3(256);
  lc.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (cudaLaunchKernelEx(&lc, bq::nvfp4_quant_kernel, static_cast<const __nv_bfloat16*>(x_bf16),
                         M, K, ldx, rows_pad, g, static_cast<uint8_t*>(q_fp4),
                         static_cast<uint8_t*>(sf_mma), static_cast<uint8_t*>(sf_rowmajor),
                         d_status) != cudaSuccess) {
    cudaGetLastError();
    return BQ_ERR_CUDA;
  }
  return launch_status();
}

int bq_grad_quant(const void* g_bf16, int64_t M, int64_t K, int64_t ldg, void* q_e5m2,
                  void* sf_mma, void* sf_rowmajor, int* d_status, int rounding, uint64_t seed,
                  bq_stream_t stream) {
  if (rounding != BQ_ROUND_NEAREST && rounding != BQ_ROUND_STOCHASTIC) return BQ_ERR_INVALID;
  return act_quant_launch(bq::kQE5M2, rounding == BQ_ROUND_STOCHASTIC, seed, g_bf16, M, K, ldg,
                          q_e5m2, sf_mma, sf_rowmajor, d_status, stream);
}

int bq_grad_quant_dual(const void* g_bf16, int64_t R, int64_t C, int64_t ldg, int rounding,
                       uint64_t seed, void* q_row, void* sf_row, void* q_t, void* sf_t,
                       int* d_status, bq_stream_t stream) {
  if (rounding != BQ_ROUND_NEAREST && rounding != BQ_ROUND_STOCHASTIC) return BQ_ERR_INVALID;
  return grad_dual_launch(rounding == BQ_ROUND_STOCHASTIC, seed, g_bf16, R, C, ldg, q_row, sf_row,
                          q_t, sf_t, d_status, stream);
}

int bq_quant_transposed(const void* x_bf16, int64_t R, int64_t C, int64_t ldx, int fmt,
                        int rounding, uint64_t seed, void* q_t, void* sf_mma, int* d_status,
                        bq_stream_t stream) {
  if (fmt != BQ_FMT_E4M3 && fmt != BQ_FMT_E5M2) return BQ_ERR_INVALID;
  if (rounding != BQ_ROUND_NEAREST && rounding != BQ_ROUND_STOCHASTIC) return BQ_ERR_INVALID;
  if (rounding == BQ_ROUND_STOCHASTIC && fmt != BQ_FMT_E5M2) return BQ_ERR_INVALID;
  return quant_t_launch(fmt == BQ_FMT_E5M2 ? bq::kQE5M2 : bq::kQE4M3,
                        rounding == BQ_ROUND_STOCHASTIC, seed, x_bf16, R, C, ldx, q_t, sf_mma,
                        d_status, stream);
}

int bq_pack_weight_scales(const void* scales_u8, int kind, int64_t N, int64_t K, void* sf_mma,
                          const void* e4m3_codes, bq_stream_t stream) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  if (kind != BQ_SF_ROW32 && kind != BQ_SF_BLK32x32 && kind != BQ_SF_ROW16_E4M3)
    return BQ_ERR_INVALID;
  if (N < 0 || K <= 0 || K % (kind == BQ_SF_ROW16_E4M3 ? 16 : 32) != 0) return BQ_ERR_SHAPE;
  if (N == 0) return BQ_OK;
  if (!scales_u8 || !sf_mma) return BQ_ERR_NULL;
  if (!aligned(sf_mma, 4) || (e4m3_codes && !aligned(e4m3_codes, 16))) return BQ_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(dev->flags_ptr, 0, sizeof(int), s) != cudaSuccess) return BQ_ERR_CUDA;
  const int64_t G = K / (kind == BQ_SF_ROW16_E4M3 ? 16 : 32);
  const int64_t rows_pad = (N + 127) / 128 * 128;
  const int64_t words = rows_pad * ((G + 3) / 4);
  const int64_t blocks = (words + 255) / 256 < 4096 ? (words + 255) / 256 : 4096;
  bq::pack_scales_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      static_cast<const uint8_t*>(scales_u8), kind, N, G, rows_pad, static_cast<uint8_t*>(sf_mma),
      dev->flags_ptr);
  if (launch_status() != BQ_OK) return BQ_ERR_CUDA;
  if (e4m3_codes) {
    const int64_t n = N * K;
    int64_t nb = (n / 16 + 255) / 256;
    if (nb < 1) nb = 1;
    if (nb > 4096) nb = 4096;
    bq::scan_e4m3_nan_kernel<<<static_cast<unsigned>(nb), 256, 0, s>>>(
        static_cast<const uint8_t*>(e4m3_codes), n, dev->flags_ptr);
    if (launch_status() != BQ_OK) return BQ_ERR_CUDA;
  }
  int flags = 0;
  if (cudaMemcpyAsync(&flags, dev->flags_ptr, sizeof(int), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return BQ_ERR_CUDA;
  if (flags & 1) return BQ_ERR_NAN_SCALE;
  if (flags & 2) return BQ_ERR_NAN_CODE;
  return BQ_OK;
}

int bq_unpack_scales(const void* sf_mma, int64_t rows, int64_t K, void* rowmajor,
                     bq_stream_t stream) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  if (rows < 0 || K <= 0 || K % 32 != 0) return BQ_ERR_SHAPE;
  if (rows == 0) return BQ_OK;
  if (!sf_mma || !rowmajor) return BQ_ERR_NULL;
  const int64_t total = rows * (K / 32);
  const int64_t blocks = (total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096;
  bq::unpack_scales_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                             reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(sf_mma), rows, K / 32, static_cast<uint8_t*>(rowmajor));
  return launch_status();
}

// The plain entries take no workspace, so their schedule never splits K.
static const bq_gemm_config kNoSplit = {0, 1, -1, BQ_SPLIT_AUTO, 0, 0};

int bq_gemm_mxfp8_mxfp4(const void* a_q, const void* a_sf, const void* b_fp4, const void* b_sf,
                        int64_t M, int64_t N, int64_t K, void* y_bf16, bq_stream_t stream) {
  return gemm_entry(kMxfp4, a_q, a_sf, b_fp4, b_sf, M, N, K, y_bf16, nullptr, nullptr, nullptr, 0,
                    &kNoSplit, stream);
}

int bq_gemm_mxfp8_fp8blk32(const void* a_q, const void* a_sf, const void* b_e4m3,
                           const void* b_sf, int64_t M, int64_t N, int64_t K, void* y_bf16,
                           bq_stream_t stream) {
  return gemm_entry(kFp8Blk32, a_q, a_sf, b_e4m3, b_sf, M, N, K, y_bf16, nullptr, nullptr,
                    nullptr, 0, &kNoSplit, stream);
}

int bq_gemm_mxfp8_mxfp8(const void* a_q, const void* a_sf, const void* b_e4m3, const void* b_sf,
                        int64_t M, int64_t N, int64_t K, void* y_bf16, bq_stream_t stream) {
  return gemm_entry(kMxfp8, a_q, a_sf, b_e4m3, b_sf, M, N, K, y_bf16, nullptr, nullptr, nullptr,
                    0, &kNoSplit, stream);
}

int bq_gemm_e5m2_mxfp8(const void* a_e5m2, const void* a_sf, const void* b_e4m3,
                       const void* b_sf, int64_t M, int64_t N, int64_t K, void* y_bf16,
                       bq_stream_t stream) {
  return gemm_entry(kGrad, a_e5m2, a_sf, b_e4m3, b_sf, M, N, K, y_bf16, nullptr, nullptr, nullptr,
                    0, &kNoSplit, stream);
}

int bq_gemm_e5m2_mxfp8_epilogue(const void* a_e5m2, const void* a_sf, const void* b_e4m3,
                                const void* b_sf, int64_t M, int64_t N, int64_t K, void* y_bf16,
                                const bq_epilogue* epi, const bq_batch* batch, void* workspace,
                                size_t workspace_bytes, const bq_gemm_config* cfg,
                                bq_stream_t stream) {
  return gemm_entry(kGrad, a_e5m2, a_sf, b_e4m3, b_sf, M, N, K, y_bf16, epi, batch, workspace,
                    workspace_bytes, cfg, stream);
}

int bq_gemm_nvfp4_nvfp4(const void* a_fp4, const void* a_sf, const void* b_fp4, const void* b_sf,
                        int64_t M, int64_t N, int64_t K, void* y_bf16, bq_stream_t stream) {
  return gemm_entry(kNv4, a_fp4, a_sf, b_fp4, b_sf, M, N, K, y_bf16, nullptr, nullptr, nullptr, 0,
                    nullptr, stream);
}

int bq_gemm_nvfp4_nvfp4_epilogue(const void* a_fp4, const void* a_sf, const void* b_fp4,
                                 const void* b_sf, int64_t M, int64_t N, int64_t K, void* y_bf16,
                                 const bq_epilogue* epi, const bq_batch* batch, void* workspace,
                                 size_t workspace_bytes, const bq_gemm_config* cfg,
                                 bq_stream_t stream) {
  return gemm_entry(kNv4, a_fp4, a_sf, b_fp4, b_sf, M, N, K, y_bf16, epi, batch, workspace,
                    workspace_bytes, cfg, stream);
}

int bq_gemm_mxfp4_mxfp4(const void* a_fp4, const void* a_sf, const void* b_fp4, const void* b_sf,
                        int64_t M, int64_t N, int64_t K, void* y_bf16, bq_stream_t stream) {
  return gemm_entry(kA4W4, a_fp4, a_sf, b_fp4, b_sf, M, N, K, y_bf16, nullptr, nullptr, nullptr, 0,
                    &kNoSplit, stream);
}

int bq_gemm_mxfp4_mxfp4_epilogue(const void* a_fp4, const void* a_sf, const void* b_fp4,
                                 const void* b_sf, int64_t M, int64_t N, int64_t K, void* y_bf16,
                                 const bq_epilogue* epi, const bq_batch* batch, void* workspace,
                                 size_t workspace_bytes, const bq_gemm_config* cfg,
                                 bq_stream_t stream) {
  return gemm_entry(kA4W4, a_fp4, a_sf, b_fp4, b_sf, M, N, K, y_bf16, epi, batch, workspace,
                    workspace_bytes, cfg, stream);
}

size_t bq_gemm_workspace_bytes(int weight_kind, int64_t M, int64_t N, int64_t K, int64_t batch,
                               const bq_gemm_config* cfg) {
  if (weight_kind < 0 || weight_kind > 5 || M <= 0 || N <= 0 || K <= 0 || batch <= 0) return 0;
  DevInfo* dev = nullptr;
  if (current_device(&dev) != BQ_OK) return 0;
  Plan pl;
  if (plan_kind(static_cast<WeightKind>(weight_kind), M, N, K, batch, cfg, dev->num_sms, &pl) !=
      BQ_OK)
    return 0;
  return plan_ws_bytes(pl);
}

int bq_gemm_plan(int weight_kind, int64_t M, int64_t N, int64_t K, int64_t batch,
                 const bq_gemm_config* cfg, int num_sms, bq_gemm_config* out) {
  if (!out) return BQ_ERR_NULL;
  if (weight_kind < 0 || weight_kind > 5) return BQ_ERR_INVALID;
  if (M <= 0 || N <= 0 || K <= 0 || K % 32 != 0 || batch <= 0 || num_sms < 1)
    return BQ_ERR_SHAPE;
  Plan pl;
  const int st = plan_kind(static_cast<WeightKind>(weight_kind), M, N, K, batch, cfg, num_sms,
                           &pl);
  if (st != BQ_OK) return st;
  out->block_n = pl.bn;
  out->split_k = pl.splits;
  out->swap_ab = pl.swap ? 1 : 0;
  out->split_mode =
      pl.splits > 1 ? (pl.cluster ? BQ_SPLIT_CLUSTER : BQ_SPLIT_WORKSPACE) : BQ_SPLIT_AUTO;
  out->k_chunks = pl.kc;
  out->cta_pair = pl.pair ? 2 : 1;
  return BQ_OK;
}

int bq_gemm_mxfp8_mxfp4_epilogue(const void* a_q, const void* a_sf, const void* b_fp4,
                                 const void* b_sf, int64_t M, int64_t N, int64_t K, void* y_bf16,
                                 const bq_epilogue* epi, const bq_batch* batch, void* workspace,
                                 size_t workspace_bytes, const bq_gemm_config* cfg,
                                 bq_stream_t stream) {
  return gemm_entry(kMxfp4, a_q, a_sf, b_fp4, b_sf, M, N, K, y_bf16, epi, batch, workspace,
                    workspace_bytes, cfg, stream);
}

// ------------------------------------------------ allocation-free variant --
//
// For callers that cannot allocate device memory themselves -- an inference
// plugin that is handed only its input and output buffers, or a latency-bound
// serving loop whose memory is fixed when it starts -- this entry point runs
// the MXFP4-weight GEMM (with its K-split schedule) against a scratch area the
// library owns: a fixed-size array in the module's global memory, created
// when the library is loaded on a device and kept until the process exits.

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB per device

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on each device, looked up once per device
// (with that device current).  In host code the array's name is only a
// host-side stand-in, never a device address.
static void* g_noalloc_ptr[kMaxDevices] = {};

static int noalloc_scratch(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return BQ_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return BQ_OK;
}

int bq_gemm_mxfp8_fp8blk32_epilogue(const void* a_q, const void* a_sf, const void* b_e4m3,
                                    const void* b_sf, int64_t M, int64_t N, int64_t K,
                                    void* y_bf16, const bq_epilogue* epi, const bq_batch* batch,
                                    void* workspace, size_t workspace_bytes,
                                    const bq_gemm_config* cfg, bq_stream_t stream) {
  return gemm_entry(kFp8Blk32, a_q, a_sf, b_e4m3, b_sf, M, N, K, y_bf16, epi, batch, workspace,
                    workspace_bytes, cfg, stream);
}

int bq_gemm_bf16act_epilogue(int weight_kind, const void* x_bf16, int64_t ldx, const void* b,
                             const void* b_sf, int64_t M, int64_t N, int64_t K, void* y_bf16,
                             const bq_epilogue* epi, void* a_q_out, void* a_sf_out,
                             int* d_status, bq_stream_t stream) {
  if (weight_kind < 0 || weight_kind > 2) return BQ_ERR_INVALID;
  // A long K loop is faster split over a cluster than in one CTA: then the
  // activations are quantized by bq_act_quant into the caller's buffers and
  // the split GEMM consumes them (two launches).  The quantized output needs
  // an unsplit tile, so it always takes the fused kernel.
  if (M > 0 && M <= 64 && N > 0 && K > 0 && !(epi && epi->q_out)) {
    DevInfo* dev = nullptr;
    int st = current_device(&dev);
    if (st != BQ_OK) return st;
    Plan pl;
    if (make_plan(M, N, K, 1, nullptr, dev->num_sms, &pl) == BQ_OK && pl.splits > 1) {
      if (!a_q_out || !a_sf_out) return BQ_ERR_NULL;
      st = bq_act_quant(x_bf16, M, K, ldx, a_q_out, a_sf_out, nullptr, d_status, stream);
      if (st != BQ_OK) return st;
      return gemm_entry(static_cast<WeightKind>(weight_kind), a_q_out, a_sf_out, b, b_sf, M, N,
                        K, y_bf16, epi, nullptr, nullptr, 0, nullptr, stream);
    }
  }
  const FusedAct f{x_bf16, ldx, a_q_out, a_sf_out, d_status};
  return gemm_entry(static_cast<WeightKind>(weight_kind), nullptr, nullptr, b, b_sf, M, N, K,
                    y_bf16, epi, nullptr, nullptr, 0, nullptr, stream, &f);
}

int bq_gemm_mxfp8_mxfp8_epilogue(const void* a_q, const void* a_sf, const void* b_e4m3,
                                 const void* b_sf, int64_t M, int64_t N, int64_t K, void* y_bf16,
                                 const bq_epilogue* epi, const bq_batch* batch, void* workspace,
                                 size_t workspace_bytes, const bq_gemm_config* cfg,
                                 bq_stream_t stream) {
  return gemm_entry(kMxfp8, a_q, a_sf, b_e4m3, b_sf, M, N, K, y_bf16, epi, batch, workspace,
                    workspace_bytes, cfg, stream);
}

int bq_gemm_mxfp8_mxfp4_epilogue_noalloc(const void* a_q, const void* a_sf, const void* b_fp4,
                                         const void* b_sf, int64_t M, int64_t N, int64_t K,
                                         void* y_bf16, const bq_epilogue* epi,
                                         const bq_batch* batch, const bq_gemm_config* cfg,
                                         bq_stream_t stream) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  const int64_t count = batch ? batch->count : 1;
  if (M < 0 || N < 0 || K <= 0 || K % 32 != 0 || count < 0) return BQ_ERR_SHAPE;
  if (M == 0 || N == 0 || count == 0) return BQ_OK;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != BQ_OK) return st;
  // The scratch keeps whatever the previous call left: the call zeroes this
  // problem's ticket counters itself, after its argument checks, just before
  // the kernel.
  return gemm_entry(kMxfp4, a_q, a_sf, b_fp4, b_sf, M, N, K, y_bf16, epi, batch, scratch,
                    kNoAllocScratchBytes, cfg, stream, nullptr, /*clear_tickets=*/true);
}

size_t bq_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int bq_device_status_detail(bq_stream_t stream, int* detail) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int err = 0;
  if (cudaMemcpyAsync(&err, dev->err_ptr, sizeof(int), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaMemsetAsync(dev->err_ptr, 0, sizeof(int), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return BQ_ERR_CUDA;
  if (detail) *detail = err;
  if (err & BQ_DEV_ERR_TIMEOUT) return BQ_ERR_TIMEOUT;
  return (err & BQ_DEV_ERR_NONFINITE) ? BQ_ERR_NONFINITE : BQ_OK;
}

int bq_selftest_wait_timeout(int64_t limit_us, bq_stream_t stream) {
  DevInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != BQ_OK) return st;
  if (limit_us < 1 || limit_us > 1000000) return BQ_ERR_SHAPE;
  wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      dev->err_ptr, static_cast<uint64_t>(limit_us) * 1000u);
  return launch_status();
}

int bq_debug_override_compute_capability(int major, int minor) {
  if (major < 0 || minor < 0) {
    g_cc_override.store(-1);
    return BQ_OK;
  }
  if (major > 99 || minor > 9) return BQ_ERR_INVALID;
  g_cc_override.store(major * 10 + minor);
  return BQ_OK;
}

int bq_device_status(bq_stream_t stream) { return bq_device_status_detail(stream, nullptr); }

int bq_device_report(char* buf, size_t n) {
  if (!buf || n == 0) return BQ_ERR_NULL;
  int dev = 0;
  cudaDeviceProp p;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&p, dev) != cudaSuccess) {
    snprintf(buf, n, "no CUDA device");
    return BQ_ERR_CUDA;
  }
  int clk = 0, mclk = 0;
  cudaDeviceGetAttribute(&clk, cudaDevAttrClockRate, dev);
  cudaDeviceGetAttribute(&mclk, cudaDevAttrMemoryClockRate, dev);
  snprintf(buf, n, "%s cc %d.%d, %d SMs, L2 %d KiB, smem/block optin %zu KiB, sm clock %d MHz, mem clock %d MHz",
           p.name, p.major, p.minor, p.multiProcessorCount, p.l2CacheSize / 1024,
           p.sharedMemPerBlockOptin / 1024, clk / 1000, mclk / 1000);
  return (p.major == 10 && p.minor == 0) ? BQ_OK : BQ_ERR_ARCH;
}

}  // extern "C"
