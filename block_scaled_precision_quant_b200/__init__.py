"""Python binding of libbq, the C-ABI library declared in include/bq.h.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libbq.so``.  Tensors must live on a CUDA device of compute
capability 10.0 (B200); torch is used for device memory, streams and the
optional allocation of outputs.  If ``libbq.so`` has not been built, the first
call raises -- there is no CPU fallback.

Build the library with ``python -m block_scaled_precision_quant_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbq.so")

# status codes (include/bq.h)
BQ_OK = 0
BQ_ERR_NULL = 1
BQ_ERR_SHAPE = 2
BQ_ERR_ALIGN = 3
BQ_ERR_NAN_SCALE = 4
BQ_ERR_NAN_CODE = 5
BQ_ERR_ARCH = 6
BQ_ERR_WORKSPACE = 7
BQ_ERR_CUDA = 8
BQ_ERR_TIMEOUT = 9
BQ_ERR_NONFINITE = 10
BQ_ERR_INVALID = 11

BQ_SF_ROW32 = 0
BQ_SF_BLK32x32 = 1
BQ_SF_ROW16_E4M3 = 2
BQ_ACT_NONE = 0
BQ_ACT_GELU = 1
BQ_SPLIT_AUTO, BQ_SPLIT_WORKSPACE, BQ_SPLIT_CLUSTER = 0, 1, 2
W_MXFP4, W_FP8BLK32, W_MXFP8 = 0, 1, 2
W_A4W4 = 3  # MXFP4 weights with MXFP4 (packed E2M1) activations
W_GRAD = 4  # E5M2 gradient codes x MXFP8 (E4M3) operand: the backward products
W_NVFP4 = 5  # NVFP4 x NVFP4 (E2M1 with E4M3 scales per 16)
BQ_ROUND_NEAREST, BQ_ROUND_STOCHASTIC = 0, 1
BQ_FMT_E4M3, BQ_FMT_E5M2 = 0, 1

EXPORTS = (
    "bq_status_string", "bq_version", "bq_sf_bytes", "bq_act_quant", "bq_pack_weight_scales",
    "bq_unpack_scales", "bq_gemm_mxfp8_mxfp4", "bq_gemm_mxfp8_fp8blk32", "bq_gemm_mxfp8_mxfp8",
    "bq_gemm_workspace_bytes", "bq_gemm_mxfp8_mxfp4_epilogue", "bq_gemm_mxfp8_fp8blk32_epilogue",
    "bq_gemm_mxfp8_mxfp8_epilogue", "bq_device_status", "bq_device_status_detail",
    "bq_device_report", "bq_gemm_mxfp8_mxfp4_epilogue_noalloc", "bq_noalloc_scratch_bytes",
    "bq_gemm_bf16act_epilogue", "bq_gemm_plan", "bq_act_quant_mxfp4", "bq_gemm_mxfp4_mxfp4",
    "bq_gemm_mxfp4_mxfp4_epilogue", "bq_grad_quant", "bq_quant_transposed", "bq_gemm_e5m2_mxfp8",
    "bq_gemm_e5m2_mxfp8_epilogue", "bq_grad_quant_dual", "bq_sf_bytes_nvfp4", "bq_act_quant_nvfp4",
    "bq_gemm_nvfp4_nvfp4", "bq_gemm_nvfp4_nvfp4_epilogue", "bq_selftest_wait_timeout",
    "bq_debug_override_compute_capability",
)


class BqError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = lib().bq_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{what}: {msg}" if what else msg)


class Epilogue(ctypes.Structure):
    _fields_ = [("bias", ctypes.c_void_p), ("residual", ctypes.c_void_p),
                ("ld_residual", ctypes.c_int64), ("alpha", ctypes.c_float), ("act", ctypes.c_int),
                ("q_out", ctypes.c_void_p), ("sf_out", ctypes.c_void_p)]


class Batch(ctypes.Structure):
    _fields_ = [("count", ctypes.c_int64), ("stride_a", ctypes.c_int64),
                ("stride_a_sf", ctypes.c_int64), ("stride_b", ctypes.c_int64),
                ("stride_b_sf", ctypes.c_int64), ("stride_y", ctypes.c_int64),
                ("stride_res", ctypes.c_int64)]


class GemmConfig(ctypes.Structure):
    _fields_ = [("block_n", ctypes.c_int), ("split_k", ctypes.c_int), ("swap_ab", ctypes.c_int),
                ("split_mode", ctypes.c_int), ("k_chunks", ctypes.c_int),
                ("cta_pair", ctypes.c_int)]


_lib = None
_lock = threading.Lock()


def lib():
    """The loaded libbq.so (ctypes.CDLL); raises if it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_scaled_precision_quant_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.bq_status_string.argtypes = [i32]
        L.bq_status_string.restype = ctypes.c_char_p
        L.bq_version.restype = i32
        L.bq_sf_bytes.argtypes = [i64, i64]
        L.bq_sf_bytes.restype = sz
        L.bq_act_quant.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp]
        L.bq_act_quant.restype = i32
        L.bq_act_quant_mxfp4.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp]
        L.bq_act_quant_mxfp4.restype = i32
        L.bq_act_quant_nvfp4.argtypes = [vp, i64, i64, i64, ctypes.c_float, vp, vp, vp, vp, vp]
        L.bq_act_quant_nvfp4.restype = i32
        L.bq_sf_bytes_nvfp4.argtypes = [i64, i64]
        L.bq_sf_bytes_nvfp4.restype = sz
        L.bq_grad_quant.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, i32, ctypes.c_uint64, vp]
        L.bq_grad_quant.restype = i32
        L.bq_quant_transposed.argtypes = [vp, i64, i64, i64, i32, i32, ctypes.c_uint64, vp, vp,
                                          vp, vp]
        L.bq_quant_transposed.restype = i32
        L.bq_grad_quant_dual.argtypes = [vp, i64, i64, i64, i32, ctypes.c_uint64, vp, vp, vp, vp,
                                         vp, vp]
        L.bq_grad_quant_dual.restype = i32
        L.bq_pack_weight_scales.argtypes = [vp, i32, i64, i64, vp, vp, vp]
        L.bq_pack_weight_scales.restype = i32
        L.bq_unpack_scales.argtypes = [vp, i64, i64, vp, vp]
        L.bq_unpack_scales.restype = i32
        for name in ("bq_gemm_mxfp8_mxfp4", "bq_gemm_mxfp8_fp8blk32", "bq_gemm_mxfp8_mxfp8",
                     "bq_gemm_mxfp4_mxfp4", "bq_gemm_e5m2_mxfp8", "bq_gemm_nvfp4_nvfp4"):
            f = getattr(L, name)
            f.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
            f.restype = i32
        for name in ("bq_gemm_mxfp8_mxfp4_epilogue", "bq_gemm_mxfp8_fp8blk32_epilogue",
                     "bq_gemm_mxfp8_mxfp8_epilogue", "bq_gemm_mxfp4_mxfp4_epilogue",
                     "bq_gemm_e5m2_mxfp8_epilogue", "bq_gemm_nvfp4_nvfp4_epilogue"):
            f = getattr(L, name)
            f.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, ctypes.POINTER(Epilogue),
                          ctypes.POINTER(Batch), vp, sz, ctypes.POINTER(GemmConfig), vp]
            f.restype = i32
        L.bq_gemm_mxfp8_mxfp4_epilogue_noalloc.argtypes = [
            vp, vp, vp, vp, i64, i64, i64, vp, ctypes.POINTER(Epilogue), ctypes.POINTER(Batch),
            ctypes.POINTER(GemmConfig), vp]
        L.bq_gemm_mxfp8_mxfp4_epilogue_noalloc.restype = i32
        L.bq_noalloc_scratch_bytes.restype = sz
        L.bq_gemm_bf16act_epilogue.argtypes = [i32, vp, i64, vp, vp, i64, i64, i64, vp,
                                               ctypes.POINTER(Epilogue), vp, vp, vp, vp]
        L.bq_gemm_bf16act_epilogue.restype = i32
        L.bq_gemm_workspace_bytes.argtypes = [i32, i64, i64, i64, i64, ctypes.POINTER(GemmConfig)]
        L.bq_gemm_workspace_bytes.restype = sz
        L.bq_gemm_plan.argtypes = [i32, i64, i64, i64, i64, ctypes.POINTER(GemmConfig), i32,
                                   ctypes.POINTER(GemmConfig)]
        L.bq_gemm_plan.restype = i32
        L.bq_device_status.argtypes = [vp]
        L.bq_device_status.restype = i32
        L.bq_device_status_detail.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.bq_device_status_detail.restype = i32
        L.bq_device_report.argtypes = [ctypes.c_char_p, sz]
        L.bq_device_report.restype = i32
        L.bq_selftest_wait_timeout.argtypes = [i64, vp]
        L.bq_selftest_wait_timeout.restype = i32
        L.bq_debug_override_compute_capability.argtypes = [i32, i32]
        L.bq_debug_override_compute_capability.restype = i32
        _lib = L
        return L


# ------------------------------------------------------------------ helpers --

def _torch():
    import torch
    return torch


def _stream():
    return ctypes.c_void_p(_torch().cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(status: int, what: str):
    if status != BQ_OK:
        raise BqError(status, what)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libbq works on CUDA tensors only")


def sf_bytes(rows: int, K: int) -> int:
    """Bytes of an MMA-layout scale buffer for rows x K (K % 32 == 0)."""
    return int(lib().bq_sf_bytes(int(rows), int(K)))


def version() -> int:
    return int(lib().bq_version())


def status_string(status: int) -> str:
    return lib().bq_status_string(int(status)).decode()


def device_report() -> str:
    buf = ctypes.create_string_buffer(512)
    lib().bq_device_report(buf, 512)
    return buf.value.decode()


def device_status():
    """Synchronizes the current stream; raises BqError(BQ_ERR_TIMEOUT) if a
    kernel gave up on a barrier wait since the last check (the message carries
    the raw error word naming the wait site), BqError(BQ_ERR_NONFINITE) if a
    quantized-output GEMM epilogue met a NaN or Inf output."""
    detail = ctypes.c_int(0)
    st = lib().bq_device_status_detail(_stream(), ctypes.byref(detail))
    _check(st, f"device status (detail 0x{detail.value:x})")


# ----------------------------------------------------------- act_quant -----

def act_quant(x, q=None, sf_mma=None, sf_rowmajor=None, status=None):
    """Per-32 MX quantization of a bf16 [M, K] CUDA tensor (row stride may
    exceed K).  Returns (q uint8 [M, K] E4M3 codes, sf_mma uint8 MMA-layout
    scales).  sf_rowmajor ([M, K/32] uint8) and status (int32 [1]) are
    optional outputs filled when given."""
    torch = _torch()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [M, K] tensor with unit column stride")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if sf_mma is None:
        sf_mma = torch.empty((max(sf_bytes(M, K), 1),), dtype=torch.uint8, device=x.device)
    _check(lib().bq_act_quant(_ptr(x), M, K, x.stride(0), _ptr(q), _ptr(sf_mma),
                              _ptr(sf_rowmajor), _ptr(status), _stream()), "bq_act_quant")
    return q, sf_mma


def act_quant_mxfp4(x, q=None, sf_mma=None, sf_rowmajor=None, status=None):
    """Per-32 MXFP4 quantization of a bf16 [M, K] CUDA tensor: returns (q
    uint8 [M, K/2] packed E2M1 codes, low nibble = even element, sf_mma uint8
    MMA-layout scales), the operands of gemm(W_A4W4, ...)."""
    torch = _torch()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [M, K] tensor with unit column stride")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if sf_mma is None:
        sf_mma = torch.empty((max(sf_bytes(M, K), 1),), dtype=torch.uint8, device=x.device)
    _check(lib().bq_act_quant_mxfp4(_ptr(x), M, K, x.stride(0), _ptr(q), _ptr(sf_mma),
                                    _ptr(sf_rowmajor), _ptr(status), _stream()),
           "bq_act_quant_mxfp4")
    return q, sf_mma


def sf_bytes_nvfp4(rows: int, K: int) -> int:
    return int(lib().bq_sf_bytes_nvfp4(rows, K))


def act_quant_nvfp4(x, g=1.0, q=None, sf_mma=None, sf_rowmajor=None, status=None):
    """NVFP4 quantization of a bf16 [M, K] CUDA tensor scaled by the per-tensor
    g: returns (q uint8 [M, K/2] packed E2M1, sf_mma MMA-layout E4M3 scales per
    16), the operands of gemm(W_NVFP4, ...) (with alpha = 1 / (g_a g_b))."""
    torch = _torch()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [M, K] tensor with unit column stride")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if sf_mma is None:
        sf_mma = torch.empty((max(sf_bytes_nvfp4(M, K), 1),), dtype=torch.uint8, device=x.device)
    _check(lib().bq_act_quant_nvfp4(_ptr(x), M, K, x.stride(0), float(g), _ptr(q), _ptr(sf_mma),
                                    _ptr(sf_rowmajor), _ptr(status), _stream()),
           "bq_act_quant_nvfp4")
    return q, sf_mma


def grad_quant(g, stochastic=False, seed=0, q=None, sf_mma=None, sf_rowmajor=None,
               status=None):
    """Per-32 E5M2 quantization of a bf16 [M, K] gradient along K (round to
    nearest even, or stochastic with Philox draws keyed by seed): returns (q
    uint8 [M, K] E5M2 codes, sf_mma MMA-layout scales)."""
    torch = _torch()
    _need_cuda(g)
    if g.dtype != torch.bfloat16 or g.dim() != 2 or g.stride(1) != 1:
        raise ValueError("g must be a bf16 [M, K] tensor with unit column stride")
    M, K = g.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=g.device)
    if sf_mma is None:
        sf_mma = torch.empty((max(sf_bytes(M, K), 1),), dtype=torch.uint8, device=g.device)
    _check(lib().bq_grad_quant(_ptr(g), M, K, g.stride(0), _ptr(q), _ptr(sf_mma),
                               _ptr(sf_rowmajor), _ptr(status),
                               BQ_ROUND_STOCHASTIC if stochastic else BQ_ROUND_NEAREST,
                               int(seed) & (2 ** 64 - 1), _stream()), "bq_grad_quant")
    return q, sf_mma


def grad_quant_dual(g, stochastic=False, seed=0, out=None, status=None):
    """Both E5M2 quantizations of a bf16 [R, C] gradient in one pass: returns
    (q_row [R, C], sf_row, q_t [C, R], sf_t), equal to grad_quant(g) and
    quant_transposed(g, BQ_FMT_E5M2) with the same seed."""
    torch = _torch()
    _need_cuda(g)
    if g.dtype != torch.bfloat16 or g.dim() != 2 or g.stride(1) != 1:
        raise ValueError("g must be a bf16 [R, C] tensor with unit column stride")
    R, C = g.shape
    if out is None:
        u8 = dict(dtype=torch.uint8, device=g.device)
        out = (torch.empty((R, C), **u8), torch.empty((max(sf_bytes(R, C), 1),), **u8),
               torch.empty((C, R), **u8), torch.empty((max(sf_bytes(C, R), 1),), **u8))
    q_row, sf_row, q_t, sf_t = out
    _check(lib().bq_grad_quant_dual(_ptr(g), R, C, g.stride(0),
                                    BQ_ROUND_STOCHASTIC if stochastic else BQ_ROUND_NEAREST,
                                    int(seed) & (2 ** 64 - 1), _ptr(q_row), _ptr(sf_row),
                                    _ptr(q_t), _ptr(sf_t), _ptr(status), _stream()),
           "bq_grad_quant_dual")
    return q_row, sf_row, q_t, sf_t


def quant_transposed(x, fmt=BQ_FMT_E4M3, stochastic=False, seed=0, q=None, sf_mma=None,
                     status=None):
    """Quantize a bf16 [R, C] tensor along R (per 32 rows of each column) and
    write it transposed: returns (q uint8 [C, R] codes, sf_mma MMA-layout
    scales of a [C, R] operand).  fmt BQ_FMT_E4M3 or BQ_FMT_E5M2 (stochastic
    rounding for E5M2 only)."""
    torch = _torch()
    _need_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [R, C] tensor with unit column stride")
    R, C = x.shape
    if q is None:
        q = torch.empty((C, R), dtype=torch.uint8, device=x.device)
    if sf_mma is None:
        sf_mma = torch.empty((max(sf_bytes(C, R), 1),), dtype=torch.uint8, device=x.device)
    _check(lib().bq_quant_transposed(_ptr(x), R, C, x.stride(0), int(fmt),
                                     BQ_ROUND_STOCHASTIC if stochastic else BQ_ROUND_NEAREST,
                                     int(seed) & (2 ** 64 - 1), _ptr(q), _ptr(sf_mma),
                                     _ptr(status), _stream()), "bq_quant_transposed")
    return q, sf_mma


def pack_weight_scales(scales, kind: int, N: int, K: int, out=None, e4m3_codes=None):
    """Weight scales (E8M0 ROW32 [N, K/32] or BLK32x32 [ceil(N/32), K/32], or
    E4M3 ROW16_E4M3 [N, K/16] for NVFP4) to the MMA layout.  Synchronizes the stream; raises on NaN scales or codes."""
    torch = _torch()
    _need_cuda(scales, e4m3_codes)
    if out is None:
        n = sf_bytes_nvfp4(N, K) if kind == BQ_SF_ROW16_E4M3 else sf_bytes(N, K)
        out = torch.empty((max(n, 1),), dtype=torch.uint8, device=scales.device)
    _check(lib().bq_pack_weight_scales(_ptr(scales), int(kind), N, K, _ptr(out),
                                       _ptr(e4m3_codes), _stream()), "bq_pack_weight_scales")
    return out


def unpack_scales(sf_mma, rows: int, K: int, out=None):
    """MMA-layout scales back to row-major [rows, K/32] uint8."""
    torch = _torch()
    _need_cuda(sf_mma)
    if out is None:
        out = torch.empty((rows, K // 32), dtype=torch.uint8, device=sf_mma.device)
    _check(lib().bq_unpack_scales(_ptr(sf_mma), rows, K, _ptr(out), _stream()),
           "bq_unpack_scales")
    return out


# ---------------------------------------------------------------- GEMM -----

_ws = {}
_ENTRY = {W_MXFP4: "bq_gemm_mxfp8_mxfp4", W_FP8BLK32: "bq_gemm_mxfp8_fp8blk32",
          W_MXFP8: "bq_gemm_mxfp8_mxfp8", W_A4W4: "bq_gemm_mxfp4_mxfp4",
          W_GRAD: "bq_gemm_e5m2_mxfp8", W_NVFP4: "bq_gemm_nvfp4_nvfp4"}


def _config(block_n=0, split_k=0, swap_ab=-1, split_mode=0, k_chunks=0, cta_pair=0):
    return GemmConfig(int(block_n), int(split_k), int(swap_ab), int(split_mode), int(k_chunks),
                      int(cta_pair))


def workspace_bytes(weight_kind, M, N, K, batch=1, config=None) -> int:
    cfg = config if config is not None else None
    return int(lib().bq_gemm_workspace_bytes(int(weight_kind), M, N, K, batch,
                                             ctypes.byref(cfg) if cfg is not None else None))


def plan(M, N, K, batch=1, config=None, num_sms=148, weight_kind=0) -> GemmConfig:
    """The schedule the built-in dispatch picks (host-only, no device): every
    GemmConfig field resolved for a device with num_sms SMs."""
    out = GemmConfig()
    _check(lib().bq_gemm_plan(int(weight_kind), M, N, K, batch,
                              ctypes.byref(config) if config is not None else None, num_sms,
                              ctypes.byref(out)), "bq_gemm_plan")
    return out


def _workspace(device, nbytes):
    """A zero-initialized per-device workspace, grown on demand.  The kernels
    leave its ticket counters at zero after every call."""
    torch = _torch()
    key = device.index if device.index is not None else torch.cuda.current_device()
    buf = _ws.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros((max(nbytes, 256),), dtype=torch.uint8, device=device)
        _ws[key] = buf
    return buf


def gemm(weight_kind, a_q, a_sf, b, b_sf, M, N, K, y=None, bias=None, residual=None,
         alpha=1.0, act=BQ_ACT_NONE, batch=None, config=None, workspace=None,
         quantize_out=False, write_y=True, q_out=None, sf_out=None):
    """y = bf16(act(alpha * A B^T + bias) + residual) for weight_kind W_MXFP4,
    W_FP8BLK32, W_MXFP8 (E4M3 activations a_q [.., M, K]), W_A4W4 (packed
    E2M1 activations a_q [.., M, K/2] from act_quant_mxfp4), W_NVFP4 (packed
    E2M1 activations and weights with E4M3 scales per 16, from act_quant_nvfp4;
    alpha = 1 / (g_a g_b) undoes the per-tensor scales) or W_GRAD (E5M2
    gradient codes a_q [.., M, K], MXFP8 b).  batch: None or a dict with 'count' and byte
    strides ('stride_a', 'stride_a_sf', 'stride_b', 'stride_b_sf', 'stride_y',
    'stride_res'; 0 broadcasts).  config: GemmConfig or None (auto).
    quantize_out: also return y quantized for the next GEMM (E4M3 codes
    [.., M, N] u8 and MMA-layout scales, exactly act_quant of y, written to
    q_out / sf_out when given); then returns (y or None, q, sf), with no bf16
    y written when write_y is False."""
    torch = _torch()
    _need_cuda(a_q, a_sf, b, b_sf, bias, residual)
    count = 1 if batch is None else int(batch["count"])
    shape = (M, N) if batch is None else (count, M, N)
    if not write_y and not quantize_out:
        raise ValueError("write_y=False needs quantize_out=True")
    if y is None and write_y:
        y = torch.empty(shape, dtype=torch.bfloat16, device=a_q.device)
    if quantize_out:
        if q_out is None:
            q_out = torch.empty(shape, dtype=torch.uint8, device=a_q.device)
        if sf_out is None:
            per = sf_bytes(M, N)
            sf_out = torch.empty((per,) if batch is None else (count, per), dtype=torch.uint8,
                                 device=a_q.device)
    else:
        q_out = sf_out = None
    need = workspace_bytes(weight_kind, M, N, K, count, config)
    plain = (bias is None and residual is None and alpha == 1.0 and act == BQ_ACT_NONE
             and batch is None and config is None and workspace is None and need == 0
             and not quantize_out)
    if plain:
        f = getattr(lib(), _ENTRY[weight_kind])
        _check(f(_ptr(a_q), _ptr(a_sf), _ptr(b), _ptr(b_sf), M, N, K, _ptr(y), _stream()),
               _ENTRY[weight_kind])
        return y
    epi = Epilogue(bias.data_ptr() if bias is not None else None,
                   residual.data_ptr() if residual is not None else None,
                   residual.stride(-2) if residual is not None else 0, float(alpha), int(act),
                   q_out.data_ptr() if q_out is not None else None,
                   sf_out.data_ptr() if sf_out is not None else None)
    bt = None
    if batch is not None:
        bt = Batch(count, *(int(batch.get(k, 0)) for k in (
            "stride_a", "stride_a_sf", "stride_b", "stride_b_sf", "stride_y", "stride_res")))
    ws = workspace
    if need and ws is None:
        ws = _workspace(a_q.device, need)
    f = getattr(lib(), _ENTRY[weight_kind] + "_epilogue")
    _check(f(_ptr(a_q), _ptr(a_sf), _ptr(b), _ptr(b_sf), M, N, K, _ptr(y), ctypes.byref(epi),
             ctypes.byref(bt) if bt is not None else None, _ptr(ws),
             ws.numel() if ws is not None else 0,
             ctypes.byref(config) if config is not None else None, _stream()),
           _ENTRY[weight_kind] + "_epilogue")
    if quantize_out:
        return (y if write_y else None), q_out, sf_out
    return y


def gemm_bf16act(weight_kind, x, b, b_sf, M, N, K, y=None, bias=None, residual=None, alpha=1.0,
                 act=BQ_ACT_NONE, store_act=False, status=None, quantize_out=False, write_y=True,
                 a_q=None, a_sf=None):
    """act_quant(x) and the GEMM of weight_kind in one launch (decode shapes:
    M <= 64, K % 128 == 0): the GEMM quantizes the bf16 activations x [M, K]
    itself.  store_act: also return the activation codes and MMA-layout scales
    bq_act_quant would write.  Returns y, or a tuple (y, [q, sf], [a_q, a_sf])
    when quantize_out / store_act ask for more."""
    torch = _torch()
    _need_cuda(x, b, b_sf, bias, residual, status)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a bf16 [M, K] tensor with unit column stride")
    if not write_y and not quantize_out:
        raise ValueError("write_y=False needs quantize_out=True")
    dev = x.device
    if y is None and write_y:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    q_out = sf_out = None
    if quantize_out:
        q_out = torch.empty((M, N), dtype=torch.uint8, device=dev)
        sf_out = torch.empty((sf_bytes(M, N),), dtype=torch.uint8, device=dev)
    # the library may need the activation buffers (a long-K shape runs act_quant
    # into them and a split GEMM); they are returned only with store_act
    a_q = torch.empty((M, K), dtype=torch.uint8, device=dev) if a_q is None else a_q
    a_sf = torch.empty((sf_bytes(M, K),), dtype=torch.uint8, device=dev) if a_sf is None else a_sf
    epi = Epilogue(bias.data_ptr() if bias is not None else None,
                   residual.data_ptr() if residual is not None else None,
                   residual.stride(-2) if residual is not None else 0, float(alpha), int(act),
                   q_out.data_ptr() if q_out is not None else None,
                   sf_out.data_ptr() if sf_out is not None else None)
    _check(lib().bq_gemm_bf16act_epilogue(
        int(weight_kind), _ptr(x), x.stride(0), _ptr(b), _ptr(b_sf), M, N, K,
        _ptr(y) if write_y else None, ctypes.byref(epi), _ptr(a_q), _ptr(a_sf), _ptr(status),
        _stream()), "bq_gemm_bf16act_epilogue")
    out = [y if write_y else None]
    if quantize_out:
        out += [q_out, sf_out]
    if store_act:
        out += [a_q, a_sf]
    return out[0] if len(out) == 1 else tuple(out)


def gemm_mxfp8_mxfp4(a_q, a_sf, b_fp4, b_sf, M, N, K, **kw):
    return gemm(W_MXFP4, a_q, a_sf, b_fp4, b_sf, M, N, K, **kw)


def gemm_mxfp8_fp8blk32(a_q, a_sf, b_e4m3, b_sf, M, N, K, **kw):
    return gemm(W_FP8BLK32, a_q, a_sf, b_e4m3, b_sf, M, N, K, **kw)


def gemm_mxfp8_mxfp8(a_q, a_sf, b_e4m3, b_sf, M, N, K, **kw):
    return gemm(W_MXFP8, a_q, a_sf, b_e4m3, b_sf, M, N, K, **kw)


def gemm_mxfp4_mxfp4(a_fp4, a_sf, b_fp4, b_sf, M, N, K, **kw):
    return gemm(W_A4W4, a_fp4, a_sf, b_fp4, b_sf, M, N, K, **kw)


def gemm_nvfp4_nvfp4(a_fp4, a_sf, b_fp4, b_sf, M, N, K, **kw):
    return gemm(W_NVFP4, a_fp4, a_sf, b_fp4, b_sf, M, N, K, **kw)


def gemm_e5m2_mxfp8(a_e5m2, a_sf, b_e4m3, b_sf, M, N, K, **kw):
    return gemm(W_GRAD, a_e5m2, a_sf, b_e4m3, b_sf, M, N, K, **kw)


config = _config
