"""CPU oracle for block-scaled (MX) activation quantization and GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product library never calls it, and it shares no code with the CUDA path.

The arithmetic lives in ``bq_oracle.c`` (plain C, fp64 sums, exact decode of
every operand); this module only builds that file with gcc and marshals numpy
arrays into it.  Each function cites the passage of the "formats.py" page
(dsv41-sampled-drafting, code/offload/dspark/native/formats.py) that it
follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, ERR_NAN_SCALE, ERR_NAN_CODE, ERR_SHAPE, ERR_NONFINITE = 0, -1, -2, -3, -4
B_FP4, B_FP8BLK, B_FP8ROW, B_NVFP4 = 0, 1, 2, 3
A_E4M3, A_FP4, A_E5M2, A_NVFP4 = 0, 1, 2, 3
Q_E4M3, Q_E5M2 = 0, 1  # code formats of the transposed quantizer
ACT_NONE, ACT_GELU = 0, 1

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-Wall", "-Wextra"]


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile bq_oracle.c into liboracle.so next to it (gcc, no fast-math,
    no FMA contraction).  Rebuilds when the source is newer than the library."""
    with _lock:
        if (not force and os.path.exists(_LIB)
                and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
            return _LIB
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
        return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    u16p = ctypes.POINTER(ctypes.c_uint16)
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    i64p = ctypes.POINTER(ctypes.c_int64)
    i64 = ctypes.c_int64
    lib.oracle_decode_e8m0.argtypes = [ctypes.c_uint8, f64p]
    lib.oracle_decode_e8m0.restype = ctypes.c_int
    lib.oracle_decode_fp4.argtypes = [ctypes.c_uint8]
    lib.oracle_decode_fp4.restype = ctypes.c_double
    lib.oracle_decode_e4m3.argtypes = [ctypes.c_uint8, f64p]
    lib.oracle_decode_e4m3.restype = ctypes.c_int
    lib.oracle_encode_e4m3.argtypes = [ctypes.c_float]
    lib.oracle_encode_e4m3.restype = ctypes.c_uint8
    lib.oracle_encode_e4m3_n.argtypes = [f32p, i64, u8p]
    lib.oracle_encode_e4m3_n.restype = None
    lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
    lib.oracle_act_quant.argtypes = [u16p, i64, i64, i64, u8p, u8p]
    lib.oracle_act_quant.restype = ctypes.c_int
    lib.oracle_act_quant_f32.argtypes = [f32p, i64, i64, u8p, u8p]
    lib.oracle_act_quant_f32.restype = ctypes.c_int
    lib.oracle_act_qdq.argtypes = [u8p, u8p, i64, i64, u16p]
    lib.oracle_act_qdq.restype = ctypes.c_int
    lib.oracle_encode_fp4.argtypes = [ctypes.c_float]
    lib.oracle_encode_fp4.restype = ctypes.c_uint8
    lib.oracle_encode_fp4_n.argtypes = [f32p, i64, u8p]
    lib.oracle_encode_fp4_n.restype = None
    lib.oracle_act_quant_fp4.argtypes = [u16p, i64, i64, i64, u8p, u8p]
    lib.oracle_act_quant_fp4.restype = ctypes.c_int
    lib.oracle_act_quant_fp4_f32.argtypes = [f32p, i64, i64, u8p, u8p]
    lib.oracle_act_quant_fp4_f32.restype = ctypes.c_int
    u64 = ctypes.c_uint64
    u64p = ctypes.POINTER(ctypes.c_uint64)
    lib.oracle_decode_e5m2.argtypes = [ctypes.c_uint8, f64p]
    lib.oracle_decode_e5m2.restype = ctypes.c_int
    lib.oracle_encode_e5m2.argtypes = [ctypes.c_float]
    lib.oracle_encode_e5m2.restype = ctypes.c_uint8
    lib.oracle_encode_e5m2_n.argtypes = [f32p, i64, u8p]
    lib.oracle_encode_e5m2_n.restype = None
    lib.oracle_encode_e5m2_sr.argtypes = [ctypes.c_float, ctypes.c_double]
    lib.oracle_encode_e5m2_sr.restype = ctypes.c_uint8
    lib.oracle_philox4x64_10.argtypes = [u64p, u64p, u64p]
    lib.oracle_philox4x64_10.restype = None
    lib.oracle_uniform.argtypes = [u64, u64]
    lib.oracle_uniform.restype = ctypes.c_double
    lib.oracle_grad_quant.argtypes = [u16p, i64, i64, i64, ctypes.c_int, u64, u8p, u8p]
    lib.oracle_grad_quant.restype = ctypes.c_int
    lib.oracle_quant_transposed.argtypes = [u16p, i64, i64, i64, ctypes.c_int, ctypes.c_int, u64,
                                            u8p, u8p]
    lib.oracle_quant_transposed.restype = ctypes.c_int
    lib.oracle_e4m3_ceil.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_ceil.restype = ctypes.c_uint8
    lib.oracle_act_quant_nvfp4.argtypes = [u16p, i64, i64, i64, ctypes.c_float, u8p, u8p]
    lib.oracle_act_quant_nvfp4.restype = ctypes.c_int
    lib.oracle_gemm_ex.argtypes = [u8p, u8p, ctypes.c_int, u8p, u8p, ctypes.c_int, i64, i64, i64,
                                   u16p, u16p, i64, ctypes.c_double, ctypes.c_int, f64p, f64p,
                                   ctypes.c_int]
    lib.oracle_gemm_ex.restype = ctypes.c_int
    lib.oracle_gemm_sampled_ex.argtypes = [u8p, u8p, ctypes.c_int, u8p, u8p, ctypes.c_int, i64,
                                           i64, i64, u16p, u16p, i64, ctypes.c_double,
                                           ctypes.c_int, i64p, i64p, i64, f64p, f64p,
                                           ctypes.c_int]
    lib.oracle_gemm_sampled_ex.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check(st: int, what: str):
    if st != OK:
        names = {ERR_NAN_SCALE: "E8M0 NaN scale (255)", ERR_NAN_CODE: "E4M3 NaN code",
                 ERR_SHAPE: "bad shape", ERR_NONFINITE: "non-finite activation"}
        raise OracleError(f"{what}: {names.get(st, st)}")


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


# ---------------------------------------------------------------- formats ----

def decode_e8m0(b: int) -> float:
    """2^(b-127); 255 refused (formats.py page, "Formats": E8M0 scale)."""
    out = ctypes.c_double()
    _check(_load().oracle_decode_e8m0(int(b), ctypes.byref(out)), "decode_e8m0")
    return out.value


def decode_fp4(code: int) -> float:
    """E2M1 code -> value (formats.py page, FP4_TABLE; sign bit 3, 8 = -0.0)."""
    return _load().oracle_decode_fp4(int(code))


def decode_e4m3(b: int) -> float:
    """e4m3fn byte -> value; 0x7F/0xFF refused (formats.py page, "Formats")."""
    out = ctypes.c_double()
    _check(_load().oracle_decode_e4m3(int(b), ctypes.byref(out)), "decode_e4m3")
    return out.value


def encode_e4m3(v: float) -> int:
    """binary32 -> E4M3 byte, round to nearest even, saturating at +-448
    (the conversion act_quant applies after its clamp)."""
    return int(_load().oracle_encode_e4m3(float(v)))


def encode_e4m3_array(v: np.ndarray) -> np.ndarray:
    """encode_e4m3 applied element-wise; returns uint8 of v's shape."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_encode_e4m3_n(_ptr(v, ctypes.c_float), v.size, _ptr(out, ctypes.c_uint8))
    return out


def encode_fp4(v: float) -> int:
    """binary32 -> E2M1 code (0..15), round to nearest even, saturating at
    +-6, sign kept (the conversion the MXFP4 activation quantizer applies
    after its clamp)."""
    return int(_load().oracle_encode_fp4(float(v)))


def encode_fp4_array(v: np.ndarray) -> np.ndarray:
    """encode_fp4 applied element-wise; one code per uint8, v's shape."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_encode_fp4_n(_ptr(v, ctypes.c_float), v.size, _ptr(out, ctypes.c_uint8))
    return out


def decode_e5m2(b: int) -> float:
    """E5M2 byte -> value (bias 15, 2 mantissa bits); Inf / NaN codes refused."""
    out = ctypes.c_double()
    _check(_load().oracle_decode_e5m2(int(b), ctypes.byref(out)), "decode_e5m2")
    return out.value


def encode_e5m2(v: float) -> int:
    """binary32 -> E5M2 byte, round to nearest even, saturating at +-57344."""
    return int(_load().oracle_encode_e5m2(float(v)))


def encode_e5m2_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_encode_e5m2_n(_ptr(v, ctypes.c_float), v.size, _ptr(out, ctypes.c_uint8))
    return out


def encode_e5m2_sr(v: float, u: float) -> int:
    """Stochastic E5M2 rounding of v with the uniform draw u in [0, 1): the
    upper neighbour when u < (|v| - lo) / (hi - lo)."""
    return int(_load().oracle_encode_e5m2_sr(float(v), float(u)))


def philox4x64_10(ctr, key):
    """Philox4x64-10 of a 4-word counter under a 2-word key (4 uint64 words)."""
    c = np.ascontiguousarray(ctr, dtype=np.uint64)
    k = np.ascontiguousarray(key, dtype=np.uint64)
    out = np.empty(4, dtype=np.uint64)
    _load().oracle_philox4x64_10(_ptr(c, ctypes.c_uint64), _ptr(k, ctypes.c_uint64),
                                 _ptr(out, ctypes.c_uint64))
    return out


def uniform(seed: int, index: int) -> float:
    """The stochastic-rounding draw of element `index` under `seed`."""
    return _load().oracle_uniform(int(seed), int(index))


def grad_quant(x_bf16_bits: np.ndarray, stochastic=False, seed=0):
    """Per-32 E5M2 gradient quantization along the last dimension ("hip_quant"
    README: "Stochastic E5M2 Backward Gradients", "Block-wise FP8 Scaling"; the
    scale rule of the formats.py page with 57344 in place of 448).
    Returns (q uint8 [M, K] E5M2 codes, sf uint8 [M, K/32] E8M0 bytes)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    sf = np.empty((M, K // 32), dtype=np.uint8)
    if M:
        _check(_load().oracle_grad_quant(_ptr(x, ctypes.c_uint16), M, K, K, int(bool(stochastic)),
                                         int(seed), _ptr(q, ctypes.c_uint8),
                                         _ptr(sf, ctypes.c_uint8)), "grad_quant")
    return q, sf


def quant_transposed(x_bf16_bits: np.ndarray, fmt=Q_E4M3, stochastic=False, seed=0):
    """Quantization along the FIRST dimension of x [R, C] (per 32 rows of a
    column), written transposed: (q uint8 [C, R], sf uint8 [C, R/32]).  fmt
    Q_E4M3 (the act_quant rule) or Q_E5M2 (the gradient rule; its stochastic
    draws use the element's index r * C + c in x)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    R, C = x.shape
    q = np.empty((C, R), dtype=np.uint8)
    sf = np.empty((C, R // 32), dtype=np.uint8)
    if C:
        _check(_load().oracle_quant_transposed(_ptr(x, ctypes.c_uint16), R, C, C, int(fmt),
                                               int(bool(stochastic)), int(seed),
                                               _ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8)),
               "quant_transposed")
    return q, sf


def f32_to_bf16_bits(v: float) -> int:
    return int(_load().oracle_f32_to_bf16(float(v)))


# ---------------------------------------------------------- activations ----

def act_quant(x_bf16_bits: np.ndarray):
    """Per-32 activation quantization (formats.py page: act_scale + act_quant).

    x_bf16_bits: uint16 array [..., K] of bf16 bit patterns.
    Returns (q uint8 [..., K] E4M3 codes, sf uint8 [..., K/32] E8M0 bytes)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    K = x.shape[-1]
    M = x.size // K if K else 0
    q = np.empty(x.shape, dtype=np.uint8)
    sf = np.empty(x.shape[:-1] + (K // 32,), dtype=np.uint8)
    if M:
        _check(_load().oracle_act_quant(_ptr(x, ctypes.c_uint16), M, K, K,
                                        _ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8)),
               "act_quant")
    return q, sf


def act_quant_f32(x: np.ndarray):
    """The same steps on binary32 input [M, K]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    K = x.shape[-1]
    M = x.size // K
    q = np.empty(x.shape, dtype=np.uint8)
    sf = np.empty(x.shape[:-1] + (K // 32,), dtype=np.uint8)
    _check(_load().oracle_act_quant_f32(_ptr(x, ctypes.c_float), M, K,
                                        _ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8)),
           "act_quant_f32")
    return q, sf


def act_quant_fp4(x_bf16_bits: np.ndarray):
    """Per-32 MXFP4 activation quantization: the act_quant steps with the
    E2M1 maximum 6 in place of 448 (the pages define the per-32 rule for
    E4M3 activations and the E2M1 format with E8M0 scales for weights; the
    FP4 x FP4 GEMMs of the "fp4-gemm" page need FP4 activations).

    Returns (q uint8 [..., K/2] packed E2M1, low nibble = even element,
    sf uint8 [..., K/32] E8M0 bytes)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    K = x.shape[-1]
    M = x.size // K if K else 0
    q = np.empty(x.shape[:-1] + (K // 2,), dtype=np.uint8)
    sf = np.empty(x.shape[:-1] + (K // 32,), dtype=np.uint8)
    if M:
        _check(_load().oracle_act_quant_fp4(_ptr(x, ctypes.c_uint16), M, K, K,
                                            _ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8)),
               "act_quant_fp4")
    return q, sf


def act_quant_fp4_f32(x: np.ndarray):
    """The MXFP4 steps on binary32 input [M, K]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    K = x.shape[-1]
    M = x.size // K
    q = np.empty(x.shape[:-1] + (K // 2,), dtype=np.uint8)
    sf = np.empty(x.shape[:-1] + (K // 32,), dtype=np.uint8)
    _check(_load().oracle_act_quant_fp4_f32(_ptr(x, ctypes.c_float), M, K,
                                            _ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8)),
           "act_quant_fp4_f32")
    return q, sf


def e4m3_ceil(t: float) -> int:
    """The smallest positive E4M3 value >= t, as its byte (the NVFP4 block
    scale): 0x01 (2^-9) at or below it, 0x7E (448) above 448."""
    return int(_load().oracle_e4m3_ceil(float(t)))


def act_quant_nvfp4(x_bf16_bits: np.ndarray, g: float = 1.0):
    """NVFP4 quantization: every value first fp32(x * g) (g the per-tensor
    scale), then per 16 consecutive values an E4M3 scale s = the smallest E4M3
    value >= fp32(amax * fp32(1/6)) and E2M1 codes of fp32(x / s) (round to
    nearest even, sign kept).  Returns (q uint8 [M, K/2] packed, low nibble
    first, sf uint8 [M, K/16] E4M3 bytes)."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K // 2), dtype=np.uint8)
    sf = np.empty((M, K // 16), dtype=np.uint8)
    if M:
        _check(_load().oracle_act_quant_nvfp4(_ptr(x, ctypes.c_uint16), M, K, K, float(g),
                                              _ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8)),
               "act_quant_nvfp4")
    return q, sf


def unpack_fp4(q: np.ndarray) -> np.ndarray:
    """Packed E2M1 bytes [..., K/2] -> one code per byte [..., K] (low nibble
    first)."""
    q = np.asarray(q, dtype=np.uint8)
    out = np.empty(q.shape[:-1] + (2 * q.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = q & 0x0F
    out[..., 1::2] = q >> 4
    return out


def act_qdq(q: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """bf16 bits of fp32(q) * s (formats.py page: act_qdq)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    K = q.shape[-1]
    M = q.size // K
    y = np.empty(q.shape, dtype=np.uint16)
    _check(_load().oracle_act_qdq(_ptr(q, ctypes.c_uint8), _ptr(sf, ctypes.c_uint8), M, K,
                                  _ptr(y, ctypes.c_uint16)), "act_qdq")
    return y


# ----------------------------------------------------------------- GEMM ----

def gemm(aq, asf, b, bsf, bkind, M, N, K, bias=None, residual=None, alpha=1.0,
         act=ACT_NONE, nthreads=None, a_kind=A_E4M3):
    """Exact-decode fp64 GEMM with the fused epilogue.

    ref[m, n] = act(alpha * sum_k a[m,k] b[n,k] + bias[n]) + residual[m, n] and
    sumabs[m, n] = sum_k |a[m,k] b[n,k]|, where a and b are the exactly decoded
    operands (formats.py page: decode_fp4, decode_fp8_block, e8m0_to_f32).
    a_kind: A_E4M3 (aq [M, K]), A_FP4 (aq [M, K/2] packed E2M1), A_E5M2
    (aq [M, K] E5M2 gradient codes) or A_NVFP4 (aq [M, K/2] packed E2M1 with
    E4M3 scales asf [M, K/16]); bkind B_NVFP4 likewise for b."""
    aq = np.ascontiguousarray(aq, dtype=np.uint8)
    asf = np.ascontiguousarray(asf, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    bsf = np.ascontiguousarray(bsf, dtype=np.uint8)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
    residual = None if residual is None else np.ascontiguousarray(residual, dtype=np.uint16)
    ref = np.empty((M, N), dtype=np.float64)
    sumabs = np.empty((M, N), dtype=np.float64)
    if M and N:
        _check(_load().oracle_gemm_ex(
            _ptr(aq, ctypes.c_uint8), _ptr(asf, ctypes.c_uint8), int(a_kind),
            _ptr(b, ctypes.c_uint8), _ptr(bsf, ctypes.c_uint8), int(bkind), M, N, K,
            _ptr(bias, ctypes.c_uint16),
            _ptr(residual, ctypes.c_uint16), N, float(alpha), int(act),
            _ptr(ref, ctypes.c_double), _ptr(sumabs, ctypes.c_double),
            int(nthreads or default_threads())), "gemm")
    return ref, sumabs


def gemm_sampled(aq, asf, b, bsf, bkind, M, N, K, ms, ns, bias=None, residual=None,
                 alpha=1.0, act=ACT_NONE, nthreads=None, a_kind=A_E4M3):
    """The same per-element definition at the (ms[i], ns[i]) pairs only."""
    aq = np.ascontiguousarray(aq, dtype=np.uint8)
    asf = np.ascontiguousarray(asf, dtype=np.uint8)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    bsf = np.ascontiguousarray(bsf, dtype=np.uint8)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
    residual = None if residual is None else np.ascontiguousarray(residual, dtype=np.uint16)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    ref = np.empty(ms.size, dtype=np.float64)
    sumabs = np.empty(ms.size, dtype=np.float64)
    if ms.size:
        _check(_load().oracle_gemm_sampled_ex(
            _ptr(aq, ctypes.c_uint8), _ptr(asf, ctypes.c_uint8), int(a_kind),
            _ptr(b, ctypes.c_uint8), _ptr(bsf, ctypes.c_uint8), int(bkind), M, N, K,
            _ptr(bias, ctypes.c_uint16),
            _ptr(residual, ctypes.c_uint16), N, float(alpha), int(act),
            _ptr(ms, ctypes.c_int64), _ptr(ns, ctypes.c_int64), ms.size,
            _ptr(ref, ctypes.c_double), _ptr(sumabs, ctypes.c_double),
            int(nthreads or default_threads())), "gemm_sampled")
    return ref, sumabs


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """One bf16 ulp at |x|: 2^(floor(log2|x|) - 7) for normal |x|, and the
    subnormal spacing 2^-133 at or below the smallest normal."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(ax)  # ax = f * 2^e with f in [0.5, 1)
    ulp = np.ldexp(1.0, (e - 1) - 7)
    return np.where(ax < 2.0 ** -126, 2.0 ** -133, ulp)


def gemm_tolerance(ref, sumabs, alpha=1.0, bias_abs=None, res_abs=None, act=ACT_NONE):
    """Per-element bound |y - ref| <= ulp_bf16(|ref|) + 2^-20 * S, with
    S = |alpha| sum_k |a b| (+ |bias| + |residual|), the GELU branch scaled by
    its largest slope 1.13."""
    s = abs(alpha) * np.asarray(sumabs, dtype=np.float64)
    if bias_abs is not None:
        s = s + bias_abs
    if act == ACT_GELU:
        s = 1.13 * s
    if res_abs is not None:
        s = s + res_abs
    return bf16_ulp(ref) + 2.0 ** -20 * s
