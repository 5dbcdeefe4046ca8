"""Pins for the oracle's block-scaled GEMM and epilogue.

The oracle is checked against (a) exact rational brute force on tiny inputs,
decoding the operands with the page's printed FP4 table and torch's E4M3
conversion, (b) special cases that reduce to a known product or to a plain
fp64 matmul, and (c) the QDQ invariant of the "formats.py" page: a GEMM over
act_qdq'd bf16 activations and exactly decoded weights forms the same products
as the GEMM over the codes.
"""
from fractions import Fraction
import math

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_quant_b200 import synth
from conftest import read_golden

FP4 = {int(c): Fraction(float(v)) for c, v in read_golden("fp4_table.txt")}
E4M3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).numpy()


def e8(b):
    return Fraction(2) ** (int(b) - 127)


def frac_a(aq, asf):
    M, K = aq.shape
    return [[Fraction(float(E4M3[aq[m, k]])) * e8(asf[m, k // 32]) for k in range(K)]
            for m in range(M)]


def frac_b(b, bsf, kind, N, K):
    out = []
    for n in range(N):
        row = []
        for k in range(K):
            if kind == oracle.B_FP4:
                byte = int(b[n, k // 2])
                code = byte & 0xF if k % 2 == 0 else byte >> 4  # low nibble = even input
                row.append(FP4[code] * e8(bsf[n, k // 32]))
            elif kind == oracle.B_FP8BLK:
                row.append(Fraction(float(E4M3[b[n, k]])) * e8(bsf[n // 32, k // 32]))
            else:
                row.append(Fraction(float(E4M3[b[n, k]])) * e8(bsf[n, k // 32]))
        out.append(row)
    return out


def bf16v(bits):
    return float((np.uint32(bits) << np.uint32(16)).view(np.float32))


def make_operands(rng, M, N, K, kind, lo=123, hi=127):
    """Random finite codes; scale bytes U{lo..hi}.  With the default span the
    products' exponents (codes 2^-9..2^8.8 each, scales 2^4 each) plus log2 K
    stay under 53 bits, so fp64 sums are exact."""
    aq = rng.choice([c for c in range(256) if (c & 0x7F) != 0x7F], size=(M, K)).astype(np.uint8)
    asf = rng.integers(lo, hi + 1, size=(M, K // 32)).astype(np.uint8)
    if kind == oracle.B_FP4:
        b = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
        bsf = rng.integers(lo, hi + 1, size=(N, K // 32)).astype(np.uint8)
    elif kind == oracle.B_FP8BLK:
        b = rng.choice([c for c in range(256) if (c & 0x7F) != 0x7F], size=(N, K)).astype(np.uint8)
        bsf = rng.integers(lo, hi + 1, size=((N + 31) // 32, (K + 31) // 32)).astype(np.uint8)
    else:
        b = rng.choice([c for c in range(256) if (c & 0x7F) != 0x7F], size=(N, K)).astype(np.uint8)
        bsf = rng.integers(lo, hi + 1, size=(N, K // 32)).astype(np.uint8)
    return aq, asf, b, bsf


@pytest.mark.parametrize("kind", [oracle.B_FP4, oracle.B_FP8BLK, oracle.B_FP8ROW])
@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (3, 5, 64), (8, 7, 96), (2, 40, 64)])
def test_brute_force_exact(kind, M, N, K):
    """Dyadic products whose exponents span well under 53 bits sum exactly in
    fp64, so the oracle must equal the exact rational result bit for bit."""
    rng = np.random.default_rng(100 * M + 10 * N + K + kind)
    aq, asf, b, bsf = make_operands(rng, M, N, K, kind)
    ref, sabs = oracle.gemm(aq, asf, b, bsf, kind, M, N, K, nthreads=2)
    A = frac_a(aq, asf)
    B = frac_b(b, bsf, kind, N, K)
    for m in range(M):
        for n in range(N):
            exact = sum(A[m][k] * B[n][k] for k in range(K))
            exact_abs = sum(abs(A[m][k] * B[n][k]) for k in range(K))
            assert ref[m, n] == float(exact), (m, n)
            assert sabs[m, n] == float(exact_abs)


@pytest.mark.parametrize("kind", [oracle.B_FP4, oracle.B_FP8BLK])
def test_brute_force_epilogue(kind):
    """bias, alpha, residual and erf-GELU against exact sums plus math.erf."""
    M, N, K = 4, 6, 64
    rng = np.random.default_rng(5 + kind)
    aq, asf, b, bsf = make_operands(rng, M, N, K, kind)
    asf[:] = rng.integers(120, 128, size=asf.shape)
    bsf[:] = rng.integers(120, 128, size=bsf.shape)
    bias = synth.bias(N, seed=3, std=0.5)
    res = synth.residual(M, N, seed=4)
    A = frac_a(aq, asf)
    B = frac_b(b, bsf, kind, N, K)
    for act in (oracle.ACT_NONE, oracle.ACT_GELU):
        ref, _ = oracle.gemm(aq, asf, b, bsf, kind, M, N, K, bias=bias, residual=res,
                             alpha=0.75, act=act, nthreads=1)
        for m in range(M):
            for n in range(N):
                acc = sum(A[m][k] * B[n][k] for k in range(K))
                t = Fraction(3, 4) * acc + Fraction(bf16v(bias[n]))
                if act == oracle.ACT_NONE:
                    want = float(t + Fraction(bf16v(res[m, n])))
                    assert ref[m, n] == want
                else:
                    tf = float(t)
                    want = 0.5 * tf * (1.0 + math.erf(tf / math.sqrt(2.0))) + bf16v(res[m, n])
                    assert abs(ref[m, n] - want) <= 1e-12 * (abs(want) + 1.0)


def test_single_nonzero_weight_selects_a_column():
    """A weight row holding one nonzero code c at input j with scale 2^e gives
    Y[:, n] = a[:, j] * c * 2^e exactly, and a transposed or mis-indexed
    operand could not."""
    M, N, K = 5, 64, 128
    rng = np.random.default_rng(9)
    aq, asf, _, _ = make_operands(rng, M, N, K, oracle.B_FP8ROW)
    b = np.zeros((N, K), dtype=np.uint8)
    bsf = np.full((N, K // 32), 127, dtype=np.uint8)
    picks = rng.integers(0, K, size=N)
    for n in range(N):
        b[n, picks[n]] = 0x40 + (n % 24)  # positive normal codes
        bsf[n, picks[n] // 32] = 120 + n % 9
    ref, _ = oracle.gemm(aq, asf, b, bsf, oracle.B_FP8ROW, M, N, K)
    A = frac_a(aq, asf)
    for n in range(N):
        w = Fraction(float(E4M3[b[n, picks[n]]])) * e8(bsf[n, picks[n] // 32])
        for m in range(M):
            assert ref[m, n] == float(A[m][picks[n]] * w)
    # FP4: nibble j of byte j//2 -- low nibble for even j
    b4 = np.zeros((N, K // 2), dtype=np.uint8)
    s4 = np.full((N, K // 32), 127, dtype=np.uint8)
    for n in range(N):
        j = picks[n]
        b4[n, j // 2] = 0x07 if j % 2 == 0 else 0x70  # code 7 = 6.0
    ref4, _ = oracle.gemm(aq, asf, b4, s4, oracle.B_FP4, M, N, K)
    for n in range(N):
        for m in range(M):
            assert ref4[m, n] == float(A[m][picks[n]] * 6)


def test_unit_scales_reduce_to_plain_matmul():
    """With every scale byte 127 (= 1.0) the GEMM is a plain matmul of the
    decoded codes: torch.matmul in fp64 over torch's E4M3 decode and the
    printed FP4 table."""
    M, N, K = 33, 47, 256
    rng = np.random.default_rng(21)
    aq, _, b8, _ = make_operands(rng, M, N, K, oracle.B_FP8ROW)
    ones_a = np.full((M, K // 32), 127, dtype=np.uint8)
    A = torch.from_numpy(E4M3[aq])
    ref, _ = oracle.gemm(aq, ones_a, b8, np.full((N, K // 32), 127, np.uint8),
                         oracle.B_FP8ROW, M, N, K)
    want = A @ torch.from_numpy(E4M3[b8]).T
    assert np.allclose(ref, want.numpy(), rtol=1e-15, atol=0)
    refb, _ = oracle.gemm(aq, ones_a, b8, np.full(((N + 31) // 32, K // 32), 127, np.uint8),
                          oracle.B_FP8BLK, M, N, K)
    assert np.array_equal(refb, ref)
    b4 = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
    lut = np.array([float(FP4[c]) for c in range(16)])
    codes = np.stack([b4 & 0xF, b4 >> 4], axis=-1).reshape(N, K)
    ref4, _ = oracle.gemm(aq, ones_a, b4, np.full((N, K // 32), 127, np.uint8),
                          oracle.B_FP4, M, N, K)
    want4 = A @ torch.from_numpy(lut[codes]).T
    assert np.allclose(ref4, want4.numpy(), rtol=1e-15, atol=0)


def test_block_scale_index_is_row_block_by_col_block():
    """FP8 32x32 blocks: scale [n // 32, k // 32].  Scaling one block by 2
    doubles exactly the contributions of rows n in that block and inputs k
    in that block."""
    M, N, K = 3, 96, 128
    rng = np.random.default_rng(2)
    aq, asf, b, bsf = make_operands(rng, M, N, K, oracle.B_FP8BLK)
    bsf[:] = 127
    base, _ = oracle.gemm(aq, asf, b, bsf, oracle.B_FP8BLK, M, N, K)
    bsf2 = bsf.copy()
    bsf2[2, 1] = 128  # rows 64..95, inputs 32..63
    bumped, _ = oracle.gemm(aq, asf, b, bsf2, oracle.B_FP8BLK, M, N, K)
    A = frac_a(aq, asf)
    B = frac_b(b, bsf, oracle.B_FP8BLK, N, K)
    for n in range(N):
        for m in range(M):
            extra = sum(A[m][k] * B[n][k] for k in range(32, 64)) if 64 <= n < 96 else 0
            assert bumped[m, n] == float(Fraction(base[m, n]) + extra) or \
                abs(bumped[m, n] - float(Fraction(base[m, n]) + extra)) <= 1e-15 * abs(bumped[m, n])


def test_bias_only():
    M, N, K = 4, 16, 32
    aq = np.zeros((M, K), np.uint8)
    asf = np.full((M, 1), 127, np.uint8)
    b = np.zeros((N, K // 2), np.uint8)
    bsf = np.full((N, 1), 127, np.uint8)
    bias = synth.bias(N, seed=1)
    ref, sabs = oracle.gemm(aq, asf, b, bsf, oracle.B_FP4, M, N, K, bias=bias)
    for n in range(N):
        assert np.all(ref[:, n] == bf16v(bias[n]))
    assert np.all(sabs == 0)


def test_qdq_invariant_gemm_over_bf16_activations():
    """formats.py page, docstring: a GEMM over the QDQ'd bf16 activations and
    exactly decoded weights forms the same products as the GEMM over codes.
    The bf16 side is evaluated with torch.matmul in fp64."""
    M, N, K = 12, 40, 256
    x = synth.activations(M, K, seed=4, group_pow2=(-4, 4))
    q, sf = oracle.act_quant(x)
    y = oracle.act_qdq(q, sf)
    yv = torch.from_numpy((y.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    b4, s4 = synth.mxfp4_weight(N, K, seed=8)
    codes = np.stack([b4 & 0xF, b4 >> 4], axis=-1).reshape(N, K)
    lut = np.array([float(FP4[c]) for c in range(16)])
    W = lut[codes] * np.ldexp(1.0, s4.astype(np.int64) - 127).repeat(32, axis=1)
    want = (yv @ torch.from_numpy(W).T).numpy()
    ref, _ = oracle.gemm(q, sf, b4, s4, oracle.B_FP4, M, N, K)
    assert np.allclose(ref, want, rtol=1e-14, atol=1e-300)


def test_refuses_nan_scale_and_nan_code():
    M, N, K = 2, 3, 32
    aq = np.zeros((M, K), np.uint8)
    asf = np.full((M, 1), 127, np.uint8)
    b = np.zeros((N, K), np.uint8)
    bsf = np.full((1, 1), 127, np.uint8)
    bad = bsf.copy()
    bad[0, 0] = 255
    with pytest.raises(oracle.OracleError):
        oracle.gemm(aq, asf, b, bad, oracle.B_FP8BLK, M, N, K)
    b2 = b.copy()
    b2[1, 7] = 0x7F
    with pytest.raises(oracle.OracleError):
        oracle.gemm(aq, asf, b2, bsf, oracle.B_FP8BLK, M, N, K)


def test_sampled_equals_full():
    M, N, K = 20, 70, 160
    rng = np.random.default_rng(31)
    aq, asf, b, bsf = make_operands(rng, M, N, K, oracle.B_FP8BLK)
    bias = synth.bias(N, seed=2)
    res = synth.residual(M, N, seed=3)
    ref, sabs = oracle.gemm(aq, asf, b, bsf, oracle.B_FP8BLK, M, N, K, bias=bias, residual=res,
                            act=oracle.ACT_GELU)
    ms = rng.integers(0, M, 50)
    ns = rng.integers(0, N, 50)
    r2, s2 = oracle.gemm_sampled(aq, asf, b, bsf, oracle.B_FP8BLK, M, N, K, ms, ns, bias=bias,
                                 residual=res, act=oracle.ACT_GELU)
    assert np.array_equal(r2, ref[ms, ns]) and np.array_equal(s2, sabs[ms, ns])


def test_tolerance_helper():
    ulp = oracle.bf16_ulp(np.array([1.0, 1.5, 2.0, 0.0, 3e-39, -256.0]))
    assert ulp.tolist() == [2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -133, 2.0 ** -133, 2.0]
