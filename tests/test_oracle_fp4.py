"""Pins for the oracle's MXFP4 activation path (E2M1 codes, E8M0 per 32) and
its FP4 x FP4 GEMM decode.

The pages define the per-32 scale rule for E4M3 activations ("formats.py"
page: act_scale, act_quant) and the E2M1 format with E8M0 scales (FP4_TABLE,
fp4_codes); the A4W4 GEMMs of the "fp4-gemm" page (README "Available
Functions", "Tensor Contract") take packed E2M1 activations.  The oracle's
FP4 quantizer is that rule with 6 in place of 448.  It is pinned here by
(a) brute force over the printed FP4 table for the encoder, (b) hand-worked
scales and a hand-worked group, (c) a second restatement of the rule in numpy
that must agree bit for bit, (d) invariants of the ceil rule, and (e) exact
rational brute force and a plain-matmul special case for the GEMM.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_quant_b200 import synth
from conftest import parse_float, parse_int, read_golden

TABLE = {int(c): float(v) for c, v in read_golden("fp4_table.txt")}
MAG = np.array([TABLE[c] for c in range(8)])  # codes 0..7, increasing
E4M3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).numpy()


def brute_encode(v):
    """Nearest E2M1 code by exhaustive distance to the printed table's
    magnitudes; ties to the even code; saturate at 6; sign bit from v."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), 6.0)
    d = np.abs(a[..., None] - MAG)                      # [..., 8]
    best = d.min(axis=-1, keepdims=True)
    cand = d == best                                    # one or two (a tie) candidates
    even = cand & (np.arange(8) % 2 == 0)
    code = np.where(even.any(axis=-1), even.argmax(axis=-1), cand.argmax(axis=-1))
    return (code | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def test_decode_table_is_the_printed_one():
    for c in range(16):
        assert oracle.decode_fp4(c) == TABLE[c]
        assert np.signbit(oracle.decode_fp4(c)) == (c >= 8)


def test_encoder_midpoints_and_saturation():
    # every grid point, every midpoint (the ties), and points just off them
    grid = np.concatenate([MAG, (MAG[1:] + MAG[:-1]) / 2])
    vals = np.concatenate([grid, np.nextafter(grid, 10), np.nextafter(grid, -10),
                           [6.5, 7.0, 1e30, np.float32(3.4e38)]])
    vals = np.concatenate([vals, -vals]).astype(np.float32)
    assert np.array_equal(oracle.encode_fp4_array(vals), brute_encode(vals))
    # the ties, by hand: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    hand = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 7.0: 7, -0.25: 8,
            -0.1: 8, -5.0: 14}
    for v, c in hand.items():
        assert oracle.encode_fp4(v) == c, v


def test_encoder_all_bf16_values():
    """Every finite bf16 bit pattern (the scaled inputs the quantizer meets are
    bf16 values times a power of two) against the brute force."""
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)]
    for scale in (1.0, 2.0 ** -3, 2.0 ** 5):
        with np.errstate(over="ignore"):
            v = (f * np.float32(scale)).astype(np.float32)
        v = v[np.isfinite(v)]
        assert np.array_equal(oracle.encode_fp4_array(v), brute_encode(v))


@pytest.mark.parametrize("row", read_golden("act_scale_fp4_worked.txt"))
def test_hand_worked_scales(row):
    amax, byte = parse_float(row[0]), int(row[1])
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 5] = amax
    x[0, 9] = -amax / 2
    _, sf = oracle.act_quant_fp4_f32(x)
    assert sf[0, 0] == byte


def test_hand_worked_group():
    rows = read_golden("act_quant_fp4_worked_group.txt")
    x = np.zeros((1, 32), dtype=np.uint16)
    codes = {}
    packed = scale = None
    for r in rows:
        if r[0] == "PACKED":
            packed = [parse_int(t) for t in r[1:]]
        elif r[0] == "SCALE":
            scale = int(r[1])
        else:
            x[0, int(r[0])] = parse_int(r[1])
            codes[int(r[0])] = int(r[2])
    q, sf = oracle.act_quant_fp4(x)
    assert sf[0, 0] == scale
    assert list(q[0, :4]) == packed
    assert np.all(q[0, 4:] == 0)
    unpacked = oracle.unpack_fp4(q)[0]
    for i, c in codes.items():
        assert unpacked[i] == c


def restated_quant(xf):
    """The MXFP4 rule restated in numpy, step by step: amax with the 1e-4
    floor, t = fp32(amax * fp32(1/6)), e = ceil(log2 t) via frexp, q the
    brute-force nearest code of clamp(x / 2^e, +-6)."""
    M, K = xf.shape
    g = xf.reshape(M, K // 32, 32)
    amax = np.maximum(np.abs(g).max(axis=-1), np.float32(1e-4)).astype(np.float32)
    t = (amax * np.float32(1.0 / 6.0)).astype(np.float32)
    mant, ex = np.frexp(t.astype(np.float64))  # t = mant * 2^ex, mant in [0.5, 1)
    e = np.where(mant == 0.5, ex - 1, ex)
    y = np.clip(g.astype(np.float64) / np.ldexp(1.0, e)[..., None], -6.0, 6.0)
    codes = brute_encode(y).reshape(M, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, (e + 127).astype(np.uint8)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_restatement_agrees(seed):
    x = synth.activations(64, 1024, seed=seed, group_pow2=(-12, 12))
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    q, sf = oracle.act_quant_fp4(x)
    q2, sf2 = restated_quant(xf)
    assert np.array_equal(sf, sf2)
    assert np.array_equal(q, q2)


def test_ceil_rule_invariants():
    x = synth.activations(128, 2048, seed=7, group_pow2=(-8, 8))
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    q, sf = oracle.act_quant_fp4(x)
    s = np.ldexp(1.0, sf.astype(np.int64) - 127)
    g = xf.reshape(128, -1, 32)
    r = np.abs(g).max(axis=-1) / s
    assert np.all((r > 3.0) & (r <= 6.0))          # the group maximum lands in (3, 6]
    codes = oracle.unpack_fp4(q).reshape(128, -1, 32)
    vals = np.vectorize(TABLE.get)(codes)
    y = g / s[..., None]
    half_gap = np.where(np.abs(y) <= 2.0, 0.25, np.where(np.abs(y) <= 4.0, 0.5, 1.0))
    assert np.all(np.abs(y - vals) <= half_gap)    # round to nearest on the E2M1 grid
    top = np.take_along_axis(codes & 7, np.abs(g).argmax(axis=-1)[..., None], axis=-1)
    assert np.all(np.isin(top, [5, 6, 7]))         # 3, 4 or 6


def test_nonfinite_refused():
    x = np.zeros((1, 32), dtype=np.uint16)
    x[0, 3] = 0x7FC0
    with pytest.raises(oracle.OracleError):
        oracle.act_quant_fp4(x)


# ------------------------------------------------------------------ GEMM ----

def e8(b):
    return Fraction(2) ** (int(b) - 127)


def frac_fp4_rows(q, sf):
    rows, kh = q.shape
    out = []
    for r in range(rows):
        row = []
        for k in range(2 * kh):
            byte = int(q[r, k // 2])
            code = byte & 0xF if k % 2 == 0 else byte >> 4
            row.append(Fraction(TABLE[code]) * e8(sf[r, k // 32]))
        out.append(row)
    return out


def frac_b(b, bsf, kind, N, K):
    if kind == oracle.B_FP4:
        return frac_fp4_rows(b, bsf)
    out = []
    for n in range(N):
        if kind == oracle.B_FP8BLK:
            out.append([Fraction(float(E4M3[b[n, k]])) * e8(bsf[n // 32, k // 32])
                        for k in range(K)])
        else:
            out.append([Fraction(float(E4M3[b[n, k]])) * e8(bsf[n, k // 32]) for k in range(K)])
    return out


@pytest.mark.parametrize("kind", [oracle.B_FP4, oracle.B_FP8BLK, oracle.B_FP8ROW])
@pytest.mark.parametrize("M,N,K", [(1, 1, 32), (3, 5, 64), (8, 7, 96)])
def test_fp4_activation_gemm_brute_force(kind, M, N, K):
    rng = np.random.default_rng(1000 + 100 * M + N + K + kind)
    aq = rng.integers(0, 256, size=(M, K // 2)).astype(np.uint8)
    asf = rng.integers(120, 128, size=(M, K // 32)).astype(np.uint8)
    if kind == oracle.B_FP4:
        b = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
        bsf = rng.integers(120, 128, size=(N, K // 32)).astype(np.uint8)
    else:
        b = rng.choice([c for c in range(256) if (c & 0x7F) != 0x7F],
                       size=(N, K)).astype(np.uint8)
        shape = ((N + 31) // 32, (K + 31) // 32) if kind == oracle.B_FP8BLK else (N, K // 32)
        bsf = rng.integers(120, 128, size=shape).astype(np.uint8)
    ref, sabs = oracle.gemm(aq, asf, b, bsf, kind, M, N, K, a_kind=oracle.A_FP4)
    A = frac_fp4_rows(aq, asf)
    B = frac_b(b, bsf, kind, N, K)
    for m in range(M):
        for n in range(N):
            exact = sum(A[m][k] * B[n][k] for k in range(K))
            assert ref[m, n] == float(exact)
            assert sabs[m, n] == float(sum(abs(A[m][k] * B[n][k]) for k in range(K)))


def test_fp4_gemm_unit_scales_is_plain_matmul():
    """All scale bytes 127 (2^0): the GEMM is the fp64 matmul of the decoded
    codes."""
    rng = np.random.default_rng(5)
    M, N, K = 17, 23, 256
    aq = rng.integers(0, 256, size=(M, K // 2)).astype(np.uint8)
    b = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
    ones_a = np.full((M, K // 32), 127, np.uint8)
    ones_b = np.full((N, K // 32), 127, np.uint8)
    ref, _ = oracle.gemm(aq, ones_a, b, ones_b, oracle.B_FP4, M, N, K, a_kind=oracle.A_FP4)
    dec = np.vectorize(TABLE.get)
    A = dec(oracle.unpack_fp4(aq)).astype(np.float64)
    B = dec(oracle.unpack_fp4(b)).astype(np.float64)
    assert np.array_equal(ref, (torch.from_numpy(A) @ torch.from_numpy(B).T).numpy())


def test_fp4_gemm_sampled_matches_full():
    rng = np.random.default_rng(9)
    M, N, K = 40, 33, 128
    x = synth.activations(M, K, seed=3)
    aq, asf = oracle.act_quant_fp4(x)
    b, bsf = synth.mxfp4_weight(N, K, seed=4)
    ref, sabs = oracle.gemm(aq, asf, b, bsf, oracle.B_FP4, M, N, K, a_kind=oracle.A_FP4)
    ms = rng.integers(0, M, 50)
    ns = rng.integers(0, N, 50)
    r2, s2 = oracle.gemm_sampled(aq, asf, b, bsf, oracle.B_FP4, M, N, K, ms, ns,
                                 a_kind=oracle.A_FP4)
    assert np.array_equal(r2, ref[ms, ns])
    assert np.array_equal(s2, sabs[ms, ns])
