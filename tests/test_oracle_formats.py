"""Pins for the oracle's number formats and activation quantizer.

Each check ties the oracle to something other than itself: the values the
"formats.py" page prints (fixtures under tests/golden), the library conversion
the page's own definition calls (torch.float8_e4m3fn), hand-worked cases, and
mathematical properties of the definition (power-of-two ceiling, exactness).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_quant_b200 import synth
from conftest import parse_float, parse_int, read_golden


def facts():
    return {r[0]: parse_int(r[1]) for r in read_golden("format_facts.txt")}


# ------------------------------------------------------------------ FP4 ----

def test_fp4_matches_printed_table():
    rows = read_golden("fp4_table.txt")
    assert len(rows) == 16
    for code_s, val_s in rows:
        code, val = int(code_s), float(val_s)
        got = oracle.decode_fp4(code)
        assert got == val, (code, got, val)
        assert math.copysign(1.0, got) == math.copysign(1.0, val), code  # -0.0 at code 8


# ----------------------------------------------------------------- E8M0 ----

def test_e8m0_is_power_of_two_and_refuses_255():
    for b in range(255):
        assert oracle.decode_e8m0(b) == math.ldexp(1.0, b - 127)
    assert oracle.decode_e8m0(facts()["E8M0_ONE"]) == 1.0
    assert oracle.decode_e8m0(0) == 2.0 ** -127  # an fp32 subnormal, still exact
    with pytest.raises(oracle.OracleError):
        oracle.decode_e8m0(facts()["E8M0_NAN"])


# ----------------------------------------------------------------- E4M3 ----

def test_e4m3_decode_matches_torch_e4m3fn_on_all_finite_codes():
    f = facts()
    nan_codes = {f["E4M3_NAN_POS"], f["E4M3_NAN_NEG"]}
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib_vals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        if c in nan_codes:
            assert math.isnan(lib_vals[c])
            with pytest.raises(oracle.OracleError):
                oracle.decode_e4m3(c)
            continue
        got = oracle.decode_e4m3(c)
        assert got == lib_vals[c], (hex(c), got, lib_vals[c])
        assert math.copysign(1.0, got) == math.copysign(1.0, lib_vals[c])
    assert oracle.decode_e4m3(f["E4M3_MAX_CODE"]) == f["FP8_MAX"]
    assert oracle.decode_e4m3(f["E4M3_BIAS"] << 3) == 1.0  # exponent field = bias -> 2^0


def test_decoded_values_exact_in_fp32_below_overflow():
    """Every decoded value code * 2^(b-127) is exact in binary32 (formats.py
    page, docstring "Formats": <= 4 significant bits times a power of two) for
    every scale byte up to the point where the product overflows binary32:
    E4M3 (max 448 = 1.75 * 2^8) for b <= 246, FP4 (max 6 = 1.5 * 2^2) for b <= 252."""
    e4m3 = np.array([oracle.decode_e4m3(c) for c in range(256) if (c & 0x7F) != 0x7F])
    fp4 = np.array([oracle.decode_fp4(c) for c in range(16)])
    for vals, last_ok in ((e4m3, 246), (fp4, 252)):
        for b in range(255):
            s = oracle.decode_e8m0(b)
            exact = vals * s  # fp64: exact (<= 4 significant bits)
            f32 = vals.astype(np.float32) * np.float32(s)
            if b <= last_ok:
                assert np.array_equal(f32.astype(np.float64), exact), b
            else:
                assert not np.all(np.isfinite(f32)), b


# -------------------------------------------------------------- encoder ----

def test_encoder_tie_cases():
    for v_s, code_s in read_golden("e4m3_rne_ties.txt"):
        assert oracle.encode_e4m3(parse_float(v_s)) == parse_int(code_s), v_s


def test_encoder_matches_torch_on_every_bf16_value_and_scale():
    """All 65536 bf16 patterns x, divided by every power-of-two scale 2^e the
    quantizer can pick (e in [-22, 120]), clamped to +-448 and converted: the
    oracle's encoder against torch's float8_e4m3fn conversion, the conversion
    the page's act_quant calls."""
    bits = np.arange(65536, dtype=np.uint32)
    x = (bits << 16).view(np.float32)
    x = x[np.isfinite(x)]
    for e in range(-22, 121):
        y = torch.from_numpy(x) / torch.tensor(2.0 ** e, dtype=torch.float32)
        y = y.clamp(-448.0, 448.0)
        want = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        got = oracle.encode_e4m3_array(y.numpy())
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (e, x[bad[:5]], got[bad[:5]], want[bad[:5]])


# ----------------------------------------------------------- act_quant ----

def test_scale_hand_worked_table():
    rows = read_golden("act_scale_worked.txt")
    for amax_s, byte_s in rows:
        amax = parse_float(amax_s)
        x = np.zeros((1, 32), dtype=np.float32)
        x[0, 5] = amax
        x[0, 9] = -amax / 2
        _, sf = oracle.act_quant_f32(x)
        assert int(sf[0, 0]) == int(byte_s), (amax_s, int(sf[0, 0]), byte_s)
        _, sf_neg = oracle.act_quant_f32(-x)  # amax is of |x|
        assert int(sf_neg[0, 0]) == int(byte_s)


def test_worked_group():
    rows = read_golden("act_quant_worked_group.txt")
    scale = [r for r in rows if r[0] == "SCALE"][0]
    vals = [r for r in rows if r[0] != "SCALE"]
    x = np.zeros((1, 64), dtype=np.uint16)
    for idx, xh, _, _ in vals:
        x[0, int(idx)] = parse_int(xh)
        x[0, 32 + int(idx)] = parse_int(xh)  # the same group again in the second block
    q, sf = oracle.act_quant(x)
    assert sf.tolist() == [[int(scale[1]), int(scale[1])]]
    qdq = oracle.act_qdq(q, sf)
    qdq_f = (qdq.astype(np.uint32) << 16).view(np.float32)
    for idx, _, code, v in vals:
        for base in (0, 32):
            assert int(q[0, base + int(idx)]) == parse_int(code)
            assert float(qdq_f[0, base + int(idx)]) == float(v)
    assert np.all(q[0, 4:32] == 0)


def _scale_properties(x_f32, q, sf):
    """Properties the definition fixes for every group:
    - s = 2^(b-127) is the smallest power of two >= t, t = fp32(amax * fp32(1/448)),
      amax = max(max|x|, fp32(1e-4)); checked by comparison, not exponent bits;
    - q = E4M3(clamp(x / s)) through torch's float8_e4m3fn conversion;
    - the largest |q| of a group whose amax is above the floor lies in [224, 448]."""
    M, K = x_f32.shape
    g = x_f32.reshape(M, K // 32, 32)
    amax = np.maximum(np.abs(g).max(-1), np.float32(1e-4)).astype(np.float32)
    t = (amax * np.float32(1.0 / 448.0)).astype(np.float32).astype(np.float64)
    s = np.ldexp(1.0, sf.astype(np.int64) - 127)
    assert np.all(t <= s) and np.all(t > s / 2)
    y = torch.from_numpy(g) / torch.from_numpy(s.astype(np.float32))[..., None]
    want = y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy().reshape(M, K)
    assert np.array_equal(q, want)
    qv = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy().reshape(M, K // 32, 32)
    above = np.abs(g).max(-1) >= np.float32(1e-4)  # the floor is not what set the scale
    top = np.abs(qv).max(-1)
    assert np.all(top[above] >= 224) and np.all(top <= 448)


@pytest.mark.parametrize("seed,group_pow2,std", [(0, (-4, 4), 1.0), (1, None, 1.0),
                                                  (7, (-30, 30), 1.0), (9, None, 1e-6)])
def test_act_quant_properties_random(seed, group_pow2, std):
    x = synth.activations(37, 512, seed=seed, std=std, group_pow2=group_pow2)
    q, sf = oracle.act_quant(x)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    _scale_properties(xf, q, sf)


def test_act_quant_properties_extreme_bf16_groups():
    """Groups built from bf16 patterns at the edges: subnormals, the largest
    finite bf16, zeros and signed zeros, powers of two."""
    rng = np.random.default_rng(3)
    pats = [0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x0080, 0x7F7F, 0xFF7F, 0x3F80, 0x4380,
            0x38D1, 0x3A83, 0x4040]
    x = rng.choice(np.array(pats, dtype=np.uint16), size=(64, 96))
    x[:, 32:64] = rng.integers(0, 0x7F80, size=(64, 32)).astype(np.uint16)
    q, sf = oracle.act_quant(x)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    _scale_properties(xf, q, sf)
    assert sf.min() >= 105 and sf.max() <= 247


def test_act_quant_refuses_nonfinite_and_bad_k():
    x = np.zeros((1, 32), dtype=np.uint16)
    x[0, 3] = 0x7F80  # +Inf
    with pytest.raises(oracle.OracleError):
        oracle.act_quant(x)
    x[0, 3] = 0x7FC0  # NaN
    with pytest.raises(oracle.OracleError):
        oracle.act_quant(x)
    with pytest.raises(oracle.OracleError):
        oracle.act_quant_f32(np.zeros((1, 48), dtype=np.float32))


def test_qdq_value_is_exactly_q_times_s():
    """The dequantized bf16 value equals q * s exactly (formats.py page,
    docstring: 4 significant bits times a power of two survive bf16), so
    act_qdq loses nothing beyond act_quant -- below the top of the range."""
    for seed, gp in ((2, (-4, 4)), (5, (-60, 60))):
        x = synth.activations(16, 256, seed=seed, group_pow2=gp)
        q, sf = oracle.act_quant(x)
        y = oracle.act_qdq(q, sf)
        yv = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        qv = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        s = np.ldexp(1.0, sf.astype(np.int64) - 127).repeat(32, axis=1)
        assert np.array_equal(yv, qv * s)
        # bf16 round trip of those values is the identity (torch's conversion)
        yt = torch.from_numpy(yv).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.array_equal(yt, yv)


def test_qdq_identity_breaks_only_at_the_top_of_bf16():
    """At amax = the largest bf16 the scale is 2^120 and x/s rounds up to
    2^8 = 256, so q * s = 2^128 overflows: the one place the page's
    exactness claim cannot hold."""
    x = np.zeros((1, 32), dtype=np.uint16)
    x[0, 0] = 0x7F7F
    q, sf = oracle.act_quant(x)
    assert int(sf[0, 0]) == 247 and int(q[0, 0]) == 0x78  # 256 = 2^8 -> E=15, m=0
    y = oracle.act_qdq(q, sf)
    assert int(y[0, 0]) == 0x7F80  # +Inf


def test_bf16_rounding_helper_matches_torch():
    rng = np.random.default_rng(11)
    v = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    v = np.concatenate([v, np.float32([1.00390625, 1.01171875, -1.00390625, 0.0, -0.0])])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16_bits(float(t)) for t in v], dtype=np.uint16)
    assert np.array_equal(got, want)
