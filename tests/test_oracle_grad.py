"""Pins for the oracle's backward-pass pieces: E5M2 codes, the counter-based
generator of the stochastic draws, the per-32 E5M2 gradient quantizer (round
to nearest even and stochastic), the transposed quantizer and the GEMM over
E5M2 gradient codes.

The "hip_quant" README on the pages describes E5M2 backward gradients with
optional stochastic rounding (the upper neighbour is taken with a probability
that grows linearly with the value's position between the two E5M2 values,
the random number a function of the seed and the element's index alone) and
block-wise scaling along the last dimension; the scale rule is the formats.py
page's with 57344 in place of 448.  Pins: torch's float8_e5m2 for the format,
numpy's Philox bit generator for the draws, hand-worked scales, a numpy
restatement, the stochastic rule's bracket and frequency, the plain
definition of the transposed quantization, rational brute force for the GEMM.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_quant_b200 import synth
from conftest import parse_float, read_golden

E5M2 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e5m2) \
    .to(torch.float64).numpy()
E4M3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).numpy()
FINITE = [c for c in range(256) if np.isfinite(E5M2[c])]


def bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def torch_e5m2(v):
    """torch's E5M2 conversion (round to nearest even) of values already
    clamped to +-57344."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    return t.to(torch.float8_e5m2).view(torch.uint8).numpy()


def test_decode_matches_torch():
    assert len(FINITE) == 248
    for c in range(256):
        if c in FINITE:
            v = oracle.decode_e5m2(c)
            assert v == E5M2[c] and np.signbit(v) == np.signbit(E5M2[c])
        else:
            with pytest.raises(oracle.OracleError):
                oracle.decode_e5m2(c)
    assert oracle.decode_e5m2(0x7B) == 57344.0


def test_encode_rne_matches_torch_on_all_bf16_values():
    f = bits_to_f32(np.arange(65536, dtype=np.uint32))
    f = f[np.isfinite(f)]
    for scale in (1.0, 2.0 ** -20, 2.0 ** 10):
        with np.errstate(over="ignore"):
            v = (f * np.float32(scale)).astype(np.float32)
        v = np.clip(v[np.isfinite(v)], -57344.0, 57344.0).astype(np.float32)
        assert np.array_equal(oracle.encode_e5m2_array(v), torch_e5m2(v))


@pytest.mark.parametrize("key,ctr", [((0, 0), (0, 0, 0, 0)), ((1234, 0), (7, 0, 0, 0)),
                                     ((2 ** 64 - 1, 99), (2 ** 40, 3, 5, 9)),
                                     ((42, 0), (2 ** 64 - 1, 5, 0, 0))])
def test_philox_matches_numpy(key, ctr):
    """numpy's Philox (4x64, 10 rounds) increments its 256-bit counter before
    each block: its first block is Philox(counter + 1)."""
    bg = np.random.Philox(key=np.array(key, dtype=np.uint64),
                          counter=np.array(ctr, dtype=np.uint64))
    raw = bg.random_raw(8)
    c = list(ctr)
    for blk in range(2):
        c[0] += 1  # with carry into the next words
        for w in range(3):
            if c[w] == 2 ** 64:
                c[w] = 0
                c[w + 1] += 1
        assert list(oracle.philox4x64_10(c, key)) == list(raw[4 * blk:4 * blk + 4])


def test_uniform_draw_is_philox_word():
    """Element i's draw: 32-bit half (i % 2) of word (i / 2) % 4 of the Philox
    block at counter i / 8 (numpy's block j comes from counter j + 1)."""
    for seed, idx in ((0, 0), (5, 3), (99, 12), (2 ** 63, 12345), (7, 8)):
        blk = idx >> 3
        ctr = [blk - 1, 0, 0, 0] if blk else [2 ** 64 - 1] * 4
        bg = np.random.Philox(key=np.array([seed, 0], dtype=np.uint64),
                              counter=np.array(ctr, dtype=np.uint64))
        word = int(bg.random_raw(4)[(idx >> 1) & 3])
        half = (word >> 32) if idx & 1 else (word & 0xFFFFFFFF)
        assert oracle.uniform(seed, idx) == half * 2.0 ** -32
    u = np.array([oracle.uniform(7, i) for i in range(20000)])
    assert u.min() >= 0.0 and u.max() < 1.0 and abs(u.mean() - 0.5) < 0.01


def test_stochastic_rounding_rule():
    # representable values never move
    for c in FINITE[:120:7]:
        v = np.float32(E5M2[c])
        for u in (0.0, 0.3, 0.999999):
            assert oracle.encode_e5m2_sr(v, u) == oracle.encode_e5m2(v)
    # a value a quarter of the way from 1.0 to 1.25 rounds up for u < 0.25
    v = np.float32(1.0625)
    assert oracle.encode_e5m2_sr(v, 0.2499) == 0x3D     # 1.25
    assert oracle.encode_e5m2_sr(v, 0.25) == 0x3C       # 1.0
    assert oracle.encode_e5m2_sr(-v, 0.1) == 0xBD       # sign kept
    assert oracle.encode_e5m2_sr(np.float32(1e-9), 0.0) == 0x01  # subnormal bin above 0
    assert oracle.encode_e5m2_sr(np.float32(-1e-9), 0.5) == 0x80  # -0
    assert oracle.encode_e5m2_sr(np.float32(60000.0), 0.0) == 0x7B  # saturates
    # over a fine grid of draws the rounded-up fraction is d (to 2^-12): unbiased
    rng = np.random.default_rng(0)
    grid = (np.arange(4096) + 0.5) / 4096
    for v in rng.uniform(-100, 100, 20).astype(np.float32):
        codes = [oracle.encode_e5m2_sr(v, u) for u in grid]
        vals = E5M2[codes]
        assert abs(vals.mean() - float(v)) <= 2.0 ** -12 * abs(np.diff(np.unique(vals))).max() + 1e-12


@pytest.mark.parametrize("row", read_golden("grad_scale_worked.txt"))
def test_hand_worked_grad_scales(row):
    amax, byte = parse_float(row[0]), int(row[1])
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 3] = amax
    x[0, 30] = -amax / 4
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert float(bits_to_f32(bits)[0, 3]) == amax  # every listed amax is a bf16 value
    _, sf = oracle.grad_quant(bits)
    assert sf[0, 0] == byte


def restated_grad_quant(x_bits):
    xf = bits_to_f32(x_bits).astype(np.float32)
    M, K = xf.shape
    g = xf.reshape(M, K // 32, 32)
    amax = np.maximum(np.abs(g).max(axis=-1), np.float32(1e-4)).astype(np.float32)
    t = (amax * np.float32(1.0 / 57344.0)).astype(np.float32)
    mant, ex = np.frexp(t.astype(np.float64))
    e = np.where(mant == 0.5, ex - 1, ex)
    y = np.clip(g.astype(np.float64) / np.ldexp(1.0, e)[..., None], -57344.0, 57344.0)
    return torch_e5m2(y.astype(np.float32)).reshape(M, K), (e + 127).astype(np.uint8)


@pytest.mark.parametrize("seed", [0, 1])
def test_grad_quant_rne_restatement(seed):
    x = synth.activations(48, 1024, seed=seed, group_pow2=(-30, 30))
    q, sf = oracle.grad_quant(x)
    q2, sf2 = restated_grad_quant(x)
    assert np.array_equal(sf, sf2)
    assert np.array_equal(q, q2)


def test_grad_quant_stochastic_brackets_and_index():
    M, K = 16, 256
    x = synth.activations(M, K, seed=3, group_pow2=(-6, 6))
    q_rne, sf = oracle.grad_quant(x)
    q_sr, sf_sr = oracle.grad_quant(x, stochastic=True, seed=77)
    assert np.array_equal(sf, sf_sr)
    s = np.ldexp(1.0, sf.astype(np.int64) - 127).repeat(32, axis=1)
    y = bits_to_f32(x).astype(np.float64) / s
    v = E5M2[q_sr]
    # the stochastic code is one of the two E5M2 neighbours of y, same sign
    step = np.maximum(np.abs(y), 2.0 ** -14) * 2.0 ** -2
    assert np.all(np.abs(v - y) <= step + 1e-30)
    assert np.all((v == 0) | (np.sign(v) == np.sign(y)))
    # element (m, k) draws uniform(seed, m * K + k)
    for m, k in ((0, 0), (3, 17), (15, 255), (7, 128)):
        assert q_sr[m, k] == oracle.encode_e5m2_sr(np.float32(y[m, k]),
                                                   oracle.uniform(77, m * K + k))
    # deterministic per seed, different across seeds
    assert np.array_equal(q_sr, oracle.grad_quant(x, stochastic=True, seed=77)[0])
    assert not np.array_equal(q_sr, oracle.grad_quant(x, stochastic=True, seed=78)[0])


def test_transposed_is_rowwise_of_transpose():
    R, C = 96, 40
    x = synth.activations(R, C, seed=5)
    xt = np.ascontiguousarray(x.T)
    q, sf = oracle.quant_transposed(x, oracle.Q_E4M3)
    q2, sf2 = oracle.act_quant(xt)
    assert np.array_equal(q, q2) and np.array_equal(sf, sf2)
    q, sf = oracle.quant_transposed(x, oracle.Q_E5M2)
    q2, sf2 = oracle.grad_quant(xt)
    assert np.array_equal(q, q2) and np.array_equal(sf, sf2)
    # stochastic: element (r, c) of x keeps its own index r * C + c
    q, sf = oracle.quant_transposed(x, oracle.Q_E5M2, stochastic=True, seed=9)
    s = np.ldexp(1.0, sf.astype(np.int64) - 127)
    xf = bits_to_f32(x).astype(np.float64)
    for r, c in ((0, 0), (31, 39), (64, 7), (95, 20)):
        y = np.float32(xf[r, c] / s[c, r // 32])
        assert q[c, r] == oracle.encode_e5m2_sr(y, oracle.uniform(9, r * C + c))


@pytest.mark.parametrize("M,N,K", [(2, 3, 32), (5, 4, 96)])
def test_e5m2_activation_gemm_brute_force(M, N, K):
    rng = np.random.default_rng(M * N + K)
    # Narrow exponent ranges so that fp64 sums are exact: E5M2 exponent fields 12..18
    # (7 binades), E4M3 fields 5..10 (6), scale spans 4 and 3 binades; with 3 + 4 mantissa
    # bits and log2 K < 7 the products of a sum span under 34 bits.
    a_codes = [c for c in FINITE if 12 <= (c >> 2) & 0x1F <= 18]
    b_codes = [c for c in range(256) if 5 <= (c >> 3) & 0xF <= 10]
    aq = rng.choice(a_codes, size=(M, K)).astype(np.uint8)
    asf = rng.integers(120, 124, size=(M, K // 32)).astype(np.uint8)
    b = rng.choice(b_codes, size=(N, K)).astype(np.uint8)
    bsf = rng.integers(125, 128, size=(N, K // 32)).astype(np.uint8)
    ref, sabs = oracle.gemm(aq, asf, b, bsf, oracle.B_FP8ROW, M, N, K, a_kind=oracle.A_E5M2)
    e8 = lambda v: Fraction(2) ** (int(v) - 127)  # noqa: E731
    for m in range(M):
        for n in range(N):
            terms = [Fraction(E5M2[aq[m, k]]) * e8(asf[m, k // 32]) *
                     Fraction(E4M3[b[n, k]]) * e8(bsf[n, k // 32]) for k in range(K)]
            assert ref[m, n] == float(sum(terms))
            assert sabs[m, n] == float(sum(abs(t) for t in terms))
