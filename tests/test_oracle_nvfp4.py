"""Pins for the oracle's NVFP4 path: E2M1 codes with one E4M3 scale per 16
values after a per-tensor scale (the A4W4 kernels of the "fp4-gemm" page), the
block scale read as the smallest E4M3 value that holds the block's largest
value.  Pinned by brute force over torch's float8_e4m3fn values for the
round-up scale, hand-worked groups, a numpy restatement, the no-clip and
minimality invariants, and rational brute force for the GEMM."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_quant_b200 import synth
from conftest import parse_int, read_golden

TABLE = {int(c): float(v) for c, v in read_golden("fp4_table.txt")}
MAG = np.array([TABLE[c] for c in range(8)])
E4M3 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).numpy()
POS = np.array([E4M3[c] for c in range(1, 127)])  # positive finite E4M3 values, increasing


def brute_ceil(t):
    """Index (byte) of the smallest positive E4M3 value >= t, capped at 448."""
    idx = np.searchsorted(POS, np.asarray(t, dtype=np.float64), side="left")
    return (np.minimum(idx, 125) + 1).astype(np.uint8)


def brute_fp4(v):
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), 6.0)
    d = np.abs(a[..., None] - MAG)
    cand = d == d.min(axis=-1, keepdims=True)
    even = cand & (np.arange(8) % 2 == 0)
    code = np.where(even.any(axis=-1), even.argmax(axis=-1), cand.argmax(axis=-1))
    return (code | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def test_e4m3_ceil_brute_force():
    ts = np.concatenate([POS, np.nextafter(POS, 0), np.nextafter(POS, 1e9), [0.0, 1e-30, 500.0],
                         np.random.default_rng(0).uniform(0, 460, 2000)]).astype(np.float32)
    got = np.array([oracle.e4m3_ceil(float(t)) for t in ts], dtype=np.uint8)
    assert np.array_equal(got, brute_ceil(ts.astype(np.float64)))


def test_hand_worked_groups():
    rows = read_golden("nvfp4_worked_group.txt")
    groups = {}
    for r in rows:
        if r[0] == "SCALE":
            groups.setdefault(r[1], [{}, None])[1] = parse_int(r[2])
        else:
            groups.setdefault(r[0], [{}, None])[0][int(r[1])] = (parse_int(r[2]), int(r[3]))
    names = sorted(groups)
    x = np.zeros((1, 16 * len(names)), np.uint16)
    for gi, nm in enumerate(names):
        for i, (bits, _) in groups[nm][0].items():
            x[0, 16 * gi + i] = bits
    q, sf = oracle.act_quant_nvfp4(x)
    codes = oracle.unpack_fp4(q)[0]
    for gi, nm in enumerate(names):
        assert sf[0, gi] == groups[nm][1], nm
        for i, (_, c) in groups[nm][0].items():
            assert codes[16 * gi + i] == c, (nm, i)


def restated(x_bits, g):
    xf = ((x_bits.astype(np.uint32) << 16).view(np.float32) * np.float32(g)).astype(np.float32)
    M, K = xf.shape
    blk = xf.reshape(M, K // 16, 16)
    amax = np.abs(blk).max(axis=-1).astype(np.float32)
    t = (amax * np.float32(1.0 / 6.0)).astype(np.float32)
    sb = brute_ceil(t.astype(np.float64))
    s = E4M3[sb].astype(np.float32)
    y = np.clip((blk / s[..., None]).astype(np.float32), -6.0, 6.0)
    codes = brute_fp4(y).reshape(M, K)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8), sb


@pytest.mark.parametrize("g", [1.0, 0.37, 2688.0 / 7.5])
def test_restatement_agrees(g):
    x = synth.activations(40, 512, seed=int(g * 10), group_pow2=(-6, 2))
    q, sf = oracle.act_quant_nvfp4(x, g)
    q2, sf2 = restated(x, g)
    assert np.array_equal(sf, sf2)
    assert np.array_equal(q, q2)


def test_no_clip_and_minimal_scale():
    x = synth.activations(64, 1024, seed=3)
    q, sf = oracle.act_quant_nvfp4(x)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64).reshape(64, -1, 16)
    amax = np.abs(xf).max(axis=-1)
    s = E4M3[sf]
    assert np.all(amax / s <= 6.0)                     # no value clips
    below = E4M3[np.maximum(sf.astype(int) - 1, 0)]    # the next smaller E4M3 value
    t = (amax.astype(np.float32) * np.float32(1.0 / 6.0)).astype(np.float64)
    assert np.all((sf == 1) | (below < t))             # and none smaller would hold it


@pytest.mark.parametrize("M,N,K", [(2, 3, 32), (4, 5, 64)])
def test_nvfp4_gemm_brute_force(M, N, K):
    rng = np.random.default_rng(M + N + K)
    aq = rng.integers(0, 256, size=(M, K // 2)).astype(np.uint8)
    b = rng.integers(0, 256, size=(N, K // 2)).astype(np.uint8)
    # E4M3 scales 2^-3 .. 2^3 (bytes 0x20 .. 0x50): sums stay exact in fp64
    asf = rng.integers(0x20, 0x51, size=(M, K // 16)).astype(np.uint8)
    bsf = rng.integers(0x20, 0x51, size=(N, K // 16)).astype(np.uint8)
    ref, sabs = oracle.gemm(aq, asf, b, bsf, oracle.B_NVFP4, M, N, K, a_kind=oracle.A_NVFP4)
    ua, ub = oracle.unpack_fp4(aq), oracle.unpack_fp4(b)
    for m in range(M):
        for n in range(N):
            terms = [Fraction(TABLE[int(ua[m, k])]) * Fraction(E4M3[asf[m, k // 16]]) *
                     Fraction(TABLE[int(ub[n, k])]) * Fraction(E4M3[bsf[n, k // 16]])
                     for k in range(K)]
            assert ref[m, n] == float(sum(terms))
            assert sabs[m, n] == float(sum(abs(t) for t in terms))
