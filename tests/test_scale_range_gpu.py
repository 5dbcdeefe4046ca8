"""Parity of the block-scaled GEMMs at the ends of the E8M0 scale range and
under heavy cancellation.

The "formats.py" page (docstring "Formats", e8m0_to_f32) makes every scale
byte 0..254 a valid power of two 2^(b-127), byte 0 included; the activation
quantizer only ever produces 105..247, so these tests build both operands
directly (random finite codes with scale bytes drawn from a band) and feed
them to the GEMMs through the same prepacked MMA scale layout.  Every
element is compared with the oracle's exact-decode fp64 result at the
tolerance of every GEMM test, |y - ref| <= ulp_bf16(|ref|) + 2^-20 sum|a b|.

Scale bands (bytes drawn uniformly per 32-group; byte 0 / 254 forced into
some groups): one side at the bottom of the range (0..20) against the other
at the top (234..254), the top of the weights' range (230..246) against the
bottom of the activations', and both sides spread over 94..160 (products
spanning 2^+-60 inside one output).  The exponent sums stay where fp32 holds
the result.  Products that fall into fp32's subnormal range (a separate
case) are held to the same bound.

The cancellation cases pair every term of the first half of K with its
negation in the second half (same magnitudes, same scales), so sum a b = 0
exactly while sum |a b| is large and the running sum climbs to half of it
before it comes back; a variant leaves one pair a code step apart, so the
exact result is small but not zero, and another pairs each term with its
negation inside the same 32-input block.
"""
import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_quant_b200 as bq

pytestmark = pytest.mark.gpu

# weight kind -> (A code format, B code format, oracle B kind, oracle A kind)
KINDS = {
    bq.W_MXFP4: ("e4m3", "fp4", oracle.B_FP4, oracle.A_E4M3),
    bq.W_MXFP8: ("e4m3", "e4m3", oracle.B_FP8ROW, oracle.A_E4M3),
    bq.W_FP8BLK32: ("e4m3", "e4m3", oracle.B_FP8BLK, oracle.A_E4M3),
    bq.W_A4W4: ("fp4", "fp4", oracle.B_FP4, oracle.A_FP4),
}
FINITE_E4M3 = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
# E4M3 codes of magnitude >= 2^-2 (exponent field >= 5), for the cancellation
# cases: with them every partial sum of a row fits fp64 exactly
WIDE_E4M3 = np.array([c for c in FINITE_E4M3 if (c >> 3) & 0xF >= 5], dtype=np.uint8)


def dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def f64(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def codes(fmt, rows, K, rng, e4m3_set=FINITE_E4M3):
    """Random finite codes: E4M3 bytes [rows, K] drawn from e4m3_set, or packed
    E2M1 [rows, K/2] (all 16 codes in both nibbles)."""
    if fmt == "e4m3":
        return e4m3_set[rng.integers(0, e4m3_set.size, (rows, K))]
    return rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)


def scale_bytes(shape, band, rng, force=None):
    lo, hi = band
    s = rng.integers(lo, hi + 1, shape).astype(np.uint8)
    if force is not None:  # the band's end value in a few groups
        s.reshape(-1)[rng.integers(0, s.size, max(1, s.size // 16))] = force
    return s


def gemm_gpu(wk, aq, asf, b, bsf, M, N, K, config=None):
    a_d, b_d = dev_u8(aq), dev_u8(b)
    asf_d = bq.pack_weight_scales(dev_u8(asf), bq.BQ_SF_ROW32, M, K)
    kind = bq.BQ_SF_BLK32x32 if wk == bq.W_FP8BLK32 else bq.BQ_SF_ROW32
    bsf_d = bq.pack_weight_scales(dev_u8(bsf), kind, N, K)
    y = bq.gemm(wk, a_d, asf_d, b_d, bsf_d, M, N, K, config=config)
    bq.device_status()
    return f64(y.cpu().view(torch.int16).numpy().view(np.uint16))


def check(wk, aq, asf, b, bsf, M, N, K, config=None, what=""):
    _, _, okind, akind = KINDS[wk]
    y = gemm_gpu(wk, aq, asf, b, bsf, M, N, K, config)
    ref, sabs = oracle.gemm(aq, asf, b, bsf, okind, M, N, K, a_kind=akind)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    tol = oracle.gemm_tolerance(ref, sabs)
    err = np.abs(y - ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{what}: {bad.shape[0]} of {err.size} outside tolerance; first "
                           f"{[(tuple(i), float(y[tuple(i)]), float(ref[tuple(i)])) for i in bad[:4]]}")
    return y, ref, sabs


def operands(wk, M, N, K, a_band, b_band, seed, a_force=None, b_force=None,
             e4m3_set=FINITE_E4M3):
    rng = np.random.default_rng(seed)
    afmt, bfmt, _, _ = KINDS[wk]
    aq = codes(afmt, M, K, rng, e4m3_set)
    bq_ = codes(bfmt, N, K, rng, e4m3_set)
    asf = scale_bytes((M, K // 32), a_band, rng, a_force)
    bshape = ((N + 31) // 32, K // 32) if wk == bq.W_FP8BLK32 else (N, K // 32)
    bsf = scale_bytes(bshape, b_band, rng, b_force)
    return aq, asf, bq_, bsf


# (A band, B band, byte forced on A, on B): exponent sums a + b - 254 within +-20
# for the first three, within [-60, 66] for the spread band
BANDS = {
    "weights_low": ((234, 254), (0, 20), 254, 0),
    "weights_high": ((8, 28), (230, 246), None, 246),
    "acts_low": ((0, 20), (234, 254), 0, 254),
    "spread": ((94, 160), (100, 160), None, None),
}


@pytest.mark.parametrize("band", sorted(BANDS))
@pytest.mark.parametrize("wk", sorted(KINDS))
def test_scale_bands_wide_tiles(wk, band):
    """Wide tiles (activations on the 128-row MMA side), ragged M and N."""
    a_band, b_band, af, bf = BANDS[band]
    M, N, K = 200, 264, 512
    seed = 100 * sorted(BANDS).index(band) + wk
    check(wk, *operands(wk, M, N, K, a_band, b_band, seed=seed, a_force=af, b_force=bf), M, N, K,
          what=f"{wk} {band}")


@pytest.mark.parametrize("split", [1, 4])
@pytest.mark.parametrize("band", ["weights_low", "acts_low"])
@pytest.mark.parametrize("wk", [bq.W_MXFP4, bq.W_FP8BLK32])
def test_scale_bands_decode_tiles(wk, band, split):
    """Swap-AB decode tiles (weights on the 128-row side), unsplit and as a
    cluster split of K."""
    a_band, b_band, af, bf = BANDS[band]
    M, N, K = 41, 384, 1024
    cfg = bq.config(swap_ab=1, split_k=split,
                    split_mode=bq.BQ_SPLIT_CLUSTER if split > 1 else bq.BQ_SPLIT_AUTO)
    check(wk, *operands(wk, M, N, K, a_band, b_band, seed=7 + split, a_force=af, b_force=bf),
          M, N, K, config=cfg, what=f"decode {wk} {band} split {split}")


@pytest.mark.parametrize("wk", [bq.W_MXFP4, bq.W_MXFP8, bq.W_A4W4])
def test_scale_band_subnormal_products(wk):
    """Exponent sums a + b - 254 in [-154, -107]: products and block partials
    in or below fp32's subnormal range, outputs down to ~1e-40.  The pages
    leave the treatment of such values open; the plain bound holds (the
    tensor core does not flush them on B200), so no allowance is given."""
    M, N, K = 130, 136, 256
    ops = operands(wk, M, N, K, (100, 127), (0, 20), seed=31, b_force=0)
    check(wk, *ops, M, N, K, what=f"subnormal {wk}")


# ------------------------------------------------------------- cancellation --

def negate(fmt, c):
    """The code of the negated value: the sign bit (bit 7 of an E4M3 code, bit
    3 of each E2M1 nibble)."""
    return c ^ (0x80 if fmt == "e4m3" else 0x88)


def cancelling_operands(wk, M, N, K, seed, mode):
    """A and B whose products cancel in pairs.  mode "halves": element k of
    the first half of K is paired with k + K/2 (A negated, B equal, the
    second half's scale blocks copying the first half's); "inblock": elements
    pair inside one 32-input block (16 with the 16 after them); "near": as
    halves, with one pair per row of A a code step apart, so the sums are
    small but not zero."""
    rng = np.random.default_rng(seed)
    afmt, bfmt, _, _ = KINDS[wk]
    # scale bytes 123..131 on both sides and E4M3 codes of magnitude >= 2^-2:
    # every product and partial sum of a row spans few enough bits that the
    # oracle's fp64 sums are exact, so its reference is exactly 0 where the
    # terms cancel
    aq, asf, b, bsf = operands(wk, M, N, K, (123, 131), (123, 131), seed, e4m3_set=WIDE_E4M3)
    h = K // 2
    if mode in ("halves", "near"):
        if afmt == "e4m3":
            aq[:, h:] = negate(afmt, aq[:, :h])
        else:
            aq[:, h // 2:] = negate(afmt, aq[:, :h // 2])
        if bfmt == "e4m3":
            b[:, h:] = b[:, :h]
        else:
            b[:, h // 2:] = b[:, :h // 2]
        g = K // 64
        asf[:, g:] = asf[:, :g]
        bsf[:, g:] = bsf[:, :g]
        if mode == "near":
            # one E4M3 magnitude a code step smaller (codes 0x01..0x7E keep
            # their sign bit; 0x00 stays), so each row keeps one small residue
            assert afmt == "e4m3"
            col = h + rng.integers(0, h, M)
            c = aq[np.arange(M), col]
            mag = c & 0x7F
            aq[np.arange(M), col] = np.where(mag > 0, c - 1, c).astype(np.uint8)
    else:  # inblock: positions 16..31 of each block negate positions 0..15
        if afmt == "e4m3":
            a3 = aq.reshape(M, K // 32, 32)
            a3[:, :, 16:] = negate(afmt, a3[:, :, :16])
        else:
            a3 = aq.reshape(M, K // 32, 16)
            a3[:, :, 8:] = negate(afmt, a3[:, :, :8])
        if bfmt == "e4m3":
            b3 = b.reshape(N, K // 32, 32)
            b3[:, :, 16:] = b3[:, :, :16]
        else:
            b3 = b.reshape(N, K // 32, 16)
            b3[:, :, 8:] = b3[:, :, :8]
    return aq, asf, b, bsf


@pytest.mark.parametrize("mode", ["halves", "inblock"])
@pytest.mark.parametrize("wk", sorted(KINDS))
def test_cancellation_exact_zero(wk, mode):
    """sum a b = 0 exactly with sum |a b| large; the GEMM must stay within
    2^-20 sum |a b| of zero (and the fp64 oracle gives exactly 0)."""
    M, N, K = 150, 136, 2048
    y, ref, sabs = check(wk, *cancelling_operands(wk, M, N, K, 5, mode), M, N, K,
                         what=f"cancel {wk} {mode}")
    assert np.all(ref == 0.0)
    assert np.all(sabs > 0.0)


@pytest.mark.parametrize("cfg", [None, dict(swap_ab=1, split_k=4,
                                            split_mode=bq.BQ_SPLIT_CLUSTER),
                                 dict(swap_ab=1, split_k=3, split_mode=bq.BQ_SPLIT_WORKSPACE)])
def test_cancellation_small_residue(cfg):
    """Each row keeps one term uncancelled by a code step: the exact sums are
    small against sum |a b|, across the unsplit and both split reductions."""
    wk = bq.W_MXFP8
    M, N, K = 41, 256, 3072
    config = bq.config(**cfg) if cfg else None
    y, ref, sabs = check(wk, *cancelling_operands(wk, M, N, K, 9, "near"), M, N, K,
                         config=config, what=f"near-cancel {cfg}")
    assert np.any(ref != 0.0)
    assert np.median(np.abs(ref) / sabs) < 2.0 ** -6
