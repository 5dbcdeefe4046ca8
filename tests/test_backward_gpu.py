"""Parity of the backward-pass kernels with the fp64 oracle: the E5M2 gradient
quantizer (round to nearest even and stochastic, bit-exact including every
stochastic choice), the transposed quantizer (bit-exact) and the E5M2 x MXFP8
GEMMs that form dX and dW (within |y - ref| <= ulp_bf16(|ref|) + 2^-20 * S)."""
import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_quant_b200 as bq
from block_scaled_precision_quant_b200 import synth

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def f64(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_close(y, ref, tol, what=""):
    err = np.abs(y - ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{what}: {bad.shape[0]} of {err.size} outside tolerance; first "
                           f"{[(tuple(i), float(y[tuple(i)]), float(ref[tuple(i)])) for i in bad[:4]]}")


def grads(M, K, seed, spread=(-20, 4)):
    """Gradient-like values: N(0,1) times 2^U{spread} per 32-group."""
    return synth.activations(M, K, seed=seed, group_pow2=spread)


# ------------------------------------------------------- gradient quant ----

# (5000, 5056): a grid of >= 6144 one-row blocks (two rows per warp when rounding
# to nearest), ragged rows and chunks
@pytest.mark.parametrize("M,K", [(1, 32), (7, 96), (130, 544), (512, 4096), (5000, 5056)])
@pytest.mark.parametrize("stochastic", [False, True])
def test_grad_quant_bit_exact(M, K, stochastic):
    g = grads(M, K, seed=M + K)
    q, sf = bq.grad_quant(dev_bf16(g), stochastic=stochastic, seed=1234)
    sf_row = bq.unpack_scales(sf, M, K)
    bq.device_status()
    q_ref, s_ref = oracle.grad_quant(g, stochastic=stochastic, seed=1234)
    assert np.array_equal(sf_row.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_grad_quant_stochastic_seeds_row_stride_and_padding():
    M, K, ld = 45, 160, 232
    wide = grads(M, ld - 8, seed=2)
    wide = np.concatenate([wide, np.zeros((M, 8), np.uint16)], axis=1)
    xd = dev_bf16(wide)[:, :K]
    for seed in (0, 1, 2 ** 63 + 5):
        q, sf = bq.grad_quant(xd, stochastic=True, seed=seed)
        bq.device_status()
        q_ref, s_ref = oracle.grad_quant(np.ascontiguousarray(wide[:, :K]), stochastic=True,
                                         seed=seed)
        assert np.array_equal(q.cpu().numpy(), q_ref), seed
    full = bq.unpack_scales(sf, 128, 256).cpu().numpy()
    assert np.array_equal(full[:M, :K // 32], s_ref)
    assert np.all(full[M:, :] == 127) and np.all(full[:, K // 32:] == 127)


def test_grad_quant_special_values():
    """Exact E5M2 values, E5M2 subnormals, values below the smallest bin, signed
    zeros, a group at the 1e-4 floor, bf16 max."""
    rows = []
    base = np.array([1.0, -1.0625, 1.5, 3.0e-5, -3.0e-5, 1e-6, -1e-6, 0.0, -0.0, 57344.0,
                     60000.0, -7.0, 2.0 ** -16, 2.0 ** -17, 3 * 2.0 ** -17] + [0.5] * 17,
                    dtype=np.float32)
    rows += [base, base * 2.0 ** -10, base * 2.0 ** -40]
    top = np.zeros(32, np.float32)
    top[0] = np.float32(3.3895313892515355e38)
    top[1] = -1.0
    rows.append(top)
    x = np.stack(rows).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    for sr in (False, True):
        q, sf = bq.grad_quant(dev_bf16(bits), stochastic=sr, seed=7)
        bq.device_status()
        q_ref, s_ref = oracle.grad_quant(bits, stochastic=sr, seed=7)
        assert np.array_equal(q.cpu().numpy(), q_ref), sr
        assert np.array_equal(bq.unpack_scales(sf, len(rows), 32).cpu().numpy(), s_ref)


def test_grad_quant_stochastic_is_unbiased_on_device():
    """Mean of the dequantized stochastic codes over many elements holding the
    same value equals that value (within the sampling error)."""
    M, K = 256, 4096
    v = np.float32(1.0 + 1.0 / 8 + 1.0 / 64)  # between E5M2 1.0 and 1.25 at s = 1
    x = np.full((M, K), v, np.float32)
    x[:, ::32] = 1.75  # the group maximum sets s = 2^-15 ... keep one anchor per group
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    q, sf = bq.grad_quant(dev_bf16(bits), stochastic=True, seed=99)
    bq.device_status()
    sb = bq.unpack_scales(sf, M, K).cpu().numpy().astype(np.int64)
    e5m2 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e5m2) \
        .to(torch.float64).numpy()
    vals = e5m2[q.cpu().numpy()] * np.ldexp(1.0, sb - 127).repeat(32, axis=1)
    mask = np.ones((M, K), bool)
    mask[:, ::32] = False
    xv = float(f64(bits)[0, 1])
    sel = vals[mask]
    lo, hi = sel.min(), sel.max()
    p = (xv - lo) / (hi - lo)
    n = sel.size
    assert abs((sel == hi).mean() - p) < 5 * np.sqrt(p * (1 - p) / n)


# ---------------------------------------------------- transposed quant ----

@pytest.mark.parametrize("R,C", [(32, 8), (96, 40), (160, 200), (4096, 1536)])
@pytest.mark.parametrize("mode", ["e4m3", "e5m2", "e5m2_sr"])
def test_quant_transposed_bit_exact(R, C, mode):
    x = grads(R, C, seed=R + C, spread=None) if mode == "e4m3" else \
        synth.activations(R, C, seed=R + C)
    fmt = bq.BQ_FMT_E4M3 if mode == "e4m3" else bq.BQ_FMT_E5M2
    sr = mode == "e5m2_sr"
    q, sf = bq.quant_transposed(dev_bf16(x), fmt=fmt, stochastic=sr, seed=31)
    sf_row = bq.unpack_scales(sf, C, R)
    bq.device_status()
    q_ref, s_ref = oracle.quant_transposed(x, oracle.Q_E4M3 if mode == "e4m3" else oracle.Q_E5M2,
                                           stochastic=sr, seed=31)
    assert np.array_equal(sf_row.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_quant_transposed_row_stride_and_padding():
    R, C, ld = 96, 40, 72
    wide = synth.activations(R, ld, seed=4)
    xd = dev_bf16(wide)[:, :C]
    q, sf = bq.quant_transposed(xd, fmt=bq.BQ_FMT_E5M2, stochastic=True, seed=3)
    bq.device_status()
    q_ref, s_ref = oracle.quant_transposed(np.ascontiguousarray(wide[:, :C]), oracle.Q_E5M2,
                                           stochastic=True, seed=3)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    full = bq.unpack_scales(sf, 128, 128).cpu().numpy()  # rows to 128, groups to 4
    assert np.array_equal(full[:C, :R // 32], s_ref)
    assert np.all(full[C:, :] == 127) and np.all(full[:, R // 32:] == 127)


def test_quant_transposed_refusals():
    x = dev_bf16(synth.activations(64, 40, seed=1))
    with pytest.raises(bq.BqError) as e:
        bq.quant_transposed(x, fmt=bq.BQ_FMT_E4M3, stochastic=True)
    assert e.value.status == bq.BQ_ERR_INVALID
    with pytest.raises(bq.BqError) as e:
        bq.quant_transposed(dev_bf16(synth.activations(48, 40, seed=1)))  # R % 32
    assert e.value.status == bq.BQ_ERR_SHAPE
    with pytest.raises(bq.BqError) as e:
        bq.quant_transposed(dev_bf16(synth.activations(64, 44, seed=1)))  # C % 8
    assert e.value.status == bq.BQ_ERR_SHAPE


@pytest.mark.parametrize("R,C", [(32, 32), (96, 160), (160, 96), (4096, 1536)])
@pytest.mark.parametrize("stochastic", [False, True])
def test_grad_quant_dual_equals_both_quantizers(R, C, stochastic):
    g = grads(R, C, seed=R * 3 + C)
    q_row, sf_row, q_t, sf_t = bq.grad_quant_dual(dev_bf16(g), stochastic=stochastic, seed=21)
    bq.device_status()
    o_row, o_rs = oracle.grad_quant(g, stochastic=stochastic, seed=21)
    o_t, o_ts = oracle.quant_transposed(g, oracle.Q_E5M2, stochastic=stochastic, seed=21)
    assert np.array_equal(q_row.cpu().numpy(), o_row)
    assert np.array_equal(q_t.cpu().numpy(), o_t)
    rp, cp = (R + 127) // 128 * 128, (C + 127) // 128 * 128
    full_r = bq.unpack_scales(sf_row, rp, cp).cpu().numpy()
    full_t = bq.unpack_scales(sf_t, cp, rp).cpu().numpy()
    assert np.array_equal(full_r[:R, :C // 32], o_rs)
    assert np.array_equal(full_t[:C, :R // 32], o_ts)
    assert np.all(full_r[R:, :] == 127) and np.all(full_r[:, C // 32:] == 127)
    assert np.all(full_t[C:, :] == 127) and np.all(full_t[:, R // 32:] == 127)


# ------------------------------------------------------- backward GEMMs ----

def check_grad_gemm(aq, asf, b, bsf, M, N, K, config=None, workspace=None, what=""):
    """aq/asf: oracle E5M2 codes + row-major scales [M, K]; b/bsf E4M3 [N, K]."""
    y = bq.gemm(bq.W_GRAD, dev_u8(aq), bq.pack_weight_scales(dev_u8(asf), bq.BQ_SF_ROW32, M, K),
                dev_u8(b), bq.pack_weight_scales(dev_u8(bsf), bq.BQ_SF_ROW32, N, K), M, N, K,
                config=config, workspace=workspace)
    bq.device_status()
    yv = f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    ref, sabs = oracle.gemm(aq, asf, b, bsf, oracle.B_FP8ROW, M, N, K, a_kind=oracle.A_E5M2)
    assert_close(yv, ref, oracle.gemm_tolerance(ref, sabs), what)


@pytest.mark.parametrize("M,N,K,cfg", [
    (200, 264, 384, None),
    (257, 520, 256, dict(block_n=256, split_k=1, swap_ab=0)),
    (300, 384, 1024, dict(block_n=128, split_k=1, swap_ab=0, k_chunks=2)),
    (300, 512, 2048, dict(split_k=1, swap_ab=0, cta_pair=2)),
    (41, 384, 2048, dict(split_k=1, swap_ab=1, k_chunks=4)),
    (41, 256, 6144, dict(split_k=8, swap_ab=1, split_mode=2)),
])
def test_e5m2_mxfp8_gemm(M, N, K, cfg):
    g = grads(M, K, seed=M + N)
    aq, asf = oracle.grad_quant(g, stochastic=True, seed=5)
    b, bsf = oracle.act_quant(synth.activations(N, K, seed=N + K))
    config = bq.config(**cfg) if cfg else None
    ws = None
    if config is not None:
        need = bq.workspace_bytes(bq.W_GRAD, M, N, K, 1, config)
        ws = torch.zeros((max(need, 16),), dtype=torch.uint8, device="cuda") if need else None
    check_grad_gemm(aq, asf, b, bsf, M, N, K, config, ws, f"{M}x{N}x{K} {cfg}")


def backward_case(T, N, K, seed):
    """One linear layer y = x W^T (x [T, K], W [N, K]) and its output gradient
    dY [T, N]: the GPU backward (quantizers + the two GEMMs) against the
    oracle's quantizers and GEMMs on the same bf16 inputs."""
    x = synth.activations(T, K, seed=seed)
    w = synth.activations(N, K, seed=seed + 1, std=0.05)
    dy = grads(T, N, seed=seed + 2)
    xd, wd, dyd = dev_bf16(x), dev_bf16(w), dev_bf16(dy)
    # The B operands (W^T, X^T) are quantized before dY: a GEMM may read its
    # B operand while the kernel just before it is still running, so that
    # kernel is the quantizer of its A operand.
    wtq, wtsf = bq.quant_transposed(wd, fmt=bq.BQ_FMT_E4M3)              # W^T [K, N]
    xtq, xtsf = bq.quant_transposed(xd, fmt=bq.BQ_FMT_E4M3)              # X^T [K, T]
    gq, gsf, gtq, gtsf = bq.grad_quant_dual(dyd, stochastic=True, seed=11)  # dY, dY^T [N, T]
    # dX [T, K] = dY W: contraction over N
    dx = bq.gemm(bq.W_GRAD, gq, gsf, wtq, wtsf, T, K, N)
    # dW [N, K] = dY^T X: contraction over T
    dw = bq.gemm(bq.W_GRAD, gtq, gtsf, xtq, xtsf, N, K, T)
    bq.device_status()
    og, ogs = oracle.grad_quant(dy, stochastic=True, seed=11)
    owt, owts = oracle.quant_transposed(w, oracle.Q_E4M3)
    ogt, ogts = oracle.quant_transposed(dy, oracle.Q_E5M2, stochastic=True, seed=11)
    oxt, oxts = oracle.quant_transposed(x, oracle.Q_E4M3)
    assert np.array_equal(gq.cpu().numpy(), og)
    assert np.array_equal(wtq.cpu().numpy(), owt)
    assert np.array_equal(gtq.cpu().numpy(), ogt)
    assert np.array_equal(xtq.cpu().numpy(), oxt)
    return (dx, dw), (og, ogs, owt, owts, ogt, ogts, oxt, oxts)


def test_backward_step_full_compare():
    T, N, K = 256, 384, 512
    (dx, dw), (og, ogs, owt, owts, ogt, ogts, oxt, oxts) = backward_case(T, N, K, seed=40)
    ref, sabs = oracle.gemm(og, ogs, owt, owts, oracle.B_FP8ROW, T, K, N, a_kind=oracle.A_E5M2)
    assert_close(f64(dx.cpu().view(torch.int16).numpy().view(np.uint16)), ref,
                 oracle.gemm_tolerance(ref, sabs), "dX")
    ref, sabs = oracle.gemm(ogt, ogts, oxt, oxts, oracle.B_FP8ROW, N, K, T, a_kind=oracle.A_E5M2)
    assert_close(f64(dw.cpu().view(torch.int16).numpy().view(np.uint16)), ref,
                 oracle.gemm_tolerance(ref, sabs), "dW")


def test_backward_step_full_size_sampled():
    """The benchmark's backward layer: 4096 tokens, N = 1536, K = 6144."""
    T, N, K = 4096, 1536, 6144
    (dx, dw), (og, ogs, owt, owts, ogt, ogts, oxt, oxts) = backward_case(T, N, K, seed=50)
    rng = np.random.default_rng(0)
    for y, (aq, asf, b, bsf, M, NN, KK), what in (
            (dx, (og, ogs, owt, owts, T, K, N), "dX"),
            (dw, (ogt, ogts, oxt, oxts, N, K, T), "dW")):
        ms = np.concatenate([rng.integers(0, M, 1500), [0, M - 1]])
        ns = np.concatenate([rng.integers(0, NN, 1500), [NN - 1, 0]])
        ref, sabs = oracle.gemm_sampled(aq, asf, b, bsf, oracle.B_FP8ROW, M, NN, KK, ms, ns,
                                        a_kind=oracle.A_E5M2)
        yv = f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
        assert_close(yv[ms, ns], ref, oracle.gemm_tolerance(ref, sabs), what)
