"""Parity of the NVFP4 quantizer (bit-exact) and the NVFP4 x NVFP4 GEMM
(tcgen05.mma kind::mxf4nvf4, E4M3 scales per 16) with the fp64 oracle, GEMM
within |y - ref| <= ulp_bf16(|ref|) + 2^-20 * S."""
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


def unpack16(sf, rows, K):
    """Row-major [rows, K/16] view of an NVFP4 MMA-layout scale buffer: the
    layout of 16-input groups is the one bq_unpack_scales reads for K' = 2K."""
    return bq.unpack_scales(sf, rows, 2 * K)


# ------------------------------------------------------------ quantizer ----

@pytest.mark.parametrize("M,K", [(1, 32), (7, 96), (130, 544), (300, 4096)])
@pytest.mark.parametrize("g", [1.0, 0.37, 11.5])
def test_act_quant_nvfp4_bit_exact(M, K, g):
    x = synth.activations(M, K, seed=M + K, group_pow2=(-8, 4))
    q, sf = bq.act_quant_nvfp4(dev_bf16(x), g=g)
    sf_row = unpack16(sf, M, K)
    bq.device_status()
    q_ref, s_ref = oracle.act_quant_nvfp4(x, g)
    assert np.array_equal(sf_row.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)


def test_act_quant_nvfp4_special_values_and_padding():
    base = np.array([6.0, -3.0, 0.25, -0.1, 0.0, -0.0, 7.0, 1.0] + [0.0] * 8, np.float32)
    rows = [np.concatenate([base, base * 2.0 ** -12]), np.concatenate([base * 500.0, base]),
            np.zeros(32, np.float32), np.concatenate([base * 2.0 ** -30, -base])]
    x = np.stack(rows)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    sf_row = torch.empty((4, 2), dtype=torch.uint8, device="cuda")
    q, sf = bq.act_quant_nvfp4(dev_bf16(bits), sf_rowmajor=sf_row)
    bq.device_status()
    q_ref, s_ref = oracle.act_quant_nvfp4(bits)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sf_row.cpu().numpy(), s_ref)
    full = unpack16(sf, 128, 64).cpu().numpy()  # rows to 128, groups to 4
    assert np.array_equal(full[:4, :2], s_ref)
    assert np.all(full[4:, :] == 0x38) and np.all(full[:, 2:] == 0x38)


def test_pack_row16_e4m3_and_refusal():
    N, K = 200, 320
    rng = np.random.default_rng(3)
    s = rng.integers(0x20, 0x50, size=(N, K // 16)).astype(np.uint8)
    sf = bq.pack_weight_scales(dev_u8(s), bq.BQ_SF_ROW16_E4M3, N, K)
    assert sf.numel() == bq.sf_bytes_nvfp4(N, K)
    full = unpack16(sf, 256, K + 64 - K % 64 if K % 64 else K).cpu().numpy()
    assert np.array_equal(full[:N, :K // 16], s)
    assert np.all(full[N:, :] == 0x38)
    s[5, 3] = 0x7F
    with pytest.raises(bq.BqError) as e:
        bq.pack_weight_scales(dev_u8(s), bq.BQ_SF_ROW16_E4M3, N, K)
    assert e.value.status == bq.BQ_ERR_NAN_SCALE


# ----------------------------------------------------------------- GEMM ----

class NvCase:
    def __init__(self, M, N, K, seed=0, ga=1.0, gb=1.0, bias=False, residual=False,
                 act=bq.BQ_ACT_NONE):
        self.M, self.N, self.K, self.ga, self.gb, self.act = M, N, K, ga, gb, act
        self.x = synth.activations(M, K, seed=seed)
        self.w = synth.activations(N, K, seed=seed + 1, std=0.05)
        self.bias = synth.bias(N, seed=seed + 2) if bias else None
        self.res = synth.residual(M, N, seed=seed + 3) if residual else None
        self.alpha = float(np.float32(1.0 / (ga * gb)))
        self.bq_, self.bsf = oracle.act_quant_nvfp4(self.w, gb)  # weights: prequantized

    def gpu(self, config=None):
        aq, asf = bq.act_quant_nvfp4(dev_bf16(self.x), g=self.ga)
        bsf = bq.pack_weight_scales(dev_u8(self.bsf), bq.BQ_SF_ROW16_E4M3, self.N, self.K)
        y = bq.gemm(bq.W_NVFP4, aq, asf, dev_u8(self.bq_), bsf, self.M, self.N, self.K,
                    bias=dev_bf16(self.bias) if self.bias is not None else None,
                    residual=dev_bf16(self.res) if self.res is not None else None,
                    alpha=self.alpha, act=self.act, config=config)
        bq.device_status()
        return f64(y.cpu().view(torch.int16).numpy().view(np.uint16))

    def ref(self, ms=None, ns=None):
        aq, asf = oracle.act_quant_nvfp4(self.x, self.ga)
        kw = dict(bias=self.bias, residual=self.res, alpha=self.alpha, act=self.act,
                  a_kind=oracle.A_NVFP4)
        if ms is None:
            return oracle.gemm(aq, asf, self.bq_, self.bsf, oracle.B_NVFP4, self.M, self.N,
                               self.K, **kw)
        return oracle.gemm_sampled(aq, asf, self.bq_, self.bsf, oracle.B_NVFP4, self.M, self.N,
                                   self.K, ms, ns, **kw)

    def tol(self, ref, sabs, ms=None, ns=None):
        babs = rabs = None
        if self.bias is not None:
            babs = np.abs(f64(self.bias))
            babs = babs[None, :] if ms is None else babs[ns]
        if self.res is not None:
            rabs = np.abs(f64(self.res))
            rabs = rabs if ms is None else rabs[ms, ns]
        return oracle.gemm_tolerance(ref, sabs, self.alpha, babs, rabs, self.act)

    def check_full(self, config=None):
        y = self.gpu(config)
        ref, sabs = self.ref()
        assert_close(y, ref, self.tol(ref, sabs), f"NVFP4 {self.M}x{self.N}x{self.K} {config}")

    def check_sampled(self, n=2000):
        y = self.gpu()
        rng = np.random.default_rng(2)
        ms = np.concatenate([rng.integers(0, self.M, n), [0, self.M - 1]])
        ns = np.concatenate([rng.integers(0, self.N, n), [self.N - 1, 0]])
        ref, sabs = self.ref(ms, ns)
        assert_close(y[ms, ns], ref, self.tol(ref, sabs, ms, ns), "NVFP4 sampled")


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 264, 384), (257, 520, 640)])
def test_nvfp4_multi_tile_ragged(M, N, K):
    NvCase(M, N, K, seed=M + N).check_full()


@pytest.mark.parametrize("block_n", [128, 256])
def test_nvfp4_wide_tiles_per_tensor_scales(block_n):
    NvCase(300, 520, 1024, seed=5, ga=2.5, gb=40.0, bias=True).check_full(
        bq.config(block_n=block_n, split_k=1, swap_ab=0))


@pytest.mark.parametrize("M", [1, 41, 64])
def test_nvfp4_decode_swap(M):
    NvCase(M, 384, 2048, seed=10 + M, bias=True).check_full(bq.config(split_k=1, swap_ab=1))


@pytest.mark.parametrize("bias,res,act", [(True, False, bq.BQ_ACT_GELU),
                                          (False, True, bq.BQ_ACT_NONE)])
def test_nvfp4_epilogues(bias, res, act):
    NvCase(190, 264, 512, seed=20, ga=3.0, bias=bias, residual=res, act=act).check_full()


def test_nvfp4_full_size_sampled():
    NvCase(4096, 4096, 4096, seed=30, ga=8.0, gb=64.0).check_sampled()
    NvCase(41, 4608, 1536, seed=31, bias=True).check_sampled()


def test_nvfp4_refusals():
    c = NvCase(300, 520, 512)
    aq, asf = bq.act_quant_nvfp4(dev_bf16(c.x))
    bsf = bq.pack_weight_scales(dev_u8(c.bsf), bq.BQ_SF_ROW16_E4M3, c.N, c.K)
    for cfg in (bq.config(split_k=2, swap_ab=0), bq.config(split_k=1, swap_ab=0, cta_pair=2),
                bq.config(split_k=1, swap_ab=0, k_chunks=2)):
        with pytest.raises(bq.BqError) as e:
            bq.gemm(bq.W_NVFP4, aq, asf, dev_u8(c.bq_), bsf, c.M, c.N, c.K, config=cfg)
        assert e.value.status == bq.BQ_ERR_INVALID
    with pytest.raises(bq.BqError) as e:
        bq.act_quant_nvfp4(dev_bf16(c.x), g=0.0)
    assert e.value.status == bq.BQ_ERR_INVALID
