"""Parity of the MXFP4 activation quantizer (bit-exact) and the FP4 x FP4
(A4W4, tcgen05.mma kind::mxf4) GEMM with the fp64 oracle.

GEMM tolerance as for the other GEMMs: |y - ref| <= ulp_bf16(|ref|) + 2^-20 * S
per element, ref the oracle's exact-decode fp64 result from the same codes."""
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


# ------------------------------------------------------------ act_quant ----

# (6100, 4128): a grid of >= 6144 one-row blocks, so two rows per warp, with
# ragged rows and a last chunk of one group
@pytest.mark.parametrize("M,K", [(1, 32), (7, 96), (64, 1024), (130, 544), (300, 4096),
                                 (6100, 4128)])
def test_act_quant_mxfp4_bit_exact(M, K):
    x = synth.activations(M, K, seed=M + K, group_pow2=(-10, 10))
    q, sf = bq.act_quant_mxfp4(dev_bf16(x))
    sf_row = bq.unpack_scales(sf, M, K)
    bq.device_status()
    q_ref, s_ref = oracle.act_quant_fp4(x)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sf_row.cpu().numpy(), s_ref)


def test_act_quant_mxfp4_row_stride_rowmajor_scales_and_padding():
    M, K, ld = 45, 160, 200
    wide = synth.activations(M, ld, seed=3)
    xd = dev_bf16(wide)[:, :K]
    sf_row = torch.empty((M, K // 32), dtype=torch.uint8, device="cuda")
    q, sf = bq.act_quant_mxfp4(xd, sf_rowmajor=sf_row)
    bq.device_status()
    q_ref, s_ref = oracle.act_quant_fp4(np.ascontiguousarray(wide[:, :K]))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sf_row.cpu().numpy(), s_ref)
    # MMA layout: rows padded to 128 and K/32 to a multiple of 4, pad bytes 127
    full = bq.unpack_scales(sf, 128, 256).cpu().numpy()
    assert np.array_equal(full[:M, :K // 32], s_ref)
    assert np.all(full[M:, :] == 127) and np.all(full[:, K // 32:] == 127)


def test_act_quant_mxfp4_special_values():
    """Ties on the E2M1 grid, negative values that round to zero (-0, code 8),
    saturation, all-zero and tiny groups, bf16 max."""
    vals = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, -0.25, -0.1, -5.0, 0.0] +
                    [0.0] * 20, dtype=np.float32)
    rows = [vals, vals * 2.0 ** -20, np.zeros(32, np.float32), vals * 2.0 ** 100]
    top = np.zeros(32, np.float32)
    top[0] = np.float32(3.3895313892515355e38)  # bf16 max
    top[1] = -1.0
    rows.append(top)
    x = np.stack(rows).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    q, sf = bq.act_quant_mxfp4(dev_bf16(bits))
    bq.device_status()
    q_ref, s_ref = oracle.act_quant_fp4(bits)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(bq.unpack_scales(sf, len(rows), 32).cpu().numpy(), s_ref)


def test_act_quant_mxfp4_nonfinite_status():
    x = synth.activations(4, 64, seed=1)
    x[2, 17] = 0x7F80  # +Inf
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bq.act_quant_mxfp4(dev_bf16(x), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1


# ----------------------------------------------------------------- GEMM ----

class A4Case:
    def __init__(self, M, N, K, seed=0, bias=False, residual=False, alpha=1.0,
                 act=bq.BQ_ACT_NONE, act_gp=None):
        self.M, self.N, self.K, self.alpha, self.act = M, N, K, alpha, act
        self.x = synth.activations(M, K, seed=seed, group_pow2=act_gp)
        self.b, self.bsf = synth.mxfp4_weight(N, K, seed=seed + 100)
        self.bias = synth.bias(N, seed=seed + 200) if bias else None
        self.res = synth.residual(M, N, seed=seed + 300) if residual else None

    def gpu(self, config=None, workspace=None):
        aq, asf = bq.act_quant_mxfp4(dev_bf16(self.x))
        bsf = bq.pack_weight_scales(dev_u8(self.bsf), bq.BQ_SF_ROW32, self.N, self.K)
        y = bq.gemm(bq.W_A4W4, aq, asf, dev_u8(self.b), bsf, self.M, self.N, self.K,
                    bias=dev_bf16(self.bias) if self.bias is not None else None,
                    residual=dev_bf16(self.res) if self.res is not None else None,
                    alpha=self.alpha, act=self.act, config=config, workspace=workspace)
        bq.device_status()
        return f64(y.cpu().view(torch.int16).numpy().view(np.uint16))

    def ref(self, ms=None, ns=None):
        aq, asf = oracle.act_quant_fp4(self.x)
        kw = dict(bias=self.bias, residual=self.res, alpha=self.alpha, act=self.act,
                  a_kind=oracle.A_FP4)
        if ms is None:
            return oracle.gemm(aq, asf, self.b, self.bsf, oracle.B_FP4, self.M, self.N, self.K,
                               **kw)
        return oracle.gemm_sampled(aq, asf, self.b, self.bsf, oracle.B_FP4, self.M, self.N,
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

    def check_full(self, config=None, workspace=None):
        y = self.gpu(config, workspace)
        ref, sabs = self.ref()
        assert_close(y, ref, self.tol(ref, sabs), f"A4W4 {self.M}x{self.N}x{self.K} {config}")

    def check_sampled(self, n=3000, config=None):
        y = self.gpu(config)
        rng = np.random.default_rng(1)
        ms = np.concatenate([rng.integers(0, self.M, n), [0, self.M - 1, 0, self.M - 1]])
        ns = np.concatenate([rng.integers(0, self.N, n), [0, 0, self.N - 1, self.N - 1]])
        ref, sabs = self.ref(ms, ns)
        assert_close(y[ms, ns], ref, self.tol(ref, sabs, ms, ns), "A4W4 sampled")


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 264, 384), (257, 520, 640),
                                   (130, 128, 128)])
def test_a4w4_multi_tile_ragged(M, N, K):
    """Several tiles with ragged tails in M and N; K with a half chunk (128 of
    256 K) at its end (384, 640) and K shorter than a chunk (128)."""
    A4Case(M, N, K, seed=M + N, act_gp=(-4, 4)).check_full()


@pytest.mark.parametrize("block_n", [128, 256])
@pytest.mark.parametrize("k_chunks", [1, 2])
def test_a4w4_wide_tiles(block_n, k_chunks):
    A4Case(300, 520, 1024, seed=11).check_full(
        bq.config(block_n=block_n, split_k=1, swap_ab=0, k_chunks=k_chunks))


@pytest.mark.parametrize("k_chunks,K", [(1, 1408), (2, 1536)])
def test_a4w4_pair_tiles(k_chunks, K):
    """256x256 tiles on CTA pairs with kind::mxf4 (cta_group::2): ragged M and
    N; with one chunk per stage K ends in a half chunk (128 of 256 K)."""
    A4Case(600, 776, K, seed=12 + k_chunks, bias=True, residual=True).check_full(
        bq.config(split_k=1, swap_ab=0, cta_pair=2, k_chunks=k_chunks))


def test_a4w4_pair_tiles_persistent():
    """More pair tiles than SM pairs: every pair walks several tiles."""
    A4Case(2304, 2560, 512, seed=17).check_full(bq.config(split_k=1, swap_ab=0, cta_pair=2))


def test_a4w4_pair_tiles_batched_gelu():
    count, M, N, K = 2, 300, 520, 1024
    xs = [synth.activations(M, K, seed=80 + i) for i in range(count)]
    b, bsf = synth.mxfp4_weight(N, K, seed=85)
    bias = synth.bias(N, seed=86)
    qs, sfs = zip(*[bq.act_quant_mxfp4(dev_bf16(x)) for x in xs])
    aq = torch.stack(qs).reshape(count * M, K // 2)
    asf = torch.stack(sfs)
    bsf_d = bq.pack_weight_scales(dev_u8(bsf), bq.BQ_SF_ROW32, N, K)
    y = bq.gemm(bq.W_A4W4, aq, asf, dev_u8(b), bsf_d, M, N, K, bias=dev_bf16(bias),
                act=bq.BQ_ACT_GELU, config=bq.config(split_k=1, swap_ab=0, cta_pair=2),
                batch=dict(count=count, stride_a=M * K // 2, stride_a_sf=asf.shape[1],
                           stride_b=0, stride_b_sf=0, stride_y=M * N * 2))
    bq.device_status()
    yv = f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    for i, x in enumerate(xs):
        q, s = oracle.act_quant_fp4(x)
        ref, sabs = oracle.gemm(q, s, b, bsf, oracle.B_FP4, M, N, K, bias=bias,
                                act=oracle.ACT_GELU, a_kind=oracle.A_FP4)
        tol = oracle.gemm_tolerance(ref, sabs, 1.0, np.abs(f64(bias))[None, :], None,
                                    oracle.ACT_GELU)
        assert_close(yv[i], ref, tol, f"pair batch {i}")


@pytest.mark.parametrize("M", [1, 17, 41, 64])
@pytest.mark.parametrize("k_chunks", [1, 4])
def test_a4w4_decode_swap(M, k_chunks):
    A4Case(M, 384, 2048, seed=20 + M, bias=True).check_full(
        bq.config(split_k=1, swap_ab=1, k_chunks=k_chunks))


@pytest.mark.parametrize("split,mode", [(2, bq.BQ_SPLIT_CLUSTER), (4, bq.BQ_SPLIT_CLUSTER),
                                        (8, bq.BQ_SPLIT_CLUSTER), (3, bq.BQ_SPLIT_WORKSPACE),
                                        (5, bq.BQ_SPLIT_WORKSPACE)])
def test_a4w4_decode_split_k(split, mode):
    c = A4Case(41, 256, 6144, seed=30 + split, bias=True, residual=(split == 4))
    cfg = bq.config(split_k=split, swap_ab=1, split_mode=mode)
    need = bq.workspace_bytes(bq.W_A4W4, 41, 256, 6144, 1, cfg)
    ws = torch.zeros((max(need, 16),), dtype=torch.uint8, device="cuda") if need else None
    c.check_full(cfg, ws)


def test_a4w4_split_k_wide_tiles():
    c = A4Case(256, 384, 4096, seed=40, residual=True)
    cfg = bq.config(split_k=4, swap_ab=0, block_n=128)
    need = bq.workspace_bytes(bq.W_A4W4, 256, 384, 4096, 1, cfg)
    c.check_full(cfg, torch.zeros((need,), dtype=torch.uint8, device="cuda"))


@pytest.mark.parametrize("bias,res,act,alpha", [(True, False, bq.BQ_ACT_GELU, 1.0),
                                                (True, True, bq.BQ_ACT_NONE, 0.5),
                                                (False, True, bq.BQ_ACT_NONE, 2.0)])
def test_a4w4_epilogues(bias, res, act, alpha):
    A4Case(190, 264, 512, seed=50, bias=bias, residual=res, act=act, alpha=alpha).check_full()


def test_a4w4_batched_broadcast_weight():
    count, M, N, K = 3, 200, 264, 512
    xs = [synth.activations(M, K, seed=60 + i) for i in range(count)]
    b, bsf = synth.mxfp4_weight(N, K, seed=65)
    bias = synth.bias(N, seed=66)
    qs, sfs = zip(*[bq.act_quant_mxfp4(dev_bf16(x)) for x in xs])
    aq = torch.stack(qs).reshape(count * M, K // 2)
    asf = torch.stack(sfs)
    bsf_d = bq.pack_weight_scales(dev_u8(bsf), bq.BQ_SF_ROW32, N, K)
    y = bq.gemm(bq.W_A4W4, aq, asf, dev_u8(b), bsf_d, M, N, K, bias=dev_bf16(bias),
                act=bq.BQ_ACT_GELU,
                batch=dict(count=count, stride_a=M * K // 2, stride_a_sf=asf.shape[1],
                           stride_b=0, stride_b_sf=0, stride_y=M * N * 2))
    bq.device_status()
    yv = f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    for i, x in enumerate(xs):
        q, s = oracle.act_quant_fp4(x)
        ref, sabs = oracle.gemm(q, s, b, bsf, oracle.B_FP4, M, N, K, bias=bias,
                                act=oracle.ACT_GELU, a_kind=oracle.A_FP4)
        tol = oracle.gemm_tolerance(ref, sabs, 1.0, np.abs(f64(bias))[None, :], None,
                                    oracle.ACT_GELU)
        assert_close(yv[i], ref, tol, f"batch {i}")


def test_a4w4_quantized_output():
    """The MXFP8-emitting epilogue on an A4W4 product: codes and scales equal
    act_quant of the bf16 y the same call writes."""
    c = A4Case(150, 256, 512, seed=70, bias=True)
    aq, asf = bq.act_quant_mxfp4(dev_bf16(c.x))
    bsf = bq.pack_weight_scales(dev_u8(c.bsf), bq.BQ_SF_ROW32, c.N, c.K)
    y, q, sf = bq.gemm(bq.W_A4W4, aq, asf, dev_u8(c.b), bsf, c.M, c.N, c.K,
                       bias=dev_bf16(c.bias), quantize_out=True)
    bq.device_status()
    ybits = y.cpu().view(torch.int16).numpy().view(np.uint16)
    ref, sabs = c.ref()
    assert_close(f64(ybits), ref, c.tol(ref, sabs), "A4W4 quant-out y")
    q_ref, s_ref = oracle.act_quant(ybits)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(bq.unpack_scales(sf, c.M, c.N).cpu().numpy(), s_ref)


def test_a4w4_decode_layers_full_size():
    for N, K in ((4608, 1536), (6144, 1536), (1536, 6144)):
        A4Case(41, N, K, seed=N, bias=True).check_sampled(n=2000)


def test_a4w4_square_full_size():
    """8192 x 8192 x 8192 on packed E2M1 operands, sampled outputs."""
    M = N = K = 8192
    c = A4Case.__new__(A4Case)
    c.M, c.N, c.K, c.alpha, c.act, c.bias, c.res = M, N, K, 1.0, bq.BQ_ACT_NONE, None, None
    c.x = synth.activations(M, K, seed=4)
    c.b, c.bsf = synth.mxfp4_weight(N, K, seed=5)
    c.check_sampled(n=1500)


def test_a4w4_refusals():
    c = A4Case(300, 520, 640)
    aq, asf = bq.act_quant_mxfp4(dev_bf16(c.x))
    bd = dev_u8(c.b)
    bsf = bq.pack_weight_scales(dev_u8(c.bsf), bq.BQ_SF_ROW32, c.N, c.K)
    with pytest.raises(bq.BqError) as e:  # K % 128
        bq.gemm(bq.W_A4W4, aq, asf, bd, bsf, c.M, c.N, 608)
    assert e.value.status == bq.BQ_ERR_SHAPE
    with pytest.raises(bq.BqError) as e:  # the fused quantizer emits E4M3 only
        bq.gemm_bf16act(bq.W_A4W4, dev_bf16(c.x[:41]), bd, bsf, 41, c.N, c.K)
    assert e.value.status == bq.BQ_ERR_INVALID
