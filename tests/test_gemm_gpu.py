"""Parity of the CUDA block-scaled GEMMs with the fp64 oracle.

Every output element must satisfy |y - ref| <= ulp_bf16(|ref|) + 2^-20 * S with
S = |alpha| sum_k |a_k b_k| (+ |bias| + |residual|, GELU branch scaled by 1.13),
where ref is the oracle's exact-decode fp64 result.  Small and mid sizes are
compared in full (several tiles plus ragged tails in M, N and K); the
workloads' full sizes are compared on sampled outputs, in the launch
configuration the benchmark uses.
"""
import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_quant_b200 as bq
from block_scaled_precision_quant_b200 import synth

pytestmark = pytest.mark.gpu

OKIND = {bq.W_MXFP4: oracle.B_FP4, bq.W_FP8BLK32: oracle.B_FP8BLK, bq.W_MXFP8: oracle.B_FP8ROW}


def to_dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_to_f64(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


class Case:
    """Inputs of one GEMM problem (host copies for the oracle, device copies
    for the CUDA path)."""

    def __init__(self, wk, M, N, K, seed=0, act_gp=None, bias=False, residual=False,
                 alpha=1.0, act=bq.BQ_ACT_NONE):
        self.wk, self.M, self.N, self.K = wk, M, N, K
        self.alpha, self.act = alpha, act
        self.x = synth.activations(M, K, seed=seed, group_pow2=act_gp)
        if wk == bq.W_MXFP4:
            self.b, self.bsf = synth.mxfp4_weight(N, K, seed=seed + 100)
        elif wk == bq.W_FP8BLK32:
            self.b, self.bsf = synth.fp8_weight_blk32(N, K, seed=seed + 100)
        else:
            w = synth.activations(N, K, seed=seed + 100)
            self.b, self.bsf = oracle.act_quant(w)
        self.bias = synth.bias(N, seed=seed + 200) if bias else None
        self.res = synth.residual(M, N, seed=seed + 300) if residual else None

    def gpu(self, config=None, batch=None):
        return self.gpu_with(config=config)

    def gpu_with(self, config=None, workspace=None):
        xd = to_dev_bf16(self.x)
        aq, asf = bq.act_quant(xd)
        bd = to_dev_u8(self.b)
        kind = bq.BQ_SF_BLK32x32 if self.wk == bq.W_FP8BLK32 else bq.BQ_SF_ROW32
        bsf = bq.pack_weight_scales(to_dev_u8(self.bsf), kind, self.N, self.K,
                                    e4m3_codes=bd if self.wk != bq.W_MXFP4 else None)
        y = bq.gemm(self.wk, aq, asf, bd, bsf, self.M, self.N, self.K,
                    bias=to_dev_bf16(self.bias) if self.bias is not None else None,
                    residual=to_dev_bf16(self.res) if self.res is not None else None,
                    alpha=self.alpha, act=self.act, config=config, workspace=workspace)
        bq.device_status()
        self.aq_gpu = aq.cpu().numpy()
        return bf16_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16))

    def oracle_full(self):
        aq, asf = oracle.act_quant(self.x)
        return oracle.gemm(aq, asf, self.b, self.bsf, OKIND[self.wk], self.M, self.N, self.K,
                           bias=self.bias, residual=self.res, alpha=self.alpha, act=self.act)

    def oracle_sampled(self, ms, ns):
        aq, asf = oracle.act_quant(self.x)
        return oracle.gemm_sampled(aq, asf, self.b, self.bsf, OKIND[self.wk], self.M, self.N,
                                   self.K, ms, ns, bias=self.bias, residual=self.res,
                                   alpha=self.alpha, act=self.act)

    def tol(self, ref, sabs, ms=None, ns=None):
        babs = None
        rabs = None
        if self.bias is not None:
            babs = np.abs(bf16_to_f64(self.bias))
            babs = babs[None, :] if ms is None else babs[ns]
        if self.res is not None:
            rabs = np.abs(bf16_to_f64(self.res))
            rabs = rabs if ms is None else rabs[ms, ns]
        return oracle.gemm_tolerance(ref, sabs, self.alpha, babs, rabs, self.act)


def assert_close(y, ref, tol, what=""):
    err = np.abs(y - ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{what}: {bad.shape[0]} of {err.size} outside tolerance; first "
                           f"{[(tuple(i), float(y[tuple(i)]), float(ref[tuple(i)])) for i in bad[:4]]}")


def run_full(case, config=None):
    y = case.gpu(config)
    ref, sabs = case.oracle_full()
    aq_oracle, _ = oracle.act_quant(case.x)
    assert np.array_equal(case.aq_gpu, aq_oracle)
    assert_close(y, ref, case.tol(ref, sabs), f"{case.wk} {case.M}x{case.N}x{case.K}")
    return y, ref, sabs


def run_sampled(case, n=4000, seed=0, config=None):
    y = case.gpu(config)
    rng = np.random.default_rng(seed)
    ms = rng.integers(0, case.M, n)
    ns = rng.integers(0, case.N, n)
    # always include the corners and the last tile's tail
    ms = np.concatenate([ms, [0, case.M - 1, 0, case.M - 1]])
    ns = np.concatenate([ns, [0, 0, case.N - 1, case.N - 1]])
    ref, sabs = case.oracle_sampled(ms, ns)
    assert_close(y[ms, ns], ref, case.tol(ref, sabs, ms, ns), f"{case.wk} sampled")


# ------------------------------------------------------------ small / mid --

@pytest.mark.parametrize("wk", [bq.W_MXFP4, bq.W_FP8BLK32, bq.W_MXFP8])
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (200, 264, 384), (257, 520, 256),
                                   (130, 128, 512)])
def test_multi_tile_ragged(wk, M, N, K):
    run_full(Case(wk, M, N, K, seed=M + N))


@pytest.mark.parametrize("wk", [bq.W_FP8BLK32, bq.W_MXFP8])
@pytest.mark.parametrize("K", [32, 96, 352, 640])
def test_k_tails(wk, K):
    run_full(Case(wk, 150, 136, K, seed=K))


def test_pr1_reference_config():
    """act_quant then MXFP8 x MXFP4, M=64 N=512 K=1024, A scaled by 2^U{-4..4}
    per group, no bias (compared in full)."""
    run_full(Case(bq.W_MXFP4, 64, 512, 1024, seed=0, act_gp=(-4, 4)))


@pytest.mark.parametrize("k_chunks", [1, 2])
@pytest.mark.parametrize("block_n", [128, 256])
@pytest.mark.parametrize("wk", [bq.W_MXFP4, bq.W_FP8BLK32])
def test_block_n_choices(block_n, wk, k_chunks):
    run_full(Case(wk, 300, 520, 640, seed=3), config=bq.config(block_n=block_n, split_k=1,
                                                                swap_ab=0, k_chunks=k_chunks))


@pytest.mark.parametrize("k_chunks", [1, 4])
@pytest.mark.parametrize("M", [7, 41])
def test_swap_k_chunks(M, k_chunks):
    """Swap-AB tiles with one or four 128-K chunks per stage (K = 10 chunks:
    the last stage is partial)."""
    run_full(Case(bq.W_MXFP4, M, 384, 1280, seed=M + k_chunks, bias=True),
             config=bq.config(split_k=1, swap_ab=1, k_chunks=k_chunks))


# ------------------------------------------------------------- epilogues --

@pytest.mark.parametrize("wk", [bq.W_MXFP4, bq.W_FP8BLK32])
@pytest.mark.parametrize("bias,res,act,alpha", [(True, False, bq.BQ_ACT_NONE, 1.0),
                                                (False, True, bq.BQ_ACT_NONE, 1.0),
                                                (True, True, bq.BQ_ACT_NONE, 0.5),
                                                (True, False, bq.BQ_ACT_GELU, 1.0),
                                                (False, False, bq.BQ_ACT_GELU, 2.0)])
def test_epilogues(wk, bias, res, act, alpha):
    run_full(Case(wk, 190, 264, 256, seed=7, bias=bias, residual=res, act=act, alpha=alpha))


# ------------------------------------------------- decode: swap + split-K --

@pytest.mark.parametrize("M", [1, 17, 41, 64])
@pytest.mark.parametrize("split", [0, 1, 3])
def test_decode_swap_split(M, split):
    c = Case(bq.W_MXFP4, M, 640, 1536, seed=M, bias=True)
    run_full(c, config=bq.config(split_k=split, swap_ab=1))


@pytest.mark.parametrize("M", [1, 17, 41, 64])
@pytest.mark.parametrize("split", [2, 4, 8])
def test_decode_cluster_split(M, split):
    """K slices of a tile in one thread-block cluster, reduced through DSMEM."""
    c = Case(bq.W_MXFP4, M, 640, 1536, seed=M + split, bias=True, residual=(split == 4))
    cfg = bq.config(split_k=split, swap_ab=1, split_mode=bq.BQ_SPLIT_CLUSTER)
    assert bq.workspace_bytes(bq.W_MXFP4, M, 640, 1536, 1, cfg) == 0
    run_full(c, config=cfg)


@pytest.mark.parametrize("wk", [bq.W_FP8BLK32, bq.W_MXFP8])
def test_decode_cluster_split_fp8_weights(wk):
    cfg = bq.config(split_k=8, swap_ab=1, split_mode=bq.BQ_SPLIT_CLUSTER)
    run_full(Case(wk, 41, 384, 2048, seed=5, residual=True, alpha=0.5), config=cfg)


def test_cluster_split_persistent_tiles():
    """More clusters of work than fit at once: clusters loop over several tiles
    (the partial buffer is reused after every peer finished reading it)."""
    cfg = bq.config(split_k=8, swap_ab=1, split_mode=bq.BQ_SPLIT_CLUSTER)
    run_full(Case(bq.W_MXFP4, 33, 8192, 1024, seed=8, bias=True), config=cfg)


def test_decode_auto_plan_uses_no_workspace():
    for N, K in ((4608, 1536), (6144, 1536), (1536, 6144)):
        assert bq.workspace_bytes(bq.W_MXFP4, 41, N, K, 1) == 0


@pytest.mark.parametrize("M", [1, 17, 41, 64])
@pytest.mark.parametrize("split", [2, 3, 4, 12])
def test_decode_swap_workspace_split(M, split):
    """Swap-AB split-K through the workspace: partial rows m < M only, the
    last slice sums all slices in slice order (its own from TMEM)."""
    c = Case(bq.W_MXFP4, M, 640, 1536, seed=M + 7 * split, bias=True,
             residual=(split == 3), act=bq.BQ_ACT_GELU if split == 4 else bq.BQ_ACT_NONE)
    run_full(c, config=bq.config(split_k=split, swap_ab=1, split_mode=bq.BQ_SPLIT_WORKSPACE))


def test_workspace_split_persistent_tiles():
    """More split units than CTAs: each CTA walks several tiles, reusing its
    staging buffer and ticket flag."""
    cfg = bq.config(split_k=4, swap_ab=1, split_mode=bq.BQ_SPLIT_WORKSPACE)
    run_full(Case(bq.W_MXFP4, 33, 8192, 1024, seed=18, bias=True), config=cfg)


@pytest.mark.parametrize("wk", [bq.W_FP8BLK32, bq.W_MXFP8])
def test_decode_fp8_weights(wk):
    run_full(Case(wk, 41, 384, 1024, seed=2, residual=True), config=bq.config(swap_ab=1))


def test_decode_without_swap():
    run_full(Case(bq.W_MXFP4, 41, 640, 1536, seed=9, bias=True),
             config=bq.config(swap_ab=0, split_k=1))


# ------------------------------------------------------------ CTA pairs --

PAIR = dict(split_k=1, swap_ab=0, cta_pair=2)


@pytest.mark.parametrize("kc", [1, 2])
def test_pair_tiles_ragged(kc):
    """256x256 tiles on CTA pairs (one cta_group::2 MMA per K step): ragged
    M, N and K, several tiles each way, both stage shapes."""
    c = Case(bq.W_MXFP4, 300, 520, 640, seed=61 + kc, bias=True)
    run_full(c, config=bq.config(k_chunks=kc, **PAIR))


@pytest.mark.parametrize("wk", [bq.W_FP8BLK32, bq.W_MXFP8])
def test_pair_tiles_fp8_weights_residual(wk):
    c = Case(wk, 512, 768, 512, seed=63, residual=True, alpha=0.75)
    run_full(c, config=bq.config(**PAIR))


def test_pair_tiles_persistent_gelu():
    """More pair tiles than pairs of SMs: each pair walks several tiles (the
    accumulator handed back by both CTAs' epilogues each time)."""
    c = Case(bq.W_MXFP4, 1280, 2048, 256, seed=64, bias=True, act=bq.BQ_ACT_GELU)
    run_full(c, config=bq.config(**PAIR))


def test_pair_tiles_batched_broadcast():
    count, M, N, K = 3, 260, 264, 384
    xs = [synth.activations(M, K, seed=70 + i) for i in range(count)]
    b, bsf = synth.mxfp4_weight(N, K, seed=75)
    bias = synth.bias(N, seed=76)
    aqs, sfs = zip(*[bq.act_quant(to_dev_bf16(x)) for x in xs])
    aq = torch.stack(aqs)
    asf = torch.stack(sfs)
    bsf_d = bq.pack_weight_scales(to_dev_u8(bsf), bq.BQ_SF_ROW32, N, K)
    y = bq.gemm(bq.W_MXFP4, aq.reshape(count * M, K), asf, to_dev_u8(b), bsf_d, M, N, K,
                bias=to_dev_bf16(bias), act=bq.BQ_ACT_GELU, config=bq.config(**PAIR),
                batch=dict(count=count, stride_a=M * K, stride_a_sf=asf.shape[1], stride_b=0,
                           stride_b_sf=0, stride_y=M * N * 2))
    bq.device_status()
    yb = bf16_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    for i, x in enumerate(xs):
        q, s = oracle.act_quant(x)
        ref, sabs = oracle.gemm(q, s, b, bsf, oracle.B_FP4, M, N, K, bias=bias,
                                act=bq.BQ_ACT_GELU)
        tol = oracle.gemm_tolerance(ref, sabs, 1.0, np.abs(bf16_to_f64(bias))[None, :], None,
                                    bq.BQ_ACT_GELU)
        assert_close(yb[i], ref, tol, f"pair batch {i}")


@pytest.mark.parametrize("cfg", [dict(split_k=1, swap_ab=0, block_n=256),
                                 dict(split_k=1, swap_ab=0, block_n=128, k_chunks=2), PAIR])
@pytest.mark.parametrize("layout", ["strided", "per_problem", "broadcast"])
def test_residual_layouts(cfg, layout):
    """The wide tiles load the residual tile by tile into the output staging
    buffer: a row pitch wider than N, one residual per problem, and one
    residual broadcast to every problem (batch stride 0)."""
    count = 1 if layout == "strided" else 2
    M, N, K, ld = 300, 296, 384, 296 + 40
    xs = [synth.activations(M, K, seed=110 + i) for i in range(count)]
    b, bsf = synth.mxfp4_weight(N, K, seed=115)
    nres = 1 if layout == "broadcast" else count
    res = [synth.residual(M, N, seed=120 + i) for i in range(nres)]
    wide = np.zeros((nres, M, ld), np.uint16)
    for i in range(nres):
        wide[i, :, :N] = res[i]
        wide[i, :, N:] = 0x7FC0  # NaN outside the view: must never be read
    res_d = to_dev_bf16(wide)[:, :, :N]
    aqs, sfs = zip(*[bq.act_quant(to_dev_bf16(x)) for x in xs])
    aq = torch.stack(aqs).reshape(count * M, K)
    asf = torch.stack(sfs)
    bsf_d = bq.pack_weight_scales(to_dev_u8(bsf), bq.BQ_SF_ROW32, N, K)
    batch = None
    if count > 1:
        batch = dict(count=count, stride_a=M * K, stride_a_sf=asf.shape[1], stride_b=0,
                     stride_b_sf=0, stride_y=M * N * 2,
                     stride_res=0 if layout == "broadcast" else M * ld * 2)
    y = bq.gemm(bq.W_MXFP4, aq, asf if count > 1 else asf[0], to_dev_u8(b), bsf_d, M, N, K,
                residual=res_d if count > 1 else res_d[0], batch=batch,
                config=bq.config(**cfg))
    bq.device_status()
    yb = bf16_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16)).reshape(count, M, N)
    for i, x in enumerate(xs):
        q, s = oracle.act_quant(x)
        r = res[0 if layout == "broadcast" else i]
        ref, sabs = oracle.gemm(q, s, b, bsf, oracle.B_FP4, M, N, K, residual=r)
        tol = oracle.gemm_tolerance(ref, sabs, 1.0, None, np.abs(bf16_to_f64(r)), 0)
        assert_close(yb[i], ref, tol, f"{layout} {cfg} problem {i}")


def test_pair_tiles_refusals():
    c = Case(bq.W_MXFP4, 300, 520, 640)
    for cfg in (bq.config(split_k=2, swap_ab=0, cta_pair=2),
                bq.config(swap_ab=1, cta_pair=2),
                bq.config(block_n=128, split_k=1, swap_ab=0, cta_pair=2),
                bq.config(split_k=1, swap_ab=0, cta_pair=3)):
        with pytest.raises(bq.BqError) as e:
            c.gpu(cfg)
        assert e.value.status == bq.BQ_ERR_INVALID


def test_split_k_non_swap():
    run_full(Case(bq.W_FP8BLK32, 256, 384, 2048, seed=4, residual=True),
             config=bq.config(swap_ab=0, split_k=4, block_n=128))


@pytest.mark.parametrize("M", [17, 41])
def test_decode_workspace_split_balanced(M):
    """Workspace split-K with a slice count that does not divide the K blocks."""
    run_full(Case(bq.W_MXFP4, M, 640, 1536, seed=M + 1, bias=True),
             config=bq.config(split_k=5, swap_ab=1, split_mode=bq.BQ_SPLIT_WORKSPACE))


def test_split_k_repeatable():
    """Fixed slice order: repeated launches give identical bits."""
    c = Case(bq.W_MXFP4, 41, 1536, 6144, seed=1, bias=True)
    y0 = c.gpu()
    for _ in range(3):
        assert np.array_equal(c.gpu(), y0)


@pytest.mark.parametrize("N,K", [(4608, 1536), (6144, 1536), (1536, 6144)])
def test_decode_workload_full(N, K):
    """Decode-shaped linear (M=41, fused bias), compared in full."""
    run_full(Case(bq.W_MXFP4, 41, N, K, seed=1, bias=True))


# ----------------------------------------------------------------- batch --

@pytest.mark.parametrize("cfg", [None, dict(split_k=1, swap_ab=0, block_n=256),
                                 dict(split_k=1, swap_ab=0, block_n=128)])
def test_batched_broadcast_weight_bias_gelu(cfg):
    """Independent problems over one broadcast weight (stride 0), bias+GELU, in
    the built-in schedule and on both wide tile widths (3-D output stores)."""
    count, M, N, K = 3, 200, 264, 256
    xs = [synth.activations(M, K, seed=40 + i) for i in range(count)]
    b, bsf = synth.mxfp4_weight(N, K, seed=50)
    bias = synth.bias(N, seed=51)
    aqs, sfs = zip(*[bq.act_quant(to_dev_bf16(x)) for x in xs])
    aq = torch.stack(aqs)
    asf = torch.stack(sfs)
    bsf_d = bq.pack_weight_scales(to_dev_u8(bsf), bq.BQ_SF_ROW32, N, K)
    y = bq.gemm(bq.W_MXFP4, aq, asf, to_dev_u8(b), bsf_d, M, N, K, bias=to_dev_bf16(bias),
                act=bq.BQ_ACT_GELU, config=bq.config(**cfg) if cfg else None,
                batch=dict(count=count, stride_a=M * K, stride_a_sf=asf.shape[1], stride_b=0,
                           stride_b_sf=0, stride_y=M * N * 2))
    bq.device_status()
    yv = bf16_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    for i in range(count):
        q, s = oracle.act_quant(xs[i])
        ref, sabs = oracle.gemm(q, s, b, bsf, oracle.B_FP4, M, N, K, bias=bias,
                                act=oracle.ACT_GELU)
        tol = oracle.gemm_tolerance(ref, sabs, 1.0, np.abs(bf16_to_f64(bias))[None, :], None,
                                    oracle.ACT_GELU)
        assert_close(yv[i], ref, tol, f"batch {i}")


# ------------------------------------------------------- full-size sampled --

def test_fp8blk32_residual_full_size():
    """FP8 E4M3 weights with 32x32 block scales, 1024 x 4096 x 4096, residual."""
    run_sampled(Case(bq.W_FP8BLK32, 1024, 4096, 4096, seed=2, residual=True), n=3000)


def test_square_mxfp8_full_size():
    """Square MXFP8 x MXFP8 GEMM, 8192^3, alpha 1."""
    run_sampled(Case(bq.W_MXFP8, 8192, 8192, 8192, seed=3), n=600)


def test_batched_mlp_up_full_size():
    """The MLP workload's up-projection at full size: 8 problems of 1024 x 2048 x 2048 over
    one broadcast MXFP4 weight (stride 0), bias + GELU, in the dispatch's own schedule;
    sampled outputs of every problem against the oracle."""
    count, M, N, K = 8, 1024, 2048, 2048
    xs = [synth.activations(M, K, seed=60 + i) for i in range(count)]
    b, bsf = synth.mxfp4_weight(N, K, seed=70)
    bias = synth.bias(N, seed=71)
    aqs, sfs = zip(*[bq.act_quant(to_dev_bf16(x)) for x in xs])
    aq = torch.stack(aqs)
    asf = torch.stack(sfs)
    bsf_d = bq.pack_weight_scales(to_dev_u8(bsf), bq.BQ_SF_ROW32, N, K)
    y = bq.gemm(bq.W_MXFP4, aq, asf, to_dev_u8(b), bsf_d, M, N, K, bias=to_dev_bf16(bias),
                act=bq.BQ_ACT_GELU,
                batch=dict(count=count, stride_a=M * K, stride_a_sf=asf.shape[1], stride_b=0,
                           stride_b_sf=0, stride_y=M * N * 2))
    bq.device_status()
    yv = bf16_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    babs = np.abs(bf16_to_f64(bias))
    rng = np.random.default_rng(6)
    for i in range(count):
        ms = np.concatenate([rng.integers(0, M, 400), [0, M - 1, 0, M - 1]])
        ns = np.concatenate([rng.integers(0, N, 400), [0, 0, N - 1, N - 1]])
        q, sc = oracle.act_quant(xs[i])
        ref, sabs = oracle.gemm_sampled(q, sc, b, bsf, oracle.B_FP4, M, N, K, ms, ns,
                                        bias=bias, act=oracle.ACT_GELU)
        tol = oracle.gemm_tolerance(ref, sabs, 1.0, babs[ns], None, oracle.ACT_GELU)
        assert_close(yv[i][ms, ns], ref, tol, f"batched MLP up, problem {i}")


def test_down_projection_full_size():
    """Down-projection 4096 x 1536 x 6144, MXFP4 weights."""
    run_sampled(Case(bq.W_MXFP4, 4096, 1536, 6144, seed=4), n=3000)


# ---------------------------------------------------------------- errors --

def test_argument_errors():
    c = Case(bq.W_MXFP4, 16, 128, 128)
    aq, asf = bq.act_quant(to_dev_bf16(c.x))
    bd = to_dev_u8(c.b)
    bsf = bq.pack_weight_scales(to_dev_u8(c.bsf), bq.BQ_SF_ROW32, 128, 128)
    with pytest.raises(bq.BqError) as e:  # N not a multiple of 8
        bq.gemm(bq.W_MXFP4, aq, asf, bd, bsf, 16, 124, 128)
    assert e.value.status == bq.BQ_ERR_SHAPE
    with pytest.raises(bq.BqError) as e:  # FP4 weights need K % 128 == 0
        bq.gemm(bq.W_MXFP4, aq, asf, bd, bsf, 16, 128, 96)
    assert e.value.status == bq.BQ_ERR_SHAPE
    c2 = Case(bq.W_MXFP4, 16, 128, 512)  # operands sized for K = 512 (4 K blocks)
    aq2, asf2 = bq.act_quant(to_dev_bf16(c2.x))
    bd2 = to_dev_u8(c2.b)
    bsf2 = bq.pack_weight_scales(to_dev_u8(c2.bsf), bq.BQ_SF_ROW32, 128, 512)
    with pytest.raises(bq.BqError) as e:  # workspace split-K without a workspace
        f = bq.lib().bq_gemm_mxfp8_mxfp4_epilogue
        cfg = bq.config(split_k=2, swap_ab=1, split_mode=bq.BQ_SPLIT_WORKSPACE)
        import ctypes
        st = f(aq2.data_ptr(), asf2.data_ptr(), bd2.data_ptr(), bsf2.data_ptr(), 16, 128, 512,
               torch.empty((16, 128), dtype=torch.bfloat16, device="cuda").data_ptr(), None, None,
               None, 0, ctypes.byref(cfg), None)
        bq._check(st, "split without workspace")
    assert e.value.status == bq.BQ_ERR_WORKSPACE
    with pytest.raises(bq.BqError) as e:  # cluster split needs a power-of-two slice count
        bq.gemm(bq.W_MXFP4, aq2, asf2, bd2, bsf2, 16, 128, 512,
                config=bq.config(split_k=3, swap_ab=1, split_mode=bq.BQ_SPLIT_CLUSTER))
    assert e.value.status == bq.BQ_ERR_INVALID
    with pytest.raises(bq.BqError) as e:  # invalid enum
        bq.gemm(bq.W_MXFP4, aq, asf, bd, bsf, 16, 128, 128, act=7)
    assert e.value.status == bq.BQ_ERR_INVALID


def test_pack_refuses_nan_scale_and_code():
    s = np.full((64, 4), 127, np.uint8)
    s[5, 2] = 255
    with pytest.raises(bq.BqError) as e:
        bq.pack_weight_scales(to_dev_u8(s), bq.BQ_SF_ROW32, 64, 128)
    assert e.value.status == bq.BQ_ERR_NAN_SCALE
    codes = np.zeros((64, 128), np.uint8)
    codes[7, 99] = 0xFF
    with pytest.raises(bq.BqError) as e:
        bq.pack_weight_scales(to_dev_u8(np.full((2, 4), 127, np.uint8)), bq.BQ_SF_BLK32x32, 64,
                              128, e4m3_codes=to_dev_u8(codes))
    assert e.value.status == bq.BQ_ERR_NAN_CODE


def test_pack_layout_blk32():
    """BLK32x32 scales repeat over the 32 rows of their block; padding is 127."""
    N, K = 100, 160
    s = synth.uniform_bytes(((N + 31) // 32, K // 32), seed=1, lo=100, hi=140)
    out = bq.pack_weight_scales(to_dev_u8(s), bq.BQ_SF_BLK32x32, N, K)
    rows = bq.unpack_scales(out, N, K).cpu().numpy()
    assert np.array_equal(rows, np.repeat(s, 32, axis=0)[:N])


def test_workspace_shared_across_problems():
    """One workspace serves a sequence of split-K problems of different
    shapes; the ticket region is zero again after every call."""
    shapes = [(41, 640, 1536, 5), (17, 1536, 6144, 12), (64, 384, 1024, 3), (5, 4608, 1536, 4)]
    mode = bq.BQ_SPLIT_WORKSPACE
    need = max(bq.workspace_bytes(bq.W_MXFP4, M, N, K, 1,
                                  bq.config(split_k=s, swap_ab=1, split_mode=mode))
               for M, N, K, s in shapes)
    ws = torch.zeros((need,), dtype=torch.uint8, device="cuda")
    for i, (M, N, K, s) in enumerate(shapes * 2):
        c = Case(bq.W_MXFP4, M, N, K, seed=60 + i, bias=True)
        y = c.gpu_with(config=bq.config(split_k=s, swap_ab=1, split_mode=mode), workspace=ws)
        ref, sabs = c.oracle_full()
        assert_close(y, ref, c.tol(ref, sabs), f"shared workspace {M}x{N}x{K}/{s}")
        assert int(ws[:65536].count_nonzero().item()) == 0


# ------------------------------------------------- quantized GEMM output --

def _quant_out_case(c, config=None, write_y=True):
    """GEMM with the MXFP8 output: y within tolerance of the oracle, and the
    codes and scales (padding included) byte-equal to act_quant of y."""
    aq, asf = bq.act_quant(to_dev_bf16(c.x))
    bd = to_dev_u8(c.b)
    kind = bq.BQ_SF_BLK32x32 if c.wk == bq.W_FP8BLK32 else bq.BQ_SF_ROW32
    bsf = bq.pack_weight_scales(to_dev_u8(c.bsf), kind, c.N, c.K,
                                e4m3_codes=bd if c.wk != bq.W_MXFP4 else None)
    kw = dict(bias=to_dev_bf16(c.bias) if c.bias is not None else None,
              residual=to_dev_bf16(c.res) if c.res is not None else None,
              alpha=c.alpha, act=c.act, config=config)
    y, q, sf = bq.gemm(c.wk, aq, asf, bd, bsf, c.M, c.N, c.K, quantize_out=True, **kw)
    bq.device_status()
    ref, sabs = c.oracle_full()
    yv = bf16_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    assert_close(yv, ref, c.tol(ref, sabs), "quantized-output GEMM y")
    q_ref, sf_ref = bq.act_quant(y)
    assert torch.equal(q, q_ref)
    assert torch.equal(sf, sf_ref)
    oq, osf = oracle.act_quant(y.cpu().view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(bq.unpack_scales(sf, c.M, c.N).cpu().numpy(), osf)
    if not write_y:
        y2, q2, sf2 = bq.gemm(c.wk, aq, asf, bd, bsf, c.M, c.N, c.K, quantize_out=True,
                              write_y=False, **kw)
        bq.device_status()
        assert y2 is None and torch.equal(q2, q) and torch.equal(sf2, sf)


@pytest.mark.parametrize("M,N,K,write_y,bn", [(300, 800, 640, True, 128), (128, 512, 256, False, 128),
                                               (300, 800, 640, True, 256),
                                               (136, 544, 384, False, 256)])
def test_quant_out_wide_tiles(M, N, K, write_y, bn):
    # 128 x 256 tiles keep one accumulator and read all of a row's chunks into
    # registers before the stores; N = 800 and 544 end in a tile of one
    # 32-column chunk, where the second epilogue group has no chunk at all.
    _quant_out_case(Case(bq.W_MXFP4, M, N, K, seed=81, bias=True, act=bq.BQ_ACT_GELU),
                    config=bq.config(split_k=1, swap_ab=0, block_n=bn), write_y=write_y)


def test_quant_out_pair_tiles():
    _quant_out_case(Case(bq.W_FP8BLK32, 520, 800, 512, seed=82, residual=True),
                    config=bq.config(split_k=1, swap_ab=0, cta_pair=2), write_y=True)


@pytest.mark.parametrize("M,N", [(41, 1536), (17, 800), (64, 640)])
def test_quant_out_decode(M, N):
    _quant_out_case(Case(bq.W_MXFP4, M, N, 1536, seed=83 + M, bias=True), write_y=(M != 17))


def test_quant_out_auto_schedule_does_not_split():
    """A long-K decode shape the automatic schedule would split: with the
    quantized output it runs unsplit."""
    _quant_out_case(Case(bq.W_MXFP4, 41, 1536, 6144, seed=85, bias=True))


def test_quant_out_refusals():
    c = Case(bq.W_MXFP4, 41, 520, 512)
    aq, asf = bq.act_quant(to_dev_bf16(c.x))
    bd = to_dev_u8(c.b)
    bsf = bq.pack_weight_scales(to_dev_u8(c.bsf), bq.BQ_SF_ROW32, 520, 512)
    with pytest.raises(bq.BqError) as e:  # N % 32 != 0
        bq.gemm(bq.W_MXFP4, aq, asf, bd, bsf, 41, 520, 512, quantize_out=True)
    assert e.value.status == bq.BQ_ERR_SHAPE
    c2 = Case(bq.W_MXFP4, 41, 512, 512)
    aq2, asf2 = bq.act_quant(to_dev_bf16(c2.x))
    bsf2 = bq.pack_weight_scales(to_dev_u8(c2.bsf), bq.BQ_SF_ROW32, 512, 512)
    with pytest.raises(bq.BqError) as e:  # explicit split-K
        bq.gemm(bq.W_MXFP4, aq2, asf2, to_dev_u8(c2.b), bsf2, 41, 512, 512, quantize_out=True,
                config=bq.config(split_k=2, swap_ab=1))
    assert e.value.status == bq.BQ_ERR_INVALID


# ------------------------------------- act_quant fused into the decode GEMM --

def _fused_case(c, quantize_out=False, check_oracle=True,
                ref_config=bq.config(split_k=1, swap_ab=1, k_chunks=4)):
    """bq_gemm_bf16act_epilogue against bq_act_quant + the epilogue GEMM: y,
    the stored activation codes / scales and the status word bit for bit;
    y within tolerance of the oracle."""
    xd = to_dev_bf16(c.x)
    bd = to_dev_u8(c.b)
    kind = bq.BQ_SF_BLK32x32 if c.wk == bq.W_FP8BLK32 else bq.BQ_SF_ROW32
    bsf = bq.pack_weight_scales(to_dev_u8(c.bsf), kind, c.N, c.K,
                                e4m3_codes=bd if c.wk != bq.W_MXFP4 else None)
    kw = dict(bias=to_dev_bf16(c.bias) if c.bias is not None else None,
              residual=to_dev_bf16(c.res) if c.res is not None else None,
              alpha=c.alpha, act=c.act)
    st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
    aq, asf = bq.act_quant(xd, status=st_ref)
    ref2 = bq.gemm(c.wk, aq, asf, bd, bsf, c.M, c.N, c.K, quantize_out=quantize_out,
                   config=ref_config, **kw)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = bq.gemm_bf16act(c.wk, xd, bd, bsf, c.M, c.N, c.K, store_act=True, status=st,
                          quantize_out=quantize_out, **kw)
    bq.device_status()
    if quantize_out:
        y, q, sf, gq, gsf = got
        y_ref, q_ref, sf_ref = ref2
        assert torch.equal(q, q_ref) and torch.equal(sf, sf_ref)
    else:
        y, gq, gsf = got
        y_ref = ref2
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(gq, aq) and torch.equal(gsf, asf)
    assert int(st.item()) == int(st_ref.item())
    if not check_oracle:  # a non-finite input: y carries NaN; equality above is the check
        return int(st.item())
    ref, sabs = c.oracle_full()
    yv = bf16_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
    assert_close(yv, ref, c.tol(ref, sabs), "fused act_quant GEMM")


@pytest.mark.parametrize("M", [1, 17, 41, 64])
def test_fused_act_quant_decode(M):
    """M = 41 takes the decode layer 41x4608x1536, which the library splits
    over a 4-CTA cluster: the call quantizes into the activation buffers and
    runs that split GEMM, so it is compared with the automatic schedule."""
    _fused_case(Case(bq.W_MXFP4, M, 4608 if M == 41 else 520, 640 if M != 41 else 1536,
                     seed=90 + M, bias=True),
                ref_config=None if M == 41 else bq.config(split_k=1, swap_ab=1, k_chunks=4))


@pytest.mark.parametrize("wk", [bq.W_FP8BLK32, bq.W_MXFP8])
def test_fused_act_quant_fp8_weights(wk):
    _fused_case(Case(wk, 41, 384, 1024, seed=95, residual=True, alpha=0.5))


def test_fused_act_quant_long_k_split():
    """A 6144-deep decode projection: the call quantizes into the activation
    buffers and runs the split GEMM; same results as the two calls."""
    _fused_case(Case(bq.W_MXFP4, 41, 1536, 6144, seed=98, bias=True), ref_config=None)


def test_fused_act_quant_gelu_quant_out():
    _fused_case(Case(bq.W_MXFP4, 33, 1536, 6144, seed=96, bias=True, act=bq.BQ_ACT_GELU),
                quantize_out=True)


def test_fused_act_quant_nonfinite_and_refusals():
    c = Case(bq.W_MXFP4, 8, 256, 256, seed=97)
    x = c.x.copy()
    x[3, 77] = 0x7F80  # +Inf
    c.x = x
    assert _fused_case(c, check_oracle=False) & 1  # status bit, codes as bq_act_quant's
    xd = to_dev_bf16(c.x)
    bsf = bq.pack_weight_scales(to_dev_u8(c.bsf), bq.BQ_SF_ROW32, 256, 256)
    for M, K in ((65, 256), (8, 192)):  # M > 64, K % 128 != 0
        xs = to_dev_bf16(synth.activations(M, K, seed=1))
        with pytest.raises(bq.BqError) as e:
            bq.gemm_bf16act(bq.W_MXFP8, xs, torch.zeros((256, K), dtype=torch.uint8,
                                                         device="cuda"),
                            bsf, M, 256, K)
        assert e.value.status in (bq.BQ_ERR_SHAPE,)
