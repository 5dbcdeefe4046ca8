"""The allocation-free GEMM entry point (bq_gemm_mxfp8_mxfp4_epilogue_noalloc).

Some callers cannot allocate device memory (a plugin given only its inputs and
outputs, a serving loop with a fixed memory budget); this entry point runs the
K-split MXFP4 GEMM on a scratch array the library owns.  The test calls it
through the C ABI twice in a row (the second call finds the first call's
leftovers in the shared scratch) and checks each result against the oracle's
fp64 reference, within the tolerance the parity tests use, and bit for bit
against the existing workspace entry point (both reduce the K slices in the
same fixed order).  The file is named to be collected last; it passes on its
own in a fresh process too.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_quant_b200 as bq
from block_scaled_precision_quant_b200 import synth

pytestmark = pytest.mark.gpu


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _f64(y):
    return (y.cpu().view(torch.int16).numpy().view(np.uint16).astype(np.uint32) << 16) \
        .view(np.float32).astype(np.float64)


def test_noalloc_matches_workspace_entry_twice():
    L = bq.lib()
    M, N, K = 41, 4608, 1536
    cfg = bq.config(split_k=4, swap_ab=1, split_mode=bq.BQ_SPLIT_WORKSPACE)
    need = bq.workspace_bytes(bq.W_MXFP4, M, N, K, 1, cfg)
    assert 0 < need <= L.bq_noalloc_scratch_bytes()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        x = synth.activations(M, K, seed=70 + call)
        w, ws = synth.mxfp4_weight(N, K, seed=80 + call)
        bias = synth.bias(N, seed=90 + call)
        aq, asf = bq.act_quant(_dev_bf16(x))
        wd = torch.from_numpy(w).cuda()
        wsf = bq.pack_weight_scales(torch.from_numpy(ws).cuda(), bq.BQ_SF_ROW32, N, K)
        bd = _dev_bf16(bias)
        epi = bq.Epilogue(bd.data_ptr(), None, 0, 1.0, bq.BQ_ACT_NONE)

        y_new = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = L.bq_gemm_mxfp8_mxfp4_epilogue_noalloc(
            aq.data_ptr(), asf.data_ptr(), wd.data_ptr(), wsf.data_ptr(), M, N, K,
            y_new.data_ptr(), ctypes.byref(epi), None, ctypes.byref(cfg), stream)
        assert st == bq.BQ_OK, bq.status_string(st)

        work = torch.zeros((need,), dtype=torch.uint8, device="cuda")
        y_old = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = L.bq_gemm_mxfp8_mxfp4_epilogue(
            aq.data_ptr(), asf.data_ptr(), wd.data_ptr(), wsf.data_ptr(), M, N, K,
            y_old.data_ptr(), ctypes.byref(epi), None, work.data_ptr(), need,
            ctypes.byref(cfg), stream)
        assert st == bq.BQ_OK, bq.status_string(st)
        bq.device_status()

        q, s = oracle.act_quant(x)
        assert np.array_equal(aq.cpu().numpy(), q)
        ref, sabs = oracle.gemm(q, s, w, ws, oracle.B_FP4, M, N, K, bias=bias)
        babs = np.abs((bias.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
        tol = oracle.gemm_tolerance(ref, sabs, 1.0, babs[None, :])
        new = _f64(y_new)
        assert np.all(np.isfinite(new))
        assert np.all(np.abs(new - ref) <= tol), f"call {call}: outside the oracle tolerance"
        assert torch.equal(y_new.view(torch.int16), y_old.view(torch.int16)), \
            f"call {call}: differs from the workspace entry point"


def test_noalloc_rejects_problems_beyond_the_scratch():
    L = bq.lib()
    M, N, K = 64, 16384, 4096
    cfg = bq.config(split_k=16, swap_ab=1, split_mode=bq.BQ_SPLIT_WORKSPACE)
    assert bq.workspace_bytes(bq.W_MXFP4, M, N, K, 1, cfg) > L.bq_noalloc_scratch_bytes()
    dummy = torch.zeros((1 << 20,), dtype=torch.uint8, device="cuda")
    st = L.bq_gemm_mxfp8_mxfp4_epilogue_noalloc(
        dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), M, N, K,
        dummy.data_ptr(), None, None, ctypes.byref(cfg),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bq.BQ_ERR_WORKSPACE


def test_noalloc_checks_arguments_like_the_workspace_entry():
    """Argument errors come first and in the same order as the workspace entry
    point's: a NULL output is BQ_ERR_NULL even for a problem too large for the
    scratch, and a misaligned one BQ_ERR_ALIGN, before anything is enqueued."""
    L = bq.lib()
    M, N, K = 64, 16384, 4096
    cfg = bq.config(split_k=16, swap_ab=1, split_mode=bq.BQ_SPLIT_WORKSPACE)
    dummy = torch.zeros((1 << 20,), dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for y, want in ((None, bq.BQ_ERR_NULL), (p + 2, bq.BQ_ERR_ALIGN)):
        st_new = L.bq_gemm_mxfp8_mxfp4_epilogue_noalloc(p, p, p, p, M, N, K, y, None, None,
                                                        ctypes.byref(cfg), stream)
        st_old = L.bq_gemm_mxfp8_mxfp4_epilogue(p, p, p, p, M, N, K, y, None, None, None, 0,
                                                ctypes.byref(cfg), stream)
        assert st_new == st_old == want
