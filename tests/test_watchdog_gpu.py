"""Failure detection without a GPU fault: the bounded waits, the architecture
check and the non-finite reports (the hip_quant README's memory-safety
guards on the pages, restated for this library).

* Every barrier wait in the library's kernels gives up after a time limit,
  records the timeout (and the wait site) in the device error word and
  returns; bq_selftest_wait_timeout runs that same wait on a barrier nothing
  ever completes, with a short limit, so the test sees BQ_ERR_TIMEOUT through
  bq_device_status and then checks that the context still computes correctly.
  No trap, no fault, no kernel left waiting.
* bq_debug_override_compute_capability makes the arch check compare another
  compute capability, so every entry point must refuse with BQ_ERR_ARCH
  before launching anything (the outputs keep their sentinel).
* A quantized-output GEMM whose outputs overflow reports BQ_ERR_NONFINITE and
  never writes the NaN scale byte 255.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_quant_b200 as bq
from block_scaled_precision_quant_b200 import synth

pytestmark = pytest.mark.gpu


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _f64(y):
    return (y.cpu().view(torch.int16).numpy().view(np.uint16).astype(np.uint32) << 16) \
        .view(np.float32).astype(np.float64)


def _small_gemm_matches_oracle(seed=3):
    M, N, K = 64, 256, 512
    x = synth.activations(M, K, seed=seed)
    w, ws = synth.mxfp4_weight(N, K, seed=seed + 1)
    aq, asf = bq.act_quant(_dev_bf16(x))
    wsf = bq.pack_weight_scales(torch.from_numpy(ws).cuda(), bq.BQ_SF_ROW32, N, K)
    y = bq.gemm(bq.W_MXFP4, aq, asf, torch.from_numpy(w).cuda(), wsf, M, N, K)
    bq.device_status()
    q, s = oracle.act_quant(x)
    ref, sabs = oracle.gemm(q, s, w, ws, oracle.B_FP4, M, N, K)
    assert np.all(np.abs(_f64(y) - ref) <= oracle.gemm_tolerance(ref, sabs))


def test_bounded_wait_gives_up_and_reports_the_site():
    L = bq.lib()
    bq.device_status()  # start from a clear error word
    st = _stream()
    t0 = time.perf_counter()
    assert L.bq_selftest_wait_timeout(20000, st) == bq.BQ_OK  # 20 ms
    detail = ctypes.c_int(0)
    assert L.bq_device_status_detail(st, ctypes.byref(detail)) == bq.BQ_ERR_TIMEOUT
    waited = time.perf_counter() - t0
    assert detail.value & 1
    assert (detail.value >> 8) & 0xFF == 9  # the self-test's wait site
    assert waited >= 0.02
    # the status call cleared the word, and the context is intact
    assert L.bq_device_status(st) == bq.BQ_OK
    _small_gemm_matches_oracle()


def test_two_timeouts_keep_the_first_site():
    L = bq.lib()
    bq.device_status()
    st = _stream()
    for _ in range(2):
        assert L.bq_selftest_wait_timeout(1000, st) == bq.BQ_OK
    detail = ctypes.c_int(0)
    assert L.bq_device_status_detail(st, ctypes.byref(detail)) == bq.BQ_ERR_TIMEOUT
    assert detail.value == 1 | (9 << 8)


def test_selftest_limit_is_checked():
    L = bq.lib()
    for bad in (0, -5, 1000001):
        assert L.bq_selftest_wait_timeout(bad, _stream()) == bq.BQ_ERR_SHAPE
    bq.device_status()


def test_arch_override_refuses_every_entry_before_launching():
    L = bq.lib()
    M, N, K = 64, 256, 512
    x = _dev_bf16(synth.activations(M, K, seed=5))
    w, ws = synth.mxfp4_weight(N, K, seed=6)
    wd = torch.from_numpy(w).cuda()
    wsf = bq.pack_weight_scales(torch.from_numpy(ws).cuda(), bq.BQ_SF_ROW32, N, K)
    aq, asf = bq.act_quant(x)
    torch.cuda.synchronize()
    q_out = torch.full((M, K), 0x5A, dtype=torch.uint8, device="cuda")
    sf_out = torch.full((bq.sf_bytes(M, K),), 0x5A, dtype=torch.uint8, device="cuda")
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    ws_buf = torch.zeros((1 << 20,), dtype=torch.uint8, device="cuda")
    st = _stream()
    p = lambda t: t.data_ptr()  # noqa: E731
    assert L.bq_debug_override_compute_capability(9, 0) == bq.BQ_OK
    try:
        calls = {
            "act_quant": lambda: L.bq_act_quant(p(x), M, K, K, p(q_out), p(sf_out), None, None, st),
            "act_quant_mxfp4": lambda: L.bq_act_quant_mxfp4(p(x), M, K, K, p(q_out), p(sf_out),
                                                            None, None, st),
            "pack": lambda: L.bq_pack_weight_scales(p(wd), bq.BQ_SF_ROW32, N, K, p(sf_out), None,
                                                    st),
            "gemm": lambda: L.bq_gemm_mxfp8_mxfp4(p(aq), p(asf), p(wd), p(wsf), M, N, K, p(y), st),
            "gemm_epilogue": lambda: L.bq_gemm_mxfp8_mxfp4_epilogue(
                p(aq), p(asf), p(wd), p(wsf), M, N, K, p(y), None, None, p(ws_buf),
                ws_buf.numel(), None, st),
            "gemm_noalloc": lambda: L.bq_gemm_mxfp8_mxfp4_epilogue_noalloc(
                p(aq), p(asf), p(wd), p(wsf), M, N, K, p(y), None, None, None, st),
            "selftest": lambda: L.bq_selftest_wait_timeout(1000, st),
            "device_status": lambda: L.bq_device_status(st),
        }
        for name, call in calls.items():
            assert call() == bq.BQ_ERR_ARCH, name
        torch.cuda.synchronize()
    finally:
        assert L.bq_debug_override_compute_capability(-1, -1) == bq.BQ_OK
    # nothing ran: the outputs still hold their sentinels
    assert torch.all(q_out == 0x5A) and torch.all(sf_out == 0x5A)
    assert torch.all(y == 7.0)
    assert L.bq_device_status(st) == bq.BQ_OK
    assert L.bq_debug_override_compute_capability(100, 0) == bq.BQ_ERR_INVALID
    _small_gemm_matches_oracle(seed=11)


@pytest.mark.parametrize("M", [41, 200])  # swap-AB decode tile, wide tile
def test_quant_out_overflow_reports_nonfinite(M):
    """alpha = 2^123 drives some outputs past the bf16 range: the epilogue
    must flag BQ_ERR_NONFINITE, keep every scale byte valid (never 255), and
    give the groups that stay finite the quantizer's codes and scales."""
    N, K = 256, 512
    x = synth.activations(M, K, seed=21)
    w, ws = synth.mxfp4_weight(N, K, seed=22)
    aq, asf = bq.act_quant(_dev_bf16(x))
    wsf = bq.pack_weight_scales(torch.from_numpy(ws).cuda(), bq.BQ_SF_ROW32, N, K)
    y, q, sf = bq.gemm(bq.W_MXFP4, aq, asf, torch.from_numpy(w).cuda(), wsf, M, N, K,
                       alpha=2.0 ** 123, quantize_out=True)
    with pytest.raises(bq.BqError) as err:
        bq.device_status()
    assert err.value.status == bq.BQ_ERR_NONFINITE
    bq.device_status()  # cleared
    sf_row = bq.unpack_scales(sf, M, N).cpu().numpy()
    assert sf_row.max() <= 247
    ybits = y.cpu().view(torch.int16).numpy().view(np.uint16)
    groups = ybits.reshape(M, N // 32, 32)
    finite = np.all((groups & 0x7F80) != 0x7F80, axis=2)
    assert finite.any() and not finite.all()
    gq, gs = oracle.act_quant(groups[finite])
    qv = q.cpu().numpy().reshape(M, N // 32, 32)
    assert np.array_equal(qv[finite], gq)
    assert np.array_equal(sf_row[finite], gs[:, 0])
