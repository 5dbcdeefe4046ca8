"""Host-side checks of the C-ABI library: it builds, loads without a GPU, and
exports every entry point include/bq.h declares.  No compute call is made."""
import ctypes
import os
import re

import pytest

import block_scaled_precision_quant_b200 as bq
from block_scaled_precision_quant_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "bq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bq_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return bq.lib()


def test_header_declares_the_entry_points():
    names = declared_entry_points()
    for required in ("bq_act_quant", "bq_pack_weight_scales", "bq_gemm_mxfp8_mxfp4",
                     "bq_gemm_mxfp8_fp8blk32", "bq_gemm_mxfp8_mxfp4_epilogue",
                     "bq_gemm_mxfp8_fp8blk32_epilogue", "bq_gemm_mxfp8_mxfp8_epilogue"):
        assert required in names
    assert set(names) == set(bq.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    for code in range(12):
        s = bq.status_string(code)
        assert s.startswith("BQ_")
    assert bq.status_string(0) == "BQ_OK"
    assert "UNKNOWN" in bq.status_string(99)


def test_sf_bytes(lib):
    assert bq.sf_bytes(1, 32) == 512
    assert bq.sf_bytes(128, 128) == 512
    assert bq.sf_bytes(129, 128) == 1024
    assert bq.sf_bytes(41, 1536) == 12 * 512
    assert bq.sf_bytes(8192, 8192) == 64 * 64 * 512
    assert bq.sf_bytes(4, 48) == 0  # K not a multiple of 32
    assert bq.sf_bytes(-1, 32) == 0


def test_version(lib):
    assert bq.version() >= 100


def test_built_for_sm100a_only():
    flags = build.NVCC_FLAGS
    i = flags.index("-gencode")
    assert flags[i + 1] == "arch=compute_100a,code=sm_100a"
    assert flags.count("-gencode") == 1


def test_binding_refuses_cpu_tensors(lib):
    import torch
    with pytest.raises(ValueError):
        bq.act_quant(torch.zeros((4, 32), dtype=torch.bfloat16))
