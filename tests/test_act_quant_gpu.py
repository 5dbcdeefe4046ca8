"""Parity of the CUDA activation quantizer with the oracle: bit-exact codes and
scale bytes, in both the row-major and the MMA scale layout (padding bytes
included), for the workloads' shapes, ragged and degenerate sizes, and every
bf16 bit pattern."""
import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_quant_b200 as bq
from block_scaled_precision_quant_b200 import synth

pytestmark = pytest.mark.gpu


def mma_index(rows, G):
    """Byte offsets of scale (r, c) in the MMA layout, written from the layout
    rule in include/bq.h; returns (offsets [rows, G], total bytes)."""
    katoms = (G + 3) // 4
    r = np.arange(rows)[:, None]
    c = np.arange(G)[None, :]
    off = ((r // 128) * katoms + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4
    total = ((rows + 127) // 128) * katoms * 512
    return off, total


def run_gpu(x_bits, ldx=None):
    M, K = x_bits.shape
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16)
    if ldx is not None and ldx != K:
        big = torch.zeros((M, ldx), dtype=torch.bfloat16)
        big[:, :K] = x
        xd = big.cuda()[:, :K]
    else:
        xd = x.cuda()
    G = K // 32
    sf_row = torch.full((M, G), 0xAA, dtype=torch.uint8, device="cuda")
    sf_mma = torch.full((bq.sf_bytes(M, K),), 0xAA, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, _ = bq.act_quant(xd, sf_mma=sf_mma, sf_rowmajor=sf_row, status=status)
    unpacked = bq.unpack_scales(sf_mma, M, K)
    torch.cuda.synchronize()
    return (q.cpu().numpy(), sf_row.cpu().numpy(), sf_mma.cpu().numpy(), unpacked.cpu().numpy(),
            int(status.item()))


def check(x_bits, ldx=None):
    M, K = x_bits.shape
    want_q, want_sf = oracle.act_quant(x_bits)
    q, sf_row, sf_mma, unpacked, status = run_gpu(x_bits, ldx)
    assert status == 0
    bad = np.argwhere(q != want_q)
    assert bad.size == 0, f"{bad.shape[0]} code mismatches, first {bad[:3].tolist()}"
    assert np.array_equal(sf_row, want_sf)
    assert np.array_equal(unpacked, want_sf)
    off, total = mma_index(M, K // 32)
    assert sf_mma.size == total
    expect = np.full(total, 127, dtype=np.uint8)  # padding rows / columns
    expect[off.ravel()] = want_sf.ravel()
    assert np.array_equal(sf_mma, expect)


@pytest.mark.parametrize("M,K,seed,gp", [
    (64, 1024, 0, (-4, 4)),      # PR1 reference activations
    (41, 1536, 1, None),         # decode-shaped linear
    (41, 6144, 1, None),
    (1024, 4096, 2, None),       # FP8-weight layer
    (8, 2048, 3, None),
])
def test_workload_shapes(M, K, seed, gp):
    check(synth.activations(M, K, seed=seed, group_pow2=gp))


@pytest.mark.parametrize("M,K", [(1, 32), (3, 96), (7, 544), (129, 160), (130, 4064), (255, 32)])
def test_ragged_shapes(M, K):
    check(synth.activations(M, K, seed=M + K, group_pow2=(-20, 20)))


def test_row_stride_larger_than_k():
    check(synth.activations(33, 320, seed=5), ldx=512)


@pytest.mark.parametrize("M,K,ldx", [(1000, 4128, None), (4113, 1120, None), (2050, 2048, 2304),
                                     (256, 16384, None), (6100, 4128, 4160)])
def test_large_inputs(M, K, ldx):
    """Inputs of >= 4 Mi elements: rows past a 128-row band boundary, a last
    512-column chunk holding only a few groups, a row stride wider than K,
    long rows; the last case launches >= 6144 one-row blocks' worth of work,
    so its warps take two rows each."""
    check(synth.activations(M, K, seed=M + K, group_pow2=(-12, 12)), ldx=ldx)


def test_every_bf16_pattern():
    """All finite bf16 patterns, shuffled into groups so that each value meets
    many different group maxima (and so many scales)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = bits[(bits & 0x7F80) != 0x7F80]
    rng = np.random.default_rng(0)
    xs = []
    for _ in range(4):
        xs.append(rng.permutation(finite))
    x = np.concatenate(xs)
    x = x[: (x.size // 1024) * 1024].reshape(-1, 1024)
    check(x)


def test_tiny_and_floor_groups():
    """Groups under the 1e-4 floor, all-zero and signed-zero groups."""
    x = np.zeros((4, 128), dtype=np.uint16)
    x[1, :32] = 0x8000
    x[2, 32:64] = 0x0001          # smallest bf16 subnormal
    x[3, 64:96] = 0x38D1          # ~1e-4
    x[3, 96:128] = 0xB8D0
    check(x)


def test_full_size_square_operand():
    """The 8192 x 8192 operand of the square GEMM, in the launch configuration
    the benchmark uses."""
    check(synth.activations(8192, 8192, seed=3))


def test_nonfinite_input_sets_status():
    x = synth.activations(2, 64, seed=1)
    x[1, 40] = 0x7F80  # +Inf
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, sf = bq.act_quant(xd, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    # the group holding the Inf gets a valid scale byte (the exponent's cap,
    # 247), never the NaN scale 255; the other groups are exact
    sf_row = bq.unpack_scales(sf, 2, 64).cpu().numpy()
    assert sf_row[1, 1] == 247
    q_ref, s_ref = oracle.act_quant(x[:, :32])
    assert np.array_equal(sf_row[:, 0], s_ref[:, 0])
    assert np.array_equal(q.cpu().numpy()[:, :32], q_ref)
    q_ref0, s_ref0 = oracle.act_quant(x[:1, 32:])
    assert sf_row[0, 1] == s_ref0[0, 0]


def test_empty_m_launches_nothing():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    q, sf = bq.act_quant(x)
    torch.cuda.synchronize()
    assert q.shape == (0, 64)


def test_argument_errors():
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bq.BqError) as e:
        bq.act_quant(x)
    assert e.value.status == bq.BQ_ERR_SHAPE
    x = torch.zeros((4, 72), dtype=torch.bfloat16, device="cuda")[:, 1:65]  # misaligned base
    with pytest.raises(bq.BqError) as e:
        bq.act_quant(x)
    assert e.value.status == bq.BQ_ERR_ALIGN
