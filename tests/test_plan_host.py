"""Host-side checks of the built-in GEMM dispatch (bq_gemm_plan, no device):
the schedules the sweeps measured fastest on the workloads' shapes, and the
explicit requests the dispatch must refuse or keep."""
import pytest

import block_scaled_precision_quant_b200 as bq
from block_scaled_precision_quant_b200 import build

SMS = 148


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    bq.lib()


def desc(c):
    return dict(block_n=c.block_n, split_k=c.split_k, swap_ab=c.swap_ab,
                split_mode=c.split_mode, k_chunks=c.k_chunks, cta_pair=c.cta_pair)


@pytest.mark.parametrize("N,K,split", [(4608, 1536, 4), (6144, 1536, 1), (1536, 6144, 8)])
def test_decode_layers(N, K, split):
    """M = 41: swap-AB tiles of 64 activation rows; the 6144-wide short-K
    layer unsplit with 4 chunks per stage, the 4608-wide one on 4-CTA
    cluster slices (36 x 4 CTAs fill 144 of 148 SMs), the long-K layer on
    8-CTA cluster slices."""
    d = desc(bq.plan(41, N, K, num_sms=SMS))
    assert d["swap_ab"] == 1 and d["block_n"] == 64 and d["cta_pair"] == 1
    assert d["split_k"] == split
    if split == 1:
        assert d["k_chunks"] == 4 and d["split_mode"] == bq.BQ_SPLIT_AUTO
    else:
        assert d["split_mode"] == bq.BQ_SPLIT_CLUSTER
    assert (N // 128) * split <= SMS  # one CTA per SM


def test_short_k_split_needs_nearly_every_sm():
    # 36 tiles: 4 slices fill 144 of 148 SMs; on 160 SMs 144 is below 90 %
    assert bq.plan(41, 4608, 1536, num_sms=148).split_k == 4
    assert bq.plan(41, 4608, 1536, num_sms=170).split_k == 1
    # 12 K blocks at most; fewer stay unsplit
    assert bq.plan(41, 4608, 1280, num_sms=148).split_k == 1


def test_small_m_tiles():
    assert bq.plan(16, 512, 1024).block_n == 32
    assert bq.plan(64, 512, 1024).block_n == 64
    assert bq.plan(65, 512, 1024).swap_ab == 0


@pytest.mark.parametrize("M,N,K,batch,want", [
    (1024, 4096, 4096, 1, dict(block_n=256, cta_pair=1, k_chunks=1)),   # fp8blk + residual
    (1024, 2048, 2048, 8, dict(block_n=128, cta_pair=1, k_chunks=2)),   # batched MLP up
    (4096, 1536, 6144, 1, dict(block_n=256, cta_pair=1, k_chunks=1)),   # down-projection
    (8192, 8192, 8192, 1, dict(block_n=256, cta_pair=1, k_chunks=1)),   # square
])
def test_wide_tile_workloads(M, N, K, batch, want):
    d = desc(bq.plan(M, N, K, batch=batch, num_sms=SMS))
    assert d["swap_ab"] == 0 and d["split_k"] == 1
    for k, v in want.items():
        assert d[k] == v, (k, d)


def test_pair_tiles_only_on_request():
    for shape in ((4096, 8192, 4096), (8192, 8192, 8192), (2048, 2048, 8192)):
        assert bq.plan(*shape, num_sms=SMS).cta_pair == 1
    c = bq.plan(8192, 8192, 8192, num_sms=SMS, config=bq.config(split_k=1, swap_ab=0, cta_pair=2))
    assert (c.cta_pair, c.block_n) == (2, 256)


def test_explicit_requests_kept():
    c = bq.plan(1024, 4096, 4096, config=bq.config(split_k=1, swap_ab=0, cta_pair=2))
    assert (c.cta_pair, c.block_n, c.k_chunks) == (2, 256, 2)
    c = bq.plan(41, 1536, 6144, config=bq.config(split_k=4, swap_ab=1,
                                                 split_mode=bq.BQ_SPLIT_WORKSPACE))
    assert (c.split_k, c.split_mode, c.k_chunks) == (4, bq.BQ_SPLIT_WORKSPACE, 1)
    c = bq.plan(1000, 1000, 4096, config=bq.config(block_n=128, split_k=1, swap_ab=0))
    assert (c.block_n, c.cta_pair, c.k_chunks) == (128, 1, 2)


@pytest.mark.parametrize("cfg", [
    dict(split_k=2, swap_ab=0, cta_pair=2),                 # pair tiles never split
    dict(swap_ab=1, cta_pair=2),                            # nor swap
    dict(block_n=128, split_k=1, swap_ab=0, cta_pair=2),    # 256-wide only
    dict(split_k=1, swap_ab=0, cta_pair=3),
    dict(split_k=3, swap_ab=1, split_mode=bq.BQ_SPLIT_CLUSTER),  # cluster: power of two
])
def test_refused_requests(cfg):
    with pytest.raises(bq.BqError) as e:
        bq.plan(41 if cfg.get("swap_ab") == 1 else 300, 520, 1536, config=bq.config(**cfg))
    assert e.value.status == bq.BQ_ERR_INVALID


def test_bad_sizes():
    for args in ((0, 512, 1024), (64, 512, 1000), (64, 0, 1024)):
        with pytest.raises(bq.BqError) as e:
            bq.plan(*args)
        assert e.value.status == bq.BQ_ERR_SHAPE
    with pytest.raises(bq.BqError):
        bq.plan(64, 512, 1024, num_sms=0)


def test_a4w4_plans():
    """Packed E2M1 operands: chunks of 256 K, wide tiles with 2 chunks per
    stage, no pair tiles unless asked for."""
    c = bq.plan(8192, 8192, 8192, num_sms=SMS, weight_kind=bq.W_A4W4)
    assert (c.block_n, c.cta_pair, c.k_chunks, c.swap_ab) == (256, 1, 2, 0)
    c = bq.plan(8192, 8192, 8192, num_sms=SMS, weight_kind=bq.W_A4W4,
                config=bq.config(split_k=1, swap_ab=0, cta_pair=2))
    assert (c.cta_pair, c.k_chunks) == (2, 2)
    c = bq.plan(41, 4608, 1536, num_sms=SMS, weight_kind=bq.W_A4W4)
    assert c.swap_ab == 1 and c.split_k == 1
    assert bq.plan(41, 1536, 6144, num_sms=SMS, weight_kind=bq.W_A4W4).split_k > 1
