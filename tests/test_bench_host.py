"""Host-side logic of bench.py: algorithmic byte/flop counts, the multi-rank
timing reduction (2 gloo ranks on CPU) and the reference arm's rank handling."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def test_decode_algorithmic_bytes():
    # weights 4.25 bits/weight + activations + bias + bf16 output (MB)
    got = [bench.gemm_bytes(sp) / 1e6 for sp in bench.WORKLOADS["decode"]["layers"]]
    assert [round(g, 2) for g in got] == [4.21, 5.59, 5.4]
    assert bench.gemm_flops(bench.WORKLOADS["decode"]["layers"][0]) == 2.0 * 41 * 4608 * 1536


def test_act_quant_bytes_per_element():
    assert bench.act_quant_bytes(("x", "mxfp4", 1, 0, 32, 1, {})) == 32 * 3.03125
    # packed E2M1 activations: half a byte per code; NVFP4 one scale per 16
    assert bench.act_quant_bytes(("x", "a4w4", 1, 0, 32, 1, {})) == 32 * (2 + 0.5 + 1 / 32)
    assert bench.act_quant_bytes(("x", "nvfp4", 1, 0, 32, 1, {})) == 32 * (2 + 0.5 + 1 / 16)


def test_every_workload_is_accounted():
    """Each workload names a dtype, a bound and positive flop / byte counts."""
    for name, spec in bench.WORKLOADS.items():
        assert spec["bound"] in ("hbm", "tensor"), name
        for layer in spec["layers"]:
            assert layer[1] in bench.WKIND and layer[1] in bench.DTYPE, name
            assert bench.gemm_flops(layer) > 0 and bench.gemm_bytes(layer) > 0, name
            assert bench.act_quant_bytes(layer) > 0, name
            assert bench.gemm_shapes(layer), name


def test_backward_accounting():
    """dX and dW: two GEMMs of 2 T N K flops each; the quantizers read dY twice
    (row-wise and transposed), x and W once."""
    layer = bench.WORKLOADS["backward"]["layers"][0]
    _, _, T, N, K, _, _ = layer
    assert bench.gemm_flops(layer) == 4.0 * T * N * K
    assert bench.gemm_shapes(layer) == [(T, K, N, 1), (N, K, T, 1)]
    assert bench.act_quant_bytes(layer) == 3.03125 * (2 * T * N + T * K + N * K)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p
def test_source_hash_ignores_comments_only():
    """The stored-traffic key changes with the code, not with its comments."""
    a = 'int f(int x) {  // twice\n  return 2 * x;  /* no\n overflow */\n}\n'
    b = '// header\nint f(int x) {\n\n  return 2 * x;\n}\n'
    assert bench.strip_c_comments(a) == bench.strip_c_comments(b)
    assert bench.strip_c_comments('s = "a//b /* c */";') == 's = "a//b /* c */";'
    assert bench.strip_c_comments("c = '/'; // x") == "c = '/';"
    assert bench.strip_c_comments("return 3 * x;") != bench.strip_c_comments("return 2 * x;")
    sha = bench.kernel_source_sha()
    assert len(sha) == 16 and sha == bench.kernel_source_sha()




def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    bench.init_dist(world, "gloo")
    bench.barrier(world)
    m = bench.reduce_max(10.0 + rank, world)
    bench.barrier(world)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((rank, m))


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == {0: 11.0, 1: 11.0}


def test_reference_arm_other_ranks_do_nothing(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_windows_continue_one_rotation():
    """Back-to-back windows of exactly `steps` steps walk the input sets in
    rotation order whether steps is below, equal to or above the set count,
    so a timed result does not depend on --steps through L2 reuse."""
    for steps, nsets in ((20, 28), (1, 7), (28, 28), (45, 28), (3, 2), (20, 2)):
        starts = bench.window_starts(steps, nsets)
        seq = [(s + i) % nsets for s in starts for i in range(steps)]
        assert seq == [i % nsets for i in range(len(seq))], (steps, nsets)
        # the next window after the last one starts where the first one did
        assert (starts[-1] + steps) % nsets == starts[0]
    assert bench.window_starts(20, 28) == [0, 20, 12, 4, 24, 16, 8]


def test_rotation_exceeds_three_l2():
    l2 = 126 * 2 ** 20
    for name, spec in bench.WORKLOADS.items():
        b = sum(bench.input_set_bytes(sp) for sp in spec["layers"])
        n = bench.rotation_sets(b, l2)
        assert 2 <= n <= 64
        assert n * b > 3 * l2 or n == 64, name


def test_input_set_bytes_by_hand():
    # decode layer 1: bf16 x 41x1536, FP4 weights 4608x768 bytes, scales
    # 36 x 12 atoms of 512 bytes, bias 4608 bf16
    qkv = bench.WORKLOADS["decode"]["layers"][0]
    assert bench.input_set_bytes(qkv) == 41 * 1536 * 2 + 4608 * 768 + 36 * 12 * 512 + 4608 * 2
    # square: bf16 x and bf16 weight operand, its E4M3 codes and scales
    sq = bench.WORKLOADS["square"]["layers"][0]
    n = 8192 * 8192
    assert bench.input_set_bytes(sq) == 2 * n + 2 * n + n + 64 * 64 * 512


def test_suite_names_every_workload_once():
    assert bench.HEADLINE not in bench.SUITE
    assert len(set(bench.SUITE)) == len(bench.SUITE)
    assert all(s in bench.WORKLOADS for s in (bench.HEADLINE,) + bench.SUITE)
    # the batched up-projection and the down-projection are separate records
    assert bench.WORKLOADS["mlp_up"]["layers"] + bench.WORKLOADS["mlp_down"]["layers"] == \
        bench.WORKLOADS["mlp"]["layers"]


def test_reference_arm_line(capsys):
    """The reference arm on the smallest workload: one JSON line with the
    oracle timed on this host, its thread count and CPU model."""
    import json
    assert bench.main(["--impl", "reference", "--workload", "pr1", "--steps", "1",
                       "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["steps"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["cpu_model"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_oracle_sample_counts_the_weight_quantization():
    """The square workload's sample quantizes rows*N/M rows of its weight
    operand on top of the activation rows (a smaller square stands in)."""
    spec = [("sq", "mxfp8", 256, 256, 256, 1, {})]
    sample = bench.OracleSample(spec)
    flops, secs, threads = sample.run(4)
    assert flops == 2.0 * 4 * 256 * 256 and secs > 0 and threads >= 1
