"""Standalone timing of the activation quantizers (E4M3 and MXFP4 codes).

For each operand shape, times bq_act_quant / bq_act_quant_mxfp4 alone: a CUDA
graph of back-to-back launches over enough distinct input copies that they
span more than 3x the L2 cache, so every launch reads its input from HBM (at
most 64 copies: decode-sized operands of a few hundred KB stay in L2), timed
with CUDA events over two graph replays after three warm-up replays.  Prints
one JSON line of {"<fmt> <M>x<K>": [us per launch, algorithmic GB/s]}, the
algorithmic bytes being 2 (bf16 read) + 1 or 1/2 (code) + 1/32 (scale) per
element.

    python quant_timing.py [--fmt e4m3,fp4] [MxK ...]
"""
from __future__ import annotations

import argparse
import json

DEFAULT_SHAPES = ("8192x8192", "1024x4096", "4096x6144", "8192x2048", "41x1536", "41x6144")


def algorithmic_bytes(fmt: str, M: int, K: int) -> float:
    """Bytes one launch must move: the bf16 input, the codes and the scales."""
    code = {"e4m3": 1.0, "fp4": 0.5}[fmt]
    return M * K * (2.0 + code + 1.0 / 32.0)


def input_copies(in_bytes: int, l2_bytes: int) -> int:
    """Distinct input copies so that one pass over them exceeds 3x L2 (2..64)."""
    return max(2, min(64, (3 * l2_bytes) // in_bytes + 1))


def parse_shape(s: str):
    m, k = s.lower().split("x")
    M, K = int(m), int(k)
    if M <= 0 or K <= 0 or K % 32:
        raise ValueError(f"bad operand shape {s}: M > 0, K > 0 and K % 32 == 0")
    return M, K


def time_one(fmt: str, M: int, K: int, device, l2_bytes: int):
    import torch
    import block_scaled_precision_quant_b200 as bq
    nbuf = input_copies(M * K * 2, l2_bytes)
    xs = [torch.randn(M, K, device=device).to(torch.bfloat16) for _ in range(nbuf)]
    qs = [torch.empty((M, K if fmt == "e4m3" else K // 2), dtype=torch.uint8, device=device)
          for _ in range(nbuf)]
    sfs = [torch.empty((bq.sf_bytes(M, K),), dtype=torch.uint8, device=device)
           for _ in range(nbuf)]
    f = bq.act_quant if fmt == "e4m3" else bq.act_quant_mxfp4
    for i in range(nbuf):
        f(xs[i], q=qs[i], sf_mma=sfs[i])
    torch.cuda.synchronize()
    reps = max(nbuf, 4 * ((200 if M * K > 4e6 else 2000) // nbuf))
    stream = torch.cuda.Stream(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for r in range(reps):
                i = r % nbuf
                f(xs[i], q=qs[i], sf_mma=sfs[i])
    torch.cuda.synchronize()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    bq.device_status()
    us = e0.elapsed_time(e1) * 1e3 / (2 * reps)
    return round(us, 2), round(algorithmic_bytes(fmt, M, K) / us / 1e3, 1)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("shapes", nargs="*", default=list(DEFAULT_SHAPES), metavar="MxK")
    ap.add_argument("--fmt", default="e4m3,fp4", help="comma-separated: e4m3, fp4")
    args = ap.parse_args(argv)
    fmts = [f for f in args.fmt.split(",") if f]
    for f in fmts:
        if f not in ("e4m3", "fp4"):
            raise SystemExit(f"unknown format {f}")
    shapes = [parse_shape(s) for s in args.shapes]
    import torch
    device = torch.device("cuda", torch.cuda.current_device())
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    out = {}
    for fmt in fmts:
        for M, K in shapes:
            out[f"{fmt} {M}x{K}"] = time_one(fmt, M, K, device, l2)
            torch.cuda.empty_cache()
    print(json.dumps(out))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
