"""Schedule sweep for the block-scaled GEMM.

For one problem shape, times every candidate schedule (bq_gemm_config) with
CUDA-graph replay over rotating weight copies (more bytes than L2 holds, so
weights stream from HBM) and prints one JSON line per candidate:

    python sweep.py M N K [kind] [--batch B] [--gelu]
        [--residual]

kind: mxfp4 (default), fp8blk32, mxfp8, a4w4 (MXFP4 activations and weights).  --batch B runs B independent problems
over one broadcast weight (batch stride 0), --gelu adds bias + GELU,
--residual adds a bf16 residual.  The
built-in dispatch of bq_api.cu is derived from these measurements.
"""
from __future__ import annotations

import argparse
import json
import sys

import numpy as np


def candidates(M, N, K):
    import block_scaled_precision_quant_b200 as bq
    out = []
    if M <= 64:
        kt = (K + 127) // 128
        for kc in (1, 4):
            if kc == 1 or K % 128 == 0:
                out.append(bq.config(split_k=1, swap_ab=1, k_chunks=kc))
        for split in (2, 4, 8):
            for kc in (1, 4):
                if split <= kt and (kc == 1 or K % 128 == 0):
                    out.append(bq.config(split_k=split, swap_ab=1, split_mode=bq.BQ_SPLIT_CLUSTER,
                                         k_chunks=kc))
        for split in (2, 3, 4, 6, 8, 12, 16):
            if split <= kt:
                out.append(bq.config(split_k=split, swap_ab=1, split_mode=bq.BQ_SPLIT_WORKSPACE,
                                     k_chunks=1))
    for bn in (128, 256):
        for kc in (1, 2):
            if kc > 1 and K % 128:
                continue
            out.append(bq.config(block_n=bn, split_k=1, swap_ab=0, k_chunks=kc))
    if M > 64:
        for kc in (1, 2):
            if kc == 1 or K % 128 == 0:
                out.append(bq.config(split_k=1, swap_ab=0, k_chunks=kc, cta_pair=2))
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("M", type=int)
    ap.add_argument("N", type=int)
    ap.add_argument("K", type=int)
    ap.add_argument("kind", nargs="?", default="mxfp4")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--gelu", action="store_true")
    ap.add_argument("--residual", action="store_true")
    args = ap.parse_args(argv)
    import torch
    import block_scaled_precision_quant_b200 as bq
    from block_scaled_precision_quant_b200 import synth
    M, N, K, B = args.M, args.N, args.K, args.batch
    wk = {"mxfp4": bq.W_MXFP4, "fp8blk32": bq.W_FP8BLK32, "mxfp8": bq.W_MXFP8,
          "a4w4": bq.W_A4W4}[args.kind]
    quant = bq.act_quant_mxfp4 if wk == bq.W_A4W4 else bq.act_quant
    kb = K // 2 if wk == bq.W_A4W4 else K  # activation bytes per row
    dev = torch.device("cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        aqs, asfs = [], []
        for b in range(B):
            x = torch.from_numpy(synth.activations(M, K, seed=1 + b).view(np.int16)) \
                .view(torch.bfloat16).to(dev)
            q, f = quant(x)
            aqs.append(q)
            asfs.append(f)
        aq = torch.stack(aqs).reshape(B * M, kb)
        asf = torch.stack(asfs)
        batch = None if B == 1 else dict(count=B, stride_a=M * kb, stride_a_sf=asf.shape[1],
                                         stride_b=0, stride_b_sf=0, stride_y=M * N * 2,
                                         stride_res=M * N * 2 if args.residual else 0)
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        wbytes = N * K // 2 if wk in (bq.W_MXFP4, bq.W_A4W4) else N * K
        copies = max(1, min(64, int(np.ceil(2.5 * l2 / max(wbytes, 1)))))
        ws = []
        for c in range(copies):
            if wk in (bq.W_MXFP4, bq.W_A4W4):
                b, s = synth.mxfp4_weight(N, K, seed=10 + c)
                kind = bq.BQ_SF_ROW32
            elif wk == bq.W_FP8BLK32:
                b, s = synth.fp8_weight_blk32(N, K, seed=10 + c)
                kind = bq.BQ_SF_BLK32x32
            else:
                b = synth.uniform_bytes((N, K), seed=10 + c, lo=0, hi=0x7E)
                s = synth.uniform_bytes((N, K // 32), seed=20 + c, lo=118, hi=126)
                kind = bq.BQ_SF_ROW32
            bd = torch.from_numpy(b).to(dev)
            ws.append((bd, bq.pack_weight_scales(torch.from_numpy(s).to(dev), kind, N, K)))
        bias = torch.from_numpy(synth.bias(N, seed=3).view(np.int16)).view(torch.bfloat16).to(dev)
        y = torch.empty((B, M, N) if B > 1 else (M, N), dtype=torch.bfloat16, device=dev)
        act = bq.BQ_ACT_GELU if args.gelu else bq.BQ_ACT_NONE
        res = None
        if args.residual:
            res = torch.from_numpy(synth.residual(B * M, N, seed=4).view(np.int16)) \
                .view(torch.bfloat16).to(dev).reshape(y.shape)
        for cfg in candidates(M, N, K):
            need = bq.workspace_bytes(wk, M, N, K, B, cfg)
            work = torch.zeros((max(need, 16),), dtype=torch.uint8, device=dev) if need else None
            desc = dict(block_n=cfg.block_n, split_k=cfg.split_k, swap_ab=cfg.swap_ab,
                        split_mode=cfg.split_mode, k_chunks=cfg.k_chunks, cta_pair=cfg.cta_pair)
            try:
                def run(c):
                    bq.gemm(wk, aq, asf, ws[c][0], ws[c][1], M, N, K, y=y, bias=bias,
                            act=act, residual=res, batch=batch, config=cfg, workspace=work)
                for c in range(copies):
                    run(c)
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for c in range(copies):
                        run(c)
                for _ in range(3):
                    g.replay()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(args.reps):
                    g.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                bq.device_status()
                us = e0.elapsed_time(e1) * 1e3 / (args.reps * copies)
                gbytes = (wbytes + N * K / 32 + B * (M * (kb + K / 32) + 2 * M * N)) / (us * 1e-6) / 1e9
                print(json.dumps(dict(shape=[M, N, K], batch=B, gelu=args.gelu, kind=args.kind,
                                      residual=args.residual,
                                      cfg=desc, us=round(us, 3),
                                      tflops=round(2 * B * M * N * K / us / 1e6, 1),
                                      gbs=round(gbytes, 1))), flush=True)
            except bq.BqError as e:
                print(json.dumps(dict(shape=[M, N, K], cfg=desc, error=str(e))), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
