"""Benchmark of the block-scaled linear-layer hot path on B200.

One step = the whole hot path over one batch: for each linear layer of the
workload, the activation quantizer (bf16 -> E4M3 + E8M0 in the MMA scale
layout) and the block-scaled GEMM with its fused epilogue.

The default run reports the square MXFP8 x MXFP8 GEMM at M = N = K = 8192
(both bf16 operands quantized by act_quant inside every step) as the headline
line, and carries every other workload of the suite as a sub-record of that
line ("suite"): the 64x512x1024 MXFP8 x MXFP4 reference case, the three
decode-shaped (M = 41) layers with bias, the FP8 32x32-block weights at
1024x4096x4096 with a residual, the batched MLP up-projection 8 x
(1024x2048x2048) with bias + GELU and its 4096x1536x6144 down-projection,
then the FP4 x FP4 rows (MXFP4 decode layers and 8192^3, NVFP4 8192^3) and
the backward of a 4096x1536x6144 layer.  Every record has its own roofline,
act_quant bandwidth, end-to-end number and CPU-oracle baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload suite|square|decode|pr1|fp8blk|mlp|mlp_up|...]

Timing: W untimed warm-up steps, then windows of exactly K steps, each window
one CUDA-graph replay between two CUDA events on the launching stream; the
windows run back to back between a barrier + device synchronize on both
sides, at least 100 of them, and the median window gives ms_per_step (max
over ranks).  Consecutive windows continue one rotation over enough copies of
the inputs (more than 3x the L2 size) that every step reads its weights and
activations from HBM.  `--impl reference` times the CPU oracle on a bounded
sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "block-scaled GEMM TFLOP/s & act_quant GB/s on 1 B200, % of FP8/FP4 & HBM peak"

# ---------------------------------------------------------------- workloads --
# Each layer: (name, weight kind, M, N, K, batch, extras)
WORKLOADS = {
    "decode": dict(
        desc="decode-shaped linear: act_quant + MXFP8xMXFP4 GEMM + bias, M=41, "
             "(N,K) in {(4608,1536),(6144,1536),(1536,6144)}",
        layers=[("qkv", "mxfp4", 41, 4608, 1536, 1, dict(bias=True)),
                ("up", "mxfp4", 41, 6144, 1536, 1, dict(bias=True)),
                ("down", "mxfp4", 41, 1536, 6144, 1, dict(bias=True))],
        bound="hbm"),
    "pr1": dict(
        desc="PR1 reference: act_quant + MXFP8xMXFP4 GEMM, M=64 N=512 K=1024, no bias",
        layers=[("pr1", "mxfp4", 64, 512, 1024, 1, dict(act_gp=(-4, 4)))], bound="hbm"),
    "fp8blk": dict(
        desc="FP8 E4M3 weights with 32x32 E8M0 block scales, M=1024 N=4096 K=4096, + residual",
        layers=[("fp8blk", "fp8blk32", 1024, 4096, 4096, 1, dict(residual=True))],
        bound="tensor"),
    "square": dict(
        desc="square MXFP8xMXFP8 GEMM M=N=K=8192 (both operands act_quant'd per step)",
        layers=[("square", "mxfp8", 8192, 8192, 8192, 1, dict())], bound="tensor"),
    "mlp": dict(
        desc="batched MLP: 8x(1024x2048x2048) MXFP4, broadcast weight, bias+GELU; then "
             "down-projection 4096x1536x6144",
        layers=[("up8", "mxfp4", 1024, 2048, 2048, 8, dict(bias=True, gelu=True)),
                ("down", "mxfp4", 4096, 1536, 6144, 1, dict())], bound="tensor"),
    "mlp_up": dict(
        desc="batched MLP up-projection: 8x(1024x2048x2048) MXFP8xMXFP4, broadcast weight, "
             "bias+GELU",
        layers=[("up8", "mxfp4", 1024, 2048, 2048, 8, dict(bias=True, gelu=True))],
        bound="tensor"),
    "mlp_down": dict(
        desc="MLP down-projection: MXFP8xMXFP4 GEMM M=4096 N=1536 K=6144",
        layers=[("down", "mxfp4", 4096, 1536, 6144, 1, dict())], bound="tensor"),
    # FP4 x FP4 (A4W4): MXFP4 activations (bq_act_quant_mxfp4) and MXFP4 weights
    # on tcgen05.mma kind::mxf4, on the decode shapes and on a large square
    "a4w4_decode": dict(
        desc="decode-shaped linear, A4W4: act_quant_mxfp4 + MXFP4xMXFP4 GEMM + bias, M=41, "
             "(N,K) in {(4608,1536),(6144,1536),(1536,6144)}",
        layers=[("qkv", "a4w4", 41, 4608, 1536, 1, dict(bias=True)),
                ("up", "a4w4", 41, 6144, 1536, 1, dict(bias=True)),
                ("down", "a4w4", 41, 1536, 6144, 1, dict(bias=True))],
        bound="hbm"),
    "a4w4_square": dict(
        desc="square MXFP4xMXFP4 GEMM M=N=K=8192 (activations act_quant_mxfp4'd per step, "
             "MXFP4 weights)",
        layers=[("square", "a4w4", 8192, 8192, 8192, 1, dict())], bound="tensor"),
    "nvfp4_square": dict(
        desc="square NVFP4xNVFP4 GEMM M=N=K=8192 (activations act_quant_nvfp4'd per step, "
             "NVFP4 weights)",
        layers=[("square", "nvfp4", 8192, 8192, 8192, 1, dict())], bound="tensor"),
    # Backward of one linear layer y = x W^T (x [T, K], W [N, K]): the output
    # gradient dY [T, N] quantized to E5M2 with stochastic rounding along N
    # (for dX) and along T (for dW), x and the bf16 master weight W quantized
    # along T and along N (transposed quantizers), then dX = dY W [T, K] and
    # dW = dY^T x [N, K] on E5M2 x MXFP8 GEMMs.  Shape: the MLP workload's
    # down-projection, T = 4096 tokens, N = 1536, K = 6144.
    "backward": dict(
        desc="backward of a 4096x1536x6144 linear layer: E5M2 stochastic gradient quantization "
             "(row-wise and transposed in one pass), transposed E4M3 quantization of x and W, "
             "dX = dY W and dW = dY^T x on E5M2 x MXFP8 GEMMs",
        layers=[("bwd", "grad", 4096, 1536, 6144, 1, dict())], bound="tensor"),
}

# The default run: the headline workload, then the suite's sub-records (the
# reference configurations, then the FP4 x FP4 and backward rows).
HEADLINE = "square"
SUITE = ("pr1", "decode", "fp8blk", "mlp_up", "mlp_down", "a4w4_decode", "a4w4_square",
         "nvfp4_square", "backward")

WKIND = {"mxfp4": 0, "fp8blk32": 1, "mxfp8": 2, "a4w4": 3, "grad": 4, "nvfp4": 5}
DTYPE = {"mxfp4": "mxfp8xmxfp4", "fp8blk32": "mxfp8xfp8blk32", "mxfp8": "mxfp8xmxfp8",
         "a4w4": "mxfp4xmxfp4", "grad": "e5m2xmxfp8", "nvfp4": "nvfp4xnvfp4"}
FP4_ACT = ("a4w4", "nvfp4")  # packed E2M1 activations


def gemm_shapes(layer):
    """(M, N, K, batch) of each GEMM launch of a layer: the backward layer
    runs dX = dY W ([T, K], contraction N) and dW = dY^T x ([N, K], over T)."""
    _, wk, M, N, K, B, _ = layer
    if wk == "grad":
        return [(M, K, N, 1), (N, K, M, 1)]
    return [(M, N, K, B)]


def gemm_flops(layer):
    _, wk, M, N, K, B, _ = layer
    return (4.0 if wk == "grad" else 2.0) * M * N * K * B  # backward: dX and dW


def act_quant_bytes(layer):
    """Algorithmic bytes of act_quant: read 2 B/elem, write 1 + 1/32 B/elem
    (E4M3 codes) or 1/2 + 1/32 B/elem (packed E2M1 codes)."""
    _, wk, M, N, K, B, _ = layer
    if wk == "grad":  # dY twice (row-wise, transposed), x^T and W^T
        return (2.0 + 1.0 + 1.0 / 32.0) * (2 * M * N + M * K + N * K)
    if wk == "nvfp4":
        return (2.0 + 0.5 + 1.0 / 16.0) * M * K * B
    code = 0.5 if wk == "a4w4" else 1.0
    return (2.0 + code + 1.0 / 32.0) * M * K * B


def gemm_bytes(layer, quant_out=False):
    """Algorithmic bytes of one GEMM launch: every operand read once, the
    output written once (weights counted once when broadcast over a batch);
    a quantized output is 1 + 1/32 bytes per element instead of 2."""
    _, wk, M, N, K, B, ex = layer
    if wk == "grad":  # dX: dY codes [M, N] x W^T codes [K, N]; dW: dY^T [N, M] x x^T [K, M]
        code = 1.0 + 1.0 / 32.0
        return code * (M * N + K * N) + 2.0 * M * K + code * (N * M + K * M) + 2.0 * N * K
    w = N * K / 2.0 if wk in ("mxfp4",) + FP4_ACT else float(N * K)
    sfb = 16.0 if wk == "nvfp4" else 32.0  # inputs per scale byte
    w += N * K / sfb  # weight scales
    a = B * (M * K * (0.5 if wk in FP4_ACT else 1.0) + M * K / sfb)
    y = B * M * N * ((1.0 + 1.0 / 32.0) if quant_out else 2.0)
    if ex.get("bias"):
        a += N * 2.0
    if ex.get("residual"):
        a += B * M * N * 2.0
    if wk == "mxfp8":  # the square workload quantizes its weight operand each step too
        w = float(N * K) + N * K / 32.0
    return w + a + y


# ------------------------------------------------------- profile evidence --

# The sources a GEMM launch is built and configured from (kernels, PTX
# wrappers, the epilogue's quantizer arithmetic, the host dispatch).
GEMM_SOURCES = ("gemm_bs.cuh", "gemm_pair.cuh", "bq_ptx.cuh", "mx_quant.cuh", "bq_api.cu")


def strip_c_comments(text):
    """C/C++ source without its comments and blank lines (string and character
    literals kept as written), so that editing a comment leaves the code's
    hash unchanged."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_sha():
    """Hash of the GEMM's sources and the header, comments left out: a stored
    DRAM-traffic figure is used only while the code it was measured on is
    unchanged."""
    import hashlib
    h = hashlib.sha256()
    files = [os.path.join(ROOT, "block_scaled_precision_quant_b200", "csrc", f)
             for f in GEMM_SOURCES]
    files.append(os.path.join(ROOT, "include", "bq.h"))
    for f in files:
        with open(f) as fh:
            h.update(os.path.basename(f).encode())
            h.update(strip_c_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def stored_traffic(workload):
    """DRAM bytes per GEMM launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the committed ncu summary, or None if the kernels changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f).get(workload)
        if d and d.get("source_sha") == kernel_source_sha():
            return float(d["bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------- peaks --

# Nominal dense figures of one B200, for the fractions stated against them
# next to the measured-peak fractions: HBM3e ~8 TB/s, FP8 4.5 PFLOP/s, FP4
# 9 PFLOP/s (NVIDIA's doubled figures assume 2:4 sparsity).
NOMINAL = dict(hbm=8000.0, fp8=4500.0, fp4=9000.0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


# ---------------------------------------------------------------- distributed --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity on one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"bq_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.remove(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        return dict(sm_mhz=statistics.median(sm) if sm else None,
                    sm_max_mhz=max(mx) if mx else None, reasons=reasons, samples=len(rows))


# -------------------------------------------------------------- GPU workload --

def _bf16_dev(bits, device):
    import torch
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)


class Layer:
    """Device buffers of one linear layer, with `sets` rotating copies of the
    inputs (activations, weights, scales, bias, residual).  The first
    `distinct` sets are drawn from their own seeds; the others are device
    copies of them (distinct memory, so the rotation still streams every
    step's operands from HBM)."""

    def __init__(self, spec, sets, seed, device, quant_out=False, fused_act=False, distinct=2):
        import torch
        import block_scaled_precision_quant_b200 as bq
        from block_scaled_precision_quant_b200 import synth
        self.spec = spec
        name, wk, M, N, K, B, ex = spec
        self.wk, self.M, self.N, self.K, self.B = WKIND[wk], M, N, K, B
        self.gelu = bool(ex.get("gelu"))
        self.sets = []
        for s in range(sets):
            if s >= distinct:
                src = self.sets[s % distinct]
                self.sets.append({k: (v.clone() if v is not None else None)
                                  for k, v in src.items()})
                continue
            sd = seed + 1000 * s
            xs = []
            for b in range(B):
                xs.append(_bf16_dev(synth.activations(M, K, seed=sd + b,
                                                      group_pow2=ex.get("act_gp")), "cpu"))
            x = torch.stack(xs).reshape(B * M, K).to(device)
            if wk == "nvfp4":  # weights quantized once here, on the device
                wx = _bf16_dev(synth.activations(N, K, seed=sd + 500, std=0.05), device)
                w, wsf = bq.act_quant_nvfp4(wx)
                wx = None
            elif wk in ("mxfp4", "a4w4"):
                wb, ws = synth.mxfp4_weight(N, K, seed=sd + 500)
                w = torch.from_numpy(wb).to(device)
                wsf = bq.pack_weight_scales(torch.from_numpy(ws).to(device), bq.BQ_SF_ROW32, N, K)
                wx = None
            elif wk == "fp8blk32":
                wb, ws = synth.fp8_weight_blk32(N, K, seed=sd + 500)
                w = torch.from_numpy(wb).to(device)
                wsf = bq.pack_weight_scales(torch.from_numpy(ws).to(device), bq.BQ_SF_BLK32x32,
                                            N, K)
                wx = None
            else:  # MXFP8 weight operand, quantized by act_quant inside the step
                wx = _bf16_dev(synth.activations(N, K, seed=sd + 500), device)
                w = torch.empty((N, K), dtype=torch.uint8, device=device)
                wsf = torch.empty((bq.sf_bytes(N, K),), dtype=torch.uint8, device=device)
            bias = _bf16_dev(synth.bias(N, seed=sd + 600), device) if ex.get("bias") else None
            res = (_bf16_dev(synth.residual(B * M, N, seed=sd + 700), device)
                   if ex.get("residual") else None)
            self.sets.append(dict(x=x, w=w, wsf=wsf, wx=wx, bias=bias, res=res))
        # outputs shared by all sets (written every step)
        self.a4 = wk in FP4_ACT  # packed E2M1 activations, two codes per byte
        self.nv = wk == "nvfp4"
        self.aq = torch.empty((B * M, K // 2 if self.a4 else K), dtype=torch.uint8,
                              device=device)
        per = bq.sf_bytes_nvfp4(M, K) if self.nv else bq.sf_bytes(M, K)
        self.asf = torch.empty((B, per), dtype=torch.uint8, device=device)
        self.y = torch.empty((B, M, N), dtype=torch.bfloat16, device=device)
        self.quant_out = quant_out
        # one call per layer: the GEMM quantizes its bf16 activations itself
        self.fused_act = fused_act and M <= 64 and B == 1 and K % 128 == 0 and not self.a4
        self.qy = torch.empty((B, M, N), dtype=torch.uint8, device=device) if quant_out else None
        self.sfy = (torch.empty((B, bq.sf_bytes(M, N)), dtype=torch.uint8, device=device)
                    if quant_out else None)
        self.need = bq.workspace_bytes(self.wk, M, N, K, B)
        self.ws = (torch.zeros((self.need,), dtype=torch.uint8, device=device)
                   if self.need else None)
        self.set_bytes = sum(t.numel() * t.element_size() for t in self.sets[0].values()
                             if t is not None)

    def step_inputs(self, s):
        """The bf16 tensors a step copies in from the host (end-to-end path):
        the activations, and for the square workload the bf16 weight operand
        that every step quantizes."""
        d = self.sets[s]
        return dict(x=d["x"]) if d["wx"] is None else dict(x=d["x"], wx=d["wx"])

    def output(self):
        return self.qy if self.quant_out else self.y

    def launches(self, s, which="all", x=None, wx=None):
        """Issue this layer's kernels for input set s on the current stream
        (x, wx: optional bf16 operands replacing the set's own)."""
        import block_scaled_precision_quant_b200 as bq
        d = dict(self.sets[s])
        if x is not None:
            d["x"] = x
        if wx is not None:
            d["wx"] = wx
        M, N, K, B = self.M, self.N, self.K, self.B
        n = 0
        if self.fused_act and which == "all":
            kw = {}
            if self.quant_out:
                kw = dict(quantize_out=True, write_y=False)
            bq.gemm_bf16act(self.wk, d["x"], d["w"], d["wsf"], M, N, K,
                            y=None if self.quant_out else self.y, bias=d["bias"],
                            residual=d["res"],
                            act=bq.BQ_ACT_GELU if self.gelu else bq.BQ_ACT_NONE,
                            a_q=self.aq, a_sf=self.asf[0], **kw)
            # one fused launch; a shape the library splits runs act_quant +
            # the split GEMM instead
            split = bq.plan(M, N, K, weight_kind=self.wk).split_k > 1
            return 2 if split and not self.quant_out else 1
        if which in ("all", "act_quant"):
            quant = (bq.act_quant_nvfp4 if self.nv else
                     bq.act_quant_mxfp4 if self.a4 else bq.act_quant)
            # The weight operand first: a GEMM may read its weights while the
            # kernel just before it is still running (programmatic launch), so
            # that kernel must be the activations' quantizer, not the weights'.
            if d["wx"] is not None:
                bq.act_quant(d["wx"], q=d["w"], sf_mma=d["wsf"])
                n += 1
            for b in range(B):
                quant(d["x"][b * M:(b + 1) * M], q=self.aq[b * M:(b + 1) * M],
                      sf_mma=self.asf[b])
                n += 1
        if which in ("all", "gemm"):
            batch = None
            if B > 1:
                batch = dict(count=B, stride_a=M * self.aq.shape[1], stride_a_sf=self.asf.shape[1],
                             stride_b=0,
                             stride_b_sf=0, stride_y=M * N * 2, stride_res=M * N * 2)
            kw = {}
            if self.quant_out:  # the output in MXFP8 for a next projection, no bf16 y
                kw = dict(quantize_out=True, write_y=False, q_out=self.qy, sf_out=self.sfy)
            bq.gemm(self.wk, self.aq, self.asf, d["w"], d["wsf"], M, N, K,
                    y=None if self.quant_out else self.y, bias=d["bias"], residual=d["res"],
                    act=bq.BQ_ACT_GELU if self.gelu else bq.BQ_ACT_NONE, batch=batch,
                    workspace=self.ws, **kw)
            n += 1
        return n


class BackwardLayer:
    """Device buffers of the backward of one linear layer (T tokens, N
    outputs, K inputs), with `sets` rotating copies of x, W and dY.  Same
    interface as Layer: launches(s, which) issues the quantizers ("act_quant")
    and the two GEMMs ("gemm"); y is dX (the step's result passed on)."""

    def __init__(self, spec, sets, seed, device, distinct=2, **_):
        import torch
        import block_scaled_precision_quant_b200 as bq
        from block_scaled_precision_quant_b200 import synth
        self.spec = spec
        name, wk, T, N, K, B, ex = spec
        self.T, self.N, self.K = T, N, K
        self.wk = WKIND[wk]
        self.quant_out = False
        self.qy = None
        self.sets = []
        for s in range(sets):
            if s >= distinct:
                self.sets.append({k: v.clone() for k, v in self.sets[s % distinct].items()})
                continue
            sd = seed + 1000 * s
            self.sets.append(dict(
                x=_bf16_dev(synth.activations(T, N, seed=sd + 2, group_pow2=(-20, 4)), device),
                xin=_bf16_dev(synth.activations(T, K, seed=sd), device),
                w=_bf16_dev(synth.activations(N, K, seed=sd + 1, std=0.05), device)))
        u8 = dict(dtype=torch.uint8, device=device)
        self.gq, self.gsf = torch.empty((T, N), **u8), torch.empty((bq.sf_bytes(T, N),), **u8)
        self.wtq, self.wtsf = torch.empty((K, N), **u8), torch.empty((bq.sf_bytes(K, N),), **u8)
        self.gtq, self.gtsf = torch.empty((N, T), **u8), torch.empty((bq.sf_bytes(N, T),), **u8)
        self.xtq, self.xtsf = torch.empty((K, T), **u8), torch.empty((bq.sf_bytes(K, T),), **u8)
        self.y = torch.empty((T, K), dtype=torch.bfloat16, device=device)   # dX
        self.dw = torch.empty((N, K), dtype=torch.bfloat16, device=device)
        self.need = max(bq.workspace_bytes(self.wk, T, K, N, 1),
                        bq.workspace_bytes(self.wk, N, K, T, 1))
        self.ws = torch.zeros((self.need,), **u8) if self.need else None
        self.set_bytes = sum(t.numel() * t.element_size() for t in self.sets[0].values())

    def step_inputs(self, s):
        return dict(x=self.sets[s]["x"])  # the output gradient dY

    def output(self):
        return self.y

    def launches(self, s, which="all", x=None, wx=None):
        import block_scaled_precision_quant_b200 as bq
        d = dict(self.sets[s])
        if x is not None:
            d["x"] = x
        T, N, K = self.T, self.N, self.K
        n = 0
        if which in ("all", "act_quant"):
            seed = 1000 + s  # a fresh stochastic-rounding seed per input set
            # dY along N (for dX) and along T (for dW) in one pass, shared draws
            bq.grad_quant_dual(d["x"], stochastic=True, seed=seed,
                               out=(self.gq, self.gsf, self.gtq, self.gtsf))
            bq.quant_transposed(d["w"], fmt=bq.BQ_FMT_E4M3, q=self.wtq, sf_mma=self.wtsf)
            bq.quant_transposed(d["xin"], fmt=bq.BQ_FMT_E4M3, q=self.xtq, sf_mma=self.xtsf)
            n += 3
        if which in ("all", "gemm"):
            bq.gemm(bq.W_GRAD, self.gq, self.gsf, self.wtq, self.wtsf, T, K, N, y=self.y,
                    workspace=self.ws)
            bq.gemm(bq.W_GRAD, self.gtq, self.gtsf, self.xtq, self.xtsf, N, K, T, y=self.dw,
                    workspace=self.ws)
            n += 2
        return n


def make_layer(spec, sets, seed, device, **kw):
    if spec[1] == "grad":
        return BackwardLayer(spec, sets, seed, device, **kw)
    return Layer(spec, sets, seed, device, **kw)


# ------------------------------------------------------------------ timing --

def _sf_bytes(rows, K, per=32):
    """Bytes of an MMA-layout scale buffer (512-byte atoms of 128 rows x 4
    scale columns)."""
    return -(-rows // 128) * -(-K // (4 * per)) * 512


def input_set_bytes(layer):
    """Device bytes of one rotating copy of a layer's step inputs: bf16
    activations, weight codes and scales (the square workload's bf16 weight
    operand, its codes and scales), bias and residual."""
    _, wk, M, N, K, B, ex = layer
    if wk == "grad":  # dY [T, N], x [T, K], W [N, K], all bf16
        return 2 * (M * N + M * K + N * K)
    x = 2 * B * M * K
    if wk in ("mxfp4", "a4w4"):
        w = N * K // 2 + _sf_bytes(N, K)
    elif wk == "nvfp4":
        w = N * K // 2 + _sf_bytes(N, K, per=16)
    elif wk == "fp8blk32":
        w = N * K + _sf_bytes(N, K)
    else:  # mxfp8: bf16 operand + its codes + scales
        w = 2 * N * K + N * K + _sf_bytes(N, K)
    return x + w + (2 * N if ex.get("bias") else 0) + (2 * B * M * N if ex.get("residual") else 0)


def rotation_sets(set_bytes, l2_bytes, cap=64):
    """Rotating input copies so that consecutive steps read more than 3x the
    L2 size before an input comes round again (at least 2, at most cap)."""
    return max(2, min(cap, int(math.ceil(3.0 * l2_bytes / max(set_bytes, 1)))))


def window_starts(steps, nsets, cap=64):
    """Input sets at which consecutive windows of `steps` steps begin when the
    windows continue one rotation over nsets sets: window j starts at set
    (j * steps) mod nsets, and the pattern repeats after nsets / gcd(steps,
    nsets) windows (capped)."""
    n = nsets // math.gcd(steps, nsets)
    return [(j * steps) % nsets for j in range(min(n, cap))]


def capture_windows(layers, nsets, which, steps):
    """One CUDA graph per window start, each holding exactly `steps` steps
    (input sets start, start+1, ... mod nsets) of the layers' launches.
    Returns (graphs, launches per step)."""
    import torch
    stream = torch.cuda.current_stream()
    per_step = 0
    for L in layers:  # warm once outside capture (function attributes, caches)
        per_step += L.launches(0, which)
    torch.cuda.synchronize()
    graphs = []
    for start in window_starts(steps, nsets):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(steps):
                for L in layers:
                    L.launches((start + i) % nsets, which)
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs, per_step


def time_windows(graphs, steps, warmup, world, device, min_windows=100, budget_s=1.0,
                 max_windows=20000):
    """Warm-up (at least `warmup` steps), then windows of exactly `steps`
    steps replayed back to back, each between two CUDA events on the
    launching stream, with a barrier + synchronize before the first and after
    the last.  The window count is sized to about budget_s of GPU time, at
    least min_windows.  Returns (median ms per window, max over ranks;
    windows; per-window ms of this rank)."""
    import torch
    stream = torch.cuda.current_stream()
    n = len(graphs)
    done = 0
    j = 0
    while done < warmup or j < n:
        graphs[j % n].replay()
        j += 1
        done += steps
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        graphs[(j + i) % n].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    j += n
    per = max(e0.elapsed_time(e1) / n, 1e-4)
    windows = int(min(max_windows, max(min_windows, budget_s * 1e3 / per)))
    windows = reduce_max(float(windows), world, device)  # same count on every rank
    windows = int(windows)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(windows + 1)]
    torch.cuda.synchronize()
    barrier(world, device)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(windows):
        graphs[(j + i) % n].replay()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    barrier(world, device)
    ts = [ev[i].elapsed_time(ev[i + 1]) for i in range(windows)]
    return reduce_max(statistics.median(ts), world, device), windows, ts


def run_e2e(layers, nsets, device, budget_s=0.3, max_steps=2000):
    """The same step through the public API with host buffers, every step:
    the step's bf16 inputs copied in from pinned host memory, act_quant + GEMM
    launched eagerly on the input set's weights (rotating like the timed
    windows), the result copied back to pinned host memory.  Runs about
    budget_s of steps (at least 5).  Returns (ms per step, steps, H2D bytes
    per step, D2H bytes per step)."""
    import torch
    host = [{k: v.cpu().pin_memory() for k, v in L.step_inputs(0).items()} for L in layers]
    dev = [{k: torch.empty_like(v, device=device) for k, v in h.items()} for h in host]
    outs = [L.output() for L in layers]
    host_y = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h2d = sum(v.numel() * v.element_size() for h in host for v in h.values())
    d2h = sum(h.numel() * h.element_size() for h in host_y)

    def step(s):
        for L, h, d, hy, o in zip(layers, host, dev, host_y, outs):
            for k in h:
                d[k].copy_(h[k], non_blocking=True)
            L.launches(s % nsets, **d)
            hy.copy_(o, non_blocking=True)

    def timed(first, count):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for s in range(first, first + count):
            step(s)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / count
    one = timed(0, 3)  # warm-up, and the size of the timed run
    steps = int(min(max_steps, max(5, budget_s * 1e3 / max(one, 1e-3))))
    return timed(3, steps), steps, h2d, d2h


# ------------------------------------------------------------- CPU oracle --

class OracleSample:
    """A workload's step on the CPU oracle, on a bounded sample: for each
    layer, the activation quantizer on `rows` activation rows and the GEMM of
    those rows against the full weight (flops 2 rows N K).  The square
    workload quantizes its bf16 weight operand every step; the sample charges
    that share too, the quantizer on rows * N / M of its rows.  Weights are
    prepared once (outside the timed sample), as the GPU path prepacks them.
    The backward workload times the gradient quantizers on `rows` rows and
    columns of dY and the dX and dW GEMMs on `rows` output rows."""

    def __init__(self, layers_spec, seed=0):
        import oracle
        from block_scaled_precision_quant_b200 import synth
        self.o, self.synth = oracle, synth
        self.layers = []
        for (name, wk, M, N, K, B, ex) in layers_spec:
            d = dict(spec=(name, wk, M, N, K, B, ex))
            if wk == "grad":
                d["dy"] = synth.activations(M, N, seed=seed + 2, group_pow2=(-20, 4))
                d["xin"] = synth.activations(M, K, seed=seed)
                d["wq"] = oracle.quant_transposed(synth.activations(N, K, seed=seed + 1, std=0.05),
                                                  oracle.Q_E4M3)
            elif wk == "nvfp4":
                d["w"] = oracle.act_quant_nvfp4(synth.activations(N, K, seed=seed + 500, std=0.05))
                d["kind"] = oracle.B_NVFP4
            elif wk in ("mxfp4", "a4w4"):
                d["w"] = synth.mxfp4_weight(N, K, seed=seed + 500)
                d["kind"] = oracle.B_FP4
            elif wk == "fp8blk32":
                d["w"] = synth.fp8_weight_blk32(N, K, seed=seed + 500)
                d["kind"] = oracle.B_FP8BLK
            else:  # mxfp8: the bf16 weight operand, quantized once for the GEMM
                d["wx"] = synth.activations(N, K, seed=seed + 500)
                d["w"] = oracle.act_quant(d["wx"])
                d["kind"] = oracle.B_FP8ROW
            if wk != "grad":
                d["bias"] = synth.bias(N, seed=seed + 600) if ex.get("bias") else None
            self.layers.append(d)

    def run(self, rows, seed=0, nthreads=None):
        """Returns (flops done, seconds, threads)."""
        o, synth = self.o, self.synth
        nthreads = nthreads or o.default_threads()
        flops, t_total = 0.0, 0.0
        for d in self.layers:
            name, wk, M, N, K, B, ex = d["spec"]
            r = min(rows, M)
            if wk == "grad":
                dy, xin = d["dy"], d["xin"]
                wq, ws = d["wq"]
                cols = max(32, r)
                t0 = time.perf_counter()
                gq, gs = o.grad_quant(dy[:r], stochastic=True, seed=seed)
                o.gemm(gq, gs, wq, ws, o.B_FP8ROW, r, K, N, a_kind=o.A_E5M2, nthreads=nthreads)
                gtq, gts = o.quant_transposed(dy[:, :cols], o.Q_E5M2, stochastic=True, seed=seed)
                xq, xs = o.quant_transposed(xin, o.Q_E4M3)
                o.gemm(gtq[:r], gts[:r], xq, xs, o.B_FP8ROW, r, K, M, a_kind=o.A_E5M2,
                       nthreads=nthreads)
                t_total += time.perf_counter() - t0
                flops += 2.0 * r * K * N + 2.0 * r * K * M
                continue
            x = synth.activations(r, K, seed=seed, group_pow2=ex.get("act_gp"))
            res = synth.residual(r, N, seed=seed + 700) if ex.get("residual") else None
            wb, ws = d["w"]
            wrows = max(1, (r * N) // M) if wk == "mxfp8" else 0
            t0 = time.perf_counter()
            if wk == "nvfp4":
                q, s = o.act_quant_nvfp4(x)
            elif wk == "a4w4":
                q, s = o.act_quant_fp4(x)
            else:
                q, s = o.act_quant(x)
            if wrows:
                o.act_quant(d["wx"][:wrows])
            a_kind = {"a4w4": o.A_FP4, "nvfp4": o.A_NVFP4}.get(wk, o.A_E4M3)
            o.gemm(q, s, wb, ws, d["kind"], r, N, K, bias=d["bias"], residual=res,
                   act=o.ACT_GELU if ex.get("gelu") else o.ACT_NONE,
                   nthreads=nthreads, a_kind=a_kind)
            t_total += time.perf_counter() - t0
            flops += 2.0 * r * N * K
        return flops, t_total, nthreads


def cpu_baseline(spec, budget_s=15.0, sample=None):
    """The oracle as it stands on this host's cores, on a bounded sample of
    the workload grown toward budget_s of CPU time."""
    import oracle
    sample = sample or OracleSample(spec["layers"])
    rows = oracle.default_threads()  # the oracle's GEMM spreads rows over its threads
    flops, secs, th = sample.run(rows)
    while secs < budget_s / 3 and rows < 1024:
        rows *= 2
        flops, secs, th = sample.run(rows)
    rows = min(rows, max(sp[2] for sp in spec["layers"]))  # at most the layers' own rows
    return dict(value=flops / secs / 1e12, unit="TFLOP/s", cores=th, kind="oracle",
                cpu_model=cpu_model(),
                sample=f"{rows} activation rows per layer (act_quant + exact-decode fp64 GEMM "
                       f"against the full weight), {flops / 1e9:.2f} GFLOP in {secs:.1f} s "
                       f"on {th} threads")


# ----------------------------------------------------------------- records --

def roofline(spec, layers_spec, gemm_ms_step, ck, peaks, kernels, workload, quant_out=False):
    """The dominant kernel's roofline object: algorithmic bytes (HBM-bound
    workloads) or flops (tensor-bound) per GEMM launch over the measured
    average launch time, against the measured peak and the nominal one."""
    flops_step = sum(gemm_flops(sp) for sp in layers_spec)
    bytes_step = sum(gemm_bytes(sp, quant_out) for sp in layers_spec)
    launches = sum(len(gemm_shapes(sp)) for sp in layers_spec)
    avg_us = gemm_ms_step * 1e3 / launches
    common = dict(kernel=kernels, avg_launch_us=round(avg_us, 3),
                  traffic=stored_traffic(workload), launches_per_step=launches)
    if spec["bound"] == "hbm":
        achieved = bytes_step / (gemm_ms_step * 1e-3) / 1e9
        return dict(bound="hbm", achieved=round(achieved, 1), peak=peaks["hbm"], unit="GB/s",
                    frac=round(achieved / peaks["hbm"], 4),
                    frac_nominal=round(achieved / NOMINAL["hbm"], 4),
                    peak_nominal=NOMINAL["hbm"],
                    algorithmic_bytes_per_launch=bytes_step / launches,
                    peak_source=f"{peaks['src']} hbm_gbs (burst)", **common)
    # A kernel whose median SM clock over the timed region sat under the power
    # cap is held to the sustained tensor figure, otherwise to the burst one.
    capped = bool(ck) and "sw_power_cap" in (ck.get("reasons") or []) and bool(
        ck.get("sm_mhz") and ck.get("sm_max_mhz") and ck["sm_mhz"] < 0.97 * ck["sm_max_mhz"])
    kind = "bf16_sus" if capped else "bf16"
    fp4 = all(sp[1] in FP4_ACT for sp in layers_spec)  # FP4 x FP4: the FP4 tensor rate
    ratio = 4.0 if fp4 else 2.0  # nominal dense fp8 (fp4) / bf16 ratio: 4.5 (9) / 2.25
    peak = ratio * peaks[kind]
    nominal = NOMINAL["fp4" if fp4 else "fp8"]
    achieved = flops_step / (gemm_ms_step * 1e-3) / 1e12
    out = dict(bound="tensor", achieved=round(achieved, 1), peak=round(peak, 1), unit="TFLOP/s",
               frac=round(achieved / peak, 4), frac_nominal=round(achieved / nominal, 4),
               peak_nominal=nominal, flops_per_launch=flops_step / launches,
               peak_source=(f"{peaks['src']} "
                            f"{'bf16_tflops_sustained' if capped else 'bf16_tflops'} x {ratio:g} "
                            f"(nominal {'fp4' if fp4 else 'fp8'}/bf16 ratio)"), **common)
    if ck and ck.get("sm_mhz"):  # clock-normalised: time x median SM clock
        out["us_x_ghz_per_launch"] = round(avg_us * ck["sm_mhz"] / 1e3, 3)
    return out


def measure(name, args, world, rank, local, device, cpu_budget_s, time_budget_s=1.0):
    """Every number of one workload's record (see the module docstring)."""
    import torch
    import block_scaled_precision_quant_b200 as bq
    spec = WORKLOADS[name]
    layers_spec = spec["layers"]
    props = torch.cuda.get_device_properties(device)
    l2 = props.L2_cache_size
    sms = props.multi_processor_count
    set_bytes = sum(input_set_bytes(sp) for sp in layers_spec)
    nsets = rotation_sets(set_bytes, l2)
    layers = [make_layer(sp, nsets, 11 * (i + 1), device, quant_out=args.quant_out,
                         fused_act=args.fused_act)
              for i, sp in enumerate(layers_spec)]
    K = args.steps
    graphs, per_step = capture_windows(layers, nsets, "all", K)
    clocks = ClockSampler(local)
    clocks.start()
    ms_win, windows, _ = time_windows(graphs, K, args.warmup, world, device,
                                      budget_s=time_budget_s)
    del graphs
    # the dominant kernel: the GEMM alone, same windows and rotation
    ggraphs, _ = capture_windows(layers, nsets, "gemm", K)
    gms_win, _, _ = time_windows(ggraphs, K, args.warmup, world, device,
                                 budget_s=time_budget_s / 2)
    del ggraphs
    ck = clocks.stop()
    qgraphs, _ = capture_windows(layers, nsets, "act_quant", K)
    qms_win, _, _ = time_windows(qgraphs, K, args.warmup, world, device,
                                 budget_s=time_budget_s / 4)
    del qgraphs
    per_layer_us = None
    if len(layers) > 1:  # each layer's GEMM alone, same rotation
        per_layer_us = []
        for L in layers:
            lg, _ = capture_windows([L], nsets, "gemm", K)
            lms, _, _ = time_windows(lg, K, args.warmup, world, device,
                                     budget_s=time_budget_s / 4)
            per_layer_us.append(round(lms / K * 1e3, 3))
            del lg
    ms_step, gemm_ms_step, aq_ms_step = ms_win / K, gms_win / K, qms_win / K
    e2e_ms, e2e_steps, h2d, d2h = run_e2e(layers, nsets, device)
    bq.device_status()  # raises if a kernel gave up on one of its waits

    flops_step = sum(gemm_flops(sp) for sp in layers_spec)
    qbytes_step = sum(act_quant_bytes(sp) for sp in layers_spec)
    qbytes_step += sum(act_quant_bytes((0, 0, sp[3], 0, sp[4], 1, 0))
                       for sp in layers_spec if sp[1] == "mxfp8")  # the quantized weight operand
    peaks = load_peaks()
    shapes = [(WKIND[sp[1]],) + g for sp in layers_spec for g in gemm_shapes(sp)]
    kernels = "+".join(sorted({("gemm_pair_kernel" if bq.plan(
        M, N, Kd, B, num_sms=sms, weight_kind=wk).cta_pair == 2 else "gemm_bs_kernel")
        for (wk, M, N, Kd, B) in shapes}))
    qgbs = qbytes_step / (aq_ms_step * 1e-3) / 1e9
    rec = {
        "workload": spec["desc"],
        "value": round(world * flops_step / (ms_step * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s",
        "ms_per_step": round(ms_step, 6),
        "steps": K,
        "windows": windows,
        "dtype": DTYPE[layers_spec[0][1]],
        "roofline": roofline(spec, layers_spec, gemm_ms_step, ck, peaks, kernels, name,
                             args.quant_out),
        "act_quant": {"achieved_gbs": round(qgbs, 1), "frac_hbm": round(qgbs / peaks["hbm"], 4),
                      "frac_hbm_nominal": round(qgbs / NOMINAL["hbm"], 4),
                      "us_per_step": round(aq_ms_step * 1e3, 3),
                      "algorithmic_bytes_per_step": qbytes_step},
        "gemm_us_per_step": round(gemm_ms_step * 1e3, 3),
        "gemm_us_per_layer": per_layer_us,
        "e2e": {"value": round(world * flops_step / (e2e_ms * 1e-3) / 1e12, 3),
                "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps},
        "clocks": ck,
        "l2": (f"{nsets} rotating input sets of {set_bytes / 1e6:.1f} MB "
               f"({nsets * set_bytes / 1e6:.0f} MB > 3 x L2 {l2 / 1e6:.0f} MB or 64 sets; "
               f"2 drawn from seeds, the rest device copies)"),
        "gpu_launches": per_step * K * windows,
        "launches_per_step": per_step,
    }
    del layers
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if world == 1 and rank == 0 and cpu_budget_s > 0:
        rec["cpu_baseline"] = cpu_baseline(spec, cpu_budget_s)
    return rec


# ------------------------------------------------------------------- main --

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20, help="steps per timed window")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["suite"] + sorted(WORKLOADS), default="suite",
                    help="suite (default): the square 8192^3 headline with every other "
                         "workload of the suite as a sub-record")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-run", type=int, default=0, metavar="R",
                    help="no timing: build one input set and run every layer's step R "
                         "times eagerly (for ncu captures of single launches)")
    ap.add_argument("--fused-act", action="store_true",
                    help="decode-shaped layers (M <= 64) run act_quant inside the GEMM: one "
                         "library call per layer")
    ap.add_argument("--quant-out", action="store_true",
                    help="every GEMM writes its output quantized (MXFP8 codes + MMA-layout "
                         "scales, for a next projection) instead of bf16 y")
    ap.add_argument("--profile-shape", default=None, metavar="M,N,K",
                    help="with --profile-run: run only the workload's first layer, at this "
                         "smaller shape (a small case of the same kernel for full captures)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)
    args.steps = max(1, args.steps)
    world, rank, local = dist_env()
    suite = args.workload == "suite"
    name = HEADLINE if suite else args.workload

    if args.impl == "reference":
        return run_reference(args, name, world, rank)

    import torch
    from block_scaled_precision_quant_b200 import build as bq_build
    bq_build.build()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    # All work on one non-default stream: graphs are captured and replayed on
    # it, and the CUDA events are recorded on it.
    with torch.cuda.stream(torch.cuda.Stream(device)):
        rc = run_ours(args, name, suite, world, rank, local, device)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return rc


def run_profile(args, name, rank, device):
    import torch
    import block_scaled_precision_quant_b200 as bq
    specs = WORKLOADS[name]["layers"]
    if args.profile_shape:
        M, N, K = (int(v) for v in args.profile_shape.split(","))
        lname, wk, _, _, _, B, ex = specs[0]
        specs = [(lname, wk, M, N, K, B, ex)]
    layers = [make_layer(sp, 1, 11 * (i + 1), device) for i, sp in enumerate(specs)]
    for _ in range(args.profile_run):
        for L in layers:
            L.launches(0)
    torch.cuda.synchronize()
    bq.device_status()
    if rank == 0:
        print(json.dumps({"profile_run": args.profile_run, "workload": WORKLOADS[name]["desc"],
                          "shape": args.profile_shape}))
    return 0


def run_ours(args, name, suite, world, rank, local, device):
    if args.profile_run:
        return run_profile(args, name, rank, device)
    cpu = not args.no_cpu_baseline
    head = measure(name, args, world, rank, local, device, cpu_budget_s=15.0 if cpu else 0,
                   time_budget_s=1.5)
    subs = {}
    if suite:
        for sub in SUITE:
            subs[sub] = measure(sub, args, world, rank, local, device,
                                cpu_budget_s=4.0 if cpu else 0, time_budget_s=0.6)
    out = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": head["dtype"],
        "data": "synthetic",
        "config": {"workload": head["workload"],
                   "parallelism": "replicas" if world > 1 else "single",
                   "timing": (f"median of {head['windows']} windows of exactly {args.steps} "
                              f"steps, each window one CUDA-graph replay between CUDA events"),
                   "l2": head["l2"],
                   "output": "mxfp8 (codes + scales, no bf16 y)" if args.quant_out else "bf16",
                   "act_quant": "fused into the GEMM (one call per decode layer)"
                                if args.fused_act else "separate launch"},
        "roofline": head["roofline"],
        "act_quant": head["act_quant"],
        "gemm_us_per_step": head["gemm_us_per_step"],
        "gemm_us_per_layer": head["gemm_us_per_layer"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    if "cpu_baseline" in head:
        out["cpu_baseline"] = head["cpu_baseline"]
    if subs:
        out["suite"] = subs
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


def run_reference(args, name, world, rank):
    """Reference arm: the CPU oracle on the host cores, on a bounded sample of
    the same workload per step (one activation row per oracle thread and
    layer).  Under torchrun only rank 0 works."""
    if rank != 0:
        return 0
    import oracle
    spec = WORKLOADS[name]
    rows = oracle.default_threads()
    sample = OracleSample(spec["layers"])
    times = []
    flops = 0.0
    th = 1
    for i in range(args.warmup + args.steps):
        f, s, th = sample.run(rows, seed=i)
        if i >= args.warmup:
            times.append(s)
            flops += f
    secs = sum(times)
    value = flops / secs / 1e12
    out = {
        "metric": METRIC, "impl": "reference", "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec["desc"], "parallelism": "cpu oracle"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": th,
                         "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": f"{rows} activation rows per layer per step (act_quant + "
                                   "exact-decode fp64 GEMM against the full weight; the square "
                                   "workload also quantizes rows*N/M of its weight operand)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
