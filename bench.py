"""Benchmark of the block-scaled linear-layer hot path on B200.

One step = the whole hot path over one batch: for each linear layer of the
workload, bq_act_quant (bf16 -> E4M3 + E8M0 in the MMA scale layout) and the
block-scaled GEMM with its fused epilogue.  The default workload is the
decode-shaped linear (M = 41 rows, MXFP8 activations x MXFP4 weights + bias,
(N, K) in {(4608, 1536), (6144, 1536), (1536, 6144)}).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode|pr1|fp8blk|square|mlp]

Prints one JSON line (rank 0).  Timing: W untimed warm-up steps, then K steps
between a barrier + device synchronize on both sides, timed with CUDA events on
the launching stream, max over ranks.  Each step's launches are replayed from
a CUDA graph (one graph per rotating input set); inputs rotate over enough
copies that every step reads its weights from HBM, not L2.  `--impl reference`
times the CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
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

class Layer:
    """Device buffers of one linear layer, with `sets` rotating copies of the
    inputs (activations, weights, scales, bias, residual)."""

    def __init__(self, spec, sets, seed, device, quant_out=False, fused_act=False):
        import torch
        import block_scaled_precision_quant_b200 as bq
        from block_scaled_precision_quant_b200 import synth
        self.spec = spec
        name, wk, M, N, K, B, ex = spec
        self.wk, self.M, self.N, self.K, self.B = WKIND[wk], M, N, K, B
        self.gelu = bool(ex.get("gelu"))
        self.sets = []
        for s in range(sets):
            sd = seed + 1000 * s
            xs = []
            for b in range(B):
                xb = synth.activations(M, K, seed=sd + b, group_pow2=ex.get("act_gp"))
                xs.append(torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16))
            x = torch.stack(xs).reshape(B * M, K).to(device)
            if wk == "nvfp4":  # weights quantized once here, on the device
                wxb = synth.activations(N, K, seed=sd + 500, std=0.05)
                wx = torch.from_numpy(wxb.view(np.int16)).view(torch.bfloat16).to(device)
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
                wxb = synth.activations(N, K, seed=sd + 500)
                wx = torch.from_numpy(wxb.view(np.int16)).view(torch.bfloat16).to(device)
                w = torch.empty((N, K), dtype=torch.uint8, device=device)
                wsf = torch.empty((bq.sf_bytes(N, K),), dtype=torch.uint8, device=device)
            bias = (torch.from_numpy(synth.bias(N, seed=sd + 600).view(np.int16))
                    .view(torch.bfloat16).to(device) if ex.get("bias") else None)
            res = (torch.from_numpy(synth.residual(B * M, N, seed=sd + 700).view(np.int16))
                   .view(torch.bfloat16).to(device) if ex.get("residual") else None)
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

    def launches(self, s, which="all", x=None):
        """Issue this layer's kernels for input set s on the current stream
        (x: optional activations replacing the set's own)."""
        import block_scaled_precision_quant_b200 as bq
        d = dict(self.sets[s])
        if x is not None:
            d["x"] = x
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
            # one fused launch; a K loop of >= 24 blocks (the library's split
            # rule) runs act_quant + the split GEMM instead
            return 2 if (K + 127) // 128 >= 24 and not self.quant_out else 1
        if which in ("all", "act_quant"):
            quant = (bq.act_quant_nvfp4 if self.nv else
                     bq.act_quant_mxfp4 if self.a4 else bq.act_quant)
            for b in range(B):
                quant(d["x"][b * M:(b + 1) * M], q=self.aq[b * M:(b + 1) * M],
                      sf_mma=self.asf[b])
                n += 1
            if d["wx"] is not None:
                bq.act_quant(d["wx"], q=d["w"], sf_mma=d["wsf"])
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

    def __init__(self, spec, sets, seed, device, **_):
        import torch
        import block_scaled_precision_quant_b200 as bq
        from block_scaled_precision_quant_b200 import synth
        self.spec = spec
        name, wk, T, N, K, B, ex = spec
        self.T, self.N, self.K = T, N, K
        self.wk = WKIND[wk]
        self.quant_out = False
        self.qy = None

        def bf16(bits):
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)
        self.sets = []
        for s in range(sets):
            sd = seed + 1000 * s
            self.sets.append(dict(
                x=bf16(synth.activations(T, N, seed=sd + 2, group_pow2=(-20, 4))),  # dY
                xin=bf16(synth.activations(T, K, seed=sd)),
                w=bf16(synth.activations(N, K, seed=sd + 1, std=0.05))))
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
        self.step = 0

    def launches(self, s, which="all", x=None):
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


def build_graphs(layers, nsets, which):
    """One CUDA graph per input set (one step each) and one rotation graph
    holding the steps of all sets back to back."""
    import torch
    graphs = []
    stream = torch.cuda.current_stream()
    for s in range(nsets):
        # warm once outside capture (sets function attributes, caches)
        for L in layers:
            L.launches_per_step = L.launches(s, which)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for L in layers:
                L.launches(s, which)
        graphs.append(g)
    rot = torch.cuda.CUDAGraph()
    with torch.cuda.graph(rot, stream=stream):
        for s in range(nsets):
            for L in layers:
                L.launches(s, which)
    torch.cuda.synchronize()
    return graphs, rot


def replay_steps(graphs, rot, start, count):
    """Replay `count` steps beginning at input set `start` (mod the number of
    sets); whole rotations go through the rotation graph."""
    n = len(graphs)
    i, left = start, count
    while left > 0 and i % n != 0:
        graphs[i % n].replay()
        i, left = i + 1, left - 1
    while left >= n:
        rot.replay()
        i, left = i + n, left - n
    while left > 0:
        graphs[i % n].replay()
        i, left = i + 1, left - 1
    return i


def time_graphs(graph_pair, steps, warmup, world, device, min_warm_s=1.0, nvtx=None):
    """Warm-up (at least `warmup` steps and `min_warm_s` seconds), then time
    exactly `steps` steps between barrier + synchronize, CUDA events on the
    launching stream, max over ranks.  Returns (ms, warm-up steps run)."""
    import torch
    graphs, rot = graph_pair
    i = replay_steps(graphs, rot, 0, warmup)
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < min_warm_s and i < 2_000_000:
        i = replay_steps(graphs, rot, i, len(graphs))
        torch.cuda.synchronize()
    torch.cuda.synchronize()
    barrier(world, device)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if nvtx:
        torch.cuda.nvtx.range_push(nvtx)
    e0.record(stream)
    replay_steps(graphs, rot, i, steps)
    e1.record(stream)
    if nvtx:
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(world, device)
    ms = e0.elapsed_time(e1)
    return reduce_max(ms, world, device), i


def run_e2e(spec_layers, layers, steps, device):
    """The same step through the public API with host buffers: pinned host
    activations copied in, act_quant + GEMM launched eagerly, outputs read
    back, every step."""
    import torch
    import block_scaled_precision_quant_b200 as bq
    host_x = [L.sets[0]["x"].cpu().pin_memory() for L in layers]
    outs = [L.qy if L.quant_out else L.y for L in layers]  # the step's result
    host_y = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h2d = sum(h.numel() * h.element_size() for h in host_x)
    d2h = sum(h.numel() * h.element_size() for h in host_y)
    dev_x = [torch.empty_like(L.sets[0]["x"]) for L in layers]

    def step():
        for L, hx, dx, hy, o in zip(layers, host_x, dev_x, host_y, outs):
            dx.copy_(hx, non_blocking=True)
            L.launches(0, x=dx)
            hy.copy_(o, non_blocking=True)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, h2d, d2h


# ------------------------------------------------------------- CPU oracle --

def oracle_step_sample(layers_spec, rows, seed=0, nthreads=None):
    """One bounded sample of the workload on the CPU oracle: for each layer,
    act_quant of `rows` activation rows and the GEMM of those rows against the
    full weight.  Returns (flops done, seconds, threads)."""
    import oracle
    from block_scaled_precision_quant_b200 import synth
    nthreads = nthreads or oracle.default_threads()
    flops = 0.0
    t_total = 0.0
    for (name, wk, M, N, K, B, ex) in layers_spec:
        r = min(rows, M)
        if wk == "grad":
            # backward: `r` rows of dX (over all N) and `r` rows of dW (over all T tokens)
            dy = synth.activations(M, N, seed=seed + 2, group_pow2=(-20, 4))
            w = synth.activations(N, K, seed=seed + 1, std=0.05)
            xin = synth.activations(M, K, seed=seed)
            t0 = time.perf_counter()
            gq, gs = oracle.grad_quant(dy[:r], stochastic=True, seed=seed)
            wq, ws = oracle.quant_transposed(w, oracle.Q_E4M3)
            oracle.gemm(gq, gs, wq, ws, oracle.B_FP8ROW, r, K, N, a_kind=oracle.A_E5M2,
                        nthreads=nthreads)
            gtq, gts = oracle.quant_transposed(dy[:, :max(8, r)], oracle.Q_E5M2, stochastic=True,
                                               seed=seed)
            xq, xs = oracle.quant_transposed(xin, oracle.Q_E4M3)
            oracle.gemm(gtq[:r], gts[:r], xq, xs, oracle.B_FP8ROW, r, K, M,
                        a_kind=oracle.A_E5M2, nthreads=nthreads)
            t_total += time.perf_counter() - t0
            flops += 2.0 * r * K * N + 2.0 * r * K * M
            continue
        x = synth.activations(r, K, seed=seed, group_pow2=ex.get("act_gp"))
        if wk == "nvfp4":
            wb, ws = oracle.act_quant_nvfp4(synth.activations(N, K, seed=seed + 500, std=0.05))
            kind = oracle.B_NVFP4
        elif wk in ("mxfp4", "a4w4"):
            wb, ws = synth.mxfp4_weight(N, K, seed=seed + 500)
            kind = oracle.B_FP4
        elif wk == "fp8blk32":
            wb, ws = synth.fp8_weight_blk32(N, K, seed=seed + 500)
            kind = oracle.B_FP8BLK
        else:
            wb, ws = oracle.act_quant(synth.activations(N, K, seed=seed + 500))
            kind = oracle.B_FP8ROW
        bias = synth.bias(N, seed=seed + 600) if ex.get("bias") else None
        res = synth.residual(r, N, seed=seed + 700) if ex.get("residual") else None
        t0 = time.perf_counter()
        if wk == "nvfp4":
            q, s = oracle.act_quant_nvfp4(x)
        elif wk == "a4w4":
            q, s = oracle.act_quant_fp4(x)
        else:
            q, s = oracle.act_quant(x)
        a_kind = {"a4w4": oracle.A_FP4, "nvfp4": oracle.A_NVFP4}.get(wk, oracle.A_E4M3)
        oracle.gemm(q, s, wb, ws, kind, r, N, K, bias=bias, residual=res,
                    act=oracle.ACT_GELU if ex.get("gelu") else oracle.ACT_NONE,
                    nthreads=nthreads, a_kind=a_kind)
        t_total += time.perf_counter() - t0
        flops += 2.0 * r * N * K
    return flops, t_total, nthreads


def cpu_baseline(spec, budget_s=15.0):
    """The oracle as it stands on this host's cores, on a bounded sample."""
    rows = 4
    flops, secs, th = oracle_step_sample(spec["layers"], rows)
    # grow the sample toward the time budget (bounded)
    while secs < budget_s / 4 and rows < 64:
        rows *= 2
        flops, secs, th = oracle_step_sample(spec["layers"], rows)
    return dict(value=flops / secs / 1e12, unit="TFLOP/s", cores=th, kind="oracle",
                sample=f"{rows} activation rows per layer (act_quant + exact-decode fp64 GEMM "
                       f"against the full weight), {flops / 1e9:.2f} GFLOP in {secs:.1f} s")


# ------------------------------------------------------------------- main --

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about 2 s of timed work)")
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
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
    if args.warmup < 3:
        args.warmup = 3
    spec = WORKLOADS[args.workload]
    world, rank, local = dist_env()

    if args.impl == "reference":
        return run_reference(args, spec, world, rank)

    import torch
    import block_scaled_precision_quant_b200 as bq
    from block_scaled_precision_quant_b200 import build as bq_build
    bq_build.build()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    # All work on one non-default stream: graphs are captured and replayed on
    # it, and the CUDA events are recorded on it.
    with torch.cuda.stream(torch.cuda.Stream(device)):
        return run_ours(args, spec, world, rank, local, device)


def run_ours(args, spec, world, rank, local, device):
    import torch
    import block_scaled_precision_quant_b200 as bq

    if args.profile_run:
        specs = spec["layers"]
        if args.profile_shape:
            M, N, K = (int(v) for v in args.profile_shape.split(","))
            name, wk, _, _, _, B, ex = specs[0]
            specs = [(name, wk, M, N, K, B, ex)]
        layers = [make_layer(sp, 1, 11 * (i + 1), device) for i, sp in enumerate(specs)]
        for _ in range(args.profile_run):
            for L in layers:
                L.launches(0)
        torch.cuda.synchronize()
        bq.device_status()
        if rank == 0:
            print(json.dumps({"profile_run": args.profile_run, "workload": spec["desc"],
                              "shape": args.profile_shape}))
        return 0

    layers_spec = spec["layers"]
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    probe = [make_layer(sp, 1, 11 * (i + 1), device) for i, sp in enumerate(layers_spec)]
    set_bytes = sum(L.set_bytes for L in probe)
    nsets = max(1, min(64, int(np.ceil(3.0 * l2 / max(set_bytes, 1)))))
    del probe
    torch.cuda.empty_cache()
    layers = [make_layer(sp, nsets, 11 * (i + 1), device, quant_out=args.quant_out,
                         fused_act=args.fused_act)
              for i, sp in enumerate(layers_spec)]
    graphs = build_graphs(layers, nsets, "all")
    launches_per_step = sum(L.launches_per_step for L in layers)

    if args.steps is None:  # calibrate: about 2 s of timed work
        rot = graphs[1]
        rot.replay()
        torch.cuda.synchronize()
        c0 = time.perf_counter()
        rot.replay()
        torch.cuda.synchronize()
        per = (time.perf_counter() - c0) / nsets
        args.steps = int(min(200000, max(50, 2.0 / max(per, 1e-7))))
    clocks = ClockSampler(local)
    clocks.start()
    ms, warm_steps = time_graphs(graphs, args.steps, args.warmup, world, device,
                                 nvtx="bq_timed")
    ck = clocks.stop()
    ms_step = ms / args.steps

    # dominant kernel: the GEMM.  Time GEMM-only graphs over the same rotation,
    # and act_quant-only graphs likewise.
    ggraphs = build_graphs(layers, nsets, "gemm")
    gms, _ = time_graphs(ggraphs, args.steps, args.warmup, world, device, min_warm_s=0.2)
    gemm_ms_step = gms / args.steps
    qgraphs = build_graphs(layers, nsets, "act_quant")
    qms, _ = time_graphs(qgraphs, args.steps, args.warmup, world, device, min_warm_s=0.2)
    aq_ms_step = qms / args.steps
    per_layer_us = None
    if len(layers) > 1:  # each layer's GEMM alone, same rotation
        per_layer_us = []
        for L in layers:
            lg = build_graphs([L], nsets, "gemm")
            lms, _ = time_graphs(lg, args.steps, args.warmup, world, device, min_warm_s=0.1)
            per_layer_us.append(round(lms / args.steps * 1e3, 3))
            del lg
    bq.device_status()

    flops_step = sum(gemm_flops(sp) for sp in layers_spec)
    gbytes_step = sum(gemm_bytes(sp, args.quant_out) for sp in layers_spec)
    qbytes_step = sum(act_quant_bytes(sp) for sp in layers_spec)
    if any(sp[1] == "mxfp8" for sp in layers_spec):
        qbytes_step += sum(act_quant_bytes((0, 0, sp[3], 0, sp[4], 1, 0))
                           for sp in layers_spec if sp[1] == "mxfp8")
    value = world * flops_step / (ms_step * 1e-3) / 1e12
    peaks = load_peaks()
    # A kernel whose median SM clock over the timed region sat under the power
    # cap is held to the sustained tensor figure, otherwise to the burst one.
    capped = bool(ck) and "sw_power_cap" in (ck.get("reasons") or []) and bool(
        ck.get("sm_mhz") and ck.get("sm_max_mhz") and ck["sm_mhz"] < 0.97 * ck["sm_max_mhz"])
    tensor_kind = "bf16_sus" if capped else "bf16"
    # nominal dense fp8 / bf16 ratio 4.5 / 2.25; FP4 x FP4 (kind::mxf4) 9 / 2.25
    a4 = all(sp[1] in FP4_ACT for sp in layers_spec)  # FP4 x FP4: the FP4 tensor rate
    tensor_ratio = 4.0 if a4 else 2.0
    fp8_peak = tensor_ratio * peaks[tensor_kind]
    shapes = [(WKIND[sp[1]],) + g for sp in layers_spec for g in gemm_shapes(sp)]
    gemm_launches = len(shapes)
    # the GEMM kernel(s) the built-in dispatch runs for these layers
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    kernels = sorted({("gemm_pair_kernel" if bq.plan(M, N, K, B, num_sms=sms,
                                                     weight_kind=wk).cta_pair == 2
                       else "gemm_bs_kernel") for (wk, M, N, K, B) in shapes})
    kernel_name = "+".join(kernels)
    if spec["bound"] == "hbm":
        achieved = gbytes_step / (gemm_ms_step * 1e-3) / 1e9
        roof = dict(bound="hbm", achieved=round(achieved, 1), peak=peaks["hbm"], unit="GB/s",
                    frac=round(achieved / peaks["hbm"], 4), traffic=stored_traffic(args.workload),
                    kernel=kernel_name, algorithmic_bytes_per_launch=gbytes_step / gemm_launches,
                    avg_launch_us=round(gemm_ms_step * 1e3 / gemm_launches, 3),
                    peak_source=f"{peaks['src']} hbm_gbs (burst)")
    else:
        achieved = flops_step / (gemm_ms_step * 1e-3) / 1e12
        roof = dict(bound="tensor", achieved=round(achieved, 1), peak=round(fp8_peak, 1),
                    unit="TFLOP/s", frac=round(achieved / fp8_peak, 4),
                    traffic=stored_traffic(args.workload),
                    kernel=kernel_name, flops_per_launch=flops_step / gemm_launches,
                    avg_launch_us=round(gemm_ms_step * 1e3 / gemm_launches, 3),
                    peak_source=(f"{peaks['src']} {'bf16_tflops_sustained' if tensor_kind != 'bf16' else 'bf16_tflops'}"
                                 f" x {tensor_ratio:g} (nominal "
                                 f"{'fp4' if a4 else 'fp8'}/bf16 ratio)"))
    e2e_ms, h2d, d2h = run_e2e(layers_spec, layers, min(2000, max(10, args.steps // 4)), device)
    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE[layers_spec[0][1]],
        "data": "synthetic",
        "config": {"workload": spec["desc"], "parallelism": "replicas" if world > 1 else "single",
                   "l2": f"{nsets} rotating input sets of {set_bytes / 1e6:.1f} MB "
                         f"({nsets * set_bytes / 1e6:.0f} MB > L2 {l2 / 1e6:.0f} MB)",
                   "graphs": "one CUDA graph per input set, replayed per step",
                   "output": "mxfp8 (codes + scales, no bf16 y)" if args.quant_out else "bf16",
                   "act_quant": "fused into the GEMM (one call per decode layer)"
                                if args.fused_act else "separate launch"},
        "roofline": roof,
        "act_quant": {"achieved_gbs": round(qbytes_step / (aq_ms_step * 1e-3) / 1e9, 1),
                      "frac_hbm": round(qbytes_step / (aq_ms_step * 1e-3) / 1e9 / peaks["hbm"], 4),
                      "us_per_step": round(aq_ms_step * 1e3, 3),
                      "algorithmic_bytes_per_step": qbytes_step},
        "gemm_us_per_step": round(gemm_ms_step * 1e3, 3),
        "gemm_us_per_layer": per_layer_us,
        "e2e": {"value": round(world * flops_step / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": launches_per_step * args.steps,
        "warmup_steps_run": warm_steps,
        "clocks": ck,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(spec)
    if rank == 0:
        print(json.dumps(out), flush=True)
    del graphs, ggraphs, qgraphs
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_reference(args, spec, world, rank):
    """Reference arm: the CPU oracle on the host cores, on a bounded sample of
    the same workload per step.  Under torchrun only rank 0 works."""
    if rank != 0:
        return 0
    rows = 2
    times = []
    flops = 0.0
    th = 1
    for i in range(args.warmup + args.steps):
        f, s, th = oracle_step_sample(spec["layers"], rows, seed=i)
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
                         "kind": "oracle",
                         "sample": f"{rows} activation rows per layer per step (act_quant + "
                                   "exact-decode fp64 GEMM against the full weight)"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
