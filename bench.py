#!/usr/bin/env python3
"""Benchmark of the fine-grained FP8 W8A8 linear layer on B200.

One step = one pass of the hot path over one batch of synthetic input: one
call of the layer, fgfp8_linear (fgfp8_grouped_linear for the MoE workload),
which runs the dynamic per-token 1x128 activation quantizer and then the
block-scaled FP8 GEMM with its bf16 epilogue, launched as the quantizer's
programmatic dependent.  The two kernels are also timed apart (an event
between them) for the per-kernel roofline.  Weights are quantized once before
timing (fgfp8_quant_weight, reported separately), as a deployed layer holds
pre-quantized weights.

Default workload: the Llama-3-8B MLP in prefill as two W8A8 linear layers,
the fused gate/up projection X [8192, 4096] x W [28672, 4096] (activations
N(0, 1) with outliers) and then the down projection X [8192, 14336] x
W [4096, 14336] (a post-SiLU-like heavy-tailed input), fp32 block scales,
both bf16 outputs written: one step is two fgfp8_linear calls.  The roofline
is taken on the gate/up GEMM (the dominant kernel) and the act-quant line on
the 8192 x 14336 down-projection input (the largest activation).  Other
workloads can be chosen with --workload (see workloads/), among them the
attention projection 4096^3, the same dense shapes with per-token x
per-channel scales (the FP8_DYNAMIC scheme) or a static per-tensor activation
scale, whose step is the row / tensor quantizer and the row/column-scaled
GEMM.

Timing: W warm-up steps, then K timed steps.  L2 is flushed (a 256 MB write followed
by a 256 MB read, so no dirty line is written back inside the next step)
before every step, outside the timed events.  Each kernel is bracketed by
CUDA events on the launching stream.  For N > 1 (torchrun) every rank runs
its own replica of the workload with no collective on the data path, and
rank 0 reports the max over ranks.

--impl reference runs the CPU oracle (the plain C implementation under
oracle/) on the host cores: on each step it quantizes and multiplies a
bounded sample of rows of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "block-scaled FP8 GEMM TFLOP/s (% FP8 peak); act-quant GB/s (% HBM)"
L2_FLUSH_BYTES = 256 << 20
# Idle time before each timed pass (the step pass and the per-kernel pass), so
# that both start from the same power state: the per-kernel breakdown then
# describes the step it breaks down instead of a GPU already heated by it.
REST_S = 0.25
FP8_OVER_BF16 = 2.0            # nominal dense fp8 / bf16 tensor ratio on B200 (4.5 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}

# Row / tensor scale granularity on the dense shapes ("FP8 W8A8", "Applying
# quantization"): "fp8_dynamic" = per-token activations x per-output-channel
# weights; "static_tensor" = one static activation scale (AbsMax over the
# layer's input, calibrated once before timing) x per-channel weights.
ROWCOL_SCHEMES = ("fp8_dynamic", "static_tensor")
ROWCOL = {f"{c.name}_{sch}": (c, sch) for c in (workloads.LLAMA_ATTN, workloads.LLAMA_GATE_UP, workloads.LLAMA_DOWN)
          for sch in ROWCOL_SCHEMES}

WORKLOAD_ALIASES = {
    "llama_attn": workloads.LLAMA_ATTN.name, "tiny": workloads.TINY.name,
    "llama_gate_up": workloads.LLAMA_GATE_UP.name, "llama_down": workloads.LLAMA_DOWN.name,
    **{f"ds_decode_m{m}": workloads.DS_DECODE[m].name for m in (1, 8, 32, 64)},
    **{f"ds_decode_m{m}_layers": f"ds_decode_m{m}_layers" for m in (1, 8, 32, 64)},
    "moe": workloads.MOE.name, "moe_small": workloads.MOE_SMALL.name, "moe_fp32": workloads.MOE_F32.name,
    "llama_attn_dynamic": f"{workloads.LLAMA_ATTN.name}_fp8_dynamic",
    "llama_attn_static": f"{workloads.LLAMA_ATTN.name}_static_tensor",
    "llama_gate_up_dynamic": f"{workloads.LLAMA_GATE_UP.name}_fp8_dynamic",
    "llama_down_dynamic": f"{workloads.LLAMA_DOWN.name}_fp8_dynamic",
    "llama_mlp_fused": "llama3_8b_mlp_8192x4096x14336_swiglu_fused",
    "llama_mlp_prefill": "llama3_8b_mlp_prefill_gate_up_8192x28672x4096_down_8192x4096x14336",
    "moe_decode_masked": workloads.MOE_DECODE.name,
    "moe_decode_masked_small": workloads.MOE_DECODE_SMALL.name,
    **{f"{a}_ue8m0": workloads.LLAMA_UE8M0[c.name].name
       for a, c in (("llama_attn", workloads.LLAMA_ATTN), ("llama_gate_up", workloads.LLAMA_GATE_UP),
                    ("llama_down", workloads.LLAMA_DOWN))},
}
MLP_NAME = "llama3_8b_mlp_8192x4096x14336_swiglu_fused"
PREFILL_NAME = "llama3_8b_mlp_prefill_gate_up_8192x28672x4096_down_8192x4096x14336"
DEFAULT_WORKLOAD = "llama_mlp_prefill"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {**FALLBACK_PEAKS, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_sha256(root=None):
    """sha256 over the CUDA sources in name order: each file's name, then its
    text with comments and blank lines removed.  A comment-only edit keeps
    committed ncu counters valid; any change to the code invalidates them."""
    import glob
    import hashlib
    import re
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(root or ROOT, "fine_grained_fp8_token_b200", "csrc", "*"))):
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        code = [line.rstrip() for line in text.splitlines() if line.strip()]
        h.update("\n".join(code).encode())
    return h.hexdigest()


def ncu_traffic(workload_name):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when there is none for this workload or the kernel
    sources changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            cap = json.load(f)["captures"].get(workload_name)
    except (OSError, ValueError, KeyError):
        return None
    if not cap or cap.get("source_sha256") != kernel_source_sha256():
        return None
    return cap["dram_read_bytes"] + cap["dram_write_bytes"]


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle reasons of this GPU, sampled every 10 ms through
    NVML (read-only queries) while the timed region runs."""

    def __init__(self, device_index: int):
        self.ok = False
        self.samples = []
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid).replace("GPU-", "")
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid:
                    handle = h
            if handle is None:
                return
            self.nv, self.h, self.threading = pynvml, handle, threading
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _loop(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                try:
                    watts = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                except Exception:
                    watts = None
                self.samples.append((mhz, reasons, watts))
            except Exception:
                pass
            self.stop_flag.wait(0.01)

    def start(self):
        if not self.ok:
            return
        self.stop_flag = self.threading.Event()
        self.thread = self.threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def stop(self):
        if not self.ok:
            return None
        self.stop_flag.set()
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        nv = self.nv
        names = {"hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
                 "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                 "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                 "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4)}
        seen = set()
        for _, r, _ in self.samples:
            for n, bit in names.items():
                if r & bit:
                    seen.add(n)
        out = {"sm_mhz": statistics.median(m for m, _, _ in self.samples), "sm_max_mhz": self.max_mhz,
               "samples": len(self.samples), "reasons": sorted(seen)}
        watts = [w for _, _, w in self.samples if w is not None]
        if watts:
            out["power_w"] = round(statistics.median(watts), 1)
            out["power_w_max"] = round(max(watts), 1)
        return out


def flush_l2(buf_w, buf_r):
    """Evict L2: write a buffer larger than L2, then read another one so the
    lines left behind are clean (no write-back lands in the next kernel)."""
    buf_w.fill_(1)
    buf_r.sum(dtype=torch.int32)


# ---------------------------------------------------------------- workloads on the GPU
class DenseLayer:
    """X [M, K] bf16 and pre-quantized W for one dense linear layer."""

    def __init__(self, cfg: workloads.Linear, dev):
        import fine_grained_fp8_token_b200 as fg
        self.fg, self.cfg, self.dev = fg, cfg, dev
        self.X = workloads.activations((cfg.M, cfg.K), cfg.x_kind, cfg.seed, device=dev)
        W = workloads.weights((cfg.N, cfg.K), cfg.seed + 1, device=dev)
        sdt = torch.float32 if cfg.fmt == 0 else torch.uint8
        self.W = W
        self.Wq = torch.empty((cfg.N, cfg.K), dtype=torch.uint8, device=dev)
        self.Ws = torch.empty((cfg.N // 128, cfg.K // 128), dtype=sdt, device=dev)
        self.ld_s = fg.scale_rows(cfg.M, cfg.fmt)
        self.Xq = torch.empty((cfg.M, cfg.K), dtype=torch.uint8, device=dev)
        self.Xs = torch.empty((cfg.K // 128, self.ld_s), dtype=sdt, device=dev)
        self.Y = torch.empty((cfg.M, cfg.N), dtype=torch.bfloat16, device=dev)
        self.quant_weight()

    def quant_weight(self):
        self.fg.quant_weight(self.W, self.cfg.fmt, Wq=self.Wq, Ws=self.Ws)

    def quant_act(self, X=None):
        self.fg.quant_act(self.X if X is None else X, self.cfg.fmt, Xq=self.Xq, Xs=self.Xs, ld_s=self.ld_s)

    def gemm(self):
        self.fg.gemm(self.Xq, self.Xs, self.Wq, self.Ws, self.cfg.fmt, Y=self.Y)

    def linear(self, X=None):
        self.fg.linear(self.X if X is None else X, self.Wq, self.Ws, self.cfg.fmt, Y=self.Y, Xq=self.Xq, Xs=self.Xs,
                       ld_s=self.ld_s)

    def flops(self):
        c = self.cfg
        return 2.0 * c.M * c.N * c.K

    def act_bytes(self):
        c = self.cfg
        return 2.0 * c.M * c.K + c.M * c.K + (4 if c.fmt == 0 else 1) * c.M * c.K / 128

    def gemm_bytes(self):
        c = self.cfg
        sb = 4 if c.fmt == 0 else 1
        return c.M * c.K + c.N * c.K + sb * (c.M * c.K / 128 + c.N * c.K / 16384) + 2.0 * c.M * c.N

    def weight_bytes(self):
        c = self.cfg
        return 3.0 * c.N * c.K + (4 if c.fmt == 0 else 1) * c.N * c.K / 16384

    def describe(self):
        c = self.cfg
        return {"workload": c.name, "M": c.M, "N": c.N, "K": c.K,
                "scales": "fp32" if c.fmt == 0 else "ue8m0", "x": c.x_kind}

    def host_io(self):
        return [self.X], [self.Y]

    def gemm_kernel_name(self):
        if self.cfg.M <= 64:
            return "gemm_decode_kernel" if self.cfg.fmt == 0 else "gemm_decode_mx_kernel"
        return "gemm_blockscaled_kernel" if self.cfg.fmt == 0 else "gemm_mx_kernel"


class DecodeSweep:
    """Config-4 decode through L layers: M tokens (1..64) times L distinct
    [18432, 7168] UE8M0 weights (8 x 132 MB, far above the 126 MB L2), as a
    decode step walks through a model's layers.  One step is L calls of
    fgfp8_linear (each quantizer, then its GEMM as the programmatic
    dependent).  Timed apart, the L quantizers run back to back in one event
    pair and the L GEMMs in another, so a kernel's time is its average over a
    stream of launches rather than one launch behind an event (whose fixed
    cost is several microseconds on this GPU)."""

    LAYERS = 8

    def __init__(self, cfg: workloads.Linear, dev):
        import fine_grained_fp8_token_b200 as fg
        self.fg, self.cfg, self.dev = fg, cfg, dev
        self.layers = []
        sdt = torch.float32 if cfg.fmt == 0 else torch.uint8
        for i in range(self.LAYERS):
            sub = workloads.replace(cfg, seed=cfg.seed + 16 * i)
            d = DenseLayer(sub, dev)
            del d.W                                       # keep only the quantized weight
            self.layers.append(d)
        self.W = workloads.weights((cfg.N, cfg.K), cfg.seed + 1, device=dev)   # for the weight-quantizer timing
        self.Wq1 = torch.empty((cfg.N, cfg.K), dtype=torch.uint8, device=dev)
        self.Ws1 = torch.empty((cfg.N // 128, cfg.K // 128), dtype=sdt, device=dev)
        self.X = self.layers[0].X
        self.launches_per_step = 2 * self.LAYERS

    def quant_weight(self):
        self.fg.quant_weight(self.W, self.cfg.fmt, Wq=self.Wq1, Ws=self.Ws1)

    def quant_act(self, X=None):
        for d in self.layers:
            d.quant_act()

    def gemm(self):
        for d in self.layers:
            d.gemm()

    def linear(self, X=None):
        for i, d in enumerate(self.layers):
            d.linear(None if X is None else X[i])

    def flops(self):
        return self.LAYERS * self.layers[0].flops()

    def act_bytes(self):
        return self.LAYERS * self.layers[0].act_bytes()

    def gemm_bytes(self):
        return self.LAYERS * self.layers[0].gemm_bytes()

    def weight_bytes(self):
        return self.layers[0].weight_bytes()

    def describe(self):
        c = self.cfg
        return {"workload": f"{c.name}_x{self.LAYERS}layers", "M": c.M, "N": c.N, "K": c.K, "layers": self.LAYERS,
                "scales": "fp32" if c.fmt == 0 else "ue8m0", "x": c.x_kind,
                "timing": "per-kernel times: L launches back to back in one event pair, divided by L"}

    def host_io(self):
        return [d.X for d in self.layers], [d.Y for d in self.layers]

    def gemm_kernel_name(self):
        return self.layers[0].gemm_kernel_name()


class RowColLayer:
    """One dense layer with row / tensor scale granularity: per-output-channel
    weight scales (fgfp8_quant_rows on W) and either per-token activation
    scales (fgfp8_quant_rows on X, the FP8_DYNAMIC scheme) or one static
    activation scale calibrated once from the layer's input
    (fgfp8_tensor_scale, then fgfp8_quant_static per step).  The GEMM is
    fgfp8_gemm_rowcol."""

    def __init__(self, cfg: workloads.Linear, scheme: str, dev):
        import fine_grained_fp8_token_b200 as fg
        self.fg, self.cfg, self.scheme, self.dev = fg, cfg, scheme, dev
        self.X = workloads.activations((cfg.M, cfg.K), cfg.x_kind, cfg.seed, device=dev)
        self.W = workloads.weights((cfg.N, cfg.K), cfg.seed + 1, device=dev)
        self.Wq = torch.empty((cfg.N, cfg.K), dtype=torch.uint8, device=dev)
        self.sw = torch.empty((cfg.N,), dtype=torch.float32, device=dev)
        self.Xq = torch.empty((cfg.M, cfg.K), dtype=torch.uint8, device=dev)
        if scheme == "fp8_dynamic":
            self.sx = torch.empty((cfg.M,), dtype=torch.float32, device=dev)
        else:
            self.sx = fg.tensor_scale(self.X)             # calibration, before timing
        self.Y = torch.empty((cfg.M, cfg.N), dtype=torch.bfloat16, device=dev)
        self.quant_weight()

    def quant_weight(self):
        self.fg.quant_rows(self.W, Xq=self.Wq, scales=self.sw)

    def quant_act(self, X=None):
        X = self.X if X is None else X
        if self.scheme == "fp8_dynamic":
            self.fg.quant_rows(X, Xq=self.Xq, scales=self.sx)
        else:
            self.fg.quant_static(X, self.sx, Xq=self.Xq)

    def gemm(self):
        self.fg.gemm_rowcol(self.Xq, self.sx, self.Wq, self.sw, Y=self.Y)

    def linear(self, X=None):
        self.quant_act(X)
        self.gemm()

    def flops(self):
        c = self.cfg
        return 2.0 * c.M * c.N * c.K

    def act_bytes(self):
        c = self.cfg
        return 3.0 * c.M * c.K + (4.0 * c.M if self.scheme == "fp8_dynamic" else 0.0)

    def gemm_bytes(self):
        c = self.cfg
        return c.M * c.K + c.N * c.K + 4.0 * (c.M + c.N) + 2.0 * c.M * c.N

    def weight_bytes(self):
        c = self.cfg
        return 3.0 * c.N * c.K + 4.0 * c.N

    def describe(self):
        c = self.cfg
        x = "per-token (dynamic)" if self.scheme == "fp8_dynamic" else "per-tensor (static, calibrated once)"
        return {"workload": f"{c.name}_{self.scheme}", "M": c.M, "N": c.N, "K": c.K,
                "scales": f"fp32, activations {x}, weights per output channel", "x": c.x_kind}

    def host_io(self):
        return [self.X], [self.Y]

    def gemm_kernel_name(self):
        return "gemm_rowcol_kernel"


class PrefillMLP:
    """The Llama-3-8B MLP in prefill as two dense W8A8 linear layers, each one
    fgfp8_linear call (the 1x128 quantizer, then the block-scaled GEMM as its
    programmatic dependent), fp32 block scales: the fused gate/up projection
    X [8192, 4096] (N(0, 1) with 0.1% outliers x50) x W [28672, 4096], then
    the down projection X [8192, 14336] (sign(z)|z|^1.5, a post-SiLU-like
    heavy tail) x W [4096, 14336].  Both bf16 outputs are written.  The down
    input is its own seeded synthetic tensor, not derived from the gate/up
    output (the SwiGLU chain between them is the separate fused workload)."""

    launches_per_step = 4

    def __init__(self, dev, tokens=None):
        import fine_grained_fp8_token_b200 as fg
        self.fg, self.dev = fg, dev
        g, d = workloads.LLAMA_GATE_UP, workloads.LLAMA_DOWN
        if tokens:                            # a smaller token batch (profiling captures)
            g = workloads.replace(g, name=f"{g.name}@{tokens}tok", M=tokens)
            d = workloads.replace(d, name=f"{d.name}@{tokens}tok", M=tokens)
        self.tokens = tokens
        self.gu = DenseLayer(g, dev)
        self.down = DenseLayer(d, dev)
        self.X = self.gu.X

    def quant_weight(self):
        self.gu.quant_weight()

    def linear(self, X=None):
        self.gu.linear(None if X is None else X[0])
        self.down.linear(None if X is None else X[1])

    def kernel_steps(self):
        """The step's kernels in launch order, for timing them apart."""
        return [("quant_act_gate_up", self.gu.quant_act), ("gemm", self.gu.gemm),
                ("quant_act", self.down.quant_act), ("gemm_down", self.down.gemm)]

    def flops(self):
        return self.gu.flops() + self.down.flops()

    def kernel_flops(self):
        return {"gemm": self.gu.flops(), "gemm_down": self.down.flops()}

    def act_bytes(self):
        return self.down.act_bytes()           # the act-quant line: the 8192 x 14336 input

    def kernel_bytes(self):
        return {"quant_act_gate_up": self.gu.act_bytes(), "quant_act": self.down.act_bytes(),
                "gemm": self.gu.gemm_bytes(), "gemm_down": self.down.gemm_bytes()}

    def gemm_bytes(self):
        return self.gu.gemm_bytes()            # the roofline kernel: the gate/up GEMM

    def weight_bytes(self):
        return self.gu.weight_bytes()

    def describe(self):
        g, d = self.gu.cfg, self.down.cfg
        return {"workload": PREFILL_NAME if not self.tokens else f"{PREFILL_NAME}@{self.tokens}tok",
                "layers": [{"name": "gate_up", "M": g.M, "N": g.N, "K": g.K, "x": g.x_kind},
                           {"name": "down", "M": d.M, "N": d.N, "K": d.K, "x": d.x_kind}],
                "scales": "fp32 (1x128 activations, 128x128 weights)",
                "roofline_kernel": "gate/up GEMM", "act_quant_line": "down-projection input 8192 x 14336"}

    def host_io(self):
        return [self.gu.X, self.down.X], [self.gu.Y, self.down.Y]

    def gemm_kernel_name(self):
        return "gemm_blockscaled_kernel (gate/up 8192x28672x4096)"


class MLPLayer:
    """The Llama-3-8B MLP in prefill (X [8192, 4096], gate/up [2 x 14336,
    4096], down [4096, 14336], fp32 block scales) as three kernels: the 1x128
    activation quantizer, the gate/up GEMM fused with SiLU * up and the down
    projection's quantizer (fgfp8_gemm_swiglu_quant: the bf16 [8192, 28672]
    gate/up output is never written), and the down GEMM."""

    M, K, I, N_DOWN = 8192, 4096, 14336, 4096
    launches_per_step = 3

    def __init__(self, dev, tokens=None):
        import fine_grained_fp8_token_b200 as fg
        self.fg, self.dev = fg, dev
        if tokens:
            self.M = tokens                 # a smaller token batch of the same layer (profiling captures)
        c = workloads.LLAMA_GATE_UP
        self.X = workloads.activations((self.M, self.K), c.x_kind, c.seed, device=dev)
        Wg = workloads.weights((self.I, self.K), c.seed + 1, device=dev)
        Wu = workloads.weights((self.I, self.K), c.seed + 2, device=dev)
        self.W_gu = fg.interleave_gate_up(Wg, Wu)
        del Wg, Wu
        self.W_down = workloads.weights((self.N_DOWN, self.I), c.seed + 3, device=dev)
        self.Wq_gu = torch.empty((2 * self.I, self.K), dtype=torch.uint8, device=dev)
        self.Ws_gu = torch.empty((2 * self.I // 128, self.K // 128), dtype=torch.float32, device=dev)
        self.Wq_d = torch.empty((self.N_DOWN, self.I), dtype=torch.uint8, device=dev)
        self.Ws_d = torch.empty((self.N_DOWN // 128, self.I // 128), dtype=torch.float32, device=dev)
        self.ld_s = fg.scale_rows(self.M, 0)
        self.Xq = torch.empty((self.M, self.K), dtype=torch.uint8, device=dev)
        self.Xs = torch.empty((self.K // 128, self.ld_s), dtype=torch.float32, device=dev)
        self.Hq = torch.empty((self.M, self.I), dtype=torch.uint8, device=dev)
        self.Hs = torch.empty((self.I // 128, self.ld_s), dtype=torch.float32, device=dev)
        self.Y = torch.empty((self.M, self.N_DOWN), dtype=torch.bfloat16, device=dev)
        self.quant_weight()
        fg.quant_weight(self.W_down, 0, Wq=self.Wq_d, Ws=self.Ws_d)
        self.W = self.W_gu

    def quant_weight(self):
        self.fg.quant_weight(self.W_gu, 0, Wq=self.Wq_gu, Ws=self.Ws_gu)

    def quant_act(self, X=None):
        self.fg.quant_act(self.X if X is None else X, 0, Xq=self.Xq, Xs=self.Xs, ld_s=self.ld_s)

    def gemm(self):
        self.fg.gemm_swiglu_quant(self.Xq, self.Xs, self.Wq_gu, self.Ws_gu, Hq=self.Hq, Hs=self.Hs, ld_h=self.ld_s)
        self.fg.gemm(self.Hq, self.Hs, self.Wq_d, self.Ws_d, 0, Y=self.Y)

    def linear(self, X=None):
        self.quant_act(X)
        self.gemm()

    def flops(self):
        return 2.0 * self.M * (2 * self.I) * self.K + 2.0 * self.M * self.N_DOWN * self.I

    def act_bytes(self):
        return 3.0 * self.M * self.K + 4.0 * self.M * self.K / 128

    def gemm_bytes(self):
        # operands read once, h written once and read once (codes and scales), Y written
        h = self.M * self.I * (1 + 4.0 / 128)
        return (self.M * self.K + 2 * self.I * self.K + self.N_DOWN * self.I + 4.0 * (self.M * self.K + 2 * self.I
                * self.K + self.N_DOWN * self.I) / 128 / 128 + 2 * h + 2.0 * self.M * self.N_DOWN)

    def weight_bytes(self):
        return 3.0 * 2 * self.I * self.K + 4.0 * 2 * self.I * self.K / 16384

    def describe(self):
        return {"workload": MLP_NAME if self.M == MLPLayer.M else f"{MLP_NAME}@{self.M}tok", "M": self.M,
                "K": self.K, "I": self.I, "N_down": self.N_DOWN,
                "scales": "fp32 (1x128 activations, 128x128 weights)", "x": "normal_outliers",
                "chain": "quant_act -> gate/up GEMM + SiLU*up + quant (fused) -> down GEMM"}

    def host_io(self):
        return [self.X], [self.Y]

    def gemm_kernel_name(self):
        return "gemm_blockscaled_kernel (fused SwiGLU) + gemm_blockscaled_kernel"


class MaskedMoELayer:
    """Decode step of the expert layer in the masked layout: 128 tokens
    routed top-8 (Zipf-skewed) to 256 experts, every expert a fixed block of
    cap = 128 rows of which the first counts[e] hold tokens; the step is
    fgfp8_masked_linear: the 1x128 quantizer over the token rows only, then
    the masked GEMM as its programmatic dependent.  Experts without tokens
    are skipped, so the GEMM streams the weights of the active experts only."""

    CAP = 128

    def __init__(self, cfg: workloads.MoE, dev):
        import fine_grained_fp8_token_b200 as fg
        self.fg, self.cfg, self.dev = fg, cfg, dev
        self.r = workloads.moe_routing(cfg)
        self.X = workloads.moe_masked_rows(workloads.moe_tokens(cfg, device=dev), self.r, cfg.E, self.CAP)
        sdt = torch.float32 if cfg.fmt == 0 else torch.uint8
        self.Wq = torch.empty((cfg.E, cfg.N, cfg.K), dtype=torch.uint8, device=dev)
        self.Ws = torch.empty((cfg.E, cfg.N // 128, cfg.K // 128), dtype=sdt, device=dev)
        for e in range(cfg.E):
            fg.quant_weight(workloads.moe_expert_weight(cfg, e, device=dev), cfg.fmt, Wq=self.Wq[e], Ws=self.Ws[e])
        self.counts = torch.as_tensor(self.r.counts.astype(np.int32), device=dev)
        M = cfg.E * self.CAP
        self.ld_s = fg.scale_rows(M, cfg.fmt)
        self.Xq = torch.empty((M, cfg.K), dtype=torch.uint8, device=dev)
        self.Xs = torch.empty((cfg.K // 128, self.ld_s), dtype=sdt, device=dev)
        self.Y = torch.empty((M, cfg.N), dtype=torch.bfloat16, device=dev)
        self.W = workloads.moe_expert_weight(cfg, 0, device=dev)
        self.active = int((self.r.counts > 0).sum())

    def quant_weight(self):
        self.fg.quant_weight(self.W, self.cfg.fmt, Wq=self.Wq[0], Ws=self.Ws[0])

    def quant_act(self, X=None):
        # the token rows only: padding rows are never read by the masked GEMM
        self.fg.quant_act_masked(self.X if X is None else X, self.counts, self.cfg.E, self.cfg.fmt, Xq=self.Xq,
                                 Xs=self.Xs, ld_s=self.ld_s)

    def gemm(self):
        self.fg.masked_gemm(self.Xq, self.Xs, self.Wq, self.Ws, self.counts, self.cfg.fmt, Y=self.Y)

    def linear(self, X=None):
        self.fg.masked_linear(self.X if X is None else X, self.Wq, self.Ws, self.counts, self.cfg.fmt, Y=self.Y,
                              Xq=self.Xq, Xs=self.Xs, ld_s=self.ld_s)

    def flops(self):
        c = self.cfg
        return 2.0 * float(self.r.counts.sum()) * c.N * c.K

    def act_bytes(self):
        # the token rows read and their codes and scales written
        c = self.cfg
        rows = float(self.r.counts.sum())
        return 3.0 * rows * c.K + (4 if c.fmt == 0 else 1) * rows * c.K / 128

    def gemm_bytes(self):
        # the active experts' weights and scales, the token rows' codes and scales, Y's token rows
        c = self.cfg
        rows = float(self.r.counts.sum())
        sb = 4 if c.fmt == 0 else 1
        return (self.active * c.N * c.K * (1 + sb / 16384.0) + rows * c.K * (1 + sb / 128.0)
                + 2.0 * rows * c.N)

    def weight_bytes(self):
        c = self.cfg
        return 3.0 * c.N * c.K + (4 if c.fmt == 0 else 1) * c.N * c.K / 16384

    def describe(self):
        c = self.cfg
        return {"workload": c.name, "experts": c.E, "active_experts": self.active, "cap": self.CAP, "N": c.N,
                "K": c.K, "tokens": c.tokens, "topk": c.topk, "zipf": c.zipf,
                "rows_routed": int(self.r.counts.sum()), "max_rows_per_expert": int(self.r.counts.max()),
                "scales": "fp32" if c.fmt == 0 else "ue8m0"}

    def host_io(self):
        return [self.X], [self.Y]

    def gemm_kernel_name(self):
        return ("gemm_blockscaled_kernel" if self.cfg.fmt == 0 else "gemm_mx_kernel") + " (masked)"


class MoELayer:
    """Grouped expert layer: routed token rows and pre-quantized experts."""

    def __init__(self, cfg: workloads.MoE, dev):
        import fine_grained_fp8_token_b200 as fg
        self.fg, self.cfg, self.dev = fg, cfg, dev
        self.r = workloads.moe_routing(cfg)
        self.X = workloads.moe_grouped_rows(workloads.moe_tokens(cfg, device=dev), self.r)
        sdt = torch.float32 if cfg.fmt == 0 else torch.uint8
        self.Wq = torch.empty((cfg.E, cfg.N, cfg.K), dtype=torch.uint8, device=dev)
        self.Ws = torch.empty((cfg.E, cfg.N // 128, cfg.K // 128), dtype=sdt, device=dev)
        for e in range(cfg.E):
            fg.quant_weight(workloads.moe_expert_weight(cfg, e, device=dev), cfg.fmt, Wq=self.Wq[e], Ws=self.Ws[e])
        self.offs = torch.as_tensor(self.r.group_offs, device=dev)
        M = self.r.M_total
        self.ld_s = fg.scale_rows(M, cfg.fmt)
        self.Xq = torch.empty((M, cfg.K), dtype=torch.uint8, device=dev)
        self.Xs = torch.empty((cfg.K // 128, self.ld_s), dtype=sdt, device=dev)
        self.Y = torch.empty((M, cfg.N), dtype=torch.bfloat16, device=dev)
        self.W = workloads.moe_expert_weight(cfg, 0, device=dev)     # for timing the weight quantizer

    def quant_weight(self):
        self.fg.quant_weight(self.W, self.cfg.fmt, Wq=self.Wq[0], Ws=self.Ws[0])

    def quant_act(self, X=None):
        self.fg.quant_act(self.X if X is None else X, self.cfg.fmt, Xq=self.Xq, Xs=self.Xs, ld_s=self.ld_s)

    def gemm(self):
        self.fg.grouped_gemm(self.Xq, self.Xs, self.Wq, self.Ws, self.offs, self.cfg.fmt, Y=self.Y)

    def linear(self, X=None):
        self.fg.grouped_linear(self.X if X is None else X, self.Wq, self.Ws, self.offs, self.cfg.fmt, Y=self.Y,
                               Xq=self.Xq, Xs=self.Xs, ld_s=self.ld_s)

    def flops(self):
        c = self.cfg
        return 2.0 * float(self.r.counts.sum()) * c.N * c.K      # useful rows only, no padding

    def act_bytes(self):
        c = self.cfg
        M = self.r.M_total
        return 3.0 * M * c.K + (4 if c.fmt == 0 else 1) * M * c.K / 128

    def gemm_bytes(self):
        c = self.cfg
        M = self.r.M_total
        sb = 4 if c.fmt == 0 else 1
        return M * c.K + c.E * c.N * c.K + sb * (M * c.K / 128 + c.E * c.N * c.K / 16384) + 2.0 * M * c.N

    def weight_bytes(self):
        c = self.cfg
        return 3.0 * c.N * c.K + (4 if c.fmt == 0 else 1) * c.N * c.K / 16384

    def describe(self):
        c = self.cfg
        return {"workload": c.name, "experts": c.E, "N": c.N, "K": c.K, "tokens": c.tokens, "topk": c.topk,
                "zipf": c.zipf, "M_total_padded": self.r.M_total, "rows_routed": int(self.r.counts.sum()),
                "max_rows_per_expert": int(self.r.counts.max()), "scales": "fp32" if c.fmt == 0 else "ue8m0"}

    def host_io(self):
        return [self.X], [self.Y]

    def gemm_kernel_name(self):
        return ("gemm_blockscaled_kernel" if self.cfg.fmt == 0 else "gemm_mx_kernel") + " (grouped)"


def make_layer(name, dev, tokens=None):
    name = WORKLOAD_ALIASES.get(name, name)
    for cfg in (workloads.MOE_DECODE, workloads.MOE_DECODE_SMALL):
        if name == cfg.name:
            return MaskedMoELayer(cfg, dev)
    if name == MLP_NAME:
        return MLPLayer(dev, tokens)
    if name == PREFILL_NAME:
        return PrefillMLP(dev, tokens)
    if name in ROWCOL:
        cfg, scheme = ROWCOL[name]
        return RowColLayer(cfg, scheme, dev)
    for cfg in (workloads.MOE, workloads.MOE_SMALL, workloads.MOE_F32):
        if name == cfg.name:
            return MoELayer(cfg, dev)
    for m, cfg in workloads.DS_DECODE.items():
        if name in (f"{cfg.name}_x{DecodeSweep.LAYERS}layers", f"ds_decode_m{m}_layers"):
            return DecodeSweep(cfg, dev)
    cfg = workloads.LINEARS[name]
    if tokens:                                # a smaller token batch of the same layer (profiling captures)
        cfg = workloads.replace(cfg, name=f"{cfg.name}@{tokens}tok", M=tokens)
    return DenseLayer(cfg, dev)


# ---------------------------------------------------------------- ranks
def max_over_ranks(times, world, device):
    """Element-wise max of per-rank timings: the job takes as long as its
    slowest replica.  Every rank calls this exactly once per run, in the same
    order, so the collective sequence matches on all ranks."""
    t = torch.tensor([float(x) for x in times], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(world, units_per_rank, ms):
    """Units processed by all ranks per second, in units / 1e12 (TFLOP/s for
    FLOPs), when each of `world` replicas processes `units_per_rank` and the
    slowest takes `ms` milliseconds."""
    return world * units_per_rank / (ms / 1e3) / 1e12


# ---------------------------------------------------------------- end to end
E2E_CHUNKS = 4


def streamed_parts(layer):
    """The dense layers of a step whose token rows can be streamed through
    host copies in chunks (each output row depends on its own input row
    only), or None for workloads run in one piece."""
    if isinstance(layer, PrefillMLP):
        return [layer.gu, layer.down]
    if type(layer) is DenseLayer and layer.cfg.M >= 1024:
        return [layer]
    return None


def e2e_streamed(parts, X_hosts, X_stages, Y_hosts, stream, dev, start):
    """One end-to-end step of the dense layers `parts`, streamed over
    E2E_CHUNKS token chunks each: chunk copies host -> device on one stream,
    fgfp8_linear of the chunk on the compute stream once its rows are in,
    and the chunk's output device -> host on a third stream once computed,
    so the two copy directions overlap each other and the compute.  Every
    stream starts after `start` and the compute stream waits for the last
    copy out, so an event recorded next on it closes the step."""
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_in.wait_event(start)
    s_out.wait_event(start)
    chunks = []                                  # (part index, r0, r1)
    for i, d in enumerate(parts):
        M = d.cfg.M
        bounds = [(M * c // E2E_CHUNKS) // 16 * 16 for c in range(E2E_CHUNKS)] + [M]
        chunks += [(i, r0, r1) for r0, r1 in zip(bounds, bounds[1:]) if r1 > r0]
    ev_in = []
    for i, r0, r1 in chunks:
        with torch.cuda.stream(s_in):
            X_stages[i][r0:r1].copy_(X_hosts[i][r0:r1], non_blocking=True)
        e = torch.cuda.Event()
        e.record(s_in)
        ev_in.append(e)
    ev_c = []
    for (i, r0, r1), e in zip(chunks, ev_in):
        d = parts[i]
        stream.wait_event(e)
        d.fg.linear(X_stages[i][r0:r1], d.Wq, d.Ws, d.cfg.fmt, Y=d.Y[r0:r1], Xq=d.Xq[r0:r1], Xs=d.Xs[:, r0:],
                    ld_s=d.ld_s, stream=stream)
        e2 = torch.cuda.Event()
        e2.record(stream)
        ev_c.append(e2)
    for (i, r0, r1), e2 in zip(chunks, ev_c):
        s_out.wait_event(e2)
        with torch.cuda.stream(s_out):
            Y_hosts[i][r0:r1].copy_(parts[i].Y[r0:r1], non_blocking=True)
    done = torch.cuda.Event()
    done.record(s_out)
    stream.wait_event(done)


# ---------------------------------------------------------------- timing
def run_gpu(args, rank, world, dev):
    """Times the hot path on this rank.  The step is one call of the layer
    (fgfp8_linear / fgfp8_grouped_linear: the quantizer, then the GEMM as its
    programmatic dependent; two such calls for the prefill MLP), bracketed by
    CUDA events; a second pass of the same length times the kernels apart (an
    event between consecutive ones) for the per-kernel roofline."""
    layer = make_layer(args.workload, dev, args.tokens)
    stream = torch.cuda.current_stream(dev)
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    launches_per_step = getattr(layer, "launches_per_step", 2)
    kernels = (layer.kernel_steps() if hasattr(layer, "kernel_steps")
               else [("quant_act", layer.quant_act), ("gemm", layer.gemm)])

    for _ in range(args.warmup):
        flush_l2(flush_w, flush_r)
        layer.linear()
        flush_l2(flush_w, flush_r)
        for _, f in kernels:
            f()
    layer.fg.check_device_status()

    n = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(kernels) + 1)] for _ in range(n)]
    sampler = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    time.sleep(REST_S)
    sampler.start()
    for i in range(n):
        flush_l2(flush_w, flush_r)
        ev[i][0].record(stream)
        layer.linear()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    layer.fg.check_device_status()
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(n)]
    total_ms = sum(step_ms)

    # the kernels timed apart (same flush between steps), from the same idle
    # start as the step pass
    ksampler = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    time.sleep(REST_S)
    ksampler.start()
    for i in range(n):
        flush_l2(flush_w, flush_r)
        kev[i][0].record(stream)
        for j, (_, f) in enumerate(kernels):
            f()
            kev[i][j + 1].record(stream)
    torch.cuda.synchronize(dev)
    kclocks = ksampler.stop()
    layer.fg.check_device_status()
    kern_ms = [sum(kev[i][j].elapsed_time(kev[i][j + 1]) for i in range(n)) for j in range(len(kernels))]

    # weight quantization (offline step, reported, not part of the step)
    wq_ms = []
    for _ in range(max(3, min(n, 10))):
        flush_l2(flush_w, flush_r)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        layer.quant_weight()
        b.record(stream)
        torch.cuda.synchronize(dev)
        wq_ms.append(a.elapsed_time(b))

    # end to end through the public API with host buffers: pinned X in,
    # quantize + GEMM, pinned Y out, copies inside the timed events
    X_devs, Y_devs = layer.host_io()
    X_hosts = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in X_devs]
    for xh, xd in zip(X_hosts, X_devs):
        xh.copy_(xd)
    Y_hosts = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for y in Y_devs]
    X_stages = [torch.empty_like(x) for x in X_devs]
    e2e_ms = []
    e2e_steps = max(3, min(n, 10))
    parts = streamed_parts(layer)
    for i in range(e2e_steps + 2):
        flush_l2(flush_w, flush_r)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if parts:
            e2e_streamed(parts, X_hosts, X_stages, Y_hosts, stream, dev, a)
        else:
            for xs, xh in zip(X_stages, X_hosts):
                xs.copy_(xh, non_blocking=True)
            layer.linear(X_stages[0] if len(X_stages) == 1 else X_stages)
            for yh, yd in zip(Y_hosts, Y_devs):
                yh.copy_(yd, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize(dev)
        if i >= 2:
            e2e_ms.append(a.elapsed_time(b))
    h2d = sum(x.numel() * x.element_size() for x in X_hosts)
    d2h = sum(y.numel() * y.element_size() for y in Y_hosts)

    vals = max_over_ranks([total_ms, *kern_ms, statistics.mean(e2e_ms), statistics.mean(wq_ms)], world, dev)
    total_ms, kern_tot, e2e_mean, wq_mean = vals[0], vals[1:1 + len(kernels)], vals[-2], vals[-1]
    kernel_ms = {name: t / n for (name, _), t in zip(kernels, kern_tot)}
    return layer, {"total_ms": total_ms, "kernel_ms": kernel_ms, "gemm_ms": kernel_ms["gemm"],
                   "quant_ms": kernel_ms["quant_act"], "e2e_ms": e2e_mean, "wq_ms": wq_mean, "clocks": clocks,
                   "clocks_kernels": kclocks,
                   "h2d": h2d, "d2h": d2h, "launches": launches_per_step * n}


# ---------------------------------------------------------------- CPU oracle timing
def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleSample:
    """The oracle on a bounded sample of the workload: r rows of X quantized
    and multiplied by the (pre-quantized, untimed) full weight."""

    def __init__(self, name, rows):
        import oracle
        self.oracle = oracle
        name = WORKLOAD_ALIASES.get(name, name)
        self.scheme = None
        if name == MLP_NAME:
            c = workloads.LLAMA_GATE_UP
            X = workloads.activations((MLPLayer.M, MLPLayer.K), c.x_kind, c.seed)[:rows]
            Wg = workloads.weights((MLPLayer.I, MLPLayer.K), c.seed + 1)
            Wu = workloads.weights((MLPLayer.I, MLPLayer.K), c.seed + 2)
            Wd = workloads.weights((MLPLayer.N_DOWN, MLPLayer.I), c.seed + 3)
            b = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
            self.scheme, self.fmt = "mlp", 0
            self.X = b(X)
            self.Wq_g, self.Ws_g = oracle.quant_weight(b(Wg), 0)
            self.Wq_u, self.Ws_u = oracle.quant_weight(b(Wu), 0)
            self.Wq_d, self.Ws_d = oracle.quant_weight(b(Wd), 0)
            self.rows = self.X.shape[0]
            self.N, self.K = MLPLayer.N_DOWN, MLPLayer.K
            self.desc = (f"first {self.rows} of {MLPLayer.M} tokens through gate/up, SiLU * up, the 1x128 "
                         f"quantizer and down")
            return
        if name == PREFILL_NAME:
            b = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
            self.scheme, self.fmt = "prefill", 0
            self.layers = []
            for cfg in (workloads.LLAMA_GATE_UP, workloads.LLAMA_DOWN):
                X, W = workloads.linear_inputs(cfg)
                Wq, Ws = oracle.quant_weight(b(W), 0)
                self.layers.append((np.ascontiguousarray(b(X[:rows])), Wq, Ws))
            self.rows = self.layers[0][0].shape[0]
            self.N, self.K = workloads.LLAMA_DOWN.N, workloads.LLAMA_GATE_UP.K
            self.desc = (f"first {self.rows} of 8192 tokens through the gate/up layer [28672, 4096] and the down "
                         f"layer [4096, 14336]")
            return
        if name in ROWCOL:
            cfg, self.scheme = ROWCOL[name]
            X, W = workloads.linear_inputs(cfg)
            self.N, self.K, self.fmt = cfg.N, cfg.K, cfg.fmt
            xb = X.contiguous().view(torch.int16).numpy().view(np.uint16)
            self.sx_static = oracle.tensor_scale(xb) if self.scheme == "static_tensor" else None
            self.X = np.ascontiguousarray(xb[:rows])
            self.Wq, self.sw = oracle.quant_rows(W.contiguous().view(torch.int16).numpy().view(np.uint16))
            self.rows = self.X.shape[0]
            self.desc = (f"first {self.rows} of {cfg.M} rows x the full [{cfg.N}, {cfg.K}] weight, "
                         f"{self.scheme} scales")
            return
        moe = {c.name: c for c in (workloads.MOE, workloads.MOE_SMALL, workloads.MOE_F32, workloads.MOE_DECODE,
                                   workloads.MOE_DECODE_SMALL)}
        if name in moe:
            cfg = moe[name]
            r = workloads.moe_routing(cfg)
            e = int(np.argmax(r.counts))                    # the busiest expert's rows
            tok = r.row_token[r.group_offs[e]:r.group_offs[e] + r.counts[e]]
            X = workloads.moe_tokens(cfg)[torch.as_tensor(tok[:rows])]
            W = workloads.moe_expert_weight(cfg, e)
            self.N, self.K, self.fmt = cfg.N, cfg.K, cfg.fmt
            self.desc = f"{min(rows, len(tok))} routed rows of expert {e} x its [4096, 7168] weight"
        else:
            cfg = workloads.LINEARS.get(name)
            if cfg is None:                             # the decode sweep: one layer's sample
                cfg = next(c for m, c in workloads.DS_DECODE.items()
                           if name in (f"{c.name}_x{DecodeSweep.LAYERS}layers", f"ds_decode_m{m}_layers"))
            X, W = workloads.linear_inputs(cfg)
            X = X[:rows]
            self.N, self.K, self.fmt = cfg.N, cfg.K, cfg.fmt
            self.desc = f"first {min(rows, cfg.M)} of {cfg.M} rows x the full [{cfg.N}, {cfg.K}] weight"
        self.X = X.contiguous().view(torch.int16).numpy().view(np.uint16)
        self.Wq, self.Ws = oracle.quant_weight(W.contiguous().view(torch.int16).numpy().view(np.uint16), self.fmt)
        self.rows = self.X.shape[0]

    def step(self):
        if self.scheme == "prefill":
            for X, Wq, Ws in self.layers:
                Xq, Xs = self.oracle.quant_act(X, 0)
                self.oracle.gemm(Xq, Xs, Wq, Ws, 0)
            return
        if self.scheme == "mlp":
            Xq, Xs = self.oracle.quant_act(self.X, 0)
            g, _ = self.oracle.gemm(Xq, Xs, self.Wq_g, self.Ws_g, 0)
            u, _ = self.oracle.gemm(Xq, Xs, self.Wq_u, self.Ws_u, 0)
            h = self.oracle.bf16_rne(self.oracle.silu_mul(g, u))
            Hq, Hs = self.oracle.quant_act(h, 0)
            self.oracle.gemm(Hq, Hs, self.Wq_d, self.Ws_d, 0)
            return
        if self.scheme == "fp8_dynamic":
            Xq, sx = self.oracle.quant_rows(self.X)
            self.oracle.gemm_rowcol(Xq, sx, self.Wq, self.sw)
            return
        if self.scheme == "static_tensor":
            Xq = self.oracle.quant_static(self.X, self.sx_static)
            self.oracle.gemm_rowcol(Xq, np.array([self.sx_static], dtype=np.float32), self.Wq, self.sw)
            return
        Xq, Xs = self.oracle.quant_act(self.X, self.fmt)
        self.oracle.gemm(Xq, Xs, self.Wq, self.Ws, self.fmt)

    def flops(self):
        if self.scheme == "prefill":
            g, d = workloads.LLAMA_GATE_UP, workloads.LLAMA_DOWN
            return 2.0 * self.rows * (g.N * g.K + d.N * d.K)
        if self.scheme == "mlp":
            return 2.0 * self.rows * (2 * MLPLayer.I * MLPLayer.K + MLPLayer.N_DOWN * MLPLayer.I)
        return 2.0 * self.rows * self.N * self.K


def calibrated_sample(name, target_s):
    """Grow the row sample until one oracle step takes about target_s."""
    rows = 4
    s = OracleSample(name, rows)
    t0 = time.perf_counter()
    s.step()
    dt = max(time.perf_counter() - t0, 1e-3)
    rows = max(1, int(rows * target_s / dt))
    return OracleSample(name, rows)


def cpu_baseline(name, target_s=15.0):
    os.environ.setdefault("OMP_NUM_THREADS", str(cpu_cores()))
    s = calibrated_sample(name, target_s / 3)
    t0 = time.perf_counter()
    reps = 0
    while time.perf_counter() - t0 < target_s or reps == 0:
        s.step()
        reps += 1
    dt = (time.perf_counter() - t0) / reps
    return {"value": s.flops() / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{s.desc}, fmt {'fp32' if s.fmt == 0 else 'ue8m0'}; quantize + GEMM per step, "
                      f"{reps} steps of {dt:.2f} s"}


REFERENCE_RUN_SECONDS = 150.0


def reference_step_seconds(steps, warmup, budget_s=REFERENCE_RUN_SECONDS):
    """Target duration of one oracle step so that warm-up plus timed steps end
    within about budget_s (at most 2 s a step)."""
    return min(2.0, budget_s / max(1, steps + warmup))


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    os.environ.setdefault("OMP_NUM_THREADS", str(cpu_cores()))
    s = calibrated_sample(args.workload, reference_step_seconds(args.steps, args.warmup))
    for _ in range(args.warmup):
        s.step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        s.step()
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = s.flops() / (ms / 1e3) / 1e12
    name = WORKLOAD_ALIASES.get(args.workload, args.workload)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name, "sample_rows": s.rows, "parallelism": "host cores (OpenMP)"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                             "sample": s.desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fgfp8", choices=["fgfp8", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="one of: " + ", ".join(WORKLOAD_ALIASES))
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing (quick runs)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--tokens", type=int, default=None,
                    help="token batch M of the MLP and dense workloads (default: the workload's own; smaller for "
                         "profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        return run_reference(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    layer, r = run_gpu(args, rank, world, dev)
    peaks = measured_peaks()
    n = args.steps
    step_ms = r["total_ms"] / n
    flops = layer.flops()
    value = whole_job_rate(world, flops, step_ms)
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    gemm_flops = layer.kernel_flops()["gemm"] if hasattr(layer, "kernel_flops") else flops
    gemm_tflops = gemm_flops / (r["gemm_ms"] / 1e3) / 1e12
    gemm_gbs = layer.gemm_bytes() / (r["gemm_ms"] / 1e3) / 1e9
    act_gbs = layer.act_bytes() / (r["quant_ms"] / 1e3) / 1e9
    wq_gbs = layer.weight_bytes() / (r["wq_ms"] / 1e3) / 1e9
    hbm_bound = gemm_tflops / fp8_peak < gemm_gbs / peaks["hbm_gbs"]
    if hbm_bound:
        roofline = {"bound": "hbm", "achieved": gemm_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": gemm_gbs / peaks["hbm_gbs"], "traffic": ncu_traffic(layer.describe()["workload"]),
                    "kernel": layer.gemm_kernel_name(),
                    "peak_source": f"{peaks['source']} HBM copy bandwidth"}
    else:
        roofline = {"bound": "tensor", "achieved": gemm_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                    "frac": gemm_tflops / fp8_peak, "traffic": ncu_traffic(layer.describe()["workload"]),
                    "kernel": layer.gemm_kernel_name(),
                    "peak_source": f"{peaks['source']} cuBLAS bf16 burst x {FP8_OVER_BF16:g} (nominal fp8/bf16)"}
    line = {
        "impl": "fgfp8", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": n,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3xe4m3->f32", "data": "synthetic (seeded, see workloads/)",
        "config": {**layer.describe(), "l2": "flushed before every timed step (256 MB write, then 256 MB read)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": roofline,
        "kernels": {
            "gemm": {"us": 1e3 * r["gemm_ms"], "tflops": gemm_tflops, "frac_fp8_peak": gemm_tflops / fp8_peak,
                     "gbs": gemm_gbs, "frac_hbm": gemm_gbs / peaks["hbm_gbs"]},
            "quant_act": {"us": 1e3 * r["quant_ms"], "gbs": act_gbs, "frac_hbm": act_gbs / peaks["hbm_gbs"],
                          "bytes": layer.act_bytes()},
            "quant_weight_offline": {"us": 1e3 * r["wq_ms"], "gbs": wq_gbs, "frac_hbm": wq_gbs / peaks["hbm_gbs"],
                                     "bytes": layer.weight_bytes()},
            "apart_sum_us": 1e3 * sum(r["kernel_ms"].values()),
        },
        "step_call": ("fgfp8_quant_act + fgfp8_gemm_swiglu_quant + fgfp8_gemm" if isinstance(layer, MLPLayer) else
                      "fgfp8_linear (gate/up) + fgfp8_linear (down)" if isinstance(layer, PrefillMLP) else
                      "fgfp8_masked_linear" if isinstance(layer, MaskedMoELayer) else
                      "fgfp8_grouped_linear" if isinstance(layer, MoELayer) else
                      ("fgfp8_quant_rows + fgfp8_gemm_rowcol" if getattr(layer, "scheme", None) == "fp8_dynamic"
                       else "fgfp8_quant_static + fgfp8_gemm_rowcol") if isinstance(layer, RowColLayer)
                      else "fgfp8_linear"),
        "e2e": {"value": whole_job_rate(world, flops, r["e2e_ms"]), "unit": "TFLOP/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"], "ms_per_step": r["e2e_ms"],
                "pipeline": (f"{E2E_CHUNKS} token chunks per layer: copy in, fgfp8_linear, copy out on three "
                             f"streams" if streamed_parts(layer) else "copy in, the step, copy out on one stream")},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
        "clocks_kernels": r["clocks_kernels"],
        "peaks": peaks,
    }
    if hasattr(layer, "kernel_flops"):
        kb = layer.kernel_bytes()
        for name, f in layer.kernel_flops().items():
            if name != "gemm":
                t = r["kernel_ms"][name] / 1e3
                line["kernels"][name] = {"us": 1e6 * t, "tflops": f / t / 1e12, "frac_fp8_peak": f / t / 1e12 / fp8_peak,
                                         "gbs": kb[name] / t / 1e9, "frac_hbm": kb[name] / t / 1e9 / peaks["hbm_gbs"]}
        for name, b in kb.items():
            if name.startswith("quant_act") and name != "quant_act":
                t = r["kernel_ms"][name] / 1e3
                line["kernels"][name] = {"us": 1e6 * t, "gbs": b / t / 1e9, "frac_hbm": b / t / 1e9 / peaks["hbm_gbs"],
                                         "bytes": b}
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
