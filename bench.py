#!/usr/bin/env python
"""Benchmark of the activation-sparse decode path on B200.

Workload: Llama-3-8B-shaped decoder-layer projections at batch 1, bf16 weights
~ N(0, 0.02^2): q/k/v (4096 -> 4096/1024/1024, one fused [4096 x 6144] matrix),
o (4096 -> 4096), SwiGLU FFN d=4096, ffn=14336 (gate|up interleaved
[4096 x 28672], down [14336 x 4096]). Inputs are Laplace(0, 1); TEAL magnitude
thresholds are calibrated per block input (qkv-in, o-in, gate/up-in, down-in)
on 64 seeded draws for the target sparsity (down-in on the dense FFN's h).

One step = one batch-1 token through a stack of 32 such layers with distinct
weights (13.9 GB of bf16 weights, far larger than the 126 MB L2, so every
weight byte comes from HBM). Each layer runs three library calls: sparse GEMV
(qkv), sparse GEMV (o), sparse SwiGLU FFN (two kernels); the 32-layer step is
captured once in a CUDA graph and replayed.

Metric: effective HBM GB/s = algorithmic bytes (active weight rows x row bytes
+ activations in + outputs) / time, whole job (summed over ranks); also
us/layer. With --gpus N each rank runs an independent replica (no collective:
the path does not shard across GPUs here).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

OTHER_WORKLOADS = ("gemv", "phi2", "moe", "ffn70b")
METRIC = "sparse FFN µs/layer and effective HBM GB/s vs sparsity at batch 1–16"
D, FFN, NQKV = 4096, 14336, 6144
WORKLOAD = ("Llama-3-8B-shaped decoder layer at batch 1: q/k/v/o 4096->4096/1024/1024/4096, "
            "SwiGLU FFN d=4096 ffn=14336, bf16 weights ~N(0,0.02^2), Laplace inputs, per-block "
            "TEAL thresholds on all four block inputs")


# ---------------------------------------------------------------- helpers

def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(ms, dist=None, device=None):
    """The slowest rank's time: replicas finish when the last one does."""
    if dist is None:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_gbs(bytes_per_step, steps, world, ms):
    """Whole-job GB/s of `world` replicas that each ran `steps` steps, the slowest in `ms`."""
    return bytes_per_step * steps * world / (ms * 1e-3) / 1e9


class ClockSampler:
    """Samples SM clock, max clock and clock-event reasons with NVML in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML missing: report no clocks rather than fail
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = get_reasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


KERNEL_SOURCES = ("sparse_input_gemv_b200/csrc/sfx_gemv_kernel.cuh",
                  "sparse_input_gemv_b200/csrc/sfx_gemv.cu",
                  "sparse_input_gemv_b200/csrc/sfx_common.cuh")
PROFILE_SUMMARIES = {"ffn_gate_up": "profiles/sparse_gemv_gate_up_llama3_8b.md"}


def _code_only(src: str) -> str:
    """C/C++/CUDA source without comments and blank lines (string literals are
    kept; the sources hold no comment markers inside strings)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_source_hash() -> str:
    """Hash of the GEMV sources' code: a comment edit keeps it, a code edit changes it."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, sparsity: float):
    """DRAM traffic per launch from the committed ncu summary of `kernel`.

    The summary records `traffic_bytes_per_launch`, the `sparsity` it was
    taken at and `kernel_source_sha256_16` of the GEMV sources; the figure is
    used only while those sources are unchanged (else None).
    """
    path = PROFILE_SUMMARIES.get(kernel)
    if not path or not os.path.exists(os.path.join(ROOT, path)):
        return None, "no ncu summary for this kernel"
    fields = {}
    for line in open(os.path.join(ROOT, path)):
        if ":" in line and line.strip().startswith("- `"):
            k, v = line.strip()[3:].split("`", 1)[0], line.split(":", 1)[1].strip().strip("`")
            fields[k] = v
    try:
        if fields.get("kernel_source_sha256_16") != kernel_source_hash():
            return None, "kernel changed since the ncu capture"
        if abs(float(fields.get("sparsity", "nan")) - sparsity) > 1e-9:
            return None, "ncu capture taken at another sparsity"
        return int(fields["traffic_bytes_per_launch"]), f"ncu capture, {path}"
    except (KeyError, ValueError):
        return None, "ncu summary unreadable"


def time_graph(graph, reps, stream):
    """Device time of `reps` replays of a captured graph (CUDA events, ms)."""
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(reps):
        graph.replay()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


# ---------------------------------------------------------------- the model stack

class Stack:
    """L Llama-3-8B-shaped layers with sparse-decode buffers and thresholds."""

    def __init__(self, layers: int, dev, keep_layer0_fp64: bool):
        from sparse_input_gemv_b200 import binding as sb
        from sparse_input_gemv_b200 import synth
        self.sb, self.synth, self.L, self.dev = sb, synth, layers, dev
        bf = "bf16"
        self.Wqkv, self.Wo, self.Wgu, self.Wd = [], [], [], []
        self.layer0 = None
        for l in range(layers):
            key = ("llama3-8b", l)
            self.Wqkv.append(synth.normal((D, NQKV), synth.seed_of(*key, "Wqkv"), 0.02, bf, dev))
            self.Wo.append(synth.normal((D, D), synth.seed_of(*key, "Wo"), 0.02, bf, dev))
            Wg = synth.normal((D, FFN), synth.seed_of(*key, "Wg"), 0.02, bf, dev)
            Wu = synth.normal((D, FFN), synth.seed_of(*key, "Wu"), 0.02, bf, dev)
            self.Wgu.append(sb.sfx_pack_gate_up(Wg, Wu))
            self.Wd.append(synth.normal((FFN, D), synth.seed_of(*key, "Wd"), 0.02, bf, dev))
            if l == 0 and keep_layer0_fp64:
                self.layer0 = {k: v.to("cpu", torch.float64).numpy() for k, v in
                               (("Wqkv", self.Wqkv[0]), ("Wo", self.Wo[0]), ("Wg", Wg),
                                ("Wu", Wu), ("Wd", self.Wd[0]))}
            del Wg, Wu
        torch.cuda.synchronize()
        # calibration draws (64 per site) and evaluation inputs (draw 64 + layer)
        self.calib = {s: synth.calib_draws("llama3-8b", s, 64, D, bf).to(dev)
                      for s in ("qkv-in", "o-in", "ffn-in")}
        self.xq = synth.eval_draw("llama3-8b", "qkv-in", layers, D, bf).to(dev)
        self.xo = synth.eval_draw("llama3-8b", "o-in", layers, D, bf).to(dev)
        self.xf = synth.eval_draw("llama3-8b", "ffn-in", layers, D, bf).to(dev)
        self.yq = torch.empty((layers, NQKV), dtype=torch.bfloat16, device=dev)
        self.yo = torch.empty((layers, D), dtype=torch.bfloat16, device=dev)
        self.yf = torch.empty((layers, D), dtype=torch.bfloat16, device=dev)
        self.h = torch.empty((layers, FFN), dtype=torch.float32, device=dev)
        self.ws = sb.Workspace(dev)
        need = max(sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, 1, D, NQKV, sb.SFX_BF16),
                   sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, 1, D, 2 * FFN, sb.SFX_BF16),
                   sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, 1, FFN, D, sb.SFX_F32),
                   sb.sfx_workspace_bytes(sb.SFX_OP_FFN_SWIGLU, 16, D, FFN, sb.SFX_BF16),
                   sb.sfx_workspace_bytes(sb.SFX_OP_CALIBRATE, 64, FFN, 8, sb.SFX_F32))
        self.ws.reserve(need)
        # down-site calibration input: the dense FFN's h of layer 0 on the ffn-in draws
        hc = []
        for c0 in range(0, 64, 16):
            hc.append(sb.sfx_sparse_ffn_swiglu(self.calib["ffn-in"][c0:c0 + 16], self.Wgu[0],
                                               self.Wd[0], want_h=True, ws=self.ws)["h"])
        self.calib["down-in"] = torch.cat(hc).contiguous()

    def set_sparsity(self, p: float):
        sb = self.sb
        self.p = p
        self.t = {s: sb.sfx_calibrate_thresholds(self.calib[s], [p], ws=self.ws)[0]
                  for s in ("qkv-in", "o-in", "ffn-in", "down-in")}
        # active rows per layer and site (for the algorithmic byte count)
        xq, xo, xf = self.xq.float(), self.xo.float(), self.xf.float()
        self.act_q = (xq.abs() > self.t["qkv-in"]).sum(1).tolist()
        self.act_o = (xo.abs() > self.t["o-in"]).sum(1).tolist()
        self.act_f = (xf.abs() > self.t["ffn-in"]).sum(1).tolist()
        self.act_d = []
        for l in range(self.L):
            out = sb.sfx_sparse_ffn_swiglu(self.xf[l], self.Wgu[l], self.Wd[l], self.t["ffn-in"],
                                           self.t["down-in"], h=self.h[l:l + 1], y=self.yf[l:l + 1],
                                           want_bitmaps=True, ws=self.ws)
            bits = out["bitmap_h"].view(torch.uint8).cpu().numpy()
            self.act_d.append(int(np.unpackbits(bits).sum()))

    # one layer = three library calls (four kernels)
    def layer(self, l: int):
        sb, ws, t = self.sb, self.ws, self.t
        sb.sfx_sparse_gemv(self.xq[l], self.Wqkv[l], t=t["qkv-in"], y=self.yq[l:l + 1], ws=ws)
        sb.sfx_sparse_gemv(self.xo[l], self.Wo[l], t=t["o-in"], y=self.yo[l:l + 1], ws=ws)
        sb.sfx_sparse_ffn_swiglu(self.xf[l], self.Wgu[l], self.Wd[l], t["ffn-in"], t["down-in"],
                                 y=self.yf[l:l + 1], ws=ws)

    def step(self):
        for l in range(self.L):
            self.layer(l)

    # the four kernels of a layer on their own (same launch configuration)
    def kernel_fns(self):
        sb, ws, t = self.sb, self.ws, self.t
        return {
            "qkv_gemv": lambda l: sb.sfx_sparse_gemv(self.xq[l], self.Wqkv[l], t=t["qkv-in"],
                                                     y=self.yq[l:l + 1], ws=ws),
            "o_gemv": lambda l: sb.sfx_sparse_gemv(self.xo[l], self.Wo[l], t=t["o-in"],
                                                   y=self.yo[l:l + 1], ws=ws),
            "ffn_gate_up": lambda l: sb.sfx_sparse_gemv(self.xf[l], self.Wgu[l], t=t["ffn-in"],
                                                        flags=sb.SFX_FLAG_SWIGLU,
                                                        y=self.h[l:l + 1], ws=ws),
            "ffn_down": lambda l: sb.sfx_sparse_gemv(self.h[l], self.Wd[l], t=t["down-in"],
                                                     y=self.yf[l:l + 1], ws=ws),
        }

    def kernel_bytes(self, name: int, l: int) -> int:
        if name == "qkv_gemv":
            return self.act_q[l] * NQKV * 2 + D * 2 + NQKV * 2
        if name == "o_gemv":
            return self.act_o[l] * D * 2 + D * 2 + D * 2
        if name == "ffn_gate_up":
            return self.act_f[l] * 2 * FFN * 2 + D * 2 + FFN * 4
        if name == "ffn_down":
            return self.act_d[l] * D * 2 + FFN * 4 + D * 2
        raise KeyError(name)

    def step_bytes(self) -> int:
        return sum(self.kernel_bytes(k, l) for l in range(self.L)
                   for k in ("qkv_gemv", "o_gemv", "ffn_gate_up", "ffn_down"))

    def dense_step_bytes(self) -> int:
        return self.L * ((NQKV + D + 2 * FFN) * D * 2 + FFN * D * 2)


def dense_library_us_per_layer(stack, stream, reps=5):
    """Dense reference: the same layers through torch.matmul (cuBLAS) and torch
    elementwise ops (SiLU(g) * u in bf16), all rows read, µs per layer. A library
    yardstick only; it is not on the measured path."""
    L = stack.L
    dev = stack.Wqkv[0].device
    yq = torch.empty((1, NQKV), dtype=torch.bfloat16, device=dev)
    yo = torch.empty((1, D), dtype=torch.bfloat16, device=dev)
    gu = torch.empty((1, 2 * FFN), dtype=torch.bfloat16, device=dev)
    yf = torch.empty((1, D), dtype=torch.bfloat16, device=dev)

    def layers():
        for l in range(L):
            torch.mm(stack.xq[l:l + 1], stack.Wqkv[l], out=yq)
            torch.mm(stack.xo[l:l + 1], stack.Wo[l], out=yo)
            torch.mm(stack.xf[l:l + 1], stack.Wgu[l], out=gu)
            h = torch.nn.functional.silu(gu[:, 0::2]) * gu[:, 1::2]
            torch.mm(h, stack.Wd[l], out=yf)

    layers()
    torch.cuda.synchronize()
    g = capture(layers, stream)
    g.replay()
    ms = time_graph(g, reps, stream)
    del g
    return ms * 1e3 / (reps * L)


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def graph_us(fns, stream, reps=5):
    """Mean device time (us) of one call of `fns` (a list of callables replayed
    round-robin, one per weight copy) captured in a CUDA graph."""
    for f in fns:
        f()
    torch.cuda.synchronize()
    g = capture(lambda: [f() for f in fns], stream)
    g.replay()
    ms = time_graph(g, reps, stream)
    del g
    return ms * 1e3 / (reps * len(fns))


def copies_for(nbytes, floor=2):
    """Weight copies needed so that one pass over them is >= 3x the 126 MB L2."""
    return max(floor, math.ceil(400e6 / max(nbytes, 1)))


def bench_other_workloads(stream, dev, which=OTHER_WORKLOADS):
    """The other workloads of the path, short graph-timed runs (not the headline).

    `which` selects among "gemv" (single input-sparse GEMV), "phi2" (GeLU FFN with
    GxO top-k / GLASS), "moe" (128-expert MoE) and "ffn70b" (batch sweep).
    """
    from sparse_input_gemv_b200 import binding as sb
    from sparse_input_gemv_b200 import synth
    out = {}
    ws = sb.Workspace(dev)
    ws.reserve(256 << 20)

    if "gemv" in which:
        # single input-sparse GEMV: x fp16 [1 x 256], W fp16 [256 x 512], t_p for 50%
        calib = synth.calib_draws("single", "x", 64, 256, "f16").to(dev)
        t = sb.sfx_calibrate_thresholds(calib, [0.5], ws=ws)[0]
        n = copies_for(256 * 512 * 2, floor=2)
        Ws = [synth.normal((256, 512), synth.seed_of("single", "W", c), 0.02, "f16", dev) for c in range(n)]
        x = synth.eval_draw("single", "x", 1, 256, "f16").to(dev)
        y = torch.empty((1, 512), dtype=torch.float16, device=dev)
        us = graph_us([lambda W=W: sb.sfx_sparse_gemv(x, W, t=t, y=y, ws=ws) for W in Ws[:64]], stream)
        act = int((x.float().abs() > t).sum())
        out["single_gemv_fp16_256x512_p50"] = {
            "us": us, "active_rows": act, "gbs": (act * 1024 + 512 + 1024) / (us * 1e-6) / 1e9,
            "note": "latency-bound: 128 KB of active weights; 64 distinct weight copies per graph"}
        del Ws

    if "phi2" in which:
        # Phi-2-shaped GeLU FFN d=2560, ffn=10240, fp16: dense up + GeLU, top-k of |g h|
        # (or a static GLASS mask), sparse down
        d, f = 2560, 10240
        n = copies_for(2 * d * f * 2)
        W1 = [synth.normal((d, f), synth.seed_of("phi2", "W1", c), 0.02, "f16", dev) for c in range(n)]
        W2 = [synth.normal((f, d), synth.seed_of("phi2", "W2", c), 0.02, "f16", dev) for c in range(n)]
        x = synth.eval_draw("phi2", "x", 1, d, "f16").to(dev)
        g = synth.normal((1, f), synth.seed_of("phi2", "g"), 1.0, "f32", dev)
        sl = synth.abs_normal((1, f), synth.seed_of("phi2", "local"), device=dev)
        sgl = synth.abs_normal((1, f), synth.seed_of("phi2", "global"), device=dev)
        W1T = [w.t().contiguous() for w in W1]  # one row per neuron, for the static set
        h = torch.empty((1, f), dtype=torch.float32, device=dev)
        y = torch.empty((1, d), dtype=torch.float16, device=dev)
        bitmap = torch.zeros((1, (f + 31) // 32), dtype=torch.int32, device=dev)
        idx = torch.zeros((1, f), dtype=torch.int32, device=dev)
        cnt = torch.zeros((1,), dtype=torch.int32, device=dev)
        lib = sb.load()
        import ctypes
        P = lambda tns: ctypes.c_void_p(tns.data_ptr())

        def select_gxo(k, sel=sb.SFX_SEL_TOPK_GXO):
            lib.sfx_mask_compact(P(h), sb.SFX_F32, 1, f, sel, 0.0, k, P(g), None, 0.5,
                                 P(bitmap), P(idx), P(cnt), None, None, P(ws.buf), ws.buf.numel(),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        phi = {}
        for keep in (0.3, 0.5, 0.7):
            k = int(keep * f + 0.5)
            steps = []
            for c in range(n):
                def step(c=c, k=k):
                    sb.sfx_sparse_gemv(x, W1[c], flags=sb.SFX_FLAG_GELU, y=h, ws=ws)
                    select_gxo(k)
                    sb.sfx_sparse_gemv(h[0], W2[c], idx=idx[0], cnt=cnt, y=y[0], ws=ws)
                steps.append(step)
            us = graph_us(steps, stream)
            # the same step with the corrected GxO score (ATTR "correction term")
            csteps = []
            for c in range(n):
                def cstep(c=c, k=k):
                    sb.sfx_sparse_gemv(x, W1[c], flags=sb.SFX_FLAG_GELU, y=h, ws=ws)
                    select_gxo(k, sb.SFX_SEL_TOPK_CGXO)
                    sb.sfx_sparse_gemv(h[0], W2[c], idx=idx[0], cnt=cnt, y=y[0], ws=ws)
                csteps.append(cstep)
            us_c = graph_us(csteps, stream)
            nbytes = d * f * 2 + k * d * 2 + d * 2 + f * 4 * 3 + d * 2
            # GLASS: the mask is fixed after prefill, so a decode step is up + down only
            sb.sfx_mask_compact(None, sb.SFX_SEL_TOPK_GLASS, k=k, score_l=sl, score_g=sgl, lam=0.5, ws=ws)
            gl = sb.sfx_mask_compact(None, sb.SFX_SEL_TOPK_GLASS, k=k, score_l=sl, score_g=sgl, lam=0.5,
                                     ws=ws)
            us_gl = graph_us([lambda c=c: (sb.sfx_sparse_gemv(x, W1[c], flags=sb.SFX_FLAG_GELU, y=h, ws=ws),
                                           sb.sfx_sparse_gemv(h[0], W2[c], idx=gl["idx"][0],
                                                              cnt=gl["cnt"], y=y[0], ws=ws))
                              for c in range(n)], stream)
            # GLASS set on both projections: up rows and down rows of the kept neurons only
            us_both = graph_us([lambda c=c: sb.sfx_static_ffn(x, W1T[c], W2[c], gl["idx"][0],
                                                              gl["cnt"], y=y, ws=ws)
                                for c in range(n)], stream)
            bytes_both = 2 * k * d * 2 + 2 * d * 2
            phi[f"keep{int(keep * 100)}"] = {"us_gxo": us, "us_corrected_gxo": us_c,
                                             "us_glass_static_mask": us_gl,
                                             "us_glass_both_projections": us_both,
                                             "gbs_glass_both_projections":
                                                 bytes_both / (us_both * 1e-6) / 1e9,
                                             "gbs_gxo": nbytes / (us * 1e-6) / 1e9}
        out["phi2_gelu_ffn_fp16_topk"] = phi
        del W1, W2, W1T

    if "moe" in which:
        # MoE: 128 experts, d=2048, expert ffn=768, top-8, shared expert ffn=2048, bf16.
        # Four layers with their own weights (1.2 GB each) are replayed round-robin,
        # so a replay reads its active experts from HBM, not from the 126 MB L2.
        E, d, f, fs, top, L = 128, 2048, 768, 2048, 8, 4
        layers = []
        xc = synth.calib_draws("moe", "x", 16, d, "bf16").to(dev)
        zl = torch.zeros((16, E), dtype=torch.float32, device=dev)
        ninf = torch.full((E,), -math.inf, dtype=torch.float32, device=dev)
        for li in range(L):
            WgT = synth.normal((E, f, d), synth.seed_of("moe", "WgT", li), 0.02, "bf16", dev)
            WuT = synth.normal((E, f, d), synth.seed_of("moe", "WuT", li), 0.02, "bf16", dev)
            Wd = synth.normal((E, f, d), synth.seed_of("moe", "Wd", li), 0.02, "bf16", dev)
            SgT = synth.normal((fs, d), synth.seed_of("moe", "SgT", li), 0.02, "bf16", dev)
            SuT = synth.normal((fs, d), synth.seed_of("moe", "SuT", li), 0.02, "bf16", dev)
            Sd = synth.normal((fs, d), synth.seed_of("moe", "Sd", li), 0.02, "bf16", dev)
            # per-expert gate activations of 16 calibration tokens routed to every expert
            a_all = sb.sfx_moe_expert_sparse(xc, zl, WgT, WuT, Wd, ninf, E, want_a=True, ws=ws)["a"]
            a_e = a_all.permute(1, 0, 2).contiguous()  # [E x 16 x ffn], experts in index order
            te = {p: torch.tensor([sb.sfx_calibrate_thresholds(a_e[e], [p], ws=ws)[0]
                                   for e in range(E)], dtype=torch.float32, device=dev)
                  for p in (0.5, 0.8, 0.9)}
            layers.append((WgT, WuT, Wd, SgT, SuT, Sd, te))
            del a_all, a_e
        moe = {}
        for p in (0.5, 0.8, 0.9):
            for B in (1, 4, 16):
                xb = synth.eval_draw("moe", "x", B, d, "bf16").to(dev)
                lgs = [synth.normal((B, E), synth.seed_of("moe", "logits", B, li), 1.0, "f32", dev)
                       for li in range(L)]
                yb = torch.empty((B, d), dtype=torch.bfloat16, device=dev)
                nbytes, n_exp, kept_all = 0, 0, 0
                for li, (WgT, WuT, Wd, SgT, SuT, Sd, te) in enumerate(layers):
                    r = sb.sfx_moe_expert_sparse(xb, lgs[li], WgT, WuT, Wd, te[p], top, Ws_gT=SgT,
                                                 Ws_upT=SuT, Ws_d=Sd, y=yb, want_a=True, ws=ws)
                    sel = r["sel"].cpu().numpy()
                    a = r["a"]
                    experts = sorted({int(e) for e in sel.ravel()})
                    # bytes: dense gate rows of every active expert, kept up/down rows
                    # (union over the expert's tokens), shared expert, activations
                    kept = 0
                    for e in experts:
                        mask = torch.zeros(f, dtype=torch.bool, device=dev)
                        for t_ in range(B):
                            for k_ in range(top):
                                if sel[t_, k_] == e:
                                    mask |= a[t_, k_].abs() > te[p][e]
                        kept += int(mask.sum())
                    nbytes += len(experts) * f * d * 2 + kept * 2 * d * 2 + 3 * d * fs * 2 + 2 * B * d * 2
                    n_exp += len(experts)
                    kept_all += kept
                us = graph_us([lambda li=li, l=l: sb.sfx_moe_expert_sparse(
                    xb, lgs[li], l[0], l[1], l[2], l[6][p], top, Ws_gT=l[3], Ws_upT=l[4], Ws_d=l[5],
                    y=yb, ws=ws) for li, l in enumerate(layers)], stream, reps=20)
                moe[f"p{int(p * 100)}_b{B}"] = {"us": us, "gbs": nbytes / L / (us * 1e-6) / 1e9,
                                                "active_experts": n_exp / L,
                                                "kept_frac": kept_all / (n_exp * f)}
        out["moe_128x768_top8_shared2048"] = {"results": moe,
                                              "note": "us per MoE layer; 4 layers with distinct "
                                                      "weights replayed round-robin (HBM-resident)"}
        del layers

    if "ffn70b" in which:
        # Llama-3-70B-shaped SwiGLU FFN d=8192, ffn=28672 bf16, batch 1/4/8/16,
        # per-batch union of magnitude masks, sparsity 0..0.9
        d, f = 8192, 28672
        n = 2
        Wgu = []
        Wdn = []
        for c in range(n):
            Wg = synth.normal((d, f), synth.seed_of("l70", "Wg", c), 0.02, "bf16", dev)
            Wu = synth.normal((d, f), synth.seed_of("l70", "Wu", c), 0.02, "bf16", dev)
            Wgu.append(sb.sfx_pack_gate_up(Wg, Wu))
            del Wg, Wu
            Wdn.append(synth.normal((f, d), synth.seed_of("l70", "Wd", c), 0.02, "bf16", dev))
        calib = synth.calib_draws("l70", "x", 64, d, "bf16").to(dev)
        hc = torch.cat([sb.sfx_sparse_ffn_swiglu(calib[i:i + 16], Wgu[0], Wdn[0], want_h=True, ws=ws)["h"]
                        for i in range(0, 64, 16)]).contiguous()
        sweep = []
        for B in (1, 4, 8, 16):
            xb = synth.eval_draw("l70", "x", B, d, "bf16").to(dev)
            yb = torch.empty((B, d), dtype=torch.bfloat16, device=dev)
            hb = torch.empty((B, f), dtype=torch.float32, device=dev)
            for p in [i / 10 for i in range(10)]:
                t_in = sb.sfx_calibrate_thresholds(calib, [p], ws=ws)[0]
                t_h = sb.sfx_calibrate_thresholds(hc, [p], ws=ws)[0]
                r = sb.sfx_sparse_ffn_swiglu(xb, Wgu[0], Wdn[0], t_in, t_h, h=hb, y=yb,
                                             want_bitmaps=True, ws=ws)
                ux = int(np.unpackbits(r["bitmap_x"].view(torch.uint8).cpu().numpy().reshape(B, -1),
                                       axis=1).any(0).sum())
                uh = int(np.unpackbits(r["bitmap_h"].view(torch.uint8).cpu().numpy().reshape(B, -1),
                                       axis=1).any(0).sum())
                nbytes = ux * 2 * f * 2 + uh * d * 2 + B * (d * 2 * 2 + f * 4 * 2)
                us = graph_us([lambda c=c: sb.sfx_sparse_ffn_swiglu(xb, Wgu[c], Wdn[c], t_in, t_h, h=hb,
                                                                    y=yb, ws=ws) for c in range(n)],
                              stream, reps=3)
                sweep.append({"batch": B, "sparsity": p, "us": us, "gbs": nbytes / (us * 1e-6) / 1e9,
                              "union_frac_in": ux / d, "union_frac_h": uh / f})
        # the same layer on correlated tokens (shared per-neuron scales; masks of
        # different tokens overlap with pairwise Jaccard ~0.56 at p = 0.5)
        ccal = synth.correlated_draws("l70c", "x", 64, d, "bf16", draw=0).to(dev)
        chc = torch.cat([sb.sfx_sparse_ffn_swiglu(ccal[i:i + 16], Wgu[0], Wdn[0], want_h=True,
                                                  ws=ws)["h"] for i in range(0, 64, 16)]).contiguous()
        csweep = []
        for B in (4, 8, 16):
            xb = synth.correlated_draws("l70c", "x", B, d, "bf16").to(dev)
            yb = torch.empty((B, d), dtype=torch.bfloat16, device=dev)
            hb = torch.empty((B, f), dtype=torch.float32, device=dev)
            for p in (0.5, 0.7, 0.9):
                t_in = sb.sfx_calibrate_thresholds(ccal, [p], ws=ws)[0]
                t_h = sb.sfx_calibrate_thresholds(chc, [p], ws=ws)[0]
                r = sb.sfx_sparse_ffn_swiglu(xb, Wgu[0], Wdn[0], t_in, t_h, h=hb, y=yb,
                                             want_bitmaps=True, ws=ws)
                ux = int(np.unpackbits(r["bitmap_x"].view(torch.uint8).cpu().numpy().reshape(B, -1),
                                       axis=1).any(0).sum())
                uh = int(np.unpackbits(r["bitmap_h"].view(torch.uint8).cpu().numpy().reshape(B, -1),
                                       axis=1).any(0).sum())
                nbytes = ux * 2 * f * 2 + uh * d * 2 + B * (d * 2 * 2 + f * 4 * 2)
                us = graph_us([lambda c=c: sb.sfx_sparse_ffn_swiglu(xb, Wgu[c], Wdn[c], t_in, t_h, h=hb,
                                                                    y=yb, ws=ws) for c in range(n)],
                              stream, reps=3)
                csweep.append({"batch": B, "sparsity": p, "us": us, "gbs": nbytes / (us * 1e-6) / 1e9,
                               "union_frac_in": ux / d, "union_frac_h": uh / f})
        out["llama3_70b_ffn_bf16_correlated_tokens"] = {
            "sweep": csweep,
            "note": "x_bi = exp(1.5 n_i) z_bi (shared per-neuron scales); pairwise mask Jaccard "
                    "~0.56 at p = 0.5"}
        # dense library reference: torch.matmul (cuBLAS) for both projections and
        # torch ops for SiLU(g) * u, every row read
        lib = []
        for B in (1, 4, 8, 16):
            xb = synth.eval_draw("l70", "x", B, d, "bf16").to(dev)
            gu = torch.empty((B, 2 * f), dtype=torch.bfloat16, device=dev)
            yb = torch.empty((B, d), dtype=torch.bfloat16, device=dev)

            def dense(c, xb=xb, gu=gu, yb=yb):
                torch.mm(xb, Wgu[c], out=gu)
                torch.mm(torch.nn.functional.silu(gu[:, 0::2]) * gu[:, 1::2], Wdn[c], out=yb)

            us = graph_us([lambda c=c: dense(c) for c in range(n)], stream, reps=3)
            lib.append({"batch": B, "us": us, "gbs": 3 * d * f * 2 / (us * 1e-6) / 1e9})
        out["llama3_70b_ffn_bf16"] = {"sweep": sweep, "dense_bytes": 3 * d * f * 2,
                                      "dense_library": lib,
                                      "note": "2 weight copies (2.8 GB) alternate between calls; "
                                              "dense_library = torch.matmul (cuBLAS) reference"}
    return out


# ---------------------------------------------------------------- CPU oracle leg

def oracle_layer_pass(W, x, t):
    """One layer (qkv, o, SwiGLU FFN) of the fp64 oracle as it stands."""
    import oracle as O
    O.masked_gemv(x["qkv-in"], O.magnitude_mask(x["qkv-in"], t["qkv-in"]), W["Wqkv"])
    O.masked_gemv(x["o-in"], O.magnitude_mask(x["o-in"], t["o-in"]), W["Wo"])
    O.ffn_swiglu(x["ffn-in"], t["ffn-in"], W["Wg"], W["Wu"], W["Wd"], t["down-in"])


def oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def eval_inputs_fp64():
    from sparse_input_gemv_b200 import synth
    return {s: synth.eval_draw("llama3-8b", s, 1, D, "bf16").double().numpy()
            for s in ("qkv-in", "o-in", "ffn-in")}


def layer_bytes_fp64(W, x, t, frac=1.0):
    """Algorithmic bytes of one layer (bf16 weights), same accounting as the GPU arm."""
    import oracle as O
    nq, no_, nf = W["Wqkv"].shape[1], W["Wo"].shape[1], W["Wg"].shape[1]
    _, h, mx, mh = O.ffn_swiglu(x["ffn-in"], t["ffn-in"], W["Wg"], W["Wu"], W["Wd"], t["down-in"])
    aq = int((np.abs(x["qkv-in"]) > t["qkv-in"]).sum())
    ao = int((np.abs(x["o-in"]) > t["o-in"]).sum())
    return (aq * nq * 2 + D * 2 + nq * 2 + ao * no_ * 2 + D * 2 + no_ * 2
            + int(mx.sum()) * 2 * nf * 2 + D * 2 + nf * 4 + int(mh.sum()) * D * 2 + nf * 4 + D * 2)


def oracle_layer0():
    """fp64 host copies of layer 0's weights, drawn exactly as the GPU stack draws them."""
    from sparse_input_gemv_b200 import synth
    dev = torch.device("cuda")
    key = ("llama3-8b", 0)
    out = {}
    for name, shape in (("Wqkv", (D, NQKV)), ("Wo", (D, D)), ("Wg", (D, FFN)), ("Wu", (D, FFN)),
                        ("Wd", (FFN, D))):
        out[name] = synth.normal(shape, synth.seed_of(*key, name), 0.02, "bf16",
                                 dev).to("cpu", torch.float64).numpy()
    return out


def reference_arm(args):
    """The oracle, as it stands, timed on the host cores on this workload.

    Thresholds come from the oracle's own calibration (down-in on its dense
    FFN h over the 64 calibration draws). One step is one layer pass; if the
    requested steps would take more than about 150 s, every weight matrix is
    cut to its first columns (the same fraction for all) so the run stays
    within a few minutes, and the bytes are counted on that sample.
    """
    import oracle as O
    from sparse_input_gemv_b200 import synth
    p = args.sparsity
    W = oracle_layer0()
    t = {s: O.calibrate_threshold(synth.calib_draws("llama3-8b", s, 64, D, "bf16")
                                  .double().numpy(), p) for s in ("qkv-in", "o-in", "ffn-in")}
    cf = synth.calib_draws("llama3-8b", "ffn-in", 64, D, "bf16").double().numpy()
    _, hc, _, _ = O.ffn_swiglu(cf, -math.inf, W["Wg"], W["Wu"], W["Wd"], -math.inf)
    t["down-in"] = O.calibrate_threshold(hc, p)
    x = eval_inputs_fp64()
    t0 = time.perf_counter()
    oracle_layer_pass(W, x, t)
    t_full = time.perf_counter() - t0
    frac = min(1.0, 150.0 / max(t_full * (args.steps + args.warmup), 1e-9))
    if frac < 1.0:
        cut = lambda n: max(8, int(n * frac) // 8 * 8)
        W = {"Wqkv": np.ascontiguousarray(W["Wqkv"][:, :cut(NQKV)]),
             "Wo": np.ascontiguousarray(W["Wo"][:, :cut(D)]),
             "Wg": np.ascontiguousarray(W["Wg"][:, :cut(FFN)]),
             "Wu": np.ascontiguousarray(W["Wu"][:, :cut(FFN)]),
             "Wd": np.ascontiguousarray(W["Wd"][:cut(FFN), :])}
    for _ in range(args.warmup):
        oracle_layer_pass(W, x, t)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_layer_pass(W, x, t)
    el = time.perf_counter() - t0
    nbytes = layer_bytes_fp64(W, x, t)
    gbs = nbytes * args.steps / el / 1e9
    cores = oracle_cores()
    sample = ("one layer pass (qkv, o, SwiGLU FFN) of the fp64 numpy oracle per step on layer 0"
              + (f", weights cut to the first {frac:.3f} of their columns" if frac < 1 else ""))
    return {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / max(args.steps, 1) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1, "sparsity": p, "layers_per_step": 1,
                   "parallelism": "host cores"},
        "us_per_layer": el / max(args.steps, 1) * 1e6 / max(frac, 1e-9),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sfx", "reference"], default="sfx")
    ap.add_argument("--sparsity", type=float, default=0.5)
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--sweep", default="0,0.25,0.4,0.5,0.65,0.9",
                    help="comma list of sparsities for the sweep ('' to skip)")
    ap.add_argument("--sweep-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-other", action="store_true",
                    help="skip the other workloads (single GEMV, Phi-2, MoE, Llama-3-70B FFN)")
    ap.add_argument("--other", default=",".join(OTHER_WORKLOADS),
                    help="comma list of the other workloads to run: " + ", ".join(OTHER_WORKLOADS))
    args = ap.parse_args()

    rank, local_rank, world = env_rank()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return

    from sparse_input_gemv_b200 import binding as sb
    sb.load()
    stack = Stack(args.layers, dev, keep_layer0_fp64=(rank == 0 and not args.no_cpu))
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)

    def measure(p, steps, warmup, clocks=False, e2e=False):
        stack.set_sparsity(p)
        for _ in range(max(warmup, 1)):
            stack.step()
        torch.cuda.synchronize()
        g = capture(stack.step, stream)
        for _ in range(2):
            g.replay()
        res = {"p": p, "t": dict(stack.t)}
        sampler = ClockSampler(local_rank) if clocks else None
        if sampler:
            sampler.__enter__()
            t_soak = time.perf_counter()
            while time.perf_counter() - t_soak < 1.0:  # clock soak before the timed region
                g.replay()
                torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        ms = time_graph(g, steps, stream)
        torch.cuda.synchronize()
        if sampler:
            sampler.__exit__()
            res["clocks"] = sampler.summary()
        res["ms"] = max_over_ranks(ms, dist, dev)
        res["bytes_step"] = stack.step_bytes()
        res["graph"] = g
        if e2e:
            # same step through host buffers: H2D of the step's inputs, D2H of its outputs
            xs = [stack.xq, stack.xo, stack.xf]
            ys = [stack.yq, stack.yo, stack.yf]
            hx = [x.cpu().pin_memory() for x in xs]
            hy = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for y in ys]
            start = torch.cuda.Event(enable_timing=True)
            end = torch.cuda.Event(enable_timing=True)
            if dist is not None:
                dist.barrier()
            torch.cuda.synchronize()
            start.record(stream)
            for _ in range(steps):
                for d_, h_ in zip(xs, hx):
                    d_.copy_(h_, non_blocking=True)
                g.replay()
                for h_, d_ in zip(hy, ys):
                    h_.copy_(d_, non_blocking=True)
            end.record(stream)
            end.synchronize()
            ems = start.elapsed_time(end)
            res["e2e_ms"] = max_over_ranks(ems, dist, dev)
            res["h2d"] = sum(x.numel() * x.element_size() for x in xs)
            res["d2h"] = sum(y.numel() * y.element_size() for y in ys)
        return res

    # headline
    main_res = measure(args.sparsity, args.steps, args.warmup, clocks=True, e2e=True)
    ms = main_res["ms"]
    K = args.steps
    bytes_step = main_res["bytes_step"]
    value = replica_gbs(bytes_step, K, world, ms)
    us_layer = ms * 1e3 / (K * args.layers)

    # per-kernel device times: each kernel alone, replayed over the 32 layers
    kernels = {}
    fns = stack.kernel_fns()
    reps = max(3, min(20, args.steps))
    for name, fn in fns.items():
        for l in range(args.layers):
            fn(l)
        torch.cuda.synchronize()
        g = capture(lambda: [fn(l) for l in range(args.layers)], stream)
        g.replay()
        kms = time_graph(g, reps, stream)
        avg_us = kms * 1e3 / (reps * args.layers)
        kb = sum(stack.kernel_bytes(name, l) for l in range(args.layers)) / args.layers
        kernels[name] = {"us": avg_us, "bytes": kb, "gbs": kb / (avg_us * 1e-6) / 1e9}
        del g
    ffn_us = kernels["ffn_gate_up"]["us"] + kernels["ffn_down"]["us"]
    dense_lib_us = dense_library_us_per_layer(stack, stream)

    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    peak = peaks.get("hbm_gbs")
    peak_src = "measured" if peak else "fallback"
    peak = peak or 6650.0
    dom = max(kernels, key=lambda k: kernels[k]["us"])
    roofline = {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["gbs"], "peak": peak,
                "unit": "GB/s", "frac": kernels[dom]["gbs"] / peak, "peak_source": peak_src,
                "traffic": None}
    roofline["traffic"], roofline["traffic_note"] = profiled_traffic(dom, args.sparsity)

    # sweep over sparsity (shorter runs, graph replay only)
    sweep = []
    dense_us = None
    if args.sweep:
        for p in [float(v) for v in args.sweep.split(",") if v.strip() != ""]:
            r = measure(p, args.sweep_steps, 2)
            us = r["ms"] * 1e3 / (args.sweep_steps * args.layers)
            sweep.append({"sparsity": p, "us_per_layer": us,
                          "gbs": r["bytes_step"] * args.sweep_steps / (r["ms"] * 1e-3) / 1e9,
                          "active_bytes_per_layer": r["bytes_step"] / args.layers})
            if p == 0:
                dense_us = us
            del r["graph"]
        stack.set_sparsity(args.sparsity)

    # CPU oracle baseline on rank 0 (bounded sample of about cpu_seconds)
    cpu = None
    if rank == 0 and not args.no_cpu and stack.layer0 is not None:
        t = dict(stack.t)
        x = eval_inputs_fp64()
        reps_o, t0 = 0, time.perf_counter()
        while reps_o == 0 or time.perf_counter() - t0 < args.cpu_seconds:
            oracle_layer_pass(stack.layer0, x, t)
            reps_o += 1
        el = time.perf_counter() - t0
        nbytes = layer_bytes_fp64(stack.layer0, x, t)
        cpu = {"value": nbytes * reps_o / el / 1e9, "unit": "GB/s", "cores": oracle_cores(),
               "kind": "oracle", "us_per_layer": el / reps_o * 1e6,
               "sample": f"{reps_o} passes of one layer (qkv, o, SwiGLU FFN) of the fp64 numpy "
                         f"oracle on layer 0 in {el:.1f} s"}

    other = None
    if rank == 0 and not args.no_other:
        other = bench_other_workloads(stream, dev, tuple(w for w in args.other.split(",") if w))

    e2e_val = replica_gbs(bytes_step, K, world, main_res["e2e_ms"])
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1, "sparsity": args.sparsity,
                   "layers_per_step": args.layers,
                   "l2": f"inputs larger than L2: {args.layers} distinct layers, "
                         f"{stack.dense_step_bytes() / 1e9:.1f} GB of weights per step",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "us_per_layer": us_layer, "us_per_layer_ffn": ffn_us,
        "dense_us_per_layer": dense_us,
        "speedup_vs_dense": (dense_us / us_layer) if dense_us else None,
        "dense_library_us_per_layer": dense_lib_us,
        "speedup_vs_dense_library": dense_lib_us / us_layer,
        "thresholds": main_res["t"],
        "kernels": kernels, "roofline": roofline, "sweep": sweep,
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": main_res["h2d"],
                "d2h_bytes_per_step": main_res["d2h"], "ms_per_step": main_res["e2e_ms"] / K,
                "path": "CUDA graph of the public entry points + pinned host copies"},
        "gpu_launches": 4 * args.layers * K,
        "clocks": main_res.get("clocks"),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if other is not None:
        line["other_workloads"] = other
    del main_res["graph"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
