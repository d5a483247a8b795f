#!/usr/bin/env python
"""Benchmark of the activation-sparse decode path on B200.

Headline workload: a Llama-3-70B-shaped SwiGLU FFN layer, d = 8192,
ffn = 28672, bf16 weights ~ N(0, 0.02^2) (1.41 GB dense per layer), at batch 1
with TEAL magnitude thresholds on its two block inputs (gate/up-in and
down-in) calibrated for p = 0.5 on 64 seeded Laplace(0, 1) draws (down-in on
the dense FFN's h of those draws).

One step = one token through a stack of 8 such layers with distinct weights
(11.3 GB, far larger than the 126 MB L2, so every weight byte comes from HBM);
each layer is one sfx_sparse_ffn_swiglu call (two kernels), and the step is
captured once in a CUDA graph and replayed.

Metric: effective HBM GB/s = algorithmic bytes (active weight rows x row bytes
+ activations in and out, h written and read) / time, whole job (summed over
ranks), and µs per layer. The line also carries the metric's sweep (batch 1,
4, 8, 16 x sparsity 0-0.9 on the same layer, iid and correlated tokens), the
per-kernel roofline, the cuBLAS dense reference, the fp64 oracle timed on the
host cores, the mask flips of the GPU path against the oracle, and the other
workloads of the path (Llama-3-8B decoder layer, single GEMV, Phi-2 top-k
FFN, 128-expert MoE) as secondary keys. With --gpus N each rank runs an
independent replica (no collective: the path does not shard across GPUs).
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

OTHER_WORKLOADS = ("llama8b", "gemv", "phi2", "moe")
METRIC = "sparse FFN µs/layer and effective HBM GB/s vs sparsity at batch 1–16"
D70, F70 = 8192, 28672
WORKLOAD = ("Llama-3-70B-shaped SwiGLU FFN layer d=8192 ffn=28672, bf16 weights ~N(0,0.02^2) "
            "(1.41 GB dense), batch 1, Laplace(0,1) inputs, TEAL thresholds on the gate/up and "
            "down inputs")
D, FFN, NQKV = 4096, 14336, 6144
WORKLOAD_8B = ("Llama-3-8B-shaped decoder layer at batch 1: q/k/v/o 4096->4096/1024/1024/4096, "
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
PROFILE_SUMMARIES = {"ffn_gate_up": "profiles/sparse_gemv_gate_up_llama3_70b_p50.md"}


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

    SITES = ("qkv-in", "o-in", "ffn-in", "down-in")

    def set_sparsity(self, p):
        """One sparsity for every site, or a dict {site: p} (a per-site allocation)."""
        sb = self.sb
        self.p = p
        ps = p if isinstance(p, dict) else {s: p for s in self.SITES}
        self.t = {s: sb.sfx_calibrate_thresholds(self.calib[s], [ps[s]], ws=self.ws)[0]
                  for s in self.SITES}
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
    GxO top-k / GLASS) and "moe" (128-expert MoE).
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

        def select_gxo(k, sel=sb.SFX_SEL_TOPK_GXO, with_idx=False):
            lib.sfx_mask_compact(P(h), sb.SFX_F32, 1, f, sel, 0.0, k, P(g), None, 0.5,
                                 P(bitmap), P(idx) if with_idx else None, P(cnt), None, None,
                                 P(ws.buf), ws.buf.numel(),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))

        def gxo_steps(k, sel, with_idx):
            # up GEMV (GeLU) -> top-k select -> down GEMV on the select's bitmap
            # (or on its ascending index list)
            steps = []
            for c in range(n):
                def step(c=c):
                    sb.sfx_sparse_gemv(x, W1[c], flags=sb.SFX_FLAG_GELU, y=h, ws=ws)
                    select_gxo(k, sel, with_idx)
                    if with_idx:
                        sb.sfx_sparse_gemv(h[0], W2[c], idx=idx[0], cnt=cnt, y=y[0], ws=ws)
                    else:
                        sb.sfx_sparse_gemv_mask(h[0], W2[c], bitmap[0], y=y[0], ws=ws)
                steps.append(step)
            return steps
        phi = {}
        for keep in (0.3, 0.5, 0.7):
            k = int(keep * f + 0.5)
            us = graph_us(gxo_steps(k, sb.SFX_SEL_TOPK_GXO, False), stream)
            us_idx = graph_us(gxo_steps(k, sb.SFX_SEL_TOPK_GXO, True), stream)
            # the same step with the corrected GxO score (ATTR "correction term")
            us_c = graph_us(gxo_steps(k, sb.SFX_SEL_TOPK_CGXO, False), stream)
            nbytes = d * f * 2 + k * d * 2 + d * 2 + f * 4 * 3 + d * 2
            # GLASS: the mask is fixed after prefill, so a decode step is up + down only
            sb.sfx_mask_compact(None, sb.SFX_SEL_TOPK_GLASS, k=k, score_l=sl, score_g=sgl, lam=0.5, ws=ws)
            gl = sb.sfx_mask_compact(None, sb.SFX_SEL_TOPK_GLASS, k=k, score_l=sl, score_g=sgl, lam=0.5,
                                     ws=ws)
            us_gl = graph_us([lambda c=c: (sb.sfx_sparse_gemv(x, W1[c], flags=sb.SFX_FLAG_GELU, y=h, ws=ws),
                                           sb.sfx_sparse_gemv_mask(h[0], W2[c], gl["bitmap"][0],
                                                                   y=y[0], ws=ws))
                              for c in range(n)], stream)
            # GLASS set on both projections: up rows and down rows of the kept neurons only
            us_both = graph_us([lambda c=c: sb.sfx_static_ffn(x, W1T[c], W2[c], gl["idx"][0],
                                                              gl["cnt"], y=y, ws=ws)
                                for c in range(n)], stream)
            bytes_both = 2 * k * d * 2 + 2 * d * 2
            phi[f"keep{int(keep * 100)}"] = {"us_gxo": us, "us_corrected_gxo": us_c,
                                             "us_gxo_index_list": us_idx,
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

    return out


# ---------------------------------------------------------------- the headline: Llama-3-70B FFN

def ffn_bytes(ux: int, uh: int, B: int, d: int = D70, f: int = F70) -> int:
    """Algorithmic bytes of one SwiGLU FFN call with `ux` gate/up rows and `uh`
    down rows read (the batch union): bf16 rows of 4 f and 2 d bytes, x in,
    y out (bf16), h written and read once (fp32)."""
    return ux * 4 * f + uh * 2 * d + B * (2 * d * 2 + 2 * f * 4)


def union_counts(bitmap: torch.Tensor, B: int, n: int) -> int:
    """Rows of the batch union in a [B x words] int32 bitmap of n columns."""
    bits = np.unpackbits(bitmap.view(torch.uint8).cpu().numpy().reshape(B, -1), axis=1,
                         bitorder="little")[:, :n]
    return int(bits.any(0).sum())


class Ffn70Stack:
    """L Llama-3-70B-shaped SwiGLU FFN layers with distinct bf16 weights."""

    def __init__(self, layers: int, dev, table=None):
        from sparse_input_gemv_b200 import binding as sb
        from sparse_input_gemv_b200 import synth
        from sparse_input_gemv_b200.thresholds import ThresholdTable
        self.sb, self.synth, self.L, self.dev = sb, synth, layers, dev
        self.table = table if table is not None else ThresholdTable()
        self.Wgu, self.Wd = [], []
        for l in range(layers):
            Wg = synth.normal((D70, F70), synth.seed_of("l70", "Wg", l), 0.02, "bf16", dev)
            Wu = synth.normal((D70, F70), synth.seed_of("l70", "Wu", l), 0.02, "bf16", dev)
            self.Wgu.append(sb.sfx_pack_gate_up(Wg, Wu))
            del Wg, Wu
            self.Wd.append(synth.normal((F70, D70), synth.seed_of("l70", "Wd", l), 0.02, "bf16", dev))
        torch.cuda.synchronize()
        self.ws = sb.Workspace(dev)
        self.ws.reserve(max(sb.sfx_workspace_bytes(sb.SFX_OP_FFN_SWIGLU, 16, D70, F70),
                            sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, 16, D70, 2 * F70, sb.SFX_BF16),
                            sb.sfx_workspace_bytes(sb.SFX_OP_SPARSE_GEMV, 16, F70, D70, sb.SFX_F32),
                            sb.sfx_workspace_bytes(sb.SFX_OP_CALIBRATE, 64, F70, 8, sb.SFX_F32)))
        self.calib = {}
        self.hcal = {}
        for kind in ("iid", "corr"):
            self.calib[kind] = self.draws(kind, 64, draw=0)
            hs = [sb.sfx_sparse_ffn_swiglu(self.calib[kind][i:i + 16], self.Wgu[0], self.Wd[0],
                                           want_h=True, ws=self.ws)["h"] for i in range(0, 64, 16)]
            self.hcal[kind] = torch.cat(hs).contiguous()

    def draws(self, kind, B, draw=64):
        s = self.synth
        if kind == "iid":
            return s.eval_draw("l70", "x", B, D70, "bf16", draw=draw).to(self.dev)
        return s.correlated_draws("l70c", "x", B, D70, "bf16", draw=draw).to(self.dev)

    def thresholds(self, p, kind="iid"):
        """(t_in, t_h) for sparsity p, from the threshold table (calibrated on a miss)."""
        seed = "draws 0-63"
        return (self.table.calibrate(f"l70-{kind}", "gate_up-in", self.calib[kind], [p], seed,
                                     ws=self.ws)[0],
                self.table.calibrate(f"l70-{kind}", "down-in", self.hcal[kind], [p], seed,
                                     ws=self.ws)[0])

    def call(self, l, x, t_in, t_h, y, h=None):
        return self.sb.sfx_sparse_ffn_swiglu(x, self.Wgu[l], self.Wd[l], t_in, t_h, y=y, h=h,
                                             ws=self.ws)

    def active_bytes(self, l, x, t_in, t_h):
        """(bytes, union rows in, union rows h) of one call, from the fused bitmaps."""
        B = x.shape[0]
        r = self.sb.sfx_sparse_ffn_swiglu(x, self.Wgu[l], self.Wd[l], t_in, t_h,
                                          want_bitmaps=True, ws=self.ws)
        ux = union_counts(r["bitmap_x"], B, D70)
        uh = union_counts(r["bitmap_h"], B, F70)
        return ffn_bytes(ux, uh, B), ux, uh


def sweep_70b(stack, stream, batches=(1, 4, 8, 16), ps=None, kind="iid", reps=3):
    """µs per FFN call over batch x sparsity, the layers replayed round-robin."""
    ps = ps if ps is not None else [i / 10 for i in range(10)]
    rows = []
    for B in batches:
        xs = [stack.draws(kind, B, draw=64 + 16 * l) for l in range(stack.L)]
        y = torch.empty((B, D70), dtype=torch.bfloat16, device=stack.dev)
        for p in ps:
            t_in, t_h = stack.thresholds(p, kind)
            nb, ux, uh = stack.active_bytes(0, xs[0], t_in, t_h)
            us = graph_us([lambda l=l: stack.call(l, xs[l], t_in, t_h, y) for l in range(stack.L)],
                          stream, reps=reps)
            rows.append({"batch": B, "sparsity": p, "us": round(us, 2), "bytes": nb,
                         "gbs": round(nb / (us * 1e-6) / 1e9, 1),
                         "union_in": round(ux / D70, 4), "union_h": round(uh / F70, 4)})
    return rows


def dense_library_70b(stack, stream, batches=(1, 4, 8, 16), reps=3):
    """torch.matmul (cuBLAS) for both projections and torch SiLU * mul, every row
    read: the dense library yardstick, not on the measured path."""
    out = []
    for B in batches:
        x = stack.draws("iid", B)
        gu = torch.empty((B, 2 * F70), dtype=torch.bfloat16, device=stack.dev)
        y = torch.empty((B, D70), dtype=torch.bfloat16, device=stack.dev)

        def dense(l):
            torch.mm(x, stack.Wgu[l], out=gu)
            torch.mm(torch.nn.functional.silu(gu[:, 0::2]) * gu[:, 1::2], stack.Wd[l], out=y)

        us = graph_us([lambda l=l: dense(l) for l in range(stack.L)], stream, reps=reps)
        out.append({"batch": B, "us": round(us, 2),
                    "gbs": round(3 * D70 * F70 * 2 / (us * 1e-6) / 1e9, 1)})
    return out


def stage_kernels_70b(stack, stream, t_in, t_h, reps=10):
    """Each of the FFN's two kernels alone at batch 1, in graphs of L launches:
    gate|up with the SiLU(g) * u epilogue (writes h), and down on that h."""
    sb = stack.sb
    xs = [stack.draws("iid", 1, draw=64 + 16 * l) for l in range(stack.L)]
    hs = [torch.empty((1, F70), dtype=torch.float32, device=stack.dev) for _ in range(stack.L)]
    y = torch.empty((1, D70), dtype=torch.bfloat16, device=stack.dev)
    fns = {
        "ffn_gate_up": lambda l: sb.sfx_sparse_gemv(xs[l], stack.Wgu[l], t=t_in,
                                                    flags=sb.SFX_FLAG_SWIGLU, y=hs[l], ws=stack.ws),
        "ffn_down": lambda l: sb.sfx_sparse_gemv(hs[l], stack.Wd[l], t=t_h, y=y, ws=stack.ws),
    }
    for l in range(stack.L):
        fns["ffn_gate_up"](l)
    torch.cuda.synchronize()
    act_x = [int((xs[l].float().abs() > t_in).sum()) for l in range(stack.L)]
    act_h = [int((hs[l].abs() > t_h).sum()) for l in range(stack.L)]
    nbytes = {"ffn_gate_up": sum(a * 4 * F70 + D70 * 2 + F70 * 4 for a in act_x) / stack.L,
              "ffn_down": sum(a * 2 * D70 + F70 * 4 + D70 * 2 for a in act_h) / stack.L}
    out = {}
    for name, fn in fns.items():
        us = graph_us([lambda l=l: fn(l) for l in range(stack.L)], stream, reps=reps)
        out[name] = {"us": us, "bytes": nbytes[name], "gbs": nbytes[name] / (us * 1e-6) / 1e9,
                     "launches_timed": reps * stack.L}
    return out


def oracle_chunks_70b(stack, l, x, t_in, t_h, chunk=2048):
    """The oracle's FFN on layer l, one block of intermediate neurons at a time.

    h_j depends only on neuron j's gate/up columns and y sums the neurons'
    down rows, so the oracle's definition (O.ffn_swiglu) runs on blocks of
    neurons and the block outputs add up to y. Returns (y, h, m_x, m_h) in fp64.
    """
    import oracle as O
    x64 = x.to("cpu", torch.float64).numpy()
    y = np.zeros((x64.shape[0], D70))
    hs, mhs, m_x = [], [], None
    Wgu = stack.Wgu[l]
    for j0 in range(0, F70, chunk):
        j1 = min(F70, j0 + chunk)
        Wg = Wgu[:, 2 * j0:2 * j1:2].to("cpu", torch.float64).numpy()
        Wu = Wgu[:, 2 * j0 + 1:2 * j1:2].to("cpu", torch.float64).numpy()
        Wd = stack.Wd[l][j0:j1].to("cpu", torch.float64).numpy()
        yc, hc, m_x, mhc = O.ffn_swiglu(x64, t_in, Wg, Wu, Wd, t_h)
        y += yc
        hs.append(hc)
        mhs.append(mhc)
    return y, np.concatenate(hs, 1), m_x, np.concatenate(mhs, 1)


def flips_vs_oracle(stack, t_in, t_h):
    """Mask agreement of the GPU path with the oracle on layer 0 at batch 1.

    The oracle takes the GPU's thresholds; the x mask must match bit for bit,
    the h mask may differ where the fp32 and fp64 h straddle t_h (counted).
    """
    import oracle as O
    sb = stack.sb
    x = stack.draws("iid", 1)
    r = sb.sfx_sparse_ffn_swiglu(x, stack.Wgu[0], stack.Wd[0], t_in, t_h, want_bitmaps=True,
                                 want_h=True, ws=stack.ws)
    y, h, m_x, m_h = oracle_chunks_70b(stack, 0, x, t_in, t_h)
    bx = np.unpackbits(r["bitmap_x"].view(torch.uint8).cpu().numpy(), bitorder="little")[:D70]
    bh = np.unpackbits(r["bitmap_h"].view(torch.uint8).cpu().numpy(), bitorder="little")[:F70]
    yg = r["y"].to("cpu", torch.float64).numpy()
    want = O.round_to(y, "bf16")
    return {"x_mask_flips": int(np.count_nonzero(bx.astype(bool) != m_x[0])),
            "h_mask_flips": int(np.count_nonzero(bh.astype(bool) != m_h[0])),
            "h_active": int(m_h.sum()), "x_active": int(m_x.sum()),
            "y_rel_l2_vs_oracle": float(np.linalg.norm(yg - want) / np.linalg.norm(want)),
            "note": "layer 0, batch 1; the oracle (fp64, blocks of 2048 neurons) takes the GPU's "
                    "thresholds, so flips count only where fp32 and fp64 h straddle t_h"}


# ---------------------------------------------------------------- CPU oracle legs

def oracle_sample_70b(stack, frac):
    """Layer 0 of the headline FFN restricted to its first `frac` of the
    intermediate neurons: fp64 host copies (W_g, W_u [d x n], W_d [n x d])."""
    n = max(64, int(F70 * frac) // 64 * 64)
    Wgu = stack.Wgu[0]
    return {"Wg": Wgu[:, 0:2 * n:2].to("cpu", torch.float64).numpy(),
            "Wu": Wgu[:, 1:2 * n:2].to("cpu", torch.float64).numpy(),
            "Wd": stack.Wd[0][:n].to("cpu", torch.float64).numpy(), "n": n}


def oracle_pass(W, x64, t_in, t_h):
    import oracle as O
    return O.ffn_swiglu(x64, t_in, W["Wg"], W["Wu"], W["Wd"], t_h)


def oracle_pass_bytes(W, x64, t_in, t_h):
    """Algorithmic bytes of one sampled pass, counted as the GPU arm counts them."""
    _, _, m_x, m_h = oracle_pass(W, x64, t_in, t_h)
    n = W["n"]
    return int(m_x.sum()) * 4 * n + int(m_h.sum()) * 2 * D70 + 2 * D70 * 2 + 2 * n * 4


def time_oracle(W, x64, t_in, t_h, seconds, threads):
    """Passes of the sampled oracle FFN in about `seconds`, on `threads` BLAS threads."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=threads):
        reps, t0 = 0, time.perf_counter()
        while reps == 0 or time.perf_counter() - t0 < seconds:
            oracle_pass(W, x64, t_in, t_h)
            reps += 1
        el = time.perf_counter() - t0
    return reps, el


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline_70b(stack, t_in, t_h, seconds):
    """The fp64 oracle as it stands on a bounded sample of the headline layer,
    on one host thread and on one thread per core (BLAS threads)."""
    W = oracle_sample_70b(stack, 1 / 16)
    x64 = stack.draws("iid", 1).to("cpu", torch.float64).numpy()
    nbytes = oracle_pass_bytes(W, x64, t_in, t_h)
    cores = host_cores()
    r1, e1 = time_oracle(W, x64, t_in, t_h, seconds / 2, 1)
    rn, en = time_oracle(W, x64, t_in, t_h, seconds / 2, cores)
    return {"value": nbytes * rn / en / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "single_thread_gbs": nbytes * r1 / e1 / 1e9,
            "us_per_layer_all_cores": en / rn * 1e6 * (F70 / W["n"]),
            "us_per_layer_single_thread": e1 / r1 * 1e6 * (F70 / W["n"]),
            "sample": f"layer 0 of the headline FFN on its first {W['n']} of {F70} intermediate "
                      f"neurons (1/16), batch 1: {r1} passes on 1 thread in {e1:.1f} s, {rn} "
                      f"passes on {cores} threads in {en:.1f} s; value = the all-core run"}


def reference_arm(args):
    """The oracle, as it stands, timed on the host cores on the headline workload.

    Each step is one pass of the oracle's SwiGLU FFN (fp64, all host cores
    through BLAS) over a sample of layer 0: its first intermediate neurons,
    as many as keep the whole run within about two minutes. Thresholds are the
    oracle's own (calibrated on the same 64 draws; down-in on its h of them).
    """
    import oracle as O
    from sparse_input_gemv_b200 import synth
    p = args.sparsity
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))

    class One:
        pass

    st = One()
    Wg = synth.normal((D70, F70), synth.seed_of("l70", "Wg", 0), 0.02, "bf16", dev)
    Wu = synth.normal((D70, F70), synth.seed_of("l70", "Wu", 0), 0.02, "bf16", dev)
    st.Wgu = [torch.stack([Wg, Wu], 2).reshape(D70, 2 * F70)]
    del Wg, Wu
    st.Wd = [synth.normal((F70, D70), synth.seed_of("l70", "Wd", 0), 0.02, "bf16", dev)]
    calib = synth.calib_draws("l70", "x", 64, D70, "bf16", draw=0).double().numpy()
    x64 = synth.eval_draw("l70", "x", 1, D70, "bf16").double().numpy()
    t_in = O.calibrate_threshold(calib, p)
    W = oracle_sample_70b(st, 1 / 64)
    _, hc, _, _ = O.ffn_swiglu(calib, -math.inf, W["Wg"], W["Wu"], W["Wd"], -math.inf)
    t_h = O.calibrate_threshold(hc, p)
    t0 = time.perf_counter()
    oracle_pass(W, x64, t_in, t_h)
    t_one = time.perf_counter() - t0
    frac = min(0.25, (1 / 64) * 120.0 / max(t_one * (args.steps + args.warmup), 1e-9))
    if frac > 1 / 64:
        W = oracle_sample_70b(st, frac)
    for _ in range(args.warmup):
        oracle_pass(W, x64, t_in, t_h)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_pass(W, x64, t_in, t_h)
    el = time.perf_counter() - t0
    nbytes = oracle_pass_bytes(W, x64, t_in, t_h)
    gbs = nbytes * args.steps / el / 1e9
    cores = host_cores()
    sample = (f"one pass of the fp64 numpy oracle's SwiGLU FFN per step on layer 0, its first "
              f"{W['n']} of {F70} intermediate neurons, batch 1, BLAS on the host cores")
    return {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / max(args.steps, 1) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1, "sparsity": p, "layers_per_step": 1,
                   "parallelism": "host cores"},
        "us_per_layer": el / max(args.steps, 1) * 1e6 * (F70 / W["n"]),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------- profiling cases

PROFILE_CASES = {
    "ffn_gate_up": "the headline gate|up GEMV (SiLU(g) * u epilogue), batch 1",
    "ffn_down": "the headline down GEMV on the gate|up stage's h, batch 1",
    "ffn": "the headline SwiGLU FFN call, batch 1",
    "union_gate_up_b16": "the gate|up product of 16 tokens (batch-union kernels), same layer",
    "union_down_b16": "the down product of 16 tokens on their fp32 h (batch-union kernels; the "
                      "union keeps every row, so the dense kernel with the split x runs), same layer",
    "union_mma_gate_up_8b_b16": "a Llama-3-8B-shaped gate|up product (W 4096 x 28672) of 16 "
                                "correlated tokens on the gathered-union mma.sync kernel",
    "union_tc_gate_up_8b_b16": "the same product on the tcgen05 union kernel (kept for comparison)",
    "moe_b1": "the 128-expert MoE layer (d=2048, expert ffn=768, top-8, shared ffn=2048), batch 1",
    "topk_phi2": "the Phi-2-shaped GeLU up GEMV (2560 -> 10240) and the GxO top-k select, keep "
                 "1 - sparsity",
    "static_up_phi2": "the Phi-2-shaped FFN on a static GLASS set (keep 1 - sparsity) on both "
                      "projections, batch 1",
}


def profile_other(name, p, dev, launches):
    """The small cases of profile_case outside the headline layer."""
    from sparse_input_gemv_b200 import binding as sb
    from sparse_input_gemv_b200 import synth
    ws = sb.Workspace(dev)
    if name in ("union_mma_gate_up_8b_b16", "union_tc_gate_up_8b_b16"):
        K, N = 4096, 28672
        W = synth.normal((K, N), synth.seed_of("prof-8b", "Wgu"), 0.02, "bf16", dev)
        x = synth.correlated_draws("prof-8b", "x", 16, K, "bf16").to(dev)
        calib = synth.calib_draws("prof-8b", "x", 64, K, "bf16").to(dev)
        t = sb.sfx_calibrate_thresholds(calib, [p], ws=ws)[0]
        h = torch.empty((16, N // 2), dtype=torch.float32, device=dev)
        kern = sb.UNION_MMA if name.startswith("union_mma") else sb.UNION_TCGEN05
        with sb.plan_overrides(union_kernel=kern, dense=sb.DENSE_UNION_ONLY):
            for _ in range(launches):
                sb.sfx_sparse_gemv(x, W, t=t, flags=sb.SFX_FLAG_SWIGLU, y=h, ws=ws)
    elif name == "moe_b1":
        E, d, f, fs, top = 128, 2048, 768, 2048, 8
        WgT = synth.normal((E, f, d), synth.seed_of("prof-moe", "WgT"), 0.02, "bf16", dev)
        WuT = synth.normal((E, f, d), synth.seed_of("prof-moe", "WuT"), 0.02, "bf16", dev)
        Wd = synth.normal((E, f, d), synth.seed_of("prof-moe", "Wd"), 0.02, "bf16", dev)
        Sg = synth.normal((fs, d), synth.seed_of("prof-moe", "SgT"), 0.02, "bf16", dev)
        Su = synth.normal((fs, d), synth.seed_of("prof-moe", "SuT"), 0.02, "bf16", dev)
        Sd = synth.normal((fs, d), synth.seed_of("prof-moe", "Sd"), 0.02, "bf16", dev)
        # per-expert thresholds: the gate activations of 16 calibration tokens routed to
        # every expert, calibrated per expert
        xc = synth.calib_draws("prof-moe", "x", 16, d, "bf16").to(dev)
        ninf = torch.full((E,), -math.inf, dtype=torch.float32, device=dev)
        a = sb.sfx_moe_expert_sparse(xc, torch.zeros((16, E), dtype=torch.float32, device=dev),
                                     WgT, WuT, Wd, ninf, E, want_a=True, ws=ws)["a"]
        a_e = a.permute(1, 0, 2).contiguous()
        te = torch.tensor([sb.sfx_calibrate_thresholds(a_e[e], [p], ws=ws)[0] for e in range(E)],
                          dtype=torch.float32, device=dev)
        x = synth.eval_draw("prof-moe", "x", 1, d, "bf16").to(dev)
        logits = synth.normal((1, E), synth.seed_of("prof-moe", "logits"), 1.0, "f32", dev)
        y = torch.empty((1, d), dtype=torch.bfloat16, device=dev)
        for _ in range(launches):
            sb.sfx_moe_expert_sparse(x, logits, WgT, WuT, Wd, te, top, Ws_gT=Sg, Ws_upT=Su,
                                     Ws_d=Sd, y=y, ws=ws)
    else:  # the Phi-2-shaped FFN cases
        d, f = 2560, 10240
        k = int((1.0 - p) * f + 0.5)
        W1 = synth.normal((d, f), synth.seed_of("prof-phi2", "W1"), 0.02, "f16", dev)
        W2 = synth.normal((f, d), synth.seed_of("prof-phi2", "W2"), 0.02, "f16", dev)
        x = synth.eval_draw("prof-phi2", "x", 1, d, "f16").to(dev)
        g = synth.normal((1, f), synth.seed_of("prof-phi2", "g"), 1.0, "f32", dev)
        h = torch.empty((1, f), dtype=torch.float32, device=dev)
        if name == "topk_phi2":
            for _ in range(launches):
                sb.sfx_sparse_gemv(x, W1, flags=sb.SFX_FLAG_GELU, y=h, ws=ws)
                sb.sfx_mask_compact(h, sb.SFX_SEL_TOPK_GXO, k=k, score_l=g, ws=ws)
        else:
            sl = synth.abs_normal((1, f), synth.seed_of("prof-phi2", "local"), device=dev)
            sgl = synth.abs_normal((1, f), synth.seed_of("prof-phi2", "global"), device=dev)
            gl = sb.sfx_mask_compact(None, sb.SFX_SEL_TOPK_GLASS, k=k, score_l=sl, score_g=sgl,
                                     lam=0.5, ws=ws)
            W1T = W1.t().contiguous()
            y = torch.empty((1, d), dtype=torch.float16, device=dev)
            for _ in range(launches):
                sb.sfx_static_ffn(x, W1T, W2, gl["idx"][0], gl["cnt"], y=y, ws=ws)
    torch.cuda.synchronize()


def profile_case(name, p, dev, launches=6):
    """One kernel (or call) of a small case, `launches` times, then exit: the
    headline layer's, or another workload's. The ncu captures in profiles/ run this."""
    if name not in ("ffn_gate_up", "ffn_down", "ffn", "union_gate_up_b16", "union_down_b16"):
        profile_other(name, p, dev, launches)
        print(json.dumps({"profile_case": name, "sparsity": p, "launches": launches,
                          "what": PROFILE_CASES[name]}), flush=True)
        return
    stack = Ffn70Stack(1, dev)
    sb = stack.sb
    t_in, t_h = stack.thresholds(p)
    x = stack.draws("iid", 1)
    h = torch.empty((1, F70), dtype=torch.float32, device=dev)
    y = torch.empty((1, D70), dtype=torch.bfloat16, device=dev)
    sb.sfx_sparse_gemv(x, stack.Wgu[0], t=t_in, flags=sb.SFX_FLAG_SWIGLU, y=h, ws=stack.ws)
    x16 = stack.draws("iid", 16)
    h16 = torch.empty((16, F70), dtype=torch.float32, device=dev)
    y16 = torch.empty((16, D70), dtype=torch.bfloat16, device=dev)
    if name == "union_down_b16":
        sb.sfx_sparse_gemv(x16, stack.Wgu[0], t=t_in, flags=sb.SFX_FLAG_SWIGLU, y=h16, ws=stack.ws)
    for _ in range(launches):
        if name == "ffn_gate_up":
            sb.sfx_sparse_gemv(x, stack.Wgu[0], t=t_in, flags=sb.SFX_FLAG_SWIGLU, y=h, ws=stack.ws)
        elif name == "ffn_down":
            sb.sfx_sparse_gemv(h, stack.Wd[0], t=t_h, y=y, ws=stack.ws)
        elif name == "ffn":
            stack.call(0, x, t_in, t_h, y)
        elif name == "union_gate_up_b16":
            sb.sfx_sparse_gemv(x16, stack.Wgu[0], t=t_in, flags=sb.SFX_FLAG_SWIGLU, y=h16,
                               ws=stack.ws)
        elif name == "union_down_b16":
            sb.sfx_sparse_gemv(h16, stack.Wd[0], t=t_h, y=y16, ws=stack.ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "sparsity": p, "launches": launches,
                      "what": PROFILE_CASES[name]}), flush=True)


# ---------------------------------------------------------------- main

def measure_step(step_fn, stream, steps, warmup, dist, dev, clocks_index=None, e2e_bufs=None):
    """Capture `step_fn` in a graph and time `steps` replays (CUDA events,
    barrier + synchronize on both sides, max over ranks). With `e2e_bufs`
    = (device inputs, device outputs) also time the same replays with a pinned
    host->device copy of the inputs and a device->host copy of the outputs."""
    for _ in range(max(warmup, 1)):
        step_fn()
    torch.cuda.synchronize()
    g = capture(step_fn, stream)
    for _ in range(2):
        g.replay()
    res = {}
    sampler = ClockSampler(clocks_index) if clocks_index is not None else None
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
    if e2e_bufs is not None:
        xs, ys = e2e_bufs
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
        res["e2e_ms"] = max_over_ranks(start.elapsed_time(end), dist, dev)
        res["h2d"] = sum(x.numel() * x.element_size() for x in xs)
        res["d2h"] = sum(y.numel() * y.element_size() for y in ys)
    del g
    return res


def greedy_allocation_8b(stack, stream, steps, target, step=0.05):
    """TEAL slide 10 on the 8B layer: per-site sparsities from the greedy rounds on
    the sites' l2 error curves (GPU, layer 0's weights and calibration draws), at
    the model-wide target (sites weighted by their parameter counts), then the
    layer timed at that allocation next to the uniform one."""
    sb = stack.sb
    levels = [round(step * i, 4) for i in range(int(round(0.95 / step)) + 1)]
    weights_of = {"qkv-in": stack.Wqkv[0], "o-in": stack.Wo[0], "ffn-in": stack.Wgu[0],
                  "down-in": stack.Wd[0]}
    curves, weights = [], []
    for site in stack.SITES:
        W = weights_of[site]
        err, _ = sb.sfx_block_error_curve(stack.calib[site].contiguous(), W, levels)
        curves.append(err)
        weights.append(W.shape[0] * W.shape[1])  # the weights the site's sparsity skips
    lv = sb.sfx_greedy_allocate(curves, weights, step, target)
    alloc = {site: round(l * step, 4) for site, l in zip(stack.SITES, lv)}
    stack.set_sparsity(alloc)
    r = measure_step(stack.step, stream, steps, 2, None, stack.dev)
    us = r["ms"] * 1e3 / (steps * stack.L)
    overall = sum(w * alloc[s] for s, w in zip(stack.SITES, weights)) / sum(weights)
    return {"target": target, "step": step, "allocation": alloc, "overall_sparsity": overall,
            "us_per_layer": round(us, 2),
            "gbs": round(stack.step_bytes() * steps / (r["ms"] * 1e-3) / 1e9, 1),
            "error_at_allocation": {s: curves[i][lv[i]] for i, s in enumerate(stack.SITES)},
            "error_uniform": {s: curves[i][int(round(target / step))]
                              for i, s in enumerate(stack.SITES)},
            "note": "l2 output error of each site on its 64 calibration draws (layer 0)"}


def llama8b_layer(stream, dev, sparsity, steps, sweep_ps, layers=32):
    """The Llama-3-8B-shaped decoder layer (qkv, o, SwiGLU FFN) at batch 1,
    secondary workload: µs per layer at `sparsity` and over a sweep."""
    stack = Stack(layers, dev, keep_layer0_fp64=False)
    out = {"workload": WORKLOAD_8B, "layers": layers}
    sweep = []
    for p in sweep_ps:
        stack.set_sparsity(p)
        r = measure_step(stack.step, stream, steps, 2, None, dev)
        us = r["ms"] * 1e3 / (steps * layers)
        sweep.append({"sparsity": p, "us_per_layer": round(us, 2),
                      "gbs": round(stack.step_bytes() * steps / (r["ms"] * 1e-3) / 1e9, 1)})
    out["sweep"] = sweep
    base = next((s["us_per_layer"] for s in sweep if s["sparsity"] == 0), None)
    if base:
        for s in sweep:
            s["time_ratio_vs_p0"] = round(s["us_per_layer"] / base, 3)
    stack.set_sparsity(sparsity)
    kernels = {}
    for name, fn in stack.kernel_fns().items():
        us = graph_us([lambda l=l: fn(l) for l in range(layers)], stream, reps=5)
        kb = sum(stack.kernel_bytes(name, l) for l in range(layers)) / layers
        kernels[name] = {"us": round(us, 2), "gbs": round(kb / (us * 1e-6) / 1e9, 1)}
    out["kernels_at_sparsity"] = {"sparsity": sparsity, **kernels}
    out["dense_library_us_per_layer"] = round(dense_library_us_per_layer(stack, stream), 2)
    out["greedy_allocation"] = greedy_allocation_8b(stack, stream, steps, target=sparsity)
    del stack
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sfx", "reference"], default="sfx")
    ap.add_argument("--sparsity", type=float, default=0.5)
    ap.add_argument("--layers", type=int, default=8, help="70B FFN layers in the stack")
    ap.add_argument("--no-sweep", action="store_true", help="skip the batch x sparsity sweep")
    ap.add_argument("--cpu-seconds", type=float, default=16.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-other", action="store_true",
                    help="skip the other workloads (" + ", ".join(OTHER_WORKLOADS) + ")")
    ap.add_argument("--other", default=",".join(OTHER_WORKLOADS),
                    help="comma list of the other workloads to run: " + ", ".join(OTHER_WORKLOADS))
    ap.add_argument("--threshold-table", default=None,
                    help="JSON threshold table to read (if present) and write: the headline "
                         "layer's calibrated thresholds keyed by (config, site, p, seed)")
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES), default=None,
                    help="run one kernel of the headline layer a few times and exit (the small "
                         "case an ncu capture runs: one 1.4 GB layer on the device)")
    args = ap.parse_args()

    rank, local_rank, world = env_rank()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return

    from sparse_input_gemv_b200 import binding as sb
    sb.load()
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    if args.profile_case:
        profile_case(args.profile_case, args.sparsity, dev)
        return
    from sparse_input_gemv_b200.thresholds import ThresholdTable
    table = ThresholdTable(args.threshold_table)
    stack = Ffn70Stack(args.layers, dev, table)
    L = args.layers
    t_in, t_h = stack.thresholds(args.sparsity)
    # the step's inputs and outputs each live in one device buffer (a row per
    # layer), so the end-to-end leg moves them with one copy each way
    X = torch.cat([stack.draws("iid", 1, draw=64 + 16 * l) for l in range(L)]).contiguous()
    Y = torch.empty((L, D70), dtype=torch.bfloat16, device=dev)
    xs = [X[l:l + 1] for l in range(L)]
    ys = [Y[l:l + 1] for l in range(L)]
    layer_bytes = [stack.active_bytes(l, xs[l], t_in, t_h)[0] for l in range(L)]
    bytes_step = sum(layer_bytes)

    def step():
        for l in range(L):
            stack.call(l, xs[l], t_in, t_h, ys[l])

    # headline: K timed steps of the 8-layer stack
    K = args.steps
    main_res = measure_step(step, stream, K, args.warmup, dist, dev, clocks_index=local_rank,
                            e2e_bufs=([X], [Y]))
    ms = main_res["ms"]
    value = replica_gbs(bytes_step, K, world, ms)
    us_layer = ms * 1e3 / (K * L)

    # the FFN's two kernels alone (roofline), and p = 0 for the dense reference point
    kernels = stage_kernels_70b(stack, stream, t_in, t_h)
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
                "bytes_per_launch": kernels[dom]["bytes"], "traffic": None}
    roofline["traffic"], roofline["traffic_note"] = profiled_traffic(dom, args.sparsity)
    ffn_roof = {"achieved": bytes_step / L / (us_layer * 1e-6) / 1e9}
    ffn_roof["frac"] = ffn_roof["achieved"] / peak

    sweep = corr = lib = None
    if not args.no_sweep:
        sweep = sweep_70b(stack, stream)
        corr = sweep_70b(stack, stream, batches=(4, 8, 16), ps=(0.5, 0.7, 0.9), kind="corr")
        lib = dense_library_70b(stack, stream)
    scaling = None
    if sweep:
        b1 = {r["sparsity"]: r["us"] for r in sweep if r["batch"] == 1}
        dense_b1 = b1.get(0.0)
        nb1 = {r["sparsity"]: r["bytes"] for r in sweep if r["batch"] == 1}
        if dense_b1:
            scaling = [{"sparsity": p, "time_ratio": round(u / dense_b1, 3),
                        "byte_ratio": round(nb1[p] / nb1[0.0], 3)} for p, u in sorted(b1.items())]

    flips = None
    cpu = None
    if rank == 0 and not args.no_cpu:
        flips = flips_vs_oracle(stack, t_in, t_h)
        cpu = cpu_baseline_70b(stack, t_in, t_h, args.cpu_seconds)
    e2e_val = replica_gbs(bytes_step, K, world, main_res["e2e_ms"])
    del stack
    torch.cuda.empty_cache()

    other = None
    if rank == 0 and not args.no_other:
        which = tuple(w for w in args.other.split(",") if w)
        other = {}
        if "llama8b" in which:
            other["llama3_8b_decoder_layer_b1"] = llama8b_layer(
                stream, dev, args.sparsity, 20, (0.0, 0.25, 0.4, 0.5, 0.65, 0.9))
        rest = tuple(w for w in which if w != "llama8b")
        if rest:
            other.update(bench_other_workloads(stream, dev, rest))

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1, "sparsity": args.sparsity,
                   "layers_per_step": L,
                   "l2": f"inputs larger than L2: {L} distinct layers, "
                         f"{L * 3 * D70 * F70 * 2 / 1e9:.1f} GB of weights per step",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "us_per_layer": us_layer, "thresholds": {"gate_up_in": t_in, "down_in": t_h},
        "active_bytes_per_layer": bytes_step / L, "dense_bytes_per_layer": 3 * D70 * F70 * 2,
        "ffn_roofline": ffn_roof,
        "kernels": kernels, "roofline": roofline,
        "sweep": sweep, "scaling_b1": scaling, "sweep_correlated": corr, "dense_library": lib,
        "mask_flips": flips,
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": main_res["h2d"],
                "d2h_bytes_per_step": main_res["d2h"], "ms_per_step": main_res["e2e_ms"] / K,
                "path": "CUDA graph of sfx_sparse_ffn_swiglu calls; the step's inputs and "
                        "outputs in one pinned host buffer each, one copy each way"},
        "gpu_launches": 2 * L * K,
        "clocks": main_res.get("clocks"),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if other is not None:
        line["other_workloads"] = other
    if rank == 0:
        if args.threshold_table:
            table.save()
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
