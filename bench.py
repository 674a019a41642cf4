#!/usr/bin/env python
"""Benchmark of the RPTQ data path on B200; rank 0 prints one JSON line.

A step is one pass of the whole path over one synthetic batch of the workload:
  1. calibration statistics of LayerNorm(x) over the calibration batch   (rptq_calib_minmax)
  2. KMeans -> reorder index R and per-cluster (s, z)                    (rptq_kmeans)
  3. the LayerNorm rewrite of this calibration, then the reorder-fused LayerNorm + per-cluster
     quantization of the batch       (rptq_ln_quant_plan, rptq_ln_reorder_quant_planned; the
     unplanned rptq_ln_reorder_quant is timed beside it)
  3a. the explicit-reorder baseline, dynamic ranges, and the reordered linear layer on one
      2048-token micro-batch of the codes  (rptq_baseline_..., rptq_linear_prepare, rptq_reordered_linear)
  4. K/V calibration statistics, KMeans for K and for V                   (rptq_kv_calib_minmax, rptq_kmeans)
  5. K/V cache quantization                                               (rptq_kv_quant)
  6. dequantization of the activation codes and of the K/V codes         (rptq_dequant)
`value` is the metric's own kernel, measured inside those steps: the algorithmic GB/s of the
fused LN-reorder-quant (read x, write the packed codes), its bytes summed over ranks and its
device time the slowest rank's (the K/V quantizer for the K/V-only workload).  `step` gives
the same for the whole step, `kernels` every stage (see
post_activation_quantization_b200/workloads.py for the byte counts).  Inputs are larger than
the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl rptq|reference]
Multi-GPU: one process per GPU (run under torchrun, or `--gpus N` starts N ranks itself), weak
scaling (every rank its own batch); the calibration statistics are combined with one MAX/MIN
all-reduce (NCCL).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from post_activation_quantization_b200 import dist as pdist  # noqa: E402
from post_activation_quantization_b200 import synthetic  # noqa: E402
from post_activation_quantization_b200 import workloads as W  # noqa: E402

METRIC = "fused LN+reorder+cluster-quant GB/s & Mtokens/s; % of B200 HBM peak"
DEFAULT_WORKLOAD = "opt175b-12288"
L2_BYTES = 126 * 2 ** 20
HBM_FALLBACK_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return HBM_FALLBACK_GBS, "fallback"


def tensor_peak() -> float:
    """Measured dense bf16 GEMM TFLOP/s (burst), else the pool's earlier measurement."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def has_act(w: W.Workload) -> bool:
    """Whether the workload carries the activation path (the K/V-only workload does not)."""
    return w.T > 0 and w.C > 0


def stage_flops(w: W.Workload):
    """Stages bound by the tensor cores: name -> operations per call."""
    return {"reordered_linear": W.flops_linear(*W.linear_shape(w))} if has_act(w) else {}


def stage_list(w: W.Workload):
    """(name, algorithmic bytes per call, launches of this library's kernels per call) of the
    step's stages, in order.  A calibration call without `accumulate` is an init launch + the
    reduction; a KMeans call is two launches (the workspace clear and the cooperative kernel)."""
    k, a = w.kv, has_act(w)
    n = w.T * w.C
    st = [("calib_ln", W.bytes_calib(w.T_cal or w.T, w.C, w.dtype), 2)] if a else []
    if k:
        st += [("kv_calib", 2 * W.bytes_calib(k.B * k.S, k.channels, k.dtype), 4)]
    st += [("kmeans", 0, 2 * ((1 if a else 0) + (2 if k else 0)))]
    if a:
        # the offline LayerNorm rewrite of this calibration (per-channel offsets and
        # coefficients), then the fused kernel reading it; the same kernel building those tables
        # in every CTA is timed beside it
        st += [("ln_quant_plan", W.bytes_ln_quant_plan(w.C), 1),
               ("ln_reorder_quant", W.bytes_ln_quant(w.T, w.C, w.dtype, w.bits), 1),
               ("ln_reorder_quant_unplanned", W.bytes_ln_quant(w.T, w.C, w.dtype, w.bits), 1)]
        # the unfused pipeline the fused kernel replaces (a measurement baseline, same results)
        st += [("explicit_reorder_baseline", W.bytes_explicit_reorder(w.T, w.C, w.dtype, w.bits), 3)]
        # what dynamic (per-batch) cluster ranges add before the same fused kernel: the batch's
        # LayerNorm statistics and the per-cluster (s, z) of the fixed clusters
        st += [("dynamic_ranges", W.bytes_calib(w.T, w.C, w.dtype), 3)]
        # the layer after the LayerNorm: its weights re-prepared for this calibration's R and
        # (s, z), then one micro-batch of the codes through it (tensor cores; FLOPS below)
        Tl, C, N = W.linear_shape(w)
        st += [("linear_prepare", W.bytes_linear_prepare(N, C), 1), ("reordered_linear", 0, 1)]
    if k:
        st += [("kv_quant", W.bytes_kv_quant(k.elems, k.dtype, k.bits), 1)]
        # the layout variant: the K cache quantized into token rows in cluster order (a comparison
        # beside the kept layout's K/V quantizer: one tensor, the same codes)
        st += [("kv_quant_cluster_ordered", W.bytes_kv_quant(k.elems, k.dtype, k.bits, tensors=1), 1)]
    if a:
        st += [("dequant_act", W.bytes_dequant(n, w.dtype, w.bits), 1)]
    if k:
        st += [("dequant_kv", 2 * W.bytes_dequant(k.elems, k.dtype, k.bits), 2)]
        # one decode step: a token appended to K and V, then attention over the whole cache
        st += [("kv_append", W.bytes_kv_append(k.B, k.H, k.D, k.dtype, k.bits), 1),
               ("kv_decode_attention", W.bytes_kv_attention(k.B, k.H, k.S, k.D, k.bits), 1)]
    return st


# ------------------------------------------------------------------------------------------
class Step:
    """Device buffers of one rank and the sequence of library calls that makes a step."""

    def __init__(self, w: W.Workload, rank: int, device):
        from post_activation_quantization_b200 import rptq
        self.r = rptq
        self.w, self.dev = w, device
        self.kvw = w.kv
        self.act = has_act(w)  # the K/V-only workload has no activation stages
        if self.act:
            dt = synthetic.torch_dtype(w.dtype)
            m = synthetic.channel_model(w.C, w.seed, w.outlier_frac, w.outlier_factor)
            g, b = synthetic.ln_params(w.C, w.seed)
            self.gamma, self.beta = g.to(device), b.to(device)
            # every rank draws its own tokens of the same model
            self.xcal = synthetic.activations(w.T_cal or w.T, m, w.seed + 7919 * rank, dtype=w.dtype,
                                              calibration=True, device=device)
            self.x = synthetic.activations(w.T, m, w.seed + 7919 * rank, dtype=w.dtype, device=device)
            self.mx = torch.empty(w.C, dtype=torch.float32, device=device)
            self.mn = torch.empty_like(self.mx)
            self.km = self._km_out(w.C, w.g)
            self.ws = torch.empty(rptq.rptq_kmeans_workspace_size(w.C, w.g), dtype=torch.uint8, device=device)
            self.codes = torch.empty((w.T, w.C * w.bits // 8), dtype=torch.uint8, device=device)
            self.plan = torch.empty(rptq.rptq_ln_quant_plan_bytes(w.C), dtype=torch.uint8, device=device)
            self.xr_y = torch.empty((w.T, w.C), dtype=torch.float32, device=device)
            self.xr_yr = torch.empty_like(self.xr_y)
            self.xr_codes = torch.empty_like(self.codes)
            self.dmx, self.dmn = torch.empty_like(self.mx), torch.empty_like(self.mx)
            self.dsc = torch.empty(w.g, dtype=torch.float32, device=device)
            self.dz = torch.empty(w.g, dtype=torch.int32, device=device)
            self.xhat = torch.empty((w.T, w.C), dtype=dt, device=device)
            Tl, _, N = W.linear_shape(w)
            self.lin_T = Tl
            self.wq, self.wsc, self.wz = synthetic.weight_codes(N, w.C, w.seed, device=device)
            self.wprep = torch.empty((N, w.C), dtype=torch.float16, device=device)
            self.wbias = torch.empty(N, dtype=torch.float32, device=device)
            self.wlam = torch.empty(N, dtype=torch.float32, device=device)
            self.ylin = torch.empty((Tl, N), dtype=torch.float32, device=device)
        if self.kvw:
            k = self.kvw
            mk = synthetic.channel_model(k.channels, w.seed, k.outlier_frac, k.outlier_factor, tag=1)
            mv = synthetic.channel_model(k.channels, w.seed, k.outlier_frac, k.outlier_factor, tag=2)
            self.k = synthetic.kv_cache(k.B, k.H, k.S, k.D, mk, w.seed + 7919 * rank, "k", k.dtype, device)
            self.v = synthetic.kv_cache(k.B, k.H, k.S, k.D, mv, w.seed + 7919 * rank, "v", k.dtype, device)
            self.kst = [torch.empty(k.channels, dtype=torch.float32, device=device) for _ in range(4)]
            self.kmk = self._km_out(k.channels, k.g)
            self.kmv = self._km_out(k.channels, k.g)
            self.wsk = torch.empty(rptq.rptq_kmeans_workspace_size(k.channels, k.g), dtype=torch.uint8,
                                   device=device)
            self.wsv = torch.empty_like(self.wsk)
            shape = (k.B, k.H, k.S, k.D * k.bits // 8)
            self.kq = torch.empty(shape, dtype=torch.uint8, device=device)
            self.vq = torch.empty(shape, dtype=torch.uint8, device=device)
            self.kq_co = torch.empty((k.B, k.S, k.H * k.D * k.bits // 8), dtype=torch.uint8, device=device)
            kvdt = synthetic.torch_dtype(k.dtype)
            self.khat = torch.empty((k.B, k.H, k.S, k.D), dtype=kvdt, device=device)
            self.vhat = torch.empty_like(self.khat)
            # the decode step's new token and query
            self.knew = synthetic.kv_cache(k.B, k.H, 1, k.D, mk, w.seed + 7919 * rank + 1, "k", k.dtype, device)
            self.vnew = synthetic.kv_cache(k.B, k.H, 1, k.D, mv, w.seed + 7919 * rank + 1, "v", k.dtype, device)
            gq = torch.Generator(device=device)
            gq.manual_seed(w.seed * 31 + rank)
            self.q = torch.randn((k.B, k.H, k.D), generator=gq, device=device, dtype=torch.float32) * 0.05
            self.attn = torch.empty((k.B, k.H, k.D), dtype=torch.float32, device=device)
        # the three KMeans problems are independent: they run concurrently on their own streams
        self.side = [torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)]

    def _km_out(self, C, g):
        d = self.dev
        return dict(labels=torch.empty(C, dtype=torch.int32, device=d),
                    centroids=torch.empty((g, 2), dtype=torch.float64, device=d),
                    R=torch.empty(C, dtype=torch.int32, device=d),
                    col_cluster=torch.empty(C, dtype=torch.int32, device=d),
                    offsets=torch.empty(g + 1, dtype=torch.int32, device=d),
                    scale=torch.empty(g, dtype=torch.float32, device=d),
                    zero=torch.empty(g, dtype=torch.int32, device=d))

    def stages(self):
        return stage_list(self.w)

    def repeat_calls(self):
        """The two headline kernels as single calls on the step's full-size buffers (for the
        back-to-back measurement): the planned fused LN-reorder-quant and the K/V quantizer."""
        r, w, k = self.r, self.w, self.kvw
        calls = {}
        if self.act:
            calls["ln_reorder_quant"] = lambda: r.rptq_ln_reorder_quant_planned(self.x, self.plan, w.bits, eps=w.eps,
                                                                                codes=self.codes)
        if k:
            calls["kv_quant"] = lambda: r.rptq_kv_quant(self.k, self.v, self.kmk["labels"], self.kmk["scale"],
                                                        self.kmk["zero"], self.kmv["labels"], self.kmv["scale"],
                                                        self.kmv["zero"], k.bits, k_codes=self.kq, v_codes=self.vq)
        return calls

    def run(self, ev=None):
        """Enqueue one step on the current stream; ev: optional dict name -> (start, end).

        Order: the streaming calibrations, then the activation, K and V KMeans concurrently
        (three small cooperative grids on three streams), then quantization and dequantization."""
        r, w, k = self.r, self.w, self.kvw
        main = torch.cuda.current_stream(self.dev)

        def mark(name, i):
            if ev is not None:
                ev[name][i].record(main)

        if self.act:
            mark("calib_ln", 0)
            r.rptq_calib_minmax(self.xcal, self.gamma, self.beta, w.eps, ch_max=self.mx, ch_min=self.mn)
            mark("calib_ln", 1)
            pdist.allreduce_minmax(self.mx, self.mn)
        if k:
            mark("kv_calib", 0)
            r.rptq_kv_calib_minmax(self.k, ch_max=self.kst[0], ch_min=self.kst[1])
            r.rptq_kv_calib_minmax(self.v, ch_max=self.kst[2], ch_min=self.kst[3])
            mark("kv_calib", 1)
            pdist.allreduce_minmax(self.kst[0], self.kst[1])
            pdist.allreduce_minmax(self.kst[2], self.kst[3])
        mark("kmeans", 0)
        if k:
            for s in self.side:
                s.wait_stream(main)
            with torch.cuda.stream(self.side[0]):
                r.rptq_kmeans(self.kst[0], self.kst[1], k.g, k.iters, k.bits, workspace=self.wsk, out=self.kmk,
                              stream=self.side[0])
            with torch.cuda.stream(self.side[1]):
                r.rptq_kmeans(self.kst[2], self.kst[3], k.g, k.iters, k.bits, workspace=self.wsv, out=self.kmv,
                              stream=self.side[1])
        if self.act:
            r.rptq_kmeans(self.mx, self.mn, w.g, w.iters, w.bits, workspace=self.ws, out=self.km)
        if k:
            for s in self.side:
                main.wait_stream(s)
        mark("kmeans", 1)
        if self.act:
            mark("ln_quant_plan", 0)
            r.rptq_ln_quant_plan(self.gamma, self.beta, self.km["R"], self.km["col_cluster"], self.km["scale"],
                                 self.km["zero"], w.bits, plan=self.plan)
            mark("ln_quant_plan", 1)
            mark("ln_reorder_quant", 0)
            r.rptq_ln_reorder_quant_planned(self.x, self.plan, w.bits, eps=w.eps, codes=self.codes)
            mark("ln_reorder_quant", 1)
            mark("ln_reorder_quant_unplanned", 0)
            r.rptq_ln_reorder_quant(self.x, self.gamma, self.beta, self.km["R"], self.km["col_cluster"],
                                    self.km["scale"], self.km["zero"], w.bits, eps=w.eps, codes=self.xr_codes)
            mark("ln_reorder_quant_unplanned", 1)
            mark("explicit_reorder_baseline", 0)
            r.rptq_baseline_explicit_reorder_quant(self.x, self.gamma, self.beta, self.km["R"], self.km["col_cluster"],
                                                   self.km["scale"], self.km["zero"], w.bits, eps=w.eps,
                                                   y=self.xr_y, y_reordered=self.xr_yr, codes=self.xr_codes)
            mark("explicit_reorder_baseline", 1)
            mark("dynamic_ranges", 0)
            r.rptq_calib_minmax(self.x, self.gamma, self.beta, w.eps, ch_max=self.dmx, ch_min=self.dmn)
            r.rptq_cluster_params(self.dmx, self.dmn, self.km["labels"], w.g, w.bits, scale=self.dsc, zero=self.dz)
            mark("dynamic_ranges", 1)
            mark("linear_prepare", 0)
            r.rptq_linear_prepare(self.wq, self.wz, self.km["R"], self.km["col_cluster"], self.km["scale"],
                                  self.km["zero"], w_prep=self.wprep, w_bias=self.wbias, w_lambda=self.wlam)
            mark("linear_prepare", 1)
            mark("reordered_linear", 0)
            r.rptq_reordered_linear(self.codes[:self.lin_T], w.C, w.bits, self.wprep, self.wbias, self.wlam, self.wsc,
                                    out=self.ylin)
            mark("reordered_linear", 1)
        if k:
            mark("kv_quant", 0)
            r.rptq_kv_quant(self.k, self.v, self.kmk["labels"], self.kmk["scale"], self.kmk["zero"],
                            self.kmv["labels"], self.kmv["scale"], self.kmv["zero"], k.bits,
                            k_codes=self.kq, v_codes=self.vq)
            mark("kv_quant", 1)
            mark("kv_quant_cluster_ordered", 0)
            r.rptq_kv_quant_cluster_ordered(self.k, self.kmk["R"], self.kmk["col_cluster"], self.kmk["scale"],
                                            self.kmk["zero"], k.bits, codes=self.kq_co)
            mark("kv_quant_cluster_ordered", 1)
        if self.act:
            mark("dequant_act", 0)
            r.rptq_dequant(self.codes, self.km["col_cluster"], self.km["scale"], self.km["zero"], w.bits,
                           out=self.xhat)
            mark("dequant_act", 1)
        if k:
            mark("dequant_kv", 0)
            r.rptq_dequant(self.kq, self.kmk["labels"], self.kmk["scale"], self.kmk["zero"], k.bits,
                           layout=r.RPTQ_LAYOUT_BHSD, out=self.khat)
            r.rptq_dequant(self.vq, self.kmv["labels"], self.kmv["scale"], self.kmv["zero"], k.bits,
                           layout=r.RPTQ_LAYOUT_BHSD, out=self.vhat)
            mark("dequant_kv", 1)
            mark("kv_append", 0)
            r.rptq_kv_append(self.knew, self.vnew, self.kmk["labels"], self.kmk["scale"], self.kmk["zero"],
                             self.kmv["labels"], self.kmv["scale"], self.kmv["zero"], k.bits,
                             k_cache=self.kq, v_cache=self.vq, s_begin=k.S - 1)
            mark("kv_append", 1)
            mark("kv_decode_attention", 0)
            r.rptq_kv_decode_attention(self.q, self.kq, self.vq, k.S, self.kmk["labels"], self.kmk["scale"],
                                       self.kmk["zero"], self.kmv["labels"], self.kmv["scale"], self.kmv["zero"],
                                       k.bits, out=self.attn)
            mark("kv_decode_attention", 1)


# ------------------------------------------------------------------------------------------
class Clocks:
    """SM clock, power and clock-event reasons sampled every `period_s` by a thread (NVML, in
    process) while the timed region runs; only samples taken between start() and end() are kept.
    Falls back to `nvidia-smi -lms 100` when NVML cannot be opened."""
    REASONS = (("hw_slowdown", "HwSlowdown"), ("hw_thermal_slowdown", "HwThermalSlowdown"),
               ("sw_thermal_slowdown", "SwThermalSlowdown"), ("sw_power_cap", "SwPowerCap"),
               ("hw_power_brake", "HwPowerBrakeSlowdown"))

    def __init__(self, device, period_s: float = 0.002):
        import threading
        self.period, self.rows, self.on = period_s, [], False
        self.t0 = self.t1 = None
        self.stop_ev = threading.Event()
        self.how = "nvml"
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.bits = {name: getattr(nv, "nvmlClocksEventReason" + suffix, 0) for name, suffix in self.REASONS}
            self.th = threading.Thread(target=self._loop, daemon=True)
            self.th.start()
        except Exception as e:  # noqa: BLE001 -- any NVML failure falls back to nvidia-smi
            self.how, self.nv, self.err = "unavailable", None, str(e)

    def _loop(self):
        nv, h = self.nv, self.h
        while not self.stop_ev.is_set():
            if self.on:
                t = time.time()
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                except Exception:  # noqa: BLE001
                    mhz, rs, pw = None, 0, None
                self.rows.append((t, mhz, rs, pw))
            time.sleep(self.period)

    def start(self):
        self.t0 = time.time()
        self.on = True

    def end(self):
        self.on = False
        self.t1 = time.time()

    def stop(self) -> dict:
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "reasons": ["clock sampling unavailable"],
                    "how": self.how}
        self.stop_ev.set()
        self.th.join(timeout=2)
        rows = [r for r in self.rows if r[1] is not None and self.t0 <= r[0] <= self.t1]
        sm = [r[1] for r in rows]
        reasons = sorted({n for r in rows for n, b in self.bits.items() if b and (r[2] & b)})
        bins = {}
        for v in sm:
            bins[str(int(v))] = bins.get(str(int(v)), 0) + 1
        pw = [r[3] for r in rows if r[3] is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "samples": len(rows), "period_ms": self.period * 1e3, "reasons": reasons,
                "sm_mhz_bins": bins, "power_w_max": round(max(pw), 1) if pw else None, "how": "nvml in-process"}


def _traffic(kernel: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, if it still matches
    the kernel's source (null once the source has changed)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    h = hashlib.sha256()
    for src in d["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    return d["dram_bytes_per_launch"] if h.hexdigest()[:16] == d["sources_sha"] else None


# ------------------------------------------------------------------------------------------
COMPARISON_STAGES = ("explicit_reorder_baseline", "ln_reorder_quant_unplanned", "kv_quant_cluster_ordered")
GRAPH_SLOTS = 8
B2B_LAUNCHES = 20


def back_to_back_ms(call, graph: bool) -> float:
    """Device time per launch of `call` launched B2B_LAUNCHES times back to back (one CUDA graph
    of them when `graph`, else eagerly), timed by one event pair around the run: what a kernel
    costs inside a served layer, without an event round trip around every launch.  Inputs are
    the step's full-size buffers (larger than L2), so every launch streams them from HBM."""
    g = None
    if graph:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(B2B_LAUNCHES):
                    call()
            g.replay()
        except Exception:  # noqa: BLE001 -- fall back to eager launches
            torch.cuda.synchronize()
            g = None
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    if g is not None:
        g.replay()
    else:
        for _ in range(B2B_LAUNCHES):
            call()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / B2B_LAUNCHES


def capture_steps(step, stages):
    """GRAPH_SLOTS CUDA graphs of one step each, with external (timing) event nodes around every
    stage; graphs share one memory pool (the step allocates nothing)."""
    graphs, evsets, pool = [], [], None
    for _ in range(GRAPH_SLOTS):
        ev = {n: [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for n, _, _ in stages}
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, pool=pool):
            step.run(ev)
        pool = g.pool()
        graphs.append(g)
        evsets.append(ev)
    torch.cuda.synchronize()
    return graphs, evsets


def headline_stage(w: W.Workload) -> str:
    """The stage the metric names: the fused LN-reorder-quant, or the K/V quantizer for the
    K/V-only workload."""
    return "ln_reorder_quant" if has_act(w) else "kv_quant"


def headline_tokens(w: W.Workload) -> int:
    return w.T if has_act(w) else w.kv.B * w.kv.S


def run_rptq(args):
    rank, ws, local = pdist.world()
    if ws > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", device_id=torch.device("cuda", local),
                                             timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)
    from post_activation_quantization_b200 import build, rptq
    if rank == 0:
        build.build()
    if ws > 1:
        torch.distributed.barrier()
    rptq.lib()
    w = scaled_workload(args)
    step = Step(w, rank, dev)
    stages = step.stages()
    tw = time.perf_counter()
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    tw = (time.perf_counter() - tw) / max(1, args.warmup)
    assert rptq.rptq_device_error() == 0, "device error word set during warm-up"

    # One GPU: the step is captured as CUDA graphs (GRAPH_SLOTS copies, each with its own
    # timing-event nodes between stages) and the timed region replays them K times, so the
    # stages run back to back as a served layer would, without a host launch or an event
    # round trip between kernels.  Several GPUs (a collective in the step) or --eager: the
    # step's calls are issued one by one with an event pair around each stage.
    graphs, gev = [], []
    mode = "eager"
    if ws == 1 and not args.eager:
        try:
            graphs, gev = capture_steps(step, stages)
            mode = "graph"
        except Exception as e:  # noqa: BLE001 -- any capture failure falls back to eager timing
            torch.cuda.synchronize()
            sys.stderr.write(f"CUDA graph capture failed ({e}); timing the step eagerly\n")
            graphs, gev = [], []
    if mode == "graph":
        for g in graphs:  # warm replays
            g.replay()
        torch.cuda.synchronize()
        assert rptq.rptq_device_error() == 0, "device error word set during the graph warm-up"
    else:
        ev = {n: [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
              for n, _, _ in stages}
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = Clocks(dev) if rank == 0 else None
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if clk:
        clk.start()
    t0.record()
    if mode == "graph":
        for i in range(args.steps):
            graphs[i % len(graphs)].replay()
    else:
        for i in range(args.steps):
            step.run({n: ev[n][i] for n in ev})
    t1.record()
    torch.cuda.synchronize()
    # the two headline kernels once more, launched back to back (inside the clock record)
    b2b = {n: back_to_back_ms(c, mode == "graph") for n, c in step.repeat_calls().items()}
    if clk:
        clk.end()
    if ws > 1:
        torch.distributed.barrier()
    clocks = clk.stop() if clk else None
    ms = pdist.max_over_ranks(t0.elapsed_time(t1), dev)
    step_bytes = sum(b for _, b, _ in stages)
    assert rptq.rptq_device_error() == 0, "device error word set during the timed steps"

    hbm, peak_kind = peaks()
    tpeak = tensor_peak()
    flops = stage_flops(w)
    kern = {}
    for n, b, launches in stages:
        if mode == "graph":  # each slot's events hold that slot's last replay
            per = [e[n][0].elapsed_time(e[n][1]) for e in gev[:min(len(gev), args.steps)]]
        else:
            per = [ev[n][i][0].elapsed_time(ev[n][i][1]) for i in range(args.steps)]
        mean_ms = sum(per) / len(per)
        kern[n] = {"ms_per_call": round(mean_ms, 4), "bytes_per_call": b, "gpu_launches_per_call": launches}
        if b:
            kern[n]["gbs"] = round(b / (mean_ms * 1e-3) / 1e9, 1)
            kern[n]["frac_of_measured_hbm"] = round(b / (mean_ms * 1e-3) / 1e9 / hbm, 4)
        if n in flops:
            # fp16 operands: the measured bf16 GEMM peak (same nominal tensor rate), burst figure
            kern[n]["flops_per_call"] = flops[n]
            kern[n]["tflops"] = round(flops[n] / (mean_ms * 1e-3) / 1e12, 1)
            kern[n]["frac_of_measured_tensor_peak"] = round(flops[n] / (mean_ms * 1e-3) / 1e12 / tpeak, 4)
    for n, t in b2b.items():
        b = kern[n]["bytes_per_call"]
        kern[n]["back_to_back"] = {"ms_per_launch": round(t, 4), "launches": B2B_LAUNCHES,
                                   "gbs": round(b / (t * 1e-3) / 1e9, 1),
                                   "frac_of_measured_hbm": round(b / (t * 1e-3) / 1e9 / hbm, 4)}
    # the headline: the metric's own kernel launched back to back over the full batch (its
    # in-step figure, with an event pair around each launch, is kernels[head]), the slowest
    # rank's time, bytes summed over ranks
    head = headline_stage(w)
    head_bytes = kern[head]["bytes_per_call"]
    value_in_step = pdist.sum_over_ranks(head_bytes, dev) / (
        pdist.max_over_ranks(kern[head]["ms_per_call"], dev) * 1e-3) / 1e9
    head_launch_ms = pdist.max_over_ranks(b2b.get(head, kern[head]["ms_per_call"]), dev)
    head_ms = head_launch_ms * args.steps
    value = pdist.sum_over_ranks(head_bytes, dev) / (head_launch_ms * 1e-3) / 1e9
    tokens = headline_tokens(w)
    kern[head]["mtokens_per_s"] = round(tokens / (kern[head]["ms_per_call"] * 1e-3) / 1e6, 2)
    # the longest stage of the path itself (the comparison stages -- the unfused baseline and the
    # unplanned fused launch -- are left out)
    dom = max((n for n, b, _ in stages if b and n not in COMPARISON_STAGES), key=lambda n: kern[n]["ms_per_call"])

    def roof(n):
        t = b2b.get(n, kern[n]["ms_per_call"])
        ach = kern[n]["bytes_per_call"] / (t * 1e-3) / 1e9
        return {"bound": "hbm", "kernel": n, "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(ach / hbm, 4), "peak_kind": peak_kind, "traffic": _traffic(n),
                "algorithmic_bytes_per_launch": kern[n]["bytes_per_call"],
                "launch_ms": round(t, 4),
                "launch_timing": (f"{B2B_LAUNCHES} launches back to back, one event pair around them" if n in b2b
                                  else "event pair around each call in the step")}

    launches = sum(l for _, _, l in stages) * args.steps
    e2e = run_e2e(step, args, dev, ws) if args.e2e_steps > 0 else None

    if rank == 0:
        cpu = cpu_baseline(w, args) if (ws == 1 and not args.no_cpu_baseline) else None
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded per-channel uniform ranges with outlier channels)",
            "config": workload_config(w),
            "headline_kernel": head,
            "value_in_step": round(value_in_step, 1),
            "headline_timing": (f"the headline kernel launched {B2B_LAUNCHES} times back to back over the full batch "
                                "(inputs larger than L2), one event pair around the run; value_in_step: the same kernel "
                                "inside the timed steps, an event pair around each launch"),
            "timing": {"mode": mode, "graph_slots": len(graphs),
                       "what": ("the step captured as CUDA graphs and replayed back to back; per-stage times from "
                                "timing-event nodes inside the graphs (the last replay of each slot)")
                       if mode == "graph" else "the step's calls issued eagerly, an event pair around each stage"},
            "mtokens_per_s": round(tokens * ws * args.steps / (head_ms * 1e-3) / 1e6, 3),
            "frac_of_measured_hbm": round(value / ws / hbm, 4),
            "step": {"what": "every stage of the path once: calibration, KMeans, the LayerNorm plan, fused quantization "
                             "(planned, and unplanned for comparison), the "
                             "explicit-reorder baseline, dynamic ranges, the reordered linear layer (weight "
                             "preparation, one 2048-token micro-batch), K/V quantization, dequantization, "
                             "one decode step (append, attention)",
                     "ms": round(ms / args.steps, 4),
                     "gbs": round(pdist.sum_over_ranks(step_bytes * args.steps, dev) / (ms * 1e-3) / 1e9, 1),
                     "frac_of_measured_hbm": round(step_bytes * args.steps / (ms * 1e-3) / 1e9 / hbm, 4),
                     "bytes": step_bytes},
            "roofline": roof(head),
            "roofline_step_dominant": roof(dom),
            "kernels": kern,
            "gpu_launches": launches,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def scaled_workload(args) -> W.Workload:
    """The named workload; with --token-scale f < 1 its token counts (T, calibration tokens,
    K/V sequence length) shrink by f -- a smaller case of the same kernels for ncu captures,
    never the configuration a bench number is quoted on."""
    w = W.WORKLOADS[args.workload]
    f = args.token_scale
    if f == 1.0:
        return w
    kv = w.kv and dataclasses.replace(w.kv, S=max(1, int(w.kv.S * f)))
    return dataclasses.replace(w, T=max(4, int(w.T * f)) if w.T else 0,
                               T_cal=max(4, int(w.T_cal * f)) if w.T_cal else 0, kv=kv,
                               name=f"{w.name} (tokens x{f:g}, profiling case)")


def workload_config(w):
    es = W.ESIZE
    ins = [(w.T_cal or w.T) * w.C * es[w.dtype], w.T * w.C * es[w.dtype]] if has_act(w) else []
    if w.kv:
        ins += [w.kv.elems * es[w.kv.dtype]] * 2
    streamed = sum(ins)
    if min(ins) > L2_BYTES:
        l2 = f"inputs larger than L2 (a step streams about {streamed / 1e9:.1f} GB of inputs), no flush needed"
    else:
        l2 = (f"some inputs fit in the 126 MB L2 (a step streams {streamed / 1e6:.0f} MB of inputs): "
              "stage times are partly L2-warm, not HBM numbers")
    c = {"workload": w.name, "tokens": w.T, "channels": w.C, "calib_tokens": w.T_cal or w.T,
         "g": w.g, "iters": w.iters, "bits": w.bits, "io_dtype": w.dtype, "l2": l2}
    if w.kv:
        k = w.kv
        c["kv"] = {"B": k.B, "H": k.H, "S": k.S, "D": k.D, "dtype": k.dtype, "g": k.g,
                   "iters": k.iters, "bits": k.bits}
    return c


E2E_CHUNKS = 8


def run_e2e(step: Step, args, dev, ws):
    """The headline call through the public API with host buffers: every step copies its input
    from pinned host memory, runs the call, and reads its codes back, all inside the timing
    (the calibration results of the timed steps are the call's tables).  The batch goes in
    E2E_CHUNKS chunks (token rows, or whole batch entries of the K/V cache) over three streams --
    upload, the call on the chunk, readback -- so the upload of one chunk overlaps the readback of
    the one before (the host link is full duplex); every byte still crosses the link once per
    step."""
    r, w = step.r, step.w
    main = torch.cuda.current_stream(dev)
    if step.act:
        ins, outs = [step.x], [step.codes]
        T = w.T
        nch = max(1, min(E2E_CHUNKS, T // 4))
        bounds = [(T * i // nch) // 4 * 4 for i in range(nch)] + [T]
    else:
        k = step.kvw
        ins, outs = [step.k, step.v], [step.kq, step.vq]
        nch = max(1, min(E2E_CHUNKS, k.B))  # chunks of whole batch entries
        bounds = [k.B * i // nch for i in range(nch)] + [k.B]
    h_in = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ins]
    for h, t in zip(h_in, ins):
        h.copy_(t)
    h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    bi = sum(t.numel() * t.element_size() for t in ins)
    bo = sum(t.numel() * t.element_size() for t in outs)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nch)]
    ev_k = [torch.cuda.Event() for _ in range(nch)]
    ev_out = [torch.cuda.Event() for _ in range(nch)]
    for e in ev_in + ev_k + ev_out:  # every event recorded once, so the first waits are valid
        e.record(main)

    def call(t0, t1):
        if step.act:
            r.rptq_ln_reorder_quant_planned(step.x[t0:t1], step.plan, w.bits, eps=w.eps, codes=step.codes[t0:t1])
        else:
            r.rptq_kv_quant(step.k[t0:t1], step.v[t0:t1], step.kmk["labels"], step.kmk["scale"], step.kmk["zero"],
                            step.kmv["labels"], step.kmv["scale"], step.kmv["zero"], k.bits,
                            k_codes=step.kq[t0:t1], v_codes=step.vq[t0:t1])

    def one():
        for c in range(nch):
            t0, t1 = bounds[c], bounds[c + 1]
            if t1 == t0:
                continue
            # upload: the chunk's rows are free once the previous step's call on them is done
            s_in.wait_event(ev_k[c])
            with torch.cuda.stream(s_in):
                for h, t in zip(h_in, ins):
                    t[t0:t1].copy_(h[t0:t1], non_blocking=True)
            ev_in[c].record(s_in)
            # the call: after the upload, and after the previous readback of the chunk's codes
            main.wait_event(ev_in[c])
            main.wait_event(ev_out[c])
            call(t0, t1)
            ev_k[c].record(main)
            # readback
            s_out.wait_event(ev_k[c])
            with torch.cuda.stream(s_out):
                for h, t in zip(h_out, outs):
                    h[t0:t1].copy_(t[t0:t1], non_blocking=True)
            ev_out[c].record(s_out)

    one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    a.record(main)
    s_in.wait_stream(main)
    s_out.wait_stream(main)
    for _ in range(args.e2e_steps):
        one()
    main.wait_stream(s_in)
    main.wait_stream(s_out)
    b.record(main)
    torch.cuda.synchronize()
    ms = pdist.max_over_ranks(a.elapsed_time(b), dev)
    nbytes = stage_bytes(w, headline_stage(w))
    total = pdist.sum_over_ranks(nbytes * args.e2e_steps, dev)
    return {"value": round(total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "steps": args.e2e_steps,
            "what": (f"{headline_stage(w)} through the C ABI with host buffers"
                     + (f", {nch} chunks ({'tokens' if step.act else 'batch entries'}) pipelined over upload / call / "
                        "readback streams" if nch > 1 else "")),
            "ms_per_step": round(ms / args.e2e_steps, 3), "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo}


def stage_bytes(w: W.Workload, name: str) -> int:
    return dict((n, b) for n, b, _ in stage_list(w))[name]


# ------------------------------------------------------------------------------------------
def host_cpu() -> dict:
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": os.cpu_count(), "cpu_model": model}


class OracleHeadline:
    """The CPU oracle on a bounded sample of the headline stage: the fused LN-reorder-quant of
    `n` tokens of the workload's batch (the oracle's own calibration on a small calibration
    sample gives its R, clusters, s and z), or the K/V quantization of `n` sequence positions of
    the K and V caches (calibrated on that sample).  Inputs are generated once, outside the
    timing; `run()` times one pass and returns the seconds."""

    def __init__(self, w: W.Workload, n: int):
        import oracle
        oracle.build()
        self.o, self.w = oracle, w
        gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
        if has_act(w):
            self.n = n = max(1, min(n, w.T))
            m = synthetic.channel_model(w.C, w.seed, w.outlier_frac, w.outlier_factor)
            self.gamma, self.beta = synthetic.ln_params(w.C, w.seed)
            xc = oracle._f32(synthetic.activations(256, m, w.seed, dtype=w.dtype, calibration=True,
                                                   device=gen_dev).cpu())
            mx, mn = oracle.minmax_ln(xc, self.gamma, self.beta, w.eps)
            self.cal = oracle.calibrate(mx, mn, w.g, w.iters, w.bits)
            self.x = oracle._f32(synthetic.activations(n, m, w.seed, dtype=w.dtype, device=gen_dev).cpu())
            self.nbytes = W.bytes_ln_quant(n, w.C, w.dtype, w.bits)
            self.desc = (f"oracle fused LN-reorder-quant (LayerNorm, gather through R, quantize, pack) of {n} of "
                         f"the {w.T} tokens, single-threaded")
        else:
            k = w.kv
            self.n = n = max(1, min(n, k.S))
            self.kv = []
            for tag, which in ((1, "k"), (2, "v")):
                mk = synthetic.channel_model(k.channels, w.seed, k.outlier_frac, k.outlier_factor, tag=tag)
                kvf = oracle._f32(synthetic.kv_cache(k.B, k.H, n, k.D, mk, w.seed, which, k.dtype,
                                                    device=gen_dev).cpu())
                flat = kvf.transpose(0, 2, 1, 3).reshape(-1, k.channels)
                mx, mn = oracle.minmax(flat)
                self.kv.append((kvf, oracle.calibrate(mx, mn, k.g, k.iters, k.bits)))
            self.nbytes = W.bytes_kv_quant(k.B * k.H * n * k.D, k.dtype, k.bits)
            self.desc = f"oracle K/V quantization of {n} of the {k.S} sequence positions of K and V, single-threaded"

    def run(self) -> float:
        o, w = self.o, self.w
        t = time.perf_counter()
        if has_act(w):
            c = self.cal
            o.ln_reorder_quant(self.x, self.gamma, self.beta, c["R"], c["col_cluster"], c["scale"], c["zero"],
                               w.bits, eps=w.eps)
        else:
            for kvf, c in self.kv:
                o.kv_quant(kvf, c["labels"], c["scale"], c["zero"], w.kv.bits)
        return time.perf_counter() - t


def oracle_units_for(w: W.Workload, seconds: float) -> int:
    """Sample size (tokens, or K/V positions) the oracle processes in about `seconds`."""
    probe = OracleHeadline(w, 16)
    probe.run()
    per = probe.run() / probe.n
    full = w.T if has_act(w) else w.kv.S
    return int(max(1, min(full, seconds / max(per, 1e-9))))


def cpu_baseline(w, args):
    smp = OracleHeadline(w, oracle_units_for(w, args.cpu_seconds))
    secs = smp.run()
    return {"value": round(smp.nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": smp.desc, "seconds": round(secs, 2), **host_cpu()}


def run_reference(args):
    """The reference arm: the oracle on the host cores, each step one bounded sample of the
    headline stage, sized so the whole --steps K --warmup W run takes about --ref-budget-s."""
    rank, ws, _ = pdist.world()
    if rank != 0:
        return  # under torchrun only rank 0 runs the CPU reference
    w = W.WORKLOADS[args.workload]
    per_step = args.ref_budget_s / max(1, args.steps + args.warmup)
    smp = OracleHeadline(w, oracle_units_for(w, per_step))
    for _ in range(args.warmup):
        smp.run()
    secs = [smp.run() for _ in range(args.steps)]
    total = sum(secs)
    value = smp.nbytes * args.steps / total / 1e9
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w), "impl": "reference",
            "headline_kernel": headline_stage(w),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": smp.desc + " per step", **host_cpu()},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def relaunch(n: int) -> int:
    """Run this command again as n ranks under torchrun (one process per GPU) and return its
    exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["rptq", "reference"], default="rptq")
    ap.add_argument("--workload", choices=W.ORDER, default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="about how long the CPU oracle's baseline sample runs")
    ap.add_argument("--ref-budget-s", type=float, default=120.0,
                    help="target seconds of host work for the whole --impl reference run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="issue the timed steps call by call instead of replaying CUDA graphs of the step")
    ap.add_argument("--token-scale", type=float, default=1.0,
                    help="shrink the token counts (a small case for ncu captures; not a bench config)")
    ap.add_argument("--no-clock-warmup", action="store_true",
                    help="no effect (the in-process clock sampler needs no warm-up steps)")
    ap.add_argument("--dry-run", action="store_true",
                    help="print this rank's place in the launch and exit (checks the multi-process plumbing)")
    args = ap.parse_args()
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(relaunch(args.gpus))  # one process per GPU
    rank, ws, local = pdist.world()
    if ws != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but the launcher started {ws} ranks", file=sys.stderr)
        sys.exit(2)
    if args.dry_run:
        print(json.dumps({"rank": rank, "world_size": ws, "local_rank": local, "impl": args.impl}), flush=True)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_rptq(args)


if __name__ == "__main__":
    main()
