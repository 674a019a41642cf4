#!/usr/bin/env python
"""Benchmark of the RPTQ data path on B200; rank 0 prints one JSON line.

A step is one pass of the whole path over one synthetic batch of the workload:
  1. calibration statistics of LayerNorm(x) over the calibration batch   (rptq_calib_minmax)
  2. KMeans -> reorder index R and per-cluster (s, z)                    (rptq_kmeans)
  3. reorder-fused LayerNorm + per-cluster quantization of the batch      (rptq_ln_reorder_quant)
  4. K/V calibration statistics, KMeans for K and for V                   (rptq_kv_calib_minmax, rptq_kmeans)
  5. K/V cache quantization                                               (rptq_kv_quant)
  6. dequantization of the activation codes and of the K/V codes         (rptq_dequant)
`value` is the whole-job algorithmic GB/s: the bytes every stage must move (see
post_activation_quantization_b200/workloads.py) summed over ranks, divided by the slowest
rank's device time for the K timed steps.  Inputs are larger than the 126 MB L2, so no flush
is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl rptq|reference]
Multi-GPU: launched by torchrun, one process per GPU, weak scaling (every rank its own batch);
the calibration statistics are combined with one MAX/MIN all-reduce (NCCL).
"""
from __future__ import annotations

import argparse
import csv
import dataclasses
import datetime
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
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


def has_act(w: W.Workload) -> bool:
    """Whether the workload carries the activation path (the K/V-only workload does not)."""
    return w.T > 0 and w.C > 0


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
        st += [("ln_reorder_quant", W.bytes_ln_quant(w.T, w.C, w.dtype, w.bits), 1)]
    if k:
        st += [("kv_quant", W.bytes_kv_quant(k.elems, k.dtype, k.bits), 1)]
    if a:
        st += [("dequant_act", W.bytes_dequant(n, w.dtype, w.bits), 1)]
    if k:
        st += [("dequant_kv", 2 * W.bytes_dequant(k.elems, k.dtype, k.bits), 2)]
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
            self.xhat = torch.empty((w.T, w.C), dtype=dt, device=device)
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
            kvdt = synthetic.torch_dtype(k.dtype)
            self.khat = torch.empty((k.B, k.H, k.S, k.D), dtype=kvdt, device=device)
            self.vhat = torch.empty_like(self.khat)
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
            mark("ln_reorder_quant", 0)
            r.rptq_ln_reorder_quant(self.x, self.gamma, self.beta, self.km["R"], self.km["col_cluster"],
                                    self.km["scale"], self.km["zero"], w.bits, eps=w.eps, codes=self.codes)
            mark("ln_reorder_quant", 1)
        if k:
            mark("kv_quant", 0)
            r.rptq_kv_quant(self.k, self.v, self.kmk["labels"], self.kmk["scale"], self.kmk["zero"],
                            self.kmv["labels"], self.kmv["scale"], self.kmv["zero"], k.bits,
                            k_codes=self.kq, v_codes=self.vq)
            mark("kv_quant", 1)
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


# ------------------------------------------------------------------------------------------
class Clocks:
    """nvidia-smi samples every 100 ms; only those taken inside the timed region are kept."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.t0 = self.t1 = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def start(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    def stop(self) -> dict:
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = []
        for r in csv.reader(io.StringIO(self.f.read())):
            if len(r) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            if self.t0 is not None and self.t0 <= ts <= self.t1:
                rows.append([x.strip() for x in r[1:]])
        os.unlink(self.f.name)
        num = lambda v: v.replace(".", "", 1).isdigit()  # noqa: E731
        sm = [float(r[1]) for r in rows if num(r[1])]
        mx = [float(r[2]) for r in rows if num(r[2])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if "Active" in v and "Not" not in v})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(rows), "reasons": reasons}


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
def run_rptq(args):
    rank, ws, local = pdist.world()
    if ws > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", device_id=torch.device("cuda", local),
                                             timeout=__import__("datetime").timedelta(seconds=120))
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
    # untimed steps while the clock sampler starts (every rank runs the same number)
    n_pre = int(pdist.max_over_ranks(min(2000, int(0.5 / max(tw, 1e-4)) + 1), dev))

    ev = {n: [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
          for n, _, _ in stages}
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = Clocks(dev.index) if rank == 0 else None
    for _ in range(n_pre if args.clock_warmup else 0):  # the sampler starts while these run
        step.run()
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if clk:
        clk.start()
    t0.record()
    for i in range(args.steps):
        step.run({n: ev[n][i] for n in ev})
    t1.record()
    torch.cuda.synchronize()
    if clk:
        clk.end()
    if ws > 1:
        torch.distributed.barrier()
    clocks = clk.stop() if clk else None
    ms_rank = t0.elapsed_time(t1)
    ms = pdist.max_over_ranks(ms_rank, dev)
    step_bytes = sum(b * 1 for _, b, _ in stages)
    total_bytes = pdist.sum_over_ranks(step_bytes * args.steps, dev)
    value = total_bytes / (ms * 1e-3) / 1e9
    assert rptq.rptq_device_error() == 0, "device error word set during the timed steps"

    hbm, peak_kind = peaks()
    kern = {}
    for n, b, launches in stages:
        per = [ev[n][i][0].elapsed_time(ev[n][i][1]) for i in range(args.steps)]
        mean_ms = sum(per) / len(per)
        kern[n] = {"ms_per_call": round(mean_ms, 4), "bytes_per_call": b,
                   "gpu_launches_per_call": launches}
        if b:
            kern[n]["gbs"] = round(b / (mean_ms * 1e-3) / 1e9, 1)
            kern[n]["frac_of_measured_hbm"] = round(b / (mean_ms * 1e-3) / 1e9 / hbm, 4)
    # tokens of the step: the activation batch, or the cache's B*S positions for the K/V-only workload
    tok_stage, tokens = ("ln_reorder_quant", w.T) if step.act else ("kv_quant", w.kv.B * w.kv.S)
    kern[tok_stage]["mtokens_per_s"] = round(tokens / (kern[tok_stage]["ms_per_call"] * 1e-3) / 1e6, 2)
    dom = max((n for n, b, _ in stages if b), key=lambda n: kern[n]["ms_per_call"])
    dom_bytes = kern[dom]["bytes_per_call"]
    ach = dom_bytes / (kern[dom]["ms_per_call"] * 1e-3) / 1e9
    launches = sum(l for _, _, l in stages) * args.steps

    e2e = run_e2e(step, args, dev, step_bytes, ws) if args.e2e_steps > 0 else None

    if rank == 0:
        cpu = cpu_baseline(w, args) if (ws == 1 and not args.no_cpu_baseline) else None
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded per-channel uniform ranges with outlier channels)",
            "config": workload_config(w),
            "mtokens_per_s": round(tokens * ws * args.steps / (ms * 1e-3) / 1e6, 3),
            "frac_of_measured_hbm": round(value / ws / hbm, 4),
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(ach / hbm, 4), "peak_kind": peak_kind,
                         "traffic": _traffic(dom), "algorithmic_bytes_per_launch": dom_bytes},
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


def run_e2e(step: Step, args, dev, step_bytes, ws):
    """Same step through the public API with host inputs: each step copies its inputs from
    pinned host memory and reads the codes (and calibration results) back, inside the timing."""
    ins = ([step.xcal, step.x] if step.act else []) + ([step.k, step.v] if step.kvw else [])
    outs = ([step.codes] if step.act else []) + ([step.kq, step.vq] if step.kvw else [])
    outs += [step.km["R"], step.km["scale"], step.km["zero"]] if step.act else \
        [step.kmk["labels"], step.kmk["scale"], step.kmk["zero"]]
    h_in = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in ins]
    for h, t in zip(h_in, ins):
        h.copy_(t)
    h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    bi = sum(t.numel() * t.element_size() for t in ins)
    bo = sum(t.numel() * t.element_size() for t in outs)

    def one():
        for h, t in zip(h_in, ins):
            t.copy_(h, non_blocking=True)
        step.run()
        for h, t in zip(h_out, outs):
            h.copy_(t, non_blocking=True)

    one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    a.record()
    for _ in range(args.e2e_steps):
        one()
    b.record()
    torch.cuda.synchronize()
    ms = pdist.max_over_ranks(a.elapsed_time(b), dev)
    total = pdist.sum_over_ranks(step_bytes * args.e2e_steps, dev)
    return {"value": round(total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "steps": args.e2e_steps,
            "ms_per_step": round(ms / args.e2e_steps, 3), "h2d_bytes_per_step": bi,
            "d2h_bytes_per_step": bo}


# ------------------------------------------------------------------------------------------
class OracleSample:
    """The CPU oracle on a bounded sample of one step: `frac` of the tokens of every
    token-parallel stage (inputs generated once, outside the timing), the three KMeans problems
    in full.  `time_tokens()` times the token-parallel stages once; `time_kmeans()` the KMeans
    problems (deterministic: the same inputs give the same work every time)."""

    def __init__(self, w: W.Workload, frac: float):
        import numpy as np

        import oracle
        oracle.build()
        self.o, self.w = oracle, w
        gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
        self.act = has_act(w)
        self.desc = "oracle (1 core)"
        if self.act:
            m = synthetic.channel_model(w.C, w.seed, w.outlier_frac, w.outlier_factor)
            self.gamma, self.beta = synthetic.ln_params(w.C, w.seed)
            self.t_cal = max(4, int((w.T_cal or w.T) * frac))
            self.t_x = max(4, int(w.T * frac))
            self.xc = [oracle._f32(synthetic.activations(min(4096, self.t_cal - r0), m, w.seed + r0, dtype=w.dtype,
                                                        calibration=True, device=gen_dev).cpu())
                       for r0 in range(0, self.t_cal, 4096)]
            self.x = oracle._f32(synthetic.activations(self.t_x, m, w.seed, dtype=w.dtype, device=gen_dev).cpu())
            mx = mn = None
            for xc in self.xc:
                mx, mn = oracle.minmax_ln(xc, self.gamma, self.beta, w.eps, ch_max=mx, ch_min=mn)
            self.mx, self.mn = mx, mn
            self.desc += f" on {self.t_cal} calibration tokens and {self.t_x} tokens of the batch"
        self.desc += ", full KMeans"
        self.kv = []
        if w.kv:
            k = w.kv
            self.s_s = max(1, int(k.S * frac))
            for tag, which in ((1, "k"), (2, "v")):
                mk = synthetic.channel_model(k.channels, w.seed, k.outlier_frac, k.outlier_factor, tag=tag)
                kvf = oracle._f32(synthetic.kv_cache(k.B, k.H, self.s_s, k.D, mk, w.seed, which, k.dtype,
                                                    device=gen_dev).cpu())
                flat = np.ascontiguousarray(kvf.transpose(0, 2, 1, 3).reshape(-1, k.channels))
                kmx, kmn = oracle.minmax(flat)
                self.kv.append((kvf, flat, kmx, kmn))
            self.desc += f", K and V with {self.s_s} of {k.S} sequence positions"
        self.desc += "; stage times scaled to the full step"
        self.cal = oracle.calibrate(self.mx, self.mn, w.g, w.iters, w.bits) if self.act else None
        self.kcal = [oracle.calibrate(kmx, kmn, w.kv.g, w.kv.iters, w.kv.bits) for _, _, kmx, kmn in self.kv]

    def bytes_per_step(self) -> int:
        w = self.w
        n = 0
        if self.act:
            n += W.bytes_calib(w.T_cal or w.T, w.C, w.dtype) + W.bytes_ln_quant(w.T, w.C, w.dtype, w.bits) \
                + W.bytes_dequant(w.T * w.C, w.dtype, w.bits)
        if w.kv:
            k = w.kv
            n += 2 * W.bytes_calib(k.B * k.S, k.channels, k.dtype) + \
                W.bytes_kv_quant(k.elems, k.dtype, k.bits) + 2 * W.bytes_dequant(k.elems, k.dtype, k.bits)
        return n

    def time_kmeans(self) -> float:
        o, w = self.o, self.w
        t = time.perf_counter()
        if self.act:
            o.calibrate(self.mx, self.mn, w.g, w.iters, w.bits)
        for _, _, kmx, kmn in self.kv:
            o.calibrate(kmx, kmn, w.kv.g, w.kv.iters, w.kv.bits)
        return time.perf_counter() - t

    def time_tokens(self) -> float:
        """Seconds the token-parallel stages of a full step take, scaled from the sample."""
        o, w, cal = self.o, self.w, self.cal
        secs = 0.0
        if self.act:
            t = time.perf_counter()
            for xc in self.xc:
                o.minmax_ln(xc, self.gamma, self.beta, w.eps)
            secs += (time.perf_counter() - t) / (self.t_cal / (w.T_cal or w.T))
            t = time.perf_counter()
            packed, _, _ = o.ln_reorder_quant(self.x, self.gamma, self.beta, cal["R"], cal["col_cluster"],
                                              cal["scale"], cal["zero"], w.bits, eps=w.eps)
            q = o.unpack(packed, w.C, w.bits)
            o.dequant(q, cal["col_cluster"], cal["scale"], cal["zero"])
            secs += (time.perf_counter() - t) / (self.t_x / w.T)
        if w.kv:
            k = w.kv
            t = time.perf_counter()
            for (kvf, flat, _, _), kc in zip(self.kv, self.kcal):
                o.minmax(flat)
                pk = o.kv_quant(kvf, kc["labels"], kc["scale"], kc["zero"], k.bits)
                o.kv_dequant(pk, k.D, kc["labels"], kc["scale"], kc["zero"], k.bits)
            secs += (time.perf_counter() - t) / (self.s_s / k.S)
        return secs


def cpu_baseline(w, args):
    smp = OracleSample(w, args.cpu_frac)
    secs = smp.time_tokens() + smp.time_kmeans()
    return {"value": round(smp.bytes_per_step() / secs / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": smp.desc, "seconds_per_step_extrapolated": round(secs, 2)}


def run_reference(args):
    """The reference arm: the oracle on the host, one bounded sample per step.  The sample size
    keeps the whole --steps K --warmup W run near `--ref-budget-s` seconds; the three KMeans
    problems (deterministic, the same work each step) are timed once and counted in every step."""
    rank, ws, _ = pdist.world()
    if rank != 0:
        return  # under torchrun only rank 0 runs the CPU reference
    w = W.WORKLOADS[args.workload]
    probe = OracleSample(w, 1 / 256)
    t0 = time.perf_counter()
    probe.time_tokens()
    per_frac = (time.perf_counter() - t0) * 256  # seconds of token work per full-step fraction 1
    per_step = args.ref_budget_s / max(1, args.steps + args.warmup)
    frac = min(args.ref_frac, max(1 / 4096, per_step / max(per_frac, 1e-9)))
    smp = OracleSample(w, frac)
    km_secs = smp.time_kmeans()
    for _ in range(args.warmup):
        smp.time_tokens()
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(smp.bytes_per_step() / (smp.time_tokens() + km_secs) / 1e9)
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    nbytes = smp.bytes_per_step()
    line = {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(nbytes / (value * 1e9) * 1e3, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w), "impl": "reference",
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": smp.desc + f" (token fraction {frac:.5f}; KMeans timed once)",
                             "wall_s": round(wall, 1)},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["rptq", "reference"], default="rptq")
    ap.add_argument("--workload", choices=W.ORDER, default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-frac", type=float, default=1 / 2,
                    help="fraction of the tokens the CPU oracle processes for its baseline")
    ap.add_argument("--ref-frac", type=float, default=1 / 32,
                    help="largest fraction of the tokens per step of the --impl reference arm")
    ap.add_argument("--ref-budget-s", type=float, default=120.0,
                    help="target seconds of host work for the whole --impl reference run")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clock-warmup", dest="clock_warmup", action="store_false",
                    help="skip the untimed steps that let the clock sampler start (profiling runs)")
    ap.add_argument("--token-scale", type=float, default=1.0,
                    help="shrink the token counts (a small case for ncu captures; not a bench config)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_rptq(args)


if __name__ == "__main__":
    main()
