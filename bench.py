#!/usr/bin/env python3
"""Benchmark of the Swin3D shifted-window attention hot path on B200.

Headline step (the workload the metric is quoted on): one pass of the whole path over the
Aurora 0.25-degree encoder stage-1 grid (B=1, grid 4x180x360, C=512 = 8 heads x 64,
window (2,6,12)):

    window attention, shift (0,0,0)  -> AdaLN + residual (fp32 residual stream, in place)
    window attention, shift (1,3,6)  -> AdaLN + residual

Each attention call reads its own seeded bf16 Q/K/V (N(0,1)); the AdaLN calls take the
attention output, per-sample FiLM scale/shift N(0,0.1) and the fp32 residual stream.  Every
input tensor is larger than the 126 MB L2, so no flush is needed between steps.

``value`` is windows per second over all ranks (each step processes 2 x 1800 windows of 8
heads per rank).  Besides the headline the JSON line carries:

* ``attn`` / ``adaln``: per-launch statistics of the two kernels inside the timed region;
* ``roofline``: the binding roofline of the attention kernel, max(bytes/BW, FLOPs/peak),
  with the DRAM traffic of the committed ncu capture while it still matches the code;
* ``configs``: the other workloads of the set, each timed on its own (N=1 only): the tiny
  grid, stage 2 with AdaLN at C=1024, stage 3 with padding, the six-block stage-1 stack at
  B=4, each with its algorithmic bytes, FLOPs and roofline fraction;
* ``e2e``: the headline step through the public API with pinned host buffers;
* ``cpu_baseline``: the fp64 oracle on the host cores, on bounded samples of the same
  workloads (rank 0, N=1).

``--impl reference`` times the fp64 CPU oracle on samples of the headline workload as the
reference arm (same sampler as ``cpu_baseline``).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WINDOW = (2, 6, 12)
N_TOK = WINDOW[0] * WINDOW[1] * WINDOW[2]
UNSHIFTED, SHIFTED = (0, 0, 0), (1, 3, 6)
SHIFTS = (UNSHIFTED, SHIFTED)

# The benchmark set: grid, heads x head_dim.  "stage1" is the headline workload.
WORKLOADS = {
    "tiny": dict(B=1, T=2, H=15, W=30, heads=2, hd=32),
    "stage1": dict(B=1, T=4, H=180, W=360, heads=8, hd=64),
    "stage2": dict(B=1, T=4, H=90, W=180, heads=16, hd=64),
    "stage3_padded": dict(B=2, T=4, H=45, W=90, heads=32, hd=64),
    "stack_b4": dict(B=4, T=4, H=180, W=360, heads=8, hd=64),
}
STACK_BLOCKS = 6
METRIC = "window-attn TFLOP/s, HBM GB/s & % of roofline on 1 B200; windows/s"
WORKLOAD = ("Aurora 0.25deg encoder stage 1: B=1, grid T4xH180xW360, C=512 (8 heads x 64), window (2,6,12); "
            "per step: attn shift (0,0,0) + AdaLN fp32-out, attn shift (1,3,6) + AdaLN fp32-out")
PROFILE = os.path.join("profiles", "window_attn_tc_stage1.json")
KERNEL_SOURCES = [os.path.join("swin3d_window_attention_b200", "csrc", f)
                  for f in ("attn_tcgen05.cu", "attn_common.cuh", "sm100_ptx.cuh", "s3w_common.cuh")]


def geometry(w, window=WINDOW):
    """Derived sizes of a workload: channels, tokens, windows (all samples)."""
    C = w["heads"] * w["hd"]
    tokens = w["B"] * w["T"] * w["H"] * w["W"]
    windows = w["B"] * math.prod(-(-d // a) for d, a in zip((w["T"], w["H"], w["W"]), window))
    return C, tokens, windows


def attn_bytes(w, o_bytes=2, in_bytes=2):
    """Read Q, K, V once and write O once: padding and the shift never touch HBM."""
    C, tokens, _ = geometry(w)
    return (3 * in_bytes + o_bytes) * tokens * C


def attn_flops(w, window=WINDOW):
    """4 N^2 d per (window, head): QK^T and PV, dense inside each window."""
    _, _, windows = geometry(w, window)
    n = math.prod(window)
    return windows * w["heads"] * 4 * n * n * w["hd"]


def fused_bytes(w, out_bytes=4):
    """The fused attention + AdaLN call: Q, K, V, the fp32 residual and the output once each;
    the attention output never leaves the chip (its bf16 copy goes through a per-CTA
    workspace of 2 windows that stays in L2)."""
    C, tokens, _ = geometry(w)
    return tokens * C * (3 * 2 + 4 + out_bytes)


def adaln_bytes(w, x_bytes=2, out_bytes=4):
    """x, the fp32 residual and the output, once each (scale/shift are negligible)."""
    C, tokens, _ = geometry(w)
    return tokens * C * (x_bytes + 4 + out_bytes)


S1 = WORKLOADS["stage1"]
C1, L1, N_WIN = geometry(S1)
ATTN_BYTES, ATTN_FLOPS, ADALN_BYTES = attn_bytes(S1), attn_flops(S1), adaln_bytes(S1)
CONFIG = {"workload": WORKLOAD, "global_batch": S1["B"], "windows_per_call": N_WIN, "heads": S1["heads"],
          "head_dim": S1["hd"], "l2": "inputs larger than L2 (265 MB per tensor), no flush",
          "parallelism": "single GPU"}


def config_for(world):
    c = dict(CONFIG)
    c["global_batch"] = S1["B"] * world
    if world > 1:
        c["parallelism"] = f"replicas x{world}"
    return c


def reduce_max_over_ranks(torch, dist, values, device):
    """Element-wise max over the ranks of a list of floats: the slowest rank's time, and any
    rank's error flag.  Every rank calls it at the same points, error or not, so that no rank
    is left waiting in a collective; without a process group it returns the values."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def load_peaks():
    """Measured peaks of this machine's B200s if the driver wrote them, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def roofline(nbytes, flops, ms, peaks):
    """Binding roofline: the larger of bytes/BW and FLOPs/peak; frac = that time / measured."""
    t = ms * 1e-3
    t_bw = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    if t_bw >= t_tc:
        r = {"bound": "hbm", "achieved": nbytes / t / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": t_bw / t}
    else:
        r = {"bound": "tensor", "achieved": flops / t / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
             "frac": t_tc / t}
    r["frac_of_nominal_8tbs"] = nbytes / t / 8e12
    r["tensor_frac"] = flops / t / 1e12 / peaks["bf16_tflops"]
    return r


def code_sha256(text):
    """sha256 of source code with comments and blank lines removed, so that editing a
    comment does not separate a capture from the code it measured."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln.strip()).encode()).hexdigest()


def kernel_code_sha256(root=None):
    """Code hash of the attention kernel's translation unit (kernel source + its headers)."""
    root = ROOT if root is None else root
    return code_sha256("\n".join(open(os.path.join(root, f)).read() for f in KERNEL_SOURCES))


def recorded_profile(root=None):
    """The committed ncu capture of the attention kernel, or None if its code changed since."""
    root = ROOT if root is None else root
    p = os.path.join(root, PROFILE)
    if not os.path.exists(p):
        return None
    try:
        prof = json.load(open(p))
        if prof.get("code_sha256") != kernel_code_sha256(root):
            return None
        return prof
    except (OSError, ValueError, KeyError):
        return None


def recorded_traffic(root=None):
    """DRAM bytes per attention launch (read + write) from the committed capture, or None."""
    prof = recorded_profile(root)
    if prof is None:
        return None
    return int(prof["dram_bytes_read"]) + int(prof["dram_bytes_write"])


def launch_stats(ms):
    s = sorted(ms)
    q = lambda f: s[min(len(s) - 1, int(f * len(s)))]
    return {"avg_launch_ms": statistics.fmean(s), "median_ms": statistics.median(s), "p10_ms": q(0.1),
            "p90_ms": q(0.9), "min_ms": s[0], "max_ms": s[-1], "launches": len(s)}


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while the timed region runs: NVML
    read every 5 ms from a thread (nvidia-smi at 50 ms if NVML is unavailable).  Read-only."""

    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []
        self.source = None

    def _nvml_handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.dev)
        bus = getattr(p, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(p, "pci_domain_id", 0)
            devid = getattr(p, "pci_device_id", 0)
            return pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{devid:02x}.0")
        return pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        import threading

        try:
            import pynvml

            h = self._nvml_handle()
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.stop_evt = threading.Event()

            def run():
                while not self.stop_evt.is_set():
                    try:
                        self.rows.append((time.time(), float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                          float(mx), int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except Exception:
                        pass
                    self.stop_evt.wait(0.005)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            self.source = "nvml 5 ms"
            return
        except Exception:
            self.thread = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi 50 ms"
        except (OSError, FileNotFoundError):
            self.proc = None

    def _smi_rows(self):
        import datetime

        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            try:
                bits = sum(self.REASON_BITS[nm] for nm, val in zip(names, f[6:10]) if val.lower() == "active")
                rows.append((ts, float(f[2]), float(f[3]), bits))
            except ValueError:
                continue
        os.unlink(self.path)
        return rows

    def stop(self, window=None):
        """Median SM clock and the throttle reasons seen; with window = (t0, t1) in epoch
        seconds only the samples taken inside it count (all of them if none is)."""
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            rows = list(self.rows)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            rows = self._smi_rows()
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        inside = [r for r in rows if window and (r[0] is None or window[0] <= r[0] <= window[1])]
        use = inside or rows
        reasons = sorted({nm for _, _, _, bits in use for nm, bit in self.REASON_BITS.items() if bits & bit})
        sm = [r[1] for r in use]
        mx = [r[2] for r in use]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "samples_in_timed_region": len(inside), "source": self.source,
                "reasons": reasons}


# ----------------------------------------------------------------------------- GPU arm
def device_qkv(torch, w, dev, base):
    """Seeded bf16 Q, K, V of a workload, drawn on the device."""
    from swin3d_window_attention_b200 import inputs

    C = w["heads"] * w["hd"]
    shape = (w["B"], w["T"], w["H"], w["W"], C)
    return [inputs.normal_bf16_torch(shape, dev, tensor_index=base + j) for j in range(3)]


def inputs_f32(torch, w, dev, index):
    """A seeded fp32 grid tensor of a workload (the TF32_ACC_FP32 mode's inputs), on the device."""
    from swin3d_window_attention_b200 import inputs

    C, tokens, _ = geometry(w)
    return inputs.normal_f32_torch(tokens * C, dev, tensor_index=index).reshape(w["B"], w["T"], w["H"], w["W"], C)


def device_film(torch, w, dev, base, sigma):
    from swin3d_window_attention_b200 import inputs

    C, tokens, _ = geometry(w)
    sc = inputs.normal_f32_torch(w["B"] * C, dev, tensor_index=base, sigma=sigma).reshape(w["B"], C)
    sh = inputs.normal_f32_torch(w["B"] * C, dev, tensor_index=base + 1, sigma=sigma).reshape(w["B"], C)
    res = inputs.normal_f32_torch(tokens * C, dev, tensor_index=base + 2).reshape(w["B"], tokens // w["B"], C)
    return sc, sh, res


def timed(torch, stream, fn, reps, warmup=3):
    """Per-call device times (ms) of fn, CUDA events on the launching stream."""
    for _ in range(warmup):
        fn()
    ev = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        ev.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def bench_configs(torch, s3w, dev, stream, peaks, reps, only=None):
    """Every workload of the set besides the headline, each timed on its own (or only the one
    named by ``only``)."""

    def want(name):
        return only is None or only == name

    out = {}
    launches = 0
    if want("tiny"):
        # tiny grid: launch-bound, latency reported
        w = WORKLOADS["tiny"]
        q, k, v = device_qkv(torch, w, dev, 900)
        o = torch.empty_like(q)
        ms = timed(torch, stream, lambda: s3w.swin3d_window_attn_fwd(q, k, v, o, w["heads"], w["hd"], WINDOW, SHIFTED),
                   reps)
        launches += len(ms)
        out["tiny"] = {"grid": "B=1 T2xH15xW30 (padded 2x18x36), 2 heads x 32, shift (1,3,6), 9 windows",
                       "attn": launch_stats(ms), "latency_us_median": 1e3 * statistics.median(ms)}
        del q, k, v, o

    if want("stage2"):
        # stage 2: shifted attention + AdaLN at C = 1024
        w = WORKLOADS["stage2"]
        C, tokens, windows = geometry(w)
        q, k, v = device_qkv(torch, w, dev, 910)
        sc, sh, res = device_film(torch, w, dev, 920, 0.1)
        o = torch.empty_like(q)
        ms_a = timed(torch, stream, lambda: s3w.swin3d_window_attn_fwd(q, k, v, o, w["heads"], w["hd"], WINDOW, SHIFTED),
                     reps)
        x = o.view(w["B"], tokens // w["B"], C)
        ms_n = timed(torch, stream, lambda: s3w.adaln_residual_fwd(x, res, sc, sh, res, eps=1e-5), reps)
        launches += len(ms_a) + len(ms_n)
        a_med, n_med = statistics.median(ms_a), statistics.median(ms_n)
        out["stage2"] = {"grid": "B=1 T4xH90xW180, 16 heads x 64, shift (1,3,6), 450 windows; AdaLN C=1024 fp32 out",
                         "attn": {**launch_stats(ms_a), "bytes": attn_bytes(w), "flops": attn_flops(w),
                                  "windows_per_s": windows / (a_med * 1e-3),
                                  "roofline": roofline(attn_bytes(w), attn_flops(w), a_med, peaks)},
                         "adaln": {**launch_stats(ms_n), "bytes": adaln_bytes(w),
                                   "roofline": roofline(adaln_bytes(w), 0, n_med, peaks)}}
        del q, k, v, o, x, sc, sh, res

    if want("stage3_padded"):
        # stage 3: padded grid (45 -> 48, 90 -> 96), padded keys masked, padded outputs dropped
        w = WORKLOADS["stage3_padded"]
        _, _, windows = geometry(w)
        q, k, v = device_qkv(torch, w, dev, 930)
        o = torch.empty_like(q)
        ms_a = timed(torch, stream, lambda: s3w.swin3d_window_attn_fwd(q, k, v, o, w["heads"], w["hd"], WINDOW, SHIFTED),
                     reps)
        launches += len(ms_a)
        a_med = statistics.median(ms_a)
        out["stage3_padded"] = {
            "grid": "B=2 T4xH45xW90 (padded 4x48x96), 32 heads x 64, shift (1,3,6), 256 windows",
            "attn": {**launch_stats(ms_a), "bytes": attn_bytes(w), "flops": attn_flops(w),
                     "windows_per_s": windows / (a_med * 1e-3),
                     "roofline": roofline(attn_bytes(w), attn_flops(w), a_med, peaks)}}
        del q, k, v, o

    if want("stage1_tf32"):
        # TF32_ACC_FP32 mode on the stage-1 grid: fp32 Q/K/V in, fp32 O out
        w = WORKLOADS["stage1"]
        C, tokens, windows = geometry(w)
        q, k, v = (inputs_f32(torch, w, dev, 940 + j) for j in range(3))
        o = torch.empty_like(q)
        ms_a = timed(torch, stream, lambda: s3w.swin3d_window_attn_fwd(q, k, v, o, w["heads"], w["hd"], WINDOW, SHIFTED),
                     reps)
        launches += len(ms_a)
        a_med = statistics.median(ms_a)
        nbytes = attn_bytes(w, o_bytes=4, in_bytes=4)
        out["stage1_tf32"] = {
            "grid": "B=1 T4xH180xW360, 8 heads x 64, shift (1,3,6), 1800 windows; fp32 Q/K/V/O, TF32 MMAs (TF32_ACC_FP32)",
            "attn": {**launch_stats(ms_a), "bytes": nbytes, "flops": attn_flops(w), "windows_per_s": windows / (a_med * 1e-3),
                     "roofline": roofline(nbytes, attn_flops(w), a_med,
                                          {**peaks, "bf16_tflops": peaks["bf16_tflops"] / 2})}}
        del q, k, v, o

    if want("stage1_window_2x12x12"):
        # windows larger than one tile: the streaming path on the stage-1 grid with (2,12,12)
        # windows (N = 288), shift (1,6,6)
        w = WORKLOADS["stage1"]
        big = (2, 12, 12)
        C, tokens, windows = geometry(w, big)
        q, k, v = device_qkv(torch, w, dev, 945)
        o = torch.empty_like(q)
        ms_a = timed(torch, stream, lambda: s3w.swin3d_window_attn_fwd(q, k, v, o, w["heads"], w["hd"], big, (1, 6, 6)),
                     reps)
        launches += len(ms_a)
        a_med = statistics.median(ms_a)
        out["stage1_window_2x12x12"] = {
            "grid": "B=1 T4xH180xW360, 8 heads x 64, window (2,12,12) N=288, shift (1,6,6), 900 windows; streaming "
                    "path (K/V blocks of 72 slots, online softmax)",
            "attn": {**launch_stats(ms_a), "bytes": attn_bytes(w), "flops": attn_flops(w, big),
                     "windows_per_s": windows / (a_med * 1e-3),
                     "roofline": roofline(attn_bytes(w), attn_flops(w, big), a_med, peaks)}}
        del q, k, v, o

    if want("stage1_qkv_proj"):
        # QKV projection (the attention's prologue) on the stage-1 grid: 259,200 tokens x 512 ->
        # 1536 (bf16, fp32 accumulate), then the attention on its grid-layout output
        w = WORKLOADS["stage1"]
        C, tokens, windows = geometry(w)
        from swin3d_window_attention_b200 import inputs as _inp
        x = _inp.normal_bf16_torch((w["B"], w["T"], w["H"], w["W"], C), dev, tensor_index=960)
        wq = _inp.normal_bf16_torch((3 * C, C), dev, tensor_index=961, sigma=C ** -0.5)
        bq = _inp.normal_f32_torch(3 * C, dev, tensor_index=962, sigma=0.1)
        qkv = torch.empty((w["B"], w["T"], w["H"], w["W"], 3 * C), dtype=torch.bfloat16, device=dev)
        o = torch.empty_like(x)
        ms_p = timed(torch, stream, lambda: s3w.swin3d_qkv_proj_fwd(x, wq, bq, qkv), reps)
        ms_c = timed(torch, stream, lambda: s3w.swin3d_qkv_window_attn_fwd(x, wq, bq, qkv, o, w["heads"], w["hd"], WINDOW,
                                                                           SHIFTED), reps)
        launches += len(ms_p) + 2 * len(ms_c)
        p_med, c_med = statistics.median(ms_p), statistics.median(ms_c)
        p_flops = 2 * tokens * C * 3 * C
        p_bytes = tokens * C * 2 + 3 * C * C * 2 + tokens * 3 * C * 2
        out["stage1_qkv_proj"] = {
            "grid": "B=1 T4xH180xW360: 259,200 tokens x C=512 -> 3C=1536 (bf16 in/out, fp32 accumulate, bias), then "
                    "the shifted-window attention on the projection's [tokens][3C] output",
            "proj": {**launch_stats(ms_p), "bytes": p_bytes, "flops": p_flops, "tflops": p_flops / (p_med * 1e-3) / 1e12,
                     "roofline": roofline(p_bytes, p_flops, p_med, peaks)},
            "proj_then_attn_ms": launch_stats(ms_c),
            "windows_per_s": windows / (c_med * 1e-3)}
        del x, wq, bq, qkv, o

    if want("stage1_fused"):
        # fused attention + AdaLN (one kernel per block) on the stage-1 grid: one launch, and the
        # headline step (two blocks) made of fused calls against the two-call step
        w = WORKLOADS["stage1"]
        C, tokens, windows = geometry(w)
        qkv = [device_qkv(torch, w, dev, 950 + 10 * b) for b in range(2)]
        films = [device_film(torch, w, dev, 970 + 10 * b, 0.1)[:2] for b in range(2)]
        res = device_film(torch, w, dev, 990, 1.0)[2]
        o = torch.empty_like(qkv[0][0])
        x = o.view(w["B"], tokens // w["B"], C)
        ws = torch.empty(s3w.window_attn_adaln_workspace_bytes(w["B"], w["T"], w["H"], w["W"], w["heads"], w["hd"],
                                                               WINDOW), dtype=torch.uint8, device=dev)

        def fused_call(b):
            q, k, v = qkv[b]
            s3w.swin3d_window_attn_adaln_fwd(q, k, v, res, films[b][0], films[b][1], res, w["heads"], w["hd"], WINDOW,
                                             SHIFTS[b], workspace=ws, eps=1e-5)

        def two_call_block(b):
            q, k, v = qkv[b]
            s3w.swin3d_window_attn_fwd(q, k, v, o, w["heads"], w["hd"], WINDOW, SHIFTS[b])
            s3w.adaln_residual_fwd(x, res, films[b][0], films[b][1], res, eps=1e-5)

        ms_f = timed(torch, stream, lambda: fused_call(1), reps)
        ms_fs = timed(torch, stream, lambda: [fused_call(b) for b in range(2)], reps)
        ms_ts = timed(torch, stream, lambda: [two_call_block(b) for b in range(2)], reps)
        launches += len(ms_f) + 2 * len(ms_fs) + 4 * len(ms_ts)
        f_med = statistics.median(ms_f)
        nbytes = fused_bytes(w)
        out["stage1_fused"] = {
            "grid": "B=1 T4xH180xW360, 8 heads x 64, shift (1,3,6), 1800 windows; attention + AdaLN in one kernel, "
                    "fp32 residual in place",
            "fused": {**launch_stats(ms_f), "bytes": nbytes, "flops": attn_flops(w), "windows_per_s": windows / (f_med * 1e-3),
                      "roofline": roofline(nbytes, attn_flops(w), f_med, peaks)},
            "step_fused_ms": launch_stats(ms_fs), "step_two_call_ms": launch_stats(ms_ts),
            "step_bytes_fused": 2 * nbytes, "step_bytes_two_call": 2 * (attn_bytes(w) + adaln_bytes(w)),
            "step_windows_per_s_fused": 2 * windows / (statistics.median(ms_fs) * 1e-3),
            "step_windows_per_s_two_call": 2 * windows / (statistics.median(ms_ts) * 1e-3)}
        del qkv, films, res, o, x, ws

    if want("stack_b4"):
        # six-block stage-1 stack at B = 4: fresh Q/K/V per block, fp32 residual chained
        w = WORKLOADS["stack_b4"]
        C, tokens, windows = geometry(w)
        qkv = [device_qkv(torch, w, dev, 1000 + 10 * b) for b in range(STACK_BLOCKS)]
        films = [device_film(torch, w, dev, 1100 + 10 * b, 1.0)[:2] for b in range(STACK_BLOCKS)]
        res = device_film(torch, w, dev, 1190, 1.0)[2]
        o = torch.empty_like(qkv[0][0])
        x = o.view(w["B"], tokens // w["B"], C)

        def stack():
            for b in range(STACK_BLOCKS):
                q, k, v = qkv[b]
                s3w.swin3d_window_attn_fwd(q, k, v, o, w["heads"], w["hd"], WINDOW, SHIFTS[b % 2])
                s3w.adaln_residual_fwd(x, res, films[b][0], films[b][1], res, eps=1e-5)

        ws = torch.empty(s3w.window_attn_adaln_workspace_bytes(w["B"], w["T"], w["H"], w["W"], w["heads"], w["hd"],
                                                               WINDOW), dtype=torch.uint8, device=dev)

        def stack_fused():
            for b in range(STACK_BLOCKS):
                q, k, v = qkv[b]
                s3w.swin3d_window_attn_adaln_fwd(q, k, v, res, films[b][0], films[b][1], res, w["heads"], w["hd"], WINDOW,
                                                 SHIFTS[b % 2], workspace=ws, eps=1e-5)

        stack_reps = max(3, reps // 4)
        ms_s = timed(torch, stream, stack, stack_reps, warmup=2)
        ms_sf = timed(torch, stream, stack_fused, stack_reps, warmup=2)
        launches += 3 * STACK_BLOCKS * stack_reps
        s_med = statistics.median(ms_s)
        nbytes = STACK_BLOCKS * (attn_bytes(w) + adaln_bytes(w))
        flops = STACK_BLOCKS * attn_flops(w)
        out["stack_b4"] = {
            "grid": "B=4 T4xH180xW360, 8 heads x 64, 6 x (attn alternating shift + AdaLN fp32 out), 7200 windows per call",
            "ms_per_stack": launch_stats(ms_s), "bytes": nbytes, "flops": flops,
            "floor_ms_at_measured_hbm": nbytes / (peaks["hbm_gbs"] * 1e9) * 1e3,
            "windows_per_s": STACK_BLOCKS * windows / (s_med * 1e-3),
            "roofline": roofline(nbytes, flops, s_med, peaks),
            "fused": {"ms_per_stack": launch_stats(ms_sf), "bytes": STACK_BLOCKS * fused_bytes(w),
                      "windows_per_s": STACK_BLOCKS * windows / (statistics.median(ms_sf) * 1e-3),
                      "roofline": roofline(STACK_BLOCKS * fused_bytes(w), flops, statistics.median(ms_sf), peaks)}}
        del qkv, films, res, o, x, ws
        torch.cuda.empty_cache()
    return out, launches


CONFIG_NAMES = ("tiny", "stage2", "stage3_padded", "stage1_tf32", "stage1_window_2x12x12", "stage1_qkv_proj",
                "stage1_fused", "stack_b4")


def bench_one_config(args):
    """One workload of the set on its own (``--config NAME``): its entry of ``configs``."""
    import torch

    import swin3d_window_attention_b200 as s3w

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s3w.load_library()
    out, launches = bench_configs(torch, s3w, dev, torch.cuda.current_stream(dev), load_peaks(), args.config_reps,
                                  only=args.config)
    if s3w.poll_device_error() != 0:
        raise SystemExit("device error word set")
    print(json.dumps({"config": args.config, "gpu_launches": launches, **out[args.config]}), flush=True)


def bench_cuda(args):
    import torch

    import swin3d_window_attention_b200 as s3w

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod

        dist = dist_mod
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    s3w.load_library()
    stream = torch.cuda.current_stream(dev)
    peaks = load_peaks()

    # headline inputs: one Q/K/V set per attention call, FiLM vectors, residual stream
    d = {}
    for i, _ in enumerate(SHIFTS):
        d[f"q{i}"], d[f"k{i}"], d[f"v{i}"] = device_qkv(torch, S1, dev, 100 + 10 * i)
    d["scale"], d["shift"], d["res"] = device_film(torch, S1, dev, 200, 0.1)
    o = torch.empty((S1["B"], S1["T"], S1["H"], S1["W"], C1), dtype=torch.bfloat16, device=dev)
    res = d["res"]
    x = o.view(S1["B"], L1 // S1["B"], C1)
    launches_per_step = 4
    attn_ev, adaln_ev = [], []

    def ev_pair():
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def step(record=False, dd=None, oo=None):
        dd = d if dd is None else dd
        oo = o if oo is None else oo
        xx = oo.view(S1["B"], L1 // S1["B"], C1)
        for i, shift in enumerate(SHIFTS):
            if record:
                a0, a1 = ev_pair()
                a0.record(stream)
            s3w.swin3d_window_attn_fwd(dd[f"q{i}"], dd[f"k{i}"], dd[f"v{i}"], oo, S1["heads"], S1["hd"], WINDOW, shift)
            if record:
                a1.record(stream)
                attn_ev.append((a0, a1))
            s3w.adaln_residual_fwd(xx, dd["res"], dd["scale"], dd["shift"], dd["res"], eps=1e-5)
            if record:
                a2 = torch.cuda.Event(enable_timing=True)
                a2.record(stream)
                adaln_ev.append((a1, a2))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    wall0 = time.time()
    t0.record(stream)
    for _ in range(args.steps):
        step(record=True)
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if dist:
        dist.barrier()
    clk = clocks.stop((wall0, wall1))
    ms, bad = reduce_max_over_ranks(torch, dist, [t0.elapsed_time(t1), s3w.poll_device_error() != 0], dev)
    if bad:
        if dist:
            dist.destroy_process_group()
        raise SystemExit("device error word set during the timed region (on at least one rank)")
    attn_ms = [a.elapsed_time(b) for a, b in attn_ev]
    adaln_ms = [a.elapsed_time(b) for a, b in adaln_ev]
    attn = launch_stats(attn_ms)
    adaln = launch_stats(adaln_ms)
    attn_med, adaln_med = attn["median_ms"], adaln["median_ms"]

    # For context: the same attention call on the legacy mma.sync baseline kernel.
    leg = timed(torch, stream, lambda: s3w.swin3d_window_attn_fwd_legacy_mma(
        d["q1"], d["k1"], d["v1"], o, S1["heads"], S1["hd"], WINDOW, SHIFTED), 3, warmup=1)

    # End to end through the public API with host buffers: every step copies its inputs from
    # pinned host memory and reads the step's result (the residual stream) back.  Two device
    # buffer sets and two copy streams: step i's inputs come in while step i - 1 computes, and
    # its result goes out while step i + 1's inputs come in (the host link is full duplex).
    pinned = {k: t.cpu().pin_memory() for k, t in d.items()}
    res_out = torch.empty(res.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = res_out.numel() * 4
    bufs = [d, {k: torch.empty_like(t) for k, t in d.items()}]
    obufs = [o, torch.empty_like(o)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        read_done = [None, None]   # the D2H of a buffer set's result (after its compute) is done
        s_in.wait_stream(stream)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if read_done[b] is not None:
                    s_in.wait_event(read_done[b])
                for kname, t in pinned.items():
                    bufs[b][kname].copy_(t, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            step(dd=bufs[b], oo=obufs[b])
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c)
                res_out.copy_(bufs[b]["res"], non_blocking=True)
                ev_r = torch.cuda.Event()
                ev_r.record(s_out)
            read_done[b] = ev_r
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0, e1 = ev_pair()
    e0.record(stream)
    e2e_run(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, = reduce_max_over_ranks(torch, dist, [e0.elapsed_time(e1) / args.steps], dev)
    del pinned, res_out, bufs, obufs

    configs, extra_launches = None, 0
    if world == 1 and not args.no_configs:
        del d, o, x, res
        torch.cuda.empty_cache()
        configs, extra_launches = bench_configs(torch, s3w, dev, stream, peaks, args.config_reps)
        if s3w.poll_device_error() != 0:
            raise SystemExit("device error word set during the per-config runs")

    ms_step = ms / args.steps
    windows_per_step = len(SHIFTS) * N_WIN
    rl = roofline(ATTN_BYTES, ATTN_FLOPS, attn_med, peaks)
    prof = recorded_profile()
    rl.update({"traffic": None if prof is None else int(prof["dram_bytes_read"]) + int(prof["dram_bytes_write"]),
               "traffic_source": None if prof is None else PROFILE, "peak_source": peaks["source"],
               "kernel": "window_attn_tc_kernel<64, bf16 out> (window attention)",
               "algorithmic_bytes_per_launch": ATTN_BYTES, "flops_per_launch": ATTN_FLOPS,
               "timing": "median of the per-launch CUDA-event times inside the timed region"})
    line = {
        "metric": METRIC,
        "value": windows_per_step * world / (ms_step * 1e-3),
        "unit": "windows/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, N(0,0.1) FiLM, N(0,1) fp32 residual)",
        "config": config_for(world),
        "attn": {**attn, "bytes": ATTN_BYTES, "flops": ATTN_FLOPS, "hbm_gbs": ATTN_BYTES / (attn_med * 1e-3) / 1e9,
                 "tflops": ATTN_FLOPS / (attn_med * 1e-3) / 1e12, "windows_per_s": N_WIN / (attn_med * 1e-3),
                 "legacy_mma_baseline_ms": min(leg)},
        "adaln": {**adaln, "bytes": ADALN_BYTES, "hbm_gbs": ADALN_BYTES / (adaln_med * 1e-3) / 1e9,
                  "frac": ADALN_BYTES / (adaln_med * 1e-3) / 1e9 / peaks["hbm_gbs"], "peak_source": peaks["source"]},
        "roofline": rl,
        "e2e": {"value": windows_per_step * world / (e2e_ms * 1e-3), "unit": "windows/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": args.steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if configs is not None:
        line["configs"] = configs
        line["gpu_launches_outside_timed_region"] = extra_launches + len(leg) + 1
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if dist:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- CPU oracle
class OracleSampler:
    """The fp64 oracle timed on bounded samples of a workload's windows.

    One sample = a batch of random windows (all heads) of the workload's grid through
    ``oracle.window_attn``, plus AdaLN on those windows' tokens where the workload has
    AdaLN.  Both benchmark arms use this one procedure: a short untimed warm-up, then
    batches until the time budget is spent.  Host inputs are seeded draws of the workload's
    shape (made once, not timed)."""

    BATCH = 8

    def __init__(self):
        import oracle

        oracle.build()
        self.oracle = oracle
        self.cache = {}

    def inputs(self, name):
        if name not in self.cache:
            import torch

            from swin3d_window_attention_b200 import inputs

            w = WORKLOADS[name]
            C = w["heads"] * w["hd"]
            shape = (w["B"], w["T"], w["H"], w["W"], C)
            qkv = [inputs.torch_bf16_to_bits(inputs.normal_bf16_torch(shape, "cpu", tensor_index=1300 + j))
                   for j in range(3)]
            film = [inputs.normal_f32_tensor((w["B"], C), tensor_index=1310 + j, sigma=0.1) for j in range(2)]
            self.cache[name] = (qkv, film)
            del torch
        return self.cache[name]

    def run(self, name, shifts, adaln, seconds, seed=0):
        """Windows per second of the oracle; returns (windows, seconds, threads)."""
        w = WORKLOADS[name]
        C, _, windows = geometry(w)
        (q, k, v), (sc, sh) = self.inputs(name)
        rng = np.random.default_rng(seed)
        batch = min(self.BATCH, windows)

        def one(shift):
            ids = rng.integers(0, windows, size=batch)
            out, tok, _ = self.oracle.window_attn(q, k, v, w["heads"], w["hd"], WINDOW, shift, window_ids=ids)
            if adaln:
                xo = out.reshape(1, -1, C)
                self.oracle.adaln(xo, np.zeros(xo.shape, dtype=np.float32), sc[:1], sh[:1], eps=1e-5)

        one(shifts[0])   # warm-up: threads started, pages touched
        done, i = 0, 0
        t0 = time.perf_counter()
        while True:
            one(shifts[i % len(shifts)])
            i += 1
            done += batch
            el = time.perf_counter() - t0
            if el >= seconds:
                return done, el, self.oracle.num_threads()


_SAMPLER = []


def sampler():
    if not _SAMPLER:
        _SAMPLER.append(OracleSampler())
    return _SAMPLER[0]


def cpu_baseline(seconds):
    """The oracle on the headline workload and on every other workload of the set."""
    smp = sampler()
    wins, el, thr = smp.run("stage1", SHIFTS, True, seconds)
    rate = wins / el
    per = {}
    other = max(2.0, seconds / 5)
    for name, shifts, adaln in (("tiny", (SHIFTED,), False), ("stage2", (SHIFTED,), True),
                                ("stage3_padded", (SHIFTED,), False)):
        wn, e, _ = smp.run(name, shifts, adaln, other)
        per[name] = {"windows_per_s": wn / e, "sample": f"{wn} random windows in {e:.1f} s"}
    per["stage1"] = {"windows_per_s": rate, "sample": f"{wins} random windows in {el:.1f} s"}
    # One block of the B=4 stack has the per-window work of stage 1 (same grid and heads).
    stack_windows = STACK_BLOCKS * geometry(WORKLOADS["stack_b4"])[2]
    per["stack_b4"] = {"windows_per_s": rate, "extrapolated": True,
                       "seconds_per_stack": stack_windows / rate,
                       "sample": "one block timed on stage-1 windows (same per-window work), x6 blocks extrapolated"}
    return {"value": rate, "unit": "windows/s", "cores": thr, "kind": "oracle",
            "sample": f"{wins} random stage-1 windows (8 heads each, both shifts alternating) + AdaLN on their "
                      f"tokens, {el:.1f} s on {thr} threads, after one untimed batch",
            "configs": per}


def bench_reference(args):
    """The fp64 oracle as the reference arm, on the host cores: same metric, unit, config
    and sampler as the CUDA arm's cpu_baseline."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    smp = sampler()
    per_step = max(0.5, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        smp.run("stage1", SHIFTS, True, 0.2)
    wins_total, el_total, thr = 0, 0.0, 1
    for k in range(args.steps):
        wn, el, thr = smp.run("stage1", SHIFTS, True, per_step, seed=k)
        wins_total += wn
        el_total += el
    value = wins_total / el_total
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "windows/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el_total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, same generator as the CUDA arm)",
        "config": config_for(world),
        "cpu_baseline": {"value": value, "unit": "windows/s", "cores": thr, "kind": "oracle",
                         "sample": f"{wins_total} random stage-1 windows + AdaLN on their tokens over {args.steps} "
                                   f"steps of ~{per_step:.1f} s on {thr} threads"},
        "e2e": {"value": value, "unit": "windows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--config-reps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--config", choices=CONFIG_NAMES, default=None,
                    help="time only this workload of the set (no headline step)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        bench_reference(args)
    elif args.config is not None:
        bench_one_config(args)
    else:
        bench_cuda(args)


if __name__ == "__main__":
    main()
