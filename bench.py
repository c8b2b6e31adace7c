#!/usr/bin/env python3
"""Benchmark of the Swin3D shifted-window attention hot path on B200.

One step = one pass of the whole path over one batch of the Aurora 0.25-degree
encoder stage-1 workload (B=1, grid 4x180x360, C=512 = 8 heads x 64, window (2,6,12)):

    window attention, shift (0,0,0)  -> AdaLN + residual (fp32 residual stream, in place)
    window attention, shift (1,3,6)  -> AdaLN + residual

Each attention call reads fresh seeded bf16 Q/K/V (N(0,1)), the AdaLN calls take the
attention output, per-sample FiLM scale/shift N(0,0.1) and the fp32 residual stream.
Every input tensor is larger than the 126 MB L2, so no flush is needed between steps.

Output: one JSON line (rank 0).  ``value`` is windows per second over all ranks (each
step processes 2 x 1800 windows x 8 heads per rank).  ``--impl reference`` times the
fp64 CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# Workload: Aurora 0.25-degree encoder stage 1.
B, T, H, W = 1, 4, 180, 360
HEADS, HD = 8, 64
C = HEADS * HD
WINDOW = (2, 6, 12)
SHIFTS = ((0, 0, 0), (1, 3, 6))
N_TOK = 144
L = T * H * W
N_WIN = B * (T // 2) * (H // 6) * (W // 12)          # 1800 windows per call
ATTN_BYTES = 4 * B * L * C * 2                         # read Q, K, V once, write O once (bf16)
ATTN_FLOPS = N_WIN * HEADS * 4 * N_TOK * N_TOK * HD    # QK^T and PV, dense in each window
ADALN_BYTES = B * L * C * (2 + 4 + 4)                  # bf16 x, fp32 residual in, fp32 out
WORKLOAD = ("Aurora 0.25deg encoder stage 1: B=1, grid T4xH180xW360, C=512 (8 heads x 64), window (2,6,12); "
            "per step: attn shift (0,0,0) + AdaLN fp32-out, attn shift (1,3,6) + AdaLN fp32-out")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self, window=None):
        """Median SM clock and the throttle reasons seen; with window = (t0, t1) in epoch
        seconds only the samples taken inside it count (all of them if none is)."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        import datetime

        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            try:
                rows.append((ts, float(f[2]), float(f[3]), f[6:10]))
            except ValueError:
                continue
        os.unlink(self.path)
        inside = [r for r in rows if window and (r[0] is None or window[0] <= r[0] <= window[1])]
        for _, s_mhz, m_mhz, flags in (inside or rows):
            sm.append(s_mhz)
            mx.append(m_mhz)
            for nm, val in zip(names, flags):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def make_device_inputs(torch, dev):
    """Seeded inputs: two Q/K/V sets (one per attention call), FiLM vectors, residual."""
    from swin3d_window_attention_b200 import inputs

    host = {}
    for i, _ in enumerate(SHIFTS):
        for j, name in enumerate("qkv"):
            host[f"{name}{i}"] = inputs.normal_bf16_bits((B, T, H, W, C), tensor_index=100 + 10 * i + j)
    host["scale"] = inputs.normal_f32_tensor((B, C), tensor_index=200, sigma=0.1)
    host["shift"] = inputs.normal_f32_tensor((B, C), tensor_index=201, sigma=0.1)
    host["res"] = inputs.normal_f32_tensor((B, L, C), tensor_index=202)
    devt = {}
    for kname, a in host.items():
        t = inputs.bits_to_torch_bf16(a) if a.dtype == np.uint16 else torch.from_numpy(a)
        devt[kname] = t.to(dev)
    return host, devt



def kernel_code_sha256(text):
    """sha256 of a source file's code: comments and blank lines removed, so that editing a
    comment does not separate a capture from the kernel it measured."""
    import hashlib
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln.strip()).encode()).hexdigest()


def recorded_traffic():
    """DRAM bytes per attention launch (dram__bytes_read.sum + dram__bytes_write.sum) from the
    committed ncu summary, or None if the kernel's code changed since that capture."""
    import re
    summ = os.path.join(ROOT, "profiles", "window_attn_tc_stage1_full.md")
    src = os.path.join(ROOT, "swin3d_window_attention_b200", "csrc", "attn_tcgen05.cu")
    if not (os.path.exists(summ) and os.path.exists(src)):
        return None
    text = open(summ).read()
    sha = re.search(r"code sha256 `([0-9a-f]{64})`", text)
    nbytes = re.search(r"dram_bytes_per_launch: (\d+)", text)
    if not sha or not nbytes:
        return None
    if kernel_code_sha256(open(src).read()) != sha.group(1):
        return None
    return int(nbytes.group(1))

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
    host, d = make_device_inputs(torch, dev)
    o = torch.empty((B, T, H, W, C), dtype=torch.bfloat16, device=dev)
    res = d["res"]
    launches_per_step = 4
    attn_events = []

    def step(record=False):
        for i, shift in enumerate(SHIFTS):
            if record:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            s3w.swin3d_window_attn_fwd(d[f"q{i}"], d[f"k{i}"], d[f"v{i}"], o, HEADS, HD, WINDOW, shift)
            if record:
                e1.record(stream)
                attn_events.append((e0, e1))
            s3w.adaln_residual_fwd(o.view(B, L, C), res, d["scale"], d["shift"], res, eps=1e-5)

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
    wall0 = time.time()
    t0.record(stream)
    for _ in range(args.steps):
        step(record=True)
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    ms = t0.elapsed_time(t1)
    clk = clocks.stop((wall0, wall1))
    if s3w.poll_device_error() != 0:
        raise SystemExit("device error word set during the timed region")
    if dist:
        tt = torch.tensor([ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
        dist.barrier()
    attn_ms = [a.elapsed_time(b) for a, b in attn_events]
    attn_avg_ms = sum(attn_ms) / len(attn_ms)

    # For context: the same attention call on the legacy mma.sync baseline kernel.
    leg = []
    for i in range(3):
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        s3w.swin3d_window_attn_fwd_legacy_mma(d["q1"], d["k1"], d["v1"], o, HEADS, HD, WINDOW, SHIFTS[1])
        a1.record(stream)
        leg.append((a0, a1))
    torch.cuda.synchronize()
    legacy_ms = min(a.elapsed_time(b) for a, b in leg)

    # End-to-end through the public API with host buffers: every step copies its inputs
    # from pinned host memory and reads the step's result (the residual stream) back.
    pinned = {k: (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16
                  else torch.from_numpy(v)).pin_memory() for k, v in host.items()}
    res_out = torch.empty((B, L, C), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = res_out.numel() * 4
    e2e_steps = max(1, min(args.steps, 5))

    def e2e_step():
        for kname, t in pinned.items():
            d[kname].copy_(t, non_blocking=True)
        step()
        res_out.copy_(res, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if dist:
        tt = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_ms = float(tt.item())

    hbm_peak, tc_peak, peak_src = load_peaks()
    ms_step = ms / args.steps
    windows_per_step = len(SHIFTS) * N_WIN
    value = windows_per_step * world / (ms_step * 1e-3)
    attn_gbs = ATTN_BYTES / (attn_avg_ms * 1e-3) / 1e9
    attn_tflops = ATTN_FLOPS / (attn_avg_ms * 1e-3) / 1e12
    line = {
        "metric": "window-attn TFLOP/s, HBM GB/s & % of roofline on 1 B200; windows/s",
        "value": value,
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
        "config": {"workload": WORKLOAD, "global_batch": B * world, "windows_per_call": N_WIN, "heads": HEADS,
                   "head_dim": HD, "l2": "inputs larger than L2 (265 MB per tensor), no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "attn": {"avg_launch_ms": attn_avg_ms, "hbm_gbs": attn_gbs, "tflops": attn_tflops,
                 "windows_per_s": N_WIN / (attn_avg_ms * 1e-3),
                 "hbm_frac": attn_gbs / hbm_peak, "tensor_frac": attn_tflops / tc_peak,
                 "legacy_mma_baseline_ms": legacy_ms},
        "roofline": {"bound": "hbm", "achieved": attn_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": attn_gbs / hbm_peak, "traffic": recorded_traffic(), "peak_source": peak_src,
                     "kernel": "window attention", "algorithmic_bytes_per_launch": ATTN_BYTES},
        "e2e": {"value": windows_per_step * world / (e2e_ms * 1e-3), "unit": "windows/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if dist:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


_CPU_INPUTS = []


def cpu_sample(seconds_budget):
    """Time the fp64 oracle on a bounded sample of the workload: whole windows (all heads)
    of both attention calls plus AdaLN on those windows' tokens.  Returns (windows, s, threads)."""
    import oracle
    from swin3d_window_attention_b200 import inputs

    oracle.build()
    rng = np.random.default_rng(0)
    # The oracle indexes the full grid, so one full-size input set is built once (not timed).
    if not _CPU_INPUTS:
        _CPU_INPUTS.extend([inputs.normal_bf16_bits((B, T, H, W, C), tensor_index=100 + j) for j in range(3)])
        _CPU_INPUTS.append(inputs.normal_f32_tensor((B, C), tensor_index=200, sigma=0.1))
        _CPU_INPUTS.append(inputs.normal_f32_tensor((B, C), tensor_index=201, sigma=0.1))
    q, k, v, sc, sh = _CPU_INPUTS
    done = 0
    t_start = time.perf_counter()
    batch = 8
    while True:
        for shift in SHIFTS:
            ids = rng.integers(0, N_WIN, size=batch)
            out, tok, _ = oracle.window_attn(q, k, v, HEADS, HD, WINDOW, shift, window_ids=ids)
            x = out.reshape(1, -1, C)
            res = np.zeros((1, x.shape[1], C), dtype=np.float32)
            oracle.adaln(x, res, sc, sh, eps=1e-5)
            done += batch
        el = time.perf_counter() - t_start
        if el >= seconds_budget:
            break
    return done, el, oracle.num_threads()


def cpu_baseline(seconds_budget):
    wins, el, thr = cpu_sample(seconds_budget)
    return {"value": wins / el, "unit": "windows/s", "cores": thr, "kind": "oracle",
            "sample": f"{wins} random windows (all 8 heads, both shifts alternating) + AdaLN on their tokens, "
                      f"{el:.1f} s on {thr} threads"}


def bench_reference(args):
    """The fp64 oracle as the reference arm, on the host cores, same metric and unit."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = max(1.0, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        cpu_sample(0.5)
    wins_total, el_total, thr = 0, 0.0, 1
    for _ in range(args.steps):
        w, el, thr = cpu_sample(per_step)
        wins_total += w
        el_total += el
    value = wins_total / el_total
    line = {
        "impl": "reference",
        "metric": "window-attn TFLOP/s, HBM GB/s & % of roofline on 1 B200; windows/s",
        "value": value, "unit": "windows/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el_total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, same generator as the CUDA arm)",
        "config": {"workload": WORKLOAD, "global_batch": B, "windows_per_call": N_WIN, "heads": HEADS,
                   "head_dim": HD},
        "cpu_baseline": {"value": value, "unit": "windows/s", "cores": thr, "kind": "oracle",
                         "sample": f"{wins_total} random windows over {args.steps} steps of ~{per_step:.1f} s"},
        "e2e": {"value": value, "unit": "windows/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_cuda(args)


if __name__ == "__main__":
    main()
