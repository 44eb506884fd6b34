#!/usr/bin/env python
"""Benchmark of the FP8 quantization hot path on B200.

Step = one pass of the Llama-3-8B-shaped quantization workload, both tensors in one launch
(fp8_quantize_many):
    128x128 block-wise E4M3 quantization of a 14336x4096 bf16 weight
  + 1x128 per-token-group E4M3 quantization of 8192x4096 bf16 activations
Inputs are seeded synthetic tensors (N(0,0.02) weights with 0.01% entries x20; N(0,1)
activations with 8 channels x50) resident in HBM before timing.  Four input sets rotate
(about 1.1 GB, far above the 126 MB L2), so no step reads another step's data from L2.

value  = algorithmic bytes of all ranks' steps / max-over-ranks device time (GB/s), where a
         step moves 2 B read + 1 B written per element plus 4 B per scale.
e2e    = the same metric through the Python binding of the C ABI with pinned host buffers:
         each step copies the bf16 inputs host->device and codes + scales device->host.
         Steps are pipelined over upload / compute / download streams and two device buffer
         sets, as a streaming user would run them: one step's upload overlaps the previous
         step's download (PCIe is full duplex), so a step costs about its upload time.
The timed region holds exactly K launches of the step's kernel, queued behind a short GPU
sleep (outside the region) so that it measures the kernels rather than the host's launch rate.
roofline: the step's kernel (k_quant_many): algorithmic bytes per launch over the mean launch
         duration in the timed region (region time / K, one launch per step).
clocks: nvidia-smi sampled every 50 ms for the whole run, summarised over the timed region
         (the nearest samples when the region is shorter than the interval) and over a 300 ms
         run of the same steps right after it; every GEMM line carries its own.
cpu_baseline: the CPU oracle on bounded samples (rank 0, N = 1): the step's two quantizers
         (all threads and one thread), the KV quantizers, the dequantizer, and the GEMM (8B
         decode shape in full, 70B prefill on sampled rows with the full time extrapolated).
supplementary: the other measured kernels (per-tensor, KV cache, dequantize, GEMM), each the
         median of at least 20 CUDA-event timings.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantize/KV-quant GB/s vs HBM peak; block-scaled FP8 GEMM TFLOPS vs FP8 peak"
W_SHAPE = (14336, 4096)
X_SHAPE = (8192, 4096)
N_SETS = 4
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def cdiv(a, b):
    return -(-a // b)


def bytes_w(n, k):       # 128x128 blocks: read bf16, write codes, one fp32 scale per block
    return n * k * 3 + cdiv(n, 128) * cdiv(k, 128) * 4


def bytes_x(m, k):       # 1x128 groups
    return m * k * 3 + cdiv(k, 128) * m * 4


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, if still current."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)[kernel_key]
        if d.get("source_sha") != source_sha(d["sources"]):
            return None
        return float(d["bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi in loop mode for the whole run (reads settings only); summaries are taken over
    the wall-clock window of each timed region."""

    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.samples = []
        self.proc = None

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits", "-lms", "50"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                ts, frac = parts[0].rsplit(".", 1) if "." in parts[0] else (parts[0], "0")
                t = time.mktime(time.strptime(ts, "%Y/%m/%d %H:%M:%S")) + float("0." + frac)
                self.samples.append((t, float(parts[1]), float(parts[2]), parts[4:]))
            except Exception:
                continue

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        """Median SM clock, max clock and throttle reasons of the samples inside [t0, t1]; a
        window shorter than the sampling interval takes the three samples nearest its middle."""
        samples = list(self.samples)
        inside = [s for s in samples if t0 - 0.01 <= s[0] <= t1 + 0.01]
        window = "timed region"
        if len(inside) < 3 and samples:
            mid = 0.5 * (t0 + t1)
            inside = sorted(samples, key=lambda s: abs(s[0] - mid))[:3]
            window = (f"the 3 samples nearest a {1e3 * (t1 - t0):.1f} ms timed region "
                      f"(max {1e3 * max(abs(s[0] - mid) for s in inside):.0f} ms from its middle)")
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for s in inside:
            for n, v in zip(names, s[3][1:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": max(s[2] for s in inside),
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ------------------------------------------------------------------ cross-rank aggregation

def reduce_max(value: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput_gbs(bytes_per_step: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's steps' bytes over the slowest rank's device time."""
    return world * bytes_per_step * steps / (ms_max * 1e-3) / 1e9


# ------------------------------------------------------------------ helpers

def dev_bf16(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16).to(device)


def timed(fn, reps, stream, flush=None, min_reps=20):
    """Median device time (ms) of fn over reps (at least min_reps), CUDA events on `stream`,
    optional L2 flush between reps (outside the events)."""
    import torch
    times = []
    for _ in range(max(reps, min_reps)):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


def timed_graph(fn, reps, stream, flush=None):
    """Median device time (ms) of one replay of fn captured as a CUDA graph (how a decode step's
    launches run: no host work between them), CUDA events on `stream`, optional L2 flush
    between replays (outside the timed region), at least 20 replays.  fn runs once before
    capture so any lazily created buffers exist outside the graph."""
    import torch
    with torch.cuda.stream(stream):
        fn()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        g.replay()
        stream.synchronize()
        times = []
        for _ in range(max(reps, 20)):
            if flush is not None:
                flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
    del g
    return statistics.median(times)


def gpu_identity(device):
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[0] if vis else "0"


# ------------------------------------------------------------------ reference arm (CPU oracle)

def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle as orc
    import synth
    rows = 256
    w = synth.weight_8b(seed=1)[:rows]
    x = synth.activations(seed=1)[:rows]
    nbytes = bytes_w(rows, W_SHAPE[1]) + bytes_x(rows, X_SHAPE[1])
    threads = orc._threads(None)

    def step():
        orc.quantize(w, orc.E4M3, orc.BLOCK_128x128)
        orc.quantize(x, orc.E4M3, orc.GROUP_1x128)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    value = nbytes / dt / 1e9
    sample = (f"rows 0..{rows - 1} of the 14336x4096 weight (128x128 blocks) and of the 8192x4096 "
              f"activations (1x128 groups) per step")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "llama3-8b quantization: 128x128 weight blocks 14336x4096 + 1x128 activation "
                               "groups 8192x4096, E4M3", "parallelism": "none (CPU oracle)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _cpu_loop(fn, min_s, max_reps=200):
    """Mean wall time (s) of fn, repeated until min_s has passed (at least once)."""
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        if time.perf_counter() - t0 > min_s or reps >= max_reps:
            break
    return (time.perf_counter() - t0) / reps, reps


def cpu_baseline_leg():
    """The oracle as it stands, timed on this host's cores on bounded samples of each workload:
    the benchmarked step (all threads and one thread), the KV quantizers, the dequantizer and
    the block-scaled GEMM (the 8B decode shape in full, the 70B prefill on sampled rows)."""
    import oracle as orc
    import synth
    rows = 512
    w = synth.weight_8b(seed=1)
    x = synth.activations(seed=1)
    ws_, xs_ = w[:rows], x[:rows]
    nbytes = bytes_w(rows, W_SHAPE[1]) + bytes_x(rows, X_SHAPE[1])
    threads = orc._threads(None)

    def step(th):
        orc.quantize(ws_, orc.E4M3, orc.BLOCK_128x128, threads=th)
        orc.quantize(xs_, orc.E4M3, orc.GROUP_1x128, threads=th)

    dt, reps = _cpu_loop(lambda: step(threads), 5.0)
    dt1, reps1 = _cpu_loop(lambda: step(1), 2.0)
    out = {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
           "sample": f"rows 0..{rows - 1} of the weight (128x128 blocks) and of the activations (1x128 groups), "
                     f"{reps} repetitions, {threads} threads",
           "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
           "single_thread": {"value": round(nbytes / dt1 / 1e9, 4), "unit": "GB/s", "reps": reps1}}
    # KV cache (config 3): the first 8192 tokens of the [131072][8][128] K and V caches; the
    # oracle's KV quantizer is one thread
    k, v = synth.kv_70b(seed=3, tokens=8192)
    e2 = 2 * k.size
    kv = {}
    for gran, name, fmt, per_elem in ((orc.KV_PER_HEAD_TOK128, "kv_head_tok128_e4m3", orc.E4M3, 3),
                                      (orc.KV_PER_HEAD, "kv_head_e4m3", orc.E4M3, 5),
                                      (orc.KV_PER_TENSOR, "kv_tensor_e5m2", orc.E5M2, 5)):
        dtk, _ = _cpu_loop(lambda: orc.kv_quantize(k, v, fmt, gran), 1.0, 20)
        kv[name] = {"GB/s": round(e2 * per_elem / dtk / 1e9, 4), "ms": round(dtk * 1e3, 2)}
    out["kv"] = {"threads": 1, "sample": "tokens 0..8191 of the config-3 K and V caches (8 heads x 128)", **kv}
    # dequantize: the 8B weight's first 512 rows from their 128x128 codes (one thread)
    wc, wsc = orc.quantize(ws_, orc.E4M3, orc.BLOCK_128x128)
    dtd, _ = _cpu_loop(lambda: orc.dequantize(wc, wsc, orc.E4M3, orc.BLOCK_128x128), 1.0, 50)
    out["dequant"] = {"GB/s": round(wc.size * 3 / dtd / 1e9, 4), "threads": 1,
                      "sample": "rows 0..511 of the 14336x4096 weight, 128x128 scales"}
    # GEMM (fp64 over dequantized operands): the 8B decode shape (M = 16) in full
    b8, sb8 = orc.quantize(w, orc.E4M3, orc.BLOCK_128x128, threads=threads)
    a16, sa16 = orc.quantize(x[:16], orc.E4M3, orc.GROUP_1x128)
    t0 = time.perf_counter()
    orc.gemm_rows(a16, sa16, 1, b8, sb8, 2, np.arange(16), threads=threads)
    dtg = time.perf_counter() - t0
    gemm = {"gemm_8b_up_m16": {"ms": round(dtg * 1e3, 1), "GFLOP/s": round(2.0 * 16 * W_SHAPE[0] * W_SHAPE[1] / dtg / 1e9, 3),
                               "threads": threads, "sample": "all 16 rows (full)"}}
    del b8, sb8, w
    # the 70B up-projection prefill (M = 16384) on sampled rows: one row per 128-row M tile in
    # tile order, a batch of `threads` rows at a time, until about 5 s have passed
    b70, sb70 = orc.quantize(synth.weight_70b(seed=4, which="up"), orc.E4M3, orc.BLOCK_128x128, threads=threads)
    x70 = synth.activations_70b(seed=4, m=16384, which="up")
    rng = np.random.default_rng(0)
    sample = np.array([t * 128 + int(rng.integers(0, 128)) for t in range(128)], np.int64)
    done, t0 = 0, time.perf_counter()
    while done < sample.size and time.perf_counter() - t0 < 5.0:
        rws = sample[done:done + threads]
        a, sa = orc.quantize(x70[rws], orc.E4M3, orc.GROUP_1x128)     # 1x128 groups are row-local
        orc.gemm_rows(a, sa, 1, b70, sb70, 2, np.arange(rws.size), threads=threads)
        done += rws.size
    dtr = time.perf_counter() - t0
    rows_s = done / dtr
    n70, k70 = b70.shape
    gemm["gemm_70b_up_m16384"] = {"rows_per_s": round(rows_s, 3),
                                  "GFLOP/s": round(2.0 * n70 * k70 * rows_s / 1e9, 3),
                                  "extrapolated_full_s": round(16384 / rows_s, 1), "threads": threads,
                                  "sample": f"{done} rows (one per 128-row M tile, tiles 0..{done - 1}), all 28672 "
                                            f"columns; the full time is extrapolated"}
    out["gemm"] = gemm
    return out


def supplementary(device, stream, peaks, flush, sampler):
    """Other kernels of the path, each on its own workload (short, device-timed); each GEMM line
    carries the SM clock sampled while it ran."""
    import torch

    import fp8_quantization_amax_b200 as fq
    import synth
    out = {}
    hbm = peaks["hbm_gbs"]
    fp8_peak = 2.0 * peaks["bf16_tflops"]                                   # burst
    fp8_peak_sustained = 2.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])   # under the power cap

    window = [(0.0, 0.0)]

    def ctimed(fn, reps, fl, graph=False):
        """timed / timed_graph, remembering the wall-clock window for the clock record."""
        t0 = time.time()
        ms = (timed_graph if graph else timed)(fn, reps, stream, fl)
        window[0] = (t0, time.time())
        return ms

    def add_clocks(key):
        c = sampler.summary(*window[0])
        mhz = c["sm_mhz"]
        out[key]["clocks"] = {"sm_mhz": mhz, "reasons": c["reasons"], "samples": c["samples"],
                              "sm_cycles_M": round(out[key]["us"] * mhz / 1e6, 3) if mhz else None}

    def gbs(nbytes, ms):
        return {"us": round(ms * 1e3, 2), "GB/s": round(nbytes / ms / 1e6, 1), "frac_hbm": round(nbytes / ms / 1e6 / hbm, 3)}

    def back_to_back(entry, fn, nbytes, calls=40):
        """Add the mean of `calls` dependent launches (fn(i) over rotating inputs, no event in
        between) to an entry timed per launch."""
        ms = timed(lambda: [fn(i) for i in range(calls)], 5, stream, None) / calls
        b = gbs(nbytes, ms)
        entry["back_to_back"] = {"us": b["us"], "GB/s": b["GB/s"], "frac_hbm": b["frac_hbm"]}

    with torch.cuda.stream(stream):
        # per-tensor 1024x1024, E4M3 and E5M2, quantize + dequantize (launch-latency bound)
        t = dev_bf16(synth.per_tensor_1024(seed=0), device)
        for fmt, name in ((fq.E4M3, "e4m3"), (fq.E5M2, "e5m2")):
            c, s = fq.fp8_quantize(t, fmt, fq.PER_TENSOR)
            ms_q = timed(lambda: fq.fp8_quantize(t, fmt, fq.PER_TENSOR, codes=c, scales=s), 50, stream, flush)
            y = torch.empty_like(t)
            ms_d = timed(lambda: fq.fp8_dequantize(c, s, fmt, fq.PER_TENSOR, out=y), 50, stream, flush)
            e = t.numel()
            out[f"per_tensor_1024_{name}_quant"] = gbs(e * 5 + 4, ms_q)
            out[f"per_tensor_1024_{name}_dequant"] = gbs(e * 3 + 4, ms_d)
        del t
        # dequantize of the 8B weight codes (128x128)
        w = dev_bf16(synth.weight_8b(seed=1), device)
        wc, ws = fq.fp8_quantize(w, fq.E4M3, fq.BLOCK_128x128)
        y = torch.empty_like(w)
        ms = timed(lambda: fq.fp8_dequantize(wc, ws, fq.E4M3, fq.BLOCK_128x128, out=y), 20, stream, flush)
        out["dequant_14336x4096_128x128"] = gbs(w.numel() * 3 + ws.numel() * 4, ms)
        wcs = [wc.clone() for _ in range(4)]          # 4 x 58.7 MB of codes and 2 x 117 MB of output > L2
        ys = [y, torch.empty_like(w)]
        back_to_back(out["dequant_14336x4096_128x128"],
                     lambda i: fq.fp8_dequantize(wcs[i % 4], ws, fq.E4M3, fq.BLOCK_128x128, out=ys[i % 2]),
                     w.numel() * 3 + ws.numel() * 4)
        del y, ys, wcs
        # KV cache, 70B layer: [131072][8][128] for K and V
        k, v = synth.kv_70b(seed=3)
        kd, vd = dev_bf16(k, device), dev_bf16(v, device)
        e2 = 2 * kd.numel()
        for gran, name, fmt, passes in ((fq.KV_PER_HEAD_TOK128, "kv_head_tok128_e4m3", fq.E4M3, 1),
                                        (fq.KV_PER_HEAD, "kv_head_e4m3", fq.E4M3, 2),
                                        (fq.KV_PER_TENSOR, "kv_tensor_e5m2", fq.E5M2, 2)):
            r = fq.fp8_kv_quantize(kd, vd, fmt, gran)
            ms = timed(lambda: fq.fp8_kv_quantize(kd, vd, fmt, gran, *r, ws=None), 10, stream, flush)
            nbytes = e2 * (3 if passes == 1 else 5) + 2 * r[2].numel() * 4
            out[name] = gbs(nbytes, ms)
            # steady state: 8 dependent calls over the same 805 MB cache (> L2), each also draining
            # the previous call's codes still dirty in L2
            back_to_back(out[name], lambda i: fq.fp8_kv_quantize(kd, vd, fmt, gran, *r, ws=None), nbytes, calls=8)
        # delayed scaling (per head, E4M3): after the first call every call reads the cache once
        hk = torch.zeros((4, 8), dtype=torch.float32, device=device)
        hv = torch.zeros_like(hk)
        r = fq.fp8_kv_quantize_delayed(kd, vd, hk, hv, 0, fq.E4M3, fq.KV_PER_HEAD)
        step_no = [0]

        def delayed_call():
            step_no[0] += 1
            fq.fp8_kv_quantize_delayed(kd, vd, hk, hv, step_no[0], fq.E4M3, fq.KV_PER_HEAD, *r)

        ms = timed(delayed_call, 10, stream, flush)
        out["kv_head_e4m3_delayed"] = gbs(e2 * 3 + 2 * r[2].numel() * 4, ms)
        back_to_back(out["kv_head_e4m3_delayed"], lambda i: delayed_call(), e2 * 3 + 2 * r[2].numel() * 4, calls=8)
        del kd, vd, r
        # MXFP8 (1x32 groups, power-of-two scales) on the config-1 activations, and its dequantizer
        xa = dev_bf16(synth.activations(seed=1), device)
        mc, ms_ = fq.fp8_quantize_mx(xa)
        ms = timed(lambda: fq.fp8_quantize_mx(xa, fq.E4M3, codes=mc, scales=ms_), 20, stream, flush)
        out["mx_1x32_activations_8b"] = gbs(xa.numel() * 3 + ms_.numel(), ms)
        xas = [xa] + [xa.clone() for _ in range(3)]    # 4 x 67 MB of activations > L2
        back_to_back(out["mx_1x32_activations_8b"],
                     lambda i: fq.fp8_quantize_mx(xas[i % 4], fq.E4M3, codes=mc, scales=ms_), xa.numel() * 3 + ms_.numel())
        del xas
        ymx = torch.empty_like(xa)
        ms = timed(lambda: fq.fp8_dequantize_mx(mc, ms_, fq.E4M3, out=ymx), 20, stream, flush)
        out["mx_dequant_8b"] = gbs(xa.numel() * 3 + ms_.numel(), ms)
        mcs = [mc.clone() for _ in range(8)]          # 8 x 33.5 MB of codes and 4 x 67 MB of output > L2
        ymxs = [ymx] + [torch.empty_like(xa) for _ in range(3)]
        back_to_back(out["mx_dequant_8b"], lambda i: fq.fp8_dequantize_mx(mcs[i % 8], ms_, fq.E4M3, out=ymxs[i % 4]),
                     xa.numel() * 3 + ms_.numel())
        del xa, mc, ms_, ymx, mcs, ymxs
        # GEMM (8B up-proj shape) on the quantized config-1 operands
        x8 = dev_bf16(synth.activations(seed=1), device)
        xc, xs = fq.fp8_quantize(x8, fq.E4M3, fq.GROUP_1x128)

        def gemm_entry(m, n, k, ms, a, sa, wscale, c):
            flops = 2.0 * m * n * k
            nbytes = a.numel() + n * k + c.numel() * 2 + sa.numel() * sa.element_size() + \
                wscale.numel() * wscale.element_size()
            return {"us": round(ms * 1e3, 2), "TFLOP/s": round(flops / ms / 1e9, 1),
                    "frac_fp8_peak": round(flops / ms / 1e9 / fp8_peak, 3),
                    "frac_fp8_peak_sustained": round(flops / ms / 1e9 / fp8_peak_sustained, 3),
                    "GB/s": round(nbytes / ms / 1e6, 1), "frac_hbm": round(nbytes / ms / 1e6 / hbm, 3)}

        try:
            # prefill: one call per timing, L2 flushed before each
            m = 8192
            a, sa = xc[:m].contiguous(), xs[:, :m].contiguous()
            cbuf = torch.empty((m, W_SHAPE[0]), dtype=torch.bfloat16, device=device)
            fq.fp8_gemm_blockscaled(a, sa, wc, ws, out=cbuf)
            ms = ctimed(lambda: fq.fp8_gemm_blockscaled(a, sa, wc, ws, out=cbuf), 20, flush)
            out["gemm_8b_up_m8192"] = gemm_entry(m, W_SHAPE[0], W_SHAPE[1], ms, a, sa, ws, cbuf)
            add_clocks("gemm_8b_up_m8192")
            # the prefill linear layer from bf16 activations (1x128 quantizer, then the GEMM: two
            # dependent launches), beside the quantizer alone: the most any fusion of the two saves
            act8 = torch.empty(fq.linear_act_workspace_bytes(m, W_SHAPE[1]), dtype=torch.uint8, device=device)
            ms_lin = ctimed(lambda: fq.fp8_linear_dynamic(x8, wc, ws, out=cbuf, act_ws=act8), 20, flush)
            ms_q1 = timed(lambda: fq.fp8_quantize(x8, fq.E4M3, fq.GROUP_1x128, codes=a, scales=sa), 20, stream, flush)
            out["linear_8b_m8192_dynamic"] = gemm_entry(m, W_SHAPE[0], W_SHAPE[1], ms_lin, a, sa, ws, cbuf)
            out["linear_8b_m8192_dynamic"].update({"gemm_alone_us": round(ms * 1e3, 2),
                                                   "quantize_alone_us": round(ms_q1 * 1e3, 2)})
            add_clocks("linear_8b_m8192_dynamic")
            del act8
            # the same layer as one cooperative launch (quantize phase, grid barrier, GEMM)
            actf = torch.zeros(fq.linear_fused_workspace_bytes(m, W_SHAPE[1]), dtype=torch.uint8, device=device)
            fq.fp8_linear_dynamic_fused(x8, wc, ws, out=cbuf, act_ws=actf)
            ms_f = ctimed(lambda: fq.fp8_linear_dynamic_fused(x8, wc, ws, out=cbuf, act_ws=actf), 20, flush)
            out["linear_8b_m8192_fused"] = gemm_entry(m, W_SHAPE[0], W_SHAPE[1], ms_f, a, sa, ws, cbuf)
            out["linear_8b_m8192_fused"]["two_launch_us"] = round(ms_lin * 1e3, 2)
            add_clocks("linear_8b_m8192_fused")
            del actf
            # the same GEMM with C quantized to E4M3 1x128 groups in the epilogue, against the two
            # steps it replaces (bf16 C, then the 1x128 quantizer)
            qc = torch.empty((m, W_SHAPE[0]), dtype=torch.uint8, device=device)
            qs = torch.empty(fq.scale_shape(m, W_SHAPE[0], fq.GROUP_1x128), dtype=torch.float32, device=device)
            fq.fp8_gemm_blockscaled_to_fp8(a, sa, wc, ws, codes=qc, scales=qs)
            ms_f = ctimed(lambda: fq.fp8_gemm_blockscaled_to_fp8(a, sa, wc, ws, codes=qc, scales=qs), 20, flush)
            ms_2 = timed(lambda: (fq.fp8_gemm_blockscaled(a, sa, wc, ws, out=cbuf),
                                  fq.fp8_quantize(cbuf, fq.E4M3, fq.GROUP_1x128, codes=qc, scales=qs)), 20, stream,
                         flush)
            flops = 2.0 * m * W_SHAPE[0] * W_SHAPE[1]
            out["gemm_8b_up_m8192_to_fp8"] = {"us": round(ms_f * 1e3, 2), "TFLOP/s": round(flops / ms_f / 1e9, 1),
                                              "frac_fp8_peak": round(flops / ms_f / 1e9 / fp8_peak, 3),
                                              "two_steps_us": round(ms_2 * 1e3, 2)}
            add_clocks("gemm_8b_up_m8192_to_fp8")
            del qc, qs
            # MXFP8 on the native block-scaled MMA, same shape: both operands quantized in 1x32
            # groups with power-of-two scales (blocked layout)
            am, sam = fq.fp8_quantize_mx_blocked(dev_bf16(synth.activations(seed=1), device))
            bm, sbm = fq.fp8_quantize_mx_blocked(dev_bf16(synth.weight_8b(seed=1), device))
            fq.fp8_gemm_mx(am, sam, bm, sbm, out=cbuf)
            ms = ctimed(lambda: fq.fp8_gemm_mx(am, sam, bm, sbm, out=cbuf), 20, flush)
            out["gemm_mx_8b_up_m8192"] = gemm_entry(m, W_SHAPE[0], W_SHAPE[1], ms, am, sam, sbm, cbuf)
            add_clocks("gemm_mx_8b_up_m8192")
            del cbuf, am, sam, bm, sbm
            # decode: back-to-back calls as in a decode step, each on one of four copies of the
            # weight codes (4 x 58.7 MB > L2), so every call streams its weights from HBM
            m = 16
            a, sa = xc[:m].contiguous(), xs[:, :m].contiguous()
            cbuf = torch.empty((m, W_SHAPE[0]), dtype=torch.bfloat16, device=device)
            copies = [wc.clone() for _ in range(4)]
            calls = 32
            fq.fp8_gemm_blockscaled(a, sa, copies[0], ws, out=cbuf)

            def batch():
                for i in range(calls):
                    fq.fp8_gemm_blockscaled(a, sa, copies[i % 4], ws, out=cbuf)

            ms = ctimed(batch, 20, flush, graph=True) / calls
            ms_py = timed(batch, 20, stream, flush) / calls
            out["gemm_8b_up_m16"] = gemm_entry(m, W_SHAPE[0], W_SHAPE[1], ms, a, sa, ws, cbuf)
            out["gemm_8b_up_m16"]["timing"] = (f"{calls} back-to-back calls over 4 weight copies replayed from a "
                                               f"CUDA graph, median per call")
            out["gemm_8b_up_m16"]["python_loop_us"] = round(ms_py * 1e3, 2)
            add_clocks("gemm_8b_up_m16")
            # the same decode GEMM from bf16 activations: the caller's two calls, and the linear
            # entry point (the same two kernels as one call)
            xb = dev_bf16(synth.activations(seed=1)[:m], device)

            def two_step():
                for i in range(calls):
                    a2, s2 = fq.fp8_quantize(xb, fq.E4M3, fq.GROUP_1x128, codes=a, scales=sa)
                    fq.fp8_gemm_blockscaled(a2, s2, copies[i % 4], ws, out=cbuf)

            act_ws = torch.empty(fq.linear_act_workspace_bytes(m, W_SHAPE[1]), dtype=torch.uint8, device=device)

            def fused():
                for i in range(calls):
                    fq.fp8_linear_dynamic(xb, copies[i % 4], ws, out=cbuf, act_ws=act_ws)

            ms2 = ctimed(two_step, 20, flush, graph=True) / calls
            ms3 = ctimed(fused, 20, flush, graph=True) / calls
            out["linear_8b_m16_quantize_then_gemm"] = gemm_entry(m, W_SHAPE[0], W_SHAPE[1], ms2, a, sa, ws, cbuf)
            out["linear_8b_m16_dynamic"] = gemm_entry(m, W_SHAPE[0], W_SHAPE[1], ms3, a, sa, ws, cbuf)
            out["linear_8b_m16_dynamic"]["timing"] = "bf16 activations in; same batching and graph replay as gemm_8b_up_m16"
            add_clocks("linear_8b_m16_dynamic")
            del copies, cbuf, x8
            # decode on the 70B up-projection (one weight, 235 MB > L2)
            w70 = dev_bf16(synth.weight_70b(seed=4, which="up"), device)
            b70, s70 = fq.fp8_quantize(w70, fq.E4M3, fq.BLOCK_128x128)
            b70m, s70m = fq.fp8_quantize_mx_blocked(w70)
            del w70
            x70 = dev_bf16(synth.activations_70b(seed=4, m=64, which="up"), device)
            a70, sa70 = fq.fp8_quantize(x70, fq.E4M3, fq.GROUP_1x128)
            c70 = torch.empty((64, b70.shape[0]), dtype=torch.bfloat16, device=device)
            fq.fp8_gemm_blockscaled(a70, sa70, b70, s70, out=c70)
            calls = 8

            def batch70():
                for _ in range(calls):
                    fq.fp8_gemm_blockscaled(a70, sa70, b70, s70, out=c70)

            ms = ctimed(batch70, 20, flush, graph=True) / calls
            out["gemm_70b_up_m64"] = gemm_entry(64, b70.shape[0], b70.shape[1], ms, a70, sa70, s70, c70)
            out["gemm_70b_up_m64"]["timing"] = (f"{calls} back-to-back calls (weight 235 MB > L2) replayed from a CUDA "
                                                f"graph, median per call")
            add_clocks("gemm_70b_up_m64")
            del a70, sa70, c70
            # prefill on the 70B up and down projections (M = 16384), block-scaled and per-tensor
            for which in ("up", "down"):
                if which == "down":
                    del b70, s70
                    w70 = dev_bf16(synth.weight_70b(seed=4, which="down"), device)
                    b70, s70 = fq.fp8_quantize(w70, fq.E4M3, fq.BLOCK_128x128)
                    del w70
                x70 = dev_bf16(synth.activations_70b(seed=4, m=16384, which=which), device)
                a70, sa70 = fq.fp8_quantize(x70, fq.E4M3, fq.GROUP_1x128)
                if which == "up":
                    a70m, sa70m = fq.fp8_quantize_mx_blocked(x70)
                c70 = torch.empty((16384, b70.shape[0]), dtype=torch.bfloat16, device=device)
                fq.fp8_gemm_blockscaled(a70, sa70, b70, s70, out=c70)
                ms = ctimed(lambda: fq.fp8_gemm_blockscaled(a70, sa70, b70, s70, out=c70), 20, flush)
                out[f"gemm_70b_{which}_m16384"] = gemm_entry(16384, b70.shape[0], b70.shape[1], ms, a70, sa70, s70, c70)
                add_clocks(f"gemm_70b_{which}_m16384")
                if which == "up":
                    act70 = torch.empty(fq.linear_act_workspace_bytes(16384, b70.shape[1]), dtype=torch.uint8,
                                        device=device)
                    ms_lin = ctimed(lambda: fq.fp8_linear_dynamic(x70, b70, s70, out=c70, act_ws=act70), 20, flush)
                    ms_q1 = timed(lambda: fq.fp8_quantize(x70, fq.E4M3, fq.GROUP_1x128, codes=a70, scales=sa70), 20,
                                  stream, flush)
                    out["linear_70b_up_m16384_dynamic"] = gemm_entry(16384, b70.shape[0], b70.shape[1], ms_lin, a70,
                                                                     sa70, s70, c70)
                    out["linear_70b_up_m16384_dynamic"].update({"gemm_alone_us": round(ms * 1e3, 2),
                                                                "quantize_alone_us": round(ms_q1 * 1e3, 2)})
                    add_clocks("linear_70b_up_m16384_dynamic")
                    del act70
                    actf = torch.zeros(fq.linear_fused_workspace_bytes(16384, b70.shape[1]), dtype=torch.uint8,
                                       device=device)
                    fq.fp8_linear_dynamic_fused(x70, b70, s70, out=c70, act_ws=actf)
                    ms_f = ctimed(lambda: fq.fp8_linear_dynamic_fused(x70, b70, s70, out=c70, act_ws=actf), 20, flush)
                    out["linear_70b_up_m16384_fused"] = gemm_entry(16384, b70.shape[0], b70.shape[1], ms_f, a70,
                                                                   sa70, s70, c70)
                    out["linear_70b_up_m16384_fused"]["two_launch_us"] = round(ms_lin * 1e3, 2)
                    add_clocks("linear_70b_up_m16384_fused")
                    del actf
                del x70
                if which == "up":
                    one = torch.ones(1, dtype=torch.float32, device=device)
                    fq.fp8_gemm_blockscaled(a70, one, b70, one, fq.PER_TENSOR, fq.PER_TENSOR, out=c70)
                    ms = ctimed(lambda: fq.fp8_gemm_blockscaled(a70, one, b70, one, fq.PER_TENSOR, fq.PER_TENSOR,
                                                                out=c70), 20, flush)
                    out["gemm_70b_up_m16384_per_tensor"] = gemm_entry(16384, b70.shape[0], b70.shape[1], ms, a70, one,
                                                                      one, c70)
                    add_clocks("gemm_70b_up_m16384_per_tensor")
                    fq.fp8_gemm_mx(a70m, sa70m, b70m, s70m, out=c70)
                    ms = ctimed(lambda: fq.fp8_gemm_mx(a70m, sa70m, b70m, s70m, out=c70), 20, flush)
                    out["gemm_mx_70b_up_m16384"] = gemm_entry(16384, b70.shape[0], b70.shape[1], ms, a70m, sa70m,
                                                              s70m, c70)
                    add_clocks("gemm_mx_70b_up_m16384")
                    del a70m, sa70m, b70m, s70m
                del a70, sa70, c70
            del b70, s70
        except fq.Fp8qError as err:
            out["gemm"] = f"not measured: {err}"
    return out


def our_arm(args):
    import torch
    import torch.distributed as dist

    import fp8_quantization_amax_b200 as fq
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    fq.lib()
    peaks = load_peaks()
    stream = torch.cuda.Stream(device)
    sampler = ClockSampler(gpu_identity(device))
    sampler.start()

    # inputs: N_SETS rotating copies of the weight and activations
    w_np = synth.weight_8b(seed=1)
    x_np = synth.activations(seed=1)
    W = [dev_bf16(w_np, device) for _ in range(N_SETS)]
    X = [dev_bf16(x_np, device) for _ in range(N_SETS)]
    n, k = W_SHAPE
    m, _ = X_SHAPE
    WC = [torch.empty(W_SHAPE, dtype=torch.uint8, device=device) for _ in range(N_SETS)]
    WS = [torch.empty(fq.scale_shape(n, k, fq.BLOCK_128x128), dtype=torch.float32, device=device) for _ in range(N_SETS)]
    XC = [torch.empty(X_SHAPE, dtype=torch.uint8, device=device) for _ in range(N_SETS)]
    XS = [torch.empty(fq.scale_shape(m, k, fq.GROUP_1x128), dtype=torch.float32, device=device) for _ in range(N_SETS)]
    step_bytes = bytes_w(n, k) + bytes_x(m, k)
    flush_buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=device)
    flush_rd = torch.ones(64 * 1024 * 1024, dtype=torch.int64, device=device)   # 512 MB

    def flush():
        # write a buffer 4x the L2, then read another: the write evicts everything the timed
        # kernel could reuse, the read makes the flush's own dirty lines write back now, before
        # the timed launch starts, instead of during it
        flush_buf.zero_()
        flush_rd.sum()

    jobs = [[(W[j], fq.BLOCK_128x128, WC[j], WS[j]), (X[j], fq.GROUP_1x128, XC[j], XS[j])] for j in range(N_SETS)]

    def step(i):
        # both tensors in one launch (fp8_quantize_many)
        fq.fp8_quantize_many(jobs[i % N_SETS], fq.E4M3)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize(device)
        barrier()
        torch.cuda.synchronize(device)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        # the GPU sleeps (outside the timed region) while the host queues the start event and
        # the steps behind it, so the region measures the kernels, not the host's launch rate
        torch.cuda._sleep(int(min(2e9, 2e6 + 40e3 * args.steps)))
        t_start.record(stream)
        for i in range(args.steps):
            step(i)
        t_end.record(stream)
        t_start.synchronize()
        wall0 = time.time()
        torch.cuda.synchronize(device)
        wall1 = time.time()
        barrier()
    ms_total = reduce_max(t_start.elapsed_time(t_end), device)
    ms_step = ms_total / max(args.steps, 1)
    value = job_throughput_gbs(step_bytes, args.steps, world, ms_total)
    s_ms = ms_step
    # the timed region is shorter than nvidia-smi's sampling interval at small step counts:
    # also sample a longer run of the same steps right after it (reported beside it)
    clocks = sampler.summary(wall0, wall1)
    if not args.skip_extras:
        with torch.cuda.stream(stream):
            n_long = max(args.steps, int(300.0 / max(ms_step, 1e-3)))
            torch.cuda._sleep(int(2e6))
            wl0 = time.time()
            for i in range(n_long):
                step(i)
            torch.cuda.synchronize(device)
            wl1 = time.time()
        clocks["same_steps_300ms"] = sampler.summary(wl0, wl1)

    if args.skip_extras:
        sampler.stop()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
                              "note": "profiling run: steps only", "kernels_us": [round(s_ms * 1e3, 2)]}),
                  flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    # end to end through the binding, pinned host buffers, copies inside the timed region
    hw = torch.from_numpy(w_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    hx = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    hwc = torch.empty(W_SHAPE, dtype=torch.uint8).pin_memory()
    hxc = torch.empty(X_SHAPE, dtype=torch.uint8).pin_memory()
    hws = torch.empty(WS[0].shape, dtype=torch.float32).pin_memory()
    hxs = torch.empty(XS[0].shape, dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    # a streaming pipeline: step i's upload (pinned host -> device), quantization and download
    # (codes and scales -> pinned host) run on three streams over two device buffer sets, so the
    # upload of step i + 1 and the download of step i - 1 overlap (PCIe is full duplex); events
    # keep a set's inputs until its kernels have read them and its codes until they are copied
    s_up, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_up = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_down = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        j = i % 2
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(ev_done[j])
            W[j].copy_(hw, non_blocking=True)
            X[j].copy_(hx, non_blocking=True)
            ev_up[j].record(s_up)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_up[j])
            if i >= 2:
                stream.wait_event(ev_down[j])
            fq.fp8_quantize_many(jobs[j], fq.E4M3)
            ev_done[j].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev_done[j])
            hwc.copy_(WC[j], non_blocking=True)
            hws.copy_(WS[j], non_blocking=True)
            hxc.copy_(XC[j], non_blocking=True)
            hxs.copy_(XS[j], non_blocking=True)
            ev_down[j].record(s_down)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(device)
    barrier()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_up)
    for i in range(2, 2 + e2e_steps):
        e2e_step(i)
    b.record(s_down)
    torch.cuda.synchronize(device)
    barrier()
    e2e_ms = reduce_max(a.elapsed_time(b), device)
    h2d = (hw.numel() + hx.numel()) * 2
    d2h = hwc.numel() + hxc.numel() + (hws.numel() + hxs.numel()) * 4
    e2e_value = job_throughput_gbs(step_bytes, e2e_steps, world, e2e_ms)

    result = None
    if rank == 0:
        achieved = step_bytes / (s_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        traffic = ncu_traffic("k_quant_many_step")
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "llama3-8b quantization: 128x128 E4M3 weight blocks of a 14336x4096 bf16 weight "
                                   "+ 1x128 E4M3 activation groups of 8192x4096 bf16 activations (seed 1)",
                       "weight": list(W_SHAPE), "activations": list(X_SHAPE), "fmt": "e4m3",
                       "l2": f"{N_SETS} rotating input sets ({N_SETS * (w_np.nbytes + x_np.nbytes) / 1e9:.2f} GB) > 126 MB L2",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "kernel": "k_quant_many (the step: 128x128 weight blocks + 1x128 activation groups, "
                                   "one launch)", "bytes_per_launch": step_bytes,
                         "launch_us": round(s_ms * 1e3, 2),
                         "timing": "CUDA events around the timed region on the launching stream, which holds "
                                   "exactly one launch of this kernel per step: mean launch duration = "
                                   "region time / steps",
                         "peak_source": f"{peaks['source']} hbm_gbs"},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clocks,
        }
    if rank == 0 and world == 1 and not args.no_supplementary:
        # 40 back-to-back launches over the input sets (dependent launches overlap each launch's
        # start with the previous one's tail; no event between launches): the step's kernel, and
        # for reference the two single-tensor kernels the step replaces
        b2b = {}
        with torch.cuda.stream(stream):
            for name, fn, nbytes in (
                    ("quant_step_one_launch", lambda j: fq.fp8_quantize_many(jobs[j], fq.E4M3), step_bytes),
                    ("quant_128x128_weight", lambda j: fq.fp8_quantize(W[j], fq.E4M3, fq.BLOCK_128x128, codes=WC[j],
                                                                      scales=WS[j]), bytes_w(n, k)),
                    ("quant_1x128_activations", lambda j: fq.fp8_quantize(X[j], fq.E4M3, fq.GROUP_1x128, codes=XC[j],
                                                                         scales=XS[j]), bytes_x(m, k))):
                ms = timed(lambda: [fn(i % N_SETS) for i in range(40)], 5, stream, None) / 40
                b2b[name] = {"us": round(ms * 1e3, 2), "GB/s": round(nbytes / ms / 1e6, 1),
                             "frac_hbm": round(nbytes / ms / 1e6 / peaks["hbm_gbs"], 3)}
        result["kernels_back_to_back"] = b2b
    del W, X, WC, XC, WS, XS, jobs
    if rank == 0 and world == 1:
        if not args.no_supplementary:
            result["supplementary"] = supplementary(device, stream, peaks, flush, sampler)
        result["cpu_baseline"] = cpu_baseline_leg()
    sampler.stop()
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def profile_target(name, reps):
    """Set up one workload, run it `reps` times (after two warm-up runs) and print the mean time."""
    import torch

    import fp8_quantization_amax_b200 as fq
    import synth
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        if name.startswith("gemm") and not name.startswith("gemm_mx"):
            if name in ("gemm_70b_up_m16384", "gemm_70b_up_m64"):
                w = dev_bf16(synth.weight_70b(seed=4, which="up"), device)
                m70 = 64 if name == "gemm_70b_up_m64" else 16384
                x = dev_bf16(synth.activations_70b(seed=4, m=m70, which="up"), device)
            else:
                w = dev_bf16(synth.weight_8b(seed=1), device)
                x = dev_bf16(synth.activations(seed=1), device)
                if name == "gemm_8b_m16":
                    x = x[:16].contiguous()
            a, sa = fq.fp8_quantize(x, fq.E4M3, fq.GROUP_1x128)
            b, sb = fq.fp8_quantize(w, fq.E4M3, fq.BLOCK_128x128)
            c = torch.empty((a.shape[0], b.shape[0]), dtype=torch.bfloat16, device=device)
            fn = lambda: fq.fp8_gemm_blockscaled(a, sa, b, sb, out=c)  # noqa: E731
        elif name == "linear_fused_8b_m8192":
            x = dev_bf16(synth.activations(seed=1), device)
            b, sb = fq.fp8_quantize(dev_bf16(synth.weight_8b(seed=1), device), fq.E4M3, fq.BLOCK_128x128)
            c = torch.empty((x.shape[0], b.shape[0]), dtype=torch.bfloat16, device=device)
            actf = torch.zeros(fq.linear_fused_workspace_bytes(x.shape[0], x.shape[1]), dtype=torch.uint8,
                               device=device)
            fn = lambda: fq.fp8_linear_dynamic_fused(x, b, sb, out=c, act_ws=actf)  # noqa: E731
        elif name == "gemm_mx_8b_m8192":
            a, sa = fq.fp8_quantize_mx_blocked(dev_bf16(synth.activations(seed=1), device))
            b, sb = fq.fp8_quantize_mx_blocked(dev_bf16(synth.weight_8b(seed=1), device))
            c = torch.empty((a.shape[0], b.shape[0]), dtype=torch.bfloat16, device=device)
            fn = lambda: fq.fp8_gemm_mx(a, sa, b, sb, out=c)  # noqa: E731
        elif name == "kv_delayed":
            k, v = synth.kv_70b(seed=3)
            kd, vd = dev_bf16(k, device), dev_bf16(v, device)
            hk = torch.zeros((4, 8), dtype=torch.float32, device=device)
            hv = torch.zeros_like(hk)
            r = fq.fp8_kv_quantize_delayed(kd, vd, hk, hv, 0, fq.E4M3, fq.KV_PER_HEAD)
            step_no = [0]

            def fn():
                step_no[0] += 1
                fq.fp8_kv_quantize_delayed(kd, vd, hk, hv, step_no[0], fq.E4M3, fq.KV_PER_HEAD, *r)
        elif name.startswith("kv"):
            k, v = synth.kv_70b(seed=3)
            kd, vd = dev_bf16(k, device), dev_bf16(v, device)
            gran = fq.KV_PER_HEAD_TOK128 if name == "kv_tok128" else fq.KV_PER_HEAD
            r = fq.fp8_kv_quantize(kd, vd, fq.E4M3, gran)
            fn = lambda: fq.fp8_kv_quantize(kd, vd, fq.E4M3, gran, *r)  # noqa: E731
        elif name == "mx_8b":
            xa = dev_bf16(synth.activations(seed=1), device)
            mc, msc = fq.fp8_quantize_mx(xa)
            fn = lambda: fq.fp8_quantize_mx(xa, fq.E4M3, codes=mc, scales=msc)  # noqa: E731
        else:
            w = dev_bf16(synth.weight_8b(seed=1), device)
            wc, ws = fq.fp8_quantize(w, fq.E4M3, fq.BLOCK_128x128)
            y = torch.empty_like(w)
            fn = lambda: fq.fp8_dequantize(wc, ws, fq.E4M3, fq.BLOCK_128x128, out=y)  # noqa: E731
        for _ in range(2):
            fn()
        ms = timed(fn, max(reps, 1), stream, min_reps=1)
    print(json.dumps({"profile_target": name, "reps": reps, "ms": round(ms, 4)}), flush=True)
    return 0 if fq.device_status() == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-supplementary", action="store_true")
    ap.add_argument("--skip-extras", action="store_true",
                    help="time the steps only: no e2e, CPU baseline or supplementary kernels (for profiling)")
    ap.add_argument("--profile-target", default=None,
                    choices=["gemm_8b_m8192", "gemm_8b_m16", "linear_fused_8b_m8192", "gemm_mx_8b_m8192", "gemm_70b_up_m16384", "gemm_70b_up_m64", "kv_tok128", "kv_head",
                             "kv_delayed", "mx_8b", "dequant_8b"],
                    help="run one workload a few times and exit (a small target for ncu)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return reference_arm(args)
    if args.profile_target:
        return profile_target(args.profile_target, args.steps)
    return our_arm(args)


if __name__ == "__main__":
    sys.exit(main())
