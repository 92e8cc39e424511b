"""Benchmark of the OPQ hot path on B200: quantize -> linear -> dequantize.

One step = opq_quantize(W) + opq_linear(x, W') + opq_dequantize(W') on the DiT
attention-projection workload (x 3072x3840 N(0,1), W 3840x3840 Student-t(4),
std 0.02, 0.1% outlier rows, alpha = 0.73), inputs resident in HBM. The line's
value is the step's linear TFLOP/s (2 M N K per step over the step time,
summed over ranks); per-kernel figures, the small-M weight-streaming sweep
and the roofline of the dominant kernel are reported beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl opq|reference]

Multi-GPU runs (torchrun, one rank per GPU) are weak-scaling replicas: every
rank runs the same independent step; timing is the max over ranks.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["bit_diffusion_transformer_b200/csrc/opq_linear_wide.cuh",
                  "bit_diffusion_transformer_b200/csrc/opq_linear.cuh", "bit_diffusion_transformer_b200/csrc/opq_bits.h",
                  "bit_diffusion_transformer_b200/csrc/opq_device.cuh"]
METRIC = "opq_linear TFLOP/s (% bf16 peak) & quantize/small-M weight GB/s (% HBM)"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it matches the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (all ranks take part; one rank returns its own)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_replica: float, ms: float) -> float:
    """Weak-scaling replicas: every rank runs the same step; the job's rate is all ranks' work
    over the slowest rank's time."""
    return world * flops_per_replica / (ms * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.reader = threading.Thread(target=self._read, daemon=True)
            self.reader.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, start: bool):
        """Bracket the timed region: only samples taken inside it are summarised."""
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        t0, t1 = getattr(self, "t0", 0.0), getattr(self, "t1", float("inf"))
        out = self._summarise(t0, t1 + 0.05)
        if out["sm_mhz"] is None:
            # a timed region shorter than the sampling interval: the samples next to it
            out = self._summarise(t0 - 0.15, t1 + 0.15)
            if out["sm_mhz"] is not None:
                out["window"] = "adjacent samples (timed region shorter than the 20 ms sampling interval)"
        return out

    def _summarise(self, lo, hi):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if not (lo <= ts <= hi):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- GPU arm
def gpu_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bit_diffusion_transformer_b200 as opq
    import workloads

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    opq.load()
    lin = workloads.dit_attn_proj()
    M, N, K, alpha = lin.M, lin.N, lin.K, lin.alpha
    x, w = lin.make(dev)
    codes = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
    signs = torch.empty((N, K // 32), dtype=torch.int32, device=dev)
    scales = torch.empty((N,), dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    wq = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    ws_bytes = opq.workspace_size(M, N, K)
    ws = torch.zeros((max(ws_bytes, 16),), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty((4 * max(l2, 64 << 20),), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        # ev: optional 4 events bracketing the three launches (timed region only)
        if ev is not None:
            ev[0].record(stream)
        opq.quantize(w, alpha, out=(codes, signs, scales))
        if ev is not None:
            ev[1].record(stream)
        opq.linear(x, codes, signs, scales, alpha, out=y, workspace=ws)
        if ev is not None:
            ev[2].record(stream)
        opq.dequantize(codes, signs, scales, alpha, out=wq)
        if ev is not None:
            ev[3].record(stream)

    launches_per_step = 1 + opq.plan(M, N, K)[2] + 1

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert opq.device_error() == 0

    # ---- timed region: K steps, L2 flushed between steps (outside the event pairs); the
    # events bracketing each launch give the per-kernel durations of the same region
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        clocks.mark(True)
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
        clocks.mark(False)
    barrier()
    per_step = [e[0].elapsed_time(e[3]) for e in evs]
    live = {name: statistics.fmean(e[a].elapsed_time(e[b]) for e in evs)
            for name, a, b in (("quantize", 0, 1), ("linear", 1, 2), ("dequantize", 2, 3))}
    ms_step = max_over_ranks(sum(per_step) / len(per_step), world, dev)
    assert opq.device_error() == 0
    flops = 2.0 * M * N * K
    value = whole_job_tflops(world, flops, ms_step)

    # ---- per-kernel timings (events on the launching stream, L2 flushed before each)
    def time_kernel(fn, reps=20):
        ts = []
        for _ in range(reps):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts), ts

    peaks, peak_src = load_peaks()
    # mean launch durations inside the timed region (each launch starts with a flushed L2)
    t_q, t_l, t_d = live["quantize"], live["linear"], live["dequantize"]
    q_bytes = N * K * 2 + N * K // 8 * 5 + 4 * N      # read W, write codes (K/2 B) + signs (K/8 B) + scales
    d_bytes = N * K // 8 * 5 + 4 * N + N * K * 2
    l_bytes = N * K * 5 // 8 + 4 * N + 2 * M * K + 2 * M * N
    linear_tflops = flops / (t_l * 1e-3) / 1e12
    kernels = {
        "quantize": {"ms": t_q, "gbs": q_bytes / (t_q * 1e-3) / 1e9,
                     "frac_hbm": q_bytes / (t_q * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "linear": {"ms": t_l, "tflops": linear_tflops, "frac_bf16": linear_tflops / peaks["bf16_tflops"],
                   "path": opq.plan(M, N, K)[0]},
        "dequantize": {"ms": t_d, "gbs": d_bytes / (t_d * 1e-3) / 1e9,
                       "frac_hbm": d_bytes / (t_d * 1e-3) / 1e9 / peaks["hbm_gbs"]},
    }

    # ---- weight-streaming sweep (fused-QKV 11520x3840, M in {1, 16, 64, 256})
    small = {}
    if not args.no_sweep:
        qkv = workloads.small_m(1)
        wqkv = qkv.make_weights(dev)
        pq = opq.quantize(wqkv, alpha)
        for m in workloads.SMALL_M_SWEEP:
            xm = workloads.small_m(m).make_x(dev)
            ym = torch.empty((m, qkv.N), dtype=torch.bfloat16, device=dev)
            wsm = torch.zeros((max(opq.workspace_size(m, qkv.N, qkv.K), 16),), dtype=torch.uint8, device=dev)
            fn = lambda: opq.linear(xm, *pq, alpha, out=ym, workspace=wsm)
            for _ in range(3):
                fn()
            tm, _ = time_kernel(fn, reps=30)
            wbytes = qkv.N * qkv.K * 5 // 8 + 4 * qkv.N
            abytes = wbytes + 2 * m * qkv.K + 2 * m * qkv.N
            fl = 2.0 * m * qkv.N * qkv.K
            small[str(m)] = {"us": tm * 1e3, "weight_gbs": wbytes / (tm * 1e-3) / 1e9,
                             "bytes_gbs": abytes / (tm * 1e-3) / 1e9,
                             "frac_hbm": abytes / (tm * 1e-3) / 1e9 / peaks["hbm_gbs"],
                             "tflops": fl / (tm * 1e-3) / 1e12, "plan": list(opq.plan(m, qkv.N, qkv.K))}
        del wqkv, pq
        assert opq.device_error() == 0

    # ---- the group-wise format (the model card's own storage: one float16 max per GS weights)
    # on the same weight and activations: quantize, linear, dequantize at GS = 128 and 32
    grouped = {}
    if not args.no_sweep:
        wq_g = torch.empty_like(w)
        y_g = torch.empty_like(y)
        for gs in (128, 32):
            cg, sg, gg = opq.quantize_grouped(w, gs, alpha)
            ws_g = torch.zeros((max(opq.grouped_workspace_size(M, N, K, gs), 16),), dtype=torch.uint8, device=dev)
            fq = lambda: opq.quantize_grouped(w, gs, alpha, out=(cg, sg, gg))
            fl_ = lambda: opq.linear_grouped(x, cg, sg, gg, alpha, out=y_g, workspace=ws_g)
            fd = lambda: opq.dequantize_grouped(cg, sg, gg, alpha, out=wq_g)
            for f_ in (fq, fl_, fd):
                for _ in range(3):
                    f_()
            tq_, _ = time_kernel(fq)
            tl_, _ = time_kernel(fl_)
            td_, _ = time_kernel(fd)
            gq_bytes = N * K * 2 + N * K // 8 * 5 + 2 * N * (K // gs)
            gd_bytes = N * K // 8 * 5 + 2 * N * (K // gs) + N * K * 2
            g_tflops = flops / (tl_ * 1e-3) / 1e12
            grouped[str(gs)] = {
                "quantize": {"ms": tq_, "gbs": gq_bytes / (tq_ * 1e-3) / 1e9,
                             "frac_hbm": gq_bytes / (tq_ * 1e-3) / 1e9 / peaks["hbm_gbs"]},
                "linear": {"ms": tl_, "tflops": g_tflops, "frac_bf16": g_tflops / peaks["bf16_tflops"]},
                "dequantize": {"ms": td_, "gbs": gd_bytes / (td_ * 1e-3) / 1e9,
                               "frac_hbm": gd_bytes / (td_ * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            }
            del ws_g
        del wq_g, y_g
        assert opq.device_error() == 0

    # ---- the other bit widths of the card's configuration (3, 5, 6: 2^bits - 1 levels, codes as
    # one bit stream per row) on the same weight: quantize, dequantize, and the SNR of each width
    bits_out = {}
    fused = {}
    if not args.no_sweep:
        wq_b = torch.empty_like(w)
        for b_ in (3, 5, 6):
            cb, sb, fb = opq.quantize_bits(w, b_, alpha)
            fq = lambda: opq.quantize_bits(w, b_, alpha, out=(cb, sb, fb))
            fd = lambda: opq.dequantize_bits(cb, sb, fb, b_, alpha, out=wq_b)
            for f_ in (fq, fd):
                for _ in range(3):
                    f_()
            tq_, _ = time_kernel(fq)
            td_, _ = time_kernel(fd)
            packed = N * K * b_ // 8 + N * K // 8 + 4 * N
            bq_bytes = N * K * 2 + packed
            bd_bytes = packed + N * K * 2
            bits_out[str(b_)] = {
                "quantize": {"ms": tq_, "gbs": bq_bytes / (tq_ * 1e-3) / 1e9,
                             "frac_hbm": bq_bytes / (tq_ * 1e-3) / 1e9 / peaks["hbm_gbs"]},
                "dequantize": {"ms": td_, "gbs": bd_bytes / (td_ * 1e-3) / 1e9,
                               "frac_hbm": bd_bytes / (td_ * 1e-3) / 1e9 / peaks["hbm_gbs"]},
                "snr_db": None}
            opq.dequantize_bits(cb, sb, fb, b_, alpha, out=wq_b)
            r_ = w.double()
            bits_out[str(b_)]["snr_db"] = float(10.0 * torch.log10((r_ * r_).sum() / ((r_ - wq_b.double()) ** 2).sum()))
            del cb, sb, fb
        del wq_b
        # the linear with its epilogue fused (bias + SiLU), as the layer an nn.Linear + activation
        # becomes: same weight, activations and schedule as the step's linear
        bias = (torch.arange(N, device=dev, dtype=torch.float32) * 1e-3 - 1.0).to(torch.bfloat16)
        y_f = torch.empty_like(y)
        for act in ("silu", "gelu_tanh"):
            ff = lambda: opq.linear_fused(x, codes, signs, scales, alpha, bias=bias, act=act, out=y_f, workspace=ws)
            for _ in range(3):
                ff()
            tf_, _ = time_kernel(ff)
            f_tflops = flops / (tf_ * 1e-3) / 1e12
            fused[act] = {"ms": tf_, "tflops": f_tflops, "frac_bf16": f_tflops / peaks["bf16_tflops"]}
        del y_f
        assert opq.device_error() == 0

    # ---- SNR context (the model card's "+7.2 dB" claim is on Z-Image weights; these are the
    # synthetic Student-t weights of the bench workload): OPQ through the library at alpha 0.73
    # and 1.0 (same 4-bit + sign + row max format), and per-row symmetric INT4 round(w/(max/7))
    def snr_db(ref, rec):
        r = ref.double()
        return float(10.0 * torch.log10((r * r).sum() / ((r - rec.double()) ** 2).sum()))

    w_rec = torch.empty_like(w)
    snr = {}
    for a_ in (alpha, 1.0):
        p_ = opq.quantize(w, a_)
        opq.dequantize(*p_, a_, out=w_rec)
        snr[f"opq_alpha_{a_:g}"] = snr_db(w, w_rec)
    wf = w.float()
    step7 = wf.abs().amax(dim=1, keepdim=True).clamp_min(1e-30) / 7.0
    snr["int4_symmetric_row"] = snr_db(w, (torch.round(wf / step7).clamp(-7, 7) * step7).to(torch.bfloat16))
    p_ = opq.quantize_grouped(w, 128, alpha)
    opq.dequantize_grouped(*p_, alpha, out=w_rec)
    snr[f"opq_alpha_{alpha:g}_group128"] = snr_db(w, w_rec)
    if not args.no_sweep:
        # the alpha search over 0.30 .. 1.00 (the card's configuration range) on this weight
        for gs_ in (0, 128):
            best_a, snrs = opq.alpha_search(w, opq.ALPHA_GRID, gs_)
            snr[f"alpha_search_{'row' if gs_ == 0 else 'group128'}"] = {
                "best_alpha": best_a, "snr_db": dict(zip([f"{a_:.2f}" for a_ in opq.ALPHA_GRID], snrs))}
    snr["gain_vs_int4_db"] = snr[f"opq_alpha_{alpha:g}"] - snr["int4_symmetric_row"]
    snr["gain_vs_alpha1_db"] = snr[f"opq_alpha_{alpha:g}"] - snr["opq_alpha_1"]
    snr["model_card_claim_db"] = 7.2
    del w_rec

    # ---- end to end through the public API with host buffers
    w_host = w.cpu().pin_memory()
    x_host = x.cpu().pin_memory()
    y_host = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    w_dev = torch.empty_like(w)
    x_dev = torch.empty_like(x)

    def e2e_step():
        w_dev.copy_(w_host, non_blocking=True)
        x_dev.copy_(x_host, non_blocking=True)
        opq.quantize(w_dev, alpha, out=(codes, signs, scales))
        opq.linear(x_dev, codes, signs, scales, alpha, out=y, workspace=ws)
        opq.dequantize(codes, signs, scales, alpha, out=wq)
        y_host.copy_(y, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(args.steps):
        e2e_step()
    eb.record(stream)
    eb.synchronize()
    ms_e2e = max_over_ranks(ea.elapsed_time(eb) / args.steps, world, dev)
    barrier()

    traffic = recorded_traffic("wide_kernel")
    roof = {"bound": "tensor", "kernel": "wide_kernel<256>", "achieved": linear_tflops,
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": linear_tflops / peaks["bf16_tflops"],
            "traffic": traffic, "algorithmic_flops": flops, "algorithmic_bytes": l_bytes,
            "launch_ms": t_l, "peak_source": f"bf16 dense burst, {peak_src}"}
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Student-t(4) weights, N(0,1) activations)",
        "config": {"workload": lin.name, "M": M, "N": N, "K": K, "alpha": alpha,
                   "step": "quantize W + linear x W'^T + dequantize W'", "parallelism": f"replicas{world}",
                   "l2": "flushed between timed steps (4x L2 buffer write outside the event pairs)"},
        "kernels": kernels, "small_m": small, "grouped": grouped, "bits": bits_out, "fused": fused,
        "roofline": roof, "snr_db": snr,
        "e2e": {"value": whole_job_tflops(world, flops, ms_e2e), "unit": "TFLOP/s", "ms_per_step": ms_e2e,
                "h2d_bytes_per_step": w.numel() * 2 + x.numel() * 2, "d2h_bytes_per_step": y.numel() * 2},
        "gpu_launches": launches_per_step * args.steps,
        "kernels_live_ms": live,
        "clocks": clocks.summary(),
        "peaks": peaks,
    }
    return out


# --------------------------------------------------------------------------- CPU arms
def cpu_oracle_sample(budget_s: float = 12.0):
    """Time the fp64 oracle on a bounded sample of the bench workload: quantize 256
    weight rows and the linear for 16 activation rows against those 256 weight rows."""
    import numpy as np
    import oracle
    import workloads

    lin = workloads.dit_attn_proj()
    x, w = lin.make("cpu")
    rows = 256
    xs, ws = x[:16].contiguous(), w[:rows].contiguous()
    oracle.build()
    t0 = time.perf_counter()
    reps = 0
    while True:
        r = oracle.quantize(ws, lin.alpha)
        oracle.linear(xs, r["codes"], r["signs"], r["scales"], lin.alpha)
        reps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = (time.perf_counter() - t0) / reps
    flops = 2.0 * xs.shape[0] * rows * lin.K
    cores = oracle.num_threads()
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"quantize {rows}x{lin.K} + linear {xs.shape[0]}x{lin.K} @ {rows}x{lin.K}^T "
                      f"({reps} reps, {dt:.3f} s each)",
            "seconds_per_sample": dt}


def reference_arm(args):
    import oracle
    import workloads
    lin = workloads.dit_attn_proj()
    x, w = lin.make("cpu")
    xs, ws = x[:16].contiguous(), w[:256].contiguous()
    oracle.build()
    for _ in range(args.warmup):
        r = oracle.quantize(ws, lin.alpha)
        oracle.linear(xs, r["codes"], r["signs"], r["scales"], lin.alpha)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        r = oracle.quantize(ws, lin.alpha)
        oracle.linear(xs, r["codes"], r["signs"], r["scales"], lin.alpha)
        ts.append(time.perf_counter() - t0)
    dt = sum(ts) / len(ts)
    flops = 2.0 * xs.shape[0] * ws.shape[0] * lin.K
    v = flops / dt / 1e12
    cores = oracle.num_threads()
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": lin.name, "sample": "quantize 256 weight rows + linear 16 x 256 outputs",
                       "parallelism": "cpu"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": "quantize 256x3840 + linear 16x3840 @ 256x3840^T per step"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_run(args):
    """A short, fixed launch sequence of one kernel for ncu (no timing, no sweep)."""
    import torch
    import bit_diffusion_transformer_b200 as opq
    import workloads
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.profile.startswith("small"):
        lin = workloads.small_m(int(args.profile[5:]))
    else:
        lin = workloads.dit_attn_proj()
    x, w = lin.make(dev)
    planes = opq.quantize(w, lin.alpha)
    y = torch.empty((lin.M, lin.N), dtype=torch.bfloat16, device=dev)
    wq = torch.empty_like(w)
    ws = torch.zeros((max(opq.workspace_size(lin.M, lin.N, lin.K), 16),), dtype=torch.uint8, device=dev)
    gplanes = opq.quantize_grouped(w, 128, lin.alpha)
    gws = torch.zeros((max(opq.grouped_workspace_size(lin.M, lin.N, lin.K, 128), 16),), dtype=torch.uint8, device=dev)
    fns = {"quantize": lambda: opq.quantize(w, lin.alpha, out=planes),
           "dequantize": lambda: opq.dequantize(*planes, lin.alpha, out=wq),
           "grouped_quantize": lambda: opq.quantize_grouped(w, 128, lin.alpha, out=gplanes),
           "grouped_linear": lambda: opq.linear_grouped(x, *gplanes, lin.alpha, out=y, workspace=gws)}
    fn = fns.get(args.profile, lambda: opq.linear(x, *planes, lin.alpha, out=y, workspace=ws))
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    assert opq.device_error() == 0
    print(json.dumps({"profile": args.profile, "workload": lin.name, "launches": args.steps}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="opq", choices=["opq", "reference"])
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", default=None,
                    help="profiling run: warm up, then launch only this kernel --steps times "
                         "(quantize | linear | dequantize | grouped_quantize | grouped_linear | small<M>) "
                         "on the bench workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(reference_arm(args)), flush=True)
        return 0

    if args.profile:
        return profile_run(args)

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    out = gpu_arm(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_oracle_sample()
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
