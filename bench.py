"""Benchmark of the OPQ hot path on B200: quantize -> linear -> dequantize.

Headline workload: the whole-model pass of a synthetic diffusion transformer,
30 blocks x (4 attention matrices 3840x3840, two FFN up-projections 10240x3840,
one down-projection 3840x10240) = 210 matrices, 5.31 G weights (10.62 GB bf16,
Student-t(4), std 0.02, alpha = 0.73), activations 3072 x K N(0,1). One step =
quantize all 210 matrices, opq_linear at M = 3072 on every layer, dequantize
all 210; inputs resident in HBM and 84x larger than L2. The line's value is the
step's linear TFLOP/s (2 M N K summed over the layers, over the step time,
summed over ranks); quantize-all GB/s, linear TFLOP/s per shape class and the
roofline of the dominant kernel are reported beside it, with the FFN pair at
three alphas, the attention projection, the small-M weight-streaming sweep
and the library's other formats as extras.

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
import math
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




# --------------------------------------------------------------------------- byte / flop counts
def quant_bytes(N, K):
    """quantize: read W (2 B), write codes (K/2 B) + signs (K/8 B) per row, and the fp32 scales."""
    return N * K * 2 + N * K // 8 * 5 + 4 * N


def dequant_bytes(N, K):
    return N * K // 8 * 5 + 4 * N + N * K * 2


def linear_bytes(M, N, K):
    return N * K * 5 // 8 + 4 * N + 2 * M * K + 2 * M * N


# shape classes of the whole-model pass: (name, N, K)
WM_CLASSES = (("attn_3840x3840", 3840, 3840), ("ffn_up_10240x3840", 10240, 3840),
              ("ffn_down_3840x10240", 3840, 10240))


def wm_class(N, K):
    for name, n, k in WM_CLASSES:
        if (n, k) == (N, K):
            return name
    raise ValueError((N, K))


class WholeModelState:
    """Device buffers of the whole-model pass: every layer's W, packed planes and W' are
    views into one allocation per tensor kind; one activation tensor per K and one output
    per N (every layer runs at M = 3072)."""

    def __init__(self, dev, opq, workloads, torch):
        self.model = workloads.WholeModel()
        self.M, self.alpha = self.model.M, self.model.alpha
        total = self.model.weights
        rows = sum(l.N for l in self.model.layers)
        bf16 = torch.bfloat16
        self.W = torch.empty((total,), dtype=bf16, device=dev)
        self.Wq = torch.empty((total,), dtype=bf16, device=dev)
        self.codes = torch.empty((total // 8,), dtype=torch.int32, device=dev)
        self.signs = torch.empty((total // 32,), dtype=torch.int32, device=dev)
        self.scales = torch.empty((rows,), dtype=torch.float32, device=dev)
        self.layers = []
        off = roff = 0
        for l in self.model.layers:
            n, k = l.N, l.K
            L = {"name": l.name, "N": n, "K": k, "cls": wm_class(n, k), "off": off,
                 "w": self.W[off:off + n * k].view(n, k), "wq": self.Wq[off:off + n * k].view(n, k),
                 "c": self.codes[off // 8:(off + n * k) // 8].view(n, k // 8),
                 "s": self.signs[off // 32:(off + n * k) // 32].view(n, k // 32),
                 "sc": self.scales[roff:roff + n]}
            # each layer's draw comes from its own seeded generator on the device
            L["w"].copy_(l.make_weights(dev))
            self.layers.append(L)
            off += n * k
            roff += n
        first = {}
        for l in self.model.layers:
            first.setdefault(l.K, l)
        self.x = {k: l.make_x(dev) for k, l in first.items()}
        self.y = {n: torch.empty((self.M, n), dtype=bf16, device=dev) for n in {l.N for l in self.model.layers}}
        need = max(opq.workspace_size(self.M, l.N, l.K) for l in self.model.layers)
        self.ws = torch.zeros((max(need, 16),), dtype=torch.uint8, device=dev)
        self.by_class = {c[0]: [L for L in self.layers if L["cls"] == c[0]] for c in WM_CLASSES}
        # one opq_quantize_batched call per shape class quantizes all its matrices in one stream
        self.jobs = {c: (opq.quantize_jobs([L["w"] for L in Ls], [(L["c"], L["s"], L["sc"]) for L in Ls],
                                           self.alpha), [L["w"] for L in Ls],
                         [(L["c"], L["s"], L["sc"]) for L in Ls]) for c, Ls in self.by_class.items()}
        # and one opq_dequantize_batched call per shape class decodes them back
        self.djobs = {c: (opq.dequantize_jobs([(L["c"], L["s"], L["sc"]) for L in Ls], [L["wq"] for L in Ls]),
                          [(L["c"], L["s"], L["sc"]) for L in Ls], [L["wq"] for L in Ls])
                      for c, Ls in self.by_class.items()}

    def phase(self, opq, what, cls):
        a, M = self.alpha, self.M
        if what == "quantize":
            jobs, ws, outs = self.jobs[cls]
            opq.quantize_batched(ws, a, outs=outs, jobs=jobs)
            return
        if what == "dequantize":
            jobs, planes, outs = self.djobs[cls]
            opq.dequantize_batched(planes, a, outs=outs, jobs=jobs)
            return
        for L in self.by_class[cls]:
            opq.linear(self.x[L["K"]], L["c"], L["s"], L["sc"], a, out=self.y[L["N"]], workspace=self.ws)

    def counts(self, cls):
        Ls = self.by_class[cls]
        return {"matrices": len(Ls),
                "quantize_bytes": sum(quant_bytes(L["N"], L["K"]) for L in Ls),
                "dequantize_bytes": sum(dequant_bytes(L["N"], L["K"]) for L in Ls),
                "linear_flops": sum(2.0 * self.M * L["N"] * L["K"] for L in Ls),
                "linear_bytes": sum(linear_bytes(self.M, L["N"], L["K"]) for L in Ls)}


PHASES = ("quantize", "linear", "dequantize")


def capture_graph(torch, fn):
    """One CUDA graph of the launches `fn` enqueues (the library's calls are plain kernel
    launches on the current stream; nothing is allocated inside)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        fn()
    return g


# --------------------------------------------------------------------------- GPU arm
def gpu_arm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bit_diffusion_transformer_b200 as opq
    import workloads

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    opq.load()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty((4 * max(l2, 64 << 20),), dtype=torch.uint8, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def time_kernel(fn, reps=20, flush_l2=True):
        """Median duration of one call, events on the launching stream, L2 flushed before each."""
        ts = []
        for _ in range(reps):
            if flush_l2:
                flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    # ---------------------------------------------------------------- the whole-model step
    S = WholeModelState(dev, opq, workloads, torch)
    M, alpha = S.M, S.alpha
    cls_names = [c[0] for c in WM_CLASSES]
    for what in PHASES:                      # eager pass: kernel attributes, TMA encoder lookup
        for c in cls_names:
            S.phase(opq, what, c)
    torch.cuda.synchronize()
    assert opq.device_error() == 0
    graphs = {(what, c): capture_graph(torch, lambda w_=what, c_=c: S.phase(opq, w_, c_))
              for what in PHASES for c in cls_names}
    order = [(what, c) for what in PHASES for c in cls_names]

    def step(ev=None):
        for i, key in enumerate(order):
            if ev is not None:
                ev[i].record(stream)
            graphs[key].replay()
        if ev is not None:
            ev[len(order)].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert opq.device_error() == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(order) + 1)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        clocks.mark(True)
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
        clocks.mark(False)
    barrier()
    assert opq.device_error() == 0
    per_step = [e[0].elapsed_time(e[-1]) for e in evs]
    seg = {key: statistics.fmean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, key in enumerate(order)}
    ms_step = max_over_ranks(statistics.fmean(per_step), world, dev)
    cnt = {c: S.counts(c) for c in cls_names}
    flops = sum(cnt[c]["linear_flops"] for c in cls_names)
    value = whole_job_tflops(world, flops, ms_step)
    hbm, bf16 = peaks["hbm_gbs"], peaks["bf16_tflops"]
    bf16_sus = peaks.get("bf16_tflops_sustained", bf16)

    def gbs_entry(ms, nbytes, extra=None):
        g = nbytes / (ms * 1e-3) / 1e9
        d = {"ms": ms, "gbs": g, "frac_hbm": g / hbm, "bytes": nbytes}
        d.update(extra or {})
        return d

    def tf_entry(ms, fl, extra=None):
        t = fl / (ms * 1e-3) / 1e12
        d = {"ms": ms, "tflops": t, "frac_bf16": t / bf16, "frac_bf16_sustained": t / bf16_sus}
        d.update(extra or {})
        return d

    kernels = {}
    for what, key_b in (("quantize", "quantize_bytes"), ("dequantize", "dequantize_bytes")):
        ms = sum(seg[(what, c)] for c in cls_names)
        kernels[f"{what}_all"] = gbs_entry(ms, sum(cnt[c][key_b] for c in cls_names), {
            "matrices": len(S.layers),
            "by_class": {c: gbs_entry(seg[(what, c)], cnt[c][key_b], {"matrices": cnt[c]["matrices"]})
                         for c in cls_names}})
    ms_lin = sum(seg[("linear", c)] for c in cls_names)
    kernels["linear_all"] = tf_entry(ms_lin, flops, {
        "layers": len(S.layers), "M": M,
        "by_class": {c: tf_entry(seg[("linear", c)], cnt[c]["linear_flops"],
                                 {"layers": cnt[c]["matrices"], "plan": list(opq.plan(M, *[(n, k) for nm, n, k in WM_CLASSES if nm == c][0]))})
                     for c in cls_names}})
    # library kernels per step: the batched quantize and dequantize (one launch per 128 matrices of
    # a class each) and one linear per layer
    launches_per_step = 2 * sum(-(-cnt[c]["matrices"] // 128) for c in cls_names) + len(S.layers)
    linear_tflops = kernels["linear_all"]["tflops"]

    # ---------------------------------------------------------------- e2e: host buffers
    # Every step copies all 210 weights and both activation tensors from host memory, runs
    # the three phases through the public calls and copies every layer's y back to the host.
    # The step is pipelined by transformer block (7 layers): the block's weights go up on a
    # copy stream, its quantize (one batched call), linears and dequantizes run on the compute
    # stream once they have landed, and each layer's y goes down on a second copy stream as
    # soon as its linear is done (both copy directions run at once). Steps do not overlap.
    e2e = None
    if not args.no_e2e:
        total_bytes = S.W.numel() * 2
        w_host = torch.empty((S.W.numel(),), dtype=torch.bfloat16)
        w_host.copy_(S.W)
        cudart = torch.cuda.cudart()
        reg = cudart.cudaHostRegister(w_host.data_ptr(), total_bytes, 0)
        registered = int(reg) == 0
        x_host = {k: v.cpu().pin_memory() for k, v in S.x.items()}
        blocks = [S.layers[i:i + 7] for i in range(0, len(S.layers), 7)]
        bjobs = [(opq.quantize_jobs([L["w"] for L in B], [(L["c"], L["s"], L["sc"]) for L in B], alpha),
                  [L["w"] for L in B], [(L["c"], L["s"], L["sc"]) for L in B]) for B in blocks]
        bdjobs = [(opq.dequantize_jobs([(L["c"], L["s"], L["sc"]) for L in B], [L["wq"] for L in B]),
                   [(L["c"], L["s"], L["sc"]) for L in B], [L["wq"] for L in B]) for B in blocks]
        y_dev = [torch.empty((M, L["N"]), dtype=torch.bfloat16, device=dev) for L in S.layers]
        y_host = [torch.empty((M, L["N"]), dtype=torch.bfloat16).pin_memory() for L in S.layers]
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def e2e_step():
            s_up.wait_stream(stream)
            s_down.wait_stream(stream)
            landed = []
            with torch.cuda.stream(s_up):
                for k in S.x:
                    S.x[k].copy_(x_host[k], non_blocking=True)
                for B in blocks:
                    for L in B:
                        n, k = L["N"], L["K"]
                        L["w"].copy_(w_host[L["off"]:L["off"] + n * k].view(n, k), non_blocking=True)
                    e = torch.cuda.Event()
                    e.record(s_up)
                    landed.append(e)
            done = []
            i = 0
            for B, (jobs, ws_, outs_), (djobs, dplanes, douts), e in zip(blocks, bjobs, bdjobs, landed):
                stream.wait_event(e)
                opq.quantize_batched(ws_, alpha, outs=outs_, jobs=jobs)
                for L in B:
                    opq.linear(S.x[L["K"]], L["c"], L["s"], L["sc"], alpha, out=y_dev[i], workspace=S.ws)
                    ev = torch.cuda.Event()
                    ev.record(stream)
                    done.append(ev)
                    i += 1
                opq.dequantize_batched(dplanes, alpha, outs=douts, jobs=djobs)
            with torch.cuda.stream(s_down):
                for i, ev in enumerate(done):
                    s_down.wait_event(ev)
                    y_host[i].copy_(y_dev[i], non_blocking=True)
            stream.wait_stream(s_up)
            stream.wait_stream(s_down)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e_steps = max(1, min(args.steps, 3))
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record(stream)
        for _ in range(e_steps):
            e2e_step()
        eb.record(stream)
        eb.synchronize()
        ms_e2e = max_over_ranks(ea.elapsed_time(eb) / e_steps, world, dev)
        barrier()
        assert opq.device_error() == 0
        h2d = total_bytes + sum(v.numel() * 2 for v in S.x.values())
        d2h = sum(M * L["N"] * 2 for L in S.layers)
        e2e = {"value": whole_job_tflops(world, flops, ms_e2e), "unit": "TFLOP/s", "ms_per_step": ms_e2e,
               "steps": e_steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "host_weights": "registered (page-locked) host memory" if registered else "pageable host memory",
               "copies": "210 weight H2D + 2 activation H2D + 210 y D2H per step",
               "pipeline": "per transformer block: weights up on one copy stream, quantize (one batched call) + "
                           "linears + dequantize (one batched call) on the compute stream, each y down on another "
                           "copy stream"}
        if registered:
            cudart.cudaHostUnregister(w_host.data_ptr())
        del w_host, y_dev, y_host
    traffic = recorded_traffic("wide_kernel_whole_model")
    roof = {"bound": "tensor", "kernel": "opqk_wide::wide_kernel<256, 0>", "achieved": linear_tflops,
            "peak": bf16, "unit": "TFLOP/s", "frac": linear_tflops / bf16,
            "frac_of_sustained_peak": linear_tflops / bf16_sus, "traffic": traffic,
            "algorithmic_flops_per_launch": flops / len(S.layers),
            "algorithmic_bytes_per_launch": sum(cnt[c]["linear_bytes"] for c in cls_names) / len(S.layers),
            "launch_ms": ms_lin / len(S.layers), "launches": len(S.layers),
            "peak_source": f"bf16 dense burst, {peak_src} (frac_of_sustained_peak: the power-capped loop)",
            "note": "achieved = the 210 layers' 2 M N K over their summed launch durations (the mean "
                    "launch of the mix); traffic = ncu DRAM bytes per launch averaged over the mix"}
    # free the whole-model buffers before the extras
    whole = {"ms_per_step": ms_step, "per_step_ms": {f"{w}:{c}": seg[(w, c)] for (w, c) in order}}
    del graphs, S
    torch.cuda.empty_cache()

    extras = {}
    if not args.no_sweep:
        extras = gpu_extras(args, opq, workloads, torch, dev, peaks, time_kernel, flush)

    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Student-t(4) weights std 0.02 drawn per layer on the device, N(0,1) activations)",
        "config": {"workload": "dit_whole_model_30blocks_210layers_m3072", "blocks": 30, "layers": 210,
                   "weights": 5308416000, "M": M, "alpha": alpha,
                   "step": "quantize all 210 W (one batched call per shape class) + linear x W'^T on every "
                           "layer (M 3072) + dequantize all 210 (one batched call per shape class)",
                   "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (10.62 GB of weights per step against a 126 MB L2); no flush",
                   "launch": "each phase and shape class is one CUDA graph of the library's launches"},
        "kernels": kernels, "whole_model": whole, "roofline": roof,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
        "peaks": peaks,
    }
    if e2e is not None:
        out["e2e"] = e2e
    out.update(extras)
    return out


def gpu_extras(args, opq, workloads, torch, dev, peaks, time_kernel, flush):
    """The FFN pair at three alphas, the attention projection step, the small-M weight
    stream, the group-wise format, other bit widths, the fused epilogue, SNR context."""
    hbm, bf16 = peaks["hbm_gbs"], peaks["bf16_tflops"]
    stream = torch.cuda.current_stream(dev)
    out = {}

    # ---- the DiT FFN pair: x 4096x3840 through W1 10240x3840, x' 4096x10240 through W2
    # 3840x10240, at alpha 0.45, 0.73 and 1.0 (the draws do not depend on alpha)
    up0, down0 = workloads.dit_ffn_pair(workloads.ALPHA)
    xu, wu = up0.make(dev)
    xd, wd = down0.make(dev)
    yu = torch.empty((up0.M, up0.N), dtype=torch.bfloat16, device=dev)
    yd = torch.empty((down0.M, down0.N), dtype=torch.bfloat16, device=dev)
    wsu = torch.zeros((max(opq.workspace_size(up0.M, up0.N, up0.K), 16),), dtype=torch.uint8, device=dev)
    wsd = torch.zeros((max(opq.workspace_size(down0.M, down0.N, down0.K), 16),), dtype=torch.uint8, device=dev)
    ffn = {}
    for a in (0.45, 0.73, 1.0):
        pu = opq.quantize(wu, a)
        pd = opq.quantize(wd, a)
        fu = lambda: opq.linear(xu, *pu, a, out=yu, workspace=wsu)
        fd = lambda: opq.linear(xd, *pd, a, out=yd, workspace=wsd)
        fq = lambda: opq.quantize(wu, a, out=pu)
        for f_ in (fu, fd, fq):
            for _ in range(3):
                f_()
        tu, td, tq = time_kernel(fu, 10), time_kernel(fd, 10), time_kernel(fq, 10)
        flu, fld = 2.0 * up0.M * up0.N * up0.K, 2.0 * down0.M * down0.N * down0.K
        qb = quant_bytes(up0.N, up0.K)
        ffn[f"{a:g}"] = {
            "up": {"ms": tu, "tflops": flu / tu / 1e9, "frac_bf16": flu / tu / 1e9 / bf16,
                   "plan": list(opq.plan(up0.M, up0.N, up0.K))},
            "down": {"ms": td, "tflops": fld / td / 1e9, "frac_bf16": fld / td / 1e9 / bf16,
                     "plan": list(opq.plan(down0.M, down0.N, down0.K))},
            "pair": {"ms": tu + td, "tflops": (flu + fld) / (tu + td) / 1e9,
                     "frac_bf16": (flu + fld) / (tu + td) / 1e9 / bf16},
            "quantize_w1": {"ms": tq, "gbs": qb / tq / 1e6, "frac_hbm": qb / tq / 1e6 / hbm}}
        del pu, pd
    assert opq.device_error() == 0
    out["ffn_pair"] = {"workload": "dit_ffn_pair x 4096x3840 @ W1 10240x3840, x' 4096x10240 @ W2 3840x10240",
                       "l2": "flushed before each launch", "by_alpha": ffn}
    del xu, wu, xd, wd, yu, yd, wsu, wsd

    # ---- the attention projection step (x 3072x3840, W 3840x3840 with outlier rows)
    lin = workloads.dit_attn_proj()
    M, N, K, alpha = lin.M, lin.N, lin.K, lin.alpha
    x, w = lin.make(dev)
    codes, signs, scales = opq.quantize(w, alpha)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    wq = torch.empty_like(w)
    ws = torch.zeros((max(opq.workspace_size(M, N, K), 16),), dtype=torch.uint8, device=dev)
    fq = lambda: opq.quantize(w, alpha, out=(codes, signs, scales))
    fl = lambda: opq.linear(x, codes, signs, scales, alpha, out=y, workspace=ws)
    fdq = lambda: opq.dequantize(codes, signs, scales, alpha, out=wq)
    for f_ in (fq, fl, fdq):
        for _ in range(3):
            f_()
    t_q, t_l, t_d = time_kernel(fq, 50), time_kernel(fl, 50), time_kernel(fdq, 50)
    flops = 2.0 * M * N * K
    out["attn_proj"] = {
        "workload": lin.name, "l2": "flushed before each launch",
        "quantize": {"ms": t_q, "gbs": quant_bytes(N, K) / t_q / 1e6, "frac_hbm": quant_bytes(N, K) / t_q / 1e6 / hbm},
        "linear": {"ms": t_l, "tflops": flops / t_l / 1e9, "frac_bf16": flops / t_l / 1e9 / bf16,
                   "plan": list(opq.plan(M, N, K))},
        "dequantize": {"ms": t_d, "gbs": dequant_bytes(N, K) / t_d / 1e6,
                       "frac_hbm": dequant_bytes(N, K) / t_d / 1e6 / hbm}}

    # ---- weight-streaming sweep: fused-QKV W 11520x3840, M in {1, 16, 64, 256}. The launches
    # run back to back (one CUDA graph) over rotating copies of the packed weight that together
    # hold more than 4x L2, so every launch streams its weight from HBM and the per-launch
    # time carries no launch or event overhead; a single flushed launch is reported beside it.
    qkv = workloads.small_m(1)
    wqkv = qkv.make_weights(dev)
    pq = opq.quantize(wqkv, alpha)
    wbytes = qkv.N * qkv.K * 5 // 8 + 4 * qkv.N
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ncopy = int(math.ceil(4 * l2 / wbytes)) + 1
    copies = [tuple(t.clone() for t in pq) for _ in range(ncopy)]
    small = {}
    for m in workloads.SMALL_M_SWEEP:
        xm = workloads.small_m(m).make_x(dev)
        ym = torch.empty((m, qkv.N), dtype=torch.bfloat16, device=dev)
        wsm = torch.zeros((max(opq.workspace_size(m, qkv.N, qkv.K), 16),), dtype=torch.uint8, device=dev)
        reps = 2 * ncopy

        def run_all(xm=xm, ym=ym, wsm=wsm):
            for r in range(reps):
                opq.linear(xm, *copies[r % ncopy], alpha, out=ym, workspace=wsm)

        run_all()
        torch.cuda.synchronize()
        g = capture_graph(torch, run_all)
        for _ in range(2):
            g.replay()
        tg = time_kernel(g.replay, 10, flush_l2=False) / reps
        single = time_kernel(lambda: opq.linear(xm, *pq, alpha, out=ym, workspace=wsm), 20)
        abytes = wbytes + 2 * m * qkv.K + 2 * m * qkv.N
        fl_ = 2.0 * m * qkv.N * qkv.K
        small[str(m)] = {"us": tg * 1e3, "weight_gbs": wbytes / tg / 1e6, "bytes_gbs": abytes / tg / 1e6,
                         "frac_hbm": abytes / tg / 1e6 / hbm, "tflops": fl_ / tg / 1e9,
                         "frac_bf16": fl_ / tg / 1e9 / bf16, "single_launch_us": single * 1e3,
                         "plan": list(opq.plan(m, qkv.N, qkv.K))}
        del g
    out["small_m"] = {"workload": "qkv 11520x3840, M in {1, 16, 64, 256}",
                      "method": f"{2 * ncopy} back-to-back launches in one CUDA graph over {ncopy} copies of "
                                f"the packed weight ({ncopy * wbytes / 1e6:.0f} MB > 4x L2); per-launch time = "
                                f"graph time / launches", "by_m": small}
    del copies, wqkv, pq
    assert opq.device_error() == 0

    # ---- the group-wise format (one float16 max per GS weights) on the projection
    grouped = {}
    wq_g = torch.empty_like(w)
    y_g = torch.empty_like(y)
    for gs in (128, 32):
        cg, sg, gg = opq.quantize_grouped(w, gs, alpha)
        ws_g = torch.zeros((max(opq.grouped_workspace_size(M, N, K, gs), 16),), dtype=torch.uint8, device=dev)
        fq_ = lambda: opq.quantize_grouped(w, gs, alpha, out=(cg, sg, gg))
        fl_ = lambda: opq.linear_grouped(x, cg, sg, gg, alpha, out=y_g, workspace=ws_g)
        fd_ = lambda: opq.dequantize_grouped(cg, sg, gg, alpha, out=wq_g)
        for f_ in (fq_, fl_, fd_):
            for _ in range(3):
                f_()
        tq_, tl_, td_ = time_kernel(fq_), time_kernel(fl_), time_kernel(fd_)
        gq_bytes = N * K * 2 + N * K // 8 * 5 + 2 * N * (K // gs)
        gd_bytes = N * K // 8 * 5 + 2 * N * (K // gs) + N * K * 2
        grouped[str(gs)] = {
            "quantize": {"ms": tq_, "gbs": gq_bytes / tq_ / 1e6, "frac_hbm": gq_bytes / tq_ / 1e6 / hbm},
            "linear": {"ms": tl_, "tflops": flops / tl_ / 1e9, "frac_bf16": flops / tl_ / 1e9 / bf16},
            "dequantize": {"ms": td_, "gbs": gd_bytes / td_ / 1e6, "frac_hbm": gd_bytes / td_ / 1e6 / hbm}}
        del ws_g
    out["grouped"] = grouped
    del wq_g, y_g

    # ---- the other bit widths (3, 5, 6): quantize, dequantize and SNR on the projection weight
    bits_out = {}
    wq_b = torch.empty_like(w)
    r_ = w.double()
    for b_ in (3, 5, 6):
        cb, sb, fb = opq.quantize_bits(w, b_, alpha)
        fq_ = lambda: opq.quantize_bits(w, b_, alpha, out=(cb, sb, fb))
        fd_ = lambda: opq.dequantize_bits(cb, sb, fb, b_, alpha, out=wq_b)
        ws_b = torch.zeros((max(opq.bits_workspace_size(M, N, K, b_), 16),), dtype=torch.uint8, device=dev)
        fl_b = lambda: opq.linear_bits(x, cb, sb, fb, b_, alpha, out=y, workspace=ws_b)
        for f_ in (fq_, fd_, fl_b):
            for _ in range(3):
                f_()
        tq_, td_, tl_ = time_kernel(fq_), time_kernel(fd_), time_kernel(fl_b)
        packed = N * K * b_ // 8 + N * K // 8 + 4 * N
        opq.dequantize_bits(cb, sb, fb, b_, alpha, out=wq_b)
        bits_out[str(b_)] = {
            "quantize": {"ms": tq_, "gbs": (N * K * 2 + packed) / tq_ / 1e6,
                         "frac_hbm": (N * K * 2 + packed) / tq_ / 1e6 / hbm},
            "dequantize": {"ms": td_, "gbs": (packed + N * K * 2) / td_ / 1e6,
                           "frac_hbm": (packed + N * K * 2) / td_ / 1e6 / hbm},
            "linear": {"ms": tl_, "tflops": flops / tl_ / 1e9, "frac_bf16": flops / tl_ / 1e9 / bf16},
            "snr_db": float(10.0 * torch.log10((r_ * r_).sum() / ((r_ - wq_b.double()) ** 2).sum()))}
        del ws_b
        del cb, sb, fb
    out["bits"] = bits_out
    del wq_b, r_

    # ---- the linear with bias + activation fused into its epilogue, same shape as the step
    bias = (torch.arange(N, device=dev, dtype=torch.float32) * 1e-3 - 1.0).to(torch.bfloat16)
    y_f = torch.empty_like(y)
    fused = {"plain_ms": t_l}
    for act in ("silu", "gelu_tanh"):
        ff = lambda: opq.linear_fused(x, codes, signs, scales, alpha, bias=bias, act=act, out=y_f, workspace=ws)
        for _ in range(3):
            ff()
        tf_ = time_kernel(ff)
        fused[act] = {"ms": tf_, "tflops": flops / tf_ / 1e9, "frac_bf16": flops / tf_ / 1e9 / bf16,
                      "vs_plain": tf_ / t_l}
    out["fused"] = fused
    del y_f
    assert opq.device_error() == 0

    # ---- SNR context (the card's "+7.2 dB" is on Z-Image weights; these are the synthetic
    # Student-t weights): OPQ at alpha 0.73 and 1.0, per-row symmetric INT4, group-wise
    def snr_db(ref, rec):
        rr = ref.double()
        return float(10.0 * torch.log10((rr * rr).sum() / ((rr - rec.double()) ** 2).sum()))

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
    for gs_ in (0, 128):
        best_a, snrs = opq.alpha_search(w, opq.ALPHA_GRID, gs_)
        snr[f"alpha_search_{'row' if gs_ == 0 else 'group128'}"] = {
            "best_alpha": best_a, "snr_db": dict(zip([f"{a_:.2f}" for a_ in opq.ALPHA_GRID], snrs))}
    snr["gain_vs_int4_db"] = snr[f"opq_alpha_{alpha:g}"] - snr["int4_symmetric_row"]
    snr["gain_vs_alpha1_db"] = snr[f"opq_alpha_{alpha:g}"] - snr["opq_alpha_1"]
    snr["model_card_claim_db"] = 7.2
    out["snr_db"] = snr
    return out


# --------------------------------------------------------------------------- CPU arms
def oracle_sample():
    """A bounded sample of the whole-model pass for the fp64 oracle: 256 weight rows of an
    attention matrix and of the FFN down-projection (block 0), quantized, and the linear of
    16 activation rows against those rows."""
    import workloads
    model = workloads.WholeModel(blocks=1)
    out = []
    for l in (model.layers[0], model.layers[6]):
        x = l.make_x("cpu")[:16].contiguous()
        w = l.make_weights("cpu")[:256].contiguous()
        out.append((x, w, l.alpha))
    return out


def oracle_step(oracle, sample):
    for x, w, a in sample:
        r = oracle.quantize(w, a)
        oracle.linear(x, r["codes"], r["signs"], r["scales"], a)


def sample_counts(sample):
    flops = sum(2.0 * x.shape[0] * w.shape[0] * w.shape[1] for x, w, _ in sample)
    qbytes = sum(quant_bytes(w.shape[0], w.shape[1]) for _, w, _ in sample)
    return flops, qbytes


SAMPLE_TEXT = ("quantize 256 rows of W 3840x3840 and of W2 3840x10240 (block 0) + linear 16 x-rows against "
               "those 256 rows of each")


def cpu_oracle_sample(budget_s: float = 12.0):
    """Time the fp64 oracle on the bounded sample of the whole-model workload."""
    import oracle
    oracle.build()
    sample = oracle_sample()
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle_step(oracle, sample)
        reps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = (time.perf_counter() - t0) / reps
    flops, qbytes = sample_counts(sample)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{SAMPLE_TEXT} ({reps} reps, {dt:.3f} s each)", "seconds_per_sample": dt,
            "quantize_gbs_in_sample": qbytes / dt / 1e9}


def reference_arm(args):
    import oracle
    oracle.build()
    sample = oracle_sample()
    for _ in range(args.warmup):
        oracle_step(oracle, sample)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(oracle, sample)
        ts.append(time.perf_counter() - t0)
    dt = sum(ts) / len(ts)
    flops, _ = sample_counts(sample)
    v = flops / dt / 1e12
    cores = oracle.num_threads()
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "dit_whole_model_30blocks_210layers_m3072", "sample": SAMPLE_TEXT,
                       "parallelism": "cpu"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": SAMPLE_TEXT + " per step"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_run(args):
    """A short, fixed launch sequence of one kernel for ncu (no timing, no sweep)."""
    import torch
    import bit_diffusion_transformer_b200 as opq
    import workloads
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    shapes = {"attn": workloads.dit_attn_proj(),
              # the whole-model pass's three shape classes at M = 3072 (block 0's seeds)
              "wm_attn": workloads.WholeModel(blocks=1).layers[0],
              "wm_up": workloads.WholeModel(blocks=1).layers[4],
              "wm_down": workloads.WholeModel(blocks=1).layers[6],
              "ffn_up": workloads.dit_ffn_pair()[0], "ffn_down": workloads.dit_ffn_pair()[1]}
    if args.shape.startswith("small"):
        lin = workloads.small_m(int(args.shape[5:]))
    else:
        lin = shapes[args.shape]
    x, w = lin.make(dev)
    planes = opq.quantize(w, lin.alpha)
    y = torch.empty((lin.M, lin.N), dtype=torch.bfloat16, device=dev)
    wq = torch.empty_like(w)
    ws = torch.zeros((max(opq.workspace_size(lin.M, lin.N, lin.K), 16),), dtype=torch.uint8, device=dev)
    jobs = opq.quantize_jobs([w], [planes], lin.alpha)
    fns = {"quantize": lambda: opq.quantize(w, lin.alpha, out=planes),
           "quantize_batched": lambda: opq.quantize_batched([w], lin.alpha, outs=[planes], jobs=jobs),
           "dequantize": lambda: opq.dequantize(*planes, lin.alpha, out=wq),
           "linear": lambda: opq.linear(x, *planes, lin.alpha, out=y, workspace=ws)}
    if args.profile.startswith("grouped"):
        gplanes = opq.quantize_grouped(w, 128, lin.alpha)
        gws = torch.zeros((max(opq.grouped_workspace_size(lin.M, lin.N, lin.K, 128), 16),), dtype=torch.uint8,
                          device=dev)
        fns["grouped_quantize"] = lambda: opq.quantize_grouped(w, 128, lin.alpha, out=gplanes)
        fns["grouped_linear"] = lambda: opq.linear_grouped(x, *gplanes, lin.alpha, out=y, workspace=gws)
    fn = fns[args.profile]
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
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="opq", choices=["opq", "reference"])
    ap.add_argument("--no-sweep", action="store_true", help="skip the extras (FFN pair, projection, small M, ...)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", default=None,
                    help="profiling run: warm up, then launch only this kernel --steps times "
                         "(quantize | quantize_batched | linear | dequantize | grouped_quantize | grouped_linear) "
                         "on --shape")
    ap.add_argument("--shape", default="attn",
                    help="profiling shape: attn | wm_attn | wm_up | wm_down | ffn_up | ffn_down | small<M>")
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
