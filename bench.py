#!/usr/bin/env python
"""Benchmark of the microscaling hot path on B200: activation quantize + block-
scaled GEMM, reported as TFLOP/s with the roofline of the dominant kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload dit_mxfp8|mlp_nvfp4|skinny_nvfp4|quant_sweep]
                    [--no-extras]

Default workload (the configuration the headline metric is quoted on): the
DiT-like MXFP8 E4M3 W8A8 Linear, X bf16 [4096 x 3072] (N(0,1), 8 outlier
channels x30) times W [3072 x 3072] (N(0, 0.02^2), pre-quantized).  One step =
quantize X to MXFP8 (codes + tensor-core-tiled E8M0 scales) and run the
block-scaled GEMM to bf16 C.  Inputs are resident in HBM; each step uses the
next of several input sets whose total size exceeds the 126 MB L2, so every
step starts cold.  The K timed steps are captured once in a CUDA graph and
timed as one replay (device time, without the host's per-call cost).
Multi-GPU runs are independent replicas (weak scaling: the path has no
collective).

--impl reference times the CPU oracle (the plain fp64 C implementation) on a
bounded row sample of the same workload, per step.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 2 ** 20
# Page-quoted spec peaks (Microscaling MXFP4/NVFP4 page, section "Arquitetura
# Blackwell SM100"), reported beside the measured ones.
SPEC = {"hbm_gbs": 8000.0, "fp8_tflops": 2250.0, "fp4_tflops": 4500.0}
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    "dit_mxfp8": dict(fmt=0, M=4096, N=3072, K=3072, x="dit", wseed=2, name="dit_mxfp8_w8a8_linear_4096x3072x3072"),
    "mlp_nvfp4": dict(fmt=3, M=4608, N=12288, K=3072, x="student_t", wseed=4,
                      name="mlp_nvfp4_w4a4_gemm1_4608x12288x3072"),
    "skinny_nvfp4": dict(fmt=3, M=16, N=28672, K=8192, x="normal", wseed=7, name="skinny_nvfp4_16x28672x8192"),
}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


def tensor_peak(fmt: int, peaks: dict, sustained: bool):
    """Dense block-scaled peak for the element type: the measured bf16 GEMM peak
    times the nominal ratio (fp8 = 2x bf16, fp4 = 4x bf16; MXFP6 and mixed MX
    operands run on kind::mxf8f6f4 at the fp8 rate)."""
    base = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    return base * (4.0 if fmt in (2, 3, 5) else 2.0)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx_, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx_ = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx_, "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ inputs
def make_inputs(wl: dict):
    from fp8_quantization_block_b200 import synth
    if wl["x"] == "dit":
        X = synth.dit_activations(1, wl["M"], wl["K"])
    elif wl["x"] == "student_t":
        X = synth.student_t(3, wl["M"], wl["K"])
    else:
        X = synth.to_bf16_bits(np.random.default_rng(200 + wl["M"]).standard_normal((wl["M"], wl["K"])))
    W = synth.gaussian_weights(wl["wseed"], wl["N"], wl["K"])
    return X, W


# ------------------------------------------------------------------ multi-rank host logic
def max_over_ranks(x: float, dist, device) -> float:
    """The largest of every rank's x (a device time), so that a multi-rank
    number is the slowest rank's; x itself with one process (dist is None)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step: float, steps: int, ms_max: float, world: int) -> float:
    """Whole-job throughput of `world` replicas that each ran `steps` steps,
    timed as the slowest rank's ms_max (weak scaling: the work grows with N)."""
    return world * flops_per_step * steps / (ms_max * 1e-3) / 1e12


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, wl, rank, world, device):
    import torch
    from fp8_quantization_block_b200 import mx, synth

    fmt, M, N, K = wl["fmt"], wl["M"], wl["N"], wl["K"]
    X_bits, W_bits = make_inputs(wl)
    X0 = synth.bits_to_tensor(X_bits).to(device)
    W0 = synth.bits_to_tensor(W_bits).to(device)
    per_set = M * K * 2 + mx.mx_codes_bytes(fmt, N, K) + mx.mx_scales_bytes(fmt, N, K) + M * N * 2 + \
        mx.mx_codes_bytes(fmt, M, K) + mx.mx_scales_bytes(fmt, M, K)
    n_sets = max(2, int(np.ceil(3 * L2_BYTES / per_set)))
    sets = []
    for i in range(n_sets):
        X = X0.clone()
        Wq = mx.quantize(W0, fmt)               # weights pre-quantized (outside the step)
        Xq = mx.empty(fmt, M, K)
        C = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        ws = mx.fused_workspace(fmt, M, K, device)
        sets.append((X, Wq, Xq, C, ws))
    torch.cuda.synchronize()
    mx.check_device_error()
    stream = torch.cuda.current_stream()

    def step(i, ev=None):
        """One step: the fused call, X quantized inside the GEMM kernel."""
        X, Wq, Xq, C, ws = sets[i % n_sets]
        if ev is not None:
            ev[0].record(stream)
        mx.gemm_fused_act(X, Wq, out=C, workspace=ws)
        if ev is not None:
            ev[1].record(stream)

    def two_kernel_step(i):
        """The same work as two kernels: mx_quantize, then mx_gemm."""
        X, Wq, Xq, C, ws = sets[i % n_sets]
        mx.quantize(X, fmt, out=Xq)
        mx.gemm(Xq, Wq, out=C)

    def quantize_only(i):
        X, Wq, Xq, C, ws = sets[i % n_sets]
        mx.quantize(X, fmt, out=Xq)

    def gemm_only(i):
        X, Wq, Xq, C, ws = sets[i % n_sets]
        mx.gemm(Xq, Wq, out=C)

    def capture(fn, first, n):
        """A CUDA graph of fn(first), ..., fn(first + n - 1): the library's
        launches (with their programmatic-serialization edges) become graph
        nodes, so a replay costs the device time alone, not the host's ~5 us
        per C-ABI call (~12 us through the Python marshalling)."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for j in range(n):
                fn(first + j)
        return g

    def replay_ms(g):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    for i in range(args.warmup):
        step(i)
        two_kernel_step(i)
    torch.cuda.synchronize()
    # the eager step time (host-issued launches), for comparison
    e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_a.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    e_b.record(stream)
    torch.cuda.synchronize()
    eager_ms = e_a.elapsed_time(e_b)
    g_step = capture(step, args.warmup, args.steps)
    g_two = capture(two_kernel_step, args.warmup, args.steps)
    g_quant = capture(quantize_only, args.warmup, args.steps)
    g_gemm = capture(gemm_only, args.warmup, args.steps)
    g_step.replay()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    # replays of the same K steps fill a ~1.5 s window under the clock sampler
    # immediately before (and including) the timed region
    n_load = int(min(100000, max(0, args.load_window_s * 1000.0 / max(eager_ms, 1e-3))))
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        for i in range(n_load):
            g_step.replay()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        # the step time: one replay of the K steps
        t0.record(stream)
        g_step.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        # the fused kernel alone for the roofline: the same K calls replayed once
        # more right after the timed replay (average launch duration; each call is
        # the GEMM kernel plus the one-block kernel that clears the workspace's
        # counters, which overlaps the previous GEMM's tail)
        fused_graph_ms = replay_ms(g_step)
        # the same work as two kernels, and each of the two alone
        two_graph_ms = replay_ms(g_two)
        quant_graph_ms = replay_ms(g_quant)
        gemm_graph_ms = replay_ms(g_gemm)
        # and each call on its own, with events around it (the launch's ramp-up
        # and drain then count in full)
        for i in range(args.steps):
            step(args.warmup + i, evs[i])
        torch.cuda.synchronize()
    clocks = clk.summary()
    mx.check_device_error()
    del g_step, g_two, g_quant, g_gemm
    ms = t0.elapsed_time(t1)
    f_ms = [fused_graph_ms / args.steps]
    f_ms_iso = [e[0].elapsed_time(e[1]) for e in evs]
    ms = max_over_ranks(ms, dist, device)

    # end-to-end through the C ABI with host buffers: every step copies its X
    # from pinned host memory, runs the fused quantize + GEMM and copies C back.
    # Copies and compute run on three streams with double-buffered device
    # tensors, so step i+1's upload, step i's compute and step i-1's download
    # overlap (PCIe moves both directions at once); events order each buffer's
    # reuse.
    X_host = synth.bits_to_tensor(X_bits).pin_memory()
    C_hosts = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    Wq = sets[0][1]
    Xds = [torch.empty((M, K), dtype=torch.bfloat16, device=device) for _ in range(2)]
    Cds = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(2)]
    ws = mx.fused_workspace(fmt, M, K, device)
    s_up, s_down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    up_done = [ev(), ev()]
    comp_done = [ev(), ev()]
    down_done = [ev(), ev()]
    first = [True, True]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_up):
            if not first[b]:
                s_up.wait_event(comp_done[b])          # step i-2's compute has read Xds[b]
            Xds[b].copy_(X_host, non_blocking=True)
            up_done[b].record(s_up)
        stream.wait_event(up_done[b])
        if not first[b]:
            stream.wait_event(down_done[b])            # step i-2's C has left Cds[b]
        mx.gemm_fused_act(Xds[b], Wq, out=Cds[b], workspace=ws)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_down):
            s_down.wait_event(comp_done[b])
            C_hosts[b].copy_(Cds[b], non_blocking=True)
            down_done[b].record(s_down)
        first[b] = False

    for i in range(max(3, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_up.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(down_done[(args.steps - 1) % 2])
    stream.wait_event(down_done[args.steps % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    del sets
    torch.cuda.empty_cache()
    clocks["window"] = (f"{n_load} untimed replays of the {args.steps}-step graph (~{args.load_window_s} s), then the "
                        f"timed replay")
    return dict(ms=ms, f_ms=f_ms, f_ms_iso=f_ms_iso, two_ms=two_graph_ms / args.steps,
                q_ms=quant_graph_ms / args.steps, g_ms=gemm_graph_ms / args.steps, eager_ms=eager_ms, e2e_ms=e2e_ms,
                clocks=clocks, n_sets=n_sets, per_set=per_set, h2d=M * K * 2, d2h=M * N * 2)


def qsnr_table(device):
    """Quantization SNR (dB) of each format on the synthetic configs' tensors,
    computed on the device by mx_qsnr (fp64 sums)."""
    import torch
    from fp8_quantization_block_b200 import mx, synth
    tensors = {
        "dit_activations_4096x3072": synth.dit_activations(1, 4096, 3072),
        "mlp_activations_student_t_4608x3072": synth.student_t(3, 4608, 3072),
        "weights_gaussian_3072x3072": synth.gaussian_weights(2, 3072, 3072),
    }
    table = {}
    for name, bits in tensors.items():
        x = synth.bits_to_tensor(bits).to(device)
        row = {}
        for label, quant in (("mxfp8_e4m3", lambda: mx.quantize(x, 0)), ("mxfp4", lambda: mx.quantize(x, 2)),
                             ("mxfp4_oas", lambda: mx.quantize_oas(x)), ("nvfp4", lambda: mx.quantize(x, 3)),
                             ("mxfp6_e3m2", lambda: mx.quantize(x, 4)), ("mxfp4_mbs", lambda: mx.quantize(x, 5)),
                             ("mxfp4_mbs_dynamic", lambda: mx.quantize_mbs_dynamic(x))):
            s = mx.qsnr_sums(quant(), x).cpu().numpy()
            row[label] = round(float(10.0 * np.log10(s[0] / s[1])), 3)
        for label, fmt in (("mxfp4_rht32", 2), ("nvfp4_rht32", 3)):
            row[label] = round(rotated_qsnr_db(x, mx.quantize_rht(x, fmt)), 3)
        table[name] = row
    return table


def rotated_qsnr_db(x, q):
    """QSNR of a tensor quantized after the 32-point Walsh-Hadamard rotation,
    measured in the original domain: dequantize (bf16), rotate back (the
    normalised Hadamard matrix is its own inverse), compare with x in fp64.
    The bf16 rounding of the dequantized values adds ~1e-6 of relative error
    energy, negligible next to the 4-bit error."""
    import torch
    from fp8_quantization_block_b200 import mx
    M, K = x.shape
    h = torch.ones((1, 1), dtype=torch.float64, device=x.device)
    while h.shape[0] < 32:
        h = torch.cat([torch.cat([h, h], 1), torch.cat([h, -h], 1)], 0)
    y = mx.dequantize(q).double().reshape(M, K // 32, 32)
    xr = (y @ h) / np.sqrt(32.0)
    xd = x.double().reshape(M, K // 32, 32)
    return float(10.0 * torch.log10((xd * xd).sum() / ((xd - xr) ** 2).sum()))


def kv_cache_extras(device, peaks, timed):
    """K/V-cache quantize of an 80-layer, 8-KV-head, 128-dim model: one row
    per (token, layer, K or V) of 1024 values.  Prefill writes 4096 tokens at
    once; a decode step writes one token for each of 54 concurrent sessions.
    Synthetic N(0, 1) entries (drawn on the device)."""
    import torch
    from fp8_quantization_block_b200 import mx
    rows_per_token, K = 160, 1024
    g = torch.Generator(device=device).manual_seed(300)
    res = {"bytes_per_token": {
        "mxfp4": mx.mx_codes_bytes(2, rows_per_token, K) + rows_per_token * K // 32,
        "mxfp8_e5m2": mx.mx_codes_bytes(1, rows_per_token, K) + rows_per_token * K // 32,
        "bf16": rows_per_token * K * 2}}
    for label, tokens in (("prefill_4096_tokens", 4096), ("decode_54_sessions", 54)):
        M = tokens * rows_per_token
        nsets = 2 if M * K * 2 > L2_BYTES else 8
        xs = [torch.randn((M, K), generator=g, device=device).to(torch.bfloat16) for _ in range(nsets)]
        for fmt, name in ((2, "mxfp4"), (1, "mxfp8_e5m2")):
            qs = [mx.empty(fmt, M, K) for _ in xs]
            ms = timed(lambda i: mx.quantize(xs[i % len(xs)], fmt, out=qs[i % len(xs)]), len(xs))
            gbs = M * K * quant_bytes_per_elem(fmt) / (ms * 1e-3) / 1e9
            res[f"{label}_{name}"] = {"rows": M, "us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                                      "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)}
            del qs
        del xs
    return res


def quant_bytes_per_elem(fmt):
    # bf16 read + codes + scales (MXFP4-MBS: E8M0 per 16 and one macro byte per 128)
    return {0: 3.03125, 1: 3.03125, 2: 2.53125, 3: 2.5625, 4: 2.78125, 5: 2.5703125}[fmt]


def extras_gpu(device):
    """Short measurements of the other hot-path rows (quantize sweep, NVFP4
    MLP GEMM, skinny weight-stream GEMM), each on rotating buffers > L2 and
    timed as a CUDA-graph replay of 20 calls."""
    import torch
    from fp8_quantization_block_b200 import mx

    peaks, _ = measured_peaks()
    out = {}

    def timed(fn, n, reps=20, warm=3):
        """Device ms per call of fn(warm), ..., fn(warm + reps - 1), replayed
        from a CUDA graph (so that small cases are not bound by the host's
        per-call cost).  n: the number of rotating input sets fn cycles
        through; every one of them is used in each replay (reps >= n), so a
        replay touches more than L2 holds when the sets do."""
        reps = max(reps, n)
        for i in range(warm):
            fn(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(reps):
                fn(warm + i)
        g.replay()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        g.replay()
        e.record()
        torch.cuda.synchronize()
        del g
        return s.elapsed_time(e) / reps

    g = torch.Generator(device=device).manual_seed(100)
    # quantize sweep (K = 4096, M = 256 .. 262144: 2^20 .. 2^30 elements), N(0, 1)
    # with 0.5% of the entries x100, the four formats of the hot path; each point
    # rotates over input sets totalling more than twice L2
    sweep = {}
    K = 4096
    for i in range(11):
        M = 256 << i
        n = max(2, int(np.ceil(2 * L2_BYTES / (M * K * 2))))
        n = min(n, 160)
        xs = []
        for j in range(min(n, 8)):
            x = torch.randn((M, K), generator=g, device=device)
            mask = torch.rand((M, K), generator=g, device=device) < 0.005
            xs.append(torch.where(mask, x * 100.0, x).to(torch.bfloat16))
            del x, mask
        # more sets for small tensors: copies of the drawn ones
        while len(xs) < n:
            xs.append(xs[len(xs) % 8].clone())
        for fmt in (0, 1, 2, 3):
            qs = [mx.empty(fmt, M, K) for _ in xs]
            # NVFP4 with its per-tensor scale known (as for weights): g = RU(amax / 2688)
            # of each input, from one untimed call with the amax pre-pass
            gss = [None] * len(xs)
            if fmt == 3:
                for j, x in enumerate(xs):
                    gss[j] = mx.quantize(x, fmt, out=qs[j]).gscale.clone()
            ms = timed(lambda j: mx.quantize(xs[j % len(xs)], fmt, out=qs[j % len(xs)], gscale=gss[j % len(xs)]),
                       len(xs))
            gbs = M * K * quant_bytes_per_elem(fmt) / (ms * 1e-3) / 1e9
            sweep[f"{FMT_NAMES[fmt]}_M{M}"] = {
                "elements": M * K, "us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)}
            if fmt == 3:
                ms2 = timed(lambda j: mx.quantize(xs[j % len(xs)], fmt, out=qs[j % len(xs)]), len(xs))
                gbs2 = M * K * quant_bytes_per_elem(fmt) / (ms2 * 1e-3) / 1e9
                sweep[f"nvfp4_with_amax_prepass_M{M}"] = {"elements": M * K, "us": round(ms2 * 1e3, 2),
                                                          "GB/s": round(gbs2, 1),
                                                          "frac_hbm": round(gbs2 / peaks["hbm_gbs"], 3)}
            del qs
        del xs
        torch.cuda.empty_cache()
    # MXFP4 with overflow-aware scaling: same bytes as MXFP4
    M, K = 65536, 4096
    xs = [torch.randn((M, K), generator=g, device=device).to(torch.bfloat16) for _ in range(3)]
    qs = [mx.empty(2, M, K) for _ in xs]
    ms = timed(lambda i: mx.quantize_oas(xs[i % len(xs)], out=qs[i % len(xs)]), len(xs))
    gbs = M * K * quant_bytes_per_elem(2) / (ms * 1e-3) / 1e9
    sweep[f"mxfp4_oas_M{M}"] = {"us": round(ms * 1e3, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)}
    del qs
    # MXFP6 E3M2 (2 B read + 0.75 B of codes + 1/32 B of scale per element) and
    # MXFP4 with static macro-block scaling
    for fmt, name in ((4, "mxfp6_e3m2"), (5, "mxfp4_mbs")):
        qs = [mx.empty(fmt, M, K) for _ in xs]
        ms = timed(lambda i: mx.quantize(xs[i % len(xs)], fmt, out=qs[i % len(xs)]), len(xs))
        gbs = M * K * quant_bytes_per_elem(fmt) / (ms * 1e-3) / 1e9
        sweep[f"{name}_M{M}"] = {"us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                                 "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)}
        del qs
    # MXFP4 with dynamic macro-block scaling: an exhaustive search over the 256
    # macro mantissas of every macro block (compute-bound; same bytes as MBS)
    Md = 4096
    xsd = [torch.randn((Md, K), generator=g, device=device).to(torch.bfloat16) for _ in range(2)]
    qsd = [mx.empty(5, Md, K) for _ in xsd]
    ms = timed(lambda i: mx.quantize_mbs_dynamic(xsd[i % 2], out=qsd[i % 2]), 2, reps=4)
    gbs = Md * K * quant_bytes_per_elem(5) / (ms * 1e-3) / 1e9
    sweep[f"mxfp4_mbs_dynamic_M{Md}"] = {"us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                                         "macro_blocks_per_s": round(Md * K / 128 / (ms * 1e-3), 1)}
    del xsd, qsd
    # Walsh-Hadamard rotation fused with quantization: the same HBM bytes as the plain quantize
    for fmt, name in ((2, "mxfp4_rht32"), (3, "nvfp4_rht32")):
        qs = [mx.empty(fmt, M, K) for _ in xs]
        gss = [mx.quantize_rht(x, fmt, out=qs[i]).gscale.clone() if fmt == 3 else None for i, x in enumerate(xs)]
        ms = timed(lambda i: mx.quantize_rht(xs[i % len(xs)], fmt, gscale=gss[i % len(xs)], out=qs[i % len(xs)]),
                   len(xs))
        gbs = M * K * quant_bytes_per_elem(fmt) / (ms * 1e-3) / 1e9
        sweep[f"{name}_M{M}"] = {"us": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                                 "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)}
        del qs
    del xs
    out["quantize_sweep"] = sweep
    out["qsnr_db"] = qsnr_table(device)
    out["kv_cache"] = kv_cache_extras(device, peaks, timed)
    # GEMMs (A format, B format, M, N, K); MXFP6 and mixed pairs run on kind::mxf8f6f4
    for name, (fmt, wfmt, M, N, K) in {
            "mlp_nvfp4_gemm1": (3, 3, 4608, 12288, 3072), "mlp_nvfp4_gemm2": (3, 3, 4608, 3072, 12288),
            "skinny_nvfp4_M16": (3, 3, 16, 28672, 8192), "skinny_mxfp4_M16": (2, 2, 16, 28672, 8192),
            "skinny_nvfp4_M128": (3, 3, 128, 28672, 8192),
            "dit_mxfp8_gemm_back_to_back": (0, 0, 4096, 3072, 3072),
            "dit_mxfp6_gemm": (4, 4, 4096, 3072, 3072), "dit_mxfp8_x_mxfp4w_gemm": (0, 2, 4096, 3072, 3072),
            "dit_mxfp8_x_mxfp6w_gemm": (0, 4, 4096, 3072, 3072),
            "dit_mxfp4_gemm": (2, 2, 4096, 3072, 3072), "dit_mxfp4_mbs_gemm": (5, 5, 4096, 3072, 3072)}.items():
        a = torch.randn((M, K), generator=g, device=device).to(torch.bfloat16)
        w = (torch.randn((N, K), generator=g, device=device) * 0.02).to(torch.bfloat16)
        qa = mx.quantize(a, fmt)
        wbytes = mx.mx_codes_bytes(wfmt, N, K) + mx.mx_scales_bytes(wfmt, N, K)
        nw = max(2, int(np.ceil(2 * L2_BYTES / wbytes)))
        qws = [mx.quantize(w, wfmt) for _ in range(nw)]
        C = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        ms = timed(lambda i: mx.gemm(qa, qws[i % nw], out=C), nw)
        tf = 2 * M * N * K / (ms * 1e-3) / 1e12
        bytes_ = wbytes + mx.mx_codes_bytes(fmt, M, K) + mx.mx_scales_bytes(fmt, M, K) + M * N * 2
        gbs = bytes_ / (ms * 1e-3) / 1e9
        out[name] = {"us": round(ms * 1e3, 2), "TFLOP/s": round(tf, 1),
                     "frac_tensor": round(tf / tensor_peak(fmt if fmt == wfmt else 0, peaks, False), 3),
                     "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)}
        del a, w, qa, qws, C
    # the macro-block-scaled GEMM's cost over the plain MXFP4 GEMM on the same
    # shape (the MXFP4 paper page's section 4 quotes 6.2% at prefill with
    # dedicated vector units beside the tensor cores)
    out["dit_mxfp4_mbs_gemm"]["overhead_vs_mxfp4"] = round(
        out["dit_mxfp4_mbs_gemm"]["us"] / out["dit_mxfp4_gemm"]["us"] - 1.0, 3)
    # The skinny weight-stream GEMMs as the configuration states them: bf16
    # activations X [M x 8192] ~ N(0, 1), quantized inside the fused call (NVFP4:
    # g from X's amax pre-pass), times pre-quantized weights [28672 x 8192];
    # HBM-bound, so reported against HBM with the algorithmic bytes of the call:
    # W's codes and scales, X (bf16) read, X's codes and scales written and read
    # back, C written.
    skinny = {}
    N, K = 28672, 8192
    for wfmt in (3, 2):
        w = (torch.randn((N, K), generator=g, device=device) * 0.02).to(torch.bfloat16)
        wbytes = mx.mx_codes_bytes(wfmt, N, K) + mx.mx_scales_bytes(wfmt, N, K)
        nw = max(2, int(np.ceil(2 * L2_BYTES / wbytes)))
        qws = [mx.quantize(w, wfmt) for _ in range(nw)]
        del w
        for M in (1, 16, 128):
            x = torch.randn((M, K), generator=g, device=device).to(torch.bfloat16)
            C = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            ws = mx.fused_workspace(wfmt, M, K, device)
            ms = timed(lambda i: mx.gemm_fused_act(x, qws[i % nw], out=C, workspace=ws), nw)
            xq = mx.mx_codes_bytes(wfmt, M, K) + mx.mx_scales_bytes(wfmt, M, K)
            nbytes = wbytes + 2 * M * K + 2 * xq + 2 * M * N
            gbs = nbytes / (ms * 1e-3) / 1e9
            tf = 2 * M * N * K / (ms * 1e-3) / 1e12
            skinny[f"{FMT_NAMES[wfmt]}_M{M}"] = {
                "us": round(ms * 1e3, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 3),
                "algorithmic_bytes": nbytes, "TFLOP/s": round(tf, 1)}
            del x, C, ws
        del qws
        torch.cuda.empty_cache()
    out["skinny_fused"] = {"points": skinny, "call": "mx_gemm_fused_act(X bf16 [M x 8192], W [28672 x 8192])"}
    # Few output tiles and a long K (a decode-time down projection, W [8192 x
    # 28672]: 32 tiles of 256 columns for 148 SMs): the fused call splits the
    # tiles along K over all SMs (its default plan); the same call with the
    # split turned off beside it.
    down = {}
    N, K = 8192, 28672
    for wfmt in (3, 2):
        w = (torch.randn((N, K), generator=g, device=device) * 0.02).to(torch.bfloat16)
        wbytes = mx.mx_codes_bytes(wfmt, N, K) + mx.mx_scales_bytes(wfmt, N, K)
        nw = max(2, int(np.ceil(2 * L2_BYTES / wbytes)))
        qws = [mx.quantize(w, wfmt) for _ in range(nw)]
        del w
        for M in (1, 16, 128):
            x = torch.randn((M, K), generator=g, device=device).to(torch.bfloat16)
            C = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            ws = mx.fused_workspace(wfmt, M, K, device)
            xq = mx.mx_codes_bytes(wfmt, M, K) + mx.mx_scales_bytes(wfmt, M, K)
            nbytes = wbytes + 2 * M * K + 2 * xq + 2 * M * N
            r = {}
            for key, mode in (("split", mx.MX_K_SPLIT_AUTO), ("whole_tiles", mx.MX_K_SPLIT_NEVER)):
                mx.check(mx.mx_debug_set(mx.MX_DEBUG_K_SPLIT, mode), "mx_debug_set")
                ms = timed(lambda i: mx.gemm_fused_act(x, qws[i % nw], out=C, workspace=ws), nw)
                gbs = nbytes / (ms * 1e-3) / 1e9
                r[key] = {"us": round(ms * 1e3, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 3)}
            mx.check(mx.mx_debug_set(mx.MX_DEBUG_K_SPLIT, mx.MX_K_SPLIT_AUTO), "mx_debug_set")
            r["speedup"] = round(r["whole_tiles"]["us"] / r["split"]["us"], 3)
            r["algorithmic_bytes"] = nbytes
            down[f"{FMT_NAMES[wfmt]}_M{M}"] = r
            del x, C, ws
        del qws
        torch.cuda.empty_cache()
    out["down_proj_split_fused"] = {"points": down, "call": "mx_gemm_fused_act(X bf16 [M x 28672], W [8192 x 28672])"}
    # The DiT step in each mode of the fused call (same results bit for bit)
    M, N, K = 4096, 3072, 3072
    n = 6
    xs = [torch.randn((M, K), generator=g, device=device).to(torch.bfloat16) for _ in range(n)]
    w = (torch.randn((N, K), generator=g, device=device) * 0.02).to(torch.bfloat16)
    qws = [mx.quantize(w, 0) for _ in range(n)]
    Cs = [torch.empty((M, N), dtype=torch.bfloat16, device=device) for _ in range(n)]
    wss = [mx.fused_workspace(0, M, K, device) for _ in range(n)]
    modes = {}
    for name, mode in (("pipelined", mx.MX_FUSED_PIPELINED), ("in_kernel", mx.MX_FUSED_IN_KERNEL),
                       ("two_kernels", mx.MX_FUSED_TWO_KERNELS)):
        mx.check(mx.mx_debug_set(mx.MX_DEBUG_FUSED_MODE, mode), "mx_debug_set")
        ms = timed(lambda i: mx.gemm_fused_act(xs[i % n], qws[i % n], out=Cs[i % n], workspace=wss[i % n]), n)
        modes[name] = {"us": round(ms * 1e3, 2), "TFLOP/s": round(2 * M * N * K / (ms * 1e-3) / 1e12, 1)}
    mx.mx_debug_set(mx.MX_DEBUG_FUSED_MODE, mx.MX_FUSED_PIPELINED)
    out["dit_mxfp8_fused_modes"] = modes
    del xs, w, qws, Cs, wss
    torch.cuda.empty_cache()
    # The NVFP4 MLP pair as the configuration states it: X [4608 x 3072]
    # (Student-t) quantized inside the fused call for H = GELU(X W1^T) with
    # |H| max, then H quantized inside the second fused call (g from that max)
    # for Y = H W2^T; two launches of the library per call pair, no host sync.
    from fp8_quantization_block_b200 import synth
    M, D, F = 4608, 3072, 12288
    X = synth.bits_to_tensor(synth.student_t(3, M, D)).to(device)
    W1 = mx.quantize(synth.bits_to_tensor(synth.gaussian_weights(4, F, D)).to(device), 3)
    W2 = mx.quantize(synth.bits_to_tensor(synth.gaussian_weights(5, D, F)).to(device), 3)
    H = torch.empty((M, F), dtype=torch.bfloat16, device=device)
    Y = torch.empty((M, D), dtype=torch.bfloat16, device=device)
    aH = torch.empty(1, device=device)
    ws1, ws2 = mx.fused_workspace(3, M, D, device), mx.fused_workspace(3, M, F, device)

    def mlp_pair(i):
        mx.gemm_fused_act(X, W1, out=H, epilogue=mx.MX_EPI_GELU, amax_out=aH, workspace=ws1)
        mx.gemm_fused_act(H, W2, out=Y, x_amax=aH, workspace=ws2)

    ms = timed(mlp_pair, 1)
    tf = 2 * 2 * M * D * F / (ms * 1e-3) / 1e12
    out["mlp_nvfp4_pair_fused"] = {"us": round(ms * 1e3, 2), "TFLOP/s": round(tf, 1),
                                   "frac_tensor": round(tf / tensor_peak(3, peaks, False), 3),
                                   "steps": "X->H (amax pre-pass, quantize, GEMM1 + GELU + |H| max), "
                                            "H->Y (quantize with g from |H| max, GEMM2)"}
    del X, W1, W2, H, Y, ws1, ws2
    torch.cuda.empty_cache()
    mx.check_device_error()
    return out


# ------------------------------------------------------------------ CPU oracle arm
def oracle_sample(wl, X_bits, W_bits, rows: int):
    """Time the oracle's quantize of `rows` rows of X and its fp64 GEMM of those
    rows against the whole (pre-quantized) W.  Returns seconds."""
    import oracle
    fmt, N, K = wl["fmt"], wl["N"], wl["K"]
    cw, sw, gw = oracle.quantize(fmt, W_bits)             # weights: pre-quantized, untimed
    Wd = oracle.dequantize_f64(fmt, cw, sw, gw, N, K)
    t = time.perf_counter()
    xs = np.ascontiguousarray(X_bits[:rows])
    g = oracle.nvfp4_global_scale(oracle.amax_bf16(X_bits)) if fmt == 3 else None
    cx, sx, gx = oracle.quantize(fmt, xs, gscale=g)
    Xd = oracle.dequantize_f64(fmt, cx, sx, gx, rows, K)
    oracle.gemm_f64(Xd, Wd)
    return time.perf_counter() - t


def pick_sample_rows(wl, X_bits, W_bits, target_s: float):
    rows = 8
    t = oracle_sample(wl, X_bits, W_bits, rows)
    rows = int(min(wl["M"], max(8, rows * target_s / max(t, 1e-3))))
    return rows


def cpu_baseline(wl, X_bits, W_bits, target_s=12.0, target_1thread_s=8.0):
    """The oracle on the host's cores (OpenMP over rows), and on one thread,
    each on a row sample sized to a few seconds, scaled per FLOP."""
    import oracle
    cores = oracle.get_threads()
    rows = pick_sample_rows(wl, X_bits, W_bits, target_s)
    secs = oracle_sample(wl, X_bits, W_bits, rows)
    flops = 2.0 * rows * wl["N"] * wl["K"]
    oracle.set_threads(1)
    try:
        rows1 = pick_sample_rows(wl, X_bits, W_bits, target_1thread_s)
        secs1 = oracle_sample(wl, X_bits, W_bits, rows1)
    finally:
        oracle.set_threads(cores)
    flops1 = 2.0 * rows1 * wl["N"] * wl["K"]
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{rows} of {wl['M']} activation rows: quantize + fp64 GEMM vs all {wl['N']} weight rows "
                      f"({secs:.1f} s), throughput scaled per FLOP",
            "value_1thread": round(flops1 / secs1 / 1e12, 6),
            "sample_1thread": f"{rows1} rows on one thread ({secs1:.1f} s), scaled per FLOP"}


def run_reference(args, wl):
    import oracle
    X_bits, W_bits = make_inputs(wl)
    target = max(1.0, min(20.0, 60.0 / max(1, args.steps + args.warmup)))
    rows = pick_sample_rows(wl, X_bits, W_bits, target)
    for _ in range(args.warmup):
        oracle_sample(wl, X_bits, W_bits, rows)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(wl, X_bits, W_bits, rows)
    secs = time.perf_counter() - t
    flops = 2.0 * rows * wl["N"] * wl["K"] * args.steps
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl["name"], "format": FMT_NAMES[wl["fmt"]], "M": wl["M"], "N": wl["N"], "K": wl["K"],
                   "sample_rows": rows},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.get_threads(), "kind": "oracle",
                         "sample": f"{rows} activation rows per step (quantize + fp64 GEMM), scaled per FLOP"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


PROFILE_CASES = {
    # name: (kind, fmt, M, N, K[, B's format when it differs])
    "gemm_dit_mxfp8": ("gemm", 0, 4096, 3072, 3072),
    "gemm_dit_mxfp6": ("gemm", 4, 4096, 3072, 3072),
    "gemm_dit_mxfp8_x_mxfp4w": ("gemm", 0, 4096, 3072, 3072, 2),
    "quant_mxfp6_32768x4096": ("quant", 4, 32768, 0, 4096),
    "quant_mbs_32768x4096": ("quant", 5, 32768, 0, 4096),
    "rht_mxfp4_32768x4096": ("rht", 2, 32768, 0, 4096),
    "gemm_mlp1_nvfp4": ("gemm", 3, 4608, 12288, 3072),
    "gemm_mlp2_nvfp4": ("gemm", 3, 4608, 3072, 12288),
    "gemm_skinny_nvfp4": ("gemm", 3, 16, 28672, 8192),
    "quant_mxfp8_32768x4096": ("quant", 0, 32768, 0, 4096),
    "quant_mxfp4_32768x4096": ("quant", 2, 32768, 0, 4096),
    "quant_nvfp4_32768x4096": ("quant", 3, 32768, 0, 4096),
    "quant_mxfp8_dit_4096x3072": ("quant", 0, 4096, 0, 3072),
    "fused_gelu_mlp1_nvfp4": ("fused_gelu", 3, 4608, 12288, 3072),
    "fused_dit_mxfp8": ("fused", 0, 4096, 3072, 3072),
    "gemm_dit_mxfp4_mbs": ("gemm", 5, 4096, 3072, 3072),
    "quant_mbs_dynamic_1024x4096": ("quant_mbs_dynamic", 5, 1024, 0, 4096),
    "quant_nvfp4_prepass_32768x4096": ("quant_prepass", 3, 32768, 0, 4096),
    "fused_down_nvfp4_16x8192x28672": ("fused", 3, 16, 8192, 28672),
}


def run_profile_case(name: str, reps: int = 4):
    """Run one kernel case a few times (for ncu captures; nothing is timed)."""
    import torch
    from fp8_quantization_block_b200 import build as mxbuild
    from fp8_quantization_block_b200 import mx
    mxbuild.build()
    kind, fmt, M, N, K = PROFILE_CASES[name][:5]
    wfmt = PROFILE_CASES[name][5] if len(PROFILE_CASES[name]) > 5 else fmt
    g = torch.Generator(device="cuda").manual_seed(1)
    x = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    if kind == "quant":
        q = mx.empty(fmt, M, K)
        gs = mx.quantize(x, fmt, out=q).gscale.clone() if fmt == 3 else None   # NVFP4: g of this input
        for _ in range(reps):
            mx.quantize(x, fmt, out=q, gscale=gs)
    elif kind == "rht":
        q = mx.empty(fmt, M, K)
        gs = mx.quantize_rht(x, fmt, out=q).gscale.clone() if fmt == 3 else None
        for _ in range(reps):
            mx.quantize_rht(x, fmt, out=q, gscale=gs)
    elif kind == "quant_prepass":
        q = mx.empty(fmt, M, K)
        for _ in range(reps):
            mx.quantize(x, fmt, out=q)      # NVFP4 without g: the amax pre-pass, then the quantize
    elif kind == "quant_mbs_dynamic":
        q = mx.empty(fmt, M, K)
        for _ in range(reps):
            mx.quantize_mbs_dynamic(x, out=q)
    elif kind == "fused":
        w = (torch.randn((N, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        qw = mx.quantize(w, wfmt)
        C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = mx.fused_workspace(fmt, M, K)
        for _ in range(reps):
            mx.gemm_fused_act(x, qw, out=C, workspace=ws)
    elif kind == "fused_gelu":
        w = (torch.randn((N, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        qw = mx.quantize(w, wfmt)
        C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        amax = torch.empty(1, device="cuda")
        for _ in range(reps):
            mx.gemm_fused_act(x, qw, out=C, epilogue=mx.MX_EPI_GELU, amax_out=amax)
    else:
        w = (torch.randn((N, K), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        qa, qw = mx.quantize(x, fmt), mx.quantize(w, wfmt)
        C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        for _ in range(reps):
            mx.gemm(qa, qw, out=C)
    torch.cuda.synchronize()
    mx.check_device_error()
    print(f"profile case {name}: {reps} launches done", flush=True)


METRIC = "NVFP4/MXFP8 block-scaled GEMM TFLOPS + quantize GB/s, % of roofline"

# DRAM bytes (read + write) per launch of the roofline kernel on each workload,
# from one ncu capture of that kernel on that workload; reported only while the
# sources the kernel is built and launched from (KERNEL_SOURCES: every file
# under csrc/ but those of other kernels) still hash to `src`, i.e. the
# counters were taken on the code that runs.
NCU_TRAFFIC = {
    "dit_mxfp8": {"kernel": "gemm_pair_kernel<0, 6, 256, false>", "bytes": 22813184 + 85760,
                  "src": "db2404893c911f15"},
}
# csrc files that no GEMM of gemm_sm100.cuh / gemm_pair_sm100.cuh includes
OTHER_KERNELS = ("gemm_mbs_sm100.cuh", "rotate.cuh")


def csrc_hash(exclude=OTHER_KERNELS) -> str:
    import hashlib
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "fp8_quantization_block_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f in exclude:
            continue
        h.update(f.encode())
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_bytes(workload_key: str, kernel: str):
    rec = NCU_TRAFFIC.get(workload_key)
    if rec is None or rec["kernel"] != kernel or rec["src"] != csrc_hash():
        return None
    return rec["bytes"]


def gemm_kernel_name(fmt: int, M: int, N: int, gelu: bool = False, split: bool = False) -> str:
    """The GEMM kernel mx_gemm dispatches to for this shape (both operands in
    format fmt), named as ncu shows it: CTA pairs for M > 128 and N > 128
    (256 x 256 tiles with 5 stages for the FP4 kinds, 6 otherwise; with the GELU
    epilogue 256 x 128 tiles and 7 stages; MXFP6 runs on the run-time-typed
    kernel, template format 4), else one CTA with 128-wide N tiles for
    N <= 128, 32-row A tiles and 5 stages for M <= 32, 128 x 256 tiles
    otherwise.  split: the variant compiled for a K split of the tiles (the
    fused call's plan; never with GELU)."""
    sp = "true" if split and not gelu else "false"
    if M > 128 and N > 128:
        if gelu:
            return f"gemm_pair_kernel<{fmt}, 7, 128, false>"
        return f"gemm_pair_kernel<{fmt}, {5 if fmt in (2, 3) else 6}, 256, {sp}>"
    if N <= 128:
        return f"gemm_kernel<{fmt}, 128, 4, 128, {sp}>"
    if M <= 32:
        return f"gemm_kernel<{fmt}, 256, 5, 32, {sp}>"
    return f"gemm_kernel<{fmt}, 256, 4, 128, {sp}>"


def gemm_bytes(fmt: int, M: int, N: int, K: int) -> int:
    """Algorithmic bytes of one GEMM launch: A and B codes and scales read
    once, C (bf16) written once."""
    from fp8_quantization_block_b200 import mx
    return (mx.mx_codes_bytes(fmt, M, K) + mx.mx_scales_bytes(fmt, M, K) + mx.mx_codes_bytes(fmt, N, K)
            + mx.mx_scales_bytes(fmt, N, K) + 2 * M * N)


def clock_scale(clocks) -> float | None:
    """median SM clock under load / the maximum SM clock: the factor that turns
    a measured time into the time at the maximum clock (for a kernel whose
    duration scales with the SM clock), None without clock samples."""
    if not clocks:
        return None
    sm, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if not sm or not smax:
        return None
    return float(sm) / float(smax)


def gemm_roofline(fmt: int, M: int, N: int, K: int, gemm_ms: float, peaks: dict, tpeak_burst: float,
                  tpeak_sustained: float, clocks: dict | None = None) -> dict:
    """The roofline object of the GEMM: tensor-bound when its arithmetic
    intensity (FLOPs per algorithmic byte) is above the ridge of the tensor
    peak over the measured HBM bandwidth, HBM-bound below it (the skinny
    weight-streaming shapes), each against its own measured peak.  The kernel
    is timed as a sub-millisecond graph replay, so the tensor peak is the
    burst figure; the sustained one and the page's spec are reported beside
    it, and so is the fraction at the clock-normalised time (kernel time x
    median SM clock / maximum SM clock, from the clocks sampled around the
    timed replay)."""
    flops = 2.0 * M * N * K
    nbytes = gemm_bytes(fmt, M, N, K)
    tf = flops / (gemm_ms * 1e-3) / 1e12
    gbs = nbytes / (gemm_ms * 1e-3) / 1e9
    ridge = tpeak_burst * 1e12 / (peaks["hbm_gbs"] * 1e9)
    cs = clock_scale(clocks)
    if flops / nbytes >= ridge:
        out = {"bound": "tensor", "achieved": round(tf, 1), "peak": round(tpeak_burst, 1), "unit": "TFLOP/s",
               "frac": round(tf / tpeak_burst, 4), "frac_of_sustained_peak": round(tf / tpeak_sustained, 4),
               "frac_of_page_spec": round(tf / SPEC["fp8_tflops" if fmt < 2 else "fp4_tflops"], 4)}
        if cs is not None:
            out["clock_normalised_kernel_us"] = round(gemm_ms * 1e3 * cs, 2)
            out["clock_normalised_frac"] = round(tf / cs / tpeak_burst, 4)
        return out
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(peaks["hbm_gbs"], 1), "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "algorithmic_bytes": nbytes,
            "tensor_TFLOP/s": round(tf, 1), "frac_of_tensor_peak": round(tf / tpeak_burst, 4)}


def add_clock_normalised(extras: dict, clocks: dict) -> None:
    """Beside every tensor-bound fraction of the extras (each against the burst
    peak), the fraction at the clock-normalised time: the time x median SM
    clock / maximum SM clock over the clocks sampled while the extras ran."""
    cs = clock_scale(clocks)
    if cs is None:
        return
    for v in extras.values():
        if isinstance(v, dict) and "frac_tensor" in v:
            v["clock_normalised_frac_tensor"] = round(v["frac_tensor"] / cs, 3)


FMT_NAMES = {0: "mxfp8_e4m3", 1: "mxfp8_e5m2", 2: "mxfp4", 3: "nvfp4", 4: "mxfp6_e3m2", 5: "mxfp4_mbs"}


def fused_launches(fmt: int, M: int, K: int) -> int:
    """Kernels one mx_gemm_fused_act call launches in its default mode (no g
    or amax of X given): with more than one 128-row band of X, the kernel that
    clears the workspace counters, the quantize kernel and the GEMM kernel
    launched to overlap it (NVFP4: the amax pre-pass after the clear); with
    one band, the quantize kernel and the GEMM after it (NVFP4: first a
    one-block kernel that clears the amax slot, then the pre-pass, unless X
    has at most 16384 elements, whose amax the quantize kernel takes itself)."""
    if fmt != 3:
        return 3 if M > 128 else 2
    return 2 if M <= 128 and M * K <= 16384 else 4


def result_line(args, wl: dict, r: dict, world: int) -> dict:
    """The JSON line of the GPU arm from run_gpu's measurements r (device
    times in ms, already the maximum over ranks)."""
    peaks, peak_src = measured_peaks()
    fmt, M, N, K = wl["fmt"], wl["M"], wl["N"], wl["K"]
    flops = 2.0 * M * N * K
    ms_step = r["ms"] / args.steps
    value = whole_job_tflops(flops, args.steps, r["ms"], world)
    f_avg = sum(r["f_ms"]) / len(r["f_ms"])
    f_iso = sum(r["f_ms_iso"]) / len(r["f_ms_iso"])
    # the fused GEMM's own time comes from a sub-millisecond graph replay of its
    # K launches: its peak is the burst figure (the sustained one is reported
    # beside it, with the fraction at the clock-normalised time)
    tpeak_burst = tensor_peak(fmt, peaks, sustained=False)
    tpeak_sustained = tensor_peak(fmt, peaks, sustained=True)
    q_bytes = M * K * quant_bytes_per_elem(fmt)
    q_gbs = q_bytes / (r["q_ms"] * 1e-3) / 1e9
    e2e_value = whole_job_tflops(flops, args.steps, r["e2e_ms"], world)
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": FMT_NAMES[fmt], "data": "synthetic",
        "config": {"workload": wl["name"], "format": FMT_NAMES[fmt], "M": M, "N": N, "K": K,
                   "step": "mx_gemm_fused_act(X bf16, Wq pre-quantized): X quantized to "
                           f"{FMT_NAMES[fmt]} band by band into the workspace while the block-scaled GEMM, "
                           "launched to overlap the quantize, starts on the bands already written; bf16 C",
                   "timed_as": "one replay of a CUDA graph holding the K steps' launches",
                   "ms_per_step_eager": round(r["eager_ms"] / args.steps, 4),
                   "l2": f"inputs larger than L2: {r['n_sets']} rotating input sets x {r['per_set'] / 2**20:.1f} MB",
                   "parallelism": f"replicas x{world}"},
        # the dominant kernel: the GEMM, each of its K launches of the step's
        # inputs replayed alone right after the timed replay; the fused call as a
        # whole (the GEMM overlapping the quantize) beside it
        "roofline": {"kernel": gemm_kernel_name(fmt, M, N),
                     **gemm_roofline(fmt, M, N, K, r["g_ms"], peaks, tpeak_burst, tpeak_sustained, r["clocks"]),
                     "traffic": traffic_bytes(args.workload, gemm_kernel_name(fmt, M, N)),
                     "peak_source": f"{peak_src} burst bf16 x {2 if fmt < 2 else 4} (nominal dtype ratio) "
                                    f"for the tensor bound; {peak_src} copy bandwidth for the HBM bound",
                     "kernel_us": round(r["g_ms"] * 1e3, 2),
                     "timing": "CUDA events on the launching stream around one graph replay of the GEMM kernel's K "
                               "launches on the timed steps' quantized inputs, right after the timed replay",
                     "fused_call": {
                         "us": round(f_avg * 1e3, 2), "us_isolated": round(f_iso * 1e3, 2),
                         **{k: v for k, v in gemm_roofline(fmt, M, N, K, f_avg, peaks, tpeak_burst, tpeak_sustained,
                                                           r["clocks"]).items()
                            if k in ("achieved", "frac", "clock_normalised_frac", "unit")},
                         "what": "the K fused calls (counter reset, quantize, GEMM overlapping it) replayed alone; "
                                 "us_isolated: events around each call of a further eager pass"}},
        "two_kernel_split": {
            "step_us": round(r["two_ms"] * 1e3, 2),
            "quantize_kernel": f"quantize_kernel<{FMT_NAMES[fmt]}>", "quantize_us": round(r["q_ms"] * 1e3, 2),
            "quantize_GB/s": round(q_gbs, 1), "quantize_frac_hbm": round(q_gbs / peaks["hbm_gbs"], 4),
            "gemm_kernel": gemm_kernel_name(fmt, M, N), "gemm_us": round(r["g_ms"] * 1e3, 2),
            "gemm_frac_tensor": round(flops / (r["g_ms"] * 1e-3) / 1e12 / tpeak_burst, 4),
            "what": "the same step as mx_quantize then mx_gemm (two kernels), each kernel also timed alone as a "
                    "graph replay of its K launches", "bytes_per_elem": quant_bytes_per_elem(fmt)},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"], "path": "pinned host X -> H2D -> mx_gemm_fused_act -> D2H C, upload / compute / download on three "
                        "streams with double buffers (consecutive steps overlap)"},
        "gpu_launches": fused_launches(fmt, M, K) * args.steps,
        "clocks": r["clocks"],
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="dit_mxfp8", choices=sorted(WORKLOADS))
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--load-window-s", type=float, default=1.5,
                    help="seconds of untimed steps run under the clock sampler right before the timed steps")
    ap.add_argument("--profile", default=None, choices=sorted(PROFILE_CASES),
                    help="run one kernel case a few times for an ncu capture, then exit")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args.profile)
        return
    if args.warmup < 3:
        args.warmup = 3
    wl = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl)
        return

    import torch
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    from fp8_quantization_block_b200 import build as mxbuild
    if rank == 0:
        mxbuild.build()
    if world > 1:
        torch.distributed.barrier()

    r = run_gpu(args, wl, rank, world, device)
    line = result_line(args, wl, r, world)
    if rank == 0 and world == 1 and not args.no_extras:
        with ClockSampler(device.index if device.index is not None else 0) as clk:
            extras = extras_gpu(device)
        extras["clocks"] = clk.summary()
        add_clock_normalised(extras, extras["clocks"])
        line["extras"] = extras
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        X_bits, W_bits = make_inputs(wl)
        line["cpu_baseline"] = cpu_baseline(wl, X_bits, W_bits)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
