#!/usr/bin/env python
"""Benchmark of the QLoRA frozen-base linear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Workload: the 7B-shaped linear set (q, k, v, o 4096x4096; gate, up
4096->11008; down 11008->4096), M = 4 x 512 = 2048 tokens, r = 64,
alpha = 16, W ~ N(0, 0.02) with 0.1 % outliers at +-10 sigma; synthetic
seeded inputs, generated on the device before timing.

One step = for every linear: qlora_quantize_nf4, qlora_double_quant,
qlora_dequant, qlora_linear_fwd (saving XA), qlora_linear_bwd, and a
few-token qlora_linear_fwd (the first 16 tokens: the memory-bound small-M
path) — every row of the hot path once. Under torchrun each rank runs its own batch (weak
scaling, data parallel over tokens) and the adapter gradients dA, dB of
every linear are summed across ranks with one NCCL all-reduce per step.

`value` = algorithmic FLOPs of all ranks / step time (max over ranks), sum
over linears of 4MNK + 6Mr(N+K) for the fwd+bwd plus 2mNK + 2mr(N+K) for
the m = 16 token forward. The codec phases are reported
in GB/s beside it. The reference arm (--impl reference) times the CPU
oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "llama7b_set"
METRIC = "QLoRA linear fwd+bwd TFLOP/s and quant/dequant GB/s, % of roofline, 1 B200"
UNIT = "TFLOP/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_HBM_GBS = 8000.0        # HBM roofline the workload states (~8 TB/s)
SPEC_BF16_TFLOPS = 2250.0    # dense bf16 tensor-core peak (spec)
KERNEL_SOURCES = ["bit_quantized_lora_blockwise_b200/csrc/gemm.cuh",
                  "bit_quantized_lora_blockwise_b200/csrc/skinny.cuh",
                  "bit_quantized_lora_blockwise_b200/csrc/codec.cuh",
                  "bit_quantized_lora_blockwise_b200/csrc/smallm.cuh",
                  "bit_quantized_lora_blockwise_b200/csrc/ptx.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-compare", action="store_true",
                    help="skip the dequantize-then-cuBLAS comparison leg")
    ap.add_argument("--linears", default="", help="comma list of linear names to keep (profiling runs)")
    ap.add_argument("--phase", default="",
                    help="run only this diagnostic workload phase (no headline step; a profiling aid): "
                         "single_1024, llama13b_quant_sweep, llama65b_fwd, llama7b_f16, "
                         "paged_adamw_7b_adapters or llama33b_block")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the diagnostic rows of the other workloads (single linear, 13B codec sweep, "
                         "65B forwards, 33B block)")
    return ap.parse_args()


def linear_flops(M, N, K, r):
    return 4 * M * N * K + 6 * M * r * (N + K)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def _code_only(text: str) -> str:
    """Kernel source without comments and blank space, so that an edit to a
    comment does not mark the profiled kernels as changed."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(read=None):
    """Hash of the kernel sources' code (comments and spacing ignored)."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        if read is None:
            with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
                text = f.read()
        else:
            text = read(rel)
        h.update(_code_only(text).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key: str):
    """Per-launch DRAM bytes of `kernel_key` from the committed ncu summary,
    or None when there is none or the kernels changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    src = None
    val = None
    for ln in lines:
        if ln.startswith("kernel_source_hash:"):
            src = ln.split(":", 1)[1].strip()
        if ln.startswith(kernel_key + ":"):
            val = float(ln.split(":", 1)[1].strip())
    if src != kernel_source_hash():
        return None
    return val


class ClockSampler:
    """SM clock and throttle reasons of this rank's GPU, read through NVML
    (read-only queries) every ~2 ms from a host thread, so that a timed
    region of a few tens of milliseconds still gets many samples. Only the
    samples taken between mark_start() and mark_stop() are summarised.
    Falls back to `nvidia-smi -lms 200` when NVML cannot be loaded."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index: int):
        self.idx = device_index
        self.samples = []  # (host time, sm MHz, reason names)
        self.t0 = self.t1 = None
        self.stop_flag = threading.Event()
        self.thread = None
        self.proc = None
        self.max_mhz = None
        self.how = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-")
                                                            else uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            bits = [(name, getattr(nv, attr)) for name, attr in self.REASONS if hasattr(nv, attr)]
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self.stop_flag.is_set():
                    try:
                        mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        rs = int(get_reasons(h))
                        self.samples.append((time.perf_counter(), mhz, [n for n, b in bits if rs & b]))
                    except Exception:
                        pass
                    time.sleep(0.002)
            self.how = "nvml, every ~2 ms"
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.how = "nvidia-smi -lms 200"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.proc.stdout:
            f = [x.strip() for x in ln.strip().split(",")]
            if len(f) < 9:
                continue
            try:
                mhz, self.max_mhz = float(f[1]), float(f[2])
            except ValueError:
                continue
            self.samples.append((time.perf_counter(), mhz, [n for n, v in zip(names, f[5:9])
                                                             if v.lower() == "active"]))

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_stop(self):
        self.t1 = time.perf_counter()

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.stop_flag.set()
        self.thread.join(timeout=5)
        t0 = self.t0 if self.t0 is not None else float("-inf")
        t1 = self.t1 if self.t1 is not None else float("inf")
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside and self.samples:  # a region shorter than the sampling period: nearest sample
            mid = (t0 + t1) / 2 if self.t0 is not None and self.t1 is not None else self.samples[-1][0]
            inside = [min(self.samples, key=lambda s: abs(s[0] - mid))]
        sm = [s[1] for s in inside]
        reasons = sorted({r for s in inside for r in s[2]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(sm) if sm else None, "reasons": reasons, "samples": len(sm),
                "sampled_with": self.how}


# ------------------------------------------------------------------ oracle --
def oracle_sample_step(wl, li=0, tokens=64):
    """One bounded oracle step: the full codec chain on linear `li` and the
    float64 forward+backward for `tokens` tokens. Returns its algorithmic
    FLOPs (same convention as the GPU value)."""
    import numpy as np
    import torch
    import oracle
    from bit_quantized_lora_blockwise_b200.inputs import layer_inputs, bf16_bits
    lin = wl.linears[li]
    inp = layer_inputs(wl, li, tokens, device="cpu")
    wb = bf16_bits(inp["W"])
    pk, am = oracle.quantize_nf4(wb)
    q, s2 = oracle.double_quant(am)
    wq = oracle.dequant(pk, q, s2, lin.N * lin.K).reshape(lin.N, lin.K)
    X, A, B, dY = (bf16_bits(inp[k]) for k in ("X", "A", "B", "dY"))
    Y, XA = oracle.linear_fwd(X, wq, A, B, wl.alpha, wl.r)
    dX, dA, dB = oracle.linear_bwd(X, dY, wq, A, B, wl.alpha, wl.r)
    return linear_flops(tokens, lin.N, lin.K, wl.r), f"linear '{lin.name}' {lin.N}x{lin.K}: codec on all " \
        f"{lin.N * lin.K} weights + fp64 fwd/bwd on {tokens} of {wl.M[0]} tokens"


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def _oracle_rate(wl, budget_s):
    t0 = time.perf_counter()
    flops = 0
    n = 0
    sample = ""
    while True:
        f, sample = oracle_sample_step(wl)
        flops += f
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return flops / dt / 1e12, f"{n} x ({sample}); {dt:.1f} s"


def cpu_baseline(wl, budget_s=8.0):
    """The oracle on the host: all cores (its float64 matmuls use the BLAS
    thread pool; the C codec is single-threaded), and limited to one thread."""
    value, sample = _oracle_rate(wl, budget_s)
    single = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            v1, s1 = _oracle_rate(wl, budget_s)
        single = {"value": v1, "unit": UNIT, "cores": 1, "sample": s1}
    except ImportError:
        pass
    return {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle", "sample": sample,
            "single_thread": single}


def run_reference(args, rank):
    from bit_quantized_lora_blockwise_b200.inputs import WORKLOADS
    if rank != 0:
        return
    wl = WORKLOADS[WORKLOAD]
    for _ in range(args.warmup):
        oracle_sample_step(wl)
    t0 = time.perf_counter()
    flops = 0
    sample = ""
    for _ in range(args.steps):
        f, sample = oracle_sample_step(wl)
        flops += f
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "sample_per_step": sample, "M": wl.M[0], "r": wl.r},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ native --
SMALL_M = 16  # tokens of the few-token forward in each step
# GPU sleep (SM clock cycles, ~10 ms) ahead of a diagnostic pass so that the
# host has queued the whole pass before the device starts it
QUEUE_AHEAD_CYCLES = 20_000_000


class LinearState:
    def __init__(self, wl, li, M, device):
        import torch
        from bit_quantized_lora_blockwise_b200 import binding
        from bit_quantized_lora_blockwise_b200.inputs import layer_inputs
        lin = wl.linears[li]
        self.name, self.N, self.K, self.M, self.r, self.alpha = lin.name, lin.N, lin.K, M, wl.r, wl.alpha
        inp = layer_inputs(wl, li, M, device=device)
        self.W, self.X, self.A, self.B, self.dY = (inp[k] for k in ("W", "X", "A", "B", "dY"))
        N, K, r = self.N, self.K, self.r
        e = dict(device=device)
        self.packed = torch.empty(N * K // 2, dtype=torch.uint8, **e)
        self.absmax = torch.empty(N * K // 64, dtype=torch.float32, **e)
        self.q = torch.empty(N * K // 64, dtype=torch.uint8, **e)
        self.scale2 = torch.empty((N * K // 64 + 255) // 256, dtype=torch.float32, **e)
        self.Wq = torch.empty((N, K), dtype=torch.bfloat16, **e)
        self.Y = torch.empty((M, N), dtype=torch.bfloat16, **e)
        self.XA = torch.empty((M, r), dtype=torch.bfloat16, **e)
        self.dX = torch.empty((M, K), dtype=torch.bfloat16, **e)
        self.dA = torch.empty((K, r), dtype=torch.bfloat16, **e)
        self.dB = torch.empty((r, N), dtype=torch.bfloat16, **e)
        self.ws_bytes = binding.workspace_bytes(M, N, K, r)
        self.Xs = self.X[:SMALL_M]  # a view: rows are contiguous, and it follows X's contents
        self.Ys = torch.empty((SMALL_M, N), dtype=torch.bfloat16, **e)
        self.XAs = torch.empty((SMALL_M, r), dtype=torch.bfloat16, **e)

    def smallm_flops(self):
        return 2 * SMALL_M * self.N * self.K + 2 * SMALL_M * self.r * (self.N + self.K)

    def flops(self):
        return linear_flops(self.M, self.N, self.K, self.r) + self.smallm_flops()

    def smallm_bytes(self):
        """Bytes the few-token forward must move: the packed weight with its
        block constants, X, A, B, and the outputs Y, XA."""
        N, K, r, m = self.N, self.K, self.r, SMALL_M
        nb = N * K // 64
        return N * K // 2 + nb + ((nb + 255) // 256) * 4 + 2 * (m * K + K * r + r * N + m * N + m * r)

    def codec_bytes(self):
        n = self.N * self.K
        ng = (n // 64 + 255) // 256
        return {"quantize_dq": n * 2 + n // 2 + n // 64 + ng * 4,
                "quantize": n * 2 + n // 2 + n // 64 * 4,
                "double_quant": n // 64 * 4 + n // 64 + ng * 4,
                "dequant": n // 2 + n // 64 + ((n // 64 + 255) // 256) * 4 + n * 2}


def dequant_then_library(packed, q, scale2, X, A, B, dY, alpha, N, K, Wq=None):
    """The comparison design, dequantize then multiply: this library's
    dequant writes W' (in X's 16-bit type) to HBM, then torch matmuls
    (cuBLAS) compute the layer's forward and backward products.
    Returns (Y, dX, dA, dB)."""
    import torch
    from bit_quantized_lora_blockwise_b200 import binding
    s = alpha / A.shape[1]
    Wq = binding.dequant(packed, q, scale2, N, K, out=Wq, dtype=X.dtype)
    xas = (X @ A) * s
    Y = torch.addmm(xas @ B, X, Wq.t())
    g = (dY @ B.t()) * s
    dX = torch.addmm(g @ A.t(), dY, Wq)
    return Y, dX, X.t() @ g, xas.t() @ dY


def compare_dequant_then_library_gemm(layers, ws, steps):
    """The design the pages describe, dequantize then multiply, timed against
    the fused calls (a comparison, not the product and not the headline).
    Per linear: this library's dequant writes the bf16 W' to HBM and
    cuBLAS (torch.matmul) computes the same forward and backward products
    (X A, Y, dY B^T, dX, dA, dB in bf16); against it, qlora_linear_fwd +
    qlora_linear_bwd. Both are queued behind a GPU sleep and timed on the
    device over the 7 linears."""
    import torch
    from bit_quantized_lora_blockwise_b200 import binding

    def fused(L):
        binding.linear_fwd(L.packed, L.q, L.scale2, L.X, L.A, L.B, L.alpha, L.N, L.K, Y=L.Y, XA_out=L.XA,
                           workspace=ws)
        binding.linear_bwd(L.packed, L.q, L.scale2, L.X, L.dY, L.A, L.B, L.alpha, L.N, L.K, XA=L.XA, dX=L.dX,
                           dA=L.dA, dB=L.dB, workspace=ws)

    def library(L):
        dequant_then_library(L.packed, L.q, L.scale2, L.X, L.A, L.B, L.dY, L.alpha, L.N, L.K, Wq=L.Wq)

    out = {}
    for name, fn in (("fused_ms", fused), ("dequant_then_cublas_ms", library)):
        for L in layers:  # warm (cuBLAS heuristics, allocator)
            fn(L)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
        e0.record()
        for _ in range(steps):
            for L in layers:
                fn(L)
        e1.record()
        torch.cuda.synchronize()
        out[name] = round(e0.elapsed_time(e1) / steps, 4)
    out["fused_speedup"] = round(out["dequant_then_cublas_ms"] / out["fused_ms"], 3)
    out["what"] = ("fwd + bwd of the 7 linears per step; library path = dequant kernel (bf16 W' in HBM) "
                   "+ torch.matmul (cuBLAS) bf16 GEMMs; fused path = qlora_linear_fwd + qlora_linear_bwd")
    return out


def device_ms(fn, reps, warm=2):
    """Device time of one fn() (mean of `reps` back to back), queued behind a
    GPU sleep so that the events time the device, not the host's enqueue."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def workload_phases(dev, hbm_gbs, tc_tflops, quick=False, only=None):
    """Every other workload the hot path is specified on, timed on the
    device after the headline (diagnostic rows, not the headline):
      single_1024          one 1024x1024 linear, M = 16, r = 8: fwd + bwd latency
      llama13b_quant_sweep quantize + double quant, and dequant, over 40 layers x 7 linears
      llama65b_fwd         7 linears: few-token forwards (M = 1, 4, 16) and M = 4096
      llama7b_f16          the 7B set's fused fwd + bwd with fp16 operands
      paged_adamw_7b_adapters  one AdamW step over the 7B adapters, state on the device / paged out
      llama33b_block       7 linears, M = 2048: block fwd + block bwd recomputing XA (and one by one)
    Rates are against the measured peaks and the spec ones (8 TB/s HBM,
    2.25 PFLOP/s dense bf16)."""
    import torch
    from bit_quantized_lora_blockwise_b200 import binding
    from bit_quantized_lora_blockwise_b200.inputs import WORKLOADS, layer_inputs, weight_bf16, seed_for
    out = {}

    def want(name):
        return only is None or only == name

    def frac_hbm(gbs):
        return {"GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm_gbs, 3), "frac_8tbs": round(gbs / SPEC_HBM_GBS, 3)}

    def frac_tc(tf):
        return {"TFLOP/s": round(tf, 1), "frac_tensor": round(tf / tc_tflops, 3),
                "frac_spec": round(tf / SPEC_BF16_TFLOPS, 3)}

    def quantized(W):
        pk, am = binding.quantize_nf4(W)
        q, s2 = binding.double_quant(am)
        return pk, q, s2

    if want("single_1024"):
        # -- single linear (latency; every tensor L2-resident)
        wl = WORKLOADS["single_1024"]
        inp = layer_inputs(wl, 0, wl.M[0], device=dev)
        N, K, M, r = wl.linears[0].N, wl.linears[0].K, wl.M[0], wl.r
        pk, q, s2 = quantized(inp["W"])
        ws = torch.empty(binding.workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
        Y, XA = torch.empty((M, N), dtype=torch.bfloat16, device=dev), torch.empty((M, r), dtype=torch.bfloat16, device=dev)
        dX, dA, dB = (torch.empty(sh, dtype=torch.bfloat16, device=dev) for sh in ((M, K), (K, r), (r, N)))

        def c1():
            binding.linear_fwd(pk, q, s2, inp["X"], inp["A"], inp["B"], wl.alpha, N, K, Y=Y, XA_out=XA, workspace=ws)
            binding.linear_bwd(pk, q, s2, inp["X"], inp["dY"], inp["A"], inp["B"], wl.alpha, N, K, XA=XA, dX=dX,
                               dA=dA, dB=dB, workspace=ws)
        ms = device_ms(c1, 50)
        out["single_1024"] = {"what": "qlora_linear_fwd + qlora_linear_bwd, 1024x1024, M=16, r=8 (L2-resident)",
                              "us_per_fwd_bwd": round(ms * 1e3, 2),
                              "TFLOP/s": round(linear_flops(M, N, K, r) / (ms * 1e-3) / 1e12, 3)}
        del inp, pk, q, s2, ws

    if want("llama13b_quant_sweep"):
        # -- 13B-equivalent codec sweep: one layer's buffers, refilled per layer (outside the timed calls)
        wl = WORKLOADS["llama13b_quant_sweep"]
        layers = 4 if quick else wl.layers
        bufs = []
        for lin in wl.linears:
            n = lin.N * lin.K
            bufs.append({"N": lin.N, "K": lin.K, "W": torch.empty((lin.N, lin.K), dtype=torch.bfloat16, device=dev),
                         "pk": torch.empty(n // 2, dtype=torch.uint8, device=dev),
                         "am": torch.empty(n // 64, dtype=torch.float32, device=dev),
                         "q": torch.empty(n // 64, dtype=torch.uint8, device=dev),
                         "s2": torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device=dev),
                         "Wq": torch.empty((lin.N, lin.K), dtype=torch.bfloat16, device=dev)})
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 2x L2: written between timed calls
        t_q = t_dq = t_d = t_qdq = 0.0
        params = 0
        for layer in range(layers):
            for li, b in enumerate(bufs):
                b["W"].copy_(weight_bf16(b["N"], b["K"], wl.w_std, seed_for(wl.index, li, 0, layer), device=dev))
            flush.zero_()
            t_q += device_ms(lambda: [binding.quantize_nf4(b["W"], packed=b["pk"], absmax=b["am"]) for b in bufs], 1, 0)
            flush.zero_()
            t_dq += device_ms(lambda: [binding.double_quant(b["am"], q=b["q"], scale2=b["s2"]) for b in bufs], 1, 0)
            flush.zero_()
            t_qdq += device_ms(lambda: [binding.quantize_dq(b["W"], packed=b["pk"], q=b["q"], scale2=b["s2"])
                                        for b in bufs], 1, 0)
            flush.zero_()
            t_d += device_ms(lambda: [binding.dequant(b["pk"], b["q"], b["s2"], b["N"], b["K"], out=b["Wq"])
                                      for b in bufs], 1, 0)
            params += sum(b["N"] * b["K"] for b in bufs)
        n = params
        q_in, q_out = 2 * n, n // 2 + n // 64 * 4
        dq_in, dq_out = n // 64 * 4, n // 64 + n // 16384 * 4
        d_in, d_out = n // 2 + n // 64 + n // 16384 * 4, 2 * n
        out["llama13b_quant_sweep"] = {
            "what": f"{layers} layers x 7 linears (d=5120, ffn=13824), {n / 1e9:.3f} G params, per-call events summed",
            "quantize": {"ms": round(t_q, 3), "GB_in": round(q_in / 1e9, 3), "GB_out": round(q_out / 1e9, 3),
                         **frac_hbm((q_in + q_out) / (t_q * 1e-3) / 1e9)},
            "double_quant": {"ms": round(t_dq, 3), **frac_hbm((dq_in + dq_out) / (t_dq * 1e-3) / 1e9)},
            "quantize_plus_double_quant": {"ms": round(t_q + t_dq, 3),
                                           **frac_hbm((q_in + q_out + dq_in + dq_out) / ((t_q + t_dq) * 1e-3) / 1e9)},
            "quantize_dq_one_pass": {"ms": round(t_qdq, 3), "GB_in": round(q_in / 1e9, 3),
                                     "GB_out": round((n // 2 + n // 64 + n // 16384 * 4) / 1e9, 3),
                                     **frac_hbm((q_in + n // 2 + n // 64 + n // 16384 * 4) / (t_qdq * 1e-3) / 1e9)},
            "dequant": {"ms": round(t_d, 3), "GB_in": round(d_in / 1e9, 3), "GB_out": round(d_out / 1e9, 3),
                        **frac_hbm((d_in + d_out) / (t_d * 1e-3) / 1e9)}}
        del bufs, flush

    if want("llama65b_fwd"):
        # -- 65B-shaped forwards: few tokens (HBM-bound) and M = 4096 (tensor-bound)
        wl = WORKLOADS["llama65b_fwd"]
        packed = []
        for li, lin in enumerate(wl.linears):
            W = weight_bf16(lin.N, lin.K, wl.w_std, seed_for(wl.index, li, 0), device=dev)
            packed.append((lin, *quantized(W)))
            del W
        torch.cuda.synchronize()
        Mmax = max(wl.M)
        Kmax = max(lin.K for lin in wl.linears)
        Nmax = max(lin.N for lin in wl.linears)
        acts = []
        for li, (lin, _, _, _) in enumerate(packed):
            acts.append({"X": torch.randn((Mmax, lin.K), device=dev).to(torch.bfloat16),
                         "A": (torch.randn((lin.K, wl.r), device=dev) * 0.01).to(torch.bfloat16),
                         "B": (torch.randn((wl.r, lin.N), device=dev) * 0.01).to(torch.bfloat16)})
        Ybuf = torch.empty(Mmax * Nmax, dtype=torch.bfloat16, device=dev)
        XAbuf = torch.empty(Mmax * wl.r, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(binding.workspace_bytes(m, lin.N, lin.K, wl.r) for m in wl.M for lin, *_ in packed),
                         dtype=torch.uint8, device=dev)
        c4 = {"what": "7 linears (d=8192, ffn=22016), r=64: one qlora_linear_fwd per linear, summed"}
        for m in wl.M:
            def fwd_all(m=m):
                for (lin, pk, q, s2), a in zip(packed, acts):
                    binding.linear_fwd(pk, q, s2, a["X"][:m], a["A"], a["B"], wl.alpha, lin.N, lin.K,
                                       Y=Ybuf[:m * lin.N].view(m, lin.N), XA_out=XAbuf[:m * wl.r].view(m, wl.r),
                                       workspace=ws)
            ms = device_ms(fwd_all, 3 if m > 16 else 10)
            flops = sum(2 * m * lin.N * lin.K + 2 * m * wl.r * (lin.N + lin.K) for lin, *_ in packed)
            if m <= 16:
                nbytes = sum(lin.N * lin.K // 2 + lin.N * lin.K // 64 + (lin.N * lin.K // 16384) * 4 +
                             2 * (m * lin.K + lin.K * wl.r + wl.r * lin.N + m * lin.N + m * wl.r) for lin, *_ in packed)
                c4[f"M{m}"] = {"ms": round(ms, 4), "MB": round(nbytes / 1e6, 1), **frac_hbm(nbytes / (ms * 1e-3) / 1e9)}
            else:
                c4[f"M{m}"] = {"ms": round(ms, 4), **frac_tc(flops / (ms * 1e-3) / 1e12)}
        out["llama65b_fwd"] = c4
        del packed, acts, Ybuf, XAbuf, ws

    if want("llama7b_f16") or want("paged_adamw_7b_adapters"):
        # -- 7B set in fp16 (the pages' other 16-bit compute type): fused fwd + bwd
        wl = WORKLOADS["llama7b_set"]
        M = wl.M[0]
        f16 = []
        for li, lin in enumerate(wl.linears):
            inp = layer_inputs(wl, li, M, device=dev)
            pk, q, s2 = quantized(inp["W"])
            h = {k: inp[k].to(torch.float16) for k in ("X", "A", "B", "dY")}
            del inp
            f16.append((lin, pk, q, s2, h, torch.empty((M, lin.N), dtype=torch.float16, device=dev),
                        torch.empty((M, wl.r), dtype=torch.float16, device=dev),
                        torch.empty((M, lin.K), dtype=torch.float16, device=dev),
                        torch.empty((lin.K, wl.r), dtype=torch.float16, device=dev),
                        torch.empty((wl.r, lin.N), dtype=torch.float16, device=dev)))
        ws = torch.empty(max(binding.workspace_bytes(M, lin.N, lin.K, wl.r) for lin, *_ in f16),
                         dtype=torch.uint8, device=dev)

        def fwd_bwd_f16():
            for lin, pk, q, s2, h, Y, XA, dX, dA, dB in f16:
                binding.linear_fwd(pk, q, s2, h["X"], h["A"], h["B"], wl.alpha, lin.N, lin.K, Y=Y, XA_out=XA,
                                   workspace=ws)
                binding.linear_bwd(pk, q, s2, h["X"], h["dY"], h["A"], h["B"], wl.alpha, lin.N, lin.K, XA=XA, dX=dX,
                                   dA=dA, dB=dB, workspace=ws)
        ms = device_ms(fwd_bwd_f16, 5)
        flops = sum(linear_flops(M, lin.N, lin.K, wl.r) for lin, *_ in f16)
        out["llama7b_f16"] = {"what": "7 linears of the 7B set, M=2048, r=64, fp16 operands and outputs: "
                                      "qlora_linear_fwd + qlora_linear_bwd (the _dt calls)",
                              "ms": round(ms, 4), **frac_tc(flops / (ms * 1e-3) / 1e12)}

        # -- paged AdamW over the 7B set's adapters: state on the device, and paged out to the host
        grads = [t for *_, dA, dB in f16 for t in (dA, dB)]
        params = [t.clone() for lin, pk, q, s2, h, *_ in f16 for t in (h["A"], h["B"])]
        n_el = sum(t.numel() for t in params)
        adamw = {}
        for where, reserve in (("device", 0), ("host", 1 << 62)):
            opt = binding.PagedAdamW(params, lr=1e-4, weight_decay=0.01)
            opt.set_reserve(reserve)
            opt.step(grads)  # places the state
            torch.cuda.synchronize()
            ms = device_ms(lambda: opt.step(grads), 10)
            gbs = n_el * 28 / (ms * 1e-3) / 1e9  # 2 B grad + 12 B state read + 12 B written + 2 B param
            adamw[where] = {"ms": round(ms, 4), "placement": opt.location, "GB/s": round(gbs, 1),
                            **({"frac_hbm": round(gbs / hbm_gbs, 3)} if where == "device" else {})}
            opt.close()
        out["paged_adamw_7b_adapters"] = {"what": f"one AdamW step over the 14 adapter tensors of the 7B set "
                                                  f"({n_el / 1e6:.2f} M fp16 parameters, fp32 state in managed memory)",
                                          **adamw}
        del f16, ws, grads, params
        torch.cuda.empty_cache()

    if want("llama33b_block"):
        # -- 33B-shaped block: forward saving XA, backward recomputing XA (checkpoint style)
        wl = WORKLOADS["llama33b_block"]
        M = wl.M[0]
        state = []
        for li, lin in enumerate(wl.linears):
            inp = layer_inputs(wl, li, M, device=dev)
            pk, q, s2 = quantized(inp["W"])
            del inp["W"]
            state.append((lin, pk, q, s2, inp, torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev),
                          torch.empty((M, wl.r), dtype=torch.bfloat16, device=dev),
                          torch.empty((M, lin.K), dtype=torch.bfloat16, device=dev),
                          torch.empty((lin.K, wl.r), dtype=torch.bfloat16, device=dev),
                          torch.empty((wl.r, lin.N), dtype=torch.bfloat16, device=dev)))
        ws = torch.empty(max(binding.workspace_bytes(M, lin.N, lin.K, wl.r) for lin, *_ in state),
                         dtype=torch.uint8, device=dev)

        def block():
            for lin, pk, q, s2, inp, Y, XA, dX, dA, dB in state:
                binding.linear_fwd(pk, q, s2, inp["X"], inp["A"], inp["B"], wl.alpha, lin.N, lin.K, Y=Y, XA_out=XA,
                                   workspace=ws)
            for lin, pk, q, s2, inp, Y, XA, dX, dA, dB in reversed(state):
                binding.linear_bwd(pk, q, s2, inp["X"], inp["dY"], inp["A"], inp["B"], wl.alpha, lin.N, lin.K, XA=None,
                                   dX=dX, dA=dA, dB=dB, workspace=ws)
        ms_seq = device_ms(block, 3)
        # the same work through the block executor (qlora_block_fwd/bwd: one call
        # per pass, linears over two streams), checkpoint schedule: the forward
        # saves nothing and the backward recomputes X A
        lins = [{"packed": pk, "q": q, "scale2": s2, "N": lin.N, "K": lin.K, "X": inp["X"], "A": inp["A"],
                 "B": inp["B"], "Y": Y, "XA": XA, "dY": inp["dY"], "dX": dX, "dA": dA, "dB": dB}
                for lin, pk, q, s2, inp, Y, XA, dX, dA, dB in state]
        bws = torch.empty(binding.block_workspace_bytes(lins, M, wl.r), dtype=torch.uint8, device=dev)
        rev = lins[::-1]

        def block_exec():
            binding.block_fwd(lins, M, wl.r, wl.alpha, save_xa=False, workspace=bws)
            binding.block_bwd(rev, M, wl.r, wl.alpha, save_xa=False, workspace=bws)
        ms = device_ms(block_exec, 3)
        flops = sum(linear_flops(M, lin.N, lin.K, wl.r) + 2 * M * lin.K * wl.r for lin, *_ in state)
        out["llama33b_block"] = {"what": "7 linears (d=6656, ffn=17920), M=2048, r=64: block forward saving nothing, "
                                         "block backward recomputing XA and re-dequantizing W (qlora_block_fwd/bwd, "
                                         "2 streams)",
                                 "ms": round(ms, 4), "ms_linears_one_by_one": round(ms_seq, 4),
                                 "GFLOP": round(flops / 1e9, 1), **frac_tc(flops / (ms * 1e-3) / 1e12)}
        del state, ws, bws, lins, rev
        torch.cuda.empty_cache()
    return out


def run_native(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from bit_quantized_lora_blockwise_b200 import binding
    from bit_quantized_lora_blockwise_b200.build import build
    from bit_quantized_lora_blockwise_b200.dp import allreduce_adapter_grads
    from bit_quantized_lora_blockwise_b200.inputs import WORKLOADS

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    build()
    binding.load()
    if args.phase:
        pk, _ = peaks()
        res = workload_phases(dev, pk["hbm_gbs"], pk["bf16_tflops"], only=args.phase)
        if rank == 0:
            print(json.dumps({"phase": args.phase, "workloads": res, "device_error": binding.device_error()}))
        return
    wl = WORKLOADS[WORKLOAD]
    M = wl.M[0]
    keep = [n for n in args.linears.split(",") if n]
    layers = [LinearState(wl, i, M, dev) for i in range(len(wl.linears))
              if not keep or wl.linears[i].name in keep]
    ws = torch.empty(max(max(l.ws_bytes, binding.workspace_bytes(SMALL_M, l.N, l.K, l.r)) for l in layers),
                     dtype=torch.uint8, device=dev)
    nl = len(layers)

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        return e

    # per step, per linear: events around the codec calls and the fused GEMMs
    def make_events():
        return [{k: (ev(), ev()) for k in ("quantize", "double_quant", "dequant", "fwd_gemm", "bwd_gemm",
                                            "fwd_call", "bwd_call", "smallm_fwd")}
                for _ in range(nl)]

    def linear_step(L, e=None, tr=None):
        """One linear's share of the step. e: events around every call
        (breakdown pass); tr: events around the fused GEMMs only, recorded by
        the library on its stream (headline pass)."""
        if tr is not None and e is None:
            binding.set_trace_events(*tr[0])
            binding.quantize_nf4(L.W, packed=L.packed, absmax=L.absmax)
            binding.double_quant(L.absmax, q=L.q, scale2=L.scale2)
            binding.dequant(L.packed, L.q, L.scale2, L.N, L.K, out=L.Wq)
            binding.linear_fwd(L.packed, L.q, L.scale2, L.X, L.A, L.B, L.alpha, L.N, L.K, Y=L.Y,
                               XA_out=L.XA, workspace=ws)
            binding.set_trace_events(*tr[1])
            binding.linear_bwd(L.packed, L.q, L.scale2, L.X, L.dY, L.A, L.B, L.alpha, L.N, L.K, XA=L.XA,
                               dX=L.dX, dA=L.dA, dB=L.dB, workspace=ws)
            binding.set_trace_events(None, None)
            binding.linear_fwd(L.packed, L.q, L.scale2, L.Xs, L.A, L.B, L.alpha, L.N, L.K, Y=L.Ys,
                               XA_out=L.XAs, workspace=ws)
            return
        if e: e["quantize"][0].record()
        binding.quantize_nf4(L.W, packed=L.packed, absmax=L.absmax)
        if e: e["quantize"][1].record(); e["double_quant"][0].record()
        binding.double_quant(L.absmax, q=L.q, scale2=L.scale2)
        if e: e["double_quant"][1].record(); e["dequant"][0].record()
        binding.dequant(L.packed, L.q, L.scale2, L.N, L.K, out=L.Wq)
        if e: e["dequant"][1].record(); binding.set_trace_events(*e["fwd_gemm"]); e["fwd_call"][0].record()
        binding.linear_fwd(L.packed, L.q, L.scale2, L.X, L.A, L.B, L.alpha, L.N, L.K, Y=L.Y,
                           XA_out=L.XA, workspace=ws)
        if e: e["fwd_call"][1].record(); binding.set_trace_events(*e["bwd_gemm"]); e["bwd_call"][0].record()
        binding.linear_bwd(L.packed, L.q, L.scale2, L.X, L.dY, L.A, L.B, L.alpha, L.N, L.K, XA=L.XA,
                           dX=L.dX, dA=L.dA, dB=L.dB, workspace=ws)
        if e: e["bwd_call"][1].record(); binding.set_trace_events(None, None); e["smallm_fwd"][0].record()
        binding.linear_fwd(L.packed, L.q, L.scale2, L.Xs, L.A, L.B, L.alpha, L.N, L.K, Y=L.Ys,
                           XA_out=L.XAs, workspace=ws)
        if e: e["smallm_fwd"][1].record()

    def step(evs=None, trace=None):
        """One pass of the hot path over every linear."""
        for i, L in enumerate(layers):
            linear_step(L, evs[i] if evs else None, trace[i] if trace else None)
        if world > 1:
            # data parallel over tokens: sum the adapter gradients of all ranks
            allreduce_adapter_grads([t for L in layers for t in (L.dA, L.dB)])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    evs_steps = [make_events() for _ in range(args.steps)]
    # live events around the fused GEMMs in the last timed step only: an event
    # between the call's low-rank launch and its GEMM would stop the GEMM's
    # main loop from starting under that launch, so the other steps run
    # without them
    trace_last = [((ev(), ev()), (ev(), ev())) for _ in range(nl)]
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    launches0 = binding.launch_count()
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark_start()
    t_start.record()
    for k in range(args.steps):
        step(trace=trace_last if k == args.steps - 1 else None)
    t_stop.record()
    torch.cuda.synchronize()
    sampler.mark_stop()
    if world > 1:
        dist.barrier()
    launches = binding.launch_count() - launches0
    clocks = sampler.stop()
    # fused-GEMM kernel times measured live in the last timed step
    live_ms = {"fwd_gemm": sum(trace_last[i][0][0].elapsed_time(trace_last[i][0][1]) for i in range(nl)),
               "bwd_gemm": sum(trace_last[i][1][0].elapsed_time(trace_last[i][1][1]) for i in range(nl))}
    # breakdown pass (events around every call; not part of the headline).
    # Each pass is queued behind a few milliseconds of GPU sleep, so the host
    # has enqueued it before it starts and the events time the device only
    # (a small call takes less device time than its host-side launch).
    for k in range(args.steps):
        torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
        step(evs_steps[k])
    torch.cuda.synchronize()
    # codec rows and the few-token forward back to back (the 7 linears' calls
    # in a row, one event pair, queued the same way): their device throughput
    # without the per-call event gaps of the breakdown pass
    codec_calls = {
        "quantize_dq": lambda L: binding.quantize_dq(L.W, packed=L.packed, q=L.q, scale2=L.scale2),
        "quantize": lambda L: binding.quantize_nf4(L.W, packed=L.packed, absmax=L.absmax),
        "double_quant": lambda L: binding.double_quant(L.absmax, q=L.q, scale2=L.scale2),
        "dequant": lambda L: binding.dequant(L.packed, L.q, L.scale2, L.N, L.K, out=L.Wq),
        "smallm_fwd": lambda L: binding.linear_fwd(L.packed, L.q, L.scale2, L.Xs, L.A, L.B, L.alpha, L.N, L.K,
                                                   Y=L.Ys, XA_out=L.XAs, workspace=ws),
    }
    codec_run_ms = {}
    for name, call in codec_calls.items():
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(QUEUE_AHEAD_CYCLES)
        c0.record()
        for _ in range(args.steps):
            for L in layers:
                call(L)
        c1.record()
        torch.cuda.synchronize()
        codec_run_ms[name] = c0.elapsed_time(c1) / args.steps
    compare = compare_dequant_then_library_gemm(layers, ws, args.steps) if not args.no_compare else None
    ms = t_start.elapsed_time(t_stop) / args.steps
    if world > 1:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())

    step_flops = sum(L.flops() for L in layers)
    value = step_flops * world / (ms * 1e-3) / 1e12

    # per-phase device times (mean over the timed steps)
    phase = {k: [] for k in ("quantize", "double_quant", "dequant", "fwd_gemm", "bwd_gemm", "fwd_call",
                             "bwd_call", "smallm_fwd")}
    for evs in evs_steps:
        for k in phase:
            phase[k].append(sum(evs[i][k][0].elapsed_time(evs[i][k][1]) for i in range(nl)))
    phase_ms = {k: sum(v) / len(v) for k, v in phase.items()}
    codec_bytes = {k: sum(L.codec_bytes()[k] for L in layers)
                   for k in ("quantize_dq", "quantize", "double_quant", "dequant")}
    gemm_flops = {"fwd_gemm": sum(2 * M * L.N * L.K + 2 * M * L.r * L.N for L in layers),
                  "bwd_gemm": sum(2 * M * L.N * L.K + 2 * M * L.r * L.K for L in layers)}
    pk, pk_kind = peaks()
    hbm = pk["hbm_gbs"]
    # The fused GEMMs are timed inside a region of tens of milliseconds during
    # which the clocks stay at their maximum (the sampled median is in the
    # line): the burst bf16 peak is the denominator. The clock-matched
    # fraction (burst peak scaled by median/max SM clock), the fraction of the
    # sustained peak and of the 2.25 PFLOP/s dense bf16 spec sit beside it.
    tc = pk["bf16_tflops"]
    tc_sustained = pk.get("bf16_tflops_sustained")
    clock_ratio = 1.0
    if clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        clock_ratio = min(1.0, clocks["sm_mhz"] / clocks["sm_max_mhz"])
    phases = {}
    for k in ("quantize_dq", "quantize", "double_quant", "dequant"):
        gbs_run = codec_bytes[k] / (codec_run_ms[k] * 1e-3) / 1e9
        phases[k] = {"back_to_back": {"ms": round(codec_run_ms[k], 4), "GB/s": round(gbs_run, 1),
                                      "frac_hbm": round(gbs_run / hbm, 3),
                                      "frac_8tbs": round(gbs_run / SPEC_HBM_GBS, 3)}}
        if k in phase_ms:  # in the step (per-call events)
            gbs = codec_bytes[k] / (phase_ms[k] * 1e-3) / 1e9
            phases[k].update({"ms": round(phase_ms[k], 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                              "frac_8tbs": round(gbs / SPEC_HBM_GBS, 3)})
        else:
            phases[k]["note"] = ("not in the step (the step runs quantize_nf4 + double_quant, measured faster "
                                 "than the one-pass call); back to back only")
    for k in ("fwd_gemm", "bwd_gemm"):
        tf = gemm_flops[k] / (phase_ms[k] * 1e-3) / 1e12
        phases[k] = {"ms": round(phase_ms[k], 4), "TFLOP/s": round(tf, 1), "frac_tensor": round(tf / tc, 3),
                     "frac_spec": round(tf / SPEC_BF16_TFLOPS, 3)}
    # few-token forward: a whole qlora_linear_fwd call (X A product + weight stream)
    sm_bytes = sum(L.smallm_bytes() for L in layers)
    sm_gbs = sm_bytes / (phase_ms["smallm_fwd"] * 1e-3) / 1e9
    sm_gbs_run = sm_bytes / (codec_run_ms["smallm_fwd"] * 1e-3) / 1e9
    phases["smallm_fwd"] = {"ms": round(phase_ms["smallm_fwd"], 4), "tokens": SMALL_M, "GB/s": round(sm_gbs, 1),
                            "frac_hbm": round(sm_gbs / hbm, 3), "frac_8tbs": round(sm_gbs / SPEC_HBM_GBS, 3),
                            "TFLOP/s": round(sum(L.smallm_flops() for L in layers) /
                                             (phase_ms["smallm_fwd"] * 1e-3) / 1e12, 2),
                            "back_to_back": {"ms": round(codec_run_ms["smallm_fwd"], 4), "GB/s": round(sm_gbs_run, 1),
                                             "frac_hbm": round(sm_gbs_run / hbm, 3)}}
    # whole qlora_linear_fwd / _bwd calls (fused GEMM + constants pass + adapter GEMMs)
    for k in ("fwd_call", "bwd_call"):
        phases[k] = {"ms": round(phase_ms[k], 4), "outside_fused_gemm_ms":
                     round(phase_ms[k] - phase_ms[k.replace("call", "gemm")], 4)}
    # dominant kernel: the fused dequant-GEMM with the larger live share of the step
    dom = max(("fwd_gemm", "bwd_gemm"), key=lambda k: live_ms[k])
    achieved = gemm_flops[dom] / nl / (live_ms[dom] / nl * 1e-3) / 1e12
    traffic = profiled_traffic("qgemm_" + dom)
    roofline = {"bound": "tensor", "kernel": f"fused dequant-GEMM ({dom.split('_')[0]}), per-launch average "
                "over the 7 linears of the last timed step (the only step with events around the kernel)",
                "achieved": round(achieved, 1), "peak": tc,
                "peak_kind": f"{pk_kind} bf16_tflops (burst): the kernel is timed inside a region of "
                             f"{ms * args.steps:.0f} ms at the sampled clocks",
                "unit": "TFLOP/s", "frac": round(achieved / tc, 4),
                "frac_clock_matched": round(achieved / (tc * clock_ratio), 4),
                "frac_sustained": round(achieved / tc_sustained, 4) if tc_sustained else None,
                "frac_spec": round(achieved / SPEC_BF16_TFLOPS, 4),
                "traffic": traffic, "live_ms_per_step": {k: round(v, 4) for k, v in live_ms.items()}}

    # ------------------------------------------------------------ e2e leg --
    e2e = None
    if not args.no_e2e:
        host = []
        for L in layers:
            host.append({k: getattr(L, k).cpu().pin_memory() for k in ("W", "X", "A", "B", "dY")})
        h2d = sum(t.numel() * t.element_size() for h in host for t in h.values())
        outs = [(torch.empty_like(L.dA, device="cpu").pin_memory(), torch.empty_like(L.dB, device="cpu").pin_memory())
                for L in layers]
        d2h = sum(a.numel() * a.element_size() + b.numel() * b.element_size() for a, b in outs)

        # Copies run on their own stream: linear i's inputs go up while the
        # linears before it compute, and its dA, dB come back as soon as it
        # is done. The compute of linear i waits for its copy; the next
        # step's copy into linear i's buffers waits for this step's compute
        # of linear i.
        copy_stream = torch.cuda.Stream(device=dev)
        done = [torch.cuda.Event() for _ in layers]
        for d_ev in done:
            d_ev.record()

        def e2e_step():
            main = torch.cuda.current_stream()
            start = torch.cuda.Event()
            start.record(main)
            arrived = []
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(start)
                for L, h, d_ev in zip(layers, host, done):
                    copy_stream.wait_event(d_ev)
                    for k, t in h.items():
                        getattr(L, k).copy_(t, non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(copy_stream)
                    arrived.append(ev)
            for L, ev, d_ev in zip(layers, arrived, done):
                main.wait_event(ev)
                linear_step(L)
                d_ev.record(main)
            if world > 1:
                allreduce_adapter_grads([t for L in layers for t in (L.dA, L.dB)])
                for d_ev in done:
                    d_ev.record(main)
            with torch.cuda.stream(copy_stream):
                for L, (a_h, b_h), d_ev in zip(layers, outs, done):
                    copy_stream.wait_event(d_ev)
                    a_h.copy_(L.dA, non_blocking=True)
                    b_h.copy_(L.dB, non_blocking=True)
                fin = torch.cuda.Event()
                fin.record(copy_stream)
            main.wait_event(fin)

        e2e_step()
        torch.cuda.synchronize()
        e2e_steps = max(2, min(args.steps, 5))
        if world > 1:
            dist.barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(e2e_steps):
            e2e_step()
        a1.record()
        torch.cuda.synchronize()
        ems = a0.elapsed_time(a1) / e2e_steps
        if world > 1:
            t = torch.tensor([ems], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        e2e = {"value": step_flops * world / (ems * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": ems,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}

    workloads = None
    if rank == 0 and not args.no_workloads:
        workloads = workload_phases(dev, hbm, tc)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": WORKLOAD, "linears": [f"{L.name}:{L.N}x{L.K}" for L in layers],
                           "M": M, "r": wl.r, "alpha": wl.alpha, "per_rank_tokens": M,
                           "parallelism": f"dp{world}",
                           "l2": "inputs larger than L2 (405 MB of bf16 weights + 320 MB of activations per step)",
                           "step": "per linear: quantize_nf4, double_quant, dequant, linear_fwd, linear_bwd, "
                                   f"linear_fwd on the first {SMALL_M} tokens"},
                "phases": phases, "roofline": roofline, "gpu_launches": launches,
                "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu,
                "compare_dequant_then_library_gemm": compare, "workloads": workloads,
                "device_error": binding.device_error()}
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if args.impl == "reference":
            if rank == 0:
                run_reference(args, rank)
            return
        import torch
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        try:
            run_native(args, rank, world, local_rank)
        finally:
            dist.destroy_process_group()
        return
    if args.impl == "reference":
        run_reference(args, rank)
    else:
        run_native(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
