#!/usr/bin/env python
"""Benchmark of the QLoRA quantized linear layer on B200.

One step = the whole hot path over one batch of the 65B-shaped decoder block
(q/k/v/o W[8192,8192], gate/up W[22016,8192], down W[8192,22016]; Student-t(5)
weights with 0.1% x10 outliers; 2048 tokens per GPU; LoRA r=64 alpha=16):
NF4 + Double Quantization of all 7 weights, forward of every linear, backward
(dX, dA, dB) of every linear, and with N > 1 GPUs one NCCL all-reduce of the
LoRA gradients (data parallel, weak scaling).

Printed metric: algorithmic fwd+bwd TFLOP/s of the step (sum over ranks /
max-over-ranks device time).  Extra keys: roofline of the dominant kernel
(live CUDA-event times), e2e (host buffers, copies inside the timed region),
cpu_baseline (the CPU oracle on a bounded sample), clocks, kernel launch count,
and the small-M decode sweep in HBM GB/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s and small-M GB/s, as fraction of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_HBM_GBS = 8000.0          # HBM3e, the 8 TB/s figure
NOMINAL_BF16_TFLOPS = 2250.0      # dense bf16 tensor-core peak (NVIDIA's 4.5 PFLOP/s figure is with 2:4 sparsity)
AT_MAX_CLOCK = 0.97               # median SM clock at or above this share of the maximum: not power-capped
L2_FLUSH_BYTES = 256 << 20
PACKED_BYTES_PER_WEIGHT = 0.5 + 1 / 64 + 4 / (64 * 256)     # codes + E4M3 constants + c2
ALU_OPS_PER_WEIGHT = 2.5        # exact bf16 table expansion: 19 permute/logic ops per 8 weights + 8 per 64-weight table
ALU_OPS_PER_CLK_SM = 64.0       # ALU pipe: 2 warp-instructions per clock per SM (ncu's peak_sustained for
                                # sm__inst_executed_pipe_alu), 32 lanes each


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="block65b")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--case", choices=["fwd", "bwd", "quantize", "dequantize"], default=None,
                   help="profiling mode: run one op of one linear --reps times and exit")
    p.add_argument("--shape", default="2048,22016,8192", help="M,N,K for --case")
    p.add_argument("--rank", type=int, default=64, help="LoRA rank for --case")
    p.add_argument("--reps", type=int, default=3)
    p.add_argument("--only", choices=["decode", "hbm"], default=None,
                   help="measurement mode: print only the small-M sweep or the quantize/dequantize rates")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def step_flops(wl, M):
    """Algorithmic fwd+bwd flops of one step on one rank: per linear
    fwd 2MNK + 2Mr(N+K), bwd 2MNK + 4Mr(N+K)."""
    total = 0
    for (N, K) in wl.linears:
        total += 2 * M * N * K + 2 * M * wl.r * (N + K)
        total += 2 * M * N * K + 4 * M * wl.r * (N + K)
    return total


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every 5 ms while the
    timed region runs (the region can be far shorter than nvidia-smi's interval)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self.error = None

    def _handle(self, pynvml):
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._handle(pynvml)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception as e:          # no NVML: report why
            self.error = f"nvml unavailable: {e}"
            return
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    clk = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((float(clk), int(rs)))
                except Exception as e:
                    self.error = str(e)
                self._stop.wait(0.005)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.error or "not sampled"]}
        self._stop.set()
        self._thread.join(timeout=2)
        clks = sorted(c for c, _ in self.samples)
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": clks[len(clks) // 2] if clks else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(clks),
                "sm_mhz_min": clks[0] if clks else None, "source": "NVML, every 5 ms during the timed steps"}


# ----------------------------------------------------------------------------- traffic from ncu

def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments or blank-line and trailing-space differences."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] in "\"'":                       # string and character literals stay as they are
            q, j = text[i], i + 1
            while j < n and text[j] != q:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln)


# The fused dequant-GEMM's sources: its device and launch code, its parameter structs, the PTX
# wrappers and the shared helpers it is compiled from.
FUSED_GEMM_SOURCES = ("gemm_tc.cu", "gemm_tc.cuh", "qlora_internal.cuh", "tc_ptx.cuh")


def kernel_source_sha(files=FUSED_GEMM_SOURCES):
    """Hash of the fused GEMM's sources' code (comments ignored): the DRAM counters recorded in
    profiles/traffic.txt stay valid while it is unchanged."""
    h = hashlib.sha256()
    for name in sorted(files):
        with open(os.path.join(ROOT, "bit_nf4_quantized_23_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_kind: str):
    """DRAM bytes per launch recorded from an ncu capture (profiles/traffic.txt), or None
    when the kernel sources changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha()
    with open(path) as f:
        for ln in f:
            ln = ln.split("#")[0].strip()
            if not ln:
                continue
            kv = dict(part.split("=", 1) for part in ln.split())
            if kv.get("kind") == kernel_kind and kv.get("source_sha") == sha:
                return float(kv["bytes_per_launch"])
    return None


# ----------------------------------------------------------------------------- CPU oracle sample

def oracle_sample(wl, rows: int = 256, reps: int = 1, w_rows: int | None = None):
    """Time the CPU oracle on one linear of the workload (quantize all of W, or its first
    `w_rows` rows, dequantize, forward and backward on `rows` token rows).
    Returns (flops, seconds, description)."""
    import numpy as np
    import synthetic_inputs as si
    from oracle import nf4_oracle as o
    N, K = wl.linears[0]
    W = si.bf16_bits(si.weight(wl, 0))
    if w_rows is not None and w_rows < N:
        N = w_rows
        W = W[:N]
        B_rows = N
    else:
        B_rows = N
    X = si.bf16_bits(si.activations(wl, K, wl.M if isinstance(wl.M, int) else 16))[:rows]
    A, B = (si.bf16_bits(t) for t in si.lora(wl, 0))
    B = B[:B_rows]
    dY = si.bf16_bits(si.grad_output(wl, 0, wl.M if isinstance(wl.M, int) else 16))[:rows, :N]
    t0 = time.perf_counter()
    for _ in range(reps):
        qw = o.quantize_nf4_dq(W)
        Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], N, K)
        o.linear_forward(X, Wh, A, B, wl.alpha, wl.r)
        o.linear_backward(X, dY, Wh, A, B, wl.alpha, wl.r)
    dt = (time.perf_counter() - t0) / reps
    m = X.shape[0]
    flops = 2 * m * N * K + 2 * m * wl.r * (N + K) + 2 * m * N * K + 4 * m * wl.r * (N + K)
    desc = (f"oracle (NumPy, fp64 GEMMs) on linear 0 of {wl.name} restricted to W[{N},{K}]: full NF4+DQ "
            f"quantize and dequantize of that W, then fwd+bwd on {m} of the {wl.M} token rows")
    return flops, dt, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synthetic_inputs as si
    wl = si.WORKLOADS[args.workload]
    times = []
    flops = 0
    desc = ""
    # about 2 minutes in all: a full W[8192,8192] sample takes ~16 s on 8 host cores
    n_calls = args.warmup + args.steps
    w_rows = int(max(256, min(wl.linears[0][0], wl.linears[0][0] * 120.0 / (16.0 * n_calls))) // 256 * 256)
    for i in range(n_calls):
        f, dt, desc = oracle_sample(wl, w_rows=w_rows)
        if i >= args.warmup:
            times.append(dt)
            flops = f
    sec = sum(times) / len(times)
    value = flops / sec / 1e12
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.description, "sample": desc},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm

class Linear:
    pass


def setup_workload(wl, rank, device):
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si
    M = wl.M
    xs = {}
    lins = []
    for i, (N, K) in enumerate(wl.linears):
        L = Linear()
        L.N, L.K = N, K
        L.W = si.weight(wl, i).to(device)                        # frozen weight (replicated)
        if K not in xs:
            xs[K] = si.activations(wl, K, M, seed=rank).to(device)
        L.X = xs[K]
        L.A, L.B = (t.to(device) for t in si.lora(wl, i))
        L.dY = si.grad_output(wl, i, M, seed=rank).to(device)
        L.w = q4.NF4Weight.empty(N, K, device)
        L.qws = torch.empty(q4.qlora_nf4_sizes(N, K)["workspace"], dtype=torch.uint8, device=device)
        L.lws = torch.empty(max(16, q4.qlora_linear_workspace_size(M, N, K, wl.r)), dtype=torch.uint8,
                            device=device)
        L.Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
        L.U = torch.empty(M, wl.r, dtype=torch.float32, device=device)
        L.dX = torch.empty(M, K, dtype=torch.bfloat16, device=device)
        lins.append(L)
    grads = torch.empty(grad_buffer_numel(wl), dtype=torch.float32, device=device)
    for L, (dA, dB) in zip(lins, grad_views(wl, grads)):
        L.dA, L.dB = dA, dB
    return lins, grads


def grad_buffer_numel(wl):
    """Length of the flat fp32 buffer that holds every linear's LoRA gradients."""
    return sum(wl.r * K + N * wl.r for N, K in wl.linears)


def grad_views(wl, grads):
    """Per linear (dA [r,K], dB [N,r]) as views of the flat buffer, linear after linear, dA first.
    Data parallelism all-reduces this one buffer per step (one collective for all linears)."""
    views, off = [], 0
    for N, K in wl.linears:
        dA = grads[off:off + wl.r * K].view(wl.r, K)
        off += wl.r * K
        dB = grads[off:off + N * wl.r].view(N, wl.r)
        off += N * wl.r
        views.append((dA, dB))
    assert off == grads.numel()
    return views


def make_step(wl, lins, grads, world):
    import torch
    import bit_nf4_quantized_23_b200 as q4

    def step():
        for L in lins:
            q4.qlora_quantize_nf4_dq(L.W, out=L.w, workspace=L.qws)
        for L in lins:
            q4.qlora_linear_fwd(L.w, L.X, L.A, L.B, wl.r, wl.alpha, out=L.Y, U_out=L.U, workspace=L.lws)
        for L in reversed(lins):
            q4.qlora_linear_bwd(L.w, L.X, L.dY, L.A, L.B, wl.r, wl.alpha, U_saved=L.U, dX=L.dX,
                                dA=L.dA, dB=L.dB, workspace=L.lws)
        if world > 1:
            torch.distributed.all_reduce(grads)
    return step


def timed_steps(step, steps, flush, stream):
    """Device time of `steps` steps (L2 flushed before each, outside the timing)."""
    import torch
    total = 0.0
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        b.synchronize()
        total += a.elapsed_time(b)
    return total


def decode_sweep(device, peaks):
    """Small-M forward on the decode shapes: HBM GB/s over packed NF4 + DQ constant bytes, for the
    whole forward call and for the weight-streaming kernel alone (live CUDA events)."""
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si
    wl = si.WORKLOADS["decode"]
    props = torch.cuda.get_device_properties(device)
    l2 = props.L2_cache_size
    # ALU roofline of an exact bf16 dequant (every weight through a per-block 16-entry table):
    # >= 2.5 byte-permute/logic ops per weight on a pipe that issues 64 per clock per SM
    alu_gbs = (ALU_OPS_PER_CLK_SM * props.multi_processor_count * peaks.get("sm_max_mhz", 1965.0) * 1e6
               / ALU_OPS_PER_WEIGHT * PACKED_BYTES_PER_WEIGHT / 1e9)
    out = {"alu_roofline_GB/s": round(alu_gbs, 1),
           "alu_roofline_basis": f"{ALU_OPS_PER_WEIGHT} ALU ops/weight, {ALU_OPS_PER_CLK_SM} ops/clk/SM (ncu: "
                                 "sm__inst_executed_pipe_alu peak_sustained 2 warp-instr/clk/SM), SMs x max SM clock"}
    for i, (N, K) in enumerate(wl.linears):
        W = si.weight(wl, i).to(device)
        A, B = (t.to(device) for t in si.lora(wl, i))
        wbytes = PACKED_BYTES_PER_WEIGHT * N * K
        copies = max(2, int(3 * l2 // wbytes) + 1)
        ws = [q4.qlora_quantize_nf4_dq(W) for _ in range(copies)]
        del W
        for M in wl.M:
            X = si.activations(wl, K, M).to(device)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            lws = torch.empty(max(16, q4.qlora_linear_workspace_size(M, N, K, wl.r)), dtype=torch.uint8,
                              device=device)
            call = lambda j: q4.qlora_linear_fwd(ws[j % copies], X, A, B, wl.r, wl.alpha, out=Y, save_U=False,
                                                 workspace=lws)
            for j in range(3):
                call(j)
            reps = 8 * copies
            torch.cuda.synchronize()
            q4.qlora_timing_read("decode", reset=True)
            q4.qlora_timing_enable(True)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for j in range(reps):
                call(j)
            b.record()
            b.synchronize()
            q4.qlora_timing_enable(False)
            n_k, ms_k = q4.qlora_timing_read("decode", reset=True)
            ms = a.elapsed_time(b) / reps
            kms = ms_k / max(1, n_k)
            out[f"W[{N},{K}] M={M}"] = {
                "call_us": round(ms * 1e3, 2), "call_GB/s": round(wbytes / (ms * 1e-3) / 1e9, 1),
                "kernel_us": round(kms * 1e3, 2), "kernel_GB/s": round(wbytes / (kms * 1e-3) / 1e9, 1),
                "kernel_frac_of_hbm": round(wbytes / (kms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
                "kernel_frac_of_nominal": round(wbytes / (kms * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 3),
                "kernel_frac_of_alu_roofline": round(wbytes / (kms * 1e-3) / 1e9 / alu_gbs, 3)}
        if i == len(wl.linears) - 1:
            # one base, many adapters: 16 tokens, each on its own adapter, same weight copies
            M, n_ad = 16, 16
            X = si.activations(wl, K, M).to(device)
            A_all = torch.stack([si.lora(wl, i)[0]] * n_ad).to(device)
            B_all = torch.stack([si.lora(wl, i)[1]] * n_ad).to(device)
            idx = torch.arange(n_ad, dtype=torch.int32, device=device)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            lws = torch.empty(max(16, q4.qlora_linear_workspace_size(M, N, K, wl.r)), dtype=torch.uint8,
                              device=device)
            call = lambda j: q4.qlora_linear_fwd_multi(ws[j % copies], X, A_all, B_all, idx, wl.r, wl.alpha,
                                                       out=Y, workspace=lws)
            for j in range(3):
                call(j)
            reps = 8 * copies
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for j in range(reps):
                call(j)
            b.record()
            b.synchronize()
            ms = a.elapsed_time(b) / reps
            out[f"W[{N},{K}] M=16, 16 adapters"] = {
                "call_us": round(ms * 1e3, 2), "call_GB/s": round(wbytes / (ms * 1e-3) / 1e9, 1),
                "note": "qlora_linear_fwd_multi: every token on its own adapter over one base"}
        del ws
        torch.cuda.empty_cache()
    return out


def dequant_rate(device, peaks, wl):
    """qlora_dequantize on the largest weight of the workload: GB/s over 0.516 B in + 2 B out per weight."""
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si
    i = max(range(len(wl.linears)), key=lambda j: wl.linears[j][0] * wl.linears[j][1])
    N, K = wl.linears[i]
    w = q4.qlora_quantize_nf4_dq(si.weight(wl, i).to(device))
    out = torch.empty(N, K, dtype=torch.bfloat16, device=device)
    for _ in range(3):
        q4.qlora_dequantize(w, out=out)
    reps = 20
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        q4.qlora_dequantize(w, out=out)
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b) / reps
    gbs = (PACKED_BYTES_PER_WEIGHT + 2.0) * N * K / (ms * 1e-3) / 1e9
    return {"shape": [N, K], "us": round(ms * 1e3, 1), "GB/s": round(gbs, 1),
            "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 3), "frac_of_nominal": round(gbs / NOMINAL_HBM_GBS, 3),
            "bytes_per_weight": round(PACKED_BYTES_PER_WEIGHT + 2.0, 6)}


def quantizer_variants(device, peaks, wl):
    """Quantizer variants on the workload's first weight (and on a normal one of the same shape):
    relative squared error sum (W_hat - W)^2 / sum W^2 of each codebook with and without double
    quantization (from the library's dequantized weight), and the quantize rate of each variant."""
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si
    N, K = wl.linears[0]
    weights = {wl.dist: si.weight(wl, 0).to(device),
               "normal": si.normal_bf16((N, K), wl.sigma, 0, wl.name, "W0n").to(device)}
    out = {"weight": f"W[{N},{K}]", "metric": "sum (W_hat - W)^2 / sum W^2 (fp64)"}
    for dist, W in weights.items():
        w64 = W.double()
        den = float((w64 * w64).sum())
        for codebook in ("nf4", "uniform4"):
            for dq in (True, False):
                w = q4.qlora_quantize_nf4_dq(W, codebook=codebook, double_quant=dq)
                Wh = q4.qlora_dequantize(w).double()
                key = f"{dist}/{codebook}/{'dq' if dq else 'single'}"
                out[key] = {"rel_sq_error": float(((Wh - w64) ** 2).sum()) / den}
                if dist == "normal":
                    for _ in range(2):
                        q4.qlora_quantize_nf4_dq(W, out=w)
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    for _ in range(10):
                        q4.qlora_quantize_nf4_dq(W, out=w)
                    b.record()
                    b.synchronize()
                    ms = a.elapsed_time(b) / 10
                    nbytes = (2.0 + (0.5 + 1 / 64 + 4 / 16384 if dq else 0.5 + 4 / 64)) * N * K
                    out[key]["quantize_GB/s"] = round(nbytes / (ms * 1e-3) / 1e9, 1)
        nf = out[f"{dist}/nf4/single"]["rel_sq_error"]
        out[f"{dist}/nf4_over_uniform4"] = round(nf / out[f"{dist}/uniform4/single"]["rel_sq_error"], 4)
        # the 8-bit absmax comparison quantizer (blocks of 64, one fp32 scale each)
        codes, alpha = q4.qlora_quantize_int8_absmax(W, 64)
        Wh = q4.qlora_dequantize_int8_absmax(codes, alpha, 64).double()
        key = f"{dist}/int8_absmax/b64"
        out[key] = {"rel_sq_error": float(((Wh - w64) ** 2).sum()) / den}
        if dist == "normal":
            nbytes = (2.0 + 1.0 + 4 / 64) * N * K
            Wb = torch.empty_like(W)
            for name, fn in (("quantize", lambda: q4.qlora_quantize_int8_absmax(W, 64, codes, alpha)),
                             ("dequantize", lambda: q4.qlora_dequantize_int8_absmax(codes, alpha, 64, out=Wb))):
                for _ in range(2):
                    fn()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(10):
                    fn()
                b.record()
                b.synchronize()
                ms = a.elapsed_time(b) / 10
                out[key][f"{name}_GB/s"] = round(nbytes / (ms * 1e-3) / 1e9, 1)
                out[key][f"{name}_frac_of_hbm"] = round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)
        del codes, alpha, Wh
    del weights
    torch.cuda.empty_cache()
    return out


def merge_requantize(device, peaks, wl):
    """Merge the adapters into the workload's first weight, requantize, and report the merge rate
    and the error the requantization adds against the exact merged weight W + s B A (fp64)."""
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si
    N, K = wl.linears[0]
    W = si.weight(wl, 0).to(device)
    A, B = (t.to(device) for t in si.lora(wl, 0))
    w = q4.qlora_quantize_nf4_dq(W)
    Wm = q4.qlora_merge_lora(w, A, B, wl.r, wl.alpha)
    for _ in range(3):
        q4.qlora_merge_lora(w, A, B, wl.r, wl.alpha, out=Wm)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(10):
        q4.qlora_merge_lora(w, A, B, wl.r, wl.alpha, out=Wm)
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b) / 10
    w2 = q4.qlora_quantize_nf4_dq(Wm)
    s = wl.alpha / wl.r
    exact = W.double() + s * (B.double() @ A.double())
    rel = lambda X, ref: float(((X.double() - ref) ** 2).sum() / (ref ** 2).sum())
    out = {"weight": f"W[{N},{K}]", "r": wl.r, "merge_us": round(ms * 1e3, 1),
           "merge_GB/s": round((PACKED_BYTES_PER_WEIGHT + 2.0) * N * K / (ms * 1e-3) / 1e9, 1),
           "quantize_error": rel(q4.qlora_dequantize(w), W.double()),
           "merged_rounding_error": rel(Wm, exact),
           "requantized_merged_error": rel(q4.qlora_dequantize(w2), exact),
           "metric": "sum (X - ref)^2 / sum ref^2 (fp64); ref = W for the first, W + s B A after"}
    del W, A, B, w, Wm, w2, exact
    torch.cuda.empty_cache()
    return out


def compute_dtype_compare(device, peaks, wl):
    """Forward + backward of the workload's largest linear computing in bf16 and in fp16
    (same weight, same kernels with fp16 operands): TFLOP/s of each."""
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si
    i = max(range(len(wl.linears)), key=lambda j: wl.linears[j][0] * wl.linears[j][1])
    N, K = wl.linears[i]
    M, r = wl.M, wl.r
    W = si.weight(wl, i).to(device)
    X, A, B, dY = (si.activations(wl, K, M).to(device), *[t.to(device) for t in si.lora(wl, i)],
                   si.grad_output(wl, i, M).to(device))
    flops = 4 * M * N * K + 6 * M * r * (N + K)
    out = {"linear": f"M={M}, W[{N},{K}], r={r}", "flops_per_call": flops}
    for name, dt in (("bf16", torch.bfloat16), ("fp16", torch.float16)):
        w = q4.qlora_quantize_nf4_dq(W, compute_dtype=dt)
        Xc, Ac, Bc, dYc = (t.to(dt) for t in (X, A, B, dY))
        def call():
            Y, U = q4.qlora_linear_fwd(w, Xc, Ac, Bc, r, wl.alpha)
            q4.qlora_linear_bwd(w, Xc, dYc, Ac, Bc, r, wl.alpha, U_saved=U)
        for _ in range(3):
            call()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(5):
            call()
        b.record()
        b.synchronize()
        ms = a.elapsed_time(b) / 5
        out[name] = {"ms": round(ms, 4), "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1)}
    del W, X, A, B, dY
    torch.cuda.empty_cache()
    return out


def e2e_resident(wl, lins, grads, world, device, flush, stream, steps, flops_rank, barrier):
    import torch
    import bit_nf4_quantized_23_b200 as q4
    pinned = {}

    def host_of(t):
        if id(t) not in pinned:
            pinned[id(t)] = t.cpu().pin_memory()
        return pinned[id(t)]

    x_in = [(L.X, host_of(L.X)) for L in lins]
    dy_in = [(L.dY, host_of(L.dY)) for L in lins]
    y_out = [(L.Y, torch.empty(L.Y.shape, dtype=L.Y.dtype).pin_memory()) for L in lins]
    dx_out = [(L.dX, torch.empty(L.dX.shape, dtype=L.dX.dtype).pin_memory()) for L in lins]
    grads_host = torch.empty(grads.numel(), dtype=torch.float32).pin_memory()
    h2d = sum(h.numel() * h.element_size() for h in pinned.values())
    d2h = sum(h.numel() * h.element_size() for _, h in y_out + dx_out) + grads.numel() * 4
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)

    def step():
        cur = torch.cuda.current_stream()
        s_in.wait_stream(cur)                            # after the timer starts and the last step's readers
        s_out.wait_stream(cur)
        done, ev_x, ev_dy = set(), [], {}
        with torch.cuda.stream(s_in):
            for dev_t, h in x_in:
                if id(dev_t) not in done:                # an X shared by several linears is copied once
                    dev_t.copy_(h, non_blocking=True)
                    done.add(id(dev_t))
                ev_x.append(torch.cuda.Event())
                ev_x[-1].record(s_in)
            for i in reversed(range(len(lins))):
                dy_in[i][0].copy_(dy_in[i][1], non_blocking=True)
                ev_dy[i] = torch.cuda.Event()
                ev_dy[i].record(s_in)
        for i, L in enumerate(lins):
            cur.wait_event(ev_x[i])
            q4.qlora_linear_fwd(L.w, L.X, L.A, L.B, wl.r, wl.alpha, out=L.Y, U_out=L.U, workspace=L.lws)
            s_out.wait_stream(cur)
            with torch.cuda.stream(s_out):
                y_out[i][1].copy_(y_out[i][0], non_blocking=True)
        for i in reversed(range(len(lins))):
            L = lins[i]
            cur.wait_event(ev_dy[i])
            q4.qlora_linear_bwd(L.w, L.X, L.dY, L.A, L.B, wl.r, wl.alpha, U_saved=L.U, dX=L.dX,
                                dA=L.dA, dB=L.dB, workspace=L.lws)
            s_out.wait_stream(cur)
            with torch.cuda.stream(s_out):
                dx_out[i][1].copy_(dx_out[i][0], non_blocking=True)
        if world > 1:
            torch.distributed.all_reduce(grads)
        s_out.wait_stream(cur)
        with torch.cuda.stream(s_out):
            grads_host.copy_(grads, non_blocking=True)
        cur.wait_stream(s_out)                           # the step ends when its results are on the host

    for _ in range(2):
        step()
    barrier()
    n = max(1, min(steps, 5))
    ms = timed_steps(step, n, flush, stream) / n
    if world > 1:
        t = torch.tensor([ms], device=device, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    return {"value": flops_rank * world / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "note": "weights quantized once before the timed region; per step X and dY in, Y, dX, dA and dB "
                    "out through pinned host memory, overlapping the forward and backward of all linears"}


def tensor_peak(peaks, peak_kind, clk):
    """The bf16 peak a kernel timed in the step is compared with: the burst figure when the SM clock
    stayed at its maximum during the timed steps (the kernel ran unthrottled), else the sustained
    figure measured under the power cap."""
    if peak_kind != "measured":
        return peaks["bf16_tflops"], "fallback bf16 (burst)"
    mhz, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    if mhz and mx and mhz >= AT_MAX_CLOCK * mx:
        return peaks["bf16_tflops"], (f"measured bf16 burst (MEASURED_PEAKS.json): median SM clock {mhz:.0f} "
                                      f"of max {mx:.0f} MHz during the timed steps")
    return peaks["bf16_tflops_sustained"], (f"measured bf16 sustained (MEASURED_PEAKS.json): median SM clock "
                                            f"{mhz} of max {mx} MHz during the timed steps")


def run_ours(args):
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    q4._lib.lib()
    peaks, peak_kind = load_peaks()
    wl = si.WORKLOADS[args.workload]
    lins, grads = setup_workload(wl, rank, device)
    step = make_step(wl, lins, grads, world)
    stream = torch.cuda.current_stream()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush = lambda: flush_buf.zero_()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert q4.qlora_read_device_errors(clear=True) == 0

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    q4.qlora_timing_read("fwd_main", reset=True)
    q4.qlora_timing_enable(True)
    launches0 = q4.qlora_launch_count()
    ms_total = timed_steps(step, args.steps, flush, stream)
    launches = q4.qlora_launch_count() - launches0
    barrier()
    q4.qlora_timing_enable(False)
    clk = clocks.stop()
    if world > 1:
        t = torch.tensor([ms_total], device=device, dtype=torch.float64)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms_total = float(t.item())
    ms_step = ms_total / args.steps
    flops_rank = step_flops(wl, wl.M)
    value = flops_rank * world / (ms_step * 1e-3) / 1e12

    # dominant kernel, measured live over the timed region
    kinds = {k: q4.qlora_timing_read(k) for k in ("quantize", "fwd_main", "dx_main", "lora")}
    fwd_flops = sum(2 * wl.M * L.N * L.K + 2 * wl.M * L.N * wl.r for L in lins)
    dx_flops = sum(2 * wl.M * L.N * L.K + 2 * wl.M * L.K * wl.r for L in lins)
    cand = {"fwd_main": fwd_flops, "dx_main": dx_flops}
    dom = max(cand, key=lambda k: kinds[k][1])
    n_l, ms_l = kinds[dom]
    per_launch_flops = cand[dom] / len(lins)
    achieved = per_launch_flops / (ms_l / n_l * 1e-3) / 1e12 if n_l else None
    peak, peak_source = tensor_peak(peaks, peak_kind, clk)
    frac = lambda v, p: round(v / p, 4) if (v and p) else None
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": frac(achieved, peak), "peak_source": peak_source,
                "frac_burst": frac(achieved, peaks.get("bf16_tflops")),
                "frac_sustained": frac(achieved, peaks.get("bf16_tflops_sustained")),
                "frac_nominal": frac(achieved, NOMINAL_BF16_TFLOPS),
                "traffic": recorded_traffic(dom),
                "per_launch_flops": per_launch_flops, "launches": n_l,
                "avg_launch_ms": ms_l / n_l if n_l else None}
    step_fractions = {"frac_burst": frac(value / world, peaks.get("bf16_tflops")),
                      "frac_sustained": frac(value / world, peaks.get("bf16_tflops_sustained")),
                      "frac_nominal": frac(value / world, NOMINAL_BF16_TFLOPS),
                      "note": "whole step (quantize included in the time, not in the flops) per GPU"}
    breakdown = {k: {"launches": v[0], "ms_per_step": v[1] / args.steps} for k, v in kinds.items()}
    breakdown["lora"]["note"] = ("event time of the LoRA-side kernels; the backward's dA/dB run on a side stream "
                                 "beside the dX GEMM, so part of this time overlaps it")

    # end to end through the public API with host buffers (pinned), copies inside the timed region.
    # The host-to-device copies run on their own stream in the order the kernels need them
    # (linear i's W, X, A, B, then the dY of the backward's order); each linear's quantize and
    # forward wait only for its own inputs, so copying overlaps the work already possible.  Same
    # calls and the same work as the device-timed step; quantize i runs just before forward i.
    e2e = None
    if not args.no_e2e:
        pinned = {}

        def host_of(t):
            if id(t) not in pinned:
                pinned[id(t)] = (t, t.cpu().pin_memory())
            return pinned[id(t)][1]

        fwd_in = [[(getattr(L, n), host_of(getattr(L, n))) for n in ("W", "X", "A", "B")] for L in lins]
        bwd_in = [[(L.dY, host_of(L.dY))] for L in lins]
        grads_host = torch.empty(grads.numel(), dtype=torch.float32).pin_memory()
        h2d = sum(h.numel() * h.element_size() for _, h in pinned.values())
        d2h = grads.numel() * 4
        copy_stream = torch.cuda.Stream(device=device)

        def e2e_step():
            cur = torch.cuda.current_stream()
            copy_stream.wait_stream(cur)                 # after the timer starts and the last step's readers
            done, ev_f, ev_b = set(), [], {}
            with torch.cuda.stream(copy_stream):
                for ins in fwd_in:
                    for dev_t, h in ins:
                        if id(dev_t) not in done:        # an X shared by several linears is copied once
                            dev_t.copy_(h, non_blocking=True)
                            done.add(id(dev_t))
                    ev_f.append(torch.cuda.Event())
                    ev_f[-1].record(copy_stream)
                for i in reversed(range(len(lins))):
                    for dev_t, h in bwd_in[i]:
                        dev_t.copy_(h, non_blocking=True)
                    ev_b[i] = torch.cuda.Event()
                    ev_b[i].record(copy_stream)
            for i, L in enumerate(lins):
                cur.wait_event(ev_f[i])
                q4.qlora_quantize_nf4_dq(L.W, out=L.w, workspace=L.qws)
                q4.qlora_linear_fwd(L.w, L.X, L.A, L.B, wl.r, wl.alpha, out=L.Y, U_out=L.U, workspace=L.lws)
            for i in reversed(range(len(lins))):
                L = lins[i]
                cur.wait_event(ev_b[i])
                q4.qlora_linear_bwd(L.w, L.X, L.dY, L.A, L.B, wl.r, wl.alpha, U_saved=L.U, dX=L.dX,
                                    dA=L.dA, dB=L.dB, workspace=L.lws)
            if world > 1:
                torch.distributed.all_reduce(grads)
            grads_host.copy_(grads, non_blocking=True)

        for _ in range(2):
            e2e_step()
        barrier()
        ms_e2e = timed_steps(e2e_step, max(1, min(args.steps, 5)), flush, stream) / max(1, min(args.steps, 5))
        if world > 1:
            t = torch.tensor([ms_e2e], device=device, dtype=torch.float64)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            ms_e2e = float(t.item())
        e2e = {"value": flops_rank * world / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "h2d_GB/s": round(h2d / (ms_e2e * 1e-3) / 1e9, 1),
               "note": "inputs copied on a second stream in the order the kernels need them, overlapping the work"}

    # end to end with the quantized weights resident (a training step after the one-time quantize):
    # per step the activations X and upstream gradients dY come in from pinned host memory, and Y,
    # dX and the LoRA gradients go back out.  Copies in run on one side stream in the order the
    # kernels need them, copies out on another as soon as each result is written.
    e2e_res = None
    if not args.no_e2e:
        e2e_res = e2e_resident(wl, lins, grads, world, device, flush, stream, args.steps, flops_rank, barrier)

    quant_bytes = sum((2.0 + PACKED_BYTES_PER_WEIGHT) * L.N * L.K for L in lins)
    q_ms = kinds["quantize"][1] / args.steps
    hbm = {"quantize": {"GB/s": round(quant_bytes / (q_ms * 1e-3) / 1e9, 1),
                        "frac_of_hbm": round(quant_bytes / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
                        "frac_of_nominal": round(quant_bytes / (q_ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 3),
                        "ms_per_step": round(q_ms, 4), "bytes_per_weight": round(2.0 + PACKED_BYTES_PER_WEIGHT, 6),
                        "source": "live CUDA events over the timed steps (7 calls per step)"}}
    decode = variants = merge = dtypes = None
    if rank == 0 and not args.no_decode:
        del lins
        torch.cuda.empty_cache()
        hbm["dequantize"] = dequant_rate(device, peaks, wl)
        decode = decode_sweep(device, peaks)
        variants = quantizer_variants(device, peaks, wl)
        merge = merge_requantize(device, peaks, wl)
        dtypes = compute_dtype_compare(device, peaks, wl)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, dt, desc = oracle_sample(wl)
        cpu = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc, "seconds": dt}

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.description, "tokens_per_gpu": wl.M, "global_batch_tokens": wl.M * world,
                       "r": wl.r, "alpha": wl.alpha, "parallelism": f"dp{world}",
                       "l2": "flushed before every timed step (256 MiB write, outside the timed region)",
                       "step": "quantize all 7 weights + fwd + bwd of all 7 linears"
                               + (" + NCCL all-reduce of dA/dB" if world > 1 else "")},
            "roofline": roofline, "step_fractions": step_fractions, "cpu_baseline": cpu, "e2e": e2e,
            "e2e_resident": e2e_res, "gpu_launches": launches,
            "clocks": clk, "kernels": breakdown, "hbm_bound_ops": hbm, "decode_small_m": decode,
            "quantizer_variants": variants, "merge_requantize": merge, "compute_dtype": dtypes}
    print(json.dumps(line), flush=True)
    return 0


def run_case(args):
    """Run one op of one linear a few times (for ncu captures); prints device time per call."""
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si
    M, N, K = (int(v) for v in args.shape.split(","))
    r = args.rank
    W, X, A, B, dY = (t.cuda() for t in si.custom_linear(N, K, M, r, seed=7))
    w = q4.qlora_quantize_nf4_dq(W)
    Y, U = q4.qlora_linear_fwd(w, X, A, B, r, 2.0 * r)
    ops = {
        "quantize": lambda: q4.qlora_quantize_nf4_dq(W, out=w),
        "dequantize": lambda: q4.qlora_dequantize(w),
        "fwd": lambda: q4.qlora_linear_fwd(w, X, A, B, r, 2.0 * r, out=Y, U_out=U),
        "bwd": lambda: q4.qlora_linear_bwd(w, X, dY, A, B, r, 2.0 * r, U_saved=U),
    }
    op = ops[args.case]
    op()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.reps):
        op()
    b.record()
    b.synchronize()
    assert q4.qlora_read_device_errors(clear=True) == 0
    print(json.dumps({"case": args.case, "shape": [M, N, K], "r": r, "ms_per_call": a.elapsed_time(b) / args.reps}))
    return 0


def run_only(args):
    """One auxiliary measurement on its own (for quick A/B runs): the small-M sweep, or the
    quantize (7 block weights) and dequantize rates."""
    import torch
    import bit_nf4_quantized_23_b200 as q4
    import synthetic_inputs as si
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    q4._lib.lib()
    peaks, _ = load_peaks()
    wl = si.WORKLOADS[args.workload]
    if args.only == "decode":
        out = decode_sweep(device, peaks)
    else:
        lins, grads = setup_workload(wl, 0, device)
        for L in lins:
            q4.qlora_quantize_nf4_dq(L.W, out=L.w, workspace=L.qws)
        flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        total_ms = 0.0
        for _ in range(args.steps):
            flush_buf.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for L in lins:
                q4.qlora_quantize_nf4_dq(L.W, out=L.w, workspace=L.qws)
            b.record()
            b.synchronize()
            total_ms += a.elapsed_time(b)
        q_ms = total_ms / args.steps
        nbytes = sum((2.0 + PACKED_BYTES_PER_WEIGHT) * L.N * L.K for L in lins)
        out = {"quantize_7_weights": {"ms": round(q_ms, 4), "GB/s": round(nbytes / (q_ms * 1e-3) / 1e9, 1),
                                      "frac_of_hbm": round(nbytes / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}}
        del lins, grads
        torch.cuda.empty_cache()
        out["dequantize"] = dequant_rate(device, peaks, wl)
    print(json.dumps({"only": args.only, **out}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.case:
        return run_case(args)
    if args.only:
        return run_only(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
