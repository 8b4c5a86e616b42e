"""Seeded synthetic inputs for the QLoRA quantized linear layer.

This module only draws random tensors. It holds none of the method's arithmetic
(no quantization, no dequantization, no matmul), so both the CPU oracle and the
CUDA library can be fed from it without sharing code.

Recipe (every tensor is drawn in fp32 from a NumPy PCG64 stream, then rounded to
bf16 with torch's own cast, so both sides see identical bf16 bits):

* Each tensor has its own stream, keyed by (seed, workload name, tensor tag).
  A tensor therefore does not depend on which other tensors were drawn first.
* Weights W[N,K]: N(0, sigma^2) (sigma 0.02; 0.015 for the decode sweep), or for
  the 65B-shaped block a Student-t with 5 degrees of freedom scaled to std 0.02
  in which exactly round(0.001*N*K) distinct entries (chosen by the same
  stream) are multiplied by 10.
* Activations X[M,K] and upstream gradients dY[M,N]: N(0, 1).  Linears of one
  workload that share K share the same X (gate and up projections).
* LoRA A[r,K]: N(0, 1/K).  LoRA B[N,r]: N(0, 0.01^2) (nonzero so that the LoRA
  path is exercised; a freshly initialised adapter would have B = 0).

The shapes are those of 7B- and 65B-class transformer linears (LLaMA-style), the
workloads the QLoRA pages discuss; no checkpoint or dataset is used.
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    linears: tuple          # tuple of (N, K)
    M: int | tuple          # tokens (a tuple for the decode sweep)
    r: int
    alpha: float
    sigma: float = 0.02
    dist: str = "normal"    # "normal" or "t5_outliers"
    ops: tuple = field(default=("quantize", "fwd", "bwd"))
    description: str = ""


WORKLOADS = {
    "tiny": Workload(
        "tiny", ((256, 256),), 16, 8, 16.0,
        ops=("quantize", "dequantize", "fwd", "bwd"),
        description="tiny QLoRA linear W[256,256], X[16,256], r=8 alpha=16"),
    "attn7b": Workload(
        "attn7b", ((4096, 4096),), 512, 16, 32.0,
        ops=("quantize", "fwd"),
        description="7B attention projection W[4096,4096], X[512,4096], r=16 alpha=32"),
    "mlp7b": Workload(
        "mlp7b", ((11008, 4096), (11008, 4096), (4096, 11008)), 4096, 64, 16.0,
        ops=("fwd", "bwd"),
        description="7B MLP gate/up W[11008,4096], down W[4096,11008], X[4096,*], r=64 alpha=16"),
    "decode": Workload(
        "decode", ((8192, 8192), (28672, 8192)), (1, 4, 16), 16, 32.0, sigma=0.015,
        ops=("quantize", "fwd"),
        description="decode sweep W[8192,8192] and W[28672,8192], M in {1,4,16}, r=16 alpha=32"),
    "block65b": Workload(
        "block65b",
        ((8192, 8192),) * 4 + ((22016, 8192),) * 2 + ((8192, 22016),),
        2048, 64, 16.0, dist="t5_outliers",
        ops=("quantize", "fwd", "bwd"),
        description="65B decoder block: q/k/v/o W[8192,8192], gate/up W[22016,8192], "
                    "down W[8192,22016], Student-t(5) weights with 0.1% x10 outliers, "
                    "X[2048,*], r=64 alpha=16"),
}


def _rng(seed: int, workload: str, tag: str) -> np.random.Generator:
    key = [int(seed), zlib.crc32(workload.encode()), zlib.crc32(tag.encode())]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal_bf16(shape, std: float, seed: int, workload: str, tag: str) -> torch.Tensor:
    """N(0, std^2) drawn in fp32, rounded to bf16 (CPU tensor)."""
    g = _rng(seed, workload, tag)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return _to_bf16(a)


def t5_outlier_bf16(shape, std: float, seed: int, workload: str, tag: str,
                    outlier_frac: float = 0.001, outlier_mult: float = 10.0) -> torch.Tensor:
    """Student-t(5) scaled to the given std, with exactly round(frac*numel) distinct x10 entries."""
    g = _rng(seed, workload, tag)
    n = int(np.prod(shape))
    z = g.standard_normal(size=n, dtype=np.float32)
    chi2 = g.standard_gamma(2.5, size=n, dtype=np.float32) * np.float32(2.0)   # chi^2 with 5 dof
    t = z / np.sqrt(chi2 / np.float32(5.0))
    t *= np.float32(std / np.sqrt(5.0 / 3.0))
    n_out = int(round(outlier_frac * n))
    if n_out:
        idx = g.choice(n, size=n_out, replace=False)
        t[idx] *= np.float32(outlier_mult)
    return _to_bf16(t.reshape(shape))


def weight(workload: Workload | str, i: int, seed: int = 0) -> torch.Tensor:
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    N, K = w.linears[i]
    if w.dist == "normal":
        return normal_bf16((N, K), w.sigma, seed, w.name, f"W{i}")
    return t5_outlier_bf16((N, K), w.sigma, seed, w.name, f"W{i}")


def activations(workload: Workload | str, K: int, M: int, seed: int = 0) -> torch.Tensor:
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    return normal_bf16((M, K), 1.0, seed, w.name, f"X{K}_{M}")


def grad_output(workload: Workload | str, i: int, M: int, seed: int = 0) -> torch.Tensor:
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    N, _ = w.linears[i]
    return normal_bf16((M, N), 1.0, seed, w.name, f"dY{i}_{M}")


def lora(workload: Workload | str, i: int, seed: int = 0):
    """(A[r,K] ~ N(0,1/K), B[N,r] ~ N(0, 0.01^2)) as bf16 CPU tensors."""
    w = WORKLOADS[workload] if isinstance(workload, str) else workload
    N, K = w.linears[i]
    A = normal_bf16((w.r, K), float(1.0 / np.sqrt(K)), seed, w.name, f"A{i}")
    B = normal_bf16((N, w.r), 0.01, seed, w.name, f"B{i}")
    return A, B


def custom_linear(N: int, K: int, M: int, r: int, seed: int, tag: str = "custom",
                  sigma: float = 0.02, dist: str = "normal"):
    """W, X, A, B, dY for an arbitrary shape (ragged and edge-case tests)."""
    if dist == "normal":
        W = normal_bf16((N, K), sigma, seed, tag, "W")
    else:
        W = t5_outlier_bf16((N, K), sigma, seed, tag, "W")
    X = normal_bf16((M, K), 1.0, seed, tag, "X")
    A = normal_bf16((r, K), float(1.0 / np.sqrt(K)), seed, tag, "A")
    B = normal_bf16((N, r), 0.01, seed, tag, "B")
    dY = normal_bf16((M, N), 1.0, seed, tag, "dY")
    return W, X, A, B, dY


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 CPU tensor (a view, no arithmetic)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
