"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerance (GEMM outputs and gradients): relative Frobenius error <= 1e-3 and
per-element |err| <= 1e-2 * max|ref|.  A bf16 output is compared with the fp64
reference rounded to bf16 (the rounding of the output alone is ~1.6e-3 relative,
so the unrounded reference cannot be met by any bf16 result), an fp16 output
with the reference rounded to fp16; fp32 outputs are compared with the
unrounded fp64 reference.
"""
import numpy as np
import torch

from oracle import nf4_oracle as o

REL_FRO = 1e-3
MAX_ABS_REL = 1e-2


def to_numpy_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def gpu_values(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = got - ref
    denom = np.linalg.norm(ref)
    rel_fro = float(np.linalg.norm(err) / denom) if denom > 0 else float(np.linalg.norm(err))
    mref = float(np.max(np.abs(ref))) if ref.size else 0.0
    max_rel = float(np.max(np.abs(err)) / mref) if mref > 0 else float(np.max(np.abs(err), initial=0.0))
    return rel_fro, max_rel


def assert_close(got_tensor: torch.Tensor, ref64: np.ndarray, name: str):
    got = gpu_values(got_tensor)
    if got_tensor.dtype == torch.bfloat16:
        ref = o.bf16_bits_to_f32(o.f32_to_bf16_bits(np.asarray(ref64).astype(np.float32))).astype(np.float64)
    elif got_tensor.dtype == torch.float16:
        ref = o.f16_bits_to_f32(o.f64_to_f16_bits(np.asarray(ref64))).astype(np.float64)
    else:
        ref = np.asarray(ref64, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    rel_fro, max_rel = errors(got, ref)
    assert rel_fro <= REL_FRO and max_rel <= MAX_ABS_REL, \
        f"{name}: rel_fro={rel_fro:.3e} max_abs/max|ref|={max_rel:.3e}"
    return rel_fro, max_rel
