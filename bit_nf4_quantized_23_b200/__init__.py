"""B200 (sm_100a) QLoRA quantized linear layer: NF4 + Double Quantization, dequantization,
and the LoRA-augmented forward/backward through the frozen dequantized weight.

The Python functions below carry the names of the C entry points of libqlora.so
(include/qlora.h).  They only marshal arguments: they allocate outputs with
torch (device memory), pass raw pointers and the current CUDA stream, and check
the returned status.  Every step of the computation runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes
from ctypes import byref, c_float, c_size_t, c_uint32
from dataclasses import dataclass

import torch

from ._lib import (QLORA_DTYPE_BF16, QLORA_DTYPE_F16, QLORA_DTYPE_F32, TIMER_KINDS, NF4WeightC, QloraError,
                   check, lib)

__all__ = [
    "NF4Weight", "QloraError", "CODEBOOKS", "qlora_nf4_sizes", "qlora_nf4_codebook", "qlora_codebook_values",
    "qlora_quantize_nf4_dq",
    "qlora_quantize_nf4_dq_noalloc",
    "qlora_dequantize", "qlora_quantize_int8_absmax", "qlora_dequantize_int8_absmax", "qlora_merge_lora", "qlora_linear_workspace_size", "qlora_linear_fwd", "qlora_linear_fwd_multi", "qlora_linear_bwd",
    "qlora_read_device_errors", "qlora_selftest_bounded_wait", "qlora_launch_count", "qlora_timing_enable", "qlora_timing_read",
]


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, dtype, name: str, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _dtype_code(dtype) -> int:
    if dtype == torch.bfloat16:
        return QLORA_DTYPE_BF16
    if dtype == torch.float16:
        return QLORA_DTYPE_F16
    if dtype == torch.float32:
        return QLORA_DTYPE_F32
    raise TypeError("output dtype must be torch.bfloat16, torch.float16 or torch.float32")


@dataclass
class NF4Weight:
    """The stored buffers of a 4-bit quantized weight (device tensors) and its shape.

    With double quantization (the default) the block constants are c1_codes, c2 and mu and
    `c1` is None; without it `c1` holds the fp32 block absmax values and the other three are
    None.  `codebook` is "nf4" or "uniform4" (the uniform 4-bit grid NF4 is compared with)."""
    codes: torch.Tensor                 # uint8 [N*K/2]
    c1_codes: torch.Tensor | None       # uint8 [N*K/64]  (FP8 E4M3 bit patterns)
    c2: torch.Tensor | None             # fp32 [ceil(N*K/64/256)]
    mu: torch.Tensor | None             # fp32 [1]
    N: int
    K: int
    codebook: str = "nf4"
    c1: torch.Tensor | None = None      # fp32 [N*K/64] when double quantization is off
    compute_dtype: torch.dtype = torch.bfloat16   # or torch.float16: W_hat, activations, adapters

    def c_struct(self) -> NF4WeightC:
        p = lambda t: t.data_ptr() if t is not None else None
        return NF4WeightC(self.codes.data_ptr(), p(self.c1_codes), p(self.c2), p(self.mu), self.N, self.K,
                          64, 256, CODEBOOKS[self.codebook], _dtype_code(self.compute_dtype), p(self.c1))

    _BUFFERS = ("codes", "c1_codes", "c2", "mu", "c1")

    def state_dict(self) -> dict:
        """Host copies of the stored buffers plus the shape and settings that give them meaning:
        a checkpoint of the frozen quantized weight (torch.save can write it as is)."""
        d = {"N": self.N, "K": self.K, "codebook": self.codebook, "blocksize": 64, "blocksize2": 256,
             "compute_dtype": str(self.compute_dtype).replace("torch.", "")}
        for name in self._BUFFERS:
            t = getattr(self, name)
            d[name] = None if t is None else t.detach().to("cpu", copy=True)
        return d

    @classmethod
    def from_state_dict(cls, d: dict, device="cuda") -> "NF4Weight":
        """Rebuild a weight from state_dict() output: the buffers are copied to `device` byte for byte
        after their sizes are checked against the shape."""
        N, K = int(d["N"]), int(d["K"])
        if d.get("blocksize", 64) != 64 or d.get("blocksize2", 256) != 256:
            raise ValueError("only blocksize 64 and blocksize2 256 are defined")
        dtype = {"bfloat16": torch.bfloat16, "float16": torch.float16}[d["compute_dtype"]]
        ref = cls.empty(N, K, device, d["codebook"], d.get("c1") is None, dtype)
        for name in cls._BUFFERS:
            t, src = getattr(ref, name), d.get(name)
            if (t is None) != (src is None):
                raise ValueError(f"buffer {name!r} does not match the stored settings")
            if t is not None:
                if src.dtype != t.dtype or src.numel() != t.numel():
                    raise ValueError(f"buffer {name!r}: expected {t.numel()} x {t.dtype}, got "
                                     f"{src.numel()} x {src.dtype}")
                t.copy_(src.reshape(t.shape))
        return ref

    @staticmethod
    def empty(N: int, K: int, device="cuda", codebook: str = "nf4", double_quant: bool = True,
              compute_dtype: torch.dtype = torch.bfloat16) -> "NF4Weight":
        if codebook not in CODEBOOKS:
            raise ValueError(f"codebook must be one of {sorted(CODEBOOKS)}")
        if compute_dtype not in (torch.bfloat16, torch.float16):
            raise ValueError("compute_dtype must be torch.bfloat16 or torch.float16")
        s = qlora_nf4_sizes(N, K)
        codes = torch.empty(s["codes"], dtype=torch.uint8, device=device)
        if not double_quant:
            return NF4Weight(codes, None, None, None, N, K, codebook,
                             torch.empty(s["c1_codes"], dtype=torch.float32, device=device), compute_dtype)
        return NF4Weight(codes,
                         torch.empty(s["c1_codes"], dtype=torch.uint8, device=device),
                         torch.empty(s["c2"] // 4, dtype=torch.float32, device=device),
                         torch.empty(1, dtype=torch.float32, device=device), N, K, codebook, None, compute_dtype)


CODEBOOKS = {"nf4": 0, "uniform4": 1}


def qlora_nf4_sizes(N: int, K: int, blocksize: int = 64, blocksize2: int = 256) -> dict:
    a, b, c, d = c_size_t(), c_size_t(), c_size_t(), c_size_t()
    check(lib().qlora_nf4_sizes(N, K, blocksize, blocksize2, byref(a), byref(b), byref(c), byref(d)),
          "qlora_nf4_sizes")
    return {"codes": a.value, "c1_codes": b.value, "c2": c.value, "workspace": d.value}


def qlora_nf4_codebook():
    """(values[16], thresholds[15]) of the library, as Python float lists."""
    v = (c_float * 16)()
    t = (c_float * 15)()
    check(lib().qlora_nf4_codebook(v, t), "qlora_nf4_codebook")
    return list(v), list(t)


def qlora_codebook_values(codebook: str = "nf4"):
    """(values[16], thresholds[15]) of a codebook ("nf4" or "uniform4")."""
    v = (c_float * 16)()
    t = (c_float * 15)()
    check(lib().qlora_codebook_values(CODEBOOKS[codebook], v, t), "qlora_codebook_values")
    return list(v), list(t)


def qlora_quantize_nf4_dq(W: torch.Tensor, blocksize: int = 64, blocksize2: int = 256,
                          out: NF4Weight | None = None, workspace: torch.Tensor | None = None,
                          stream=None, codebook: str = "nf4", double_quant: bool = True,
                          compute_dtype: torch.dtype = torch.bfloat16) -> NF4Weight:
    """Quantize W (bf16 [N, K]); `codebook`, `double_quant` and `compute_dtype` apply when `out`
    is None (otherwise `out` carries them)."""
    _need(W, torch.bfloat16, "W")
    if W.dim() != 2:
        raise ValueError("W must be 2-D [N, K]")
    N, K = W.shape
    sizes = qlora_nf4_sizes(N, K, blocksize, blocksize2)
    if out is None:
        out = NF4Weight.empty(N, K, W.device, codebook, double_quant, compute_dtype)
    if workspace is None:
        workspace = torch.empty(sizes["workspace"], dtype=torch.uint8, device=W.device)
    ws = out.c_struct()
    check(lib().qlora_quantize_nf4_dq(_ptr(W), N, K, blocksize, blocksize2, byref(ws), _ptr(workspace),
                                      workspace.numel(), _stream(stream)), "qlora_quantize_nf4_dq")
    return out


def qlora_quantize_nf4_dq_noalloc(W: torch.Tensor, out: NF4Weight, stream=None) -> NF4Weight:
    """Quantize into caller-allocated `out` using the library's static device scratch (no
    workspace, no allocation in the call).  At most 67,108,864 weights; calls that overlap on
    the GPU race on the shared scratch."""
    _need(W, torch.bfloat16, "W")
    N, K = W.shape
    ws = out.c_struct()
    check(lib().qlora_quantize_nf4_dq_noalloc(_ptr(W), N, K, 64, 256, byref(ws), _stream(stream)),
          "qlora_quantize_nf4_dq_noalloc")
    return out


def qlora_dequantize(w: NF4Weight, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(w.N, w.K, dtype=w.compute_dtype, device=w.codes.device)
    _need(out, w.compute_dtype, "out", (w.N, w.K))
    ws = w.c_struct()
    check(lib().qlora_dequantize(byref(ws), _ptr(out), _stream(stream)), "qlora_dequantize")
    return out


def qlora_quantize_int8_absmax(W: torch.Tensor, blocksize: int = 64, codes: torch.Tensor | None = None,
                               alpha: torch.Tensor | None = None, stream=None):
    """Blockwise absmax INT8 of a bf16 tensor: alpha = 127 / max|x| per block of
    `blocksize` consecutive elements, codes = round half away from zero of x * alpha.
    Returns (codes int8 shaped like W, alpha fp32 [W.numel() // blocksize])."""
    _need(W, torch.bfloat16, "W")
    n = W.numel()
    if codes is None:
        codes = torch.empty(W.shape, dtype=torch.int8, device=W.device)
    if alpha is None:
        alpha = torch.empty(max(n // blocksize, 1), dtype=torch.float32, device=W.device)
    _need(codes, torch.int8, "codes", tuple(W.shape))
    _need(alpha, torch.float32, "alpha")
    if blocksize <= 0 or alpha.numel() * blocksize != n:
        raise ValueError(f"alpha must hold {n // blocksize} scales")
    check(lib().qlora_quantize_int8_absmax(_ptr(W), n, blocksize, _ptr(codes), _ptr(alpha), _stream(stream)),
          "qlora_quantize_int8_absmax")
    return codes, alpha


def qlora_dequantize_int8_absmax(codes: torch.Tensor, alpha: torch.Tensor, blocksize: int = 64,
                                 dtype=torch.bfloat16, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """x_hat = code / alpha per block, rounded to `dtype` (bf16, fp16 or fp32)."""
    _need(codes, torch.int8, "codes")
    _need(alpha, torch.float32, "alpha")
    if blocksize <= 0 or alpha.numel() * blocksize != codes.numel():
        raise ValueError(f"alpha must hold codes.numel() / blocksize = {codes.numel() // max(blocksize, 1)} scales")
    if out is None:
        out = torch.empty(codes.shape, dtype=dtype, device=codes.device)
    _need(out, dtype, "out", tuple(codes.shape))
    check(lib().qlora_dequantize_int8_absmax(_ptr(codes), _ptr(alpha), codes.numel(), blocksize, _ptr(out),
                                             _dtype_code(dtype), _stream(stream)), "qlora_dequantize_int8_absmax")
    return out


def qlora_merge_lora(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, r: int, alpha: float,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W_merged = bf16(W_hat + (alpha / r) B A) for inference; requantize it with
    qlora_quantize_nf4_dq to serve the merged model in 4 bits."""
    _need(A, w.compute_dtype, "A", (r, w.K))
    _need(B, w.compute_dtype, "B", (w.N, r))
    if out is None:
        out = torch.empty(w.N, w.K, dtype=w.compute_dtype, device=w.codes.device)
    _need(out, w.compute_dtype, "out", (w.N, w.K))
    ws = w.c_struct()
    check(lib().qlora_merge_lora(byref(ws), _ptr(A), _ptr(B), r, float(alpha), _ptr(out), _stream(stream)),
          "qlora_merge_lora")
    return out


def qlora_linear_workspace_size(M: int, N: int, K: int, r: int) -> int:
    n = c_size_t()
    check(lib().qlora_linear_workspace_size(M, N, K, r, byref(n)), "qlora_linear_workspace_size")
    return n.value


def _workspace(M, N, K, r, device, workspace):
    need = qlora_linear_workspace_size(M, N, K, r)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=device)
    return workspace


def qlora_linear_fwd(w: NF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, r: int,
                     alpha: float, y_dtype=None, save_U: bool = True,
                     out: torch.Tensor | None = None, U_out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None):
    """Y = X W_hat^T + (alpha/r) (X A^T) B^T.  Returns (Y, U) with U fp32 [M,r] (or None).
    X, A, B are in the weight's compute dtype; Y is in it too unless y_dtype is torch.float32."""
    M = X.shape[0]
    y_dtype = w.compute_dtype if y_dtype is None else y_dtype
    _need(X, w.compute_dtype, "X", (M, w.K))
    _need(A, w.compute_dtype, "A", (r, w.K))
    _need(B, w.compute_dtype, "B", (w.N, r))
    if out is None:
        out = torch.empty(M, w.N, dtype=y_dtype, device=X.device)
    _need(out, y_dtype, "Y", (M, w.N))
    if save_U and U_out is None:
        U_out = torch.empty(M, r, dtype=torch.float32, device=X.device)
    if U_out is not None:
        _need(U_out, torch.float32, "U", (M, r))
    workspace = _workspace(M, w.N, w.K, r, X.device, workspace)
    ws = w.c_struct()
    check(lib().qlora_linear_fwd(byref(ws), _ptr(X), M, _ptr(A), _ptr(B), r, c_float(alpha), _ptr(out),
                                 _dtype_code(y_dtype), _ptr(U_out), _ptr(workspace), workspace.numel(),
                                 _stream(stream)), "qlora_linear_fwd")
    return out, U_out


def qlora_linear_fwd_multi(w: NF4Weight, X: torch.Tensor, A_all: torch.Tensor, B_all: torch.Tensor,
                           adapter_idx: torch.Tensor, r: int, alpha: float, y_dtype=None,
                           save_U: bool = False, out: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None, stream=None):
    """One base, many adapters (M <= 16 tokens): Y[m] = X[m] W_hat^T + (alpha/r) (X[m] A_a^T) B_a^T
    with a = adapter_idx[m] (-1: base only).  A_all [n, r, K], B_all [n, N, r] bf16; adapter_idx
    int32 [M] on the device.  Returns (Y, U or None)."""
    M = X.shape[0]
    n_ad = A_all.shape[0]
    y_dtype = w.compute_dtype if y_dtype is None else y_dtype
    _need(X, w.compute_dtype, "X", (M, w.K))
    _need(A_all, w.compute_dtype, "A_all", (n_ad, r, w.K))
    _need(B_all, w.compute_dtype, "B_all", (n_ad, w.N, r))
    _need(adapter_idx, torch.int32, "adapter_idx", (M,))
    if out is None:
        out = torch.empty(M, w.N, dtype=y_dtype, device=X.device)
    _need(out, y_dtype, "Y", (M, w.N))
    U = torch.empty(M, r, dtype=torch.float32, device=X.device) if save_U else None
    workspace = _workspace(M, w.N, w.K, r, X.device, workspace)
    ws = w.c_struct()
    check(lib().qlora_linear_fwd_multi(byref(ws), _ptr(X), M, _ptr(A_all), _ptr(B_all), n_ad, _ptr(adapter_idx),
                                       r, c_float(alpha), _ptr(out), _dtype_code(y_dtype), _ptr(U),
                                       _ptr(workspace), workspace.numel(), _stream(stream)),
          "qlora_linear_fwd_multi")
    return out, U


def qlora_linear_bwd(w: NF4Weight, X: torch.Tensor, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                     r: int, alpha: float, U_saved: torch.Tensor | None = None, need_dX: bool = True,
                     dx_dtype=None, dX: torch.Tensor | None = None,
                     dA: torch.Tensor | None = None, dB: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None):
    """(dX, dA, dB) of <dY, Y> through the frozen W_hat.  dX is None when need_dX is False."""
    M = X.shape[0]
    dx_dtype = w.compute_dtype if dx_dtype is None else dx_dtype
    _need(X, w.compute_dtype, "X", (M, w.K))
    _need(dY, w.compute_dtype, "dY", (M, w.N))
    _need(A, w.compute_dtype, "A", (r, w.K))
    _need(B, w.compute_dtype, "B", (w.N, r))
    if U_saved is not None:
        _need(U_saved, torch.float32, "U_saved", (M, r))
    if need_dX and dX is None:
        dX = torch.empty(M, w.K, dtype=dx_dtype, device=X.device)
    if dX is not None:
        _need(dX, dx_dtype, "dX", (M, w.K))
    if dA is None:
        dA = torch.empty(r, w.K, dtype=torch.float32, device=X.device)
    if dB is None:
        dB = torch.empty(w.N, r, dtype=torch.float32, device=X.device)
    _need(dA, torch.float32, "dA", (r, w.K))
    _need(dB, torch.float32, "dB", (w.N, r))
    workspace = _workspace(M, w.N, w.K, r, X.device, workspace)
    ws = w.c_struct()
    check(lib().qlora_linear_bwd(byref(ws), _ptr(X), _ptr(dY), M, _ptr(A), _ptr(B), r, c_float(alpha),
                                 _ptr(U_saved), _ptr(dX), _dtype_code(dx_dtype), _ptr(dA), _ptr(dB),
                                 _ptr(workspace), workspace.numel(), _stream(stream)), "qlora_linear_bwd")
    return dX, dA, dB


def qlora_read_device_errors(clear: bool = True, stream=None) -> int:
    """Synchronize and return the device error flags (1: timeout, 2: non-finite weight)."""
    f = c_uint32()
    lib().qlora_read_device_errors(_stream(stream), 1 if clear else 0, byref(f))
    return f.value


def qlora_selftest_bounded_wait(limit_us: int, device=None, stream=None):
    """Run the bounded-wait self-test (a wait that nothing completes, limited to `limit_us`);
    returns (completed, aborted) as read back from the device.  The timeout device flag is
    left set for qlora_read_device_errors."""
    result = torch.zeros(2, dtype=torch.int32, device=device or torch.device("cuda"))
    check(lib().qlora_selftest_bounded_wait(int(limit_us), _ptr(result), _stream(stream)),
          "qlora_selftest_bounded_wait")
    r = result.cpu().tolist()
    return bool(r[0]), bool(r[1])


def qlora_launch_count() -> int:
    return int(lib().qlora_launch_count())


def qlora_timing_enable(on: bool = True) -> None:
    check(lib().qlora_timing_enable(1 if on else 0), "qlora_timing_enable")


def qlora_timing_read(kind: str, reset: bool = False):
    """(timed units, total device ms) recorded for one kind since the last reset."""
    n = ctypes.c_uint64()
    ms = ctypes.c_double()
    check(lib().qlora_timing_read(TIMER_KINDS[kind], byref(n), byref(ms), 1 if reset else 0),
          "qlora_timing_read")
    return int(n.value), float(ms.value)
