"""ctypes loader for libqlora.so and the C signatures of include/qlora.h.

The library is built in-tree (bit_nf4_quantized_23_b200/libqlora.so).  There is
no fallback: if the library is missing, importing a compute entry point raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_int64, c_size_t, c_uint32, c_uint64, c_void_p

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libqlora.so")

QLORA_OK = 0
STATUS_NAMES = {
    0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGN",
    4: "QLORA_ERR_UNSUPPORTED", 5: "QLORA_ERR_NONFINITE", 6: "QLORA_ERR_TIMEOUT",
    7: "QLORA_ERR_CUDA", 8: "QLORA_ERR_WORKSPACE", 9: "QLORA_ERR_TOO_LARGE",
}
QLORA_DTYPE_BF16 = 0
QLORA_DTYPE_F32 = 1
QLORA_DTYPE_F16 = 2

# Every symbol include/qlora.h declares, with (restype, argtypes).
_W = None  # placeholder, replaced by POINTER(NF4WeightC) below


class NF4WeightC(ctypes.Structure):
    """Mirror of qlora_nf4_weight."""
    _fields_ = [("codes", c_void_p), ("c1_codes", c_void_p), ("c2", c_void_p), ("mu", c_void_p),
                ("N", c_int64), ("K", c_int64), ("blocksize", c_int32), ("blocksize2", c_int32),
                ("codebook", c_int32), ("compute_dtype", c_int32), ("c1", c_void_p)]


_W = POINTER(NF4WeightC)

SIGNATURES = {
    "qlora_status_string": (c_char_p, [c_int32]),
    "qlora_nf4_sizes": (c_int32, [c_int64, c_int64, c_int32, c_int32, POINTER(c_size_t), POINTER(c_size_t),
                                  POINTER(c_size_t), POINTER(c_size_t)]),
    "qlora_nf4_codebook": (c_int32, [POINTER(c_float), POINTER(c_float)]),
    "qlora_codebook_values": (c_int32, [c_int32, POINTER(c_float), POINTER(c_float)]),
    "qlora_quantize_nf4_dq": (c_int32, [c_void_p, c_int64, c_int64, c_int32, c_int32, _W, c_void_p,
                                        c_size_t, c_void_p]),
    "qlora_quantize_nf4_dq_noalloc": (c_int32, [c_void_p, c_int64, c_int64, c_int32, c_int32, _W, c_void_p]),
    "qlora_merge_lora": (c_int32, [_W, c_void_p, c_void_p, c_int32, c_float, c_void_p, c_void_p]),
    "qlora_linear_fwd_multi": (c_int32, [_W, c_void_p, c_int64, c_void_p, c_void_p, c_int32, c_void_p, c_int32,
                                         c_float, c_void_p, c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_dequantize": (c_int32, [_W, c_void_p, c_void_p]),
    "qlora_quantize_int8_absmax": (c_int32, [c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_void_p]),
    "qlora_dequantize_int8_absmax": (c_int32, [c_void_p, c_void_p, c_int64, c_int32, c_void_p, c_int32, c_void_p]),
    "qlora_linear_workspace_size": (c_int32, [c_int64, c_int64, c_int64, c_int32, POINTER(c_size_t)]),
    "qlora_linear_fwd": (c_int32, [_W, c_void_p, c_int64, c_void_p, c_void_p, c_int32, c_float, c_void_p,
                                   c_int32, c_void_p, c_void_p, c_size_t, c_void_p]),
    "qlora_linear_bwd": (c_int32, [_W, c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_int32, c_float,
                                   c_void_p, c_void_p, c_int32, c_void_p, c_void_p, c_void_p, c_size_t,
                                   c_void_p]),
    "qlora_read_device_errors": (c_int32, [c_void_p, c_int32, POINTER(c_uint32)]),
    "qlora_selftest_bounded_wait": (c_int32, [c_uint32, c_void_p, c_void_p]),
    "qlora_launch_count": (c_uint64, []),
    "qlora_timing_enable": (c_int32, [c_int32]),
    "qlora_timing_read": (c_int32, [c_int32, POINTER(c_uint64), POINTER(ctypes.c_double), c_int32]),
}

TIMER_KINDS = {"quantize": 0, "dequantize": 1, "fwd_main": 2, "dx_main": 3, "lora": 4, "decode": 5}

_lib = None


class QloraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def lib() -> ctypes.CDLL:
    """The loaded libqlora.so with argument types set.  Raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m bit_nf4_quantized_23_b200.build` (no CPU fallback exists)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def check(status: int, where: str) -> None:
    if status != QLORA_OK:
        raise QloraError(status, where)
