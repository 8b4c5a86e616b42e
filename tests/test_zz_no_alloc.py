"""The no-allocation quantize entry point, checked against the workspace one.

qlora_quantize_nf4_dq_noalloc exists for callers that cannot allocate device
memory when they quantize (a plugin whose host framework owns all device
memory and passes only input and output pointers, or a path that must not call
cudaMalloc/cudaFree).  It keeps its scratch in a static device array of the
library.  This file is collected last so that a run stopping at the first
failure has run every other test first; it also passes alone in a fresh process
(the module fixture builds the library first).
"""
import ctypes

import pytest
import torch

import bit_nf4_quantized_23_b200 as q4
import synthetic_inputs as si
from bit_nf4_quantized_23_b200 import _lib

pytestmark = pytest.mark.gpu

# both codebooks, with and without double quantization: with it off the block constants are the
# output itself and the scratch holds only the partial sums of the mean
VARIANTS = [("nf4", True), ("uniform4", True), ("nf4", False), ("uniform4", False)]


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    from bit_nf4_quantized_23_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(torch.device("cuda:0"))
    q4.qlora_read_device_errors(clear=True)
    yield


def _noalloc(W, out):
    ws = out.c_struct()
    return _lib.lib().qlora_quantize_nf4_dq_noalloc(
        ctypes.c_void_p(W.data_ptr()), W.shape[0], W.shape[1], 64, 256, ctypes.byref(ws),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same(a: q4.NF4Weight, b: q4.NF4Weight):
    # integer and bit outputs: exact equality is the tolerance
    for name in ("codes", "c1_codes", "c2", "mu", "c1"):
        x, y = getattr(a, name), getattr(b, name)
        assert (x is None) == (y is None), name
        if x is not None:
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), name


def _poison(w: q4.NF4Weight):
    for name in ("codes", "c1_codes", "c2", "mu", "c1"):
        t = getattr(w, name)
        if t is not None:
            t.view(torch.uint8).fill_(0xAB)


@pytest.mark.parametrize("codebook,dq", VARIANTS)
def test_noalloc_matches_workspace_quantize_on_two_calls_in_a_row(codebook, dq):
    dev = torch.device("cuda:0")
    # two different tensors back to back: the second call must not see the first's scratch
    cases = [si.custom_linear(8192, 8192, 1, 1, seed=101, dist="t5")[0],
             si.custom_linear(300, 4160, 1, 1, seed=102)[0]]
    for W_cpu in cases:
        W = W_cpu.to(dev)
        N, K = W.shape
        ref = q4.qlora_quantize_nf4_dq(W, codebook=codebook, double_quant=dq)
        out = q4.NF4Weight.empty(N, K, dev, codebook=codebook, double_quant=dq)
        _poison(out)
        assert _noalloc(W, out) == 0
        torch.cuda.synchronize()
        _same(out, ref)
    assert q4.qlora_read_device_errors(clear=True) == 0


def test_noalloc_rejects_tensors_beyond_its_scratch():
    dev = torch.device("cuda:0")
    N, K = 8193, 8192                       # one row more than the 67,108,864-weight limit
    W = torch.empty(64, 64, dtype=torch.bfloat16, device=dev)     # never read: rejected first
    out = q4.NF4Weight.empty(64, 64, dev)
    ws = _lib.NF4WeightC(out.codes.data_ptr(), out.c1_codes.data_ptr(), out.c2.data_ptr(),
                         out.mu.data_ptr(), N, K, 64, 256)
    before = q4.qlora_launch_count()
    st = _lib.lib().qlora_quantize_nf4_dq_noalloc(ctypes.c_void_p(W.data_ptr()), N, K, 64, 256,
                                                  ctypes.byref(ws), None)
    assert _lib.STATUS_NAMES[st] == "QLORA_ERR_TOO_LARGE"
    assert q4.qlora_launch_count() == before
