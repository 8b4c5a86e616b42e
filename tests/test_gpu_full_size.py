"""GPU parity at full size, on every linear of every workload.

For each weight the CPU oracle quantizes the whole tensor, and every stored byte
the library writes (packed codes, E4M3 constant codes, c2, mu) and its whole
dequantized bf16 weight must equal the oracle's bit for bit.  The GEMM
references are then built from the oracle's own dequantized weight (never from
the library's codes): Y and dX are compared on all token rows up to 512, else on
a seeded sample of 256 rows with every output column, and dA and dB in full.

Workloads (7B- and 65B-class transformer linears): the 7B attention projection
(forward), the three 7B MLP linears (forward and backward), the decode sweep on
both shapes at M = 1, 4 and 16 (forward), and all seven linears of the 65B
decoder block (forward and backward).  The tiny workload is compared in full in
test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_23_b200 as q4
import synthetic_inputs as si
from oracle import nf4_oracle as o
from parity import assert_close, to_numpy_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_FULL_ROWS = 512
SAMPLED_ROWS = 256


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    from bit_nf4_quantized_23_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q4.qlora_read_device_errors(clear=True)
    yield
    assert q4.qlora_read_device_errors(clear=True) == 0


CASES = ([("attn7b", 0)] + [("mlp7b", i) for i in range(3)] + [("decode", i) for i in range(2)]
         + [("block65b", i) for i in range(7)])


def _token_rows(M, seed):
    if M <= MAX_FULL_ROWS:
        return np.arange(M)
    return np.sort(np.random.default_rng(seed).choice(M, SAMPLED_ROWS, replace=False))


def _exact_quantize_and_dequantize(W):
    """Quantize on the GPU and compare all four stored buffers and the whole dequantized
    weight with the oracle's; returns the library's weight and the oracle's W_hat bits."""
    N, K = W.shape
    w = q4.qlora_quantize_nf4_dq(W.to(DEV))
    torch.cuda.synchronize()
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    assert np.array_equal(w.codes.cpu().numpy(), qw["codes"]), "packed codes differ"
    assert np.array_equal(w.c1_codes.cpu().numpy(), qw["c1_codes"]), "E4M3 constant codes differ"
    assert np.array_equal(w.c2.cpu().numpy().view(np.uint32), qw["c2"].view(np.uint32)), "c2 differs"
    assert w.mu.cpu().numpy().view(np.uint32)[0] == np.float32(qw["mu"]).view(np.uint32), "mu differs"
    Wh_ref = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], N, K)
    del qw
    Wh = q4.qlora_dequantize(w)
    assert np.array_equal(to_numpy_bits(Wh), Wh_ref), "dequantized weight differs"
    del Wh
    return w, Wh_ref


@pytest.mark.parametrize("wl_name,i", CASES, ids=[f"{a}-{b}" for a, b in CASES])
def test_linear_at_full_size(wl_name, i):
    wl = si.WORKLOADS[wl_name]
    N, K = wl.linears[i]
    w, Wh_ref = _exact_quantize_and_dequantize(si.weight(wl, i))
    Whf = o._f64(Wh_ref)                                   # the oracle's W_hat, fp64 [N, K]
    del Wh_ref
    A, B = si.lora(wl, i)
    Ad, Bd = A.to(DEV), B.to(DEV)
    bA, bB = si.bf16_bits(A), si.bf16_bits(B)
    for M in (wl.M if isinstance(wl.M, tuple) else (wl.M,)):
        X = si.activations(wl, K, M)
        Xd = X.to(DEV)
        Y, U = q4.qlora_linear_fwd(w, Xd, Ad, Bd, wl.r, wl.alpha)
        torch.cuda.synchronize()
        bX = si.bf16_bits(X)
        rows = _token_rows(M, seed=N + K + i)
        rt = torch.as_tensor(rows, device=DEV)
        Yref, Uref = o.linear_forward(bX[rows], Whf, bA, bB, wl.alpha, wl.r)
        assert_close(Y[rt].contiguous(), Yref, f"Y M={M}")
        assert_close(U[rt].contiguous(), Uref, f"U M={M}")
        if "bwd" not in wl.ops:
            continue
        dY = si.grad_output(wl, i, M)
        dX, dA, dB = q4.qlora_linear_bwd(w, Xd, dY.to(DEV), Ad, Bd, wl.r, wl.alpha, U_saved=U)
        torch.cuda.synchronize()
        bdY = si.bf16_bits(dY)
        dXref = o.backward_dx_rows(bdY, Whf, bA, bB, wl.alpha, wl.r, rows)
        assert_close(dX[rt].contiguous(), dXref, f"dX M={M}")
        g = o.lora_gradients(bX, bdY, bA, bB, wl.alpha, wl.r)
        assert_close(dA, g["dA"], "dA full")
        assert_close(dB, g["dB"], "dB full")
    del w
    torch.cuda.empty_cache()
