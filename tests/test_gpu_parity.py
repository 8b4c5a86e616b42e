"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Bit-exact: packed NF4 codes, E4M3 constant codes, c2, mu and the dequantized
bf16 weight.  Within tolerance (tests/parity.py): Y, dX, dA, dB.  Shapes here
are small, ragged and edge cases, compared element by element in full; the
full-size workloads are in test_gpu_full_size.py.
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


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    from bit_nf4_quantized_23_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q4.qlora_read_device_errors(clear=True)
    yield
    assert q4.qlora_read_device_errors(clear=True) == 0


def quantize_on_gpu(W_cpu):
    w = q4.qlora_quantize_nf4_dq(W_cpu.to(DEV))
    torch.cuda.synchronize()
    return w


def check_quantize_exact(W_cpu, w_gpu, qw=None):
    bits = si.bf16_bits(W_cpu)
    qw = o.quantize_nf4_dq(bits) if qw is None else qw
    assert np.array_equal(w_gpu.codes.cpu().numpy(), qw["codes"])
    assert np.array_equal(w_gpu.c1_codes.cpu().numpy(), qw["c1_codes"])
    assert np.array_equal(w_gpu.c2.cpu().numpy().view(np.uint32), qw["c2"].view(np.uint32))
    assert w_gpu.mu.cpu().numpy().view(np.uint32)[0] == np.float32(qw["mu"]).view(np.uint32)
    return qw


def check_dequantize_exact(w_gpu, qw):
    Wh = q4.qlora_dequantize(w_gpu)
    ref = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], qw["N"], qw["K"])
    assert np.array_equal(to_numpy_bits(Wh), ref)
    return ref


# ------------------------------------------------------------------ quantize / dequantize

SHAPES = [(256, 256), (1, 64), (3, 320), (5, 4160), (17, 1024), (64, 192), (2, 16384)]


@pytest.mark.parametrize("N,K", SHAPES)
def test_quantize_and_dequantize_bit_exact(N, K):
    W = si.custom_linear(N, K, 1, 1, seed=N * 131 + K)[0]
    w = quantize_on_gpu(W)
    qw = check_quantize_exact(W, w)
    check_dequantize_exact(w, qw)


def test_quantize_heavy_tailed_weights_bit_exact():
    W = si.custom_linear(96, 8192, 1, 1, seed=3, dist="t5")[0]
    w = quantize_on_gpu(W)
    check_dequantize_exact(w, check_quantize_exact(W, w))


def _boundary_weight(seed=0):
    """Blocks whose values straddle every decision threshold of every scale.

    Each block holds its absmax c (so c1 = c) and bf16 values next to t_j * c
    for the 15 midpoints t_j of neighbouring codes, with both signs."""
    g = np.random.default_rng(seed)
    q = o.nf4_codebook().astype(np.float64)
    mids = (q[:-1] + q[1:]) / 2
    rows = []
    for _ in range(1024):
        c = np.float32(2.0 ** g.uniform(-20, 20))
        c_bits = o.f32_to_bf16_bits(np.array([c], np.float32))
        c = o.bf16_bits_to_f32(c_bits)[0]
        centre = o.f32_to_bf16_bits((mids * c).astype(np.float32)).astype(np.int64)
        cand = np.concatenate([centre + d for d in (-2, -1, 0, 1, 2)])
        cand = cand[(cand & 0x7F80) != 0x7F80].astype(np.uint16)     # finite only
        pick = g.choice(cand, 63, replace=True)
        block = np.concatenate([c_bits, pick]).astype(np.uint16)
        g.shuffle(block)
        rows.append(block)
    return np.concatenate(rows).reshape(-1, 1024)


def test_quantize_decision_boundaries_bit_exact():
    bits = _boundary_weight()
    W = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    w = quantize_on_gpu(W)
    check_dequantize_exact(w, check_quantize_exact(W, w))


def test_quantize_every_scale_at_every_decision_boundary():
    """Every positive finite bf16 block absmax c (subnormals included), each with
    the bf16 values within +-2 ulps of t_j * c for all 15 decision thresholds."""
    g = np.random.default_rng(11)
    q = o.nf4_codebook().astype(np.float64)
    mids = (q[:-1] + q[1:]) / 2
    scales = np.arange(1, 0x7F80, dtype=np.uint32).astype(np.uint16)         # all positive finite bf16
    c = o.bf16_bits_to_f32(scales).astype(np.float64)
    centre = o.f32_to_bf16_bits((c[:, None] * mids[None, :]).astype(np.float32)).astype(np.int64)
    cand = np.concatenate([centre + d for d in (-2, -1, 0, 1, 2)], axis=1)   # [n_scales, 75]
    cand = np.where((cand & 0x7F80) == 0x7F80, 0, cand)                        # keep finite patterns
    mag = o.bf16_bits_to_f32(cand.astype(np.uint16)).astype(np.float64)
    cand = np.where(np.abs(mag) <= c[:, None], cand, 0).astype(np.uint16)     # |value| <= absmax
    filler = g.integers(0, 0x7F80, size=(scales.size, 126 - 75)).astype(np.uint16)
    fmag = o.bf16_bits_to_f32(filler).astype(np.float64)
    filler = np.where(fmag <= c[:, None], filler, 0).astype(np.uint16)
    body = np.concatenate([cand, filler], axis=1)
    blocks = np.concatenate([scales[:, None], body[:, :63], scales[:, None], body[:, 63:]], axis=1)
    bits = np.ascontiguousarray(blocks.reshape(-1, 128))               # one row = the two blocks of a scale
    W = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    w = quantize_on_gpu(W)
    check_dequantize_exact(w, check_quantize_exact(W, w))


def test_quantize_every_finite_bf16_value():
    g = np.random.default_rng(1)
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    allb = allb[(allb & 0x7F80) != 0x7F80]                      # drop Inf/NaN
    allb = np.concatenate([allb, np.zeros((-allb.size) % 1024, np.uint16)])
    # sort by magnitude within shuffled neighbourhoods so that blocks hold values of similar scale
    mag = o.bf16_bits_to_f32(allb)
    order = np.argsort(np.abs(mag) * np.exp(g.normal(0, 0.5, allb.size)))
    W = torch.from_numpy(allb[order].view(np.int16).reshape(-1, 1024)).view(torch.bfloat16)
    w = quantize_on_gpu(W)
    check_dequantize_exact(w, check_quantize_exact(W, w))


def test_zero_blocks_and_signed_zeros():
    bits = si.bf16_bits(si.custom_linear(4, 512, 1, 1, seed=9)[0]).copy()
    bits[0, :64] = 0
    bits[1, 64:128] = 0x8000          # -0.0
    bits[2, :] = 0
    W = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    w = quantize_on_gpu(W)
    check_dequantize_exact(w, check_quantize_exact(W, w))


def test_nonfinite_weight_sets_flag():
    bits = si.bf16_bits(si.custom_linear(2, 128, 1, 1, seed=4)[0]).copy()
    bits[1, 5] = 0x7F80               # +Inf
    W = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(DEV)
    q4.qlora_read_device_errors(clear=True)
    q4.qlora_quantize_nf4_dq(W)
    flags = q4.qlora_read_device_errors(clear=True)
    assert flags & 2


# ------------------------------------------------------------------ linear forward / backward

def run_linear(W, X, A, B, dY, r, alpha, y_dtype=torch.bfloat16, dx_dtype=torch.bfloat16, save_U=True):
    w = quantize_on_gpu(W)
    Xd, Ad, Bd, dYd = (t.to(DEV) for t in (X, A, B, dY))
    Y, U = q4.qlora_linear_fwd(w, Xd, Ad, Bd, r, alpha, y_dtype=y_dtype, save_U=save_U)
    dX, dA, dB = q4.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, r, alpha, U_saved=U, dx_dtype=dx_dtype)
    torch.cuda.synchronize()
    return w, Y, U, dX, dA, dB


def check_linear_full(W, X, A, B, dY, r, alpha, **kw):
    w, Y, U, dX, dA, dB = run_linear(W, X, A, B, dY, r, alpha, **kw)
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], qw["N"], qw["K"])
    bX, bA, bB, bdY = (si.bf16_bits(t) for t in (X, A, B, dY))
    Yr, Ur = o.linear_forward(bX, Wh, bA, bB, alpha, r)
    g = o.linear_backward(bX, bdY, Wh, bA, bB, alpha, r)
    assert_close(Y, Yr, "Y")
    if U is not None:
        assert_close(U, Ur, "U")
    assert_close(dX, g["dX"], "dX")
    assert_close(dA, g["dA"], "dA")
    assert_close(dB, g["dB"], "dB")
    return w


def test_tiny_workload_full():
    wl = si.WORKLOADS["tiny"]
    W = si.weight(wl, 0)
    N, K = wl.linears[0]
    X = si.activations(wl, K, wl.M)
    A, B = si.lora(wl, 0)
    dY = si.grad_output(wl, 0, wl.M)
    for y_dtype in (torch.bfloat16, torch.float32):
        check_linear_full(W, X, A, B, dY, wl.r, wl.alpha, y_dtype=y_dtype, dx_dtype=y_dtype)


@pytest.mark.parametrize("M,N,K,r", [(1, 64, 64, 1), (3, 192, 128, 5), (17, 320, 192, 16),
                                     (130, 96, 640, 64), (33, 128, 256, 256), (5, 100, 128, 3),
                                     (300, 520, 1088, 96), (257, 264, 320, 200)])
def test_ragged_linear(M, N, K, r):
    W, X, A, B, dY = si.custom_linear(N, K, M, r, seed=M + N + K + r)
    check_linear_full(W, X, A, B, dY, r, alpha=2.0 * r)


# Small-M forward (M <= 16): the work is cut into equal ranges of (128-row tile, 64-wide
# K-step) units, one per persistent CTA.  These shapes give one unit per CTA (every tile
# summed from many partials), CTAs that cross several tile boundaries, a tile split over
# ~300 CTAs, ragged N, the largest rank, and both output types.
@pytest.mark.parametrize("M,N,K,r,y_f32", [(16, 1000, 640, 16, False), (7, 2600, 64, 8, True),
                                           (16, 40000, 64, 16, False), (2, 300, 4096, 256, False),
                                           (16, 9000, 1024, 16, True), (1, 128, 19200, 4, False)])
def test_decode_stream_k_layouts(M, N, K, r, y_f32):
    W, X, A, B, dY = si.custom_linear(N, K, M, r, seed=3 * M + N + K + r)
    dt = torch.float32 if y_f32 else torch.bfloat16
    check_linear_full(W, X, A, B, dY, r, alpha=2.0 * r, y_dtype=dt, dx_dtype=dt)


# dX with more than 256 tokens on CTA pairs (512-token x 256-column pair tiles): one tile short of
# its tokens, column tails of 128 and 64 columns, tiles whose K-steps are almost all LoRA steps
# (N = 64, 192), a long reduction, and fp32 output.  Two calls give the same bits.
@pytest.mark.parametrize("M,N,K,r,dx_f32", [(512, 192, 8192, 16, False), (1024, 4096, 640, 64, True),
                                            (300, 64, 4992, 8, False), (777, 1000, 1344, 16, True)])
def test_dx_pair_layouts(M, N, K, r, dx_f32):
    W, X, A, B, dY = si.custom_linear(N, K, M, r, seed=5 * M + N + K + r)
    dt = torch.float32 if dx_f32 else torch.bfloat16
    w = check_linear_full(W, X, A, B, dY, r, alpha=2.0 * r, dx_dtype=dt)
    Xd, Ad, Bd, dYd = (t.to(DEV) for t in (X, A, B, dY))
    _, U = q4.qlora_linear_fwd(w, Xd, Ad, Bd, r, 2.0 * r)
    dX1, _, _ = q4.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, r, 2.0 * r, U_saved=U, dx_dtype=dt)
    dX2, _, _ = q4.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, r, 2.0 * r, U_saved=U, dx_dtype=dt)
    torch.cuda.synchronize()
    assert torch.equal(dX1, dX2)


def test_recompute_U_and_no_dX():
    W, X, A, B, dY = si.custom_linear(128, 256, 24, 8, seed=77)
    w = quantize_on_gpu(W)
    Xd, Ad, Bd, dYd = (t.to(DEV) for t in (X, A, B, dY))
    _, U = q4.qlora_linear_fwd(w, Xd, Ad, Bd, 8, 16.0)
    dX1, dA1, dB1 = q4.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, 8, 16.0, U_saved=U)
    dX2, dA2, dB2 = q4.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, 8, 16.0, U_saved=None, need_dX=False)
    assert dX2 is None
    assert torch.allclose(dA1, dA2, rtol=1e-5, atol=1e-6)
    assert torch.allclose(dB1, dB2, rtol=1e-5, atol=1e-6)


def test_backward_leaves_weight_buffers_untouched():
    W, X, A, B, dY = si.custom_linear(256, 512, 64, 16, seed=5)
    w = quantize_on_gpu(W)
    before = [t.clone() for t in (w.codes, w.c1_codes, w.c2, w.mu)]
    Xd, Ad, Bd, dYd = (t.to(DEV) for t in (X, A, B, dY))
    _, U = q4.qlora_linear_fwd(w, Xd, Ad, Bd, 16, 32.0)
    q4.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, 16, 32.0, U_saved=U)
    torch.cuda.synchronize()
    for a, b in zip(before, (w.codes, w.c1_codes, w.c2, w.mu)):
        assert torch.equal(a, b)


def test_alpha_zero_and_zero_B():
    W, X, A, B, dY = si.custom_linear(64, 128, 8, 4, seed=6)
    check_linear_full(W, X, A, B, dY, 4, alpha=0.0)
    Bz = torch.zeros_like(B)
    w, Y, U, dX, dA, dB = run_linear(W, X, A, Bz, dY, 4, 8.0)
    assert torch.count_nonzero(dA) == 0
