"""GPU parity of the quantizer variants against the CPU oracle.

Variants ([SD] section 4 (2) compares NF4 with a uniform 4-bit grid; section 3
part 2 adds double quantization on top of single-level absmax constants):
the uniform grid with and without double quantization, and NF4 without it
(NF4 with it is covered by test_gpu_parity.py).  Bit-exact: codes, constants
and the dequantized weight.  Within tolerance: the forward and backward of the
linear layer through every GEMM path (tensor-core large-M, small-M stream-K,
CUDA-core for N % 8 != 0).  The error study is recomputed from the GPU's
dequantized weights and must equal the oracle's figure exactly.
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

VARIANTS = [("uniform4", True), ("nf4", False), ("uniform4", False)]
CODEBOOK = {"nf4": o.nf4_codebook(), "uniform4": o.uniform4_codebook()}


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    from bit_nf4_quantized_23_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q4.qlora_read_device_errors(clear=True)
    yield
    assert q4.qlora_read_device_errors(clear=True) == 0


def oracle_variant(W_cpu, codebook, dq):
    """Oracle buffers and W_hat bits of a variant."""
    q = CODEBOOK[codebook]
    qw = o.quantize_nf4_dq(si.bf16_bits(W_cpu), q=q)
    if dq:
        Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], qw["N"], qw["K"], q=q)
    else:
        Wh = o.dequantize_single(qw["codes"], qw["c1"], qw["N"], qw["K"], q=q)
    return qw, Wh


def check_buffers(w, qw, dq):
    assert np.array_equal(w.codes.cpu().numpy(), qw["codes"])
    if dq:
        assert w.c1 is None
        assert np.array_equal(w.c1_codes.cpu().numpy(), qw["c1_codes"])
        assert np.array_equal(w.c2.cpu().numpy().view(np.uint32), qw["c2"].view(np.uint32))
        assert w.mu.cpu().numpy().view(np.uint32)[0] == np.float32(qw["mu"]).view(np.uint32)
    else:
        assert w.c1_codes is None and w.c2 is None and w.mu is None
        assert np.array_equal(w.c1.cpu().numpy().view(np.uint32), qw["c1"].view(np.uint32))


@pytest.mark.parametrize("codebook,dq", VARIANTS)
@pytest.mark.parametrize("N,K", [(256, 256), (3, 320), (17, 1024), (520, 1088)])
def test_variant_quantize_and_dequantize_bit_exact(codebook, dq, N, K):
    W = si.custom_linear(N, K, 1, 1, seed=N + K, dist="t5_outliers")[0]
    w = q4.qlora_quantize_nf4_dq(W.to(DEV), codebook=codebook, double_quant=dq)
    qw, Wh_ref = oracle_variant(W, codebook, dq)
    check_buffers(w, qw, dq)
    assert np.array_equal(to_numpy_bits(q4.qlora_dequantize(w)), Wh_ref)


def test_variant_quantize_every_finite_bf16_value():
    # every finite bf16 pattern once, in blocks with large and tiny absmax, on both grids
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = bits[(bits & 0x7F80) != 0x7F80]
    pad = (-finite.size) % 1024
    allb = np.concatenate([finite, np.zeros(pad, np.uint16)]).reshape(-1, 1024)
    W = torch.from_numpy(allb.view(np.int16)).view(torch.bfloat16)
    for codebook, dq in VARIANTS:
        w = q4.qlora_quantize_nf4_dq(W.to(DEV), codebook=codebook, double_quant=dq)
        qw, Wh_ref = oracle_variant(W, codebook, dq)
        check_buffers(w, qw, dq)
        assert np.array_equal(to_numpy_bits(q4.qlora_dequantize(w)), Wh_ref)


def run_variant_linear(codebook, dq, M, N, K, r, y_dtype=torch.bfloat16):
    W, X, A, B, dY = si.custom_linear(N, K, M, r, seed=2 * M + N + K + r)
    alpha = 2.0 * r
    w = q4.qlora_quantize_nf4_dq(W.to(DEV), codebook=codebook, double_quant=dq)
    Xd, Ad, Bd, dYd = (t.to(DEV) for t in (X, A, B, dY))
    Y, U = q4.qlora_linear_fwd(w, Xd, Ad, Bd, r, alpha, y_dtype=y_dtype)
    dX, dA, dB = q4.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, r, alpha, U_saved=U, dx_dtype=y_dtype)
    torch.cuda.synchronize()
    _, Wh = oracle_variant(W, codebook, dq)
    bX, bA, bB, bdY = (si.bf16_bits(t) for t in (X, A, B, dY))
    Yr, Ur = o.linear_forward(bX, Wh, bA, bB, alpha, r)
    g = o.linear_backward(bX, bdY, Wh, bA, bB, alpha, r)
    assert_close(Y, Yr, "Y")
    assert_close(U, Ur, "U")
    assert_close(dX, g["dX"], "dX")
    assert_close(dA, g["dA"], "dA")
    assert_close(dB, g["dB"], "dB")


@pytest.mark.parametrize("codebook,dq", VARIANTS)
@pytest.mark.parametrize("M,N,K,r", [(5, 100, 128, 3), (16, 1000, 640, 16), (130, 96, 640, 64),
                                     (300, 520, 1088, 96), (33, 130, 256, 8)])
def test_variant_linear_fwd_bwd(codebook, dq, M, N, K, r):
    run_variant_linear(codebook, dq, M, N, K, r)


def test_variant_linear_fp32_outputs():
    run_variant_linear("uniform4", False, 64, 256, 512, 16, y_dtype=torch.float32)


def test_error_study_from_gpu_dequant_equals_oracle():
    # relative squared error sum (W_hat - W)^2 / sum W^2 of each variant, from the GPU's W_hat
    W = si.custom_linear(256, 1024, 1, 1, seed=3, sigma=0.02, dist="normal")[0]
    bits = si.bf16_bits(W)
    errs = {}
    for codebook, dq in VARIANTS + [("nf4", True)]:
        w = q4.qlora_quantize_nf4_dq(W.to(DEV), codebook=codebook, double_quant=dq)
        gpu = o.relative_sq_error(bits, to_numpy_bits(q4.qlora_dequantize(w)))
        ref = o.relative_sq_error(bits, oracle_variant(W, codebook, dq)[1])
        assert gpu == ref
        errs[codebook, dq] = gpu
    assert errs["nf4", False] < 0.9 * errs["uniform4", False]


def test_variant_argument_errors():
    W = si.custom_linear(64, 128, 1, 1, seed=1)[0].to(DEV)
    w = q4.NF4Weight.empty(64, 128, DEV, "nf4", double_quant=False)
    ws = w.c_struct()
    ws.codebook = 5
    from bit_nf4_quantized_23_b200 import _lib
    import ctypes
    sizes = q4.qlora_nf4_sizes(64, 128)
    scratch = torch.empty(sizes["workspace"], dtype=torch.uint8, device=DEV)
    st = _lib.lib().qlora_quantize_nf4_dq(ctypes.c_void_p(W.data_ptr()), 64, 128, 64, 256, ctypes.byref(ws),
                                         ctypes.c_void_p(scratch.data_ptr()), scratch.numel(), None)
    assert st == 1                                    # QLORA_ERR_INVALID_ARG, nothing launched
    ws.codebook = 0
    ws.compute_dtype = 3
    st = _lib.lib().qlora_quantize_nf4_dq(ctypes.c_void_p(W.data_ptr()), 64, 128, 64, 256, ctypes.byref(ws),
                                         ctypes.c_void_p(scratch.data_ptr()), scratch.numel(), None)
    assert st == 1


# ------------------------------------------------------------------ merge and requantize

@pytest.mark.parametrize("codebook,dq", [("nf4", True), ("uniform4", False)])
@pytest.mark.parametrize("N,K,r", [(256, 256, 8), (520, 1088, 96), (3, 320, 3), (130, 640, 256)])
def test_merge_lora_matches_oracle_and_requantizes_exactly(codebook, dq, N, K, r):
    # The GPU sums the rank-r term in fp32 and rounds once to bf16; the oracle sums in fp64.
    # The two can differ by one bf16 step where the fp32 sum lands across a rounding
    # boundary (rare); the requantization of the GPU's merged weight is bit-exact.
    W, X, A, B, dY = si.custom_linear(N, K, 1, r, seed=N + K + r)
    B = (B.float() * 30.0).to(torch.bfloat16)          # make the update visible next to W
    alpha = 2.0 * r
    w = q4.qlora_quantize_nf4_dq(W.to(DEV), codebook=codebook, double_quant=dq)
    Wm = q4.qlora_merge_lora(w, A.to(DEV), B.to(DEV), r, alpha)
    _, Wh = oracle_variant(W, codebook, dq)
    ref = o.merge_lora(Wh, si.bf16_bits(A), si.bf16_bits(B), alpha, r)
    got = to_numpy_bits(Wm)
    # bound: one bf16 step of the result plus the fp32 accumulation error of r terms
    # (r * 2^-23 * sum |s B A| covers r roundings or truncations); the second term only
    # matters where the update cancels W_hat and the result is far below its terms
    gv = o.bf16_bits_to_f32(got).astype(np.float64)
    rv = o.bf16_bits_to_f32(ref).astype(np.float64)
    sumabs = (alpha / r) * (np.abs(o._f64(si.bf16_bits(B))) @ np.abs(o._f64(si.bf16_bits(A))))
    step = np.ldexp(1.0, np.maximum(np.frexp(rv)[1], -125) - 8)
    assert np.all(np.abs(gv - rv) <= step + r * 2.0 ** -23 * sumabs), "beyond one step + accumulation bound"
    assert np.count_nonzero(got != ref) <= max(2, got.size // 500)
    # requantize the merged weight: bit-exact against the oracle on the same bits
    w2 = q4.qlora_quantize_nf4_dq(Wm, codebook=codebook, double_quant=dq)
    qw2 = o.quantize_nf4_dq(got, q=CODEBOOK[codebook])
    check_buffers(w2, qw2, dq)


def test_merge_with_zero_B_is_the_dequantized_weight():
    W, X, A, B, dY = si.custom_linear(64, 512, 1, 16, seed=12)
    w = q4.qlora_quantize_nf4_dq(W.to(DEV))
    Wm = q4.qlora_merge_lora(w, A.to(DEV), torch.zeros_like(B).to(DEV), 16, 32.0)
    assert torch.equal(Wm, q4.qlora_dequantize(w))


# ------------------------------------------------------------------ one base, many adapters

@pytest.mark.parametrize("M,N,K,r,n_ad", [(16, 1000, 640, 16, 16), (7, 2600, 64, 8, 3), (1, 300, 4096, 64, 2),
                                          (16, 9000, 1024, 3, 5), (12, 264, 320, 96, 4)])
def test_multi_adapter_forward(M, N, K, r, n_ad):
    g = np.random.default_rng(M + N + K)
    W, X, A, B, dY = si.custom_linear(N, K, M, r, seed=M + N + K + r)
    A_all = torch.stack([si.custom_linear(N, K, M, r, seed=100 + a)[2] for a in range(n_ad)])
    B_all = torch.stack([(si.custom_linear(N, K, M, r, seed=200 + a)[3].float() * (a + 1)).to(torch.bfloat16)
                         for a in range(n_ad)])
    idx = g.integers(-1, n_ad, size=M).astype(np.int32)
    idx[0] = n_ad - 1                                   # at least one adapted token
    alpha = 2.0 * r
    w = q4.qlora_quantize_nf4_dq(W.to(DEV))
    Y, U = q4.qlora_linear_fwd_multi(w, X.to(DEV), A_all.to(DEV), B_all.to(DEV), torch.from_numpy(idx).to(DEV),
                                     r, alpha, save_U=True)
    torch.cuda.synchronize()
    _, Wh = oracle_variant(W, "nf4", True)
    Yr, Ur = o.linear_forward_multi(si.bf16_bits(X), Wh, si.bf16_bits(A_all), si.bf16_bits(B_all), idx, alpha, r)
    assert_close(Y, Yr, "Y multi")
    assert_close(U, Ur, "U multi")


def test_multi_adapter_out_of_range_index_sets_flag_and_uses_base():
    W, X, A, B, dY = si.custom_linear(256, 256, 2, 8, seed=21)
    w = q4.qlora_quantize_nf4_dq(W.to(DEV))
    idx = torch.tensor([0, 7], dtype=torch.int32, device=DEV)       # 7 >= n_adapters = 1
    q4.qlora_read_device_errors(clear=True)
    Y, _ = q4.qlora_linear_fwd_multi(w, X.to(DEV), A[None].to(DEV), B[None].to(DEV), idx, 8, 16.0)
    flags = q4.qlora_read_device_errors(clear=True)
    assert flags & 4
    _, Wh = oracle_variant(W, "nf4", True)
    Yr, _ = o.linear_forward_multi(si.bf16_bits(X), Wh, si.bf16_bits(A)[None], si.bf16_bits(B)[None], [0, -1],
                                   16.0, 8)
    assert_close(Y, Yr, "Y with one token on the base")


# ------------------------------------------------------------------ fp16 compute dtype

F16 = torch.float16


def _f64_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().double().cpu().numpy()


@pytest.mark.parametrize("codebook,dq", [("nf4", True), ("uniform4", False)])
@pytest.mark.parametrize("N,K", [(256, 256), (3, 320), (520, 1088)])
def test_fp16_dequantize_bit_exact(codebook, dq, N, K):
    W = si.custom_linear(N, K, 1, 1, seed=N + K + 5, dist="t5_outliers")[0]
    w = q4.qlora_quantize_nf4_dq(W.to(DEV), codebook=codebook, double_quant=dq, compute_dtype=F16)
    q = CODEBOOK[codebook]
    qw = o.quantize_nf4_dq(si.bf16_bits(W), q=q)
    check_buffers(w, qw, dq)
    ref = (o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], N, K, q=q, f16=True) if dq
           else o.dequantize_single(qw["codes"], qw["c1"], N, K, q=q, f16=True))
    Wh = q4.qlora_dequantize(w)
    assert Wh.dtype == F16
    assert np.array_equal(to_numpy_bits(Wh), ref)


@pytest.mark.parametrize("M,N,K,r", [(5, 100, 128, 3), (16, 1000, 640, 16), (130, 96, 640, 64),
                                     (300, 520, 1088, 96), (33, 130, 256, 8)])
def test_fp16_linear_fwd_bwd(M, N, K, r):
    W, X, A, B, dY = si.custom_linear(N, K, M, r, seed=3 * M + N + K + r)
    Xh, Ah, Bh, dYh = (t.float().half() for t in (X, A, B, dY))      # exact: bf16 values in fp16 range
    alpha = 2.0 * r
    w = q4.qlora_quantize_nf4_dq(W.to(DEV), compute_dtype=F16)
    Xd, Ad, Bd, dYd = (t.to(DEV) for t in (Xh, Ah, Bh, dYh))
    Y, U = q4.qlora_linear_fwd(w, Xd, Ad, Bd, r, alpha)
    dX, dA, dB = q4.qlora_linear_bwd(w, Xd, dYd, Ad, Bd, r, alpha, U_saved=U)
    torch.cuda.synchronize()
    assert Y.dtype == F16 and dX.dtype == F16
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    Wh = o.f16_bits_to_f32(o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], N, K,
                                        f16=True)).astype(np.float64)
    Xf, Af, Bf, dYf = (_f64_of(t) for t in (Xh, Ah, Bh, dYh))
    Yr, Ur = o.linear_forward(Xf, Wh, Af, Bf, alpha, r)
    g = o.linear_backward(Xf, dYf, Wh, Af, Bf, alpha, r)
    assert_close(Y, Yr, "Y fp16")
    assert_close(U, Ur, "U fp16")
    assert_close(dX, g["dX"], "dX fp16")
    assert_close(dA, g["dA"], "dA fp16")
    assert_close(dB, g["dB"], "dB fp16")


def test_fp16_multi_adapter_and_merge():
    N, K, M, r, n_ad = 1000, 640, 16, 16, 4
    W, X, A, B, dY = si.custom_linear(N, K, M, r, seed=77)
    w = q4.qlora_quantize_nf4_dq(W.to(DEV), compute_dtype=F16)
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    Whb = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], N, K, f16=True)
    Wh = o.f16_bits_to_f32(Whb).astype(np.float64)
    A_all = torch.stack([si.custom_linear(N, K, M, r, seed=300 + a)[2] for a in range(n_ad)]).float().half()
    B_all = torch.stack([si.custom_linear(N, K, M, r, seed=400 + a)[3] for a in range(n_ad)]).float().half()
    idx = np.array([0, 1, 2, 3, -1, 0, 1, 2, 3, -1, 3, 2, 1, 0, 0, 1], dtype=np.int32)
    Xh = X.float().half()
    Y, U = q4.qlora_linear_fwd_multi(w, Xh.to(DEV), A_all.to(DEV), B_all.to(DEV), torch.from_numpy(idx).to(DEV),
                                     r, 2.0 * r, save_U=True)
    Yr, Ur = o.linear_forward_multi(_f64_of(Xh), Wh, _f64_of(A_all), _f64_of(B_all), idx, 2.0 * r, r)
    assert Y.dtype == F16
    assert_close(Y, Yr, "Y fp16 multi")
    assert_close(U, Ur, "U fp16 multi")
    # merge in fp16: within one fp16 step plus the fp32 accumulation bound of the fp64 merge
    Ah, Bh = A.float().half(), (B.float() * 30.0).half()
    Wm = q4.qlora_merge_lora(w, Ah.to(DEV), Bh.to(DEV), r, 2.0 * r)
    assert Wm.dtype == F16
    ref = o.merge_lora(Wh, _f64_of(Ah), _f64_of(Bh), 2.0 * r, r, f16=True)
    gv = o.f16_bits_to_f32(to_numpy_bits(Wm)).astype(np.float64)
    rv = o.f16_bits_to_f32(ref).astype(np.float64)
    sumabs = 2.0 * (np.abs(_f64_of(Bh)) @ np.abs(_f64_of(Ah)))
    step = np.ldexp(1.0, np.maximum(np.frexp(rv)[1], -13) - 11)
    assert np.all(np.abs(gv - rv) <= step + r * 2.0 ** -23 * sumabs)
