"""GPU parity of the blockwise absmax INT8 quantizer ("Ch.09 QLoRA 与量化：缩得更小再微调",
section "2. INT8 量化") against the CPU oracle: codes, scales and the dequantized
values bit for bit, on the page's worked example, on seeded weights spanning
several CTAs with a ragged last one, at every bf16 scale near every rounding
boundary, on every finite bf16 value, on the degenerate blocks (all zero, a scale
that overflows, exact halves) and, sampled, on a full-size W[22016,8192].
"""
import numpy as np
import pytest
import torch

import bit_nf4_quantized_23_b200 as q4
import synthetic_inputs as si
from conftest import read_golden
from oracle import nf4_oracle as o

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


def _bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def _gpu(bits, bs):
    codes, alpha = q4.qlora_quantize_int8_absmax(_bf16(bits).to(DEV), bs)
    torch.cuda.synchronize()
    return codes, alpha


def check_exact(bits, bs, dequant=True):
    codes, alpha = _gpu(bits, bs)
    oc, oa = o.quantize_int8_blocks(bits, bs)
    assert np.array_equal(alpha.cpu().numpy().view(np.uint32), oa.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy().ravel(), oc)
    if dequant:
        xh = o.dequantize_int8_blocks(oc, oa, bs)
        got = q4.qlora_dequantize_int8_absmax(codes, alpha, bs, torch.float32).cpu().numpy()
        assert np.array_equal(got.view(np.uint32), xh.view(np.uint32))
        got = q4.qlora_dequantize_int8_absmax(codes, alpha, bs, torch.bfloat16).cpu()
        assert np.array_equal(si.bf16_bits(got), o.f32_to_bf16_bits(xh))
        got = q4.qlora_dequantize_int8_absmax(codes, alpha, bs, torch.float16).cpu()
        assert np.array_equal(got.view(torch.int16).numpy().view(np.uint16), o.f32_to_f16_bits(xh))
    return codes, alpha


def test_int8_worked_example_on_the_gpu():
    g = read_golden("int8_absmax_example.txt")
    x = np.zeros(64, np.float32)
    x[:3] = g["input"]
    codes, alpha = check_exact(o.f32_to_bf16_bits(x), 64)
    c = codes.cpu().numpy()
    assert c[0] == g["code_of_1.2"] and c[2] == g["peak_code"] and c[1] == -12
    assert abs(float(alpha[0]) - g["alpha_approx"]) <= g["alpha_tolerance"]


@pytest.mark.parametrize("bs", [64, 128, 256])
def test_int8_seeded_weights_several_ctas_ragged_tail(bs):
    # one CTA covers 2048 elements: 37 full CTAs and a part-filled last one
    n = 2048 * 37 + 256 * 3
    W = si.t5_outlier_bf16((n,), 0.02, 3, "int8", f"bs{bs}")
    check_exact(si.bf16_bits(W), bs)


def test_int8_every_scale_near_every_rounding_boundary():
    """Every positive finite bf16 absmax c (subnormals included), with bf16 values
    within +-2 ulps of (k + 1/2) c / 127 for 12 k spread over 0..126."""
    scales = np.arange(1, 0x7F80, dtype=np.uint32).astype(np.uint16)
    c = o.bf16_bits_to_f32(scales).astype(np.float64)
    ks = np.array([0, 1, 2, 5, 13, 27, 40, 63, 64, 90, 111, 126], np.float64)
    centre = o.f32_to_bf16_bits(((ks[None, :] + 0.5) * c[:, None] / 127.0).astype(np.float32)).astype(np.int64)
    cand = np.concatenate([centre + d for d in (-2, -1, 0, 1, 2)], axis=1)          # [n_scales, 60]
    cand = np.where((cand & 0x7F80) == 0x7F80, 0, cand)
    mag = o.bf16_bits_to_f32(cand.astype(np.uint16)).astype(np.float64)
    cand = np.where(np.abs(mag) <= c[:, None], cand, 0).astype(np.uint16)
    sign = (np.arange(60) % 2).astype(np.uint16) << 15                                # both signs
    cand = np.where(cand != 0, cand | sign[None, :], cand).astype(np.uint16)
    zeros = np.zeros((scales.size, 3), np.uint16)
    blocks = np.concatenate([scales[:, None], cand, zeros], axis=1)                   # 64 per scale
    check_exact(blocks.ravel(), 64)


def test_int8_every_finite_bf16_value():
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = allb[(allb & 0x7F80) != 0x7F80]
    for bs in (64, 256):
        pad = (-finite.size) % bs
        check_exact(np.concatenate([finite, np.zeros(pad, np.uint16)]), bs)
        g = np.random.default_rng(bs)
        check_exact(g.permutation(np.concatenate([finite, np.zeros(pad, np.uint16)])), bs)


def test_int8_degenerate_blocks():
    def block(vals):
        x = np.zeros(64, np.float32)
        x[:len(vals)] = vals
        return o.f32_to_bf16_bits(x)
    tiny = float(o.bf16_bits_to_f32(np.array([0x0001], np.uint16))[0])
    bits = np.concatenate([block([]), block([tiny, -tiny, 0.0, tiny]),
                           block([127.0, 2.5, -2.5, 0.5, -0.5, 1.5, -1.5, 126.5]), block([-3.0, 1.5])])
    codes, alpha = check_exact(bits, 64)
    a = alpha.cpu().numpy()
    assert a[0] == 0 and np.isinf(a[1]) and a[2] == 1.0
    c = codes.cpu().numpy()
    assert list(c[64:68]) == [127, -127, 0, 127]
    assert list(c[128:136]) == [127, 3, -3, 1, -1, 2, -2, 127]


def test_int8_nonfinite_block_is_flagged():
    x = (np.arange(256, dtype=np.float32) - 128) / 64
    bits = o.f32_to_bf16_bits(x)
    bits[70] = 0x7FC0                                       # NaN in block 1
    codes, alpha = _gpu(bits, 64)
    assert q4.qlora_read_device_errors(clear=True) != 0
    a = alpha.cpu().numpy()
    c = codes.cpu().numpy()
    assert a[1] == 0 and np.all(c[64:128] == 0)
    ok = np.r_[0:64, 128:256]
    oc, oa = o.quantize_int8_blocks(np.where(np.arange(256) // 64 == 1, 0, bits).astype(np.uint16), 64)
    assert np.array_equal(c[ok], oc[ok]) and np.array_equal(a[[0, 2, 3]], oa[[0, 2, 3]])


def test_int8_full_size_sampled():
    W = si.weight("block65b", 4)                             # gate projection W[22016, 8192]
    bits = si.bf16_bits(W).ravel()
    codes, alpha = _gpu(bits, 64)
    xh = q4.qlora_dequantize_int8_absmax(codes, alpha, 64, torch.bfloat16)
    torch.cuda.synchronize()
    g = np.random.default_rng(9)
    blocks = np.sort(g.choice(bits.size // 64, size=4096, replace=False))
    sel = (blocks[:, None] * 64 + np.arange(64)[None, :]).ravel()
    oc, oa = o.quantize_int8_blocks(bits[sel], 64)
    idx = torch.from_numpy(sel).to(DEV)
    assert np.array_equal(codes.view(-1)[idx].cpu().numpy(), oc)
    assert np.array_equal(alpha[torch.from_numpy(blocks).to(DEV)].cpu().numpy().view(np.uint32), oa.view(np.uint32))
    assert np.array_equal(si.bf16_bits(xh.view(-1)[idx].cpu()), o.f32_to_bf16_bits(o.dequantize_int8_blocks(oc, oa, 64)))


def test_int8_argument_errors():
    W = torch.zeros(192, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(q4.QloraError) as e:
        q4.qlora_quantize_int8_absmax(W, 96)                 # blocksize 96: QLORA_ERR_UNSUPPORTED
    assert e.value.status == 4
    codes, alpha = q4.qlora_quantize_int8_absmax(W[:128], 64)
    with pytest.raises(TypeError):
        q4.qlora_dequantize_int8_absmax(codes, alpha, 64, torch.int32)


def test_int8_dequantize_every_code_at_every_reachable_scale():
    """code / alpha must be the correctly rounded fp32 quotient for every code -128..127
    and every alpha the quantizer can produce (127 / amax for every positive finite bf16
    amax), plus random fp32 scales over the whole range (both signs, subnormals, 0, inf)."""
    amax = o.bf16_bits_to_f32(np.arange(1, 0x7F80, dtype=np.uint32).astype(np.uint16))
    with np.errstate(divide="ignore", over="ignore"):
        reach = (np.float32(127.0) / amax).astype(np.float32)
    g = np.random.default_rng(12)
    bits = g.integers(0, 0xFF800000, size=65536, dtype=np.uint64).astype(np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]                     # no NaN or Inf patterns
    rand = bits.view(np.float32)
    alpha = np.concatenate([reach, rand, np.array([0.0, -0.0, np.inf, 1.0, 2.0 ** -100, 2.0 ** 100,
                                                   2.0 ** -101, 2.0 ** 101], np.float32)])
    codes = np.tile(np.arange(-128, 128, dtype=np.int32).astype(np.int8), alpha.size)
    want = o.dequantize_int8_blocks(codes, alpha, 256)
    got = q4.qlora_dequantize_int8_absmax(torch.from_numpy(codes).to(DEV), torch.from_numpy(alpha).to(DEV),
                                          256, torch.float32).cpu().numpy()
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_int8_dequantize_rejects_a_short_scale_vector():
    codes, alpha = q4.qlora_quantize_int8_absmax(torch.zeros(256, dtype=torch.bfloat16, device=DEV), 64)
    with pytest.raises(ValueError):
        q4.qlora_dequantize_int8_absmax(codes, alpha[:3], 64)
