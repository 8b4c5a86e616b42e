"""Save and reload of the frozen quantized weight.

The adapters are what training saves; the frozen 4-bit weight is reloaded beside
them, and outputs must stay the same after the round trip ("QLoRA 的原理是什么？
4-bit 量化权重真的参与训练吗？", section 6 "如何验证配置" and section 8: check that
saving, loading and serving agree).  The quantized weight is four flat buffers
(codes, E4M3 constant codes, c2, mu; or the fp32 constants with double
quantization off), so a round trip must give the same bytes, the same
dequantized weight and the same layer outputs.

CPU: the round trip of buffers the oracle wrote, and the checks of the loader.
GPU: quantize with the library, save to a file, reload onto the device, then
bit-identical dequantization and forward/backward outputs.
"""
import io

import numpy as np
import pytest
import torch

import bit_nf4_quantized_23_b200 as q4
import synthetic_inputs as si
from oracle import nf4_oracle as o


def _roundtrip(state: dict) -> dict:
    f = io.BytesIO()
    torch.save(state, f)
    f.seek(0)
    return torch.load(f, weights_only=True)


def _oracle_weight_on_cpu(N, K, seed):
    """An NF4Weight on the CPU holding the oracle's buffers (no library call computes them)."""
    bits = si.bf16_bits(si.custom_linear(N, K, 1, 1, seed=seed)[0])
    qw = o.quantize_nf4_dq(bits)
    w = q4.NF4Weight(torch.from_numpy(qw["codes"].copy()), torch.from_numpy(qw["c1_codes"].copy()),
                     torch.from_numpy(qw["c2"].copy()), torch.from_numpy(np.array([qw["mu"]], np.float32)), N, K)
    return w, qw


def test_roundtrip_keeps_every_byte_and_the_dequantized_weight():
    w, qw = _oracle_weight_on_cpu(96, 640, seed=61)
    w2 = q4.NF4Weight.from_state_dict(_roundtrip(w.state_dict()), device="cpu")
    for name in ("codes", "c1_codes", "c2", "mu"):
        a, b = getattr(w, name), getattr(w2, name)
        assert a.dtype == b.dtype and torch.equal(a.view(torch.uint8), b.view(torch.uint8)), name
    assert w2.c1 is None and (w2.N, w2.K, w2.codebook, w2.compute_dtype) == (96, 640, "nf4", torch.bfloat16)
    Wh = o.dequantize(w2.codes.numpy(), w2.c1_codes.numpy(), w2.c2.numpy(), w2.mu.numpy()[0], 96, 640)
    ref = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 96, 640)
    assert np.array_equal(Wh, ref)


def test_loader_rejects_mismatched_buffers():
    w, _ = _oracle_weight_on_cpu(8, 128, seed=62)
    bad = w.state_dict()
    bad["codes"] = bad["codes"][:-1]
    with pytest.raises(ValueError):
        q4.NF4Weight.from_state_dict(bad, device="cpu")
    bad = w.state_dict()
    bad["c1"] = torch.zeros(16)                     # fp32 constants beside the DQ buffers
    with pytest.raises(ValueError):
        q4.NF4Weight.from_state_dict(bad, device="cpu")
    bad = w.state_dict()
    bad["blocksize"] = 128
    with pytest.raises(ValueError):
        q4.NF4Weight.from_state_dict(bad, device="cpu")


@pytest.mark.gpu
@pytest.mark.parametrize("double_quant", [True, False])
def test_gpu_save_reload_gives_identical_outputs(tmp_path, double_quant):
    from bit_nf4_quantized_23_b200.build import build
    build()
    dev = torch.device("cuda:0")
    W, X, A, B, dY = (t.to(dev) for t in si.custom_linear(384, 1024, 40, 16, seed=63))
    w = q4.qlora_quantize_nf4_dq(W, double_quant=double_quant)
    path = tmp_path / "frozen_weight.pt"
    torch.save(w.state_dict(), path)
    w2 = q4.NF4Weight.from_state_dict(torch.load(path, weights_only=True), device=dev)
    for name in ("codes", "c1_codes", "c2", "mu", "c1"):
        a, b = getattr(w, name), getattr(w2, name)
        assert (a is None) == (b is None), name
        if a is not None:
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), name
    assert torch.equal(q4.qlora_dequantize(w).view(torch.int16), q4.qlora_dequantize(w2).view(torch.int16))
    outs = []
    for ww in (w, w2):
        Y, U = q4.qlora_linear_fwd(ww, X, A, B, 16, 32.0)
        dX, dA, dB = q4.qlora_linear_bwd(ww, X, dY, A, B, 16, 32.0, U_saved=U)
        outs.append((Y, U, dX, dA, dB))
    torch.cuda.synchronize()
    for a, b in zip(*outs):                          # deterministic kernels: the same bits
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))
    assert q4.qlora_read_device_errors(clear=True) == 0
