"""Failure detection without a GPU fault.

Every mbarrier wait in the library's kernels is bounded in wall time; a wait
that runs out raises the timeout device flag and the kernel returns.  The
self-test entry point runs that same bounded wait on a barrier nothing
completes, with a short limit: the wait must give up after the limit, the host
must read QLORA_ERR_TIMEOUT's flag, and the context must stay usable (a
quantize/dequantize round trip afterwards still matches the oracle bit for bit).
"""
import time

import numpy as np
import pytest
import torch

import bit_nf4_quantized_23_b200 as q4
import synthetic_inputs as si
from oracle import nf4_oracle as o

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    from bit_nf4_quantized_23_b200.build import build
    build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    q4.qlora_read_device_errors(clear=True)
    yield
    q4.qlora_read_device_errors(clear=True)


def test_bounded_wait_gives_up_reports_and_the_context_survives():
    limit_us = 20000
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    completed, aborted = q4.qlora_selftest_bounded_wait(limit_us)
    elapsed = time.perf_counter() - t0
    assert not completed and aborted
    assert elapsed >= limit_us * 1e-6
    assert elapsed < 5.0
    assert q4.qlora_read_device_errors(clear=True) & 1          # the timeout flag, read on the host
    assert q4.qlora_read_device_errors(clear=True) == 0         # and cleared
    # the context is still usable
    W = si.custom_linear(256, 512, 16, 8, seed=31)[0]
    w = q4.qlora_quantize_nf4_dq(W.cuda())
    Wh = q4.qlora_dequantize(w).cpu()
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    ref = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 256, 512)
    assert np.array_equal(si.bf16_bits(Wh), ref)
    assert q4.qlora_read_device_errors(clear=True) == 0


def test_bounded_wait_limit_is_checked_on_the_host():
    with pytest.raises(q4.QloraError):
        q4.qlora_selftest_bounded_wait(0)
    with pytest.raises(q4.QloraError):
        q4.qlora_selftest_bounded_wait(2_000_000)
