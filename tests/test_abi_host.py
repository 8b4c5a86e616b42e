"""Host-side checks of libqlora.so that need no GPU: it loads, exports every
symbol include/qlora.h declares, its own codebook equals the oracle's bit for
bit, its decision thresholds reproduce the oracle's nearest-code rule, its size
query matches the stored-buffer sizes, and bad arguments are rejected on the
host with the documented status before anything is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

from conftest import ROOT
from oracle import nf4_oracle as o
from bit_nf4_quantized_23_b200 import _lib
from bit_nf4_quantized_23_b200.build import build

HEADER = os.path.join(ROOT, "include", "qlora.h")


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"


def test_library_codebook_equals_oracle_bit_for_bit(L):
    v = (ctypes.c_float * 16)()
    t = (ctypes.c_float * 15)()
    assert L.qlora_nf4_codebook(v, t) == 0
    lib_q = np.array(v, dtype=np.float32)
    assert np.array_equal(lib_q.view(np.uint32), o.nf4_codebook().view(np.uint32))


def test_library_thresholds_give_the_nearest_code(L):
    v = (ctypes.c_float * 16)()
    t = (ctypes.c_float * 15)()
    L.qlora_nf4_codebook(v, t)
    q = np.array(v, dtype=np.float32)
    thr = np.array(t, dtype=np.float32)
    # every fp32 in [-1, 1] that matters: a dense sweep plus the fp32 neighbourhoods of the thresholds
    g = np.random.default_rng(21)
    x = np.concatenate([g.uniform(-1, 1, 200000).astype(np.float32), q,
                        thr, np.nextafter(thr, np.float32(2)), np.nextafter(thr, np.float32(-2)),
                        np.array([0.0, -0.0, 1e-30, -1e-30, 1.0, -1.0], np.float32)])
    by_threshold = (x[:, None] > thr[None, :]).sum(axis=1)
    assert np.array_equal(by_threshold, o.nearest_code(x, q))


def test_library_uniform4_codebook_and_thresholds(L):
    v = (ctypes.c_float * 16)()
    t = (ctypes.c_float * 15)()
    assert L.qlora_codebook_values(1, v, t) == 0
    q = np.array(v, dtype=np.float32)
    assert np.array_equal(q.view(np.uint32), o.uniform4_codebook().view(np.uint32))
    thr = np.array(t, dtype=np.float32)
    g = np.random.default_rng(22)
    x = np.concatenate([g.uniform(-1, 1, 200000).astype(np.float32), q, thr,
                        np.nextafter(thr, np.float32(2)), np.nextafter(thr, np.float32(-2))])
    assert np.array_equal((x[:, None] > thr[None, :]).sum(axis=1), o.nearest_code(x, q))
    assert L.qlora_codebook_values(0, v, t) == 0
    assert np.array_equal(np.array(v, dtype=np.float32).view(np.uint32), o.nf4_codebook().view(np.uint32))
    assert L.qlora_codebook_values(7, v, t) == 1          # unknown codebook: QLORA_ERR_INVALID_ARG


def test_sizes_match_oracle(L):
    for N, K in ((256, 256), (4096, 11008), (3, 320), (1, 64)):
        a, b, c, d = (ctypes.c_size_t() for _ in range(4))
        assert L.qlora_nf4_sizes(N, K, 64, 256, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c),
                                 ctypes.byref(d)) == 0
        sb = o.stored_bytes(N, K)
        assert (a.value, b.value, c.value) == (sb["codes"], sb["c1_codes"], sb["c2"])
        assert d.value >= 4 * (N * K // 64)


def test_status_strings(L):
    for s in range(9):
        assert L.qlora_status_string(s).decode().startswith(_lib.STATUS_NAMES[s])


def _w(codes=0x10000, c1=0x20000, c2=0x30000, mu=0x40000, N=4, K=128, bs=64, bs2=256):
    return _lib.NF4WeightC(codes, c1, c2, mu, N, K, bs, bs2)


FAKE = 0x7f0000000000      # never dereferenced: every call below fails validation first


def test_host_validation_before_launch(L):
    launches_before = L.qlora_launch_count()
    sz = ctypes.c_size_t()
    E = {v: k for k, v in _lib.STATUS_NAMES.items()}
    assert L.qlora_nf4_sizes(4, 96, 64, 256, None, None, None, None) == E["QLORA_ERR_SHAPE"]
    assert L.qlora_nf4_sizes(0, 64, 64, 256, None, None, None, None) == E["QLORA_ERR_SHAPE"]
    assert L.qlora_nf4_sizes(4, 128, 32, 256, None, None, None, None) == E["QLORA_ERR_UNSUPPORTED"]
    assert L.qlora_nf4_sizes(4, 128, 64, 128, None, None, None, None) == E["QLORA_ERR_UNSUPPORTED"]
    w = _w()
    # quantize: null W, misaligned W, shape mismatch with out, missing workspace
    assert L.qlora_quantize_nf4_dq(None, 4, 128, 64, 256, ctypes.byref(w), FAKE, 1 << 20, None) == \
        E["QLORA_ERR_INVALID_ARG"]
    assert L.qlora_quantize_nf4_dq(FAKE + 2, 4, 128, 64, 256, ctypes.byref(w), FAKE, 1 << 20, None) == \
        E["QLORA_ERR_ALIGN"]
    assert L.qlora_quantize_nf4_dq(FAKE, 8, 128, 64, 256, ctypes.byref(w), FAKE, 1 << 20, None) == \
        E["QLORA_ERR_SHAPE"]
    assert L.qlora_quantize_nf4_dq(FAKE, 4, 128, 64, 256, ctypes.byref(w), None, 0, None) == \
        E["QLORA_ERR_WORKSPACE"]
    assert L.qlora_quantize_nf4_dq(FAKE, 4, 128, 64, 256, ctypes.byref(w), FAKE, 4, None) == \
        E["QLORA_ERR_WORKSPACE"]
    bad = _w(c2=0x30004)
    assert L.qlora_dequantize(ctypes.byref(bad), FAKE, None) == E["QLORA_ERR_ALIGN"]
    bad = _w(mu=0)
    assert L.qlora_dequantize(ctypes.byref(bad), FAKE, None) == E["QLORA_ERR_INVALID_ARG"]
    bad = _w(K=100)
    assert L.qlora_dequantize(ctypes.byref(bad), FAKE, None) == E["QLORA_ERR_SHAPE"]
    # linear: r out of range, alpha not finite, bad dtype, workspace too small
    args = lambda r, alpha, dt, ws: (ctypes.byref(w), FAKE, 16, FAKE, FAKE, r, alpha, FAKE, dt, None,
                                     FAKE, ws, None)
    assert L.qlora_linear_fwd(*args(0, 1.0, 0, 1 << 30)) == E["QLORA_ERR_INVALID_ARG"]
    assert L.qlora_linear_fwd(*args(257, 1.0, 0, 1 << 30)) == E["QLORA_ERR_INVALID_ARG"]
    assert L.qlora_linear_fwd(*args(8, float("nan"), 0, 1 << 30)) == E["QLORA_ERR_INVALID_ARG"]
    assert L.qlora_linear_fwd(*args(8, 1.0, 7, 1 << 30)) == E["QLORA_ERR_INVALID_ARG"]
    assert L.qlora_linear_fwd(*args(8, 1.0, 0, 1)) == E["QLORA_ERR_WORKSPACE"]
    assert L.qlora_linear_workspace_size(16, 4, 128, 8, ctypes.byref(sz)) == 0 and sz.value > 0
    assert L.qlora_linear_bwd(ctypes.byref(w), FAKE, FAKE, 0, FAKE, FAKE, 8, 1.0, None, None, 0, FAKE, FAKE,
                              FAKE, 1 << 30, None) == E["QLORA_ERR_SHAPE"]
    assert L.qlora_linear_bwd(ctypes.byref(w), FAKE, FAKE, 16, FAKE, FAKE, 8, 1.0, None, None, 0, None, FAKE,
                              FAKE, 1 << 30, None) == E["QLORA_ERR_INVALID_ARG"]
    assert L.qlora_launch_count() == launches_before


def test_int8_argument_errors_on_the_host(L):
    fake = ctypes.c_void_p(0x10000)             # aligned, never dereferenced: the checks come first
    odd = ctypes.c_void_p(0x10004)
    q, d = L.qlora_quantize_int8_absmax, L.qlora_dequantize_int8_absmax
    assert q(None, 64, 64, fake, fake, None) == 1                     # null W
    assert q(odd, 64, 64, fake, fake, None) == 3                      # misaligned
    assert q(fake, 64, 32, fake, fake, None) == 4                     # blocksize
    assert q(fake, 100, 64, fake, fake, None) == 2                    # n % blocksize
    assert q(fake, 0, 64, fake, fake, None) == 2                      # empty
    assert d(fake, fake, 128, 128, fake, 5, None) == 1                # out dtype
    assert d(fake, None, 128, 128, fake, 0, None) == 1                # null alpha
    assert d(fake, fake, 192, 128, fake, 0, None) == 2


def test_selftest_argument_errors_on_the_host(L):
    fake = ctypes.c_void_p(0x10000)
    assert L.qlora_selftest_bounded_wait(0, fake, None) == 1          # limit out of range
    assert L.qlora_selftest_bounded_wait(1000001, fake, None) == 1
    assert L.qlora_selftest_bounded_wait(1000, None, None) == 1       # null result
    assert L.qlora_selftest_bounded_wait(1000, ctypes.c_void_p(0x10004), None) == 3
