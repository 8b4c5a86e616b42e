"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each test ties an oracle function to something other than itself: values the
pages print (tests/golden), closed forms, invariants the pages state, library
routines for special cases, exact rational arithmetic or brute force.  A few
tests plant a plausible mistake in a copy of an oracle step (on the CPU) and
check that a pin catches it.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import nf4_oracle as o
import synthetic_inputs as si

Q = o.nf4_codebook()


# ---------------------------------------------------------------- inverse normal CDF

def test_phi_inv_two_implementations_agree():
    pos, neg = o.nf4_probabilities()
    ps = pos + neg + list(np.linspace(0.5, 0.999, 57)) + [0.975, 0.841344746068543]
    for p in ps:
        a, b = o.phi_inv_stdlib(p), o.phi_inv_bisect(p)
        assert abs(a - b) <= 1e-12 * max(1.0, abs(a)), (p, a, b)


def test_phi_inv_textbook_values():
    # Standard-normal table values: Phi^-1(0.975) = 1.959964, Phi(1) = 0.841345, Phi^-1(1/2) = 0.
    assert abs(o.phi_inv_bisect(0.975) - 1.959963984540054) < 1e-12
    assert abs(o.phi_cdf(1.0) - 0.8413447460685429) < 1e-15
    assert abs(o.phi_inv_bisect(0.5)) < 1e-15
    for p in (0.6, 0.9, 0.96770833):
        assert abs(o.phi_cdf(o.phi_inv_bisect(p)) - p) < 1e-15


# ---------------------------------------------------------------- NF4 codebook

def test_codebook_shape_zero_and_endpoints():
    # [SD] section 3: 16 grid points (k = 4), zero represented exactly; endpoints +-1.
    assert Q.dtype == np.float32 and Q.shape == (16,)
    assert np.all(np.diff(Q) > 0)
    assert Q[0] == -1.0 and Q[7] == 0.0 and Q[15] == 1.0
    assert (Q < 0).sum() == 7 and (Q > 0).sum() == 8


def test_codebook_values_match_the_printed_table():
    # The values written down independently of the oracle (tests/golden/nf4_codebook_values.txt).
    g = read_golden("nf4_codebook_values.txt")
    printed = np.array(g["values"], dtype=np.float64)
    assert printed.shape == (16,)
    assert np.max(np.abs(o.nf4_codebook_f64() - printed)) <= g["print_precision"] + 1e-12
    assert np.max(np.abs(Q.astype(np.float64) - printed)) <= g["print_precision"] + 2 ** -24


def test_planted_delta_and_spacing_mistakes_miss_the_printed_table():
    printed = np.array(read_golden("nf4_codebook_values.txt")["values"], dtype=np.float64)
    tol = read_golden("nf4_codebook_values.txt")["print_precision"]

    def book(delta, pos_div=8.0, neg_div=7.0):
        pos = [delta - j * (delta - 0.5) / pos_div for j in range(8)]
        neg = [delta - j * (delta - 0.5) / neg_div for j in range(7)]
        v = sorted([o.phi_inv_stdlib(p) for p in pos] + [-o.phi_inv_stdlib(p) for p in neg] + [0.0])
        return np.array(v) / max(v)

    assert np.max(np.abs(book(o.NF4_DELTA) - printed)) <= tol + 1e-12
    for wrong in (book(0.5 * ((1 - 1 / 31) + (1 - 1 / 32))), book(0.5 * ((1 - 1 / 30) + (1 - 1 / 33))),
                  book(1 - 1 / 30), book(o.NF4_DELTA, pos_div=7.0), book(o.NF4_DELTA, neg_div=8.0)):
        assert np.max(np.abs(wrong - printed)) > 100 * tol


def test_codebook_equal_probability_mass_per_half():
    # [SD] section 3: each grid point covers the same probability mass of N(0,1).
    q64 = o.nf4_codebook_f64()
    top = o.phi_inv_stdlib(o.NF4_DELTA)
    p_pos = [o.phi_cdf(v * top) for v in q64[8:]]            # ascending, 8 values
    p_neg = [o.phi_cdf(-v * top) for v in q64[:7][::-1]]     # mirrored, 7 values
    for ps, count in ((p_pos, 8), (p_neg, 7)):
        steps = np.diff(ps)
        assert np.allclose(steps, steps[0], rtol=1e-9, atol=1e-13)
        # the steps partition (1/2, delta] into `count` equal parts
        assert abs((ps[-1] - 0.5) - count * steps[0]) < 1e-12 or abs(ps[0] - 0.5 - steps[0]) < 1e-12


def test_codebook_finer_near_zero():
    # [QR] section 4.1 and [SD] section 3: finer grid near 0, coarser in the tails.
    gaps_pos = np.diff(Q[7:])
    gaps_neg = np.diff(Q[:8])[::-1]
    assert np.all(np.diff(gaps_pos) > 0)
    assert np.all(np.diff(gaps_neg) > 0)


def test_codebook_independent_of_phi_inv_routine():
    assert np.array_equal(o.nf4_codebook(o.phi_inv_stdlib).view(np.uint32),
                          o.nf4_codebook(o.phi_inv_bisect).view(np.uint32))


def _blockwise_mse(w, q):
    c1 = o.block_absmax(w, 64).astype(np.float32)
    x = o.normalize_blocks(w, c1)
    idx = o.nearest_code(x, q)
    what = q[idx].astype(np.float64) * np.repeat(c1, 64)
    return float(np.mean((w.ravel().astype(np.float64) - what) ** 2))


def test_nf4_beats_uniform_int4_on_gaussian_weights():
    # [SD] section 4 (2) and [Q103]: NF4 has lower E||W - W_hat||^2 than a uniform
    # 4-bit grid on normally distributed weights (same blockwise absmax scaling).
    w = o.bf16_bits_to_f32(si.bf16_bits(si.normal_bf16((256, 1024), 0.02, 0, "pin", "mse")))
    assert _blockwise_mse(w, Q) < 0.85 * _blockwise_mse(w, o.uniform4_codebook())


def test_uniform4_grid_is_even_with_end_points():
    # reading R10: 16 evenly spaced values on [-1, 1]
    u = o.uniform4_codebook().astype(np.float64)
    assert u[0] == -1.0 and u[-1] == 1.0 and u.size == 16
    assert np.all(np.diff(u) > 0)
    assert np.allclose(np.diff(u), 2.0 / 15.0, rtol=0, atol=2 ** -22)
    assert np.allclose(u, -u[::-1], rtol=0, atol=2 ** -23)
    assert not np.any(u == 0.0)                       # the uniform grid has no exact zero, NF4 does


def test_error_study_nf4_beats_uniform_and_double_quantization_is_cheap():
    # [SD] section 4 (2): E||W - W_hat||^2 of NF4 is below that of a uniform 4-bit grid on
    # normal weights; section 3 part 2: double quantization saves 0.37 bits/param at a small cost.
    # Whole pipeline (absmax blocks, nearest code, bf16 rounding), relative squared error in fp64.
    errs = {}
    for dist in ("normal", "t5_outliers"):
        bits = si.bf16_bits(si.custom_linear(256, 1024, 1, 1, seed=3, sigma=0.02, dist=dist)[0])
        for name, q in (("nf4", Q), ("uniform4", o.uniform4_codebook())):
            qw = o.quantize_nf4_dq(bits, q=q)
            dq = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], qw["N"], qw["K"], q=q)
            single = o.dequantize_single(qw["codes"], qw["c1"], qw["N"], qw["K"], q=q)
            errs[dist, name, "dq"] = o.relative_sq_error(bits, dq)
            errs[dist, name, "single"] = o.relative_sq_error(bits, single)
    assert errs["normal", "nf4", "single"] < 0.9 * errs["normal", "uniform4", "single"]
    assert errs["t5_outliers", "nf4", "single"] < 0.6 * errs["t5_outliers", "uniform4", "single"]
    for dist in ("normal", "t5_outliers"):
        ratio = errs[dist, "nf4", "dq"] / errs[dist, "nf4", "single"]
        assert 0.99 < ratio < 1.02, (dist, ratio)


def test_relative_error_closed_forms_and_single_level_consistency():
    bits = si.bf16_bits(si.custom_linear(64, 128, 1, 1, seed=5)[0])
    assert o.relative_sq_error(bits, bits) == 0.0
    assert o.relative_sq_error(bits, np.zeros_like(bits)) == 1.0
    # with c1 set to the rebuilt c1' the single-level dequant is the double-quantized one
    qw = o.quantize_nf4_dq(bits)
    c1p = o.dq_constants(qw["c1_codes"], qw["c2"], qw["mu"])
    assert np.array_equal(o.dequantize_single(qw["codes"], c1p, 64, 128),
                          o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 64, 128))


def test_planted_codebook_mistakes_are_caught():
    # A codebook with the pages' literal symmetric midpoints (clipped ends) has no zero.
    lit = [0.5 * (o.phi_inv_stdlib(max(i / 16, 1e-3)) + o.phi_inv_stdlib(min((i + 1) / 16, 1 - 1e-3)))
           for i in range(16)]
    lit = np.array(lit) / max(abs(v) for v in lit)
    assert not np.any(lit == 0.0)
    # Evenly spaced positive half (the uniform grid) fails the equal-mass pin.
    u = o.uniform4_codebook().astype(np.float64)
    ps = [o.phi_cdf(v * 1.85) for v in u[8:]]
    assert not np.allclose(np.diff(ps), np.diff(ps)[0], rtol=1e-3)


# ---------------------------------------------------------------- bf16 / E4M3 encodings

def test_bf16_encoder_matches_torch():
    g = np.random.default_rng(1)
    x = np.concatenate([
        g.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (g.standard_normal(5000) * 1e-39).astype(np.float32),                     # subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.4e38, -3.4e38, np.inf, -np.inf], np.float32),
    ])
    # exact ties: bf16 value plus half an ulp, for both parities of the kept bit
    base = g.integers(0x3000, 0x4F00, 4000).astype(np.uint32) << 16
    ties = (base | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, (ties.view(np.uint32) + 1).view(np.float32),
                        (ties.view(np.uint32) - 1).view(np.float32)])
    ours = o.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_e4m3_hand_points():
    path = "e4m3_points.txt"
    import os
    from conftest import ROOT
    with open(os.path.join(ROOT, "tests", "golden", path)) as f:
        rows = [ln.split("#")[0].split() for ln in f if ln.split("#")[0].strip()]
    for expr, code in rows:
        v = np.float32(eval(expr, {"__builtins__": {}}))
        assert int(o.e4m3_encode(np.array([v]))[0]) == int(code, 16), expr


def test_e4m3_encoder_matches_torch_at_all_boundaries():
    vals = np.array([o.e4m3_value(c) for c in range(0x7F)], dtype=np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)        # exact in fp32
    pts = np.concatenate([vals.astype(np.float32), mids,
                          np.nextafter(mids, np.float32(np.inf)),
                          np.nextafter(mids, np.float32(-np.inf))])
    pts = np.concatenate([pts, -pts])
    g = np.random.default_rng(2)
    pts = np.concatenate([pts, g.uniform(-1, 1, 50000).astype(np.float32),
                          g.uniform(-448, 448, 20000).astype(np.float32)])
    ours = o.e4m3_encode(pts)
    ref = torch.from_numpy(pts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    # decode is exact and inverts encode on every finite code
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(o.e4m3_encode(o.e4m3_decode(codes)), codes)
    assert np.array_equal(o.e4m3_decode(codes),
                          torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy())


def test_e4m3_saturates():
    assert int(o.e4m3_encode(np.array([1e6], np.float32))[0]) == 0x7E
    assert int(o.e4m3_encode(np.array([-500.0], np.float32))[0]) == 0xFE


# ---------------------------------------------------------------- nearest code

def test_nearest_code_matches_exact_rational_argmin():
    q64 = Q.astype(np.float64)
    mids = ((q64[:-1] + q64[1:]) / 2)
    cand = []
    for m in mids:
        f = np.float32(m)                          # nearest fp32 to the midpoint
        cand += [f, np.nextafter(f, np.float32(2)), np.nextafter(f, np.float32(-2))]
    g = np.random.default_rng(3)
    cand += list(g.uniform(-1, 1, 3000).astype(np.float32))
    cand += list(Q) + [np.float32(0.0), np.float32(-0.0), np.float32(1e-30), np.float32(-1e-30)]
    x = np.array(cand, dtype=np.float32)
    got = o.nearest_code(x, Q)
    want = np.array([o.exact_nearest_code(v, Q) for v in x])
    assert np.array_equal(got, want)


def test_nearest_code_exact_at_denormals_for_a_grid_without_zero():
    # the uniform grid has a code pair +-q around 0: a denormal x > 0 is nearer to +q
    U = o.uniform4_codebook()
    tiny = np.array([1e-45, -1e-45, 1e-38, -1e-38, 1e-30, -1e-30, 0.0, -0.0], dtype=np.float32)
    g = np.random.default_rng(4)
    x = np.concatenate([tiny, g.uniform(-1, 1, 2000).astype(np.float32), U])
    want = np.array([o.exact_nearest_code(v, U) for v in x])
    assert np.array_equal(o.nearest_code(x, U), want)


def test_nearest_code_tie_goes_to_lower_index():
    # Build a codebook whose neighbour midpoints are exact fp32 numbers: ties are real.
    q = np.array([-1.0, -0.5, 0.0, 0.25, 1.0], dtype=np.float32)
    x = np.array([-0.75, -0.25, 0.125, 0.625], dtype=np.float32)
    assert list(o.nearest_code(x, q)) == [0, 1, 2, 3]


def test_planted_tie_rule_mistake_is_caught():
    q = np.array([-1.0, -0.5, 0.0, 0.25, 1.0], dtype=np.float32)
    x = np.array([-0.75, -0.25, 0.125, 0.625], dtype=np.float32)
    d = np.abs(x[:, None].astype(np.float64) - q[None, :])
    upper = d.shape[1] - 1 - np.argmin(d[:, ::-1], axis=1)      # ties to the upper index
    assert list(upper) != [o.exact_nearest_code(v, q) for v in x]


# ---------------------------------------------------------------- quantize invariants

def _tiny():
    W = si.weight("tiny", 0)
    return si.bf16_bits(W), o.quantize_nf4_dq(si.bf16_bits(W))


def test_c1_is_blockwise_absmax_and_absmax_maps_to_an_end_code():
    bits, qw = _tiny()
    w = o.bf16_bits_to_f32(bits).reshape(-1, 64)
    assert np.array_equal(qw["c1"], np.abs(w).max(axis=1))
    idx = qw["code_idx"].reshape(-1, 64)
    amax_pos = np.abs(w).argmax(axis=1)
    ends = idx[np.arange(idx.shape[0]), amax_pos]
    assert np.all((ends == 0) | (ends == 15))


def test_packing_hand_example():
    assert list(o.pack_nibbles(np.array([1, 2, 15, 0]))) == [0x12, 0xF0]
    assert list(o.unpack_nibbles(np.array([0x12, 0xF0], np.uint8))) == [1, 2, 15, 0]


def test_sign_is_preserved_and_zero_maps_to_zero():
    for wl in ("tiny", "block65b"):
        W = si.weight("tiny", 0) if wl == "tiny" else si.custom_linear(128, 512, 1, 8, 5, dist="t5")[0]
        bits = si.bf16_bits(W)
        qw = o.quantize_nf4_dq(bits)
        c1p = o.dq_constants(qw["c1_codes"], qw["c2"], qw["mu"])
        assert np.all(c1p > 0)
        Wh = o.bf16_bits_to_f32(o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], *bits.shape))
        w = o.bf16_bits_to_f32(bits)
        assert np.all((np.sign(Wh) == np.sign(w)) | (Wh == 0))
        assert np.all(Wh[w == 0] == 0)
        # |W_hat| <= bf16(c1') of its block
        bound = o.bf16_bits_to_f32(o.f32_to_bf16_bits(c1p))
        assert np.all(np.abs(Wh).reshape(-1, 64) <= bound[:, None])


def test_all_zero_block():
    bits = np.zeros((2, 128), np.uint16)
    w = si.bf16_bits(si.normal_bf16((2, 128), 0.02, 0, "pin", "z"))
    bits[1] = w[1]                               # row 1 nonzero, row 0 two all-zero blocks
    qw = o.quantize_nf4_dq(bits)
    assert np.all(qw["code_idx"][:128] == 7)
    Wh = o.bf16_bits_to_f32(o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 2, 128))
    assert np.all(Wh[0] == 0)


def test_codebook_valued_blocks_round_trip_exactly():
    # Every block holds q_i * c with c a power of two and both end codes present, so all
    # block constants are equal: mu = c, the centred constants are 0, c2 = 0 and c1' = c.
    g = np.random.default_rng(4)
    c = np.float32(2.0 ** -6)
    idx = g.integers(0, 16, size=(8, 256)).astype(np.uint8)
    idx[:, ::64] = 0
    idx[:, 1::64] = 15
    w = o.f32_to_bf16_bits((Q[idx] * c).astype(np.float32))
    qw = o.quantize_nf4_dq(w)
    assert qw["mu"] == c and np.all(qw["c2"] == 0)
    assert np.array_equal(qw["code_idx"].reshape(8, 256), idx)
    Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 8, 256)
    assert np.array_equal(Wh, w)


def test_quantize_dequantize_is_idempotent_on_codes():
    for W in (si.weight("tiny", 0), si.custom_linear(64, 1024, 1, 8, 7, dist="t5")[0]):
        bits = si.bf16_bits(W)
        qw = o.quantize_nf4_dq(bits)
        Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], *bits.shape)
        qw2 = o.quantize_nf4_dq(Wh)
        assert np.array_equal(qw2["codes"], qw["codes"])


def test_dequantize_rows_matches_full():
    bits, qw = _tiny()
    full = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 256, 256)
    rows = np.array([0, 5, 77, 255])
    assert np.array_equal(o.dequantize_rows(qw, rows), full[rows])


def test_argument_errors():
    with pytest.raises(o.OracleShapeError):
        o.quantize_nf4_dq(np.zeros((4, 96), np.uint16))
    with pytest.raises(o.OracleUnsupported):
        o.quantize_nf4_dq(np.zeros((4, 128), np.uint16), blocksize=32)


# ---------------------------------------------------------------- double quantization

def test_pairwise_tree_order():
    # Sequential summation gives 1 here; the fixed pairwise tree gives 0.
    assert o.pairwise_tree_sum([1e16, 1.0, -1e16, 1.0]) == 0.0
    assert ((1e16 + 1.0) + -1e16) + 1.0 == 1.0
    # Exact on small integers and padding with zeros is harmless.
    assert o.pairwise_tree_sum(np.arange(1000)) == 999 * 1000 / 2
    g = np.random.default_rng(5)
    v = g.random(3001)
    assert abs(o.pairwise_tree_sum(v) - math.fsum(v)) < 1e-12


def test_dq_constant_c1_and_mean():
    c1 = np.full(512, 0.03125, np.float32)
    codes, c2, mu = o.double_quantize(c1)
    assert mu == np.float32(0.03125) and np.all(c2 == 0) and np.all(codes == 0)
    assert np.all(o.dq_constants(codes, c2, mu) == c1)


def test_dq_error_bound_and_centring():
    for W in (si.weight("tiny", 0), si.custom_linear(256, 4096, 1, 8, 9, dist="t5")[0]):
        qw = o.quantize_nf4_dq(si.bf16_bits(W))
        c1 = qw["c1"]
        x2 = o.e4m3_decode(qw["c1_codes"]).astype(np.float64)
        c2e = np.repeat(qw["c2"], 256)[:c1.size].astype(np.float64)
        c1p = o.dq_constants(qw["c1_codes"], qw["c2"], qw["mu"]).astype(np.float64)
        # E4M3 half-ulp: relative 2^-4 on normals, absolute 2^-10 in the subnormal range,
        # plus the two fp32 roundings of the rebuild.
        bound = c2e * np.maximum(2.0 ** -4 * np.abs(x2), 2.0 ** -10) + 4 * np.spacing(c1.astype(np.float32))
        assert np.all(np.abs(c1p - c1) <= bound)
        # mean of the centred constants is ~0 relative to their spread
        d = c1.astype(np.float64) - float(qw["mu"])
        assert abs(d.mean()) < 1e-5 * np.abs(d).max() + 1e-12


def test_planted_missing_mean_is_caught():
    W = si.weight("tiny", 0)
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    wrong = o.dq_constants(qw["c1_codes"], qw["c2"], 0.0)      # forgets to add mu back
    assert np.max(np.abs(wrong - qw["c1"])) > 0.5 * qw["c1"].min()


# ---------------------------------------------------------------- footprint and closed forms

def test_footprint_matches_pages():
    g = read_golden("dq_footprint.txt")
    N, K = 8192, 8192
    bits = o.constant_bits_per_param(N, K)
    assert bits == 8 / 64 + 32 / (64 * 256) == 0.126953125
    assert abs(bits - g["bits_with_dq_printed"]) <= g["bits_with_dq_print_precision"]
    nodq = o.constant_bits_per_param(N, K, double_quant=False)
    assert nodq == g["bits_without_dq"]
    saving = nodq - bits
    assert abs(saving - g["saving_printed"]) <= g["saving_print_precision"]
    gb = saving * g["params_65b"] / 8 / 1e9
    assert abs(gb - g["saving_gb_65b_printed"]) <= g["saving_gb_tolerance"] * g["saving_gb_65b_printed"]
    # the oracle's stored buffers have exactly these sizes
    qw = o.quantize_nf4_dq(si.bf16_bits(si.normal_bf16((64, 4096), 0.02, 0, "pin", "fp")))
    sb = o.stored_bytes(64, 4096)
    assert qw["codes"].nbytes == sb["codes"] and qw["c1_codes"].nbytes == sb["c1_codes"]
    assert qw["c2"].nbytes == sb["c2"]


def test_memory_closed_forms():
    g = read_golden("memory_closed_forms.txt")
    assert g["params_7b"] * 2 / 1e9 == g["bf16_gb_7b"]
    assert g["params_7b"] * (o.stored_bytes(1, 64)["codes"] / 64) / 1e9 == g["nf4_gb_7b"]
    assert g["params_65b"] * 2 / 1e9 == g["bf16_gb_65b"]
    assert 32 / 4 == g["fp32_over_int4"]
    assert o.stored_bytes(1, 64)["codes"] / 64 == g["int4_bytes_per_weight"]


def test_int8_worked_example():
    g = read_golden("int8_absmax_example.txt")
    alpha, codes, xhat = o.absmax_int8(g["input"])
    assert abs(alpha - g["alpha_approx"]) <= g["alpha_tolerance"]
    assert round(alpha) == g["alpha_rounded"]
    assert codes[0] == g["code_of_1.2"]
    assert codes[2] == g["peak_code"]
    assert abs(codes[0] / alpha - g["dequant_of_28_approx"]) <= g["dequant_tolerance"]


def _int8_block(vals, blocksize=64):
    x = np.zeros(blocksize, np.float32)
    x[:len(vals)] = vals
    return o.f32_to_bf16_bits(x)


def test_int8_blocks_worked_example():
    # the page's vector (1.2, -0.5, 5.4) as one block of 64 (the rest zeros), in bf16
    g = read_golden("int8_absmax_example.txt")
    codes, alpha = o.quantize_int8_blocks(_int8_block(g["input"]), 64)
    # (5.4 is 5.40625 in bf16, so alpha is 23.49 here: the page's "rounds to 24" holds for the
    # exact 5.4 only and is pinned by test_int8_worked_example)
    assert abs(float(alpha[0]) - g["alpha_approx"]) <= g["alpha_tolerance"]
    assert codes[0] == g["code_of_1.2"] and codes[2] == g["peak_code"] and codes[1] == -12
    assert np.all(codes[3:] == 0)
    xh = o.dequantize_int8_blocks(codes, alpha, 64)
    assert abs(float(xh[0]) - g["dequant_of_28_approx"]) <= g["dequant_tolerance"]


def test_int8_blocks_round_half_away():
    # amax = 127 makes alpha exactly 1, so x * alpha = x: exact halves must round away from zero
    codes, alpha = o.quantize_int8_blocks(_int8_block([127.0, 2.5, -2.5, 0.5, -0.5, 1.5, -1.5, 126.5]), 64)
    assert float(alpha[0]) == 1.0
    assert list(codes[:8]) == [127, 3, -3, 1, -1, 2, -2, 127]
    assert np.array_equal(o.dequantize_int8_blocks(codes, alpha, 64)[:8], codes[:8].astype(np.float32))


def test_int8_blocks_agree_with_the_fp64_example_rule():
    # per block, the fp32 rule gives the fp64 single-block rule's codes except where the
    # fp64 product sits within 1e-4 of a half-integer (fp32 rounding may then flip it by one)
    rng = np.random.default_rng(5)
    for bs in (64, 128, 256):
        x = (rng.standard_t(5, size=bs * 6) * 0.02).astype(np.float32)
        bits = o.f32_to_bf16_bits(x)
        codes, alpha = o.quantize_int8_blocks(bits, bs)
        xb = o.bf16_bits_to_f32(bits).reshape(-1, bs)
        for b in range(xb.shape[0]):
            a64, c64, _ = o.absmax_int8(xb[b])
            assert abs(float(alpha[b]) - a64) <= 2 ** -23 * a64
            s64 = xb[b].astype(np.float64) * a64
            near_tie = np.abs(np.abs(s64) - np.floor(np.abs(s64)) - 0.5) < 1e-4
            blk = codes[b * bs:(b + 1) * bs].astype(np.int64)
            assert np.all((blk == c64) | (near_tie & (np.abs(blk - c64) <= 1)))


def test_int8_blocks_invariants_and_error_bound():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(64 * 40) * 0.02).astype(np.float32)
    x[::97] *= 10.0                                         # outliers
    bits = o.f32_to_bf16_bits(x)
    codes, alpha = o.quantize_int8_blocks(bits, 64)
    xb = o.bf16_bits_to_f32(bits).reshape(-1, 64).astype(np.float64)
    cb = codes.reshape(-1, 64).astype(np.int64)
    assert np.all(np.abs(cb) <= 127)
    peak = np.argmax(np.abs(xb), axis=1)
    assert np.all(np.abs(cb[np.arange(len(peak)), peak]) == 127)           # the peak maps to 127
    assert np.all((cb == 0) | (np.sign(cb) == np.sign(xb)))                # sign kept
    xh = o.dequantize_int8_blocks(codes, alpha, 64).reshape(-1, 64).astype(np.float64)
    a = alpha.astype(np.float64)[:, None]
    # half a step from rounding, the fp32 product's and quotient's roundings on top
    bound = (0.5 + 127 * 2.0 ** -23) / a + 2.0 ** -23 * np.abs(xh)
    assert np.all(np.abs(xh - xb) <= bound)


def test_int8_blocks_degenerate():
    tiny = float(o.bf16_bits_to_f32(np.array([0x0001], np.uint16))[0])   # smallest bf16 subnormal
    bits = np.concatenate([_int8_block([]), _int8_block([tiny, -tiny, 0.0]), _int8_block([3.0, -1.5])])
    codes, alpha = o.quantize_int8_blocks(bits, 64)
    assert alpha[0] == 0 and np.all(codes[:64] == 0)                       # zero block
    assert np.isinf(alpha[1]) and list(codes[64:67]) == [127, -127, 0]     # 127 / amax overflows
    assert np.all(codes[67:128] == 0)
    assert list(codes[128:130]) == [127, -64]                              # -1.5 * 127/3 = -63.5 -> -64
    xh = o.dequantize_int8_blocks(codes, alpha, 64)
    assert np.all(xh[:128] == 0)
    assert np.signbit(xh[65]) and not np.signbit(xh[64])                   # -127 / inf = -0


def test_int8_blocks_reject():
    with pytest.raises(o.OracleShapeError):
        o.quantize_int8_blocks(_int8_block([1.0], 64), 32)
    with pytest.raises(o.OracleShapeError):
        o.quantize_int8_blocks(_int8_block([1.0], 64)[:60], 64)
    bad = _int8_block([1.0])
    bad[5] = 0x7F80                                                        # +Inf
    with pytest.raises(o.OracleNonFiniteError):
        o.quantize_int8_blocks(bad, 64)


# ---------------------------------------------------------------- the linear layer

def _small_linear(M=3, N=5, K=64, r=2, seed=11):
    W, X, A, B, dY = si.custom_linear(N, K, M, r, seed)
    bits = si.bf16_bits(W)
    qw = o.quantize_nf4_dq(bits)
    Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], N, K)
    return si.bf16_bits(X), Wh, si.bf16_bits(A), si.bf16_bits(B), si.bf16_bits(dY)


def test_forward_matches_brute_force_loops():
    X, Wh, A, B, _ = _small_linear()
    Y, U = o.linear_forward(X, Wh, A, B, alpha=4.0, r=2)
    Yb = o.brute_force_forward(X, Wh, A, B, 4.0, 2)
    assert np.allclose(Y, Yb, rtol=1e-13, atol=1e-15)


def _loss(X, Wh, A, B, dY, alpha, r):
    Y, _ = o.linear_forward(X, Wh, A, B, alpha, r)
    return float(np.sum(o._f64(dY) * Y))


def _fd_directional(X, Wh, A, B, dY, alpha, r, name, E, h=1e-3):
    """Central difference of <dY, Y> along E in the named input (exact up to rounding:
    the loss is linear in each of X, A, B separately)."""
    args = {"X": o._f64(X), "A": o._f64(A), "B": o._f64(B)}
    plus = dict(args); plus[name] = args[name] + h * E
    minus = dict(args); minus[name] = args[name] - h * E
    return (_loss(plus["X"], Wh, plus["A"], plus["B"], dY, alpha, r)
            - _loss(minus["X"], Wh, minus["A"], minus["B"], dY, alpha, r)) / (2 * h)


def _grad_passes_fd(X, Wh, A, B, dY, alpha, r, name, grad, seed=12):
    rng = np.random.default_rng(seed)
    E = rng.standard_normal(grad.shape)
    fd = _fd_directional(X, Wh, A, B, dY, alpha, r, name, E)
    return abs(fd - np.sum(grad * E)) <= 1e-8 * (abs(fd) + 1.0)


def test_backward_matches_finite_differences():
    X, Wh, A, B, dY = _small_linear(M=4, N=6, K=128, r=3)
    alpha, r = 6.0, 3
    g = o.linear_backward(X, dY, Wh, A, B, alpha, r)
    for name, key in (("X", "dX"), ("A", "dA"), ("B", "dB")):
        assert _grad_passes_fd(X, Wh, A, B, dY, alpha, r, name, g[key]), name


def test_planted_backward_mistakes_are_caught():
    X, Wh, A, B, dY = _small_linear(M=4, N=6, K=128, r=3)
    alpha, r = 6.0, 3
    Xf, Af, Bf, dYf, Wf = (o._f64(v) for v in (X, A, B, dY, Wh))
    s = alpha / r
    wrong = {
        "dB scaled by r/alpha": ("B", (r / alpha) * (dYf.T @ (Xf @ Af.T))),
        "dX without s on the LoRA term": ("X", dYf @ Wf + (dYf @ Bf) @ Af),
        "dX with the frozen-weight term negated": ("X", -(dYf @ Wf) + s * (dYf @ Bf) @ Af),
        "dA with the sign flipped": ("A", -(s * (dYf @ Bf)).T @ Xf),
    }
    for label, (name, grad) in wrong.items():
        assert not _grad_passes_fd(X, Wh, A, B, dY, alpha, r, name, grad), label


def test_adjoint_identity_and_degenerate_cases():
    X, Wh, A, B, dY = _small_linear(M=5, N=7, K=192, r=4)
    Xf, Wf, dYf = o._f64(X), o._f64(Wh), o._f64(dY)
    lhs = np.sum(dYf * (Xf @ Wf.T))
    rhs = np.sum((dYf @ Wf) * Xf)
    assert abs(lhs - rhs) <= 1e-12 * abs(lhs)
    # alpha = 0: plain matmul, no LoRA gradient signal
    Y0, _ = o.linear_forward(X, Wh, A, B, 0.0, 4)
    assert np.allclose(Y0, Xf @ Wf.T, rtol=0, atol=0)
    g0 = o.linear_backward(X, dY, Wh, A, B, 0.0, 4)
    assert np.all(g0["dA"] == 0) and np.all(g0["dB"] == 0)
    # B = 0: Y = X W^T and dA = 0
    Bz = np.zeros_like(B)
    Yb, _ = o.linear_forward(X, Wh, A, Bz, 8.0, 4)
    assert np.array_equal(Yb, Xf @ Wf.T)
    assert np.all(o.linear_backward(X, dY, Wh, A, Bz, 8.0, 4)["dA"] == 0)


def test_row_subsets_match_full():
    X, Wh, A, B, dY = _small_linear(M=6, N=5, K=64, r=2)
    rows = np.array([1, 4])
    assert np.allclose(o.forward_rows(X, Wh, A, B, 4.0, 2, rows),
                       o.linear_forward(X, Wh, A, B, 4.0, 2)[0][rows], rtol=1e-14, atol=0)
    assert np.allclose(o.backward_dx_rows(dY, Wh, A, B, 4.0, 2, rows),
                       o.linear_backward(X, dY, Wh, A, B, 4.0, 2)["dX"][rows], rtol=1e-14, atol=0)


def test_lora_gradients_equal_the_full_backward():
    X, Wh, A, B, dY = _small_linear(M=7, N=5, K=128, r=3)
    full = o.linear_backward(X, dY, Wh, A, B, 6.0, 3)
    part = o.lora_gradients(X, dY, A, B, 6.0, 3)
    for k in ("dA", "dB"):
        assert np.allclose(part[k], full[k], rtol=1e-13, atol=1e-15)


def test_row_and_column_samplers_match_full_quantize():
    W = si.custom_linear(24, 512, 1, 8, 31)[0]
    bits = si.bf16_bits(W)
    full = o.quantize_nf4_dq(bits)
    rows = np.array([0, 7, 23])
    part = o.quantize_rows(bits, rows)
    assert np.array_equal(part["codes_rows"], full["codes"].reshape(24, 256)[rows])
    for k in ("c1_codes", "c2", "mu"):
        assert np.array_equal(part[k], full[k])
    Wh = o.dequantize(full["codes"], full["c1_codes"], full["c2"], full["mu"], 24, 512)
    cols = np.array([0, 1, 63, 64, 511])
    assert np.array_equal(o.dequantize_cols(full, cols), Wh[:, cols])


# ---------------------------------------------------------------- merge and requantize

def _nearest_bf16_exact(v: float) -> int:
    """Brute force: the bf16 pattern nearest to v (exact rationals; ties to the even pattern)."""
    from fractions import Fraction
    fv = Fraction(v)
    b0 = int(o.f32_to_bf16_bits(np.array([v], np.float32))[0])   # a candidate within one step
    best = None
    for b in (b0 - 1, b0, b0 + 1):
        if b & 0x7F80 == 0x7F80:
            continue
        val = Fraction(float(o.bf16_bits_to_f32(np.array([b], np.uint16))[0]))
        key = (abs(val - fv), b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return best[1]


def test_f64_to_bf16_rounds_once():
    g = np.random.default_rng(8)
    x = np.concatenate([g.normal(0, 0.02, 3000), g.normal(0, 1e-38, 200), [0.0, -0.0, 1.0, -3.5]])
    # values just above a bf16 midpoint by less than half an fp32 ulp: fp32 first would land on the
    # midpoint and round to even (down); the direct rounding must go up
    mids = [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]
    x = np.concatenate([x, [m + 2.0 ** -30 for m in mids], [m - 2.0 ** -30 for m in mids], mids])
    got = o.f64_to_bf16_bits(x)
    want = np.array([_nearest_bf16_exact(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, want)
    assert o.f64_to_bf16_bits(np.array([1.0 + 2.0 ** -8 + 2.0 ** -30]))[0] == 0x3F81


def test_merge_definition_and_degenerate_cases():
    W, X, A, B, dY = si.custom_linear(7, 128, 1, 3, seed=9)
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 7, 128)
    bA, bB = si.bf16_bits(A), si.bf16_bits(B)
    # B = 0: the merged weight is the dequantized weight, bit for bit
    assert np.array_equal(o.merge_lora(Wh, bA, np.zeros_like(bB), 6.0, 3), Wh)
    # brute-force loops over the definition
    Whf, Af, Bf = o._f64(Wh), o._f64(bA), o._f64(bB)
    brute = np.zeros((7, 128))
    for n in range(7):
        for k in range(128):
            brute[n, k] = Whf[n, k] + 2.0 * sum(Bf[n, j] * Af[j, k] for j in range(3))
    assert np.array_equal(o.merge_lora(Wh, bA, bB, 6.0, 3), o.f64_to_bf16_bits(brute))


# ---------------------------------------------------------------- one base, many adapters

def test_multi_adapter_forward_reduces_to_single_and_base():
    W, X, A, B, dY = si.custom_linear(24, 128, 5, 4, seed=13)
    qw = o.quantize_nf4_dq(si.bf16_bits(W))
    Wh = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 24, 128)
    bX, bA, bB = si.bf16_bits(X), si.bf16_bits(A), si.bf16_bits(B)
    A2 = np.stack([np.zeros_like(bA), bA]).astype(np.uint16)
    B2 = np.stack([np.zeros_like(bB), bB]).astype(np.uint16)
    Y1, U1 = o.linear_forward(bX, Wh, bA, bB, 8.0, 4)
    Ym, Um = o.linear_forward_multi(bX, Wh, A2, B2, [1] * 5, 8.0, 4)
    assert np.array_equal(Ym, Y1) and np.array_equal(Um, U1)            # every token on one adapter
    Yb, Ub = o.linear_forward_multi(bX, Wh, A2, B2, [-1] * 5, 8.0, 4)
    assert np.array_equal(Yb, o._f64(bX) @ o._f64(Wh).T) and not Ub.any()  # no adapter: base only
    # mixed: each row equals the single-adapter result of its own adapter (brute force per row)
    idx = [1, -1, 0, 1, -1]
    Ymix, _ = o.linear_forward_multi(bX, Wh, A2, B2, idx, 8.0, 4)
    for m, a in enumerate(idx):
        ref = o.linear_forward(bX[m:m + 1], Wh, A2[max(a, 0)], B2[max(a, 0)], 8.0 if a >= 0 else 0.0, 4)[0]
        assert np.allclose(Ymix[m], ref[0], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- fp16 compute dtype

def test_fp16_rounding_matches_torch_and_rounds_once_from_fp64():
    g = np.random.default_rng(31)
    x = np.concatenate([g.normal(0, 1, 4000), g.normal(0, 1e-5, 500), [65504.0, 65519.0, 65520.0, -0.0, 6e-8]])
    x32 = x.astype(np.float32)
    assert np.array_equal(o.f32_to_f16_bits(x32),
                          torch.from_numpy(x32).to(torch.float16).view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(o.f16_bits_to_f32(o.f32_to_f16_bits(x32)),
                          torch.from_numpy(x32).to(torch.float16).float().numpy())
    # direct fp64 rounding: just above an fp16 midpoint by less than half an fp32 ulp goes up
    m = 1.0 + 2.0 ** -11
    assert o.f64_to_f16_bits(np.array([m + 2.0 ** -40]))[0] == 0x3C01
    assert o.f64_to_f16_bits(np.array([m]))[0] == 0x3C00                  # tie: to even
    y = g.normal(0, 0.3, 3000)
    assert np.array_equal(o.f64_to_f16_bits(y.astype(np.float32).astype(np.float64)),
                          o.f32_to_f16_bits(y.astype(np.float32)))        # fp32-exact inputs: same


def test_fp16_dequantize_is_the_fp16_rounding_of_the_same_products():
    bits = si.bf16_bits(si.custom_linear(16, 256, 1, 1, seed=17)[0])
    qw = o.quantize_nf4_dq(bits)
    h = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 16, 256, f16=True)
    b = o.dequantize(qw["codes"], qw["c1_codes"], qw["c2"], qw["mu"], 16, 256)
    hv, bv = o.f16_bits_to_f32(h).astype(np.float64), o.bf16_bits_to_f32(b).astype(np.float64)
    assert np.all(np.abs(hv - bv) <= np.abs(bv) * 2.0 ** -8)            # both round the same fp32 product
    assert np.all(np.sign(hv) == np.sign(bv))
