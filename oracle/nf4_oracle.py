"""Plain CPU oracle for the QLoRA quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check in the repository's
entry module and the CPU-baseline leg of the benchmark may import this module.
The CUDA library and its Python binding never import it, and it imports nothing
from them: the two implementations share no code, no table and no helper.

Everything here is written for a reader to check by eye against the pages.  It
is slow on purpose: NumPy element-wise steps, fp64 where the pages fix no
precision, and library matmuls as single steps.

Sources (web pages on QLoRA, cited by title and section)
--------------------------------------------------------
[SD]   airsota.com, "Science Depth M5-131: PEFT (LoRA / QLoRA / Prefix Tuning)".
       Section 3 "Mathematical Principles & Derivation" (Chinese text and the
       English derivation): NF4 quantile formula, absmax blocks of B=64, the
       nearest-code rule, Double Quantization to 8-bit floats with block 256,
       the 0.127 bits/param footprint.  Section 4 "Industrial Trade-offs" (1):
       on-the-fly dequantization W_hat = Dequant(W_NF4) * c1 in forward and
       backward; (2): NF4 beats uniform INT4 in E||W - W_hat||^2.
[QP]   offer.aigcbaba.com, "QLoRA 的原理是什么？4-bit 量化权重真的参与训练吗？".
       Section 7 (storage vs compute precision): 4-bit frozen weight ->
       dequantize to BF16 -> matmul, LoRA path added to the output; gradients
       reach only the LoRA parameters, never the 4-bit codes.
[QR]   ainexis.cn, walkthrough of "QLoRA: Efficient Finetuning of Quantized
       LLMs".  Section 4.4: backpropagate through the frozen 4-bit weights into
       the adapters.
[CH9]  mdooai.com, "Ch.09 QLoRA 与量化：缩得更小再微调".  Section "2. INT8
       量化" and "2. 量化怎么缩数字": the absmax INT8 worked example.
[Q103] agentalpha.top, "Q103: What is QLoRA, and how does it differ from LoRA".
       Follow-up 3: LoRA rank r and alpha (alpha usually 2r).

Readings where the pages are silent, garbled or inconsistent
------------------------------------------------------------
R1  Codebook.  [SD] prints q_i = (Phi^-1(i/16) + Phi^-1((i+1)/16)) / 2, whose
    end points are infinite, and says zero is made exact by an adjustment.
    Reading: the asymmetric construction of the QLoRA method, 8 positive
    quantiles Phi^-1(p) at p evenly spaced from delta towards 1/2 (1/2
    excluded), 7 negative ones mirrored the same way, and an exact 0, with
    delta = ((1 - 1/30) + (1 - 1/32)) / 2; sorted, divided by the largest,
    computed in fp64, rounded to fp32.  Index 0 = -1, 7 = 0, 15 = +1.
R2  Blocks of 64 run over the row-major flattening of W[N,K] (K % 64 == 0, so
    blocks never straddle rows).  x = fp32(w / c1); a block with c1 == 0 gives
    x = 0.
R3  Nearest code: argmin_i |x - q_i|, ties to the lower index.
R4  Packing: byte j holds element 2j in its high nibble, 2j+1 in its low one.
R5  Double Quantization: "8-bit FP" is OCP FP8 E4M3 (finite-only variant),
    round to nearest even with saturation.  c1 is centred first by one
    tensor-wide mean mu (fp64 sum over a fixed pairwise tree, then fp32), and
    each group of 256 centred constants is scaled by its absmax c2 (fp32).
    A short last group is allowed.
R6  Dequantization op order: c1' = fp32(fp32(v8 * c2) + mu), then
    W_hat = bf16_RN(fp32(q[code] * c1')).
R7  LoRA: Y = X W_hat^T + s (X A^T) B^T with s = alpha / r, A[r,K], B[N,r].
R8  The GEMM references are exact fp64 on the bit-exact W_hat and the bf16
    inputs; U = X A^T and dU = s dY B are never rounded.
R9  The INT8 example rounds half away from zero ("四舍五入").
R10 Quantizer variants ([SD] section 4 (2) compares NF4 with uniform INT4 by
    E||W - W_hat||^2): the uniform 4-bit grid is 16 evenly spaced values on
    [-1, 1] (linspace, fp64 then fp32), coded with the same absmax blocks and
    nearest-value rule; "double quantization off" keeps the fp32 block absmax
    c1 and dequantizes W_hat = bf16_RN(fp32(q[code] * c1)).  The error study
    measures sum (W_hat - W)^2 / sum W^2 in fp64.
R11 fp16 compute dtype ([QP] section 4: bf16 is the usual compute type, fp16
    where bf16 is poorly supported): W_hat = fp16_RN(fp32(q[code] * c1')),
    activations and adapters in fp16, the same fp32 accumulation.
R14 Blockwise INT8 ([CH9] section "2. INT8 量化" fixes the steps but not the
    precision or the block): blocks of 64, 128 or 256 consecutive elements of
    a bf16 tensor, fp32 arithmetic with round-to-nearest-even:
    alpha = fp32(127 / amax), code = round half away from zero (R9) of
    fp32(x * alpha), dequantized x_hat = fp32(code / alpha).  Degenerate
    blocks: amax = 0 gives alpha = 0, zero codes and x_hat = 0; amax below
    127 / FLT_MAX makes alpha = +inf, a zero element still codes to 0 and
    every other element to +-127 (clamp), and x_hat = code / inf = +-0.
"""
from __future__ import annotations

import math
from fractions import Fraction
from statistics import NormalDist

import numpy as np

BLOCKSIZE = 64          # [SD] Section 3: "normalized in blocks of size B=64"
BLOCKSIZE2 = 256        # [SD] Section 3: "secondary block size 256"

# Status names mirrored from the C ABI's error behaviour (the oracle raises).
class OracleShapeError(ValueError):
    pass


class OracleUnsupported(ValueError):
    pass


class OracleNonFiniteError(ValueError):
    pass


# ---------------------------------------------------------------------------
# Inverse normal CDF: two independent implementations
# ---------------------------------------------------------------------------

def phi_inv_stdlib(p: float) -> float:
    """Phi^-1(p) by Python's statistics.NormalDist (Wichura's AS241)."""
    return NormalDist().inv_cdf(p)


def phi_cdf(x: float) -> float:
    """Phi(x) = erfc(-x / sqrt(2)) / 2, the standard normal CDF."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def phi_inv_bisect(p: float) -> float:
    """Phi^-1(p) by bisection on Phi (math.erfc), to the last representable bit."""
    if not (0.0 < p < 1.0):
        raise ValueError("p must lie in (0, 1)")
    lo, hi = -40.0, 40.0
    for _ in range(400):
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if phi_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


# ---------------------------------------------------------------------------
# NF4 codebook ([SD] Section 3 (1); reading R1)
# ---------------------------------------------------------------------------

NF4_DELTA = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))


def nf4_probabilities():
    """The probabilities whose normal quantiles form the two halves (reading R1).

    Returns (positive_half, negative_half): 8 and 7 probabilities evenly spaced
    from NF4_DELTA towards 1/2, 1/2 itself excluded.
    """
    d = NF4_DELTA
    pos = [d - j * (d - 0.5) / 8.0 for j in range(8)]
    neg = [d - j * (d - 0.5) / 7.0 for j in range(7)]
    return pos, neg


def nf4_codebook_f64(phi_inv=phi_inv_stdlib) -> np.ndarray:
    """The 16 NF4 values in fp64 before rounding, ascending."""
    pos, neg = nf4_probabilities()
    values = [phi_inv(p) for p in pos] + [-phi_inv(p) for p in neg] + [0.0]
    values.sort()
    top = max(values)
    return np.array([v / top for v in values], dtype=np.float64)


def nf4_codebook(phi_inv=phi_inv_stdlib) -> np.ndarray:
    """The 16 NF4 code values as fp32, ascending: q[0] = -1, q[7] = 0, q[15] = +1."""
    return nf4_codebook_f64(phi_inv).astype(np.float32)


def uniform4_codebook() -> np.ndarray:
    """A uniform 16-level grid on [-1, 1]: the INT4-style baseline NF4 is compared with ([SD] 4 (2))."""
    return np.linspace(-1.0, 1.0, 16).astype(np.float32)


# ---------------------------------------------------------------------------
# bf16 and fp8 E4M3 encodings, written from the format definitions
# ---------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp32 values (the top half of an fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16, to nearest with ties to even; returns uint16 bits.

    The 16 dropped bits are rounded: add 0x7FFF plus the lowest kept bit, then
    truncate.  NaN stays NaN (quiet bit set); overflow rounds to infinity.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> 16) & 1
    rounded = (u + 0x7FFF + keep_lsb) >> 16
    is_nan = (u & 0x7FFFFFFF) > 0x7F800000
    rounded = np.where(is_nan, (u >> 16) | 0x40, rounded)
    return rounded.astype(np.uint16)


def e4m3_value(code: int) -> float:
    """Value of an FP8 E4M3 (finite-only) code: 1 sign, 4 exponent (bias 7), 3 mantissa bits."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3_POS = np.array([e4m3_value(c) for c in range(0x7F)], dtype=np.float64)  # codes 0..0x7E
E4M3_MAX = float(_E4M3_POS[-1])   # 448


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) -> fp32 values (exact)."""
    table = np.array([e4m3_value(c) for c in range(256)], dtype=np.float32)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """fp32 -> E4M3 code: nearest finite value, ties to the even code, saturating at +-448.

    The sign bit is copied from the input, so a small negative value that rounds
    to zero becomes the code 0x80 (negative zero).
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    hi = np.searchsorted(_E4M3_POS, a, side="left")          # first value >= a
    hi = np.clip(hi, 0, len(_E4M3_POS) - 1)
    lo = np.clip(hi - 1, 0, len(_E4M3_POS) - 1)
    d_hi = np.abs(_E4M3_POS[hi] - a)
    d_lo = np.abs(a - _E4M3_POS[lo])
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo)
    mag = np.where(a >= E4M3_MAX, 0x7E, mag)
    sign = np.signbit(x).astype(np.int64) << 7
    return (mag | sign).astype(np.uint8)


# ---------------------------------------------------------------------------
# Blockwise absmax helpers
# ---------------------------------------------------------------------------

def block_absmax(v: np.ndarray, block: int) -> np.ndarray:
    """max |v| over consecutive groups of `block` elements; the last group may be short."""
    v = np.abs(np.asarray(v).ravel())
    n = v.size
    starts = np.arange(0, n, block)
    return np.maximum.reduceat(v, starts)


# ---------------------------------------------------------------------------
# First-level NF4 quantization ([SD] Section 3 (1); readings R2-R4)
# ---------------------------------------------------------------------------

def nearest_code(x: np.ndarray, q: np.ndarray) -> np.ndarray:
    """argmin_i |x - q_i| over the ascending codebook, ties to the lower index (reading R3).

    For a sorted codebook the argmin is the number of neighbour midpoints
    m_j = (q_j + q_{j+1}) / 2 that lie strictly below x (x equal to a midpoint
    is a tie and stays with the lower code).  The midpoints of two fp32 values
    of close magnitude are exact in fp64, and so is every fp32 x, so the count
    is exact for every x, denormals included (fp64 differences |x - q_i| are
    not: for a denormal x both distances to a pair +-q round to the same value).
    """
    x = np.asarray(x, dtype=np.float32).ravel().astype(np.float64)
    qd = np.asarray(q, dtype=np.float64)
    assert np.all(np.diff(qd) > 0), "codebook must be ascending"
    mids = (qd[:-1] + qd[1:]) / 2.0
    assert np.array_equal(2.0 * mids - qd[:-1], qd[1:]), "midpoint not exact in fp64"
    return np.searchsorted(mids, x, side="left").astype(np.uint8)


def normalize_blocks(w: np.ndarray, c1: np.ndarray, block: int = BLOCKSIZE) -> np.ndarray:
    """x = fp32(w / c1) per element, with c1 the absmax of its block; c1 == 0 gives 0."""
    w = np.asarray(w, dtype=np.float32).reshape(-1, block)
    c = np.asarray(c1, dtype=np.float32)[:, None]
    x = np.zeros_like(w)
    np.divide(w, np.broadcast_to(c, w.shape), out=x, where=np.broadcast_to(c > 0, w.shape))
    return x.ravel()


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte; element 2j in the high nibble (reading R4)."""
    c = np.asarray(codes, dtype=np.uint8).ravel()
    return ((c[0::2] << 4) | c[1::2]).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).ravel()
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 0xF
    return out


def check_args(N: int, K: int, blocksize: int = BLOCKSIZE, blocksize2: int = BLOCKSIZE2):
    """Argument rules shared in meaning with the C ABI: K % 64 == 0, blocks 64 / 256."""
    if blocksize != BLOCKSIZE or blocksize2 != BLOCKSIZE2:
        raise OracleUnsupported("only blocksize 64 and second-level block 256 are defined")
    if N < 1 or K < 1 or K % BLOCKSIZE != 0:
        raise OracleShapeError("need N >= 1, K >= 1 and K % 64 == 0")


# ---------------------------------------------------------------------------
# Double Quantization ([SD] Section 3 (2); reading R5)
# ---------------------------------------------------------------------------

def pairwise_tree_sum(v: np.ndarray) -> float:
    """fp64 sum over a fixed pairwise tree: pad to a power of two with zeros,
    then add neighbours level by level, s[i] = s[2i] + s[2i+1]."""
    s = np.asarray(v, dtype=np.float64).ravel()
    n = max(1, s.size)
    size = 1 << (n - 1).bit_length()
    t = np.zeros(size, dtype=np.float64)
    t[:s.size] = s
    while t.size > 1:
        t = t[0::2] + t[1::2]
    return float(t[0])


def dq_mean(c1: np.ndarray) -> np.float32:
    """mu = fp32(fp64(sum(c1) / nb1)), the sum taken over the fixed pairwise tree."""
    c1 = np.asarray(c1, dtype=np.float32)
    S = pairwise_tree_sum(c1)
    return np.float32(S / float(c1.size))


def double_quantize(c1: np.ndarray, blocksize2: int = BLOCKSIZE2):
    """Quantize the fp32 block constants c1 to 8-bit floats (reading R5).

    Returns (c1_codes uint8[nb1], c2 fp32[nb2], mu fp32).
      d  = fp32(c1 - mu)
      c2 = max |d| over each group of 256
      x2 = fp32(d / c2)   (0 when c2 == 0)
      c1_code = E4M3(x2)
    """
    c1 = np.asarray(c1, dtype=np.float32).ravel()
    mu = dq_mean(c1)
    d = (c1 - mu).astype(np.float32)
    c2 = block_absmax(d, blocksize2).astype(np.float32)
    c2e = np.repeat(c2, blocksize2)[:d.size]
    x2 = np.zeros_like(d)
    np.divide(d, c2e, out=x2, where=c2e > 0)
    return e4m3_encode(x2), c2, mu


def dq_constants(c1_codes: np.ndarray, c2: np.ndarray, mu, blocksize2: int = BLOCKSIZE2) -> np.ndarray:
    """Rebuilt first-level constants c1' = fp32(fp32(v8 * c2) + mu) (reading R6)."""
    v8 = e4m3_decode(c1_codes)
    c2e = np.repeat(np.asarray(c2, dtype=np.float32), blocksize2)[:v8.size]
    prod = (v8 * c2e).astype(np.float32)
    return (prod + np.float32(mu)).astype(np.float32)


# ---------------------------------------------------------------------------
# Whole quantize / dequantize
# ---------------------------------------------------------------------------

def quantize_nf4_dq(W_bits: np.ndarray, blocksize: int = BLOCKSIZE, blocksize2: int = BLOCKSIZE2,
                    q: np.ndarray | None = None) -> dict:
    """NF4 + Double Quantization of a bf16 weight W[N,K] given as uint16 bit patterns.

    Returns a dict with the four stored buffers (codes, c1_codes, c2, mu) and the
    intermediate first-level constants c1 and per-element codes.
    """
    W_bits = np.asarray(W_bits, dtype=np.uint16)
    N, K = W_bits.shape
    check_args(N, K, blocksize, blocksize2)
    q = nf4_codebook() if q is None else q
    w = bf16_bits_to_f32(W_bits).ravel()
    c1 = block_absmax(w, blocksize).astype(np.float32)
    x = normalize_blocks(w, c1, blocksize)
    codes = nearest_code(x, q)
    c1_codes, c2, mu = double_quantize(c1, blocksize2)
    return {"codes": pack_nibbles(codes), "c1_codes": c1_codes, "c2": c2,
            "mu": np.float32(mu), "c1": c1, "code_idx": codes, "N": N, "K": K}


def dequantize(codes_packed: np.ndarray, c1_codes: np.ndarray, c2: np.ndarray, mu,
               N: int, K: int, q: np.ndarray | None = None, f16: bool = False) -> np.ndarray:
    """W_hat = bf16_RN(fp32(q[code] * c1')) as uint16 bf16 bits [N,K] (reading R6); with f16,
    rounded to fp16 instead (the fp16 compute dtype)."""
    q = nf4_codebook() if q is None else q
    idx = unpack_nibbles(codes_packed)[:N * K]
    c1p = dq_constants(c1_codes, c2, mu)
    c1e = np.repeat(c1p, BLOCKSIZE)[:N * K]
    prod = (q[idx] * c1e).astype(np.float32)
    return (f32_to_f16_bits(prod) if f16 else f32_to_bf16_bits(prod)).reshape(N, K)


def dequantize_single(codes_packed: np.ndarray, c1: np.ndarray, N: int, K: int,
                      q: np.ndarray | None = None, f16: bool = False) -> np.ndarray:
    """Double quantization off (reading R10): W_hat = bf16_RN(fp32(q[code] * c1)) with the
    fp32 block absmax c1 kept as is; uint16 bf16 bits [N,K]."""
    q = nf4_codebook() if q is None else q
    idx = unpack_nibbles(codes_packed)[:N * K]
    c1e = np.repeat(np.asarray(c1, dtype=np.float32), BLOCKSIZE)[:N * K]
    prod = (q[idx] * c1e).astype(np.float32)
    return (f32_to_f16_bits(prod) if f16 else f32_to_bf16_bits(prod)).reshape(N, K)


def relative_sq_error(W_bits: np.ndarray, What_bits: np.ndarray) -> float:
    """sum (W_hat - W)^2 / sum W^2 in fp64 over bf16 bit patterns ([SD] section 4 (2))."""
    w = bf16_bits_to_f32(W_bits).astype(np.float64)
    e = bf16_bits_to_f32(What_bits).astype(np.float64) - w
    return float((e * e).sum() / (w * w).sum())


def dequantize_rows(qw: dict, rows: np.ndarray, q: np.ndarray | None = None) -> np.ndarray:
    """W_hat for selected rows only (uint16 bits [len(rows), K]); same arithmetic as dequantize."""
    q = nf4_codebook() if q is None else q
    K = qw["K"]
    rows = np.asarray(rows, dtype=np.int64)
    bpr = K // BLOCKSIZE
    packed = qw["codes"].reshape(-1, K // 2)[rows]
    idx = unpack_nibbles(packed).reshape(len(rows), K)
    c1p_all = dq_constants(qw["c1_codes"], qw["c2"], qw["mu"]).reshape(-1, bpr)[rows]
    c1e = np.repeat(c1p_all, BLOCKSIZE, axis=1)
    prod = (q[idx] * c1e).astype(np.float32)
    return f32_to_bf16_bits(prod)


def quantize_rows(W_bits: np.ndarray, rows, q: np.ndarray | None = None) -> dict:
    """Quantize with the double-quantized constants of the whole tensor, but the
    per-element codes of the selected rows only (same steps as quantize_nf4_dq;
    for checking large tensors by sampling)."""
    W_bits = np.asarray(W_bits, dtype=np.uint16)
    N, K = W_bits.shape
    check_args(N, K)
    q = nf4_codebook() if q is None else q
    rows = np.asarray(rows, dtype=np.int64)
    c1 = block_absmax(bf16_bits_to_f32(W_bits).ravel(), BLOCKSIZE).astype(np.float32)
    c1_codes, c2, mu = double_quantize(c1)
    bpr = K // BLOCKSIZE
    w_rows = bf16_bits_to_f32(W_bits[rows]).ravel()
    c1_rows = c1.reshape(N, bpr)[rows].ravel()
    codes = nearest_code(normalize_blocks(w_rows, c1_rows), q)
    return {"codes_rows": pack_nibbles(codes).reshape(len(rows), K // 2), "c1_codes": c1_codes,
            "c2": c2, "mu": np.float32(mu), "c1": c1, "N": N, "K": K}


def dequantize_cols(qw: dict, cols, q: np.ndarray | None = None) -> np.ndarray:
    """W_hat for selected columns only (uint16 bits [N, len(cols)]); same arithmetic as dequantize."""
    q = nf4_codebook() if q is None else q
    N, K = qw["N"], qw["K"]
    cols = np.asarray(cols, dtype=np.int64)
    flat = np.arange(N, dtype=np.int64)[:, None] * K + cols[None, :]
    byte = np.asarray(qw["codes"], dtype=np.uint8)[flat >> 1]
    idx = np.where((flat & 1) == 1, byte & 0xF, byte >> 4)
    c1p = dq_constants(qw["c1_codes"], qw["c2"], qw["mu"])
    prod = (q[idx] * c1p[flat >> 6]).astype(np.float32)
    return f32_to_bf16_bits(prod)


# ---------------------------------------------------------------------------
# The linear layer in fp64 ([QP] Section 7 diagram; [QR] Section 4.4; R7, R8)
# ---------------------------------------------------------------------------

def _f64(bits_or_array) -> np.ndarray:
    a = np.asarray(bits_or_array)
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to IEEE fp16 (nearest, ties to even: NumPy's float16 conversion);
    uint16 bits.  The fp16 compute dtype ([QP] section 4: fp16 where bf16 is not well supported)."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def f16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """fp16 bit patterns -> exact fp32 values."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float32)


def f64_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to fp16 directly (nearest, ties to even): 11 significant bits down to
    2^-14, a fixed step of 2^-24 below, infinity past 65504 (after rounding)."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    step = np.ldexp(1.0, np.maximum(e, -13) - 11)
    r = np.rint(x / step) * step
    with np.errstate(over="ignore"):
        return r.astype(np.float16).view(np.uint16)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 directly (nearest, ties to even; no fp32 step, which could
    round twice).  bf16 keeps 8 significant bits down to 2^-126 and a fixed step of 2^-133
    below; values that round past the largest finite bf16 become infinity."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                                   # |x| = m 2^e, 0.5 <= m < 1
    step = np.ldexp(1.0, np.maximum(e, -125) - 8)        # spacing of bf16 values around x
    r = np.rint(x / step) * step                         # exact scaling; rint ties to even
    with np.errstate(over="ignore"):
        r32 = r.astype(np.float32)                       # exact: <= 8 significant bits (or overflow)
    return f32_to_bf16_bits(r32)


def merge_lora(W_hat, A, B, alpha: float, r: int, f16: bool = False) -> np.ndarray:
    """Merged weight for inference ([Q103] follow-up 1; [QP] section 5):
    W_merged = RN16(W_hat + s B A), s = alpha / r, the rank-r product and the sum in fp64
    (products of 16-bit values are exact; one rounding at the end to bf16, or fp16 when f16).
    Inputs: bf16 bits (uint16) or float arrays.  Returns uint16 bits [N,K]."""
    s = lora_scale(alpha, r)
    merged = _f64(W_hat) + s * (_f64(B) @ _f64(A))
    return f64_to_f16_bits(merged) if f16 else f64_to_bf16_bits(merged)


def lora_scale(alpha: float, r: int) -> float:
    """s = alpha / r ([Q103] follow-up 3 names r and alpha)."""
    return float(alpha) / float(r)


def linear_forward(X, W_hat, A, B, alpha: float, r: int):
    """Y = X W_hat^T + s (X A^T) B^T in fp64.  Returns (Y, U) with U = X A^T unrounded."""
    Xd, Wd, Ad, Bd = _f64(X), _f64(W_hat), _f64(A), _f64(B)
    s = lora_scale(alpha, r)
    U = Xd @ Ad.T
    Y = Xd @ Wd.T + s * (U @ Bd.T)
    return Y, U


def linear_forward_multi(X, W_hat, A_all, B_all, adapter_idx, alpha: float, r: int):
    """One base, many adapters ([CH9] section "3. 一个底座，多个适配器"): token m uses adapter
    a = adapter_idx[m] (A_all[a] [r,K], B_all[a] [N,r]); a == -1 means the base alone.
    Y[m] = X[m] W_hat^T + s (X[m] A_a^T) B_a^T in fp64.  Returns (Y, U), U[m] = X[m] A_a^T (0 for -1)."""
    Xd, Wd = _f64(X), _f64(W_hat)
    Ad, Bd = _f64(A_all), _f64(B_all)
    s = lora_scale(alpha, r)
    Y = Xd @ Wd.T
    U = np.zeros((Xd.shape[0], r))
    for m, a in enumerate(np.asarray(adapter_idx).ravel()):
        if a < 0:
            continue
        U[m] = Xd[m] @ Ad[a].T
        Y[m] += s * (U[m] @ Bd[a].T)
    return Y, U


def linear_backward(X, dY, W_hat, A, B, alpha: float, r: int):
    """Gradients of <dY, Y> through the frozen W_hat; no gradient for the codes.

    dU = s dY B;  dX = dY W_hat + dU A;  dA = dU^T X;  dB = s dY^T (X A^T).
    Returns dict(dX, dA, dB, dU) in fp64.
    """
    Xd, dYd, Wd, Ad, Bd = _f64(X), _f64(dY), _f64(W_hat), _f64(A), _f64(B)
    s = lora_scale(alpha, r)
    U = Xd @ Ad.T
    dU = s * (dYd @ Bd)
    dX = dYd @ Wd + dU @ Ad
    dA = dU.T @ Xd
    dB = s * (dYd.T @ U)
    return {"dX": dX, "dA": dA, "dB": dB, "dU": dU}


def lora_gradients(X, dY, A, B, alpha: float, r: int):
    """The adapter gradients alone, for shapes where the full dX is too large to form:
    dA = (s dY B)^T X and dB = s dY^T (X A^T), in fp64 (the same formulas as linear_backward)."""
    Xd, dYd, Ad, Bd = _f64(X), _f64(dY), _f64(A), _f64(B)
    s = lora_scale(alpha, r)
    dU = s * (dYd @ Bd)
    return {"dA": dU.T @ Xd, "dB": s * (dYd.T @ (Xd @ Ad.T))}


def forward_rows(X, W_hat, A, B, alpha, r, rows):
    """Y for a subset of token rows (the reference for large shapes)."""
    Xs = _f64(X)[rows]
    return linear_forward(Xs, W_hat, A, B, alpha, r)[0]


def backward_dx_rows(dY, W_hat, A, B, alpha, r, rows):
    """dX for a subset of token rows."""
    dYs = _f64(dY)[rows]
    s = lora_scale(alpha, r)
    dU = s * (dYs @ _f64(B))
    return dYs @ _f64(W_hat) + dU @ _f64(A)


# ---------------------------------------------------------------------------
# Brute-force loops for tiny shapes (an independent check of the matmul steps)
# ---------------------------------------------------------------------------

def brute_force_forward(X, W_hat, A, B, alpha, r):
    Xd, Wd, Ad, Bd = _f64(X), _f64(W_hat), _f64(A), _f64(B)
    M, K = Xd.shape
    N = Wd.shape[0]
    s = lora_scale(alpha, r)
    Y = np.zeros((M, N))
    for m in range(M):
        u = [sum(Xd[m, k] * Ad[j, k] for k in range(K)) for j in range(r)]
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += Xd[m, k] * Wd[n, k]
            lo = 0.0
            for j in range(r):
                lo += u[j] * Bd[n, j]
            Y[m, n] = acc + s * lo
    return Y


def exact_nearest_code(x: float, q) -> int:
    """argmin with exact rational distances (ties to the lower index)."""
    fx = Fraction(float(x))
    best, best_d = 0, None
    for i, qi in enumerate(q):
        d = abs(fx - Fraction(float(qi)))
        if best_d is None or d < best_d:
            best, best_d = i, d
    return best


# ---------------------------------------------------------------------------
# Memory footprint ([SD] Section 3 (2))
# ---------------------------------------------------------------------------

def stored_bytes(N: int, K: int, blocksize: int = BLOCKSIZE, blocksize2: int = BLOCKSIZE2) -> dict:
    """Bytes of the four stored buffers for W[N,K]."""
    n = N * K
    nb1 = -(-n // blocksize)
    nb2 = -(-nb1 // blocksize2)
    return {"codes": (n + 1) // 2, "c1_codes": nb1, "c2": 4 * nb2, "mu": 4}


def constant_bits_per_param(N: int, K: int, double_quant: bool = True) -> float:
    """Bits per weight spent on quantization constants (mu excluded)."""
    b = stored_bytes(N, K)
    if not double_quant:
        return 32.0 * (-(-N * K // BLOCKSIZE)) / (N * K)
    return 8.0 * (b["c1_codes"] + b["c2"]) / (N * K)


# ---------------------------------------------------------------------------
# Absmax INT8, the worked example of [CH9] (reading R9)
# ---------------------------------------------------------------------------

def absmax_int8(x):
    """alpha = 127 / max|x|; code = round_half_away(x * alpha); x_hat = code / alpha."""
    x = np.asarray(x, dtype=np.float64)
    amax = float(block_absmax(x, x.size)[0])
    alpha = 127.0 / amax
    scaled = x * alpha
    code = np.sign(scaled) * np.floor(np.abs(scaled) + 0.5)
    return alpha, code.astype(np.int64), code / alpha


def quantize_int8_blocks(bits, blocksize: int = 64):
    """Blockwise absmax INT8 of a bf16 tensor (bits, uint16), [CH9] section
    "2. INT8 量化" steps 1-3 in fp32 (reading R14).  Returns (codes int8 [n],
    alpha fp32 [n / blocksize])."""
    if blocksize not in (64, 128, 256):
        raise OracleShapeError("blocksize must be 64, 128 or 256")
    x = bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16).ravel())
    if x.size < 1 or x.size % blocksize:
        raise OracleShapeError("n must be a positive multiple of blocksize")
    if not np.all(np.isfinite(x)):
        raise OracleNonFiniteError("tensor holds Inf or NaN")
    xb = x.reshape(-1, blocksize)
    amax = np.max(np.abs(xb), axis=1)                                  # step 1, exact
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        alpha = np.where(amax > 0, np.float32(127.0) / amax, np.float32(0.0)).astype(np.float32)   # step 2
        s = (xb * alpha[:, None]).astype(np.float32)                   # step 3: x * alpha in fp32
    s = np.where(xb == 0, np.float32(0.0), s)
    s = np.clip(s.astype(np.float64), -127.0, 127.0)
    code = np.sign(s) * np.floor(np.abs(s) + 0.5)                      # half away from zero, exact in fp64
    return code.astype(np.int8).ravel(), alpha


def dequantize_int8_blocks(codes, alpha, blocksize: int = 64):
    """[CH9] section "2. INT8 量化" step 4 (reading R14): x_hat = fp32(code / alpha),
    0 where alpha = 0.  Returns fp32 [n]."""
    c = np.asarray(codes, dtype=np.int8).astype(np.float32).reshape(-1, blocksize)
    a = np.asarray(alpha, dtype=np.float32)
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        xh = np.where(a[:, None] == 0, np.float32(0.0), c / a[:, None]).astype(np.float32)
    return xh.ravel()
