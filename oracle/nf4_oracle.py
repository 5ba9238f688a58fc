"""Plain CPU oracle for the QLoRA linear layer: NF4 codes, double-quantized block
constants, double dequantization, and the LoRA-augmented forward and backward.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``
(its CPU-baseline leg and ``--impl reference``) may import this module. The CUDA
library under ``bit_nf4_quantized_unpack_b200/`` shares no code, table or constant
with it and never imports it.

Everything here is NumPy on the host: the codec in fp32 (the precision in which the
method's integer decisions are taken), the matrix products in fp64 from the exact
bf16/fp32 inputs. Sources, by page title and section:

* "QLoRA" (itwiki.kr), section "4비트 NormalFloat(NF4)" -- the NF4 code table
  built from N(0,1) quantiles with offset 0.9677083, the printed 16-value table,
  and blockwise absmax quantization with nearest-code search (block 64).
* same page, section "이중 양자화" (double quantization) -- the block constants are
  re-quantized to an 8-bit float in blocks of 256 after subtracting their mean;
  overhead 8/64 + 32/(64*256) bits per parameter.
* same page, section "계산 방식" (computation) -- the forward
  Y = X doubleDequant(c1, c2, W) + X L1 L2 in bf16, dequantization in forward and
  backward, gradients only for L1, L2 and for the input.
* "quantization" (minnong511 blog), sections "1. 양자화" (the uniform quantizer and
  its worked example), "QLoRA에서 학습은 어떻게 되는 걸까?" (y = Wx + (alpha/r) B A x)
  and "그런데 Base Model은 4bit인데 학습이 가능한 이유는?" (W frozen, gradients for
  A and B only).
* "QLoRA" (irregular6612 blog), section "학습 → 추론 파이프라인 (실무)" -- after
  training, merge_and_unload dequantizes the base to BF16 and adds the LoRA term, with
  the alpha/r scale (section "재양자화 시 주의사항"); itwiki "QLoRA", section
  "한계와 주의점", on merging the adapter into a 16-bit weight.

Readings where the pages are silent (each pinned or flagged in the tests):
* nibble order: byte b holds code 2b in its low nibble and code 2b+1 in its high
  nibble, row-major (the pages only say 4 bits = 0.5 byte per parameter).
  Parity unpinned beyond round trips: it is a storage convention.
* an all-zero block (absmax 0) gets x = 0, hence code 7 (the exact zero).
* the 8-bit float of the double quantization is OCP FP8 E4M3; its code table T8 is
  the 253 distinct finite E4M3 values divided by 448, rounded to fp32; a constant's
  code is the E4M3 bit pattern of its nearest T8 entry.
* one mean per tensor (the only reading that gives exactly 0.127 bits/param): the
  arithmetic mean of the block constants taken exactly and rounded once to fp32.
* nearest-level ties go to the lower index (NumPy ``argmin`` takes the first).
* the LoRA term carries the alpha/r scale of the minnong511 page; the itwiki
  equation omits it. A is K x r, B is r x N, so the LoRA product is X A B.
* merge_and_unload: W_merged = bf16(Ŵ + scale (A B)^T) with the sum exact and one
  rounding to bf16 (the pages do not say in which precision the sum is formed).
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
from scipy.stats import norm

NF4_OFFSET = 0.9677083  # top probability of the NF4 construction (itwiki "QLoRA", NF4 section)
BLOCK = 64              # weights per absmax block
DQ_BLOCK = 256          # absmax constants per double-quantization block
E4M3_MAX = 448.0        # largest finite OCP FP8 E4M3 magnitude


# ---------------------------------------------------------------------------
# Code tables
# ---------------------------------------------------------------------------

def _even_probabilities(count: int) -> np.ndarray:
    """``count`` evenly spaced probabilities from NF4_OFFSET down to 1/2, the 1/2
    end point excluded: p_i = offset + i * (1/2 - offset) / count, i < count."""
    step = (0.5 - NF4_OFFSET) / count
    return NF4_OFFSET + step * np.arange(count)


def nf4_levels_f64() -> np.ndarray:
    """The 16 NF4 levels in fp64, ascending, normalised to [-1, 1].

    itwiki "QLoRA", section "4비트 NormalFloat(NF4)": 2^(k-1) = 8 quantiles on the
    positive side, 2^(k-1) - 1 = 7 on the negative side, one shared exact zero,
    all normalised by the largest magnitude. The quantiles are those of N(0, 1)
    at evenly spaced probabilities between the offset 0.9677083 and 1/2.
    """
    positive = norm.ppf(_even_probabilities(8))      # 8 values > 0
    negative = -norm.ppf(_even_probabilities(7))     # 7 values < 0
    levels = np.sort(np.concatenate([negative, [0.0], positive]))
    return levels / np.max(np.abs(levels))


def nf4_levels() -> np.ndarray:
    """NF4 levels rounded to fp32: the table the codec works with."""
    return nf4_levels_f64().astype(np.float32)


def uniform4_levels() -> np.ndarray:
    """The 'uniform 4-bit, same method' comparison codebook of the itwiki NF4
    section: 16 evenly spaced levels on [-1, 1] (fp32)."""
    return np.linspace(-1.0, 1.0, 16).astype(np.float32)


def e4m3_decode(bits: int) -> float:
    """Value of an OCP FP8 E4M3 bit pattern (sign 1, exponent 4 with bias 7,
    mantissa 3; exponent 0 is subnormal; S.1111.111 is NaN; no infinities)."""
    sign = -1.0 if bits & 0x80 else 1.0
    exp = (bits >> 3) & 0xF
    man = bits & 0x7
    if exp == 0xF and man == 0x7:
        return float("nan")
    if exp == 0:
        return sign * man * 2.0 ** -9
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


def fp8_table() -> tuple[np.ndarray, np.ndarray]:
    """T8 of the double quantization: the distinct finite E4M3 values in ascending
    order, divided by 448 in fp32, and for each entry its E4M3 bit pattern
    (+0 for zero). Returns (values fp32 [253], codes uint8 [253])."""
    by_value: dict[float, int] = {}
    for bits in range(256):
        v = e4m3_decode(bits)
        if math.isnan(v):
            continue
        if v == 0.0:
            by_value[0.0] = 0x00
        elif v not in by_value:
            by_value[v] = bits
    vals = sorted(by_value)
    scaled = (np.array(vals, np.float32) / np.float32(E4M3_MAX)).astype(np.float32)
    codes = np.array([by_value[v] for v in vals], np.uint8)
    return scaled, codes


def fp8_code_to_t8(code: np.ndarray) -> np.ndarray:
    """T8 value (fp32) for each E4M3 bit pattern in ``code``."""
    vals, codes = fp8_table()
    lut = np.full(256, np.nan, np.float32)
    lut[codes] = vals
    lut[0x80] = 0.0  # -0 decodes to zero as well
    return lut[np.asarray(code, np.uint8)]


# ---------------------------------------------------------------------------
# Nearest-code search and rounding
# ---------------------------------------------------------------------------

def nearest_code(x: np.ndarray, table: np.ndarray, chunk: int = 1 << 16) -> np.ndarray:
    """Index of the nearest table entry for each fp32 x: argmin_i fl32(|x - table_i|),
    the first (lowest) index on ties. Plain brute force over the whole table."""
    x = np.asarray(x, np.float32).ravel()
    table = np.asarray(table, np.float32)
    out = np.empty(x.size, np.int64)
    for s in range(0, x.size, chunk):
        d = np.abs(x[s:s + chunk, None] - table[None, :])   # fp32 subtraction
        out[s:s + chunk] = np.argmin(d, axis=1)
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); returned as fp32
    holding the bf16 value. Finite inputs only."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of values already representable in bf16."""
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


# ---------------------------------------------------------------------------
# Level 1: blockwise absmax + NF4 codes (itwiki "QLoRA", NF4 section)
# ---------------------------------------------------------------------------

def block_absmax(w: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Absolute maximum of each block of ``block`` consecutive weights (row-major
    flattening), fp32 [n / block]."""
    w = np.asarray(w, np.float32).reshape(-1, block)
    return np.max(np.abs(w), axis=1).astype(np.float32)


def quantize_blocks(w: np.ndarray, levels: np.ndarray, block: int = BLOCK):
    """Flatten row-major into blocks of ``block`` weights, divide each block by its
    absolute maximum (fp32, IEEE division) and take the nearest level.
    Returns (codes uint8 [n], absmax fp32 [n / block])."""
    w = np.asarray(w, np.float32).reshape(-1, block)
    absmax = block_absmax(w, block)
    x = np.zeros_like(w)
    live = absmax > 0
    x[live] = w[live] / absmax[live, None]           # fp32 / fp32, correctly rounded
    codes = nearest_code(x, levels).astype(np.uint8)
    return codes, absmax.astype(np.float32)


def dequantize_blocks(codes: np.ndarray, absmax: np.ndarray, levels: np.ndarray,
                      block: int = BLOCK) -> np.ndarray:
    """levels[code] * absmax of the code's block (fp32, no double quantization)."""
    vals = np.asarray(levels, np.float32)[np.asarray(codes).reshape(-1, block)]
    return (vals * np.asarray(absmax, np.float32)[:, None]).ravel()


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: even index in the low nibble."""
    c = np.asarray(codes, np.uint8).reshape(-1, 2)
    return (c[:, 0] | (c[:, 1] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.size * 2, np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out


# ---------------------------------------------------------------------------
# Level 2: double quantization of the absmax constants (itwiki "QLoRA", DQ)
# ---------------------------------------------------------------------------

def f32_round(x: Fraction) -> np.float32:
    """The fp32 value nearest to the non-negative rational x (IEEE round to nearest,
    ties to even), for x below the largest finite fp32. Written from the definition:
    find the binade [2^E, 2^(E+1)) holding x (E >= -126, since subnormals share the
    spacing of the smallest normal binade), count x in units of that binade's spacing
    2^(E-23), and round the count to an integer."""
    x = Fraction(x)
    if x < 0:
        raise ValueError("f32_round takes non-negative values")
    if x == 0:
        return np.float32(0.0)
    E = x.numerator.bit_length() - x.denominator.bit_length()
    while Fraction(2) ** E > x:
        E -= 1
    while Fraction(2) ** (E + 1) <= x:
        E += 1
    E = max(E, -126)
    ulp = Fraction(2) ** (E - 23)
    units = x / ulp
    n = units.numerator // units.denominator
    rest = units - n
    if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return np.float32(float(n * ulp))   # n <= 2^24: an fp32 value, converted exactly


def exact_sum_f32(values: np.ndarray) -> Fraction:
    """The exact sum of fp32 values >= 0, as a rational. Each value is sig * 2^(e - 150)
    with sig its 24-bit significand and e its biased exponent (1 for subnormals); the
    significands of each exponent are summed as integers (exactly), then combined."""
    u = np.asarray(values, np.float32).ravel().view(np.uint32)
    if np.any(u >> 31) or np.any(((u >> 23) & 0xFF) == 0xFF):
        raise ValueError("exact_sum_f32 takes finite values >= 0")
    e = (u >> 23) & 0xFF
    sig = (u & 0x7FFFFF) | np.where(e > 0, 0x800000, 0).astype(np.uint32)
    e = np.maximum(e, 1)
    total = 0
    for ev in np.unique(e[sig > 0]):
        total += int(sig[e == ev].astype(np.int64).sum()) << int(ev)
    return Fraction(total, 1 << 150)


def constants_mean(absmax: np.ndarray) -> np.float32:
    """One mean per tensor: the arithmetic mean of all block constants, taken exactly
    (exact sum over their count) and rounded once to fp32. It does not depend on the
    order of the constants, whatever their range."""
    a = np.asarray(absmax, np.float32).ravel()
    return f32_round(exact_sum_f32(a) / a.size)


def double_quantize(absmax: np.ndarray, dq_block: int = DQ_BLOCK):
    """Centre the (all positive) constants on their mean, then quantize them
    symmetrically to the 8-bit float table T8 in blocks of ``dq_block``, keeping
    one fp32 absmax c1 per block. Returns (c2 uint8 E4M3 codes [n], c1 fp32
    [ceil(n / dq_block)], mean fp32)."""
    absmax = np.asarray(absmax, np.float32)
    n = absmax.size
    mean = constants_mean(absmax)
    centred = (absmax - mean).astype(np.float32)         # fp32 subtraction
    nblk = -(-n // dq_block)
    c1 = np.zeros(nblk, np.float32)
    y = np.zeros(n, np.float32)
    for b in range(nblk):
        seg = centred[b * dq_block:(b + 1) * dq_block]
        m = np.max(np.abs(seg))
        c1[b] = m
        if m > 0:
            y[b * dq_block:b * dq_block + seg.size] = seg / m   # fp32 division
    t8_vals, t8_codes = fp8_table()
    c2 = t8_codes[nearest_code(y, t8_vals)]
    return c2.astype(np.uint8), c1, mean


def reconstruct_absmax(c2: np.ndarray, c1: np.ndarray, mean, dq_block: int = DQ_BLOCK):
    """s_j = fl32(fl32(T8[c2_j] * c1_b) + mean): multiply, then add, each rounded."""
    t = fp8_code_to_t8(c2)
    c1_per = np.repeat(np.asarray(c1, np.float32), dq_block)[:t.size]
    prod = (t * c1_per).astype(np.float32)
    return (prod + np.float32(mean)).astype(np.float32)


# ---------------------------------------------------------------------------
# The stored weight and doubleDequant (itwiki "QLoRA", computation section)
# ---------------------------------------------------------------------------

def quantize_nf4_dq(W: np.ndarray, levels: np.ndarray | None = None):
    """W [N, K] (fp32, or bf16 values held in fp32), K % 64 == 0 ->
    dict(codes packed uint8 [N*K/2], c2 uint8 [N*K/64], c1 fp32, mean fp32, absmax,
    levels). ``levels`` is the 4-bit codebook: NF4 by default, or the evenly spaced
    comparison codebook of the itwiki NF4 section (``uniform4_levels``), which goes
    through the same blocking, search and double quantization."""
    W = np.asarray(W, np.float32)
    assert W.ndim == 2 and W.shape[1] % BLOCK == 0
    levels = nf4_levels() if levels is None else np.asarray(levels, np.float32)
    codes, absmax = quantize_blocks(W, levels)
    c2, c1, mean = double_quantize(absmax)
    return {"codes": pack_nibbles(codes), "c2": c2, "c1": c1, "mean": mean,
            "absmax": absmax, "shape": W.shape, "levels": levels}


def _levels_of(q: dict) -> np.ndarray:
    return q["levels"] if "levels" in q else nf4_levels()


def double_dequant(q: dict) -> np.ndarray:
    """doubleDequant(c1, c2, W_NF4): Ŵ = bf16(fl32(L[code] * s_block)) [N, K],
    returned as fp32 holding bf16 values."""
    n, k = q["shape"]
    s = reconstruct_absmax(q["c2"], q["c1"], q["mean"])
    codes = unpack_nibbles(q["codes"]).reshape(-1, BLOCK)
    vals = _levels_of(q)[codes] * s[:, None]            # fp32 products
    return bf16_round(vals.astype(np.float32)).reshape(n, k)


def double_dequant_rows(q: dict, rows: np.ndarray) -> np.ndarray:
    """Ŵ for selected rows only (same arithmetic as ``double_dequant``)."""
    n, k = q["shape"]
    rows = np.asarray(rows)
    bpr = k // BLOCK
    blk = (rows[:, None] * bpr + np.arange(bpr)[None, :]).ravel()
    s = reconstruct_absmax(q["c2"], q["c1"], q["mean"])[blk]
    packed = q["codes"].reshape(n, k // 2)[rows]
    codes = unpack_nibbles(packed.ravel()).reshape(-1, BLOCK)
    vals = _levels_of(q)[codes] * s[:, None]
    return bf16_round(vals.astype(np.float32)).reshape(rows.size, k)


def double_dequant_cols(q: dict, cols: np.ndarray) -> np.ndarray:
    """Ŵ for selected columns only, [N, len(cols)] (same arithmetic as ``double_dequant``):
    the code of (n, k) is nibble k % 2 of byte k // 2 of row n (low nibble first), its
    scale that of block k // 64 of row n."""
    n, k = q["shape"]
    cols = np.asarray(cols)
    bpr = k // BLOCK
    s = reconstruct_absmax(q["c2"], q["c1"], q["mean"]).reshape(n, bpr)[:, cols // BLOCK]
    packed = q["codes"].reshape(n, k // 2)[:, cols // 2]
    codes = np.where((cols % 2 == 0)[None, :], packed & 0xF, packed >> 4)
    vals = _levels_of(q)[codes] * s
    return bf16_round(vals.astype(np.float32))


# ---------------------------------------------------------------------------
# The QLoRA linear layer (itwiki "QLoRA" computation section; minnong511
# "quantization": y = W x + (alpha / r) B A x, W frozen, grads for A and B)
# ---------------------------------------------------------------------------

def linear_forward(X, W_hat, A, B, scale):
    """Y = X Ŵ^T + scale (X A) B in fp64 from the exact inputs.
    X [M, K], Ŵ [N, K], A [K, r], B [r, N]. Returns (Y fp64, T = X A fp64)."""
    X = np.asarray(X, np.float64)
    T = X @ np.asarray(A, np.float64)
    Y = X @ np.asarray(W_hat, np.float64).T + scale * (T @ np.asarray(B, np.float64))
    return Y, T


def merge_lora(q: dict, A, B, scale) -> np.ndarray:
    """merge_and_unload (blog "QLoRA", irregular6612, section on the training-to-inference
    pipeline: dequantize the base to BF16, then add the LoRA term, with the alpha/r scale
    of the section on re-quantization; itwiki "QLoRA", section "한계와 주의점"):
    W_merged = bf16(Ŵ + scale (A B)^T) [N, K]. Reading: the sum is exact (fp64 from the
    bf16 Ŵ and the bf16 A, B) and rounded once to bf16. Returns fp64 pre-rounding values
    and the bf16 result (as fp32 holding bf16 values)."""
    W_hat = double_dequant(q).astype(np.float64)
    delta = (np.asarray(A, np.float64) @ np.asarray(B, np.float64)).T
    exact = W_hat + float(scale) * delta
    return exact, bf16_round_f64(exact)


def bf16_round_f64(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 in one step (nearest, ties to even), returned as fp32
    holding bf16 values. bf16 keeps 8 significant bits, so the spacing of bf16 values
    around x is ulp = 2^(E - 8) for x = m 2^E with m in [0.5, 1), and never below the
    subnormal spacing 2^-133; x / ulp and q * ulp are exact in fp64 (powers of two).
    Rounding to fp32 first and then to bf16 could round twice."""
    x = np.asarray(x, np.float64)
    _, E = np.frexp(x)
    ulp = np.ldexp(1.0, np.maximum(E - 8, -133))
    q = np.rint(x / ulp) * ulp              # np.rint: half to even
    q = np.where(np.abs(q) > 3.3895313892515355e38, np.copysign(np.inf, x), q)
    return q.astype(np.float32)


def linear_backward(dY, X, W_hat, A, B, scale, T=None):
    """Gradients of the forward above for an upstream gradient dY [M, N]:
    G = dY B^T, dX = dY Ŵ + scale G A^T, dA = scale X^T G, dB = scale T^T dY.
    No gradient for the frozen quantized weight."""
    dY = np.asarray(dY, np.float64)
    X = np.asarray(X, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    if T is None:
        T = X @ A
    G = dY @ B.T
    dX = dY @ np.asarray(W_hat, np.float64) + scale * (G @ A.T)
    dA = scale * (X.T @ G)
    dB = scale * (np.asarray(T, np.float64).T @ dY)
    return dX, dA, dB


# ---------------------------------------------------------------------------
# Aids for pins on the pages
# ---------------------------------------------------------------------------

def uniform_affine_quantize(x: float, x_min: float, x_max: float, bits: int):
    """The uniform quantizer of the minnong511 "quantization" page, section 1:
    s = (x_max - x_min) / (2^b - 1), q = round((x - x_min) / s), x̂ = q s + x_min.
    Returns (q, s, x̂) in fp64."""
    s = (x_max - x_min) / (2 ** bits - 1)
    q = int(np.round((x - x_min) / s))
    return q, s, q * s + x_min


def constant_overhead_bits(block: int = BLOCK, dq_block: int = DQ_BLOCK,
                           code_bits: int = 8, c1_bits: int = 32) -> float:
    """Bits per parameter spent on block constants after double quantization:
    one ``code_bits`` code per ``block`` weights and one ``c1_bits`` constant per
    ``block * dq_block`` weights (itwiki "QLoRA", double quantization)."""
    return code_bits / block + c1_bits / (block * dq_block)
