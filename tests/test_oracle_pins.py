"""Pins of the CPU oracle against what the pages print and what mathematics fixes.

Each test names the passage (page title, section) or the closed form it checks.
"""
import math

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as O
from tests.conftest import read_golden


# --- NF4 table: itwiki "QLoRA", section "4비트 NormalFloat(NF4)" -------------

def test_nf4_table_matches_printed_values():
    printed = np.array([float(v) for row in read_golden("nf4_table_printed.txt") for v in row])
    got = O.nf4_levels_f64()
    assert printed.shape == (16,)
    # Index 6 is printed as -0.0911 while the construction gives -0.09105; the
    # printed digits sit 5.0e-5 away, at the rounding edge. All others agree to
    # four decimals exactly.
    assert np.max(np.abs(got - printed)) <= 5.0e-5 + 1e-7
    mismatched = [i for i in range(16) if round(got[i], 4) != printed[i]]
    assert mismatched == [6]


def test_nf4_table_structure():
    L = O.nf4_levels()
    assert L.dtype == np.float32
    assert L[0] == -1.0 and L[15] == 1.0 and L[7] == 0.0
    assert np.all(np.diff(L) > 0)
    assert (L < 0).sum() == 7 and (L > 0).sum() == 8   # asymmetric, exact zero


def test_nf4_positive_levels_are_normal_quantiles():
    # the 8 positive levels are Phi^-1 of evenly spaced probabilities from the
    # offset down to 1/2, normalised by the largest one
    L = O.nf4_levels_f64()
    p = 0.9677083 - (0.9677083 - 0.5) * np.arange(8) / 8
    q = np.array([math.sqrt(2.0) * _erfinv(2 * pi - 1) for pi in p])
    np.testing.assert_allclose(np.sort(L[8:])[::-1], q / q[0], rtol=1e-12)


def _erfinv(y):
    # bisection on math.erf: an inverse independent of scipy's ppf
    lo, hi = -6.0, 6.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if math.erf(mid) < y:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


# --- nearest-code search --------------------------------------------------

def test_nearest_code_matches_pure_python_brute_force():
    rng = np.random.default_rng(5)
    L = O.nf4_levels()
    xs = np.concatenate([rng.uniform(-1, 1, 300).astype(np.float32), L,
                         (L[:-1] + L[1:]) / np.float32(2)]).astype(np.float32)
    got = O.nearest_code(xs, L)
    for x, g in zip(xs, got):
        best, bi = None, None
        for i, l in enumerate(L):
            d = abs(np.float32(x) - np.float32(l))   # fp32, as the method decides
            if best is None or d < best:
                best, bi = d, i
        assert g == bi


def test_nearest_code_tie_goes_to_lower_index():
    table = np.array([0.0, 0.5, 1.0], np.float32)
    assert list(O.nearest_code(np.array([0.25, 0.75], np.float32), table)) == [0, 1]


# --- blockwise quantization ------------------------------------------------

def test_blockwise_invariants():
    rng = np.random.default_rng(7)
    w = rng.normal(0, 0.02, (8, 64)).astype(np.float32)
    w[3] = 0.0                                   # an all-zero block
    codes, absmax = O.quantize_blocks(w, O.nf4_levels())
    codes = codes.reshape(8, 64)
    assert absmax[3] == 0 and np.all(codes[3] == 7)
    for b in range(8):
        if b == 3:
            continue
        j = np.argmax(np.abs(w[b]))
        assert codes[b, j] == (15 if w[b, j] > 0 else 0)


def test_levels_round_trip_exactly():
    L = O.nf4_levels()
    w = np.tile(L, 4)[None, :]                  # one 64-block holding the table
    codes, absmax = O.quantize_blocks(w, L)
    assert absmax[0] == 1.0
    assert np.array_equal(codes, np.tile(np.arange(16), 4))
    q = O.quantize_nf4_dq(w)
    # one block: mean = absmax, centred constant 0, T8 code of 0, s = mean = 1
    assert q["mean"] == 1.0 and q["c1"][0] == 0.0 and q["c2"][0] == 0
    np.testing.assert_array_equal(O.double_dequant(q)[0], O.bf16_round(w[0]))


def test_mae_pins_nf4_and_uniform():
    pins = {r[0]: float(r[1]) for r in read_golden("mae_pins.txt")}
    w = np.random.default_rng(0).normal(0, 0.02, size=4096 * 64)
    for name, levels in (("nf4", O.nf4_levels()), ("uniform4", O.uniform4_levels())):
        codes, absmax = O.quantize_blocks(w.astype(np.float32), levels)
        rec = O.dequantize_blocks(codes, absmax, levels).astype(np.float64)
        mae = np.mean(np.abs(rec - w))
        assert round(mae, 5) == pins[name], (name, mae)


def test_packing_round_trip():
    c = np.random.default_rng(1).integers(0, 16, 1000).astype(np.uint8)
    p = O.pack_nibbles(c)
    assert p.size == 500 and p[0] == (c[0] | (c[1] << 4))
    assert np.array_equal(O.unpack_nibbles(p), c)


# --- FP8 E4M3 table of the double quantization ------------------------------

def test_e4m3_decode_matches_torch_float8():
    bits = torch.arange(256, dtype=torch.uint8)
    ref = bits.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    mine = np.array([O.e4m3_decode(b) for b in range(256)], np.float32)
    both_nan = np.isnan(ref) & np.isnan(mine)
    assert np.array_equal(both_nan, np.isnan(ref))
    assert np.array_equal(ref[~both_nan], mine[~both_nan])


def test_t8_table_shape():
    vals, codes = O.fp8_table()
    assert vals.size == 253 and np.all(np.diff(vals) > 0)
    assert vals[0] == -1.0 and vals[-1] == 1.0 and vals[126] == 0.0
    assert codes[-1] == 0x7E and codes[0] == 0xFE and codes[126] == 0x00
    assert vals[127] == np.float32(2.0 ** -9) / np.float32(448)


# --- double quantization: itwiki "QLoRA", section "이중 양자화" --------------

def test_overhead_pins():
    pins = {r[0]: float(r[1]) for r in read_golden("overhead.txt")}
    assert 32 / O.BLOCK == pins["plain_bits"]          # one fp32 absmax per 64 weights
    got = O.constant_overhead_bits()
    assert got == 0.126953125 and round(got, 3) == pins["dq_bits"]
    assert round(pins["plain_bits"] - got, 3) == pins["saving_bits"]
    gb = pins["params_65b"] * (pins["plain_bits"] - got) / 8 / 1e9
    assert round(gb) == pins["saving_gb_65b"]


def test_stored_sizes_match_overhead_formula():
    W = np.random.default_rng(3).normal(0, 0.02, (256, 1024)).astype(np.float32)
    q = O.quantize_nf4_dq(W)
    n = W.size
    bits = (q["c2"].size * 8 + q["c1"].size * 32) / n
    assert bits == O.constant_overhead_bits()
    assert q["codes"].size * 8 / n == 4.0


def test_dq_block_max_maps_to_unit_code_and_mean_is_global():
    rng = np.random.default_rng(11)
    absmax = rng.uniform(0.03, 0.09, 1000).astype(np.float32)
    c2, c1, mean = O.double_quantize(absmax)
    assert mean == np.float32(np.sum(absmax.astype(np.float64)) / 1000)
    cc = absmax - mean
    for b in range(c1.size):
        seg = cc[b * 256:(b + 1) * 256]
        j = np.argmax(np.abs(seg))
        assert c2[b * 256 + j] == (0x7E if seg[j] > 0 else 0xFE)
    s = O.reconstruct_absmax(c2, c1, mean)
    # the block maximum is reconstructed to fp32 rounding
    for b in range(c1.size):
        seg = slice(b * 256, (b + 1) * 256)
        j = np.argmax(np.abs(cc[seg]))
        assert abs(s[seg][j] - absmax[seg][j]) <= 2 * np.spacing(absmax[seg][j])
    # and every constant to within half a T8 step of its block's scale
    assert np.max(np.abs(s - absmax)) < np.max(c1) / 8


def test_f32_round_matches_correctly_rounded_conversion():
    """Rational -> fp32 rounding against numpy's fp64 -> fp32 conversion (one correct
    rounding from an exact fp64 value), over normals, subnormals and exact ties."""
    from fractions import Fraction
    rng = np.random.default_rng(5)
    d = np.concatenate([
        rng.uniform(0, 1, 3000) * 2.0 ** rng.integers(-149, 120, 3000),
        rng.uniform(0, 2.0 ** -126, 500),                       # subnormal range
    ])
    f = np.float32(rng.uniform(1, 2, 500)) * np.float32(2.0) ** rng.integers(-140, 100, 500)
    ties = f.astype(np.float64) + np.spacing(f).astype(np.float64) / 2  # exact fp32 midpoints
    for v in np.concatenate([d, ties, [0.0, 2.0 ** -149, 2.0 ** -150, 3 * 2.0 ** -151]]):
        assert O.f32_round(Fraction(float(v))) == np.float32(v), v
    # a value just above an fp32 midpoint whose fp64 rounding lands on the midpoint:
    # two roundings go down (to even), one correct rounding goes up
    m = np.float32(1.0)
    x = Fraction(1) + Fraction(1, 2 ** 24) + Fraction(1, 2 ** 60)
    assert np.float32(float(x)) == m
    assert O.f32_round(x) == np.nextafter(m, np.float32(2))


def test_exact_sum_and_mean_are_exact_and_order_free():
    """The mean of the block constants is their exact arithmetic mean rounded once,
    whatever their range: brute force with Fractions, and invariance under reordering
    where an fp64 running sum is not."""
    from fractions import Fraction
    rng = np.random.default_rng(9)
    a = (rng.uniform(1, 2, 4000) * 2.0 ** rng.integers(-60, 11, 4000)).astype(np.float32)
    a[::97] = 0.0
    a[5] = np.float32(2.0 ** -149)            # smallest subnormal
    a[6] = np.float32(1.5 * 2.0 ** -130)      # subnormal
    brute = sum((Fraction(float(v)) for v in a), Fraction(0))
    assert O.exact_sum_f32(a) == brute
    mean = O.constants_mean(a)
    assert mean == O.f32_round(brute / a.size)
    perm = rng.permutation(a.size)
    assert O.constants_mean(a[perm]) == mean
    # an fp64 running sum is order-dependent on these data; the exact mean is not
    sums = {float(np.cumsum(a[rng.permutation(a.size)].astype(np.float64))[-1]) for _ in range(8)}
    assert len(sums) > 1
    # equal constants: the mean is the constant itself
    assert O.constants_mean(np.full(1000, np.float32(0.0371))) == np.float32(0.0371)
    # narrow-range data, where the fp64 sum is exact and its rounding cannot tie, give
    # the same mean as the fp64 formula
    b = rng.uniform(0.03, 0.09, 5000).astype(np.float32)
    assert O.constants_mean(b) == np.float32(np.sum(b.astype(np.float64)) / b.size)


def test_dq_codes_match_brute_force_over_t8():
    rng = np.random.default_rng(2)
    absmax = rng.uniform(0.02, 0.2, 600).astype(np.float32)
    c2, c1, mean = O.double_quantize(absmax)
    vals = O.fp8_code_to_t8(c2)
    cc = (absmax - mean).astype(np.float32)
    y = np.array([cc[i] / c1[i // 256] for i in range(600)], np.float32)
    t8, _ = O.fp8_table()
    for i in range(0, 600, 7):
        d = [abs(np.float32(y[i]) - t) for t in t8]
        assert vals[i] == t8[int(np.argmin(d))]
    assert not np.any(np.isnan(vals))


# --- bf16 rounding ----------------------------------------------------------

def test_bf16_round_matches_torch():
    x = np.random.default_rng(4).normal(0, 1, 100000).astype(np.float32)
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0]  # exact ties
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(O.bf16_round(x), ref)


# --- the uniform quantizer worked example (minnong511 "quantization", 1.) -----

def test_uniform_worked_example():
    g = {r[0]: float(r[1]) for r in read_golden("uniform_example.txt")}
    q, s, x_hat = O.uniform_affine_quantize(g["x"], g["x_min"], g["x_max"], int(g["bits"]))
    assert round(s, 4) == g["s"]
    assert q == g["q"]
    assert round(x_hat, 3) == g["x_hat"]
    assert round(x_hat - g["x"], 3) == g["error"]


# --- the linear layer -------------------------------------------------------

def _brute(X, W, A, B, scale):
    M, K = X.shape
    N, r = W.shape[0], A.shape[1]
    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(X[m, k]) * float(W[n, k])
            lora = 0.0
            for j in range(r):
                t = 0.0
                for k in range(K):
                    t += float(X[m, k]) * float(A[k, j])
                lora += t * float(B[j, n])
            Y[m, n] = acc + scale * lora
    return Y


@pytest.mark.parametrize("M,K,N,r", [(1, 4, 3, 1), (3, 8, 5, 2), (8, 8, 8, 4)])
def test_forward_matches_triple_loop(M, K, N, r):
    rng = np.random.default_rng(M * 100 + K)
    X, W = rng.normal(size=(M, K)), rng.normal(size=(N, K))
    A, B = rng.normal(size=(K, r)), rng.normal(size=(r, N))
    Y, T = O.linear_forward(X, W, A, B, 0.75)
    np.testing.assert_allclose(Y, _brute(X, W, A, B, 0.75), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(T, X @ A, rtol=1e-12)


def test_backward_adjoint_identities():
    rng = np.random.default_rng(9)
    M, K, N, r, scale = 5, 12, 7, 3, 1.5
    X, W = rng.normal(size=(M, K)), rng.normal(size=(N, K))
    A, B, dY = rng.normal(size=(K, r)), rng.normal(size=(r, N)), rng.normal(size=(M, N))
    dX, dA, dB = O.linear_backward(dY, X, W, A, B, scale)
    Y0, _ = O.linear_forward(X, W, A, B, scale)
    eps = 1e-3
    for which, grad in (("X", dX), ("A", dA), ("B", dB)):
        V = rng.normal(size=grad.shape)
        args = {"X": X, "A": A, "B": B}
        args[which] = args[which] + eps * V
        Y1, _ = O.linear_forward(args["X"], W, args["A"], args["B"], scale)
        lhs = np.sum(dY * (Y1 - Y0))
        rhs = eps * np.sum(grad * V)
        if which == "X":   # the layer is linear in X: exact up to rounding
            assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(rhs))
        else:              # bilinear in (A, B): first order in eps
            assert abs(lhs - rhs) <= 1e-2 * abs(rhs) + 1e-9


def test_special_cases_reduce_to_plain_products():
    rng = np.random.default_rng(12)
    M, K, N, r = 4, 16, 6, 2
    X, A, B = rng.normal(size=(M, K)), rng.normal(size=(K, r)), rng.normal(size=(r, N))
    W = rng.normal(size=(N, K))
    Y, _ = O.linear_forward(X, np.zeros((N, K)), A, B, 2.0)
    np.testing.assert_allclose(Y, 2.0 * X @ A @ B, rtol=1e-12)
    Y, _ = O.linear_forward(X, W, np.zeros((K, r)), B, 2.0)
    np.testing.assert_allclose(Y, X @ W.T, rtol=1e-12)
    dY = rng.normal(size=(M, N))
    dX, dA, dB = O.linear_backward(dY, X, W, A, np.zeros((r, N)), 2.0)
    np.testing.assert_allclose(dX, dY @ W, rtol=1e-12)
    assert np.all(dA == 0)


def test_quantized_weight_error_is_small():
    W = np.random.default_rng(3).normal(0, 0.02, (64, 256)).astype(np.float32)
    q = O.quantize_nf4_dq(W)
    What = O.double_dequant(q)
    assert np.mean(np.abs(What - W)) < 2e-3
    rows = np.array([0, 17, 63])
    np.testing.assert_array_equal(O.double_dequant_rows(q, rows), What[rows])
    cols = np.array([0, 1, 63, 64, 130, 255])  # both nibbles, block edges
    np.testing.assert_array_equal(O.double_dequant_cols(q, cols), What[:, cols])


# ---------------------------------------------------------------- merge_and_unload
def test_bf16_round_f64_is_one_rounding():
    """On fp32 inputs it agrees with the fp32 rounding (itself pinned against torch);
    exact ties go to the even neighbour; a value just above a tie rounds up, which
    rounding to fp32 first would turn into a tie and round down."""
    rng = np.random.default_rng(30)
    x = (rng.standard_normal(50000) * 10.0 ** rng.integers(-40, 30, 50000)).astype(np.float32)
    assert np.array_equal(O.bf16_round_f64(x.astype(np.float64)).view(np.uint32),
                          O.bf16_round(x).view(np.uint32))
    u = 2.0 ** -7  # bf16 spacing in [1, 2)
    assert list(O.bf16_round_f64(np.array([1 + u / 2, 1 + 3 * u / 2, -(1 + u / 2)]))) == \
        [1.0, 1.0 + 2 * u, -1.0]
    assert O.bf16_round_f64(np.array([1 + u / 2 + 2.0 ** -40]))[0] == np.float32(1 + u)
    assert O.bf16_round(np.array([1 + u / 2 + 2.0 ** -40], np.float32))[0] == np.float32(1.0)


def test_merge_special_cases():
    """A = 0 leaves the dequantized weight unchanged bit for bit; an all-zero base
    weight leaves bf16(scale (A B)^T), a plain matrix product."""
    rng = np.random.default_rng(31)
    N, K, r = 48, 192, 8
    q = O.quantize_nf4_dq(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    B = O.bf16_round(rng.normal(0, 0.02, (r, N)).astype(np.float32))
    _, merged = O.merge_lora(q, np.zeros((K, r)), B, 2.0)
    assert np.array_equal(merged.view(np.uint32), O.double_dequant(q).view(np.uint32))
    q0 = O.quantize_nf4_dq(np.zeros((N, K), np.float32))
    A = O.bf16_round(rng.normal(0, 0.02, (K, r)).astype(np.float32))
    _, merged = O.merge_lora(q0, A, B, 2.0)
    direct = np.einsum("kj,jn->nk", A.astype(np.float64), B.astype(np.float64)) * 2.0
    assert np.array_equal(merged.view(np.uint32), O.bf16_round_f64(direct).view(np.uint32))


def test_merged_weight_reproduces_the_layer_forward():
    """X W_merged^T equals the adapter-augmented forward up to the bf16 rounding of the
    merged weight (a transposed or unscaled LoRA product would not)."""
    rng = np.random.default_rng(32)
    M, N, K, r, scale = 6, 40, 128, 16, 0.5
    q = O.quantize_nf4_dq(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    A = O.bf16_round(rng.normal(0, 0.05, (K, r)).astype(np.float32))
    B = O.bf16_round(rng.normal(0, 0.05, (r, N)).astype(np.float32))
    X = O.bf16_round(rng.normal(0, 1, (M, K)).astype(np.float32)).astype(np.float64)
    _, merged = O.merge_lora(q, A, B, scale)
    Y, _ = O.linear_forward(X, O.double_dequant(q), A, B, scale)
    Ym = X @ merged.astype(np.float64).T
    half_ulp = np.ldexp(1.0, np.frexp(merged.astype(np.float64))[1] - 9)  # bf16 half spacing
    bound = np.abs(X) @ half_ulp.T + 1e-12
    assert np.all(np.abs(Ym - Y) <= bound)
    unmerged = X @ O.double_dequant(q).astype(np.float64).T  # the LoRA term left out
    assert not np.all(np.abs(unmerged - Y) <= bound)


# ---------------------------------------------------------------- codebook swap
def test_uniform_codebook_through_the_double_quantized_path():
    """The evenly spaced codebook goes through the same blocking, search, double
    quantization and doubleDequant: on the MAE workload its round-trip error without
    double quantization is the printed 1.71e-3 (1.46e-3 for NF4), and double quantization
    adds less than 1e-5 to it for either codebook; the stored weight remembers its levels."""
    pins = {r[0]: float(r[1]) for r in read_golden("mae_pins.txt")}
    w = np.random.default_rng(0).normal(0, 0.02, size=4096 * 64).astype(np.float32)
    for name, levels in (("nf4", O.nf4_levels()), ("uniform4", O.uniform4_levels())):
        codes, absmax = O.quantize_blocks(w, levels)
        plain = np.mean(np.abs(O.dequantize_blocks(codes, absmax, levels).astype(np.float64) - w))
        assert round(plain, 5) == pins[name], (name, plain)
        q = O.quantize_nf4_dq(w.reshape(64, 4096), levels)
        mae = np.mean(np.abs(O.double_dequant(q).astype(np.float64).ravel() - w))
        assert 0.0 <= mae - plain < 1e-5, (name, mae, plain)
    q = O.quantize_nf4_dq(w.reshape(64, 4096), O.uniform4_levels())
    assert np.array_equal(q["levels"], O.uniform4_levels())
    codes = O.unpack_nibbles(q["codes"])
    assert codes.min() == 0 and codes.max() == 15    # every block's max maps to +-1
    rows = np.array([0, 31, 63])
    np.testing.assert_array_equal(O.double_dequant_rows(q, rows), O.double_dequant(q)[rows])


def test_block_absmax_brute_force():
    """Block absmax against a plain loop over each 64-block (row-major flattening)."""
    rng = np.random.default_rng(31)
    w = (rng.standard_normal((6, 192)) * 0.02).astype(np.float32)
    w[2, 70] = -0.9                      # a negative extreme sets its block's absmax
    got = O.block_absmax(w)
    flat = w.ravel()
    want = [max(abs(float(v)) for v in flat[i:i + 64]) for i in range(0, flat.size, 64)]
    assert got.dtype == np.float32 and np.array_equal(got, np.float32(want))
    assert got[(2 * 192 + 70) // 64] == np.float32(0.9)


def test_sampled_weight_helper_matches_full_quantization():
    """The full-size GPU tests build their reference weight with oracle_sampled_weight
    (every constant, codes on sampled rows and 64-column blocks only). On a small weight
    it must give the full quantization's constants and codes there."""
    from tests.gpu_util import oracle_sampled_weight
    rng = np.random.default_rng(37)
    N, K = 40, 512
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    rows, blocks = np.array([0, 7, 39]), np.array([0, 3, 7])
    q_ref, codes_rows, codes_cols = oracle_sampled_weight(W, rows, blocks)
    full = O.quantize_nf4_dq(W)
    assert np.array_equal(q_ref["c2"], full["c2"]) and np.array_equal(q_ref["c1"], full["c1"])
    assert q_ref["mean"] == full["mean"]
    codes = full["codes"].reshape(N, K // 2)
    assert np.array_equal(codes_rows, codes[rows])
    assert np.array_equal(codes_cols, np.concatenate([codes[:, 32 * b:32 * (b + 1)] for b in blocks], 1))
    # and the reference weight's rows equal the full double dequantization there
    assert np.array_equal(O.double_dequant_rows(q_ref, rows), O.double_dequant(full)[rows])
