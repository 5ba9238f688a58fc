"""GPU parity of the codec (quantize, double quantization, dequant) against the oracle.
Codes, c2, c1, mean and the dequantized bf16 weights must be bit-exact."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import host, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def quantize_on_gpu(W, bf16):
    t = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    if bf16:
        t = t.to(torch.bfloat16)
    q = qlora.qlora_quantize_nf4_dq(t)
    torch.cuda.synchronize()
    return q


def compare_full(W, bf16):
    q = quantize_on_gpu(W, bf16)
    ref = O.quantize_nf4_dq(W)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(q.c2.cpu().numpy(), ref["c2"])
    assert np.array_equal(q.c1.cpu().numpy().view(np.uint32), ref["c1"].view(np.uint32))
    assert q.mean.cpu().numpy().view(np.uint32)[0] == np.float32(ref["mean"]).view(np.uint32)
    wd = qlora.qlora_dequant(q)
    torch.cuda.synchronize()
    got = wd.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.bf16_bits(O.double_dequant(ref)))
    return q, ref


def test_pr1_weight_bit_exact():
    case = inputs.pr1()
    compare_full(case["W"], bf16=False)


@pytest.mark.parametrize("shape", [(5, 192), (1, 64), (3, 4096), (64, 11008), (300, 704)])
def test_ragged_and_small_shapes(shape):
    rng = np.random.default_rng(sum(shape))
    W = inputs.to_bf16_values(rng.normal(0, 0.02, shape).astype(np.float32))
    compare_full(W, bf16=True)


def test_mean_exact_for_wide_range_constants():
    """Block absmax values from 2^-60 to 2^10 (fp32 input): the fp64 sum of such constants
    is not exact and depends on its order, but the mean is defined as the exact
    arithmetic mean rounded once to fp32, so the GPU must match the oracle bit for bit
    (and the constants and codes with it). Also a tensor of 2^17 blocks with a few tiny
    blocks among normal ones, and a subnormal block."""
    rng = np.random.default_rng(33)
    n_rows, k = 512, 1024                     # 8192 blocks
    W = rng.normal(0, 1, (n_rows, k)).astype(np.float32)
    scale = 2.0 ** rng.integers(-60, 11, n_rows * k // 64)
    W = (W.reshape(-1, 64) * scale[:, None]).astype(np.float32).reshape(n_rows, k)
    W[7, 64:128] = np.float32(2.0 ** -140)    # a block of subnormals
    W[9, :64] = 0.0
    q, ref = compare_full(W, bf16=False)
    a64 = ref["absmax"].astype(np.float64)
    assert len({float(np.cumsum(a64[rng.permutation(a64.size)])[-1]) for _ in range(6)}) > 1

    g = np.random.default_rng(34)
    W2 = g.normal(0, 0.02, (512, 16384)).astype(np.float32)
    W2[::67, ::4096] *= np.float32(2.0 ** -40)
    q2 = quantize_on_gpu(W2, bf16=False)
    codes, absmax = O.quantize_blocks(W2[:8], O.nf4_levels())   # codes on sampled rows
    full_absmax = np.max(np.abs(W2.reshape(-1, 64)), axis=1)
    c2, c1, mean = O.double_quantize(full_absmax)
    assert q2.mean.cpu().numpy().view(np.uint32)[0] == np.float32(mean).view(np.uint32)
    assert np.array_equal(q2.c2.cpu().numpy(), c2)
    assert np.array_equal(q2.c1.cpu().numpy().view(np.uint32), c1.view(np.uint32))
    got_codes = q2.codes.cpu().numpy()[: 8 * 16384 // 2]
    assert np.array_equal(got_codes, O.pack_nibbles(codes))


def test_mean_rounding_edges():
    """Means at the bottom of the fp32 range, where the exact mean is rounded to a
    subnormal, to the smallest subnormal or to zero: the GPU's division of the exact sum
    must round as the oracle does."""
    for tiny, zeros in [(2.0 ** -149, 1), (2.0 ** -149, 2), (3 * 2.0 ** -149, 3), (2.0 ** -149, 3),
                        (3 * 2.0 ** -149, 5), (2.0 ** -126, 7), (1.5 * 2.0 ** -140, 63)]:
        W = np.zeros((1 + zeros, 64), np.float32)
        W[0, 17] = np.float32(tiny)
        compare_full(W, bf16=False)


def test_edge_values():
    rng = np.random.default_rng(21)
    W = rng.normal(0, 0.02, (40, 640)).astype(np.float32)
    W[0] = 0.0                                 # all-zero rows / blocks
    W[1, :64] = 0.0
    W[2, 5] = 7.5                              # isolated outliers of both signs
    W[3, 70] = -9.0
    W[4] = 1e-30                               # tiny magnitudes
    W[5, :64] = -0.5                           # constant blocks
    W[6, 64:128] = np.float32(2.0 ** -20) * np.arange(64)
    # absmax on both sides of 2^-64 (the quantizer's switch between its reciprocal-based
    # and its plain division), subnormal elements, and a block of subnormals only
    W[7, :64] = rng.normal(0, 1, 64) * 2.0 ** -62
    W[7, 64:128] = rng.normal(0, 1, 64) * 2.0 ** -66
    W[7, 128:192] = rng.normal(0, 1, 64) * 2.0 ** -66
    W[7, 130] = 2.0 ** -64
    W[7, 192:256] = rng.normal(0, 1, 64) * 2.0 ** -66
    W[7, 200] = np.nextafter(np.float32(2.0 ** -64), np.float32(0))
    W[8, :64] = rng.normal(0, 1, 64) * 1e-40
    W[8, 64:128] = rng.normal(0, 1, 64) * 1e-40
    W[8, 100] = 0.03
    compare_full(W, bf16=False)


def test_codes_at_every_threshold_window():
    """Blocks whose absmax is exactly 1 carry x = w unchanged, so weights taken from
    windows around every NF4 decision threshold probe the code search directly."""
    th = qlora.nf4_thresholds().numpy()
    probes = []
    for t in th:
        x = np.float32(t)
        lo = hi = x
        probes.append(x)
        for _ in range(300):
            lo = np.nextafter(lo, np.float32(-2))
            hi = np.nextafter(hi, np.float32(2))
            probes += [lo, hi]
    probes = np.array(probes, np.float32)
    probes = np.concatenate([probes, O.nf4_levels(), np.array([0.0, -0.0], np.float32)])
    per = 63
    nblk = -(-probes.size // per)
    nblk = -(-nblk // 10) * 10             # whole rows of 640 weights
    probes = np.concatenate([probes, np.zeros(nblk * per - probes.size, np.float32)])
    W = np.concatenate([np.ones((nblk, 1), np.float32), probes.reshape(nblk, per)], axis=1)
    W = W.reshape(-1, 640)[: (nblk * 64) // 640]
    q = quantize_on_gpu(W, bf16=False)
    codes, _ = O.quantize_blocks(W, O.nf4_levels())
    assert np.array_equal(q.codes.cpu().numpy(), O.pack_nibbles(codes))


@pytest.mark.parametrize("n,k", [(4096, 4096), (4096, 11008), (11008, 4096)])
def test_llama7b_shapes_with_outliers(n, k):
    """Full-size codec case: all constants compared, codes and dequantized weights on
    sampled rows (the oracle quantizes rows independently once the mean is known)."""
    rng = np.random.default_rng(1)
    W = inputs.weight(rng, n, k, bf16=True, outlier_frac=1e-3)
    q = quantize_on_gpu(W, bf16=True)
    absmax = np.max(np.abs(W.reshape(-1, 64)), axis=1)   # block absmax (exact in fp32)
    c2, c1, mean = O.double_quantize(absmax)
    assert q.mean.cpu().numpy()[0] == mean
    assert np.array_equal(q.c1.cpu().numpy().view(np.uint32), c1.view(np.uint32))
    assert np.array_equal(q.c2.cpu().numpy(), c2)
    rows = np.unique(np.concatenate([[0, n - 1], rng.choice(n, 256, replace=False)]))
    codes, _ = O.quantize_blocks(W[rows], O.nf4_levels())
    got = q.codes.cpu().numpy().reshape(n, k // 2)[rows]
    assert np.array_equal(got.ravel(), O.pack_nibbles(codes))
    ref = {"codes": q.codes.cpu().numpy(), "c2": c2, "c1": c1, "mean": mean, "shape": (n, k)}
    wd = qlora.qlora_dequant(q)
    torch.cuda.synchronize()
    got_w = wd.view(torch.int16).cpu().numpy().view(np.uint16)[rows]
    assert np.array_equal(got_w, O.bf16_bits(O.double_dequant_rows(ref, rows)))
    # round-trip error stays at the NF4 level
    mae = np.mean(np.abs(host(wd)[rows] - W[rows]))
    assert mae < 2.5e-3


def test_dequant_of_handmade_constants():
    """Dequantize constants that no quantizer would produce (negative and subnormal
    scales, every E4M3 code) and compare with the definition."""
    n, k = 16, 1024
    nb = n * k // 64
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 256, n * k // 2).astype(np.uint8)
    c2 = np.array([b for b in range(256) if b not in (0x7F, 0xFF)] * 2, np.uint8)[:nb]
    c1 = np.array([0.37, -0.0, 1e-38, 3.0], np.float32)[: -(-nb // 256)]
    mean = np.float32(-0.01)
    ref = {"codes": codes, "c2": c2, "c1": c1, "mean": mean, "shape": (n, k)}
    q = qlora.NF4Weight(torch.from_numpy(codes).cuda(), torch.from_numpy(c2).cuda(),
                        torch.from_numpy(c1).cuda(), torch.tensor([mean]).cuda(), n, k)
    wd = qlora.qlora_dequant(q)
    torch.cuda.synchronize()
    got = wd.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.bf16_bits(O.double_dequant(ref)))


def test_double_quantization_at_every_t8_threshold():
    """Block constants that put y = fl32(cc / c1) on the fp32 grid (step 2^-23) around
    every decision boundary of the T8 search, on both signs. Each 256-block of constants
    holds 0 and 2 (so c1 = 1) and pairs 1 + d, 1 - d; the fp64 sum is exact, so the mean
    is exactly 1, cc = +-d exactly and y = +-d. Probes sit from two steps below to two
    steps above each midpoint of consecutive non-negative T8 entries."""
    t8_vals, _ = O.fp8_table()
    pos = np.sort(t8_vals[t8_vals >= 0].astype(np.float64))
    mids = (pos[:-1] + pos[1:]) / 2
    step = 2.0 ** -23
    d = np.unique(np.concatenate([(np.floor(mids / step) + j) * step for j in range(-2, 3)]))
    d = d[(d > 0) & (d < 1)].astype(np.float32)
    free = 127                                    # pairs per 256-block besides 0 and 2
    nblk = -(-d.size // free)
    d = np.concatenate([d, np.zeros(nblk * free - d.size, np.float32)])
    a = []
    for b in range(nblk):
        seg = d[b * free:(b + 1) * free]
        a.append(np.concatenate([[0.0, 2.0], 1.0 + seg, 1.0 - seg]).astype(np.float32))
    a = np.concatenate(a)
    assert np.array_equal((1.0 + d).astype(np.float32) - np.float32(1.0), d)  # exact grid
    W = np.zeros((a.size, 64), np.float32)
    W[:, 0] = a                                   # one weight per block carries its absmax
    W = W.reshape(-1, 640)
    ref = O.quantize_nf4_dq(W)
    assert np.float32(ref["mean"]) == np.float32(1.0)
    compare_full(W, bf16=False)
