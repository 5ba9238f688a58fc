"""Helpers of the GPU parity tests (tolerances and host<->device moves)."""
import numpy as np
import pytest
import torch

REL_FRO = 2e-3   # relative Frobenius error bound on GEMM outputs and gradients
ABS = 2e-2       # elementwise bound on unit-scale outputs (scaled by max(1, rms(ref)))


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_nf4_quantized_unpack_b200 import build
    build.build()


def to_dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).cuda()


def to_dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def host(t):
    return t.detach().float().cpu().numpy()


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def assert_close(got, ref, bf16_out=False, what=""):
    """rel-Frobenius <= 2e-3 and |got - ref| <= 2e-2 * max(1, rms(ref)); a bf16 output
    may also differ by one bf16 ulp where fp32 and fp64 accumulation round apart."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    nrm = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / max(nrm, 1e-30)
    assert rel <= REL_FRO, f"{what}: rel-Frobenius {rel:.3e}"
    scale = max(1.0, float(np.sqrt(np.mean(ref ** 2))))
    bound = ABS * scale
    if bf16_out:
        bound = np.maximum(bound, bf16_ulp(ref) * 1.0001)
    err = np.abs(got - ref)
    bad = err > bound
    assert not np.any(bad), f"{what}: {bad.sum()} elements over the bound, max err {err.max():.3e}"
    return rel


def oracle_sampled_weight(W, rows, col_blocks, levels=None):
    """The oracle's quantization of W [N, K] where full-size tests look: every block
    constant (the absmax of all blocks, then their double quantization with one mean),
    and the codes of the sampled rows and of the sampled 64-column blocks of every row.
    Returns (q_ref, codes_rows [len(rows), K/2], codes_cols [N, 32 * len(col_blocks)]);
    q_ref holds the oracle's constants and those codes (zeros elsewhere), for
    double_dequant_rows / double_dequant_cols on the sampled rows and columns."""
    from oracle import nf4_oracle as O
    W = np.asarray(W, np.float32)
    N, K = W.shape
    levels = O.nf4_levels() if levels is None else levels
    c2, c1, mean = O.double_quantize(O.block_absmax(W))
    codes = np.zeros((N, K // 2), np.uint8)
    rc, _ = O.quantize_blocks(W[rows], levels)
    codes_rows = O.pack_nibbles(rc).reshape(len(rows), K // 2)
    cols = []
    for b in col_blocks:
        cc, _ = O.quantize_blocks(W[:, 64 * b:64 * (b + 1)], levels)
        cols.append(O.pack_nibbles(cc).reshape(N, 32))
        codes[:, 32 * b:32 * (b + 1)] = cols[-1]
    codes[rows] = codes_rows
    q_ref = {"codes": codes.ravel(), "c2": c2, "c1": c1, "mean": mean, "shape": (N, K),
             "levels": levels}
    return q_ref, codes_rows, np.concatenate(cols, axis=1)


def assert_weight_matches_oracle(q, q_ref, rows, col_blocks, codes_rows, codes_cols):
    """The library's quantized weight against the oracle's: mean, c1 and c2 in full,
    codes on the sampled rows and column blocks, all bit for bit."""
    N, K = q_ref["shape"]
    assert q.mean.cpu().numpy().view(np.uint32)[0] == np.float32(q_ref["mean"]).view(np.uint32)
    assert np.array_equal(q.c1.cpu().numpy().view(np.uint32), q_ref["c1"].view(np.uint32))
    assert np.array_equal(q.c2.cpu().numpy(), q_ref["c2"])
    got = q.codes.cpu().numpy().reshape(N, K // 2)
    assert np.array_equal(got[rows], codes_rows)
    got_cols = np.concatenate([got[:, 32 * b:32 * (b + 1)] for b in col_blocks], axis=1)
    assert np.array_equal(got_cols, codes_cols)
