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
