"""merge_and_unload on the GPU (qlora_merge_lora) against the oracle's merge_lora.

W_merged = bf16(W_hat + scale (A B)^T). The library forms the rank-r product in fp32 on
the tensor cores; the oracle sums exactly and rounds once. The two must agree bit for bit
except where the exact sum lies within the fp32 error bound of a bf16 rounding boundary;
there they may differ by one bf16 ulp, and such elements must be rare.
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu


def to_dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda().to(torch.bfloat16)


def check_rows(got, q, A, B, scale, rows):
    """got: merged bf16 rows (fp32 values) of the GPU; compares them with the oracle."""
    A64, B64 = A.astype(np.float64), B.astype(np.float64)
    W_hat = O.double_dequant_rows(q, rows).astype(np.float64)
    delta = (A64 @ B64[:, rows]).T
    exact = W_hat + scale * delta
    ref = O.bf16_round_f64(exact)
    r = A.shape[1]
    beta = 2.0 ** -22 * (r * abs(scale) * (np.abs(A64) @ np.abs(B64[:, rows])).T
                         + np.abs(W_hat) + np.abs(exact)) + 1e-45
    diff = got != ref
    mid = (got.astype(np.float64) + ref.astype(np.float64)) / 2
    near = np.abs(exact - mid) <= beta
    ulp = np.ldexp(1.0, np.maximum(np.frexp(ref.astype(np.float64))[1] - 8, -133))  # bf16 spacing
    one_ulp = np.abs(got.astype(np.float64) - ref) <= ulp
    assert np.all(~diff | (near & one_ulp)), "a merged element differs away from a rounding boundary"
    assert diff.mean() < 1e-3
    return diff.mean()


@pytest.mark.parametrize("N,K,r,scale", [(512, 1024, 8, 2.0), (72, 192, 24, 0.5), (136, 1024, 64, 0.25)])
def test_merge_matches_oracle(N, K, r, scale):
    need_gpu()
    case = inputs.linear_case(400 + r, 4, N, K, r, alpha=scale * r)
    q_np = O.quantize_nf4_dq(case["W"])
    q = qlora.qlora_quantize_nf4_dq(torch.from_numpy(case["W"]).cuda())
    A, B = case["A"], case["B"]
    got = qlora.qlora_merge_lora(q, to_dev_bf16(A), to_dev_bf16(B), scale)
    torch.cuda.synchronize()
    got = got.float().cpu().numpy()
    check_rows(got, q_np, A, B, scale, np.arange(N))


def test_merge_without_adapter_is_the_dequantized_weight():
    need_gpu()
    case = inputs.linear_case(410, 4, 256, 512, 16, alpha=32.0)
    q = qlora.qlora_quantize_nf4_dq(torch.from_numpy(case["W"]).cuda())
    zeros = torch.zeros(512, 16, dtype=torch.bfloat16, device="cuda")
    got = qlora.qlora_merge_lora(q, zeros, to_dev_bf16(case["B"]), 2.0)
    ref = qlora.qlora_dequant(q)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_merge_llama_shape_sampled_rows():
    """4096 x 11008 (out x in) at r = 64: the whole weight merged on the GPU, rows sampled
    for the oracle."""
    need_gpu()
    N, K, r, scale = 4096, 11008, 64, 0.25
    g = np.random.default_rng(6)
    W = inputs.weight(g, N, K)
    A = O.bf16_round(g.normal(0, 0.02, (K, r)).astype(np.float32))
    B = O.bf16_round(g.normal(0, 0.02, (r, N)).astype(np.float32))
    q = qlora.qlora_quantize_nf4_dq(torch.from_numpy(W).cuda())
    got = qlora.qlora_merge_lora(q, to_dev_bf16(A), to_dev_bf16(B), scale)
    torch.cuda.synchronize()
    q_np = {"codes": q.codes.cpu().numpy(), "c2": q.c2.cpu().numpy(), "c1": q.c1.cpu().numpy(),
            "mean": np.float32(q.mean.cpu().numpy()[0]), "shape": (N, K)}
    rows = np.sort(g.choice(N, 48, replace=False))
    check_rows(got[rows].float().cpu().numpy(), q_np, A, B, scale, rows)
