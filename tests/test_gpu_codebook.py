"""The evenly spaced 4-bit codebook (itwiki "QLoRA", section "4비트 NormalFloat(NF4)":
the uniform 4-bit comparison) through the same kernels: quantization and double
dequantization bit-exact, the linear layer (GEMM and decode paths) and the merge
within the tolerances of the NF4 tests."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import need_gpu
from tests.test_gpu_linear import run_case
from tests.test_gpu_merge import check_rows, to_dev_bf16

pytestmark = pytest.mark.gpu
U = qlora.CODEBOOK_UNIFORM4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


@pytest.mark.parametrize("bf16", [False, True])
def test_uniform_codec_bit_exact(bf16):
    rng = np.random.default_rng(40)
    W = rng.normal(0, 0.02, (96, 640)).astype(np.float32)
    W[0] = 0.0
    W[2, 5] = 7.5
    W[4] = 1e-30
    W[5, :64] = -0.5
    W[7, :64] = rng.normal(0, 1, 64) * 2.0 ** -66
    W[8, :64] = np.linspace(-1, 1, 64) * 0.37          # values around every uniform level
    Wt = torch.from_numpy(W).cuda()
    if bf16:
        Wt = Wt.to(torch.bfloat16)
        W = Wt.float().cpu().numpy()
    q = qlora.qlora_quantize_nf4_dq(Wt, codebook=U)
    ref = O.quantize_nf4_dq(W, O.uniform4_levels())
    assert q.codebook == U
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(q.c2.cpu().numpy(), ref["c2"])
    assert np.array_equal(q.c1.cpu().numpy().view(np.uint32), ref["c1"].view(np.uint32))
    wd = qlora.qlora_dequant(q)
    torch.cuda.synchronize()
    got = wd.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.bf16_bits(O.double_dequant(ref)))
    # the same codes read as NF4 would give other weights: the codebook is really used
    q.codebook = qlora.CODEBOOK_NF4
    assert not torch.equal(qlora.qlora_dequant(q).view(torch.int16), wd.view(torch.int16))


@pytest.mark.parametrize("M,N,K,r", [(300, 384, 640, 16), (257, 512, 576, 64)])
def test_uniform_gemm_path(M, N, K, r):
    run_case(inputs.linear_case(500 + M, M, N, K, r, alpha=2 * r), codebook=U)


@pytest.mark.parametrize("M", [1, 16])
def test_uniform_decode_path(M):
    run_case(inputs.linear_case(520 + M, M, 256, 2048, 16, alpha=32), codebook=U)


def test_uniform_merge():
    case = inputs.linear_case(530, 4, 136, 1024, 64, alpha=16.0)
    q_np = O.quantize_nf4_dq(case["W"], O.uniform4_levels())
    q = qlora.qlora_quantize_nf4_dq(torch.from_numpy(case["W"]).cuda(), codebook=U)
    got = qlora.qlora_merge_lora(q, to_dev_bf16(case["A"]), to_dev_bf16(case["B"]), 0.25)
    torch.cuda.synchronize()
    check_rows(got.float().cpu().numpy(), q_np, case["A"], case["B"], 0.25, np.arange(136))
