"""GPU parity of the QLoRA linear forward and backward against the fp64 oracle
(rel-Frobenius <= 2e-3, elementwise <= 2e-2 on unit-scale outputs)."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import assert_close, host, need_gpu, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def run_case(case, w_bf16=True, check_T=True, codebook=0):
    W, A, B, X, dY, r, scale = (case[k] for k in ("W", "A", "B", "X", "dY", "r", "scale"))
    Wt = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    q = qlora.qlora_quantize_nf4_dq(Wt.to(torch.bfloat16) if w_bf16 else Wt, codebook=codebook)
    Xd, Ad, Bd, dYd = to_dev_bf16(X), to_dev_bf16(A), to_dev_bf16(B), to_dev_bf16(dY)
    Y, T = qlora.qlora_linear_fwd(Xd, q, Ad, Bd, scale)
    dX, dA, dB = qlora.qlora_linear_bwd(dYd, Xd, T, q, Ad, Bd, scale)
    torch.cuda.synchronize()
    assert qlora.qlora_device_error() == 0
    ref = O.quantize_nf4_dq(W, O.uniform4_levels() if codebook == 1 else None)
    What = O.double_dequant(ref)
    Y64, T64 = O.linear_forward(X, What, A, B, scale)
    dX64, dA64, dB64 = O.linear_backward(dY, X, What, A, B, scale, T=T64)
    assert_close(host(Y), O.bf16_round(Y64.astype(np.float32)), bf16_out=True, what="Y")
    if check_T:
        assert_close(host(T), T64, what="T")
    assert_close(host(dX), O.bf16_round(dX64.astype(np.float32)), bf16_out=True, what="dX")
    assert_close(host(dA), dA64, what="dA")
    assert_close(host(dB), dB64, what="dB")
    return q


def test_pr1_reference_case():
    """One linear 512x1024, r=8, alpha=16, M=16 (decode kernels for the forward)."""
    run_case(inputs.pr1(), w_bf16=False)


@pytest.mark.parametrize("M,N,K,r", [
    (300, 384, 640, 16),    # ragged M over two 256-token tiles, 3 weight tiles, 10 k-steps
    (257, 512, 576, 64),    # K % 128 == 64: half-filled dX tile
    (40, 136, 1024, 8),     # N % 128 != 0, few tokens, GEMM path
    (512, 1024, 1024, 64),
])
def test_gemm_path_shapes(M, N, K, r):
    run_case(inputs.linear_case(100 + M, M, N, K, r, alpha=2 * r))


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_path_small_m(M):
    run_case(inputs.linear_case(200 + M, M, 256, 2048, 16, alpha=32))


@pytest.mark.parametrize("M,N,K,r", [
    (2, 136, 576, 8),      # last 16-row group half full; K ends 64 columns into a 256-wide unit
    (3, 1024, 2048, 64),
    (7, 264, 1280, 16),
    (8, 512, 4096, 16),    # the largest M of the one-MMA-per-step kernel
    (9, 136, 576, 8),      # the smallest M of the two-MMA kernel, ragged as above
    (12, 1024, 3072, 32),
    (15, 256, 2048, 64),
    (16, 48000, 256, 16),  # one K split: 21 row groups per CTA, so some warps take two
])
def test_decode_path_shapes(M, N, K, r):
    """The decode kernels at token counts between the bench's, with ragged row groups and
    units, every rank class, and warps that take more than one row group."""
    run_case(inputs.linear_case(300 + M, M, N, K, r, alpha=2 * r))


def test_zero_weight_isolates_lora_term():
    case = inputs.linear_case(7, 300, 256, 512, 16, alpha=32)
    case["W"] = np.zeros_like(case["W"])
    q = run_case(case)
    assert torch.count_nonzero(qlora.qlora_dequant(q)) == 0


def test_zero_adapter_isolates_base_term():
    case = inputs.linear_case(8, 300, 256, 512, 16, alpha=32)
    case["A"] = np.zeros_like(case["A"])
    case["B"] = np.zeros_like(case["B"])
    q = run_case(case)
    # and against a plain PyTorch fp32 product with the library's own dequantized weight
    Xd = to_dev_bf16(case["X"])
    Y, _ = qlora.qlora_linear_fwd(Xd, q, to_dev_bf16(case["A"]), to_dev_bf16(case["B"]), 2.0)
    ref = (Xd.float() @ qlora.qlora_dequant(q).float().T)
    assert_close(host(Y), O.bf16_round(host(ref)), bf16_out=True, what="Y vs torch")


def test_recompute_T_and_skip_dX():
    case = inputs.linear_case(9, 260, 256, 512, 16, alpha=32)
    W, A, B, X, dY, scale = (case[k] for k in ("W", "A", "B", "X", "dY", "scale"))
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(W))
    Xd, Ad, Bd, dYd = to_dev_bf16(X), to_dev_bf16(A), to_dev_bf16(B), to_dev_bf16(dY)
    _, T = qlora.qlora_linear_fwd(Xd, q, Ad, Bd, scale)
    dX1, dA1, dB1 = qlora.qlora_linear_bwd(dYd, Xd, T, q, Ad, Bd, scale)
    dX2, dA2, dB2 = qlora.qlora_linear_bwd(dYd, Xd, None, q, Ad, Bd, scale, need_dX=False)
    torch.cuda.synchronize()
    assert dX2 is None
    assert torch.equal(dA1, dA2) and torch.equal(dB1, dB2)


def test_empty_batch():
    q = qlora.qlora_quantize_nf4_dq(torch.randn(128, 256, device="cuda"))
    A = torch.zeros(256, 8, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(8, 128, dtype=torch.bfloat16, device="cuda")
    X = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    Y, _ = qlora.qlora_linear_fwd(X, q, A, B, 1.0, save_T=False)
    dA = torch.full((256, 8), 5.0, device="cuda")
    dB = torch.full((8, 128), 5.0, device="cuda")
    qlora.qlora_linear_bwd(torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda"), X, None, q,
                           A, B, 1.0, need_dX=False, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert Y.shape == (0, 128) and torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0


def _tiles(rows, M):
    return -(-rows // 128) * -(-M // 512)


@pytest.mark.parametrize("M,N,K,r", [
    (600, 10368, 512, 16),   # forward: 81 x 2 = 162 tiles, a second partial wave of CTAs
    (600, 256, 10368, 16),   # dX: 81 x 2 tiles along K, 4 code steps per tile
    (700, 9600, 256, 8),     # forward: 75 x 2 = 150 tiles, the second token tile one accumulator
])
def test_more_tiles_than_sms(M, N, K, r):
    """More weight x token tiles than SMs, not a multiple of them: the persistent CTAs take
    a second tile each until the tiles run out (full oracle comparison)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert max(_tiles(N, M), _tiles(K, M)) > sms
    run_case(inputs.linear_case(300 + M + r, M, N, K, r, alpha=2 * r))


def test_graph_replay_matches_eager():
    """Forward and backward captured once in a CUDA graph and replayed on new inputs, with
    workspaces that start as all-ones bytes: every replay equals the eager calls bit for bit."""
    M, N, K, r = 600, 10368, 512, 16
    case = inputs.linear_case(41, M, N, K, r, alpha=32)
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(case["W"]))
    Ad, Bd = to_dev_bf16(case["A"]), to_dev_bf16(case["B"])
    scale = case["scale"]
    g = torch.Generator(device="cuda").manual_seed(5)
    draws = [(torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16),
              torch.randn(M, N, device="cuda", generator=g).to(torch.bfloat16)) for _ in range(3)]
    eager = []
    for Xd, dYd in draws:
        Y, T = qlora.qlora_linear_fwd(Xd, q, Ad, Bd, scale)
        dX, dA, dB = qlora.qlora_linear_bwd(dYd, Xd, T, q, Ad, Bd, scale)
        eager.append((Y, dX, dA, dB))
    # static buffers
    Xs, dYs = draws[0][0].clone(), draws[0][1].clone()
    Ys = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    Ts = torch.empty(M, r, dtype=torch.float32, device="cuda")
    dXs = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dAs = torch.empty(K, r, dtype=torch.float32, device="cuda")
    dBs = torch.empty(r, N, dtype=torch.float32, device="cuda")
    wf = torch.full((qlora.qlora_linear_fwd_workspace_size(M, N, K, r),), 255, dtype=torch.uint8,
                    device="cuda")
    wb = torch.full((qlora.qlora_linear_bwd_workspace_size(M, N, K, r),), 255, dtype=torch.uint8,
                    device="cuda")

    def step():
        qlora.qlora_linear_fwd(Xs, q, Ad, Bd, scale, Y=Ys, T=Ts, workspace=wf)
        qlora.qlora_linear_bwd(dYs, Xs, Ts, q, Ad, Bd, scale, dX=dXs, dA=dAs, dB=dBs, workspace=wb)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    for i, (Xd, dYd) in enumerate(draws):
        Xs.copy_(Xd)
        dYs.copy_(dYd)
        graph.replay()
        torch.cuda.synchronize()
        assert qlora.qlora_device_error() == 0
        for got, want, name in zip((Ys, dXs, dAs, dBs), eager[i], ("Y", "dX", "dA", "dB")):
            assert torch.equal(got, want), f"replay {i}: {name}"
    del graph


def test_launch_count_per_call():
    """The library counts its own kernels: 3 per GEMM-path forward (T, its finalize, the
    fused GEMM), 5 per backward with T saved (G, its finalize, the fused dX GEMM, the
    grouped dA/dB GEMM and its finalize), 2 per decode-path forward, 3 per quantization
    (clearing its accumulators, level 1, the double quantization)."""
    case = inputs.linear_case(51, 300, 256, 512, 16, alpha=32)
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(case["W"]))
    Xd, Ad, Bd, dYd = (to_dev_bf16(case[k]) for k in ("X", "A", "B", "dY"))
    n0 = qlora.qlora_launch_count()
    _, T = qlora.qlora_linear_fwd(Xd, q, Ad, Bd, case["scale"])
    n1 = qlora.qlora_launch_count()
    qlora.qlora_linear_bwd(dYd, Xd, T, q, Ad, Bd, case["scale"])
    n2 = qlora.qlora_launch_count()
    qlora.qlora_linear_fwd(Xd[:4].contiguous(), q, Ad, Bd, case["scale"])
    n3 = qlora.qlora_launch_count()
    qlora.qlora_quantize_nf4_dq(to_dev_bf16(case["W"]))
    n4 = qlora.qlora_launch_count()
    torch.cuda.synchronize()
    assert (n1 - n0, n2 - n1, n3 - n2, n4 - n3) == (3, 5, 2, 3)
