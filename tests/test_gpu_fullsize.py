"""Full-size parity in the launch configuration the benchmark times: the down projection
of the 7B-shaped layer (W 4096 x 11008, out x in), M = 4096 tokens, r = 64, alpha = 16.
The oracle computes sampled output columns of Y and dX one by one (fp64 dot products
over the exact bf16 inputs) and the LoRA gradients in full."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import assert_close, host, need_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", [(4096, 11008), (11008, 4096)])
def test_layer_linear_full_size_sampled(N, K):
    need_gpu()
    M, r, alpha = 4096, 64, 16.0
    case = inputs.linear_case(3, M, N, K, r, alpha)
    W, A, B, X, dY, scale = (case[k] for k in ("W", "A", "B", "X", "dY", "scale"))
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(W))
    Xd, Ad, Bd, dYd = to_dev_bf16(X), to_dev_bf16(A), to_dev_bf16(B), to_dev_bf16(dY)
    Y, T = qlora.qlora_linear_fwd(Xd, q, Ad, Bd, scale)
    dX, dA, dB = qlora.qlora_linear_bwd(dYd, Xd, T, q, Ad, Bd, scale)
    torch.cuda.synchronize()
    assert qlora.qlora_device_error() == 0

    # the stored weight as the library wrote it (its bit-exactness is tested elsewhere)
    ref = {"codes": q.codes.cpu().numpy(), "c2": q.c2.cpu().numpy(), "c1": q.c1.cpu().numpy(),
           "mean": np.float32(q.mean.cpu().numpy()[0]), "shape": (N, K)}
    rng = np.random.default_rng(17)
    X64, A64, B64, dY64 = (np.asarray(v, np.float64) for v in (X, A, B, dY))
    T64 = X64 @ A64
    G64 = dY64 @ B64.T
    # Y columns: one weight row each
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 48, replace=False)]))
    Wr = O.double_dequant_rows(ref, rows).astype(np.float64)          # [len(rows), K]
    Y_ref = X64 @ Wr.T + scale * (T64 @ B64[:, rows])
    assert_close(host(Y)[:, rows], O.bf16_round(Y_ref.astype(np.float32)), bf16_out=True, what="Y")
    # dX columns: one weight column each (all rows of W dequantized)
    What = O.double_dequant(ref)
    cols = np.unique(np.concatenate([[0, K - 1], rng.choice(K, 48, replace=False)]))
    dX_ref = dY64 @ What[:, cols].astype(np.float64) + scale * (G64 @ A64[cols].T)
    assert_close(host(dX)[:, cols], O.bf16_round(dX_ref.astype(np.float32)), bf16_out=True,
                 what="dX")
    # LoRA gradients in full
    assert_close(host(dA), scale * (X64.T @ G64), what="dA")
    assert_close(host(dB), scale * (T64.T @ dY64), what="dB")
    # the saved T
    assert_close(host(T), T64, what="T")


@pytest.mark.parametrize("N,K", [(8192, 8192), (22016, 8192), (8192, 22016)])
def test_65b_stack_linear_full_size_sampled(N, K):
    """The 65B-shaped stack's linears (q/k/v/o 8192 x 8192, gate/up 22016 x 8192, down
    8192 x 22016, out x in) at M = 8192 tokens, r = 64, alpha = 16, seed 4: Y and dX on
    sampled columns, the LoRA gradients in full."""
    need_gpu()
    M, r, alpha = 8192, 64, 16.0
    case = inputs.linear_case(4, M, N, K, r, alpha)
    W, A, B, X, dY, scale = (case[k] for k in ("W", "A", "B", "X", "dY", "scale"))
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(W))
    del W
    Xd, Ad, Bd, dYd = to_dev_bf16(X), to_dev_bf16(A), to_dev_bf16(B), to_dev_bf16(dY)
    Y, T = qlora.qlora_linear_fwd(Xd, q, Ad, Bd, scale)
    dX, dA, dB = qlora.qlora_linear_bwd(dYd, Xd, T, q, Ad, Bd, scale)
    torch.cuda.synchronize()
    assert qlora.qlora_device_error() == 0
    del Xd, dYd

    ref = {"codes": q.codes.cpu().numpy(), "c2": q.c2.cpu().numpy(), "c1": q.c1.cpu().numpy(),
           "mean": np.float32(q.mean.cpu().numpy()[0]), "shape": (N, K)}
    rng = np.random.default_rng(19)
    A64, B64 = np.asarray(A, np.float64), np.asarray(B, np.float64)
    X64, dY64 = np.asarray(X, np.float64), np.asarray(dY, np.float64)
    del X, dY
    T64 = X64 @ A64
    G64 = dY64 @ B64.T
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 24, replace=False)]))
    Wr = O.double_dequant_rows(ref, rows).astype(np.float64)
    Y_ref = X64 @ Wr.T + scale * (T64 @ B64[:, rows])
    assert_close(host(Y[:, rows]), O.bf16_round(Y_ref.astype(np.float32)), bf16_out=True, what="Y")
    cols = np.unique(np.concatenate([[0, K - 1], rng.choice(K, 24, replace=False)]))
    Wc = O.double_dequant_cols(ref, cols).astype(np.float64)
    dX_ref = dY64 @ Wc + scale * (G64 @ A64[cols].T)
    assert_close(host(dX[:, cols]), O.bf16_round(dX_ref.astype(np.float32)), bf16_out=True,
                 what="dX")
    assert_close(host(dA), scale * (X64.T @ G64), what="dA")
    assert_close(host(dB), scale * (T64.T @ dY64), what="dB")
    assert_close(host(T), T64, what="T")
