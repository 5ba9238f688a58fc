"""Full-size parity in the launch configurations the benchmark times.

* The 7B-shaped layer's down and gate linears (W 4096 x 11008 and 11008 x 4096, out x
  in) at M = 4096 tokens, r = 64, alpha = 16, seed 3.
* The 65B-shaped stack's linears (8192 x 8192, 22016 x 8192, 8192 x 22016) at M = 8192,
  seed 4.
* The decode forward on 4096 x 11008 and 8192 x 28672 at M = 1, 4 and 16, r = 16,
  alpha = 32, seed 2.

The reference weight is the oracle's own quantization of W: every block constant (one
mean, c1, c2) is compared with the library's bit for bit, and the codes on the sampled
rows and 64-column blocks. The oracle computes sampled output columns of Y (one weight
row each) and dX (one weight column each) as fp64 dot products over the exact bf16
inputs; T, dA and dB are checked in full."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import (assert_close, assert_weight_matches_oracle, host, need_gpu,
                            oracle_sampled_weight, to_dev_bf16)

pytestmark = pytest.mark.gpu


def _samples(rng, N, K, n_rows, n_cols):
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, n_rows, replace=False)]))
    cols = np.unique(np.concatenate([[0, K - 1], rng.choice(K, n_cols, replace=False)]))
    return rows, cols, np.unique(cols // 64)


def _check_linear(case, rows, cols, blocks):
    W, A, B, X, dY, scale = (case[k] for k in ("W", "A", "B", "X", "dY", "scale"))
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(W))
    Xd, Ad, Bd, dYd = to_dev_bf16(X), to_dev_bf16(A), to_dev_bf16(B), to_dev_bf16(dY)
    Y, T = qlora.qlora_linear_fwd(Xd, q, Ad, Bd, scale)
    dX, dA, dB = qlora.qlora_linear_bwd(dYd, Xd, T, q, Ad, Bd, scale)
    torch.cuda.synchronize()
    assert qlora.qlora_device_error() == 0
    del Xd, dYd
    q_ref, codes_rows, codes_cols = oracle_sampled_weight(W, rows, blocks)
    assert_weight_matches_oracle(q, q_ref, rows, blocks, codes_rows, codes_cols)
    X64, A64, B64, dY64 = (np.asarray(v, np.float64) for v in (X, A, B, dY))
    T64 = X64 @ A64
    G64 = dY64 @ B64.T
    Wr = O.double_dequant_rows(q_ref, rows).astype(np.float64)        # [len(rows), K]
    Y_ref = X64 @ Wr.T + scale * (T64 @ B64[:, rows])
    assert_close(host(Y[:, rows]), O.bf16_round(Y_ref.astype(np.float32)), bf16_out=True, what="Y")
    Wc = O.double_dequant_cols(q_ref, cols).astype(np.float64)        # [N, len(cols)]
    dX_ref = dY64 @ Wc + scale * (G64 @ A64[cols].T)
    assert_close(host(dX[:, cols]), O.bf16_round(dX_ref.astype(np.float32)), bf16_out=True,
                 what="dX")
    assert_close(host(dA), scale * (X64.T @ G64), what="dA")
    assert_close(host(dB), scale * (T64.T @ dY64), what="dB")
    assert_close(host(T), T64, what="T")


@pytest.mark.parametrize("N,K", [(4096, 11008), (11008, 4096)])
def test_layer_linear_full_size_sampled(N, K):
    need_gpu()
    case = inputs.linear_case(3, 4096, N, K, 64, 16.0)
    rows, cols, blocks = _samples(np.random.default_rng(17), N, K, 48, 48)
    _check_linear(case, rows, cols, blocks)


@pytest.mark.parametrize("N,K", [(8192, 8192), (22016, 8192), (8192, 22016)])
def test_65b_stack_linear_full_size_sampled(N, K):
    need_gpu()
    case = inputs.linear_case(4, 8192, N, K, 64, 16.0)
    rows, cols, blocks = _samples(np.random.default_rng(19), N, K, 24, 24)
    _check_linear(case, rows, cols, blocks)


_DECODE = {}


def _decode_weight(N, K):
    """One draw, quantization and oracle reference per decode shape, shared by the M
    variants (drawing 235M weights on the host takes a while)."""
    if (N, K) not in _DECODE:
        case = inputs.decode_case(N, K)
        q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(case["W"]))
        torch.cuda.synchronize()
        rows, _, blocks = _samples(np.random.default_rng(23), N, K, 64, 4)
        ref = oracle_sampled_weight(case["W"], rows, blocks)
        assert_weight_matches_oracle(q, ref[0], rows, blocks, ref[1], ref[2])
        del case["W"]
        _DECODE.clear()
        _DECODE[(N, K)] = (case, q, rows, ref[0])
    return _DECODE[(N, K)]


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("N,K", [(4096, 11008), (8192, 28672)])
def test_decode_full_size_sampled(N, K, M):
    """The decode configuration (4096 x 11008 and 8192 x 28672, r = 16, alpha = 32,
    seed 2): the weight against the oracle's quantization, then Y on sampled rows of W
    and T in full."""
    need_gpu()
    case, q, rows, q_ref = _decode_weight(N, K)
    A, B, X, scale = case["A"], case["B"], case["X"][:M], case["scale"]
    Y, T = qlora.qlora_linear_fwd(to_dev_bf16(X), q, to_dev_bf16(A), to_dev_bf16(B), scale)
    torch.cuda.synchronize()
    assert qlora.qlora_device_error() == 0
    X64, A64, B64 = (np.asarray(v, np.float64) for v in (X, A, B))
    T64 = X64 @ A64
    Wr = O.double_dequant_rows(q_ref, rows).astype(np.float64)
    Y_ref = X64 @ Wr.T + scale * (T64 @ B64[:, rows])
    assert_close(host(Y[:, rows]), O.bf16_round(Y_ref.astype(np.float32)), bf16_out=True, what="Y")
    assert_close(host(T), T64, what="T")
