"""GPU parity of the column (N) sharded layer: the shards of one weight run one after
another on one GPU (each as its own weight view), their partial G and dX are summed on
the device as a collective would, and the results match the unsharded layer and the
oracle. The fp32 dX partials are checked against fp64 on their own."""
import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import assert_close, host, need_gpu, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,r,world", [
    (300, 512, 1024, 16, 2),      # ragged tokens, two shards of 256 rows
    (257, 4096, 4096, 64, 3),     # three shards (1360 / 1360 / 1376 rows)
    (1024, 4096, 11008, 64, 2),   # cuts every 256 rows at K = 11008
])
def test_sharded_backward_matches_unsharded_and_oracle(M, N, K, r, world):
    need_gpu()
    case = inputs.linear_case(500 + world, M, N, K, r, alpha=2.0 * r)
    W, A, B, X, dY, scale = (case[k] for k in ("W", "A", "B", "X", "dY", "scale"))
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(W))
    Xd, Ad, Bd, dYd = to_dev_bf16(X), to_dev_bf16(A), to_dev_bf16(B), to_dev_bf16(dY)
    Y, T = qlora.qlora_linear_fwd(Xd, q, Ad, Bd, scale)
    dX_ref, dA_ref, dB_ref = qlora.qlora_linear_bwd(dYd, Xd, T, q, Ad, Bd, scale)

    parts = [qlora.qlora_shard_rows(N, K, world, s) for s in range(world)]
    shards = []
    for r0, rows in parts:
        ws = qlora.qlora_shard_weight(q, r0, rows)
        shards.append((r0, rows, ws, dYd[:, r0:r0 + rows].contiguous(),
                       Bd[:, r0:r0 + rows].contiguous()))
    # forward per shard: the columns of Y
    for r0, rows, ws, _, Bs in shards:
        Ys, Ts = qlora.qlora_linear_fwd(Xd, ws, Ad, Bs, scale)
        assert_close(host(Ys), host(Y[:, r0:r0 + rows]), bf16_out=True, what="Y shard")
        assert_close(host(Ts), host(T), what="T shard")
    # backward: G summed over the shards, then dX partials summed and rounded
    G = sum(qlora.qlora_linear_bwd_shard_g(dYs, Bs) for _, _, _, dYs, Bs in shards)
    dX_sum = None
    dBs = []
    for i, (r0, rows, ws, dYs, Bs) in enumerate(shards):
        dXp, dA, dB = qlora.qlora_linear_bwd_shard(dYs, Xd, T, G, ws, Ad, Bs, scale,
                                                   lora_in_dx=(i == 0))
        dX_sum = dXp if dX_sum is None else dX_sum + dXp
        assert_close(host(dA), host(dA_ref), what=f"dA (shard {i})")
        dBs.append(dB)
    dX = qlora.qlora_f32_to_bf16(dX_sum)
    torch.cuda.synchronize()
    assert qlora.qlora_device_error() == 0
    assert_close(host(dX), host(dX_ref), bf16_out=True, what="dX against the unsharded layer")
    assert_close(host(torch.cat(dBs, dim=1)), host(dB_ref), what="dB")
    # and the oracle
    ref = O.quantize_nf4_dq(W)
    What = O.double_dequant(ref)
    T64 = np.asarray(X, np.float64) @ np.asarray(A, np.float64)
    dX64, dA64, dB64 = O.linear_backward(dY, X, What, A, B, scale, T=T64)
    assert_close(host(dX), O.bf16_round(dX64.astype(np.float32)), bf16_out=True, what="dX")
    assert_close(host(torch.cat(dBs, dim=1)), dB64, what="dB against the oracle")


def test_dx_partial_is_the_fp32_product_of_the_shard():
    """Without the LoRA term, a shard's dX_part is dY_shard W_hat_shard in fp32: compared
    with the fp64 product (fp32 accumulation error only)."""
    need_gpu()
    M, N, K, r = 200, 1024, 2048, 16
    case = inputs.linear_case(77, M, N, K, r, alpha=32.0)
    W, A, B, X, dY, scale = (case[k] for k in ("W", "A", "B", "X", "dY", "scale"))
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(W))
    r0, rows = qlora.qlora_shard_rows(N, K, 2, 1)
    ws = qlora.qlora_shard_weight(q, r0, rows)
    dYs = to_dev_bf16(np.ascontiguousarray(dY[:, r0:r0 + rows]))
    Bs = to_dev_bf16(np.ascontiguousarray(B[:, r0:r0 + rows]))
    G = torch.zeros(M, r, dtype=torch.float32, device="cuda")
    dXp, _, _ = qlora.qlora_linear_bwd_shard(dYs, to_dev_bf16(X), None, G, ws, to_dev_bf16(A), Bs,
                                             scale, lora_in_dx=False)
    torch.cuda.synchronize()
    What = O.double_dequant(O.quantize_nf4_dq(W))[r0:r0 + rows].astype(np.float64)
    ref = np.asarray(dY, np.float64)[:, r0:r0 + rows] @ What
    err = np.abs(host(dXp) - ref)
    assert np.linalg.norm(host(dXp) - ref) / np.linalg.norm(ref) < 1e-5
    assert err.max() < 1e-4 * max(1.0, float(np.abs(ref).max()))
