"""Column (N) sharding of W, host side: the planner's cut points (through the C ABI, no
GPU) and the sharded backward's reductions as world-size-2 gloo ranks on the CPU, each
rank computing its shard with the oracle (itwiki "QLoRA", section "계산 방식": dX
through the frozen W, gradients for A and B only; the split over the output features
turns G and dX into sums over the shards)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_nf4_quantized_unpack_b200 import qlora


@pytest.mark.parametrize("N,K", [(4096, 4096), (4096, 11008), (11008, 4096), (8192, 8192),
                                 (22016, 8192), (8192, 22016), (512, 1024), (136, 64)])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_rows_cover_and_cut_on_whole_constant_blocks(N, K, world):
    try:
        parts = [qlora.qlora_shard_rows(N, K, world, r) for r in range(world)]
    except qlora.QLoraError as e:
        # only when there are fewer whole cuts than shards
        unit = max(65536 // np.gcd(K, 65536), 8)
        assert N // unit < world, e
        return
    row = 0
    unit = max(65536 // np.gcd(K, 65536), 8)
    for r, (r0, rows) in enumerate(parts):
        assert r0 == row and rows > 0 and rows % 8 == 0
        assert (r0 * K) % 65536 == 0                       # whole 256-constant blocks of c1
        row += rows
        if r < world - 1:
            assert rows % unit == 0
    assert row == N
    sizes = [rows for _, rows in parts]
    assert max(sizes) - min(sizes) <= unit + (N % unit)   # near-equal


def test_shard_rows_rejects_bad_arguments():
    L = qlora.lib()
    r0, rows = qlora.ctypes.c_int64(0), qlora.ctypes.c_int64(0)
    ref = (qlora.ctypes.byref(r0), qlora.ctypes.byref(rows))
    assert L.qlora_shard_rows(512, 1024, 2, 2, *ref) == 1     # rank outside [0, world)
    assert L.qlora_shard_rows(512, 1024, 0, 0, *ref) == 1
    assert L.qlora_shard_rows(512, 1000, 2, 0, *ref) == 2     # K % 64 != 0
    assert L.qlora_shard_rows(512, 1024, 16, 0, *ref) == 2    # 8 cuts of 64 rows < 16 shards
    assert L.qlora_shard_rows(512, 1024, 2, 0, None, None) == 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _sharded_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from bit_nf4_quantized_unpack_b200 import inputs
        from oracle import nf4_oracle as O
        M, N, K, r, alpha = 32, 512, 1024, 16, 32.0
        case = inputs.linear_case(41, M, N, K, r, alpha)      # the same draw on every rank
        W, A, B, X, dY, scale = (case[k] for k in ("W", "A", "B", "X", "dY", "scale"))
        q = O.quantize_nf4_dq(W)
        What = O.double_dequant(q).astype(np.float64)
        r0, rows = qlora.qlora_shard_rows(N, K, world, rank)
        sl = slice(r0, r0 + rows)
        X64, A64, B64, dY64 = (np.asarray(v, np.float64) for v in (X, A, B, dY))
        T = X64 @ A64
        # G: each shard's dY_shard B_shard^T, summed over the shards
        G = torch.from_numpy(dY64[:, sl] @ B64[:, sl].T)
        dist.all_reduce(G)
        G = G.numpy()
        # dX: each shard's dY_shard W_hat_shard, the LoRA term on shard 0 only, summed
        dXp = dY64[:, sl] @ What[sl]
        if rank == 0:
            dXp = dXp + scale * (G @ A64.T)
        dX = torch.from_numpy(dXp)
        dist.all_reduce(dX)
        dA = scale * (X64.T @ G)
        dB_shard = scale * (T.T @ dY64[:, sl])
        dX_ref, dA_ref, dB_ref = O.linear_backward(dY, X, What, A, B, scale, T=T)
        ok = (np.allclose(dX.numpy(), dX_ref, rtol=1e-12, atol=1e-12) and
              np.allclose(dA, dA_ref, rtol=1e-12, atol=1e-12) and
              np.allclose(dB_shard, dB_ref[:, sl], rtol=1e-12, atol=1e-12))
        out.put((rank, ok, r0, rows))
    finally:
        dist.destroy_process_group()


def test_sharded_backward_sums_to_the_unsharded_one_on_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [ok for _, ok, _, _ in res] == [True, True]
    assert [(r0, rows) for _, _, r0, rows in res] == [(0, 256), (256, 256)]
