"""The multi-GPU host logic of bench.py, run as two gloo ranks on the CPU: the
data-parallel all-reduce of the LoRA gradients (the flat buffer at once, and linear by
linear with asynchronous all-reduces in the backward's order) and the max-over-ranks
timing reduction. (Only one GPU is available to this test suite; the NCCL path runs
the same calls.)"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        g = torch.Generator().manual_seed(100 + rank)
        grads = torch.randn(1000, generator=g)
        local = grads.clone()
        bench.allreduce_lora_grads(grads, world)
        gathered = [torch.zeros(1000) for _ in range(world)]
        dist.all_gather(gathered, local)
        ms = bench.max_over_ranks(1.5 + rank, world, "cpu")
        ok = torch.allclose(grads, sum(gathered), atol=1e-5)
        # per linear: the [dA | dB] slices of a 7-linear layout, summed one by one in the
        # backward's order (last linear first) by asynchronous all-reduces
        layer = [dict(k=k, n=n) for k, n in ((64, 32), (64, 32), (64, 32), (64, 64), (64, 96),
                                              (64, 96), (96, 64))]
        numel = sum(l["k"] * 4 + 4 * l["n"] for l in layer)
        flat = torch.randn(numel, generator=g)
        ref = [torch.zeros(numel) for _ in range(world)]
        dist.all_gather(ref, flat.clone())
        slices = bench.linear_grad_slices(flat, layer, r=4)
        assert sum(sl.numel() for sl in slices) == numel
        assert slices[0].data_ptr() == flat.data_ptr()
        pending = [bench.allreduce_linear_grads_async(slices[i], world)
                   for i in reversed(range(len(layer)))]
        bench.wait_all(pending)
        ok = ok and torch.allclose(flat, sum(ref), atol=1e-5)
        out.put((rank, ok, ms))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_dp_gradient_allreduce_and_max_timing(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, ms in res:
        assert ok, f"rank {rank}: all-reduced gradients differ from the sum over ranks"
        assert ms == 1.5 + (world - 1)


def test_single_rank_is_identity():
    import bench
    t = torch.ones(4)
    bench.allreduce_lora_grads(t, 1)
    assert torch.equal(t, torch.ones(4))
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
