"""GPU parity of the paged AdamW step (qlora_adamw_step) against the oracle.

Every operation of the step is one IEEE fp32 rounding in a fixed order on both sides,
so parameters, their bf16 copies, the 8-bit state codes and absmax values, and the
32-bit states must agree bit for bit."""
import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import qlora
from oracle import adamw_oracle as AW
from oracle import nf4_oracle as O
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def draw(n, seed):
    rng = np.random.default_rng(seed)
    p = rng.normal(0, 0.02, n).astype(np.float32)
    grads = []
    for _ in range(3):
        g = rng.normal(0, 1e-3, n).astype(np.float32)
        out = rng.random(n) < 1e-3
        g[out] *= 100.0                       # a few large gradients per block
        if n >= 2 * AW.STATE_BLOCK:
            g[AW.STATE_BLOCK:2 * AW.STATE_BLOCK] = 0.0   # one block without gradient
        grads.append(g)
    return p, grads


def split_state8(raw: np.ndarray, n: int):
    nblk = -(-n // AW.STATE_BLOCK)
    up = lambda x: -(-x // 256) * 256
    off_vc, off_ma = up(n), 2 * up(n)
    off_va = off_ma + up(4 * nblk)
    return dict(mc=raw[:n], vc=raw[off_vc:off_vc + n],
                ma=raw[off_ma:off_ma + 4 * nblk].view(np.float32),
                va=raw[off_va:off_va + 4 * nblk].view(np.float32))


def bits(x):
    return np.asarray(x, np.float32).view(np.uint32)


def run_gpu(p0, grads, state_bits, paged=False, host_between=False):
    n = p0.size
    p = torch.from_numpy(p0.copy()).cuda()
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    sbytes = qlora.qlora_adamw_state_bytes(n, state_bits)
    if paged:
        state = qlora.PagedBuffer(sbytes)
    else:
        state = torch.zeros(sbytes, dtype=torch.uint8, device="cuda")
    for t, g in enumerate(grads, start=1):
        if paged and host_between:
            state.prefetch(to_device=False)   # the pages go to host memory between steps
            torch.cuda.synchronize()
        qlora.qlora_adamw_step(p, torch.from_numpy(g).cuda(), state, t, state_bits=state_bits,
                               p_bf16=pb, **HP)
    torch.cuda.synchronize()
    raw = np.frombuffer(state.host_bytes(), np.uint8).copy() if paged else state.cpu().numpy()
    out_p = p.cpu().numpy()
    out_pb = pb.view(torch.int16).cpu().numpy().view(np.uint16)
    if paged:
        state.free()
    return out_p, out_pb, raw


def run_oracle8(p0, grads):
    p, st = p0.copy(), AW.zero_state_8bit(p0.size)
    for t, g in enumerate(grads, start=1):
        p, pb, st = AW.adamw_step_8bit(p, g, st, step=t, **HP)
    return p, pb, st


@pytest.mark.parametrize("n", [1000, 5 * 256, 65536 + 77])
def test_8bit_states_match_oracle(n):
    p0, grads = draw(n, n)
    p, pb, raw = run_gpu(p0, grads, 8)
    rp, rpb, rst = run_oracle8(p0, grads)
    np.testing.assert_array_equal(bits(p), bits(rp))
    np.testing.assert_array_equal(pb, O.bf16_bits(rpb))
    got = split_state8(raw, n)
    for k in ("mc", "vc"):
        np.testing.assert_array_equal(got[k], rst[k])
    for k in ("ma", "va"):
        np.testing.assert_array_equal(bits(got[k]), bits(rst[k]))


@pytest.mark.parametrize("n", [1000, 65536 + 77])
def test_32bit_states_match_oracle(n):
    p0, grads = draw(n, 100 + n)
    p, pb, raw = run_gpu(p0, grads, 32)
    rp, m, v = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    for t, g in enumerate(grads, start=1):
        rp, rpb, m, v = AW.adamw_step(rp, g, m, v, step=t, **HP)
    np.testing.assert_array_equal(bits(p), bits(rp))
    np.testing.assert_array_equal(pb, O.bf16_bits(rpb))
    off_v = -(-4 * n // 256) * 256
    np.testing.assert_array_equal(raw[:4 * n].view(np.uint32), bits(m))
    np.testing.assert_array_equal(raw[off_v:off_v + 4 * n].view(np.uint32), bits(v))


def test_paged_states_give_the_same_result():
    """States in unified memory, moved to host memory before every step, update exactly
    as states in device memory do."""
    n = 4096 + 13
    p0, grads = draw(n, 7)
    p_dev, pb_dev, raw_dev = run_gpu(p0, grads, 8)
    p_pag, pb_pag, raw_pag = run_gpu(p0, grads, 8, paged=True, host_between=True)
    np.testing.assert_array_equal(bits(p_pag), bits(p_dev))
    np.testing.assert_array_equal(pb_pag, pb_dev)
    np.testing.assert_array_equal(raw_pag[:raw_dev.size], raw_dev)


def test_lora_parameters_of_a_7b_layer_sampled_blocks():
    """The LoRA parameters of the 7B-shaped layer (r = 64 on all seven linears, 5.0M
    values) in one flat buffer; the step updates 256-blocks independently, so sampled
    blocks are checked against the oracle exactly."""
    shapes = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    n = sum(64 * (k + nn) for nn, k in shapes)
    p0, grads = draw(n, 11)
    grads = grads[:2]
    p, pb, raw = run_gpu(p0, grads, 8)
    got = split_state8(raw, n)
    nblk = -(-n // AW.STATE_BLOCK)
    rng = np.random.default_rng(12)
    blocks = np.unique(np.concatenate([[0, 1, nblk - 1], rng.choice(nblk, 200, replace=False)]))
    for b in blocks:
        s = slice(b * AW.STATE_BLOCK, min(n, (b + 1) * AW.STATE_BLOCK))
        rp, rpb, rst = run_oracle8(p0[s], [g[s] for g in grads])
        np.testing.assert_array_equal(bits(p[s]), bits(rp))
        np.testing.assert_array_equal(pb[s], O.bf16_bits(rpb))
        np.testing.assert_array_equal(got["mc"][s], rst["mc"])
        np.testing.assert_array_equal(got["vc"][s], rst["vc"])
        assert bits(got["ma"][b]) == bits(rst["ma"][0]) and bits(got["va"][b]) == bits(rst["va"][0])
