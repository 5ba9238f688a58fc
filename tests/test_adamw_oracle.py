"""Pins of the AdamW oracle (paged 32-bit and 8-bit optimizer states) against things
outside it: PyTorch's own AdamW, the closed form of Adam's first step, the
no-momentum special case, exact round trips of values on the 8-bit grid, and the
8-bit trajectory staying close to the 32-bit one."""
import numpy as np
import pytest
import torch

from oracle import adamw_oracle as AW
from oracle import nf4_oracle as O

HP = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _run32(p, grads, **hp):
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    for t, g in enumerate(grads, start=1):
        p, _, m, v = AW.adamw_step(p, g, m, v, step=t, **hp)
    return p


def test_32bit_matches_torch_adamw():
    """Five steps against torch.optim.AdamW on the CPU in fp32: the same update with
    another rounding order, so the parameters agree to a few fp32 ulps."""
    rng = np.random.default_rng(0)
    p0 = rng.normal(0, 0.02, 4099).astype(np.float32)
    grads = [rng.normal(0, 1e-3, p0.size).astype(np.float32) for _ in range(5)]
    mine = _run32(p0.copy(), grads, **HP)
    tp = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([tp], lr=HP["lr"], betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"],
                            weight_decay=HP["weight_decay"], foreach=False)
    for g in grads:
        tp.grad = torch.from_numpy(g.copy())
        opt.step()
    ref = tp.detach().numpy()
    moved = np.abs(ref - p0)
    assert np.max(np.abs(mine - ref) / np.maximum(moved, 1e-12)) < 1e-3
    assert np.max(np.abs(mine - ref)) < 4 * np.spacing(np.max(np.abs(ref)))


def test_first_step_closed_form():
    """At t = 1 the bias corrections undo the averaging: m_hat = g, v_hat = g^2, so the
    step is lr * g / (|g| + eps) after the decoupled decay."""
    rng = np.random.default_rng(1)
    p = rng.normal(0, 0.02, 1000).astype(np.float32)
    g = (rng.choice([-1, 1], 1000) * rng.uniform(1e-3, 1.0, 1000)).astype(np.float32)
    p1, _, m, v = AW.adamw_step(p, g, np.zeros_like(p), np.zeros_like(p), step=1, **HP)
    expect = p.astype(np.float64) * (1 - HP["lr"] * HP["weight_decay"]) - HP["lr"] * np.sign(g)
    assert np.max(np.abs(p1 - expect)) < 1e-9 + 3e-7 * HP["lr"] + 2 * np.spacing(np.float32(0.1))
    # (1 - b) is formed from the fp32 beta: 1 - fl32(0.999) = 0.00099998713...
    omb1 = 1.0 - np.float64(np.float32(HP["beta1"]))
    omb2 = 1.0 - np.float64(np.float32(HP["beta2"]))
    np.testing.assert_allclose(m, omb1 * g, rtol=2e-7)
    np.testing.assert_allclose(v, omb2 * g.astype(np.float64) ** 2, rtol=4e-7)


def test_no_momentum_ignores_history():
    """With beta1 = beta2 = 0 every step is lr * g / (|g| + eps), whatever came before."""
    rng = np.random.default_rng(2)
    p = rng.normal(0, 0.02, 512).astype(np.float32)
    g = rng.normal(0, 1e-2, 512).astype(np.float32)
    junk = rng.normal(0, 5.0, 512).astype(np.float32)
    hp = dict(HP, beta1=0.0, beta2=0.0, weight_decay=0.0)
    p1, _, _, _ = AW.adamw_step(p, g, junk, np.abs(junk), step=7, **hp)
    expect = p.astype(np.float64) - hp["lr"] * g / (np.abs(g) + hp["eps"])
    np.testing.assert_allclose(p1, expect, rtol=0, atol=2 * np.spacing(np.float32(0.1)))


def test_state_round_trip_on_the_grid():
    """Values that are T8 entries times a power-of-two absmax are stored exactly; the
    block maximum reads back as +-absmax; an all-zero block stores zeros."""
    vals, codes = O.fp8_table()
    rng = np.random.default_rng(3)
    n = 3 * AW.STATE_BLOCK + 17
    k = rng.integers(0, vals.size, n)
    scale = np.float32(2.0) ** rng.integers(-20, 5, -(-n // AW.STATE_BLOCK)).astype(np.float32)
    x = (vals[k] * np.repeat(scale, AW.STATE_BLOCK)[:n]).astype(np.float32)
    for b in range(scale.size):  # make each block's absmax its scale
        x[b * AW.STATE_BLOCK] = scale[b]
    c, a = AW.encode_state(x)
    np.testing.assert_array_equal(a, scale)
    np.testing.assert_array_equal(AW.decode_state(c, a), x)
    zc, za = AW.encode_state(np.zeros(300, np.float32))
    assert not zc.any() and not za.any()
    np.testing.assert_array_equal(AW.decode_state(zc, za), np.zeros(300, np.float32))


def test_state_code_is_nearest_level():
    """Every stored value is the nearest representable one up to fp32 rounding: no other
    T8 entry times the block absmax lies closer by more than the roundings of x / a and
    of the decode (brute force over the table)."""
    vals, _ = O.fp8_table()
    rng = np.random.default_rng(4)
    x = (rng.normal(0, 1, 700) * rng.choice([1e-3, 1.0], 700)).astype(np.float32)
    c, a = AW.encode_state(x)
    got = AW.decode_state(c, a).astype(np.float64)
    amax = np.repeat(a, AW.STATE_BLOCK)[:x.size].astype(np.float64)
    cand = vals.astype(np.float64)[None, :] * amax[:, None]
    best = np.min(np.abs(cand - x[:, None]), axis=1)
    slack = 2 * np.spacing(np.abs(x)).astype(np.float64) + 2 * np.spacing(amax.astype(np.float32))
    assert np.all(np.abs(got - x) <= best + slack)
    # the chosen entry is the exactly nearest one almost everywhere
    chosen = np.argmin(np.abs(cand - got[:, None]), axis=1)
    assert np.mean(chosen == np.argmin(np.abs(cand - x[:, None]), axis=1)) > 0.99


def test_8bit_trajectory_tracks_32bit():
    """Twenty steps on a noisy quadratic: the 8-bit states move the parameters almost
    exactly as the 32-bit ones do (a sign or index mistake in the 8-bit path would not)."""
    rng = np.random.default_rng(5)
    n = 2 * AW.STATE_BLOCK + 40
    target = rng.normal(0, 0.05, n).astype(np.float32)
    p32 = np.zeros(n, np.float32)
    p8 = np.zeros(n, np.float32)
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    st = AW.zero_state_8bit(n)
    hp = dict(HP, lr=1e-2)
    for t in range(1, 21):
        noise = rng.normal(0, 1e-3, n).astype(np.float32)
        p32, _, m, v = AW.adamw_step(p32, (p32 - target) + noise, m, v, step=t, **hp)
        p8, _, st = AW.adamw_step_8bit(p8, (p8 - target) + noise, st, step=t, **hp)
    scale = np.mean(np.abs(target))
    assert np.mean(np.abs(p32 - target)) < 0.25 * scale   # both runs converge
    assert np.mean(np.abs(p8 - target)) < 0.25 * scale
    moved = np.abs(p32)
    assert np.max(np.abs(p8 - p32)) < 0.1 * np.max(moved)
    assert np.mean(np.abs(p8 - p32)) < 0.05 * np.mean(moved)
