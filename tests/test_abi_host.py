"""Host-side checks of the C-ABI library: it loads, exports every declared entry point,
carries the same code tables as the oracle, derives exact nearest-entry thresholds,
and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

from bit_nf4_quantized_unpack_b200 import build, qlora
from oracle import nf4_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return qlora.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "qlora.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_nf4_table_matches_oracle_bits(L):
    got = qlora.nf4_table().numpy()
    assert np.array_equal(got.view(np.uint32), O.nf4_levels().view(np.uint32))


def _next_up(x, n=1):
    return np.nextafter(x, np.float32(np.inf), dtype=np.float32) if n == 1 else None


def _ulp_window(center, half):
    """All fp32 values within `half` ulps of center (ordered-bit walk)."""
    c = np.float32(center)
    out = [c]
    lo, hi = c, c
    for _ in range(half):
        lo = np.nextafter(lo, np.float32(-np.inf))
        hi = np.nextafter(hi, np.float32(np.inf))
        out += [lo, hi]
    return np.array(out, np.float32)


def _count_leq(th, x):
    return np.searchsorted(th, x, side="right")


def test_nf4_thresholds_reproduce_argmin(L):
    th = qlora.nf4_thresholds().numpy()
    table = O.nf4_levels()
    assert np.all(np.diff(th) > 0)
    xs = [np.random.default_rng(0).uniform(-1, 1, 1 << 18).astype(np.float32), table,
          np.array([-1.0, 1.0, 0.0, -0.0], np.float32)]
    for t in th:
        xs.append(_ulp_window(t, 2048))
        mid = np.float32((np.float64(t)))
        xs.append(_ulp_window(mid, 16))
    # every midpoint of neighbouring levels, rounded both ways
    mids = (table[:-1].astype(np.float64) + table[1:]) / 2
    for m in mids:
        xs.append(_ulp_window(np.float32(m), 64))
    x = np.concatenate(xs)
    x = x[(x >= -1) & (x <= 1)]
    assert np.array_equal(O.nearest_code(x, table), _count_leq(th, x))


def test_nf4_code_buckets_reproduce_argmin(L):
    """The quantization kernel's table form of the code search: bucket
    b = round-half-even(16 x + 16), code = code[b] + (x >= thr[b]); checked against the
    oracle's argmin on random x, around every threshold and level, and on both sides of
    every bucket edge."""
    thr, code = (t.numpy() for t in qlora.nf4_code_buckets())
    table = O.nf4_levels()
    th = qlora.nf4_thresholds().numpy()
    xs = [np.random.default_rng(2).uniform(-1, 1, 1 << 18).astype(np.float32), table,
          np.array([-1.0, 1.0, 0.0, -0.0], np.float32)]
    for t in th:
        xs.append(_ulp_window(t, 256))
    S = qlora.BUCKET_SCALE
    assert thr.shape == code.shape == (2 * S + 1,)
    edges = ((2.0 * np.arange(2 * S + 2) - 2 * S - 1.0) / (2 * S)).astype(np.float32)
    for e in edges:
        xs.append(_ulp_window(e, 3))
    x = np.concatenate(xs)
    x = x[(x >= -1) & (x <= 1)]
    b = np.rint(S * x.astype(np.float64) + S).astype(np.int64)  # rint: half to even
    got = code[b].astype(np.int64) + (x >= thr[b]).astype(np.int64)
    assert np.array_equal(O.nearest_code(x, table), got)


@pytest.mark.parametrize("codebook", [0, 1])
def test_codebook_tables_reproduce_argmin(L, codebook):
    """Each codebook's levels are the oracle's bit for bit, and its thresholds and
    bucket table both reproduce the oracle's argmin around every threshold and level."""
    lev, th, bthr, bcode = (t.numpy() for t in qlora.codebook_tables(codebook))
    table = O.nf4_levels() if codebook == 0 else O.uniform4_levels()
    assert np.array_equal(lev.view(np.uint32), table.view(np.uint32))
    xs = [np.random.default_rng(3 + codebook).uniform(-1, 1, 1 << 17).astype(np.float32), table,
          np.array([-1.0, 1.0, 0.0, -0.0], np.float32)]
    for t in th:
        xs.append(_ulp_window(t, 256))
    S = qlora.BUCKET_SCALE
    for e in ((2.0 * np.arange(2 * S + 2) - 2 * S - 1.0) / (2 * S)).astype(np.float32):
        xs.append(_ulp_window(e, 2))
    x = np.concatenate(xs)
    x = x[(x >= -1) & (x <= 1)]
    want = O.nearest_code(x, table)
    assert np.array_equal(want, _count_leq(th, x))
    b = np.rint(S * x.astype(np.float64) + S).astype(np.int64)
    assert np.array_equal(want, bcode[b].astype(np.int64) + (x >= bthr[b]).astype(np.int64))
    assert L.qlora_codebook_tables(2, None, None, None, None) == -1


def test_fp8_table_and_thresholds_match_oracle(L):
    th, vals, codes = (t.numpy() for t in qlora.fp8_thresholds())
    ovals, ocodes = O.fp8_table()
    assert np.array_equal(vals.view(np.uint32), ovals.view(np.uint32))
    assert np.array_equal(codes, ocodes)
    assert th.size == 252 and np.all(np.diff(th) > 0)
    xs = [np.random.default_rng(1).uniform(-1, 1, 1 << 16).astype(np.float32), ovals]
    for t in th:
        xs.append(_ulp_window(t, 24))
    x = np.concatenate(xs)
    x = x[(x >= -1) & (x <= 1)]
    assert np.array_equal(O.nearest_code(x, ovals), _count_leq(th, x))


def test_status_strings(L):
    for code, name in qlora.STATUS.items():
        assert L.qlora_status_str(code).decode() == name
    assert L.qlora_version() >= 100


# ----------------------------------------------------------------- argument errors
# Fake, never dereferenced device addresses: every case below is rejected on the
# host before any CUDA call.
P = 1 << 20          # 16-byte aligned fake pointer
Q = (1 << 20) + 8    # misaligned fake pointer


def W(codes=P, c2=P, c1=P, mean=P, n=512, k=1024, codebook=0):
    return qlora.CNF4Weight(codes, c2, c1, mean, n, k, codebook)


def test_quantize_rejects_bad_arguments(L):
    f = L.qlora_quantize_nf4_dq
    ws = L.qlora_quantize_workspace_size(512, 1024)
    assert ws > 0 and L.qlora_quantize_workspace_size(512, 1000) == 0
    ok = [P, 0, 512, 1024, P, P, P, P, P, ws, None]
    def call(**kw):
        a = list(ok)
        idx = {"W": 0, "dtype": 1, "n": 2, "k": 3, "codes": 4, "ws": 8, "wsb": 9}
        for k_, v in kw.items():
            a[idx[k_]] = v
        return f(*a)
    assert call(W=None) == 1
    assert call(dtype=7) == 1
    assert call(k=1000) == 2
    assert call(k=0) == 2
    assert call(n=0) == 2
    assert call(codes=Q) == 3
    assert call(ws=None) == 4
    assert call(wsb=ws - 1) == 4


def test_merge_rejects_bad_arguments(L):
    merge = L.qlora_merge_lora
    assert merge(W(), None, P, 8, 2.0, P, None) == 1
    assert merge(W(), P, P, 12, 2.0, P, None) == 1
    assert merge(W(), P, P, 8, float("inf"), P, None) == 1
    assert merge(W(k=1000), P, P, 8, 2.0, P, None) == 2
    assert merge(W(n=500), P, P, 8, 2.0, P, None) == 2
    assert merge(W(), P, P, 8, 2.0, Q, None) == 3
    assert merge(W(codes=None), P, P, 8, 2.0, P, None) == 1


def test_unknown_codebook_is_rejected(L):
    assert L.qlora_dequant(W(codebook=2), P, None) == 1
    assert L.qlora_merge_lora(W(codebook=-1), P, P, 8, 2.0, P, None) == 1
    ws = L.qlora_quantize_workspace_size(512, 1024)
    assert L.qlora_quantize_dq(P, 0, 512, 1024, 7, P, P, P, P, P, ws, None) == 1


def test_linear_rejects_bad_arguments(L):
    fwd = L.qlora_linear_fwd
    need = L.qlora_linear_fwd_workspace_size(64, 512, 1024, 8)
    assert need > 0
    base = dict(X=P, M=64, w=W(), A=P, B=P, r=8, scale=2.0, Y=P, T=None, ws=P, wsb=need)
    def call(**kw):
        a = dict(base, **kw)
        return fwd(a["X"], a["M"], a["w"], a["A"], a["B"], a["r"], a["scale"], a["Y"], a["T"],
                   a["ws"], a["wsb"], None)
    assert call(X=None) == 1
    assert call(r=0) == 1 and call(r=12) == 1 and call(r=72) == 1
    assert call(scale=float("nan")) == 1
    assert call(w=W(k=1000)) == 2
    assert call(w=W(n=500)) == 2
    assert call(M=-1) == 2
    assert call(w=W(codes=None)) == 1
    assert call(w=W(c2=Q)) == 3
    assert call(Y=Q) == 3
    assert call(ws=None) == 4
    assert call(wsb=need - 1) == 4
    assert call(M=0) == 0          # empty input: nothing to do, nothing launched
    bwd = L.qlora_linear_bwd
    bneed = L.qlora_linear_bwd_workspace_size(64, 512, 1024, 8)
    assert bneed > 0
    assert bwd(None, P, None, 64, W(), P, P, 8, 2.0, P, P, P, P, bneed, None) == 1
    assert bwd(P, P, None, 64, W(), P, P, 8, 2.0, P, None, P, P, bneed, None) == 1
    assert bwd(P, P, None, 64, W(), P, P, 8, 2.0, P, P, P, P, bneed - 1, None) == 4
    assert bwd(P, P, Q, 64, W(), P, P, 8, 2.0, P, P, P, P, bneed, None) == 3
    assert L.qlora_dequant(W(k=100), P, None) == 2
    assert L.qlora_dequant(W(), None, None) == 1


def test_adamw_rejects_bad_arguments(L):
    """The optimizer step checks every argument before it touches a device."""
    from bit_nf4_quantized_unpack_b200.qlora import CAdamwHparams
    n = 1000
    sb8, sb32 = L.qlora_adamw_state_bytes(n, 8), L.qlora_adamw_state_bytes(n, 32)
    nblk = -(-n // 256)
    assert sb8 == 2 * 1024 + 2 * 256 and sb8 >= 2 * n + 8 * nblk
    assert sb32 == 2 * 4096
    assert L.qlora_adamw_state_bytes(n, 16) == 0 and L.qlora_adamw_state_bytes(-1, 8) == 0

    def hp(**kw):
        a = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1)
        a.update(kw)
        return CAdamwHparams(a["lr"], a["beta1"], a["beta2"], a["eps"], a["weight_decay"], a["step"])

    def call(p=P, pb=None, g=P, nn=n, bits=8, st=P, sbytes=sb8, **kw):
        return L.qlora_adamw_step(p, pb, g, nn, bits, st, sbytes, hp(**kw), None)

    assert call(p=None) == 1 and call(g=None) == 1 and call(st=None) == 1
    assert call(bits=16) == 1 and call(nn=-1) == 1
    assert call(step=0) == 1
    assert call(lr=-1.0) == 1 and call(lr=float("nan")) == 1
    assert call(eps=0.0) == 1 and call(weight_decay=-0.1) == 1
    assert call(beta1=1.0) == 1 and call(beta2=-0.5) == 1 and call(beta2=float("inf")) == 1
    assert call(p=Q) == 3 and call(g=Q) == 3 and call(st=Q) == 3 and call(pb=Q) == 3
    assert call(sbytes=sb8 - 1) == 4
    assert call(bits=32, sbytes=sb8) == 4
    assert call(nn=0) == 0          # nothing to update, nothing launched
    assert L.qlora_paged_free(None) == 0
    assert L.qlora_paged_prefetch(None, 16, 1, None) == 1
    import ctypes
    out = ctypes.c_void_p()
    assert L.qlora_paged_alloc(ctypes.byref(out), 0) == 1
    assert L.qlora_paged_alloc(None, 16) == 1
