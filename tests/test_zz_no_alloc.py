"""The allocation-free decode forward, qlora_linear_fwd_decode_static.

It serves callers that cannot allocate device memory when they run the layer (a
runtime that fixes its device memory at start-up, or a decode loop that must not
synchronise the device through cudaMalloc). It keeps its partial sums in a static
device array inside the library instead of a caller workspace. This test calls it
through the C ABI twice in a row and compares each result with the workspace-based
entry point, qlora_linear_fwd, within the parity tolerance of the other tests; the
second call also shows that what the first call left in the shared array does not
leak into the next result. Each result is also compared with the oracle on sampled rows
of the weight. The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import (assert_close, assert_weight_matches_oracle, host, need_gpu,
                            oracle_sampled_weight, to_dev_bf16)

pytestmark = pytest.mark.gpu


def _static_fwd(X, q, A, B, r, scale, Y, T):
    status = qlora.lib().qlora_linear_fwd_decode_static(
        ctypes.c_void_p(X.data_ptr()), X.shape[0], q.c_struct(), ctypes.c_void_p(A.data_ptr()),
        ctypes.c_void_p(B.data_ptr()), r, ctypes.c_float(scale), ctypes.c_void_p(Y.data_ptr()),
        ctypes.c_void_p(T.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == 0, qlora.lib().qlora_last_error().decode()


@pytest.mark.parametrize("M,N,K,r", [(1, 4096, 11008, 16), (16, 512, 1024, 8), (5, 8192, 2048, 64)])
def test_static_scratch_decode_matches_workspace_path(M, N, K, r):
    need_gpu()
    case = inputs.linear_case(300 + M, M, N, K, r, alpha=2.0 * r)
    q = qlora.qlora_quantize_nf4_dq(to_dev_bf16(case["W"]))
    X, A, B = to_dev_bf16(case["X"]), to_dev_bf16(case["A"]), to_dev_bf16(case["B"])
    Y_ref, T_ref = qlora.qlora_linear_fwd(X, q, A, B, case["scale"])
    for call in range(2):
        X2 = X if call == 0 else to_dev_bf16(case["X"][::-1].copy())
        if call == 1:
            Y_ref, T_ref = qlora.qlora_linear_fwd(X2, q, A, B, case["scale"])
        Y = torch.full_like(Y_ref, float("nan"))
        T = torch.full_like(T_ref, float("nan"))
        _static_fwd(X2, q, A, B, r, case["scale"], Y, T)
        torch.cuda.synchronize()
        assert qlora.qlora_device_error() == 0
        assert_close(host(Y), host(Y_ref), bf16_out=True, what=f"Y (call {call})")
        assert_close(host(T), host(T_ref), what=f"T (call {call})")
        # and directly against the oracle, on sampled rows of W
        rows = np.unique(np.random.default_rng(M).choice(N, min(N, 48), replace=False))
        q_ref, codes_rows, codes_cols = oracle_sampled_weight(case["W"], rows, [0])
        assert_weight_matches_oracle(q, q_ref, rows, [0], codes_rows, codes_cols)
        Xh = host(X2).astype(np.float64)
        A64, B64 = (np.asarray(case[k], np.float64) for k in ("A", "B"))
        T64 = Xh @ A64
        Wr = O.double_dequant_rows(q_ref, rows).astype(np.float64)
        Y64 = Xh @ Wr.T + case["scale"] * (T64 @ B64[:, rows])
        assert_close(host(Y)[:, rows], O.bf16_round(Y64.astype(np.float32)), bf16_out=True,
                     what=f"Y against the oracle (call {call})")
        assert_close(host(T), T64, what=f"T against the oracle (call {call})")


def test_static_scratch_with_fewer_k_splits():
    """M = 16 tokens on an 8192 x 11008 weight: the usual plan's fp32 partial sums (8 K
    splits, 4.2 MB) do not fit the 4 MiB array, so the entry point plans with 7; the
    results must not change."""
    need_gpu()
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    M, N, K, r, scale = 16, 8192, 11008, 16, 2.0
    q = qlora.qlora_quantize_nf4_dq((torch.randn(N, K, generator=g, device="cuda") * 0.02)
                                    .to(torch.bfloat16))
    X = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    A = (torch.randn(K, r, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    B = (torch.randn(r, N, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    Y_ref, T_ref = qlora.qlora_linear_fwd(X, q, A, B, scale)
    for _ in range(2):
        Y = torch.full_like(Y_ref, float("nan"))
        T = torch.full_like(T_ref, float("nan"))
        _static_fwd(X, q, A, B, r, scale, Y, T)
        torch.cuda.synchronize()
        assert qlora.qlora_device_error() == 0
        assert_close(host(Y), host(Y_ref), bf16_out=True, what="Y")
        assert_close(host(T), host(T_ref), what="T")


def test_static_scratch_rejects_oversize_and_large_m():
    need_gpu()
    q = qlora.NF4Weight.empty(65536, 1024)
    X = torch.zeros(16, 1024, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(1024, 64, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(64, 65536, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(16, 65536, dtype=torch.bfloat16, device="cuda")
    L = qlora.lib()
    args = (ctypes.c_void_p(X.data_ptr()), 16, q.c_struct(), ctypes.c_void_p(A.data_ptr()),
            ctypes.c_void_p(B.data_ptr()), 64, ctypes.c_float(1.0), ctypes.c_void_p(Y.data_ptr()),
            None, None)
    assert L.qlora_linear_fwd_decode_static(*args) == 4          # QLORA_ERR_WORKSPACE
    assert b"static scratch" in L.qlora_last_error()
    big = list(args)
    big[1] = 17
    assert L.qlora_linear_fwd_decode_static(*big) == 2           # QLORA_ERR_SHAPE


def test_static_scratch_argument_errors_match_workspace_path():
    """r, scale and alignment errors come back before anything is enqueued, with the
    status qlora_linear_fwd gives for the same arguments."""
    need_gpu()
    M, N, K = 4, 256, 1024
    q = qlora.NF4Weight.empty(N, K)
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(K, 64, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(64, N, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(M * N + 8, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(qlora.qlora_linear_fwd_workspace_size(M, N, K, 16), dtype=torch.uint8,
                     device="cuda")
    L = qlora.lib()

    def both(r, scale, y_ptr):
        common = (ctypes.c_void_p(X.data_ptr()), M, q.c_struct(), ctypes.c_void_p(A.data_ptr()),
                  ctypes.c_void_p(B.data_ptr()), r, ctypes.c_float(scale), ctypes.c_void_p(y_ptr),
                  None)
        st = L.qlora_linear_fwd_decode_static(*common, None)
        ref = L.qlora_linear_fwd(*common, ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
        return st, ref

    y = Y.data_ptr()
    for r, scale, y_ptr, want in [(4, 1.0, y, 1), (12, 1.0, y, 1), (16, float("nan"), y, 1),
                                  (16, float("inf"), y, 1), (16, 1.0, y + 2, 3)]:
        st, ref = both(r, scale, y_ptr)
        assert st == ref == want, (r, scale, y_ptr - y, st, ref)
    torch.cuda.synchronize()
    assert qlora.qlora_device_error() == 0

