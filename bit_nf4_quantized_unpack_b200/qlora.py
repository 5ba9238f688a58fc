"""Python binding of the C ABI in ``include/qlora.h`` (``lib/libqlora.so``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. PyTorch supplies device memory and the current stream. There is no
fallback: if the library is missing or the device is not sm_100, calls raise.

Names follow the C entry points:
    qlora_quantize_nf4_dq(W)                          -> NF4Weight
    qlora_dequant(w)                                  -> W_hat bf16 [N, K]
    qlora_linear_fwd(X, w, A, B, scale)               -> (Y, T)
    qlora_linear_bwd(dY, X, T, w, A, B, scale)        -> (dX, dA, dB)
    qlora_adamw_step(p, g, state, step, ...)          (in place; paged states: PagedBuffer)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libqlora.so")

STATUS = {0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGN",
          4: "QLORA_ERR_WORKSPACE", 5: "QLORA_ERR_CUDA", 6: "QLORA_ERR_DEVICE",
          7: "QLORA_ERR_TIMEOUT"}
F32, BF16 = 0, 1


class QLoraError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


class CNF4Weight(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("c2", ctypes.c_void_p), ("c1", ctypes.c_void_p),
                ("mean", ctypes.c_void_p), ("n_out", ctypes.c_int64), ("k_in", ctypes.c_int64),
                ("codebook", ctypes.c_int32)]


class CAdamwHparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


_lib = None
_vp, _i64, _i32, _sz, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_float

_SIGNATURES = {
    "qlora_status_str": (ctypes.c_char_p, [_i32]),
    "qlora_last_error": (ctypes.c_char_p, []),
    "qlora_version": (_i32, []),
    "qlora_device_error": (_i32, [_i32]),
    "qlora_profile_events": (None, [_vp, _vp]),
    "qlora_launch_count": (ctypes.c_ulonglong, []),
    "qlora_nf4_table": (None, [_vp]),
    "qlora_nf4_thresholds": (None, [_vp]),
    "qlora_nf4_code_buckets": (None, [_vp, _vp]),
    "qlora_fp8_thresholds": (None, [_vp, _vp, _vp]),
    "qlora_quantize_workspace_size": (_sz, [_i64, _i64]),
    "qlora_quantize_nf4_dq": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qlora_quantize_dq": (_i32, [_vp, _i32, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qlora_codebook_tables": (_i32, [_i32, _vp, _vp, _vp, _vp]),
    "qlora_dequant": (_i32, [CNF4Weight, _vp, _vp]),
    "qlora_merge_lora": (_i32, [CNF4Weight, _vp, _vp, _i32, _f32, _vp, _vp]),
    "qlora_linear_fwd_workspace_size": (_sz, [_i64, _i64, _i64, _i32]),
    "qlora_linear_fwd": (_i32, [_vp, _i64, CNF4Weight, _vp, _vp, _i32, _f32, _vp, _vp, _vp, _sz, _vp]),
    "qlora_linear_fwd_decode_static": (_i32, [_vp, _i64, CNF4Weight, _vp, _vp, _i32, _f32, _vp,
                                              _vp, _vp]),
    "qlora_linear_bwd_workspace_size": (_sz, [_i64, _i64, _i64, _i32]),
    "qlora_linear_bwd": (_i32, [_vp, _vp, _vp, _i64, CNF4Weight, _vp, _vp, _i32, _f32, _vp, _vp,
                                _vp, _vp, _sz, _vp]),
    "qlora_shard_rows": (_i32, [_i64, _i64, _i32, _i32, ctypes.POINTER(ctypes.c_int64),
                                ctypes.POINTER(ctypes.c_int64)]),
    "qlora_shard_weight": (_i32, [CNF4Weight, _i64, _i64, ctypes.c_void_p]),
    "qlora_linear_bwd_shard_g_workspace_size": (_sz, [_i64, _i64, _i32]),
    "qlora_linear_bwd_shard_g": (_i32, [_vp, _i64, _i64, _vp, _i32, _vp, _vp, _sz, _vp]),
    "qlora_linear_bwd_shard_workspace_size": (_sz, [_i64, _i64, _i64, _i32]),
    "qlora_linear_bwd_shard": (_i32, [_vp, _vp, _vp, _vp, _i64, CNF4Weight, _vp, _vp, _i32, _f32,
                                      _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "qlora_f32_to_bf16": (_i32, [_vp, _vp, _i64, _vp]),
    "qlora_selftest_wait_timeout": (_i32, [_vp]),
    "qlora_adamw_state_bytes": (_sz, [_i64, _i32]),
    "qlora_adamw_step": (_i32, [_vp, _vp, _vp, _i64, _i32, _vp, _sz, CAdamwHparams, _vp]),
    "qlora_paged_alloc": (_i32, [ctypes.POINTER(ctypes.c_void_p), _sz]),
    "qlora_paged_free": (_i32, [_vp]),
    "qlora_paged_prefetch": (_i32, [_vp, _sz, _i32, _vp]),
}


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m bit_nf4_quantized_unpack_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise QLoraError(status, where, lib().qlora_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _as_bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 tensors travel as their uint16 bit patterns."""
    if t.dtype != torch.bfloat16:
        raise TypeError(f"expected bfloat16, got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return t


@dataclass
class NF4Weight:
    """A quantized weight [n_out, k_in] in the library's storage format (device)."""
    codes: torch.Tensor   # uint8 [N*K/2]
    c2: torch.Tensor      # uint8 [N*K/64]  E4M3 bit patterns
    c1: torch.Tensor      # float32 [ceil(N*K/16384)]
    mean: torch.Tensor    # float32 [1]
    n_out: int
    k_in: int
    codebook: int = 0     # CODEBOOK_NF4 or CODEBOOK_UNIFORM4

    def c_struct(self) -> CNF4Weight:
        return CNF4Weight(self.codes.data_ptr(), self.c2.data_ptr(), self.c1.data_ptr(),
                          self.mean.data_ptr(), self.n_out, self.k_in, self.codebook)

    @staticmethod
    def empty(n_out: int, k_in: int, device="cuda", codebook: int = 0) -> "NF4Weight":
        nb = n_out * k_in // 64
        return NF4Weight(torch.empty(n_out * k_in // 2, dtype=torch.uint8, device=device),
                         torch.empty(nb, dtype=torch.uint8, device=device),
                         torch.empty((nb + 255) // 256, dtype=torch.float32, device=device),
                         torch.empty(1, dtype=torch.float32, device=device), n_out, k_in,
                         codebook)


# ------------------------------------------------------------------ host-only tables

CODEBOOK_NF4, CODEBOOK_UNIFORM4 = 0, 1
BUCKET_SCALE = 16                    # code-search buckets: round-half-even(16 x + 16)
CODE_BUCKETS = 2 * BUCKET_SCALE + 1


def codebook_tables(codebook: int):
    """(levels [16], thresholds [15], bucket thresholds [33], bucket codes [33]) of a
    codebook, as the library builds them."""
    lev, thr = (ctypes.c_float * 16)(), (ctypes.c_float * 15)()
    bthr, bcode = (ctypes.c_float * CODE_BUCKETS)(), (ctypes.c_uint8 * CODE_BUCKETS)()
    rc = lib().qlora_codebook_tables(codebook, ctypes.cast(lev, ctypes.c_void_p),
                                     ctypes.cast(thr, ctypes.c_void_p),
                                     ctypes.cast(bthr, ctypes.c_void_p),
                                     ctypes.cast(bcode, ctypes.c_void_p))
    if rc != 0:
        raise ValueError(f"unknown codebook {codebook}")
    return (torch.tensor(list(lev), dtype=torch.float32), torch.tensor(list(thr), dtype=torch.float32),
            torch.tensor(list(bthr), dtype=torch.float32), torch.tensor(list(bcode), dtype=torch.uint8))


def nf4_table() -> torch.Tensor:
    out = (ctypes.c_float * 16)()
    lib().qlora_nf4_table(ctypes.cast(out, ctypes.c_void_p))
    return torch.tensor(list(out), dtype=torch.float32)


def nf4_thresholds() -> torch.Tensor:
    out = (ctypes.c_float * 15)()
    lib().qlora_nf4_thresholds(ctypes.cast(out, ctypes.c_void_p))
    return torch.tensor(list(out), dtype=torch.float32)


def nf4_code_buckets():
    """(thr [33] fp32, code [33] uint8): the bucket table of the quantization kernel
    (bucket b = round-half-even(16 x + 16), code = code[b] + (x >= thr[b]))."""
    thr = (ctypes.c_float * CODE_BUCKETS)()
    code = (ctypes.c_uint8 * CODE_BUCKETS)()
    lib().qlora_nf4_code_buckets(ctypes.cast(thr, ctypes.c_void_p), ctypes.cast(code, ctypes.c_void_p))
    return (torch.tensor(list(thr), dtype=torch.float32),
            torch.tensor(list(code), dtype=torch.uint8))


def fp8_thresholds():
    th, vals, codes = (ctypes.c_float * 252)(), (ctypes.c_float * 253)(), (ctypes.c_uint8 * 253)()
    lib().qlora_fp8_thresholds(ctypes.cast(th, ctypes.c_void_p), ctypes.cast(vals, ctypes.c_void_p),
                               ctypes.cast(codes, ctypes.c_void_p))
    return (torch.tensor(list(th), dtype=torch.float32), torch.tensor(list(vals), dtype=torch.float32),
            torch.tensor(list(codes), dtype=torch.uint8))


# ------------------------------------------------------------------ entry points

def qlora_quantize_workspace_size(n_out: int, k_in: int) -> int:
    return int(lib().qlora_quantize_workspace_size(n_out, k_in))


def qlora_quantize_nf4_dq(W: torch.Tensor, out: NF4Weight | None = None,
                          workspace: torch.Tensor | None = None, codebook: int = 0) -> NF4Weight:
    """4-bit (NF4 by default, or the uniform codebook) + double quantization of
    W [N, K] (fp32 or bf16, CUDA, contiguous)."""
    if W.dim() != 2 or not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D CUDA tensor")
    dtype = {torch.float32: F32, torch.bfloat16: BF16}.get(W.dtype)
    if dtype is None:
        raise TypeError(f"unsupported weight dtype {W.dtype}")
    n, k = W.shape
    q = out if out is not None else NF4Weight.empty(n, k, W.device, codebook)
    q.codebook = codebook
    need = qlora_quantize_workspace_size(n, k)
    ws = workspace if workspace is not None else torch.empty(max(need, 16), dtype=torch.uint8,
                                                             device=W.device)
    _check(lib().qlora_quantize_dq(_ptr(W), dtype, n, k, codebook, _ptr(q.codes), _ptr(q.c2),
                                   _ptr(q.c1), _ptr(q.mean), _ptr(ws), ws.numel(), _stream()),
           "qlora_quantize_dq")
    return q


def qlora_dequant(w: NF4Weight, out: torch.Tensor | None = None) -> torch.Tensor:
    """doubleDequant of the stored weight to bf16 [N, K]."""
    y = out if out is not None else torch.empty(w.n_out, w.k_in, dtype=torch.bfloat16,
                                                device=w.codes.device)
    _check(lib().qlora_dequant(w.c_struct(), _ptr(_as_bits(y)), _stream()), "qlora_dequant")
    return y


def qlora_merge_lora(w: NF4Weight, A: torch.Tensor, B: torch.Tensor, scale: float,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """merge_and_unload: bf16(W_hat + scale (A B)^T) [N, K]; A [K, r], B [r, N] bf16."""
    r = int(A.shape[1])
    y = out if out is not None else torch.empty(w.n_out, w.k_in, dtype=torch.bfloat16,
                                                device=w.codes.device)
    _check(lib().qlora_merge_lora(w.c_struct(), _ptr(_as_bits(A)), _ptr(_as_bits(B)), r,
                                  float(scale), _ptr(_as_bits(y)), _stream()), "qlora_merge_lora")
    return y


def qlora_linear_fwd_workspace_size(M: int, n_out: int, k_in: int, r: int) -> int:
    return int(lib().qlora_linear_fwd_workspace_size(M, n_out, k_in, r))


def qlora_linear_bwd_workspace_size(M: int, n_out: int, k_in: int, r: int) -> int:
    return int(lib().qlora_linear_bwd_workspace_size(M, n_out, k_in, r))


def qlora_linear_fwd(X: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor, scale: float,
                     save_T: bool = True, Y: torch.Tensor | None = None,
                     T: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Y = bf16(X W_hat^T + scale (X A) B). Returns (Y, T) with T = X A (fp32) or None."""
    M, K = X.shape
    r = A.shape[1]
    dev = X.device
    Y = Y if Y is not None else torch.empty(M, w.n_out, dtype=torch.bfloat16, device=dev)
    if save_T and T is None:
        T = torch.empty(M, r, dtype=torch.float32, device=dev)
    need = qlora_linear_fwd_workspace_size(M, w.n_out, w.k_in, r)
    ws = workspace if workspace is not None else torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().qlora_linear_fwd(_ptr(_as_bits(X)), M, w.c_struct(), _ptr(_as_bits(A)),
                                  _ptr(_as_bits(B)), r, float(scale), _ptr(_as_bits(Y)),
                                  _ptr(T if save_T else None), _ptr(ws), ws.numel(), _stream()),
           "qlora_linear_fwd")
    return Y, (T if save_T else None)


def qlora_linear_bwd(dY: torch.Tensor, X: torch.Tensor, T: torch.Tensor | None, w: NF4Weight,
                     A: torch.Tensor, B: torch.Tensor, scale: float, need_dX: bool = True,
                     dX: torch.Tensor | None = None, dA: torch.Tensor | None = None,
                     dB: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Gradients (dX bf16 or None, dA fp32 [K, r], dB fp32 [r, N]); W is frozen."""
    M = X.shape[0]
    r = A.shape[1]
    dev = X.device
    if need_dX and dX is None:
        dX = torch.empty(M, w.k_in, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(w.k_in, r, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(r, w.n_out, dtype=torch.float32, device=dev)
    need = qlora_linear_bwd_workspace_size(M, w.n_out, w.k_in, r)
    ws = workspace if workspace is not None else torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().qlora_linear_bwd(_ptr(_as_bits(dY)), _ptr(_as_bits(X)), _ptr(T), M, w.c_struct(),
                                  _ptr(_as_bits(A)), _ptr(_as_bits(B)), r, float(scale),
                                  _ptr(_as_bits(dX) if need_dX else None), _ptr(dA), _ptr(dB),
                                  _ptr(ws), ws.numel(), _stream()),
           "qlora_linear_bwd")
    return (dX if need_dX else None), dA, dB


def qlora_shard_rows(n_out: int, k_in: int, world: int, rank: int):
    """(row0, rows) of shard `rank` of `world` for a column (N) split of an n_out x k_in
    weight: near-equal parts cut only where row * k_in % 65536 == 0."""
    r0, rows = ctypes.c_int64(0), ctypes.c_int64(0)
    _check(lib().qlora_shard_rows(n_out, k_in, world, rank, ctypes.byref(r0), ctypes.byref(rows)),
           "qlora_shard_rows")
    return int(r0.value), int(rows.value)


def qlora_shard_weight(w: NF4Weight, row0: int, rows: int) -> NF4Weight:
    """Rows [row0, row0 + rows) of w as a weight of its own: views of w's buffers (no copy),
    checked by the library (cuts where row0 * k_in % 65536 == 0)."""
    out = CNF4Weight()
    _check(lib().qlora_shard_weight(w.c_struct(), row0, rows, ctypes.byref(out)), "qlora_shard_weight")
    k = w.k_in
    view = NF4Weight(w.codes[row0 * k // 2:(row0 + rows) * k // 2],
                     w.c2[row0 * k // 64:(row0 + rows) * k // 64],
                     w.c1[row0 * k // 16384:-(-(row0 + rows) * k // 16384)],
                     w.mean, rows, k, w.codebook)
    assert view.codes.data_ptr() == out.codes and view.c1.data_ptr() == out.c1
    return view


def qlora_linear_bwd_shard_g(dY: torch.Tensor, B: torch.Tensor, G_part: torch.Tensor | None = None):
    """G_part [M, r] fp32 = dY B^T for one shard's dY [M, n_shard] and B [r, n_shard]."""
    M, n = dY.shape
    r = B.shape[0]
    G_part = G_part if G_part is not None else torch.empty(M, r, dtype=torch.float32, device=dY.device)
    need = int(lib().qlora_linear_bwd_shard_g_workspace_size(M, n, r))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dY.device)
    _check(lib().qlora_linear_bwd_shard_g(_ptr(_as_bits(dY)), M, n, _ptr(_as_bits(B)), r, _ptr(G_part),
                                          _ptr(ws), ws.numel(), _stream()), "qlora_linear_bwd_shard_g")
    return G_part


def qlora_linear_bwd_shard(dY: torch.Tensor, X: torch.Tensor, T: torch.Tensor | None,
                           G: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor,
                           scale: float, lora_in_dx: bool, need_dX: bool = True):
    """One shard's (dX_part fp32 [M, K] or None, dA [K, r], dB [r, n_shard]) given G summed
    over the shards; dX_part carries scale G A^T only when lora_in_dx."""
    M = X.shape[0]
    r = A.shape[1]
    dev = X.device
    dXp = torch.empty(M, w.k_in, dtype=torch.float32, device=dev) if need_dX else None
    dA = torch.empty(w.k_in, r, dtype=torch.float32, device=dev)
    dB = torch.empty(r, w.n_out, dtype=torch.float32, device=dev)
    need = int(lib().qlora_linear_bwd_shard_workspace_size(M, w.n_out, w.k_in, r))
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _check(lib().qlora_linear_bwd_shard(_ptr(_as_bits(dY)), _ptr(_as_bits(X)), _ptr(T), _ptr(G), M,
                                        w.c_struct(), _ptr(_as_bits(A)), _ptr(_as_bits(B)), r,
                                        float(scale), int(bool(lora_in_dx)), _ptr(dXp), _ptr(dA),
                                        _ptr(dB), _ptr(ws), ws.numel(), _stream()),
           "qlora_linear_bwd_shard")
    return dXp, dA, dB


def qlora_f32_to_bf16(src: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """bf16_rn of an fp32 tensor (numel % 4 == 0)."""
    out = out if out is not None else torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    _check(lib().qlora_f32_to_bf16(_ptr(src), _ptr(_as_bits(out)), src.numel(), _stream()),
           "qlora_f32_to_bf16")
    return out


def qlora_profile_events(before=None, after=None):
    """Record torch.cuda.Event pair (or None) around each fused-GEMM launch of this thread."""
    lib().qlora_profile_events(ctypes.c_void_p(before.cuda_event) if before is not None else None,
                               ctypes.c_void_p(after.cuda_event) if after is not None else None)


def qlora_launch_count() -> int:
    """Kernel launches this library has enqueued so far in this process."""
    return int(lib().qlora_launch_count())


def qlora_selftest_wait_timeout() -> None:
    """Enqueue the failure-path self-test: one kernel whose wait runs out after 2 s and
    records QLORA_ERR_TIMEOUT in the device error word (read it with qlora_device_error)."""
    _check(lib().qlora_selftest_wait_timeout(_stream()), "qlora_selftest_wait_timeout")


def qlora_device_error(clear: bool = True) -> int:
    """Status of the device error word (QLORA_ERR_TIMEOUT after a timed-out wait)."""
    return int(lib().qlora_device_error(1 if clear else 0))


# ---------------------------------------------------------------- optimizer step
class PagedBuffer:
    """Unified (managed) memory from qlora_paged_alloc, zero-filled: a paged optimizer
    state. The driver moves its pages between host and device memory on demand;
    prefetch() moves them ahead of use. Released by free() or when collected."""

    def __init__(self, nbytes: int):
        ptr = ctypes.c_void_p()
        _check(lib().qlora_paged_alloc(ctypes.byref(ptr), nbytes), "qlora_paged_alloc")
        self.ptr, self.nbytes = ptr.value, int(nbytes)

    def prefetch(self, to_device: bool = True):
        _check(lib().qlora_paged_prefetch(ctypes.c_void_p(self.ptr), self.nbytes,
                                          1 if to_device else 0, _stream()), "qlora_paged_prefetch")

    def host_bytes(self) -> bytes:
        """A host copy of the contents (synchronise the device first)."""
        return ctypes.string_at(self.ptr, self.nbytes)

    def free(self):
        if self.ptr:
            _check(lib().qlora_paged_free(ctypes.c_void_p(self.ptr)), "qlora_paged_free")
            self.ptr = None

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


def qlora_adamw_state_bytes(n: int, state_bits: int = 8) -> int:
    return int(lib().qlora_adamw_state_bytes(n, state_bits))


def qlora_adamw_step(p: torch.Tensor, g: torch.Tensor, state, step: int, *, lr: float = 2e-4,
                     beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
                     weight_decay: float = 0.0, state_bits: int = 8,
                     p_bf16: torch.Tensor | None = None) -> None:
    """One AdamW update of the fp32 parameters p (in place) with gradient g; state is a
    uint8 CUDA tensor or a PagedBuffer of qlora_adamw_state_bytes(p.numel(), state_bits)
    bytes (zeros before the first step). p_bf16, when given, receives bf16(p)."""
    for t, name in ((p, "p"), (g, "g")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous fp32 CUDA tensor")
    if g.numel() != p.numel():
        raise ValueError("p and g differ in size")
    if p_bf16 is not None and (_as_bits(p_bf16).numel() != p.numel()):
        raise ValueError("p_bf16 differs in size from p")
    if isinstance(state, PagedBuffer):
        sptr, sbytes = ctypes.c_void_p(state.ptr), state.nbytes
    else:
        if not state.is_cuda or not state.is_contiguous():
            raise ValueError("state: expected a contiguous CUDA tensor")
        sptr, sbytes = _ptr(state), state.numel() * state.element_size()
    hp = CAdamwHparams(lr, beta1, beta2, eps, weight_decay, step)
    _check(lib().qlora_adamw_step(_ptr(p), _ptr(p_bf16), _ptr(g), p.numel(), state_bits, sptr,
                                  sbytes, hp, _stream()), "qlora_adamw_step")
