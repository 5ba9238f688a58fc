"""Why the decode kernels expand every weight to its exact bf16 value (host only, oracle
arithmetic). The layer's weight is W_hat = bf16_rn(fl32(L[code] s)) (page "QLoRA", itwiki.kr,
section "계산 방식", doubleDequant), and Y is checked against bf16(X W_hat^T) of the
oracle with a relative Frobenius bound of 2e-3.

- A GEMV that skipped the per-weight bf16 rounding (one multiply by s after the dot
  product over L[code]) would compute with L[code] s instead. Its bf16 output misses the
  bound: about 2.6e-3 on N(0, 0.02) weights, whatever the shape.
- The route the kernels take (exact bf16 weights, fp32 accumulation, one bf16 rounding)
  stays far inside it."""
import numpy as np

from oracle import nf4_oracle as O


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_scaling_after_the_dot_product_misses_the_tolerance():
    rng = np.random.default_rng(2)
    N, K, M = 256, 2048, 1
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    X = O.bf16_round(rng.normal(0, 1, (M, K)).astype(np.float32))
    q = O.quantize_nf4_dq(W)
    W_hat = O.double_dequant(q).astype(np.float64)              # exact bf16 weights
    s = O.reconstruct_absmax(q["c2"], q["c1"], q["mean"]).astype(np.float64)
    codes = O.unpack_nibbles(q["codes"]).reshape(-1, 64)
    levels = O.nf4_levels().astype(np.float64)
    W_unrounded = (levels[codes] * s[:, None]).reshape(N, K)    # L[code] * s, no rounding
    X64 = X.astype(np.float64)
    y_ref = O.bf16_round((X64 @ W_hat.T).astype(np.float32)).astype(np.float64)
    # the skipped-rounding route, even with an exact (fp64) dot product
    y_skip = O.bf16_round((X64 @ W_unrounded.T).astype(np.float32)).astype(np.float64)
    assert _rel(y_skip, y_ref) > 2e-3
    # the kernels' route: exact bf16 weights, fp32 products and sums, one bf16 rounding
    y_kernel = O.bf16_round(X @ W_hat.astype(np.float32).T).astype(np.float64)
    assert _rel(y_kernel, y_ref) < 2e-4
