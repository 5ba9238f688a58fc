"""Seeded synthetic inputs for the QLoRA linear layer.

Random draws only: no quantization, dequantization or matrix arithmetic lives
here, so both the CPU oracle (in the tests) and the CUDA path can take their
inputs from this module. NumPy ``default_rng(seed)`` throughout.

Workloads (weights are out x in = N x K):
* ``pr1``: one linear, W 512 x 1024 fp32 ~N(0, 0.02), LoRA r=8 alpha=16,
  A 1024 x 8 and B 8 x 512 ~N(0, 0.02), X 16 x 1024 and dY 16 x 512 ~N(0, 1)
  in bf16; seed 0, draw order W, A, B, X, dY.
* ``llama7b_codec``: bf16 weights 4096x4096, 4096x11008, 11008x4096
  ~N(0, 0.02) with 0.1 % of the entries multiplied by 10 (outliers); seed 1.
* decode: M in {1, 4, 16} bf16 activations against 4096x11008 and 8192x28672
  weights, r=16 alpha=32; seed 2.
* ``llama7b_layer``: q,k,v,o 4096x4096, gate/up 11008x4096, down 4096x11008,
  r=64 alpha=16, M=4096; seed 3.
"""
from __future__ import annotations

import numpy as np

LLAMA7B_LINEARS = [  # (name, N = out features, K = in features)
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
]
LLAMA65B_LINEARS = [
    ("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
    ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016),
]


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round fp32 draws to bf16 (nearest, ties to even) so that host and device
    start from identical bf16 inputs. Returned as fp32 holding bf16 values."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def normal(rng, shape, std, bf16=False):
    x = rng.normal(0.0, std, size=shape).astype(np.float32)
    return to_bf16_values(x) if bf16 else x


def weight(rng, n, k, bf16=True, outlier_frac=0.0, std=0.02):
    """~N(0, std) weights; a uniformly random ``outlier_frac`` of entries x10."""
    w = rng.normal(0.0, std, size=(n, k)).astype(np.float32)
    if outlier_frac > 0:
        cnt = int(round(outlier_frac * n * k))
        idx = rng.choice(n * k, size=cnt, replace=False)
        w.reshape(-1)[idx] *= 10.0
    return to_bf16_values(w) if bf16 else w


def pr1():
    """The small reference case (one linear, M=16)."""
    rng = np.random.default_rng(0)
    W = normal(rng, (512, 1024), 0.02)                 # fp32 weights
    A = normal(rng, (1024, 8), 0.02, bf16=True)
    B = normal(rng, (8, 512), 0.02, bf16=True)
    X = normal(rng, (16, 1024), 1.0, bf16=True)
    dY = normal(rng, (16, 512), 1.0, bf16=True)
    return dict(W=W, A=A, B=B, X=X, dY=dY, r=8, alpha=16.0, scale=16.0 / 8)


def linear_case(seed, M, N, K, r, alpha, w_fp32=False, outlier_frac=0.0):
    """A generic linear: W, A, B, X, dY drawn in that order."""
    rng = np.random.default_rng(seed)
    W = weight(rng, N, K, bf16=not w_fp32, outlier_frac=outlier_frac)
    A = normal(rng, (K, r), 0.02, bf16=True)
    B = normal(rng, (r, N), 0.02, bf16=True)
    X = normal(rng, (M, K), 1.0, bf16=True)
    dY = normal(rng, (M, N), 1.0, bf16=True)
    return dict(W=W, A=A, B=B, X=X, dY=dY, r=r, alpha=float(alpha), scale=alpha / r)


def decode_case(N, K, r=16, alpha=32.0, seed=2):
    """The decode workload on one weight: W [N, K] ~N(0, 0.02) bf16, A, B ~N(0, 0.02),
    X [16, K] ~N(0, 1) bf16, drawn in that order; a decode step of M <= 16 tokens takes
    the first M rows of X."""
    rng = np.random.default_rng(seed)
    W = weight(rng, N, K, bf16=True)
    A = normal(rng, (K, r), 0.02, bf16=True)
    B = normal(rng, (r, N), 0.02, bf16=True)
    X = normal(rng, (16, K), 1.0, bf16=True)
    return dict(W=W, A=A, B=B, X=X, r=r, alpha=float(alpha), scale=alpha / r)

