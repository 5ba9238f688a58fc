"""Plain CPU oracle for the optimizer step that follows the LoRA gradients: AdamW on the
LoRA parameters with paged optimizer states kept in 32-bit or 8-bit form.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``
may import this module. The CUDA library shares no code with it.

Sources, by page title and section:

* "QLoRA" (itwiki.kr), section "페이지드 옵티마이저" (paged optimizers): optimizer
  states are allocated in unified memory, moved to host memory automatically when the
  GPU runs short and brought back for the optimizer update; the 8-bit optimizer states
  come from the same authors' block-wise quantization work.
* same page, the training example in section "계산 방식": ``optim="paged_adamw_8bit"``
  (paged 8-bit AdamW) at learning rate 2e-4; ``paged_adamw_32bit`` is named beside it.
* same page, section "이중 양자화": the pages' own 8-bit float with one fp32 absmax per
  block of 256 values (used here for the 8-bit states, see below).

Readings where the pages are silent (each stated in the design notes):
* AdamW is Adam with decoupled weight decay. Per element, in this order, every
  operation one IEEE fp32 rounding (no fused multiply-add):
      m  = b1*m' + (1-b1)*g              v  = b2*v' + ((1-b2)*g)*g
      mh = m / bc1                       vh = v / bc2      (bc_i = fl32(1 - b_i^t), t >= 1)
      u  = mh / (sqrt(vh) + eps)
      p  = p*(1 - lr*wd) - lr*u
  with (1-b1), (1-b2) and (1 - lr*wd) formed once in fp32, and bc_i computed in fp64
  and rounded to fp32. The bf16 copy of p for the forward is bf16_rn(p).
* 8-bit states: the pages do not give the block-wise format of the optimizer work.
  The plainest reading that the pages support is their own block-wise 8-bit float:
  m and v are stored, per block of 256 consecutive elements of the flat parameter
  buffer, as one fp32 absmax a and one E4M3 code per element, the nearest entry of
  T8 (the 253 distinct finite E4M3 values / 448, ties to the lower index) to
  fl32(x / a) (0 when a = 0). A stored state reads back as fl32(T8[code] * a).
  The update uses the fp32 m and v of this step; only their stored form is 8-bit.
* The states start at zero (codes 0x00, absmax 0, or fp32 zeros).
"""
from __future__ import annotations

import math

import numpy as np

from oracle.nf4_oracle import DQ_BLOCK, fp8_code_to_t8, fp8_table, nearest_code

STATE_BLOCK = DQ_BLOCK  # elements per absmax block of an 8-bit state


def hyper(lr, beta1, beta2, eps, weight_decay, step):
    """The fp32 constants of one step, formed as the reading above states."""
    f = np.float32
    b1, b2 = f(beta1), f(beta2)
    return dict(
        b1=b1, b2=b2, omb1=f(f(1.0) - b1), omb2=f(f(1.0) - b2), lr=f(lr), eps=f(eps),
        decay=f(f(1.0) - f(f(lr) * f(weight_decay))),
        bc1=f(1.0 - math.pow(float(b1), step)), bc2=f(1.0 - math.pow(float(b2), step)))


def encode_state(x: np.ndarray, block: int = STATE_BLOCK):
    """fp32 values -> (E4M3 codes uint8 [n], absmax fp32 [ceil(n / block)])."""
    x = np.asarray(x, np.float32).ravel()
    n = x.size
    nblk = -(-n // block)
    absmax = np.zeros(nblk, np.float32)
    y = np.zeros(n, np.float32)
    for b in range(nblk):
        seg = x[b * block:(b + 1) * block]
        a = np.max(np.abs(seg)) if seg.size else np.float32(0)
        absmax[b] = a
        if a > 0:
            y[b * block:b * block + seg.size] = seg / a          # fp32 division
    vals, codes = fp8_table()
    return codes[nearest_code(y, vals)].astype(np.uint8), absmax


def decode_state(codes: np.ndarray, absmax: np.ndarray, block: int = STATE_BLOCK) -> np.ndarray:
    """Stored 8-bit state -> fp32 values fl32(T8[code] * absmax of its block)."""
    t = fp8_code_to_t8(codes)
    a = np.repeat(np.asarray(absmax, np.float32), block)[:t.size]
    return (t * a).astype(np.float32)


def adamw_step(p, g, m_prev, v_prev, *, lr, beta1, beta2, eps, weight_decay, step):
    """One AdamW update in fp32 with the operation order of the module docstring.
    Returns (p_new fp32, p_bf16 as fp32 values, m fp32, v fp32)."""
    from oracle.nf4_oracle import bf16_round
    h = hyper(lr, beta1, beta2, eps, weight_decay, step)
    p = np.asarray(p, np.float32)
    g = np.asarray(g, np.float32)
    m = (h["b1"] * np.asarray(m_prev, np.float32) + h["omb1"] * g).astype(np.float32)
    v = (h["b2"] * np.asarray(v_prev, np.float32) + (h["omb2"] * g) * g).astype(np.float32)
    mh = (m / h["bc1"]).astype(np.float32)
    vh = (v / h["bc2"]).astype(np.float32)
    u = (mh / (np.sqrt(vh) + h["eps"])).astype(np.float32)
    p_new = (p * h["decay"] - h["lr"] * u).astype(np.float32)
    return p_new, bf16_round(p_new), m, v


def adamw_step_8bit(p, g, state, **hp):
    """The same step with 8-bit states: state = dict(mc, ma, vc, va) as stored; returns
    (p_new, p_bf16, new state dict)."""
    m_prev = decode_state(state["mc"], state["ma"])
    v_prev = decode_state(state["vc"], state["va"])
    p_new, p_bf, m, v = adamw_step(p, g, m_prev, v_prev, **hp)
    mc, ma = encode_state(m)
    vc, va = encode_state(v)
    return p_new, p_bf, dict(mc=mc, ma=ma, vc=vc, va=va)


def zero_state_8bit(n: int) -> dict:
    nblk = -(-n // STATE_BLOCK)
    return dict(mc=np.zeros(n, np.uint8), ma=np.zeros(nblk, np.float32),
                vc=np.zeros(n, np.uint8), va=np.zeros(nblk, np.float32))
