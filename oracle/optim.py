"""Adapter optimizer step: AdamW with 8-bit states in paged memory.

TEST INFRASTRUCTURE ONLY (see the package header).

Sources: the "QLoRA" encyclopedia entry (tonho.wtf), section "como funciona"
(the third piece: optimizer states live in NVIDIA unified memory, are evicted
to CPU RAM when the GPU runs short and brought back for the update), and the
"Tutorial fine-tuning LLM LoRA/QLoRA 2026" (nexusinovation), section "Mão na
Massa" (the trainer uses ``paged_adamw_8bit`` at learning rate 2e-4, and the
step-by-step notes say the optimizer keeps its state in 8 bits).

The pages name the optimizer but fix neither its update nor the 8-bit format.
Readings taken here:

* the update is AdamW (Adam with decoupled weight decay) with bias
  correction; hyper-parameters are inputs (the trainer's defaults are
  beta1 = 0.9, beta2 = 0.999, eps = 1e-8, weight decay 0);
* the 8-bit state uses the pages' own two-level FP8 scheme for quantisation
  constants: blocks of 256 elements, one fp32 absmax scale per block, E4M3
  codes (RNE, saturating); the first moment m is stored directly, the second
  moment v as its square root u = sqrt(v), which halves its dynamic range so
  that small second moments in a block do not flush to zero;
* every operation is one IEEE fp32 operation rounded to nearest even, in the
  order written below; the bias corrections are host constants computed in
  fp64 and rounded once to fp32.

Per element (p the bf16 parameter widened to fp32, g the fp32 gradient):

    m  = RN(e4m3(m8) * m_scale)       u = RN(e4m3(u8) * u_scale)    v = RN(u*u)
    m1 = RN(RN(b1*m) + RN((1-b1)*g))
    v1 = RN(RN(b2*v) + RN((1-b2)*RN(g*g)))
    u1 = sqrt_RN(v1)
    d  = RN(RN(m1*bc1) / RN(RN(u1*bc2) + eps))
    d  = RN(d + RN(wd*p))
    p1 = RN(p - RN(lr*d));  stored as bf16(p1)

and per block the new state is re-encoded from m1 and u1:
m_scale = RN(max|m1| / 448), m8 = E4M3(RN(m1 / m_scale)) (0 when the scale
is 0), and the same for u1.  1 - b1 and 1 - b2 are exact in fp32 for
b in [0.5, 1].

Parity status: pinned (first-step closed form, weight-decay-only closed form,
power-of-two gradient-scale invariance with eps = 0, trajectory against an
unquantised fp64 AdamW within the state-quantisation error, block locality).
"""

import math

import numpy as np

from .numerics import bf16_bits_to_f32, e4m3_decode, e4m3_encode, f32_to_bf16_bits

STATE_BLOCK = 256   # elements per fp32 state scale (the pages' FP8 group size)
FP8_MAX = 448.0


def bias_corrections(beta1, beta2, step):
    """(bc1, bc2) = fp32(1 / (1 - b1^t)), fp32(1 / sqrt(1 - b2^t)), from fp64."""
    b1 = float(np.float32(beta1))
    b2 = float(np.float32(beta2))
    bc1 = np.float32(1.0 / (1.0 - b1 ** step))
    bc2 = np.float32(1.0 / math.sqrt(1.0 - b2 ** step))
    return bc1, bc2


def init_state(n):
    """Zero state for n parameters: (m8, u8, m_scale, u_scale)."""
    nb = -(-n // STATE_BLOCK)
    return (np.zeros(n, np.uint8), np.zeros(n, np.uint8), np.zeros(nb, np.float32), np.zeros(nb, np.float32))


def _decode(codes, scale):
    n = codes.size
    blk = np.arange(n) // STATE_BLOCK
    return (e4m3_decode(codes).astype(np.float32) * scale[blk]).astype(np.float32)


def encode_state(x):
    """Blockwise E4M3 with an fp32 absmax scale per 256 elements."""
    x = np.asarray(x, dtype=np.float32)
    n = x.size
    nb = -(-n // STATE_BLOCK)
    pad = np.zeros(nb * STATE_BLOCK, np.float32)
    pad[:n] = x
    xb = pad.reshape(nb, STATE_BLOCK)
    amax = np.max(np.abs(xb), axis=1).astype(np.float32)
    scale = (amax / np.float32(FP8_MAX)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (xb / scale[:, None]).astype(np.float32)
    y[scale == 0] = 0.0
    return e4m3_encode(y).reshape(-1)[:n], scale


def adamw8_step(p_bits, grad, state, lr, beta1, beta2, eps, weight_decay, step, return_f32=False):
    """One AdamW step with 8-bit states.  Returns (p_bits_new, state_new)
    (and the fp32 parameter before the bf16 rounding when ``return_f32``)."""
    f = np.float32
    p = bf16_bits_to_f32(np.asarray(p_bits, dtype=np.uint16)).astype(np.float32)
    g = np.asarray(grad, dtype=np.float32)
    m8, u8, ms, us = state
    b1, b2, e, lr_, wd = f(beta1), f(beta2), f(eps), f(lr), f(weight_decay)
    omb1, omb2 = f(f(1.0) - b1), f(f(1.0) - b2)
    bc1, bc2 = bias_corrections(beta1, beta2, step)

    m = _decode(m8, ms)
    u = _decode(u8, us)
    v = (u * u).astype(np.float32)
    m1 = ((b1 * m).astype(f) + (omb1 * g).astype(f)).astype(f)
    gg = (g * g).astype(f)
    v1 = ((b2 * v).astype(f) + (omb2 * gg).astype(f)).astype(f)
    u1 = np.sqrt(v1).astype(f)
    num = (m1 * bc1).astype(f)
    den = ((u1 * bc2).astype(f) + e).astype(f)
    d = (num / den).astype(f)
    d = (d + (wd * p).astype(f)).astype(f)
    p1 = (p - (lr_ * d).astype(f)).astype(f)

    m8n, msn = encode_state(m1)
    u8n, usn = encode_state(u1)
    out = (f32_to_bf16_bits(p1), (m8n, u8n, msn, usn))
    return out + (p1,) if return_f32 else out


def adamw_f64(p, grad_steps, lr, beta1, beta2, eps, weight_decay):
    """Textbook AdamW in fp64 with unquantised states (a pin, not the method).
    ``grad_steps`` is a sequence of gradients, one per step; returns the
    parameter after the last step."""
    p = np.asarray(p, dtype=np.float64).copy()
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    for t, g in enumerate(grad_steps, start=1):
        g = np.asarray(g, dtype=np.float64)
        m = beta1 * m + (1 - beta1) * g
        v = beta2 * v + (1 - beta2) * g * g
        mh = m / (1 - beta1 ** t)
        vh = v / (1 - beta2 ** t)
        p = p - lr * (mh / (np.sqrt(vh) + eps) + weight_decay * p)
    return p
