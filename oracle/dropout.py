"""LoRA dropout on the adapter input, with a counter-based mask.

TEST INFRASTRUCTURE ONLY (see the package header).

Source: "Tutorial fine-tuning LLM LoRA/QLoRA 2026" (nexusinovation), section
"Mão na Massa": the adapter configuration sets ``lora_dropout=0.05``.  The
page does not say where the dropout acts; the reading taken here is the
usual one for LoRA adapters: dropout on the adapter's input only, so the
frozen path sees X and the adapter sees X_drop:

    U  = X_drop A^T                     Y  = X W'^T + s U B^T
    dU = s dY B                         dX = dY W' + (keep * c) (dU A)
    dA = dU^T X_drop                    dB = s dY^T U

Readings for the mask and the scaling (none is on the pages):

* the mask comes from Philox-4x32-10 (Salmon, Moraes, Dror and Shaw,
  "Parallel random numbers: as easy as 1, 2, 3", SC 2011), with key
  (seed mod 2^32, seed div 2^32) and counter (g mod 2^32, g div 2^32, 0, 0)
  for the group g = e div 4 of the flattened element index e = m K + k; word
  e mod 4 of that call decides element e;
* element e is kept when its 32-bit word is below T = floor((1 - p) 2^32)
  (T = 2^32 for p = 0: everything kept), computed in fp64;
* a kept element is stored as bf16(RN32(x * c)) with c = fp32(1 / (1 - p))
  (fp64 division, one rounding), a dropped one as +0;
* the backward treats the rounding of X_drop as a rounding: the dropout's
  derivative is keep * c.

Parity status: pinned (Philox known-answer vectors, p = 0 reduces to the
plain linear bit for bit, keep fraction within binomial bounds, determinism
and seed sensitivity, central finite differences of the backward).
"""

import numpy as np

from .linear import _f64
from .numerics import bf16_bits_to_f32, f32_to_bf16_bits

_M0, _M1 = 0xD2511F53, 0xCD9E8D57      # Philox-4x32 round multipliers
_W0, _W1 = 0x9E3779B9, 0xBB67AE85      # Weyl key increments
_MASK32 = 0xFFFFFFFF


def philox4x32_10(counter, key):
    """Philox-4x32 with 10 rounds, vectorised over arrays of counters.

    counter: uint64 array [..., 4] of 32-bit words; key: uint64 array [..., 2].
    Returns a uint64 array [..., 4] of 32-bit output words.
    """
    c = np.asarray(counter, dtype=np.uint64) & np.uint64(_MASK32)
    k = np.asarray(key, dtype=np.uint64) & np.uint64(_MASK32)
    x0, x1, x2, x3 = (c[..., i].copy() for i in range(4))
    k0, k1 = k[..., 0].copy(), k[..., 1].copy()
    m0, m1, mask = np.uint64(_M0), np.uint64(_M1), np.uint64(_MASK32)
    for r in range(10):
        p0 = x0 * m0                       # < 2^64: exact in uint64
        p1 = x2 * m1
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        x0, x1, x2, x3 = (hi1 ^ x1 ^ k0) & mask, lo1, (hi0 ^ x3 ^ k1) & mask, lo0
        if r < 9:
            k0 = (k0 + np.uint64(_W0)) & mask
            k1 = (k1 + np.uint64(_W1)) & mask
    return np.stack([x0, x1, x2, x3], axis=-1)


def keep_threshold(p):
    """T = floor((1 - p) 2^32) as a Python int (2^32 when p = 0)."""
    p = float(np.float32(p))
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return int(np.floor((1.0 - p) * 2.0 ** 32))


def keep_scale(p):
    """c = fp32(1 / (1 - p)) from fp64."""
    return np.float32(1.0 / (1.0 - float(np.float32(p))))


def keep_mask(M, K, p, seed):
    """Boolean [M, K]: True where the element reaches the adapter."""
    T = keep_threshold(p)
    if T >= 1 << 32:
        return np.ones((M, K), dtype=bool)
    n = M * K
    e = np.arange(n, dtype=np.uint64)
    g = e // np.uint64(4)
    ctr = np.stack([g & np.uint64(_MASK32), g >> np.uint64(32), np.zeros_like(g), np.zeros_like(g)], axis=-1)
    seed = int(seed)
    key = np.broadcast_to(np.array([seed & _MASK32, (seed >> 32) & _MASK32], dtype=np.uint64), (n, 2))
    words = philox4x32_10(ctr, key)
    w = words[np.arange(n), (e % np.uint64(4)).astype(np.int64)]
    return (w < np.uint64(T)).reshape(M, K)


def dropout_bits(X_bits, p, seed):
    """X_drop as bf16 bit patterns: bf16(RN32(x * c)) where kept, +0 elsewhere."""
    X_bits = np.asarray(X_bits, dtype=np.uint16)
    M, K = X_bits.shape
    keep = keep_mask(M, K, p, seed)
    x = bf16_bits_to_f32(X_bits)
    scaled = f32_to_bf16_bits((x * keep_scale(p)).astype(np.float32))
    return np.where(keep, scaled, np.uint16(0)).astype(np.uint16)


def linear_fwd_dropout(X, Wd, A, B, s, p, seed):
    """Return (X_drop bits, U, Y) with U and Y in fp64."""
    Xd = dropout_bits(X, p, seed)
    X64, Xd64, Wd, A, B = _f64(X), _f64(Xd), _f64(Wd), _f64(A), _f64(B)
    U = Xd64 @ A.T
    Y = X64 @ Wd.T + float(s) * (U @ B.T)
    return Xd, U, Y


def linear_bwd_dropout(dY, X, Wd, A, B, s, p, seed):
    """Return (dX, dA, dB, dU) in fp64 for the dropout forward above."""
    M, K = np.asarray(X).shape
    keep = keep_mask(M, K, p, seed)
    Xd64 = _f64(dropout_bits(X, p, seed))
    dY, A, B = _f64(dY), _f64(A), _f64(B)
    s = float(s)
    U = Xd64 @ A.T
    dU = s * (dY @ B)
    dX = dY @ _f64(Wd) + (keep * float(keep_scale(p))) * (dU @ A)
    dA = dU.T @ Xd64
    dB = s * (dY.T @ U)
    return dX, dA, dB, dU
