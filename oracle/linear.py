"""Forward and backward of the adapter-augmented frozen linear, in fp64.

TEST INFRASTRUCTURE ONLY (see the package header).

Notation (PyTorch ``Linear`` convention): W' is the dequantised base weight
[N = out, K = in]; X is [M, K]; the LoRA adapters are A [r, K] and
B [N, r]; s = alpha / r.  The forward is

    U  = X A^T                    (the adapter's down projection)
    Y  = X W'^T + s U B^T

and, for an upstream gradient dY [M, N], the backward is

    dU = s dY B
    dX = dY W' + dU A             (the gradient crosses the frozen weight)
    dA = dU^T X
    dB = s dY^T U                 (no dW: the base is frozen)

Sources: "QLoRA" encyclopedia entry (tonho.wtf), section "a ideia" — the
frozen 4-bit weight is dequantised to BF16 for the matmul, the gradient
passes through it into the LoRA adapters, which are the only parameters with
their own gradient; "Tutorial fine-tuning LLM LoRA/QLoRA 2026"
(nexusinovation), section "LoRA: O Padrão Ouro de Eficiência" — the adapter
adds a scaled product of two low-rank matrices to the frozen weight (the
page's letters and shapes differ from the ones above; the product is the
same merged weight W' + s B A).

Every product is a plain numpy fp64 matrix product of the exact (bf16 or
fp32) inputs; nothing is rounded in between.  Parity status: pinned
(pure-Python brute force on tiny shapes, the merged-weight identity, the
special cases W' = 0 and B = 0, and central finite differences of
L = sum(Y * dY) in tests/test_oracle_linear.py).
"""

import numpy as np

from .numerics import bf16_bits_to_f32


def _f64(bits_or_f32):
    a = np.asarray(bits_or_f32)
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def linear_fwd(X, Wd, A, B, s):
    """Return (U, Y) in fp64.  Inputs are bf16 bit arrays or float arrays."""
    X, Wd, A, B = _f64(X), _f64(Wd), _f64(A), _f64(B)
    U = X @ A.T
    Y = X @ Wd.T + float(s) * (U @ B.T)
    return U, Y


def linear_bwd(dY, X, Wd, A, B, s, want_dx=True):
    """Return (dX, dA, dB, dU) in fp64 (dX is None when ``want_dx`` is False)."""
    dY, X, A, B = _f64(dY), _f64(X), _f64(A), _f64(B)
    s = float(s)
    U = X @ A.T
    dU = s * (dY @ B)
    dX = dY @ _f64(Wd) + dU @ A if want_dx else None
    dA = dU.T @ X
    dB = s * (dY.T @ U)
    return dX, dA, dB, dU


def rel_frobenius(got, ref):
    """||got - ref||_F / ||ref||_F in fp64 (0 when both are zero)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)
