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
L = sum(Y * dY) in tests/test_oracle_linear.py; for a group of linears that
share X, the same finite differences of the summed loss, and the group of
one equal to the single linear).
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


def group_fwd(X, Wd, A, B, s, n_member):
    """Forward of a group of linears that read the same X, stacked along the
    output dimension: member g owns rows off_g .. off_g + n_member[g] - 1 of
    Wd and B and rows g r .. g r + r - 1 of A.  Each member is the linear
    above; returns (U [M, G r], Y [M, N]) with the members side by side."""
    G = len(n_member)
    r = np.asarray(A).shape[0] // G
    off = np.concatenate([[0], np.cumsum(n_member)]).astype(int)
    Us, Ys = [], []
    for g in range(G):
        U, Y = linear_fwd(X, np.asarray(Wd)[off[g]:off[g + 1]], np.asarray(A)[g * r:(g + 1) * r],
                          np.asarray(B)[off[g]:off[g + 1]], s)
        Us.append(U)
        Ys.append(Y)
    return np.concatenate(Us, axis=1), np.concatenate(Ys, axis=1)


def group_bwd(dY, X, Wd, A, B, s, n_member, want_dx=True):
    """Backward of :func:`group_fwd`: each member's dA, dB as for one linear,
    stacked like A and B; dX is the sum of the members' dX (X feeds every
    member, so its gradient is the sum of theirs).  Returns (dX, dA, dB)."""
    G = len(n_member)
    r = np.asarray(A).shape[0] // G
    off = np.concatenate([[0], np.cumsum(n_member)]).astype(int)
    dX, dAs, dBs = None, [], []
    for g in range(G):
        rows = slice(off[g], off[g + 1])
        Wg = None if Wd is None else np.asarray(Wd)[rows]
        dXg, dAg, dBg, _ = linear_bwd(np.asarray(dY)[:, rows], X, Wg, np.asarray(A)[g * r:(g + 1) * r],
                                      np.asarray(B)[rows], s, want_dx=want_dx)
        if want_dx:
            dX = dXg if dX is None else dX + dXg
        dAs.append(dAg)
        dBs.append(dBg)
    return dX, np.concatenate(dAs, axis=0), np.concatenate(dBs, axis=0)


def rel_frobenius(got, ref):
    """||got - ref||_F / ||ref||_F in fp64 (0 when both are zero)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(got - ref)
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)
