"""Double quantisation with mean centring (a variant of the constants'
encoding, for an error ablation against the plain scheme).

TEST INFRASTRUCTURE ONLY (see the package header).  This module fixes what
the library's mean-centred quantiser and dequantisers must compute.

The pages describe double quantisation as "the quantisation constants are
themselves quantised to FP8 in blocks of 256" ("QLoRA" encyclopedia entry,
tonho.wtf, section "como funciona") and say nothing of centring; the
original QLoRA paper (outside the pages) subtracts the mean of the constants
first, because they are all positive and a symmetric FP8 grid would waste
its sign.  Readings taken here:

* one mean per tensor: mean = fp32(S / n) for the n block constants c_i,
  where S is their pairwise sum in fp64: the constants, padded with zeros to
  a power of two, are added in neighbouring pairs, level by level, until one
  value is left.  The order is fixed, so a parallel implementation reproduces
  it exactly, and its rounding error grows with log2(n), not n;
* per group: c' = RN32(c - mean); s2 = RN32(max|c'| / 448);
  c8 = E4M3_RNE_satfinite(RN32(c' / s2)) (0 when s2 = 0);
* dequantised constant: c_hat = RN32(RN32(e4m3(c8) * s2) + mean).

The 4-bit codes are unchanged (they come from the exact constants), and the
dequantised weight is w' = bf16(RN32(q[code] * c_hat)) as in the plain scheme.

Parity status: pinned (constant constants reconstruct exactly; the pairwise
sum's tree shape on inputs where other orders round differently, and its
textbook error bound; the mean against an exact rational mean within one
fp32 rounding; the
reconstruction error within the E4M3 half-step bound per group; the plain
scheme's error bound recovered when the mean is forced to zero).
"""

import numpy as np

from .nf4 import BLOCK, GROUP, FP8_MAX, absmax_constants, codebook, encode_codes, pack_codes, unpack_codes
from .numerics import e4m3_decode, e4m3_encode, f32_to_bf16_bits


def pairwise_sum(x):
    """fp64 pairwise sum: zero-pad to a power of two, then replace the array
    by the sums of its neighbouring pairs (x[0] + x[1], x[2] + x[3], ...)
    until one value is left."""
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    p = 1
    while p < x.size:
        p *= 2
    level = np.zeros(p, dtype=np.float64)
    level[: x.size] = x
    while level.size > 1:
        level = level[0::2] + level[1::2]
    return level[0]


def constants_mean(c):
    """fp32 mean of the block constants: their fp64 pairwise sum divided by
    their count in fp64, rounded once to fp32."""
    c = np.asarray(c, dtype=np.float32)
    return np.float32(pairwise_sum(c.astype(np.float64)) / np.float64(c.size))


def double_quantize_centered(c, mean=None):
    """(c8, s2, mean) for the block constants ``c``; ``mean`` overrides the
    tensor mean (used by the pins)."""
    c = np.asarray(c, dtype=np.float32)
    mean = constants_mean(c) if mean is None else np.float32(mean)
    n = c.size
    ng = -(-n // GROUP)
    cp = np.zeros(ng * GROUP, dtype=np.float32)
    cp[:n] = (c - mean).astype(np.float32)
    cg = cp.reshape(ng, GROUP)
    # padding entries of a short last group are 0 after centring: they cannot
    # raise the group's maximum
    amax = np.max(np.abs(cg), axis=1).astype(np.float32)
    s2 = (amax / np.float32(FP8_MAX)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (cg / s2[:, None]).astype(np.float32)
    y[s2 == 0] = 0.0
    c8 = e4m3_encode(y).reshape(-1)[:n]
    return c8, s2, mean


def dequantized_constants_centered(c8, s2, mean):
    """c_hat = RN32(RN32(e4m3(c8) * s2[group]) + mean)."""
    c8 = np.asarray(c8, dtype=np.uint8)
    s2 = np.asarray(s2, dtype=np.float32)
    g = np.arange(c8.size) // GROUP
    return ((e4m3_decode(c8) * s2[g]).astype(np.float32) + np.float32(mean)).astype(np.float32)


def quantize_centered(w_bits, numel=None):
    """NF4 quantisation with mean-centred double quantisation of a bf16
    tensor (flattened row-major): ``(codes_packed, c8, s2, mean)``.  The codes
    are those of the plain scheme; only the constants' encoding differs."""
    w_bits = np.asarray(w_bits, dtype=np.uint16).reshape(-1)
    numel = w_bits.size if numel is None else numel
    c = absmax_constants(w_bits, numel)
    codes = encode_codes(w_bits, numel, c)
    c8, s2, mean = double_quantize_centered(c)
    return pack_codes(codes), c8, s2, mean


def dequantize_centered(codes_packed, c8, s2, mean, numel):
    """bf16 bit patterns of w' = bf16(RN32(q[code] * c_hat)), c_hat from
    :func:`dequantized_constants_centered` (two roundings there, two here)."""
    nblocks = -(-numel // BLOCK)
    codes = unpack_codes(codes_packed, nblocks * BLOCK).reshape(nblocks, BLOCK)
    chat = dequantized_constants_centered(c8, s2, mean)
    vals = (codebook()[codes] * chat[:, None]).astype(np.float32)
    return f32_to_bf16_bits(vals).reshape(-1)[:numel]
