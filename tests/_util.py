"""Shared helpers of the GPU parity tests (oracle side runs on the host).

Every expected value comes from ``oracle`` applied to the inputs drawn by
``synth``; nothing computed by the CUDA path is ever fed to the oracle.
Large tensors are quantised by the oracle in chunks aligned to the
double-quantisation group (16384 elements): groups are independent, so a
chunked run equals a whole-tensor run.
"""

import numpy as np
import torch

from oracle import linear as ol
from oracle import nf4

GROUP_ELEMS = 64 * 256


def bits(t):
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def np_u8(t):
    return t.detach().to("cpu").numpy().copy()


def oracle_quantize_chunked(w_bits, chunk_groups=256):
    """oracle.nf4.quantize over a flat bf16 array, in group-aligned chunks."""
    w_bits = np.asarray(w_bits, dtype=np.uint16).reshape(-1)
    n = w_bits.size
    codes, c8, s2 = [], [], []
    step = GROUP_ELEMS * chunk_groups
    for lo in range(0, n, step):
        seg = w_bits[lo:lo + step]
        p, c, s = nf4.quantize(seg)
        codes.append(p)
        c8.append(c)
        s2.append(s)
    return np.concatenate(codes), np.concatenate(c8), np.concatenate(s2)


def oracle_dequant_full(w_bits, chunk_groups=256):
    """Oracle W' (bf16 bits, same shape) of a bf16 weight, chunked."""
    shape = w_bits.shape
    flat = np.asarray(w_bits, dtype=np.uint16).reshape(-1)
    out = np.empty_like(flat)
    step = GROUP_ELEMS * chunk_groups
    for lo in range(0, flat.size, step):
        seg = flat[lo:lo + step]
        p, c, s = nf4.quantize(seg)
        out[lo:lo + seg.size] = nf4.dequantize(p, c, s, seg.size)
    return out.reshape(shape)


def oracle_dequant_rows(w_bits2d, rows):
    """Oracle W' of selected rows only (each row's covering groups quantised)."""
    n_out, k_in = w_bits2d.shape
    flat = w_bits2d.reshape(-1)
    out = np.empty((len(rows), k_in), dtype=np.uint16)
    for i, r in enumerate(rows):
        lo = r * k_in
        hi = lo + k_in
        g0 = lo // GROUP_ELEMS * GROUP_ELEMS
        g1 = min(flat.size, -(-hi // GROUP_ELEMS) * GROUP_ELEMS)
        seg = flat[g0:g1]
        p, c, s = nf4.quantize(seg)
        d = nf4.dequantize(p, c, s, seg.size)
        out[i] = d[lo - g0:hi - g0]
    return out


rel = ol.rel_frobenius
