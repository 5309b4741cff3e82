"""Pins for oracle.nf4 against what the pages and mathematics fix.

Facts used (see the oracle headers for the page citations): 16 levels from
standard-normal quantiles, normalised to [-1, 1], asymmetric with an exact
zero so zero padding quantises without error; blocks of 64 with one absmax
constant; constants double-quantised to FP8 in groups of 256; the printed
bit costs 0.5 / 0.127 / 0.373 bit/param and about 3 GB at 65B.
"""

import json
import os

import numpy as np
import pytest
import scipy.special

import synth
from oracle import nf4
from oracle import numerics as nm

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


# ----------------------------------------------------------------- codebook

def test_codebook_invariants():
    q = nf4.codebook()
    assert q.dtype == np.float32 and q.size == GOLD["nf4_levels"]
    assert np.all(np.diff(q) > 0)                      # distinct, ascending
    assert q[0] == -1.0 and q[15] == 1.0               # normalised to [-1, 1]
    assert q[7] == 0.0 and not np.signbit(q[7])        # exact zero
    assert np.sum(q < 0) == 7 and np.sum(q > 0) == 8   # asymmetric
    assert np.all(np.abs(q) <= 1.0)


def test_codebook_levels_are_normal_quantiles():
    """Forward-CDF check: Phi(q_i * z) hits evenly spaced probabilities.

    z = Phi^-1(DELTA) from scipy (a different inverse than the oracle's), and
    Phi from scipy.special.ndtr.  Positive levels sit at 8 probabilities
    evenly spaced from 1/2 to DELTA, negative ones at 7 probabilities evenly
    spaced from 1/2 to 1 - DELTA.
    """
    q = nf4.codebook().astype(np.float64)
    z = scipy.special.ndtri(nf4.DELTA)
    p = scipy.special.ndtr(q * z)
    step_pos = (nf4.DELTA - 0.5) / 8
    step_neg = (nf4.DELTA - 0.5) / 7
    expect_pos = 0.5 + step_pos * np.arange(1, 9)
    expect_neg = 0.5 - step_neg * np.arange(7, 0, -1)
    assert np.allclose(p[8:], expect_pos, rtol=0, atol=2e-7)
    assert np.allclose(p[:7], expect_neg, rtol=0, atol=2e-7)
    assert p[7] == 0.5


def test_codebook_bins_roughly_equal_occupancy():
    """Diagnostic for "each bin gets the same expected count" (soft bound).

    The midpoint decision rule on absmax-normalised Gaussian blocks gives
    bins of similar, not identical, mass; every code must be used and none
    may dominate.
    """
    w = synth.random_bf16_bits((4096, 64), seed=7, std=0.02).reshape(-1)
    packed, _, _ = nf4.quantize(w)
    codes = nf4.unpack_codes(packed, w.size)
    frac = np.bincount(codes, minlength=16) / codes.size
    assert frac.min() > 0.01 and frac.max() < 0.15


def test_midpoints_between_levels():
    q = nf4.codebook()
    m = nf4.midpoints()
    assert m.size == 15
    assert np.all((q[:-1] < m) & (m < q[1:]))
    exact = (q[:-1].astype(np.float64) + q[1:].astype(np.float64)) / 2
    assert np.all(np.abs(m.astype(np.float64) - exact) <= np.abs(np.spacing(m.astype(np.float32))) / 2)


# --------------------------------------------------------- nearest level

def _bf16_values_up_to(c_bits):
    allb = np.arange(2**16, dtype=np.uint32).astype(np.uint16)
    v = nm.bf16_bits_to_f32(allb)
    c = nm.bf16_bits_to_f32(np.uint16(c_bits))
    keep = np.isfinite(v) & (np.abs(v) <= c)
    return allb[keep], float(c)


@pytest.mark.parametrize("c_bits", [0x3F80, 0x3CA4, 0x4049, 0x0F81, 0x7F00])
def test_nearest_level_brute_force(c_bits):
    """Codes equal argmin_i |w/c - q_i| (fp64) away from the midpoints."""
    vals, c = _bf16_values_up_to(c_bits)
    n = vals.size
    per = 63
    nb = -(-n // per)
    blocks = np.full((nb, 64), np.uint16(c_bits), dtype=np.uint16)  # element 0 = c
    flat = np.zeros(nb * per, dtype=np.uint16)
    flat[:n] = vals
    blocks[:, 1:] = flat.reshape(nb, per)
    w = blocks.reshape(-1)
    packed, _, _ = nf4.quantize(w)
    codes = nf4.unpack_codes(packed, w.size).reshape(nb, 64)[:, 1:].reshape(-1)[:n]
    x = nm.bf16_bits_to_f32(vals).astype(np.float64) / c
    q = nf4.codebook().astype(np.float64)
    best = np.argmin(np.abs(x[:, None] - q[None, :]), axis=1)
    m = nf4.midpoints().astype(np.float64)
    near_mid = np.min(np.abs(x[:, None] - m[None, :]), axis=1) <= 4 * 2.0**-24
    assert np.array_equal(codes[~near_mid], best[~near_mid])
    assert near_mid.sum() < 0.01 * n


def test_absmax_element_maps_to_an_end_code():
    w = synth.random_bf16_bits((512, 64), seed=3, std=0.02)
    packed, _, _ = nf4.quantize(w.reshape(-1))
    codes = nf4.unpack_codes(packed, w.size).reshape(512, 64)
    v = nm.bf16_bits_to_f32(w)
    idx = np.argmax(np.abs(v), axis=1)
    end = codes[np.arange(512), idx]
    sign = np.signbit(v[np.arange(512), idx])
    assert np.all(np.where(sign, end == 0, end == 15))


def test_midpoint_tie_goes_to_lower_code():
    """A value exactly on a midpoint takes the lower code; one ulp above, the upper."""
    m = nf4.midpoints()
    assert np.array_equal(nf4.nearest_code(m), np.arange(15))
    up = np.nextafter(m, np.float32(np.inf))
    assert np.array_equal(nf4.nearest_code(up), np.arange(1, 16))
    assert nf4.nearest_code(np.float32(-0.0)) == 7
    assert nf4.nearest_code(np.float32(-1.0)) == 0 and nf4.nearest_code(np.float32(1.0)) == 15


# ------------------------------------------------ zero, padding, round trip

def test_zero_block_and_padding_are_exact():
    w = np.zeros(64 * 3 + 10, dtype=np.uint16)
    w[64:128] = synth.random_bf16_bits((64,), seed=1)
    w[64 * 3:] = synth.random_bf16_bits((10,), seed=2)
    packed, c8, s2 = nf4.quantize(w)
    codes = nf4.unpack_codes(packed, 64 * 4)
    assert np.all(codes[:64] == 7)              # all-zero block
    assert np.all(codes[64 * 3 + 10:] == 7)     # zero padding of the tail block
    assert c8[0] == 0
    d = nf4.dequantize(packed, c8, s2, w.size)
    assert np.all(d[:64] == 0x0000)             # exactly +0
    negz = np.full(64, 0x8000, dtype=np.uint16)
    p2, c82, s22 = nf4.quantize(negz)
    assert np.all(nf4.unpack_codes(p2, 64) == 7)
    assert np.all(nf4.dequantize(p2, c82, s22, 64) == 0x0000)


def test_tiny_block_constant():
    """A block whose absmax is so small that 1/c overflows still codes zero as 7."""
    w = np.zeros(64, dtype=np.uint16)
    w[0] = 0x0001                    # smallest positive bf16 subnormal: 1/c = inf
    w[1] = 0x8001                    # its negative
    packed, c8, s2 = nf4.quantize(w)
    codes = nf4.unpack_codes(packed, 64)
    assert codes[0] == 15 and codes[1] == 0 and np.all(codes[2:] == 7)


def test_codebook_values_round_trip():
    q = nf4.codebook()
    qb = nm.f32_to_bf16_bits(q)
    w = np.tile(qb, 4)  # block absmax = 1 exactly
    packed, c8, s2 = nf4.quantize(w)
    assert np.array_equal(nf4.unpack_codes(packed, 64), np.tile(np.arange(16), 4))
    chat = nf4.dequantized_constants(c8, s2)
    assert chat[0] == np.float32(1.0)
    assert np.array_equal(nf4.dequantize(packed, c8, s2, 64), w)


def test_codes_are_idempotent():
    for seed, outl in ((11, False), (12, True)):
        w = synth.bf16_bits(synth.weight_bf16(256, 512, seed, outliers=outl)).reshape(-1)
        p1, c81, s21 = nf4.quantize(w)
        d = nf4.dequantize(p1, c81, s21, w.size)
        p2, _, _ = nf4.quantize(d)
        assert np.array_equal(p1, p2)


def test_block_locality():
    w = synth.bf16_bits(synth.weight_bf16(64, 64 * 512, 5)).reshape(-1)  # 512 blocks, 2 groups
    p1, c81, s21 = nf4.quantize(w)
    w2 = w.copy()
    j = 64 * 300 + 17                    # block 300, group 1
    w2[j] = nm.f32_to_bf16_bits(np.float32([0.5]))[0]
    p2, c82, s22 = nf4.quantize(w2)
    changed = np.nonzero(p1 != p2)[0]
    assert changed.size > 0 and np.all((changed >= 300 * 32) & (changed < 301 * 32))
    assert np.array_equal(c81[:256], c82[:256]) and s21[0] == s22[0]
    assert s21[1] != s22[1]


# --------------------------------------------------------- double quant

def test_double_quant_group_max_is_fp8_max():
    w = synth.bf16_bits(synth.weight_bf16(128, 64 * 256, 9)).reshape(-1)
    c = nf4.absmax_constants(w, w.size)
    c8, s2 = nf4.double_quantize(c)
    for g in range(s2.size):
        seg = c[g * 256:(g + 1) * 256]
        assert c8[g * 256 + int(np.argmax(seg))] == 0x7E
        assert s2[g] == np.float32(seg.max()) / np.float32(448.0)


def test_dequantized_constant_within_fp8_precision():
    w = synth.bf16_bits(synth.weight_bf16(256, 64 * 256, 4, outliers=True)).reshape(-1)
    c = nf4.absmax_constants(w, w.size)
    c8, s2 = nf4.double_quantize(c)
    chat = nf4.dequantized_constants(c8, s2).astype(np.float64)
    g = np.arange(c.size) // 256
    normal = c / s2[g] >= 2.0**-6
    rel = np.abs(chat - c) / c
    assert np.all(rel[normal] <= 2.0**-4 * (1 + 1e-6))


# ------------------------------------------------------- page figures

def test_bit_costs_match_the_page():
    fp32_cost = nf4.bits_per_param(const_bits=32, scale_bits=0)
    dq_cost = nf4.bits_per_param()
    assert fp32_cost == GOLD["fp32_const_bits_per_param_block64"]
    assert round(dq_cost, 3) == GOLD["fp8_dq_const_bits_per_param"]
    assert round(fp32_cost - dq_cost, 3) == GOLD["saved_bits_per_param"]
    saved_gb = (fp32_cost - dq_cost) * GOLD["params_65b"] / 8 / 1e9
    assert round(saved_gb) == GOLD["saved_gb_at_65b"]


def test_storage_bytes_match_format():
    n, k = 256, 64 * 256 * 3
    w = synth.bf16_bits(synth.weight_bf16(n, k, 1)).reshape(-1)
    packed, c8, s2 = nf4.quantize(w)
    bits = 8 * (packed.nbytes + c8.nbytes + s2.nbytes) / w.size
    assert bits == 4 + nf4.bits_per_param()
    nf4_gb = GOLD["params_70b"] * 4 / 8 / 1e9          # codes alone
    assert nf4_gb == GOLD["nf4_gb_70b"]
    assert GOLD["params_70b"] * 2 / 1e9 == GOLD["fp16_gb_70b"]
