"""Pins for oracle.dq_centered (double quantisation with mean centring) and
the error ablation against the plain scheme."""

from fractions import Fraction

import numpy as np

import synth
from oracle import dq_centered as dqc
from oracle import nf4
from oracle import numerics as nm


def _constants(n_out, k_in, seed):
    w = synth.bf16_bits(synth.weight_bf16(n_out, k_in, seed=seed))
    return nf4.absmax_constants(w.reshape(-1), w.size)


def test_constant_constants_reconstruct_exactly():
    """All constants equal: the mean is that value, every centred constant is
    0, s2 = 0, and c_hat = mean = c exactly."""
    c = np.full(1000, np.float32(0.0371), dtype=np.float32)
    c8, s2, mean = dqc.double_quantize_centered(c)
    assert mean == c[0] and not c8.any() and not s2.any()
    assert np.array_equal(dqc.dequantized_constants_centered(c8, s2, mean), c)


def test_pairwise_sum_tree_shape():
    """Inputs on which the summation orders round differently fix the tree:
    neighbours first, then the pair sums, zero padding on the right.
    [1, 0, u, u] with u = 2^-53 (half an fp64 ulp of 1): the pairs give
    1 and 2u, and 1 + 2u is exact, while a running sum loses each u to the
    tie rule.  [1, u, u]: the pairs are (1 + u) -> 1 and (u + 0), and 1 + u
    ties to 1 again, while adding the last two first would keep 2u."""
    u = 2.0 ** -53
    assert dqc.pairwise_sum([1.0, 0.0, u, u]) == 1.0 + 2 * u
    assert dqc.pairwise_sum([1.0, u, u]) == 1.0
    assert dqc.pairwise_sum([u, u, 1.0]) == 1.0 + 2 * u
    # eight leaves: ((1 + 0) + (u + u)) + ((u + u) + (u + u)) = 1 + 2u + 4u
    assert dqc.pairwise_sum([1.0, 0.0] + [u] * 6) == 1.0 + 6 * u
    assert dqc.pairwise_sum([]) == 0.0 and dqc.pairwise_sum([3.5]) == 3.5


def test_pairwise_sum_error_bound():
    """Textbook bound for pairwise summation of n values:
    |S - sum| <= ceil(log2 n) * 2^-53 * sum|x| (to first order), against the
    exact sum (math.fsum), on sizes that are not powers of two."""
    import math
    rng = np.random.default_rng(9)
    for n in (3, 1000, 4097, 100003):
        x = rng.standard_normal(n) * rng.uniform(0.5, 2.0, n) * 10.0 ** rng.integers(-3, 4, n)
        exact = math.fsum(x)
        bound = math.ceil(math.log2(n)) * 2.0 ** -53 * float(np.sum(np.abs(x))) * 1.001
        assert abs(dqc.pairwise_sum(x) - exact) <= bound, n


def test_mean_is_the_exact_mean_within_one_rounding():
    """The pairwise fp64 sum of a few thousand fp32 constants is exact
    enough that the fp32 mean is the exact rational mean rounded once (or
    its neighbour when the exact mean lies within fp64 noise of a tie)."""
    c = _constants(64, 4096, 3)
    exact = sum(Fraction(float(x)) for x in c) / c.size
    got = dqc.constants_mean(c)
    lo = np.nextafter(got, np.float32(-np.inf))
    hi = np.nextafter(got, np.float32(np.inf))
    assert Fraction(float(lo)) < exact < Fraction(float(hi))


def test_reconstruction_within_e4m3_half_step():
    """|c_hat - c| <= (half an E4M3 step at the group's scale) plus the two
    fp32 roundings, group by group."""
    c = _constants(256, 4096, 4)
    c8, s2, mean = dqc.double_quantize_centered(c)
    ch = dqc.dequantized_constants_centered(c8, s2, mean).astype(np.float64)
    g = np.arange(c.size) // nf4.GROUP
    # E4M3 relative step is 2^-3 for normals; half of it, times the largest
    # magnitude 448 * s2 of the group, bounds the error of every member
    bound = 0.5 * 2.0 ** -3 * 448.0 * s2[g].astype(np.float64) + 2 * np.abs(ch) * 2.0 ** -24
    assert np.all(np.abs(ch - c.astype(np.float64)) <= bound)


def test_zero_mean_matches_plain_double_quantisation():
    """Forcing the mean to 0 gives the plain scheme's codes and scales."""
    c = _constants(128, 2048, 5)
    c8, s2, _ = dqc.double_quantize_centered(c, mean=0.0)
    p8, ps2 = nf4.double_quantize(c)
    assert np.array_equal(c8, p8) and np.array_equal(s2.view(np.uint32), ps2.view(np.uint32))


def test_centring_lowers_the_constant_error_on_normal_weights():
    """The ablation: on N(0, 0.02) weights the centred constants are closer
    to the exact ones than the plain FP8 constants (RMS relative error)."""
    c = _constants(1024, 4096, 6).astype(np.float64)
    p8, ps2 = nf4.double_quantize(c.astype(np.float32))
    plain = nf4.dequantized_constants(p8, ps2).astype(np.float64)
    c8, s2, mean = dqc.double_quantize_centered(c.astype(np.float32))
    cent = dqc.dequantized_constants_centered(c8, s2, mean).astype(np.float64)
    e_plain = np.sqrt(np.mean(((plain - c) / c) ** 2))
    e_cent = np.sqrt(np.mean(((cent - c) / c) ** 2))
    assert e_cent < e_plain


def test_full_centred_quantize_keeps_the_plain_codes():
    """Centring changes only the constants' encoding: the packed codes equal
    the plain scheme's, and c8 / s2 / mean are double_quantize_centered of
    the exact block constants."""
    w = synth.bf16_bits(synth.weight_bf16(64, 1024, seed=7)).reshape(-1)
    codes, c8, s2, mean = dqc.quantize_centered(w)
    pcodes, _, _ = nf4.quantize(w)
    assert np.array_equal(codes, pcodes)
    r8, rs2, rmean = dqc.double_quantize_centered(nf4.absmax_constants(w, w.size))
    assert np.array_equal(c8, r8) and np.array_equal(s2.view(np.uint32), rs2.view(np.uint32)) and mean == rmean


def test_centred_dequantize_reduces_to_plain_with_zero_mean():
    """With the mean forced to 0 the centred encoding is the plain one, and
    the centred dequantisation (c_hat = RN32(RN32(e4m3 * s2) + 0)) gives the
    plain dequantised weights bit for bit."""
    w = synth.bf16_bits(synth.weight_bf16(32, 2048, seed=8)).reshape(-1)
    pcodes, p8, ps2 = nf4.quantize(w)
    got = dqc.dequantize_centered(pcodes, p8, ps2, np.float32(0.0), w.size)
    assert np.array_equal(got, nf4.dequantize(pcodes, p8, ps2, w.size))


def test_centred_dequantize_closed_form_per_element():
    """Elementwise: w'[i] = bf16(RN32(q[code_i] * c_hat[block(i)])) with c_hat
    = RN32(RN32(e4m3(c8) * s2) + mean), written out with Python floats and the
    fp32 / bf16 roundings of oracle.numerics, on a few hundred elements."""
    w = synth.bf16_bits(synth.weight_bf16(4, 256, seed=9, outliers=True)).reshape(-1)
    codes, c8, s2, mean = dqc.quantize_centered(w)
    got = dqc.dequantize_centered(codes, c8, s2, mean, w.size)
    q = nf4.codebook()
    flat_codes = nf4.unpack_codes(codes, w.size)
    for i in range(0, w.size, 7):
        b = i // 64
        chat = np.float32(np.float32(nm.e4m3_decode(np.array([c8[b]], dtype=np.uint8))[0] * s2[b // 256]) + mean)
        want = nm.f32_to_bf16_bits(np.array([np.float32(q[flat_codes[i]] * chat)], dtype=np.float32))[0]
        assert got[i] == want, i
