"""Pins for oracle.optim (AdamW with 8-bit states) against closed forms,
invariants and an unquantised fp64 AdamW.

What the pages fix is only that the optimizer is an 8-bit AdamW whose state
is paged; the update rule pinned here is the textbook AdamW, the 8-bit state
the pages' own blockwise FP8 scheme (see the oracle header for the readings).
"""

import numpy as np
import pytest

from oracle import numerics as nm
from oracle import optim

B1, B2 = 0.9, 0.999


def _params(n, seed, scale=0.01):
    rng = np.random.default_rng(seed)
    return nm.f32_to_bf16_bits((rng.standard_normal(n) * scale).astype(np.float32))


def _grads(n, seed, scale=1e-3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(n) * scale).astype(np.float32)


def test_first_step_moves_by_lr_times_sign():
    """Step 1 from a zero state: bias-corrected m = g and sqrt(v) = |g|, so
    each parameter moves by lr * g / (|g| + eps), about lr * sign(g)."""
    n, lr, eps = 1000, 1e-3, 1e-8
    p = _params(n, 0)
    g = _grads(n, 1)
    _, _, p1 = optim.adamw8_step(p, g, optim.init_state(n), lr, B1, B2, eps, 0.0, 1, return_f32=True)
    p0 = nm.bf16_bits_to_f32(p).astype(np.float64)
    g64 = g.astype(np.float64)
    np.testing.assert_allclose(p0 - p1.astype(np.float64), lr * g64 / (np.abs(g64) + eps), rtol=2e-5, atol=0)


def test_weight_decay_alone():
    """Zero gradient and state: the update is the decoupled decay
    p (1 - lr wd), and the state stays exactly zero."""
    n, lr, wd = 700, 1e-2, 0.1
    p = _params(n, 2)
    pb, st, p1 = optim.adamw8_step(p, np.zeros(n, np.float32), optim.init_state(n), lr, B1, B2, 1e-8, wd, 3,
                                   return_f32=True)
    p0 = nm.bf16_bits_to_f32(p).astype(np.float64)
    np.testing.assert_allclose(p1, p0 * (1 - lr * wd), rtol=1e-6, atol=0)
    assert not st[0].any() and not st[1].any() and not st[2].any() and not st[3].any()
    assert np.array_equal(pb, nm.f32_to_bf16_bits(p1))


def test_gradient_scale_invariance_without_eps():
    """With eps = 0, multiplying every gradient by 4 (a power of two) scales
    m by 4, v by 16 and sqrt(v) by 4 exactly, so parameters and state codes
    are identical and the state scales are 4x, step after step."""
    n = 3 * 256 + 77
    p = _params(n, 3)
    sa, sb = optim.init_state(n), optim.init_state(n)
    pa, pb = p, p
    for t in range(1, 4):
        g = _grads(n, 10 + t)
        pa, sa = optim.adamw8_step(pa, g, sa, 1e-3, B1, B2, 0.0, 0.0, t)
        pb, sb = optim.adamw8_step(pb, 4 * g, sb, 1e-3, B1, B2, 0.0, 0.0, t)
        assert np.array_equal(pa, pb)
        assert np.array_equal(sa[0], sb[0]) and np.array_equal(sa[1], sb[1])
        assert np.array_equal(4 * sa[2], sb[2]) and np.array_equal(4 * sa[3], sb[3])


def test_trajectory_matches_fp64_adamw():
    """Five steps against textbook AdamW in fp64 with unquantised states: the
    displacement agrees within the 8-bit state and bf16 parameter error
    (E4M3 keeps 3 mantissa bits: a few percent), far below what a wrong bias
    correction, moment or sign would give."""
    n, lr, wd = 4096, 1e-3, 0.01
    p = _params(n, 4)
    gs = [_grads(n, 20 + t) + np.float32(2e-4) for t in range(5)]
    st = optim.init_state(n)
    pq = p
    for t, g in enumerate(gs, start=1):
        pq, st = optim.adamw8_step(pq, g, st, lr, B1, B2, 1e-8, wd, t)
    p0 = nm.bf16_bits_to_f32(p).astype(np.float64)
    ref = optim.adamw_f64(p0, gs, lr, B1, B2, 1e-8, wd)
    got = nm.bf16_bits_to_f32(pq).astype(np.float64)
    err = np.linalg.norm((got - p0) - (ref - p0)) / np.linalg.norm(ref - p0)
    assert err < 0.08, err


def test_blocks_are_independent():
    """Each 256-element block (and the ragged tail) is updated exactly as if
    it were a tensor of its own."""
    n = 2 * 256 + 91
    p = _params(n, 5)
    g = _grads(n, 6)
    st = optim.init_state(n)
    p1, st1 = optim.adamw8_step(p, g, st, 1e-3, B1, B2, 1e-8, 0.01, 1)
    p2, st2 = optim.adamw8_step(p1, _grads(n, 7), st1, 1e-3, B1, B2, 1e-8, 0.01, 2)
    for b0 in range(0, n, 256):
        sl = slice(b0, min(n, b0 + 256))
        k = b0 // 256
        q1, s1 = optim.adamw8_step(p[sl], g[sl], optim.init_state(sl.stop - b0), 1e-3, B1, B2, 1e-8, 0.01, 1)
        q2, s2 = optim.adamw8_step(q1, _grads(n, 7)[sl], s1, 1e-3, B1, B2, 1e-8, 0.01, 2)
        assert np.array_equal(q2, p2[sl])
        assert np.array_equal(s2[0], st2[0][sl]) and np.array_equal(s2[1], st2[1][sl])
        assert s2[2][0] == st2[2][k] and s2[3][0] == st2[3][k]


def test_state_encoding_absmax_maps_to_448():
    """The block absmax of each moment is stored as the largest E4M3 code
    (448, sign kept) with scale RN(amax / 448); zero blocks store zeros."""
    n = 512
    x = np.zeros(n, np.float32)
    x[:256] = _grads(256, 8)
    codes, scale = optim.encode_state(x)
    i = int(np.argmax(np.abs(x[:256])))
    assert scale[0] == np.float32(np.float32(np.abs(x[i])) / np.float32(448.0))
    assert codes[i] == (0xFE if x[i] < 0 else 0x7E)
    assert scale[1] == 0 and not codes[256:].any()
    back = nm.e4m3_decode(codes[:256]).astype(np.float64) * float(scale[0])
    rel = np.abs(back - x[:256]) / np.abs(x[i])
    assert rel.max() <= 2.0 ** -4 + 1e-7   # within half a step of the 3-bit mantissa, or subnormal spacing


@pytest.mark.parametrize("step", [1, 2, 10, 1000])
def test_bias_corrections_closed_form(step):
    bc1, bc2 = optim.bias_corrections(B1, B2, step)
    b1, b2 = float(np.float32(B1)), float(np.float32(B2))
    assert bc1 == np.float32(1 / (1 - b1 ** step))
    assert abs(float(bc2) - 1 / np.sqrt(1 - b2 ** step)) <= 1e-7 / np.sqrt(1 - b2 ** step)
