"""Pins for oracle.dropout (LoRA dropout on the adapter input): the
counter-based generator against its published known-answer vectors, the
p = 0 special case against the plain linear, mask statistics, determinism,
and the backward against central finite differences."""

import json
import os

import numpy as np
import pytest

import synth
from oracle import dropout as dr
from oracle import linear as ol
from oracle import nf4
from oracle import numerics as nm

KAT = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")))


def test_philox_known_answer_vectors():
    for v in KAT["vectors"]:
        c = np.array([[int(x, 16) for x in v["counter"]]], dtype=np.uint64)
        k = np.array([[int(x, 16) for x in v["key"]]], dtype=np.uint64)
        got = dr.philox4x32_10(c, k)[0]
        assert [int(x) for x in got] == [int(x, 16) for x in v["output"]]


def _inputs(M=48, N=96, K=128, r=16, seed=0):
    d = synth.linear_inputs(synth.Linear("drop", N, K), M, r, seed)
    bits = {k: synth.bf16_bits(v) for k, v in d.items() if k in ("W", "X", "dY", "A", "B")}
    codes, c8, s2 = nf4.quantize(bits["W"].reshape(-1))
    bits["Wd"] = nf4.dequantize(codes, c8, s2, bits["W"].size).reshape(bits["W"].shape)
    return bits


def test_p_zero_is_the_plain_linear():
    b = _inputs()
    Xd, U, Y = dr.linear_fwd_dropout(b["X"], b["Wd"], b["A"], b["B"], 0.5, 0.0, 7)
    assert np.array_equal(Xd, b["X"])
    U0, Y0 = ol.linear_fwd(b["X"], b["Wd"], b["A"], b["B"], 0.5)
    assert np.array_equal(U, U0) and np.array_equal(Y, Y0)
    g = dr.linear_bwd_dropout(b["dY"], b["X"], b["Wd"], b["A"], b["B"], 0.5, 0.0, 7)
    g0 = ol.linear_bwd(b["dY"], b["X"], b["Wd"], b["A"], b["B"], 0.5)
    for a, c in zip(g, g0):
        assert np.array_equal(a, c)


@pytest.mark.parametrize("p", [0.05, 0.5])
def test_keep_fraction_is_binomial(p):
    M, K = 1024, 1024
    keep = dr.keep_mask(M, K, p, 12345)
    n = M * K
    sigma = np.sqrt(n * p * (1 - p))
    assert abs(keep.sum() - n * (1 - p)) < 6 * sigma
    # the four words of one generator call decide four different elements
    quads = keep.reshape(-1, 4)
    assert not np.all(quads == quads[:, :1])


def test_mask_is_deterministic_and_seed_dependent():
    a = dr.keep_mask(64, 256, 0.3, 1)
    assert np.array_equal(a, dr.keep_mask(64, 256, 0.3, 1))
    b = dr.keep_mask(64, 256, 0.3, 2)
    frac = np.mean(a != b)
    assert abs(frac - 2 * 0.3 * 0.7) < 0.05      # independent masks differ with probability 2p(1-p)
    c = dr.keep_mask(64, 256, 0.3, 1 + (1 << 32))  # the high key word matters too
    assert np.mean(a != c) > 0.3


def test_kept_values_are_scaled_and_dropped_are_zero():
    b = _inputs()
    Xd = dr.dropout_bits(b["X"], 0.5, 3)           # c = 2: scaling is exact
    keep = dr.keep_mask(*b["X"].shape, 0.5, 3)
    x = nm.bf16_bits_to_f32(b["X"]).astype(np.float64)
    xd = nm.bf16_bits_to_f32(Xd).astype(np.float64)
    assert np.array_equal(xd[keep], 2 * x[keep])
    assert np.all(Xd[~keep] == 0)


def test_backward_matches_finite_differences():
    """With the mask fixed, L = sum(Y * dY) with X_drop = keep * c * X (no
    rounding) has dL/dX = dX of the backward, and with the backward's own
    X_drop, dL/dA = dA and dL/dB = dB."""
    b = _inputs(M=12, N=20, K=64, r=16, seed=1)
    p, seed, s = 0.25, 9, 0.5
    keep = dr.keep_mask(12, 64, p, seed)
    c = float(dr.keep_scale(p))
    X, Wd, A, B, dY = (ol._f64(b[k]) for k in ("X", "Wd", "A", "B", "dY"))
    dX, dA, dB, _ = dr.linear_bwd_dropout(b["dY"], b["X"], b["Wd"], b["A"], b["B"], s, p, seed)
    Xd = ol._f64(dr.dropout_bits(b["X"], p, seed))

    def loss_x(Xv):
        return np.sum((Xv @ Wd.T + s * ((keep * c * Xv) @ A.T) @ B.T) * dY)

    def loss_ab(Av, Bv):
        return np.sum((X @ Wd.T + s * (Xd @ Av.T) @ Bv.T) * dY)

    h = 1e-3
    rng = np.random.default_rng(0)
    for _ in range(8):
        i, j = rng.integers(12), rng.integers(64)
        E = np.zeros_like(X); E[i, j] = h
        assert abs((loss_x(X + E) - loss_x(X - E)) / (2 * h) - dX[i, j]) <= 1e-6 * (1 + abs(dX[i, j]))
        a, k = rng.integers(16), rng.integers(64)
        E = np.zeros_like(A); E[a, k] = h
        assert abs((loss_ab(A + E, B) - loss_ab(A - E, B)) / (2 * h) - dA[a, k]) <= 1e-6 * (1 + abs(dA[a, k]))
        n, q = rng.integers(20), rng.integers(16)
        E = np.zeros_like(B); E[n, q] = h
        assert abs((loss_ab(A, B + E) - loss_ab(A, B - E)) / (2 * h) - dB[n, q]) <= 1e-6 * (1 + abs(dB[n, q]))
