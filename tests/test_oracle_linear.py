"""Pins for oracle.linear: brute force, identities, special cases, finite differences."""

import math

import numpy as np

from oracle import linear as ol


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _loops_fwd_bwd(X, W, A, B, dY, s):
    """Pure-Python sums (math.fsum), independent of numpy's matmul."""
    M, K = len(X), len(X[0])
    N, r = len(B), len(B[0])
    U = [[math.fsum(X[m][k] * A[j][k] for k in range(K)) for j in range(r)] for m in range(M)]
    Y = [[math.fsum([math.fsum(X[m][k] * W[n][k] for k in range(K)),
                     s * math.fsum(U[m][j] * B[n][j] for j in range(r))]) for n in range(N)]
         for m in range(M)]
    dU = [[s * math.fsum(dY[m][n] * B[n][j] for n in range(N)) for j in range(r)] for m in range(M)]
    dX = [[math.fsum([math.fsum(dY[m][n] * W[n][k] for n in range(N)),
                      math.fsum(dU[m][j] * A[j][k] for j in range(r))]) for k in range(K)]
          for m in range(M)]
    dA = [[math.fsum(dU[m][j] * X[m][k] for m in range(M)) for k in range(K)] for j in range(r)]
    dB = [[s * math.fsum(dY[m][n] * U[m][j] for m in range(M)) for j in range(r)] for n in range(N)]
    return [np.array(a) for a in (U, Y, dX, dA, dB, dU)]


def test_brute_force_tiny():
    rng = np.random.default_rng(0)
    M, N, K, r, s = 3, 5, 7, 2, 0.75
    X, W, A, B, dY = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r), _rand(rng, M, N)
    U, Y = ol.linear_fwd(X, W, A, B, s)
    dX, dA, dB, dU = ol.linear_bwd(dY, X, W, A, B, s)
    ref = _loops_fwd_bwd(X.tolist(), W.tolist(), A.tolist(), B.tolist(), dY.tolist(), s)
    for got, exp in zip((U, Y, dX, dA, dB, dU), ref):
        assert np.allclose(got, exp, rtol=1e-12, atol=1e-12)


def test_merged_weight_identity():
    rng = np.random.default_rng(1)
    M, N, K, r, s = 9, 6, 8, 3, 0.25
    X, W, A, B = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r)
    _, Y = ol.linear_fwd(X, W, A, B, s)
    assert np.allclose(Y, X @ (W + s * B @ A).T, rtol=1e-12, atol=1e-12)


def test_special_cases_w_zero_and_b_zero():
    rng = np.random.default_rng(2)
    M, N, K, r, s = 4, 6, 8, 2, 2.0
    X, W, A, B, dY = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r), _rand(rng, M, N)
    U, Y = ol.linear_fwd(X, np.zeros((N, K)), A, B, s)
    assert np.allclose(Y, s * (X @ A.T) @ B.T)
    _, Y0 = ol.linear_fwd(X, W, A, np.zeros((N, r)), s)
    assert np.allclose(Y0, X @ W.T)
    dX, dA, dB, _ = ol.linear_bwd(dY, X, W, A, np.zeros((N, r)), s)
    assert np.allclose(dX, dY @ W) and np.all(dA == 0)
    assert np.allclose(dB, s * dY.T @ (X @ A.T))


def test_gradients_by_finite_differences():
    """dX, dA, dB are the gradients of L = sum(Y * dY) (L is linear in each)."""
    rng = np.random.default_rng(3)
    M, N, K, r, s = 3, 4, 5, 2, 0.5
    X, W, A, B, dY = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r), _rand(rng, M, N)

    def loss(X_, A_, B_):
        return float(np.sum(ol.linear_fwd(X_, W, A_, B_, s)[1] * dY))

    dX, dA, dB, _ = ol.linear_bwd(dY, X, W, A, B, s)
    h = 1e-3
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(P)
        for idx in np.ndindex(P.shape):
            Pp, Pm = P.copy(), P.copy()
            Pp[idx] += h
            Pm[idx] -= h
            args_p = {"X": X, "A": A, "B": B}
            args_m = dict(args_p)
            args_p[name], args_m[name] = Pp, Pm
            num[idx] = (loss(args_p["X"], args_p["A"], args_p["B"]) -
                        loss(args_m["X"], args_m["A"], args_m["B"])) / (2 * h)
        assert np.allclose(num, G, rtol=1e-7, atol=1e-9), name


def test_rel_frobenius():
    a = np.ones((3, 3))
    assert ol.rel_frobenius(a, a) == 0.0
    assert abs(ol.rel_frobenius(a * 1.001, a) - 1e-3) < 1e-12
    assert ol.rel_frobenius(np.zeros(2), np.zeros(2)) == 0.0


def test_group_of_one_is_the_linear():
    rng = np.random.default_rng(4)
    M, N, K, r, s = 3, 4, 5, 2, 0.5
    X, W, A, B, dY = _rand(rng, M, K), _rand(rng, N, K), _rand(rng, r, K), _rand(rng, N, r), _rand(rng, M, N)
    U1, Y1 = ol.linear_fwd(X, W, A, B, s)
    Ug, Yg = ol.group_fwd(X, W, A, B, s, [N])
    assert np.array_equal(U1, Ug) and np.array_equal(Y1, Yg)
    dX1, dA1, dB1, _ = ol.linear_bwd(dY, X, W, A, B, s)
    dXg, dAg, dBg = ol.group_bwd(dY, X, W, A, B, s, [N])
    assert np.array_equal(dX1, dXg) and np.array_equal(dA1, dAg) and np.array_equal(dB1, dBg)


def test_group_gradients_by_finite_differences():
    """Three members of different widths sharing X: dX (the sum over members),
    the stacked dA and dB are the gradients of L = sum(Y * dY), Y the members'
    outputs side by side; the brute-force loops pin each member's forward."""
    rng = np.random.default_rng(5)
    M, K, r, s = 3, 5, 2, 0.5
    nm = [2, 3, 1]
    N = sum(nm)
    X, W, A, B, dY = (_rand(rng, M, K), _rand(rng, N, K), _rand(rng, 3 * r, K), _rand(rng, N, r),
                      _rand(rng, M, N))
    U, Y = ol.group_fwd(X, W, A, B, s, nm)
    off = [0, 2, 5, 6]
    for g in range(3):
        ref = _loops_fwd_bwd(X.tolist(), W[off[g]:off[g + 1]].tolist(), A[g * r:(g + 1) * r].tolist(),
                             B[off[g]:off[g + 1]].tolist(), dY[:, off[g]:off[g + 1]].tolist(), s)
        assert np.allclose(U[:, g * r:(g + 1) * r], ref[0], rtol=1e-12, atol=1e-12)
        assert np.allclose(Y[:, off[g]:off[g + 1]], ref[1], rtol=1e-12, atol=1e-12)

    def loss(X_, A_, B_):
        return float(np.sum(ol.group_fwd(X_, W, A_, B_, s, nm)[1] * dY))

    dX, dA, dB = ol.group_bwd(dY, X, W, A, B, s, nm)
    h = 1e-3
    for name, P, G in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(P)
        for idx in np.ndindex(P.shape):
            Pp, Pm = P.copy(), P.copy()
            Pp[idx] += h
            Pm[idx] -= h
            args_p = {"X": X, "A": A, "B": B}
            args_m = dict(args_p)
            args_p[name], args_m[name] = Pp, Pm
            num[idx] = (loss(args_p["X"], args_p["A"], args_p["B"]) -
                        loss(args_m["X"], args_m["A"], args_m["B"])) / (2 * h)
        assert np.allclose(num, G, rtol=1e-7, atol=1e-9), name
