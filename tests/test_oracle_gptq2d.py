"""Pins of the two-sided rounding oracle (GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding)."""
import numpy as np
import pytest

import oracle


def _problem(seed, m, n, cond=30.0, scale=3.0):
    g = np.random.default_rng(seed)
    def basis(k):
        Q1, _ = np.linalg.qr(g.standard_normal((k, k)))
        Q2, _ = np.linalg.qr(g.standard_normal((k, k)))
        return Q1 @ np.diag(np.exp(np.linspace(0, np.log(cond), k))) @ Q2
    A, B = basis(m), basis(n)
    X = g.standard_normal((m, n)) * scale
    return X, A, B, A.T @ A, B @ B.T


def _babai(M, t):
    """Textbook nearest plane for the lattice M Z^N (no clipping): M = Q L (L lower), decide
    coordinate k from row k of L, which involves coordinates 0..k only."""
    Q, L = oracle.ql_decomposition(M)
    y = Q.T @ t
    c = np.zeros(M.shape[1])
    for k in range(len(c)):
        c[k] = np.rint((y[k] - L[k, :k] @ c[:k]) / L[k, k])
    return c.astype(np.int64)


@pytest.mark.parametrize("m,n,seed", [(3, 5, 1), (6, 4, 2), (5, 5, 3), (1, 7, 4), (8, 2, 5)])
def test_antidiagonal_sweep_equals_the_vectorised_sweep(m, n, seed):
    X, A, B, G, H = _problem(seed, m, n)
    Zv = oracle.gptq2d_vectorized(X, G, H)
    Za = oracle.gptq2d_antidiagonal(X, G, H)["Z"]
    assert np.array_equal(Zv, Za)


@pytest.mark.parametrize("m,n,seed", [(3, 4, 6), (5, 3, 7), (4, 4, 8)])
def test_vectorised_sweep_is_babai_on_the_kronecker_basis(m, n, seed):
    X, A, B, G, H = _problem(seed, m, n)
    M = np.kron(B.T, A)                       # vec(A D B) = (B^T (x) A) vec(D)
    x = X.reshape(-1, order="F")
    zb = _babai(M, M @ x).reshape(m, n, order="F")
    assert np.array_equal(zb, oracle.gptq2d_vectorized(X, G, H))


def test_right_identity_is_the_one_sided_sweep_of_each_column():
    X, A, B, G, H = _problem(9, 6, 5)
    Z = oracle.gptq2d_antidiagonal(X, G, np.eye(5))["Z"]
    UG = oracle.inverse_cholesky_upper(G)
    for j in range(5):
        assert np.array_equal(Z[:, j], oracle.adaptive_round_1d(X[:, j], UG))


def test_loss_identity_and_rounding_to_nearest_under_orthogonal_bases():
    """With orthogonal A and B every coordinate is independent: plain rounding to nearest."""
    g = np.random.default_rng(10)
    A, _ = np.linalg.qr(g.standard_normal((4, 4)))
    B, _ = np.linalg.qr(g.standard_normal((6, 6)))
    X = g.standard_normal((4, 6)) * 5
    Z = oracle.gptq2d_antidiagonal(X, A.T @ A, B @ B.T)["Z"]
    assert np.array_equal(Z, np.rint(X).astype(np.int64))
    assert oracle.two_sided_loss(X, Z, A, B) == pytest.approx(((Z - X) ** 2).sum(), rel=1e-10)


def test_planted_mistakes_are_caught():
    """Pushing a column buffer along its row before the entry's own error is in it, or
    exchanging the left and right Gram matrices, changes the decisions."""
    X, A, B, G, H = _problem(11, 5, 5, cond=100.0)
    good = oracle.gptq2d_vectorized(X, G, H)
    assert not np.array_equal(oracle.gptq2d_vectorized(X, H, G), good)
    m, n = X.shape
    UG, UH = oracle.inverse_cholesky_upper(G), oracle.inverse_cholesky_upper(H)
    C = np.zeros((m, n))
    V = np.zeros((m, n))
    Z = np.zeros((m, n), dtype=np.int64)
    for s_ in range(m + n - 1):
        for p in range(max(0, s_ - n + 1), min(m - 1, s_) + 1):
            q = s_ - p
            v = X[p, q] - V[p, q] - C[p, q] * UH[q, q]
            z = np.rint(v)
            e = (v - z) / (UG[p, p] * UH[q, q])
            Z[p, q] = int(z)
            V[p, q + 1:] += C[p, q] * UH[q, q + 1:]      # planted: row push before own error
            C[p:, q] += UG[p, p:] * e
    assert not np.array_equal(Z, good)


@pytest.mark.parametrize("k,seed", [(1, 20), (6, 21), (40, 22)])
def test_reverse_cholesky_factor(k, seed):
    """R upper with M = R R^T, and R is the inverse of the upper factor of M^-1."""
    g = np.random.default_rng(seed)
    A = g.standard_normal((k, k)) + 2 * np.eye(k)
    M = A @ A.T
    R = oracle.reverse_cholesky_upper(M)
    assert np.allclose(np.tril(R, -1), 0) and np.all(np.diag(R) > 0)
    assert np.allclose(R @ R.T, M, rtol=1e-12, atol=1e-12 * np.abs(M).max())
    U = oracle.inverse_cholesky_upper(M)
    assert np.allclose(R @ U, np.eye(k), atol=1e-9)


@pytest.mark.parametrize("m,n,seed", [(7, 11, 23), (12, 5, 24), (1, 9, 25)])
def test_closed_form_residuals_match_the_sweep(m, n, seed):
    """X - Z = U_G^T E U_H: the residuals computed from Z alone equal the sweep's own v - z,
    lie in [-1/2, 1/2], and moving any single entry of Z by one step leaves that box."""
    X, A, B, G, H = _problem(seed, m, n)
    out = oracle.gptq2d_antidiagonal(X, G, H)
    c = oracle.gptq2d_residuals(X, out["Z"], G, H)
    assert np.allclose(c, out["v"] - out["Z"], atol=1e-9)
    assert np.abs(c).max() <= 0.5 + 1e-12
    g = np.random.default_rng(seed)
    for _ in range(5):
        Z2 = out["Z"].copy()
        p, q = g.integers(m), g.integers(n)
        Z2[p, q] += g.choice([-1, 1])
        assert np.abs(oracle.gptq2d_residuals(X, Z2, G, H)).max() > 0.5
