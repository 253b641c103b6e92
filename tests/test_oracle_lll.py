"""Pins of the lattice-basis-reduction oracle (The Lattice Geometry of Neural Network
Quantization, section 5.2: LLL before GPTQ / Babai, "WITHREDUCTION").

LLL is pinned by what a reduced basis must satisfy, checked with Gram-Schmidt data computed
independently (a Cholesky factor of the reduced Gram matrix), by the unimodularity of T, by the
LLL bound on the first vector against brute-force shortest vectors, and by its action on an
orthogonal basis. The rounding in the reduced basis is pinned to a data-space nearest plane on
an explicit basis, to round-to-nearest for orthogonal data, to Babai's error bound and to the
brute-force optimum."""
import itertools

import numpy as np
import pytest

import oracle
from oracle.lll import gram_schmidt, lll_gram, reduce_for_gptq, round_in_basis, withreduction


def _basis(seed, k, n, decay=0.0):
    g = np.random.default_rng(seed)
    return g.standard_normal((k, n)) * (np.arange(1, n + 1) ** -decay)[None, :]


@pytest.mark.parametrize("seed,k,n,decay,tracked", [(0, 12, 6, 0.0, True), (1, 40, 24, 1.0, True),
                                                    (2, 80, 40, 0.7, True), (3, 30, 30, 1.0, True),
                                                    (3, 30, 30, 1.5, False)])
def test_lll_output_is_reduced_and_unimodular(seed, k, n, decay, tracked):
    """The last case has cond(G) ~ 5e13: the Gram matrix tracked through the operations drifts
    (2e-4), but the basis it returns is still reduced."""
    B = _basis(seed, k, n, decay)
    # a skewed basis of the same lattice, so that there is work to do
    g = np.random.default_rng(seed + 100)
    M = (np.eye(n) + np.triu(g.integers(-1, 2, (n, n)), 1)).astype(np.int64)
    G = (B @ M).T @ (B @ M)
    T, Gr, stats = lll_gram(G)
    assert np.array_equal(T, np.rint(T))
    assert abs(abs(np.linalg.det(T)) - 1.0) < 1e-6
    # the reduced basis itself, from exact integer products; the Gram matrix tracked through the
    # elementary operations drifts by their rounding (|T| reaches ~1e4 on these skewed bases)
    Bred = B @ (M @ T.astype(np.int64))
    Gx = Bred.T @ Bred
    if tracked:
        assert np.allclose(Gr, Gx, rtol=1e-6, atol=1e-6 * np.abs(Gx).max())
    mu, Bn = gram_schmidt(Gx)
    low = np.tril(mu, -1)
    assert np.abs(low).max() <= 0.5 + 1e-9
    for i in range(1, n):
        assert Bn[i] >= (0.75 - mu[i, i - 1] ** 2) * Bn[i - 1] * (1 - 1e-9)
    assert stats["swaps"] > 0


@pytest.mark.parametrize("seed,n", [(10, 2), (11, 3), (12, 3), (13, 4), (14, 4)])
def test_lll_first_vector_bound_against_brute_force(seed, n):
    """With delta = 3/4 the first reduced vector obeys |b_1|^2 <= 2^(n-1) lambda_1^2."""
    g = np.random.default_rng(seed)
    B = g.integers(-9, 10, (n, n)).astype(float)
    while abs(np.linalg.det(B)) < 1:
        B = g.integers(-9, 10, (n, n)).astype(float)
    G = B.T @ B
    T, Gr, _ = lll_gram(G)
    # shortest nonzero vector by enumeration over a box large enough for these bases
    best = np.inf
    K = 12
    for c in itertools.product(range(-K, K + 1), repeat=n):
        if any(c):
            v = B @ np.array(c, float)
            best = min(best, v @ v)
    assert Gr[0, 0] <= 2 ** (n - 1) * best * (1 + 1e-12)


def test_lll_on_a_diagonal_gram_only_permutes():
    d = np.array([1.0, 9.0, 2.0, 50.0, 3.0])
    T, Gr, _ = lll_gram(np.diag(d))
    assert np.array_equal(np.abs(T).sum(0), np.ones(5)) and np.array_equal(np.abs(T).sum(1), np.ones(5))
    assert np.allclose(Gr, np.diag(np.diag(Gr)))
    assert sorted(np.diag(Gr)) == sorted(d)


def test_reduce_for_gptq_reverses_the_order():
    B = _basis(5, 30, 16, 1.0)
    G = B.T @ B
    T, Gr, _ = reduce_for_gptq(G)
    P = np.arange(16)[::-1]
    Tr, Grr, _ = lll_gram(G[np.ix_(P, P)])
    assert np.array_equal(T, Tr[np.ix_(P, P)])
    Bred = B @ T
    assert np.allclose(Gr, Bred.T @ Bred, rtol=1e-8, atol=1e-8 * np.abs(Gr).max())


def test_round_in_basis_is_data_space_nearest_plane():
    """GPTQ without a grid under B^T B decides like Babai on B through its QL factor."""
    g = np.random.default_rng(6)
    B = _basis(6, 20, 8, 0.8)
    U = g.standard_normal((5, 8)) * 3
    C = round_in_basis(U, B.T @ B)
    Q, L = oracle.ql_decomposition(B)
    for r in range(5):
        y = Q.T @ (B @ U[r])
        c = np.zeros(8)
        for j in range(8):
            c[j] = np.rint((y[j] - L[j, :j] @ c[:j]) / L[j, j])
        assert np.array_equal(c, C[r])


def test_round_in_basis_replay_returns_the_same_trajectory():
    B = _basis(7, 20, 8, 0.5)
    U = np.random.default_rng(7).standard_normal((4, 8)) * 2
    C, V = round_in_basis(U, B.T @ B, record_v=True)
    C2, V2 = round_in_basis(U, B.T @ B, force=C)
    assert np.array_equal(C, C2) and np.allclose(V, V2)
    assert np.array_equal(np.rint(V), C)


def test_withreduction_on_orthogonal_data_is_round_to_nearest():
    g = np.random.default_rng(8)
    Q, _ = np.linalg.qr(g.standard_normal((64, 16)))
    X = 3.0 * Q                                   # X^T X = 9 I
    W = g.standard_normal((6, 16)) * 0.05
    for bits in (2, 4):
        res = withreduction(W, oracle.hessian(X), bits, 0.01)
        maxq = (1 << bits) - 1
        rtn = np.clip(np.rint(W / res["scales"][:, None] + res["zeros"][:, None]), 0, maxq)
        assert np.array_equal(res["codes"], rtn)
        assert res["n_clipped"] == 0


@pytest.mark.parametrize("seed", [20, 21, 22])
def test_withreduction_babai_bound_and_brute_force(seed):
    """Unclipped, the reduced-basis point meets Babai's bound |X'(u - c)|^2 <= sum Bn / 4 over the
    Gram-Schmidt lengths GPTQ sees in the reduced basis; clipped, its loss is never below the
    brute-force optimum of the row over the code box."""
    n, bits = 6, 2
    g = np.random.default_rng(seed)
    X = g.standard_normal((40, n)) @ (np.eye(n) + 0.8 * g.standard_normal((n, n)))
    W = g.standard_normal((4, n)) * 0.05
    H = oracle.hessian(X)
    res = withreduction(W, H, bits, 0.01)
    Gp = (H + res["lam"] * np.eye(n)) / 2
    _, Bn = gram_schmidt(res["G_red"][::-1, ::-1])
    maxq = (1 << bits) - 1
    for r in range(W.shape[0]):
        u = W[r] / res["scales"][r] + res["zeros"][r]
        d = u - res["codes_unclipped"][r]
        assert d @ Gp @ d <= Bn.sum() / 4 * (1 + 1e-9)
        s, z = res["scales"][r], res["zeros"][r]
        best = min((W[r] - s * (np.array(c) - z)) @ (2 * Gp) @ (W[r] - s * (np.array(c) - z))
                   for c in itertools.product(range(maxq + 1), repeat=n))
        assert res["loss_rows"][r] >= best * (1 - 1e-12)
