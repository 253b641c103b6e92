"""Pins of the plain-GPTQ oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a brute-force
loop, a closed form, a hand-derived fixture, an independent algorithm
(Babai's nearest plane on the QL factor of the regularised basis), or an exact
identity. The mutation tests at the end plant plausible mistakes in a copy of
the sweep and check that the pins catch them.
"""
import itertools

import numpy as np
import pytest

import oracle
from conftest import read_golden


def _rng(seed):
    return np.random.default_rng(seed)


def _layer(seed, m, n, k, decay=0.7, std=0.02):
    r = _rng(seed)
    Q, _ = np.linalg.qr(r.standard_normal((n, n)))
    s = np.arange(1, n + 1) ** (-decay)
    X = r.standard_normal((k, n)) @ (s[:, None] * Q)
    W = r.standard_normal((m, n)) * std
    return W, X


# ------------------------------------------------------------------------ Hessian, damping

def test_hessian_matches_triple_loop():
    r = _rng(1)
    X = r.standard_normal((7, 4))
    H = oracle.hessian(X, chunk=3)
    for i in range(4):
        for j in range(4):
            acc = 0.0
            for t in range(7):
                acc += X[t, i] * X[t, j]
            assert abs(H[i, j] - 2 * acc) < 1e-12


def test_damp_is_relative_to_mean_diagonal():
    H = np.array([[4.0, 1.0], [1.0, 2.0]])
    Hd, lam = oracle.damp(H, 0.5)
    assert lam == pytest.approx(1.5)
    assert np.allclose(Hd, [[5.5, 1.0], [1.0, 3.5]])


# ------------------------------------------------------------------------ factor

def test_inverse_cholesky_upper_properties():
    r = _rng(2)
    A = r.standard_normal((30, 20))
    H, _ = oracle.damp(2 * A.T @ A, 0.01)
    U = oracle.inverse_cholesky_upper(H)
    assert np.allclose(np.tril(U, -1), 0)
    assert np.all(np.diag(U) > 0)
    assert np.abs(U.T @ U @ H - np.eye(20)).max() < 1e-10
    # the rows of U are the feedback of the trailing problems: for every j the
    # trailing block of U factors the inverse of the trailing block of H
    for j in (0, 7, 19):
        T = U[j:, j:]
        assert np.abs(T.T @ T @ H[j:, j:] - np.eye(20 - j)).max() < 1e-10


def test_gram_schmidt_lengths_are_the_inverse_diagonal():
    """Lattice geometry paper, section 4: the Babai guarantee uses the Gram-Schmidt
    lengths L_jj of [X; mu I]; they equal 1 / (sqrt 2 U_jj)."""
    W, X = _layer(3, 4, 12, 40)
    H, lam = oracle.damp(oracle.hessian(X), 0.05)
    U = oracle.inverse_cholesky_upper(H)
    _, L = oracle.ql_decomposition(np.vstack([X, np.sqrt(lam / 2) * np.eye(12)]))
    assert np.allclose(np.diag(L), 1.0 / (np.sqrt(2.0) * np.diag(U)), rtol=1e-10)


# ------------------------------------------------------------------------ grid

def test_grid_golden_rows():
    for bits, ws, s, zr, z, codes in read_golden("grid_rules.txt"):
        bits = int(bits)
        w = np.array([float(x) for x in ws.split()])[None, :]
        maxq = (1 << bits) - 1
        gs_, gz, gzr = oracle.minmax_grid(w, maxq)
        assert gs_[0] == pytest.approx(float(s), rel=1e-12)
        assert gzr[0] == pytest.approx(float(zr), rel=1e-12, abs=1e-12)
        assert int(gz[0]) == int(z)
        # a group fed through the sweep with an identity factor has no feedback:
        # its codes are round-to-nearest on the group's own grid
        out = oracle.sweep(w, np.eye(w.shape[1]), bits, 0)
        assert out["codes"][0].tolist() == [int(c) for c in codes.split()]


# ------------------------------------------------------------------------ Babai equivalence

@pytest.mark.parametrize("seed,n,k,bits", [(10, 8, 40, 2), (11, 13, 64, 3), (12, 16, 9, 4),
                                           (13, 16, 100, 2), (14, 11, 30, 4)])
def test_babai_equivalence_per_channel(seed, n, k, bits):
    """GPTQ's decisions equal Babai's nearest plane in data space (lattice paper,
    sections 3.1-3.3), with the per-channel grid fixed from the original weights."""
    W, X = _layer(seed, 6, n, k)
    res = oracle.gptq_layer(W, X, bits=bits, group_size=0, lambda_rel=0.02)
    maxq = (1 << bits) - 1
    for i in range(W.shape[0]):
        s = np.full(n, res["scales"][i, 0])
        z = np.full(n, res["zeros"][i, 0])
        c, _, _ = oracle.babai_nearest_plane(X, res["lam"], W[i], s, z, maxq)
        assert np.array_equal(c, res["codes"][i])


@pytest.mark.parametrize("seed", [20, 21, 22])
def test_babai_equivalence_grouped(seed):
    """Same, with groups of 4 columns; the grid of each group is the one the sweep
    recorded (it depends on feedback-updated weights)."""
    n, bits = 16, 3
    W, X = _layer(seed, 5, n, 48)
    res = oracle.gptq_layer(W, X, bits=bits, group_size=4, lambda_rel=0.01)
    maxq = (1 << bits) - 1
    for i in range(W.shape[0]):
        s = np.repeat(res["scales"][i], 4)
        z = np.repeat(res["zeros"][i], 4)
        c, _, _ = oracle.babai_nearest_plane(X, res["lam"], W[i], s, z, maxq)
        assert np.array_equal(c, res["codes"][i])


# ------------------------------------------------------------------------ special cases

def test_round_to_nearest_when_gram_is_identity():
    """X with orthonormal columns: H is diagonal, no feedback flows, and GPTQ is
    round-to-nearest on the grid of the original weights."""
    r = _rng(30)
    n, m, bits = 24, 7, 3
    X, _ = np.linalg.qr(r.standard_normal((64, n)))
    W = r.standard_normal((m, n)) * 0.02
    res = oracle.gptq_layer(W, X, bits=bits, group_size=8, lambda_rel=0.01)
    maxq = (1 << bits) - 1
    for g in range(n // 8):
        seg = W[:, 8 * g:8 * g + 8]
        s, z, _ = oracle.minmax_grid(seg, maxq)
        rtn = np.clip(np.rint(seg / s[:, None] + z[:, None]), 0, maxq)
        assert np.array_equal(res["codes"][:, 8 * g:8 * g + 8], rtn)


@pytest.mark.parametrize("gs", [0, 32])
def test_blocking_invariance(gs):
    """GPTQ-2D, Theorem 1: any order that respects the feedback dependencies gives
    the same rounding; the lazy block update is such a re-association."""
    W, X = _layer(40, 9, 64, 200)
    H, _ = oracle.damp(oracle.hessian(X), 0.01)
    U = oracle.inverse_cholesky_upper(H)
    ref = oracle.sweep(W, U, 3, gs)
    for B in (1, 4, 32, 64):
        out = oracle.sweep_blocked(W, U, 3, gs, B)
        assert np.array_equal(out["codes"], ref["codes"])
        assert np.array_equal(out["zeros"], ref["zeros"])
        assert np.allclose(out["err"], ref["err"], rtol=1e-9, atol=1e-12)
        assert np.allclose(out["scales"], ref["scales"], rtol=1e-12)


def test_no_better_than_brute_force():
    """GPTQ-2D, section 5: the greedy sweep does not claim the closest lattice point
    (CVP is NP-hard); on tiny n its loss is never below the exhaustive optimum
    over the same grid, for the damped objective and for the data loss."""
    n, bits = 6, 2
    W, X = _layer(50, 5, n, 30)
    res = oracle.gptq_layer(W, X, bits=bits, group_size=0, lambda_rel=0.01)
    H, G = res["H"], X.T @ X
    grid = np.array(list(itertools.product(range(4), repeat=n)), dtype=np.float64)
    for i in range(W.shape[0]):
        s, z = res["scales"][i, 0], res["zeros"][i, 0]
        Dall = W[i][None, :] - s * (grid - z)
        reg = np.einsum("ij,jk,ik->i", Dall, H, Dall)
        dat = np.einsum("ij,jk,ik->i", Dall, G, Dall)
        d = W[i] - res["Wq"][i]
        assert d @ H @ d >= reg.min() - 1e-15
        assert d @ G @ d >= dat.min() - 1e-15
        # and the sweep's damped loss is a point of the grid's loss surface
        assert np.isclose(d @ H @ d, reg[np.argmin(np.abs(grid - res["codes"][i]).sum(1))])


def test_loss_identity():
    """The OBS increments of a quadratic add up exactly: per row
    sum_j e_j^2 = d^T H d, d = w - w_hat (Gram-Schmidt lengths 1/U_jj, lattice
    paper section 4)."""
    W, X = _layer(60, 8, 48, 120)
    res = oracle.gptq_layer(W, X, bits=3, group_size=16, lambda_rel=0.01)
    reg = oracle.regularised_loss_rows(W, res["Wq"], res["H"])
    assert np.allclose(res["loss_rows"], reg, rtol=1e-9)
    G = X.T @ X
    dat = oracle.data_loss_rows(W, res["Wq"], G)
    lam_term = res["lam"] * ((W - res["Wq"]) ** 2).sum(1)
    assert np.allclose(2 * dat + lam_term, reg, rtol=1e-9)


# ------------------------------------------------------------------------ replay

def test_replay_of_own_decisions_is_clean():
    W, X = _layer(70, 6, 32, 80)
    res = oracle.gptq_layer(W, X, bits=3, group_size=16, lambda_rel=0.01)
    rep = oracle.replay(W, res["U"], 3, 16, res["codes"], res["zeros"])
    assert rep["n_code_mismatch"] == 0 and rep["n_zero_mismatch"] == 0
    assert np.allclose(rep["loss_rows"], res["loss_rows"], rtol=1e-12)


def test_replay_flags_a_planted_wrong_decision():
    W, X = _layer(71, 6, 32, 80)
    res = oracle.gptq_layer(W, X, bits=3, group_size=16, lambda_rel=0.01)
    rep0 = oracle.replay(W, res["U"], 3, 16, res["codes"], res["zeros"])
    v = rep0["v"]
    frac = np.abs(v - np.rint(v))
    i, j = np.unravel_index(np.argmin(np.where((res["codes"] > 0) & (res["codes"] < 7), frac, 9)),
                            frac.shape)
    bad = res["codes"].copy()
    bad[i, j] += 1 if v[i, j] >= bad[i, j] else -1
    rep = oracle.replay(W, res["U"], 3, 16, bad, res["zeros"])
    assert rep["n_code_mismatch"] >= 1
    assert rep["code_dist"][0] == pytest.approx(0.5 - frac[i, j], abs=1e-9)


# ------------------------------------------------------------------------ mutations

def _mutant_sweep(W, U, bits, mutation):
    """A copy of the per-channel sweep with one plausible mistake planted."""
    Wc = np.array(W, dtype=np.float64)
    m, n = Wc.shape
    maxq = (1 << bits) - 1
    s, z, _ = oracle.minmax_grid(Wc, maxq)
    codes = np.zeros((m, n), dtype=np.int64)
    Uu = U.T if mutation == "transposed" else U
    for j in range(n):
        w = Wc[:, j].copy()
        c = np.clip(np.rint(w / s + z), 0, maxq)
        q = s * (c - z)
        e = (w - q) if mutation == "no_pivot" else (w - q) / Uu[j, j]
        sign = -1.0 if mutation == "sign" else 1.0
        if mutation == "off_by_one":
            Wc[:, j + 2:] -= sign * np.outer(e, Uu[j, j + 2:])
        else:
            Wc[:, j + 1:] -= sign * np.outer(e, Uu[j, j + 1:])
        codes[:, j] = c
    return codes


@pytest.mark.parametrize("mutation", ["sign", "transposed", "no_pivot", "off_by_one"])
def test_pins_catch_planted_mistakes(mutation):
    caught = False
    for seed in range(80, 86):
        W, X = _layer(seed, 6, 12, 40, decay=0.3)
        res = oracle.gptq_layer(W, X, bits=3, group_size=0, lambda_rel=0.02)
        mut = _mutant_sweep(W, res["U"], 3, mutation)
        for i in range(W.shape[0]):
            s = np.full(12, res["scales"][i, 0])
            z = np.full(12, res["zeros"][i, 0])
            c, _, _ = oracle.babai_nearest_plane(X, res["lam"], W[i], s, z, 7)
            if not np.array_equal(c, mut[i]):
                caught = True
    assert caught
