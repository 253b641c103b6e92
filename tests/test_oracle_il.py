"""Pins of the intrinsic-LoRA oracle (GPTQ-intrinsic LoRA summary, "Method" parts 2-3)."""
import numpy as np
import pytest

import oracle


def _lowrank_layer(seed, m, n, k, r, snr=30.0):
    g = np.random.default_rng(seed)
    P, _ = np.linalg.qr(g.standard_normal((n, r)))
    a = np.sqrt(snr * n / np.arange(1, r + 1) / (1.0 / np.arange(1, r + 1)).sum())
    X = (g.standard_normal((k, r)) * a) @ P.T + g.standard_normal((k, n))
    W = g.standard_normal((m, n)) * 0.02
    return W, X


def test_top_singular_directions_are_the_svd_of_X():
    W, X = _lowrank_layer(1, 3, 20, 200, 4)
    V, sig2 = oracle.top_singular_directions(X.T @ X, 4)
    _, sv, Vt = np.linalg.svd(X, full_matrices=False)
    assert np.allclose(sig2, sv[:4] ** 2, rtol=1e-10)
    for c in range(4):
        v = Vt[c] * np.sign(Vt[c][np.argmax(np.abs(Vt[c]))])
        assert np.allclose(V[:, c], v, atol=1e-10)


def test_r0_equals_plain_gptq():
    g = np.random.default_rng(2)
    X = g.standard_normal((100, 32)) @ g.standard_normal((32, 32))
    W = g.standard_normal((6, 32)) * 0.02
    plain = oracle.gptq_layer(W, X, bits=3, group_size=8, lambda_rel=0.01)
    il = oracle.il_layer(W, X, r=0, bits=3, group_size=8, lambda_rel=0.01)
    assert il["lam"] == pytest.approx(plain["lam"], rel=1e-14)
    assert np.allclose(il["Ut"], plain["U"], rtol=1e-9, atol=1e-12)
    assert np.array_equal(il["codes"], plain["codes"])
    assert np.array_equal(il["zeros"], plain["zeros"])
    assert np.allclose(il["err"], plain["err"], rtol=1e-8, atol=1e-13)
    assert il["R"].shape == (0, 6)


@pytest.mark.parametrize("seed,r", [(3, 2), (4, 5)])
def test_literal_eig_qr_factor_equals_schur_route(seed, r):
    W, X = _lowrank_layer(seed, 4, 24, 300, r)
    H_raw = oracle.hessian(X)
    V, _ = oracle.top_singular_directions(H_raw / 2, r)
    Ht, lam = oracle.il_hessian(H_raw / 2, V, 1e-3)
    Ut = oracle.eig_qr_factor(Ht)
    assert np.allclose(np.tril(Ut, -1), 0, atol=1e-12)
    assert np.abs(Ut.T @ Ut @ Ht - np.eye(24 + r)).max() < 1e-8
    rows = oracle.schur_factor_rows(H_raw, V, lam)
    assert np.allclose(Ut[:24], rows, rtol=1e-7, atol=1e-9 * np.abs(rows).max())


def test_augmented_hessian_is_singular_before_damping():
    W, X = _lowrank_layer(5, 3, 16, 200, 3)
    G = X.T @ X
    V, _ = oracle.top_singular_directions(G, 3)
    Gt = oracle.augmented_gram(G, V)
    ev = np.linalg.eigvalsh(Gt)
    assert ev[:3].max() < 1e-9 * ev.max()
    Xt = np.hstack([X, X @ V])
    assert np.allclose(Gt, Xt.T @ Xt, rtol=1e-10)


@pytest.mark.parametrize("seed", [6, 7])
def test_R_is_the_conditional_optimum(seed):
    W, X = _lowrank_layer(seed, 5, 32, 400, 4)
    res = oracle.il_layer(W, X, r=4, bits=3, group_size=8, lambda_rel=1e-3)
    Rcf = oracle.il_R_closed_form(res["H_raw"], res["L"], res["lam"], W, res["Wq"])
    assert np.allclose(res["R"], Rcf, rtol=1e-7, atol=1e-9 * np.abs(Rcf).max())


@pytest.mark.parametrize("seed", [8, 9])
def test_il_equals_babai_on_augmented_lattice(seed):
    """The intrinsic-LoRA pass is GPTQ on X~ = [X, X V_r]; its decisions are Babai's
    nearest plane on [X~; mu~ I] with the r extra coordinates real-valued."""
    n, r, bits = 14, 3, 3
    W, X = _lowrank_layer(seed, 4, n, 120, r)
    res = oracle.il_layer(W, X, r=r, bits=bits, group_size=0, lambda_rel=1e-3)
    Xt = np.hstack([X, X @ res["L"]])
    for i in range(W.shape[0]):
        s = np.full(n, res["scales"][i, 0])
        z = np.full(n, res["zeros"][i, 0])
        w = np.concatenate([W[i], np.zeros(r)])
        c, rho, _ = oracle.babai_nearest_plane(Xt, res["lam"], w, s, z, 7, n_int=n)
        assert np.array_equal(c, res["codes"][i])
        assert np.allclose(rho, res["R"][:, i], rtol=1e-6, atol=1e-9)


def test_residual_error_bound():
    """GPTQ-intrinsic LoRA summary, "Method" part 3: the IL bound replaces ||X||_F^2
    by the rank-r residual ||X - X_r||_F^2. Made concrete with the Gram-Schmidt
    lengths (lattice paper, section 4): with no clamped code,
    sum_j e_j^2 <= sum_j s_j^2 / (4 U_jj^2) <= max s^2 / 4 * (2||X - X_r||^2 + lam (n + r)),
    while the same chain for plain GPTQ needs 2||X||^2 + lam n."""
    n, r, bits = 40, 4, 4
    W, X = _lowrank_layer(10, 6, n, 500, r, snr=50.0)
    res = oracle.il_layer(W, X, r=r, bits=bits, group_size=0, lambda_rel=1e-3)
    maxq = (1 << bits) - 1
    clamped = (res["codes"] == 0) | (res["codes"] == maxq)
    u = np.diag(res["Ut"])[:n]
    Xr = X @ res["L"] @ res["L"].T
    resid = 2 * ((X - Xr) ** 2).sum() + res["lam"] * (n + r)
    full = 2 * (X ** 2).sum() + res["lam"] * n
    assert resid < 0.2 * full
    for i in range(W.shape[0]):
        if clamped[i].any():
            continue
        s = res["scales"][i, 0]
        e2 = res["loss_rows"][i]
        per_col = (s ** 2 / 4) * (1.0 / u ** 2)
        assert e2 <= per_col.sum() * (1 + 1e-12)
        assert per_col.sum() <= (s ** 2 / 4) * resid * (1 + 1e-12)
    # the data loss is within the bound as well (factor 1/2 from H = 2 X^T X)
    Wt = np.hstack([res["Wq"], np.zeros((W.shape[0], r))])
    D = np.hstack([W, np.zeros((W.shape[0], r))]) - Wt
    D[:, n:] = -res["R"].T
    Xt = np.hstack([X, X @ res["L"]])
    dl = ((Xt @ D.T) ** 2).sum(0)
    assert np.all(dl <= res["loss_rows"] / 2 * (1 + 1e-9))


@pytest.mark.parametrize("seed,r,lam_rel", [(11, 3, 1e-3), (12, 6, 1e-4), (13, 0, 1e-2)])
def test_il_damping_closed_form(seed, r, lam_rel):
    """The relative damping of the augmented Hessian (config: lambda~ = lambda_rel * mean of
    the diagonal of H~_raw = 2 X~^T X~ over all n + r coordinates). The extra columns X V_r
    have squared norms sigma_i^2 (diag(V_r^T G V_r) = sigma^2 for exact eigenvectors), so
    lambda~ = lambda_rel * 2 (||X||_F^2 + sum_{i<=r} sigma_i^2) / (n + r), with sigma taken
    here from an SVD of X. A mean over n entries, or over X~^T X~ instead of 2 X~^T X~,
    misses this value."""
    n = 30
    W, X = _lowrank_layer(seed, 3, n, 250, max(r, 1))
    G = X.T @ X
    V, _ = oracle.top_singular_directions(G, r)
    _, lam = oracle.il_hessian(G, V, lam_rel)
    sv = np.linalg.svd(X, compute_uv=False)
    closed = lam_rel * 2.0 * ((X ** 2).sum() + (sv[:r] ** 2).sum()) / (n + r)
    assert lam == pytest.approx(closed, rel=1e-12)
    if r:
        assert abs(lam - lam_rel * 2.0 * ((X ** 2).sum() + (sv[:r] ** 2).sum()) / n) > 1e-6 * lam
