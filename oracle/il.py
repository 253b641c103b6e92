"""GPTQ-intrinsic LoRA in float64 (oracle; test infrastructure only).

GPTQ-intrinsic LoRA summary, "Method", part 2 (the IL algorithm):
  * augmented calibration X~ = [X, X L] with L = V_r, the top-r right singular
    vectors of X;
  * augmented weights W~ = [W; 0] (in x out in the page's orientation); the
    pass quantizes the original coordinates to Q, and the r zero-initialised
    extra coordinates absorb the error and end as R;
  * the augmented Hessian is singular (the extra columns of X~ are linear
    combinations of X's columns), so it is factored through an
    eigendecomposition and a QR decomposition instead of a plain Cholesky.

In this module's orientation (one neuron per row, W is out x in) the extra
coordinates are r extra *columns* of W~ = [W, 0], placed last and never
quantized; at the end R = (W~[:, n:])^T, r x m, and L = V_r, n x r.
"""
from __future__ import annotations

import numpy as np

from .gptq import hessian, inverse_cholesky_upper, sweep


def top_singular_directions(G: np.ndarray, r: int):
    """Top-r eigenpairs of G = X^T X (= the right singular vectors of X).

    GPTQ-intrinsic LoRA summary, "Method" part 2: L = V_r, the top r right
    singular vectors of X. Taken from the undamped X^T X. Sorted by decreasing
    eigenvalue; sign fixed so that each vector's largest-magnitude entry is
    positive (the page leaves sign and order open). Returns (V_r, sigma^2).
    """
    w, Z = np.linalg.eigh(G)
    idx = np.argsort(w)[::-1][:r]
    V = Z[:, idx].copy()
    for c in range(r):
        i = np.argmax(np.abs(V[:, c]))
        if V[i, c] < 0:
            V[:, c] = -V[:, c]
    return V, w[idx]


def augmented_gram(G: np.ndarray, V: np.ndarray) -> np.ndarray:
    """X~^T X~ for X~ = [X, X V]: [[G, G V], [V^T G, V^T G V]]."""
    GV = G @ V
    return np.block([[G, GV], [GV.T, V.T @ GV]])


def il_hessian(G: np.ndarray, V: np.ndarray, lambda_rel: float):
    """H~ = 2 X~^T X~ + lambda~ I, with lambda~ = lambda_rel * mean(diag(2 X~^T X~)).

    The damping is relative to the mean diagonal of the augmented (n + r)-square
    raw Hessian, extra coordinates included (the pages leave the base of the
    relative damping open in intrinsic-LoRA mode). Returns (H~, lambda~).
    """
    Ht_raw = 2.0 * augmented_gram(G, V)
    lam = float(lambda_rel * np.mean(np.diag(Ht_raw)))
    return Ht_raw + lam * np.eye(Ht_raw.shape[0]), lam


def eig_qr_factor(Ht: np.ndarray) -> np.ndarray:
    """Upper U~ (positive diagonal) with H~^-1 = U~^T U~, via eigendecomposition and QR.

    GPTQ-intrinsic LoRA summary, "Method" part 2 ("implementation details"): the
    singular augmented Hessian is factored robustly through an
    eigendecomposition and a QR decomposition. Literally: H~ = Z diag(l) Z^T;
    M = diag(l)^-1/2 Z^T satisfies M^T M = H~^-1; the R factor of M = Q R
    satisfies R^T R = M^T M, and its rows are sign-flipped so that diag > 0.
    No Cholesky of H~ is ever taken.
    """
    lvals, Z = np.linalg.eigh(Ht)
    M = (1.0 / np.sqrt(lvals))[:, None] * Z.T
    _, R = np.linalg.qr(M)
    d = np.sign(np.diag(R))
    return d[:, None] * R


def schur_factor_rows(H_raw: np.ndarray, V: np.ndarray, lam: float) -> np.ndarray:
    """Rows 0..n-1 of U~ through the Schur complement of the extra block.

    With H~ = [[A, B], [B^T, C]] (A = H_raw + lam I, B = H_raw V,
    C = V^T H_raw V + lam I) and U~ = [[U11, U12], [0, U22]]:
    S = A - B C^-1 B^T satisfies S^-1 = U11^T U11 and U12 = -U11 B C^-1.
    An algebraic identity, used to cross-check the literal eig+QR factor (and
    the route the device takes). Returns the n x (n + r) block [U11, U12].
    """
    n = H_raw.shape[0]
    A = H_raw + lam * np.eye(n)
    B = H_raw @ V
    C = V.T @ B + lam * np.eye(V.shape[1])
    Cinv_Bt = np.linalg.solve(C, B.T)
    S = A - B @ Cinv_Bt
    U11 = inverse_cholesky_upper(S)
    U12 = -U11 @ Cinv_Bt.T
    return np.hstack([U11, U12])


def il_R_closed_form(H_raw: np.ndarray, V: np.ndarray, lam: float, W, Wq) -> np.ndarray:
    """R = H~22^-1 H~21 (W - W_hat)^T: the extra coordinates at their optimum
    given the quantized ones (the sweep leaves every unquantized coordinate at
    its conditional optimum of the damped quadratic)."""
    B = H_raw @ V
    C = V.T @ B + lam * np.eye(V.shape[1])
    D = np.asarray(W, dtype=np.float64) - np.asarray(Wq, dtype=np.float64)
    return np.linalg.solve(C, B.T @ D.T)


def il_layer(W, X=None, r: int = 64, bits: int = 3, group_size: int = 128,
             lambda_rel: float = 1e-4, H_raw=None, rows=None) -> dict:
    """The intrinsic-LoRA pass, literally: V_r, H~, eig+QR factor, sweep on [W, 0].

    With r = 0 this is, operation for operation, the plain pass except for the
    factorization route; ``gptq_layer`` is then reproduced exactly when the
    factor agrees (tests check it).
    """
    if H_raw is None:
        H_raw = hessian(X)
    G = H_raw / 2.0
    n = G.shape[0]
    Wd = np.asarray(W, dtype=np.float64)
    if rows is not None:
        Wd = Wd[rows]
    m = Wd.shape[0]
    V, sig2 = top_singular_directions(G, r)
    Ht, lam = il_hessian(G, V, lambda_rel)
    Ut = eig_qr_factor(Ht)
    Wt = np.hstack([Wd, np.zeros((m, r))])
    res = sweep(Wt, Ut[:n], bits, group_size, n_quant=n)
    res.update(H_raw=H_raw, L=V, sigma2=sig2, Ht=Ht, lam=lam, Ut=Ut, R=res["extra"].T.copy())
    return res
