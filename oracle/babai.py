"""Babai's nearest-plane algorithm in data space (oracle; test infrastructure only).

Lattice Geometry of Neural Network Quantization -- A Short Equivalence Proof of
GPTQ and Babai's Algorithm:
  * section 2: quantizing one neuron w is the closest vector problem on the
    lattice spanned by the columns of X, target X w;
  * section 3.1: with regularisation the basis is [X; mu I], which matches
    GPTQ's lambda term (2 X^T X + lambda I = 2 B^T B for mu = sqrt(lambda / 2));
  * sections 3.2-3.3: through the QL decomposition of the basis, the
    nearest-plane recursion in data space takes the same decisions as GPTQ in
    parameter space;
  * section 4: the error guarantee depends on the Gram-Schmidt lengths L_ii.

This module is a second, independent route to GPTQ's decisions: it never forms
a Hessian inverse.
"""
from __future__ import annotations

import numpy as np


def ql_decomposition(B: np.ndarray):
    """B = Q L with Q orthonormal columns and L lower triangular, diag(L) > 0.

    Taken as the QR decomposition of the column-reversed matrix: B J = Q' R'
    gives B = (Q' J)(J R' J), and J R' J is lower triangular.
    """
    Qr, Rr = np.linalg.qr(B[:, ::-1])
    Q = Qr[:, ::-1]
    L = Rr[::-1, ::-1]
    d = np.sign(np.diag(L))
    return Q * d[None, :], d[:, None] * L


def babai_nearest_plane(X, lam: float, w, s, z, maxq: int, n_int: int | None = None):
    """Clipped nearest-plane decisions for one neuron.

    X: k x N calibration, w: length-N weights (for intrinsic LoRA the last
    N - n_int coordinates are real-valued and start at 0), s, z: length-n_int
    grid step and zero-point per integer coordinate.

    Basis B = [X; mu I] (mu = sqrt(lambda / 2)), B = Q L. The lattice point for
    integer codes c and real tail rho is B [s (c - z); rho]; the target is
    B [w; 0-tail]. In data space the target is projected on the Gram-Schmidt
    directions (y = Q^T t), and the coordinates are decided in the order that
    peels one Gram-Schmidt direction at a time: row j of the triangular system
    involves only coordinates 0..j, so
        c_j = clip(rint((y_j - sum_{i<j} L_ji s_i c_i) / (L_jj s_j)), 0, maxq)
    (the s z offset is folded into the target). The real tail is then solved
    exactly from the last rows. Returns (codes, rho, L).
    """
    X = np.asarray(X, dtype=np.float64)
    k, N = X.shape
    n = N if n_int is None else n_int
    mu = np.sqrt(lam / 2.0)
    B = np.vstack([X, mu * np.eye(N)])
    Q, L = ql_decomposition(B)
    u = np.array(w, dtype=np.float64).copy()
    u[:n] = u[:n] + s * z
    t = B @ u
    y = Q.T @ t
    c = np.zeros(n)
    sc = np.zeros(n)
    for j in range(n):
        r = y[j] - L[j, :j] @ sc[:j]
        c[j] = np.clip(np.rint(r / (L[j, j] * s[j])), 0, maxq)
        sc[j] = s[j] * c[j]
    rho = np.zeros(N - n)
    if N > n:
        rhs = y[n:] - L[n:, :n] @ sc
        rho = np.linalg.solve(L[n:, n:], rhs)
    return c.astype(np.int64), rho, L
