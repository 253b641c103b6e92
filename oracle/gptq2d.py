"""Two-sided adaptive rounding, GPTQ-2D, in float64 (oracle; test infrastructure only).

GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding:
  * section 1 (problem): round a real matrix X (m x n) to an integer matrix Z minimising
    ||A (Z - X) B||_F^2 with fixed non-singular A (m x m) and B (n x n); vectorised, this is
    ||(B^T (x) A)(vec Z - vec X)||^2, i.e. the one-sided adaptive rounding of vec X under the
    Gram matrix H (x) G with G = A^T A, H = B B^T;
  * section 2 (method): the feedback of the vectorised sweep is the Kronecker product of the
    two triangular factors, so rounding entry (i, j) changes only the rectangle of entries
    (p, q) with p >= i and q >= j, by a rank-1 term; entries on one anti-diagonal i + j = s
    do not affect each other and are rounded together, in m + n - 1 stages; a buffer of
    column-pushed errors (C = L E in the page's notation) is pushed along the rows, so every
    entry receives each dependency once and the sweep costs O(m n max(m, n));
  * section 3, Theorems 1 and 2: any order that respects the dependencies gives the same Z,
    so the anti-diagonal sweep reproduces the vectorised one exactly (with a deterministic
    tie-break).

Readings: the one-sided sweep is GPTQ's without a grid, on the integers: in order,
z_k = rint(v_k) (half to even), e_k = (v_k - z_k) / U_kk, v_{k+1:} -= e_k U_{k,k+1:}, with U
the upper factor of the inverse Gram matrix (Gram^-1 = U^T U). vec stacks columns (entry
(i, j) is coordinate i + j m), so the Kronecker factor is U_H (x) U_G, which is upper
triangular in that order. No damping (the page's A and B are non-singular).
"""
from __future__ import annotations

import numpy as np

from .gptq import inverse_cholesky_upper


def adaptive_round_1d(x, U) -> np.ndarray:
    """One-sided adaptive rounding of the vector x in index order with the upper factor U."""
    v = np.array(x, dtype=np.float64)
    z = np.zeros(len(v))
    for k in range(len(v)):
        z[k] = np.rint(v[k])
        e = (v[k] - z[k]) / U[k, k]
        v[k + 1:] -= e * U[k, k + 1:]
    return z.astype(np.int64)


def gptq2d_vectorized(X, G, H) -> np.ndarray:
    """The problem as stated: adaptive rounding of vec X under H (x) G (explicit mn x mn factor)."""
    X = np.asarray(X, dtype=np.float64)
    m, n = X.shape
    UK = np.kron(inverse_cholesky_upper(H), inverse_cholesky_upper(G))
    return adaptive_round_1d(X.reshape(-1, order="F"), UK).reshape(m, n, order="F")


def gptq2d_antidiagonal(X, G, H, force_Z=None) -> dict:
    """GPTQ-2D: stages s = 0 .. m+n-2 over the anti-diagonals, with two buffers:
      C[p, j] = sum_{i <= p} U_G[i, p] e_ij   (errors pushed down their column), and
      V[p, q] = sum_{j < q} C[p, j] U_H[j, q] (finished column buffers pushed along the row).
    Entry (p, q) is rounded from v = x_pq - V[p, q] - C[p, q] U_H[q, q], with C[p, q] then
    holding the errors of the entries above it in its column only. Its error
    e = (v - z) / (U_G[p, p] U_H[q, q]) is pushed down column q, after which C[p, q] is final
    and is pushed along row p. ``force_Z`` replaces the decisions (replay of another
    implementation's trajectory); the pre-rounding values v are returned either way."""
    X = np.asarray(X, dtype=np.float64)
    m, n = X.shape
    UG, UH = inverse_cholesky_upper(G), inverse_cholesky_upper(H)
    C = np.zeros((m, n))
    V = np.zeros((m, n))
    Z = np.zeros((m, n), dtype=np.int64)
    E = np.zeros((m, n))
    Vpre = np.zeros((m, n))
    for s in range(m + n - 1):
        for p in range(max(0, s - n + 1), min(m - 1, s) + 1):
            q = s - p
            v = X[p, q] - V[p, q] - C[p, q] * UH[q, q]
            z = np.rint(v) if force_Z is None else float(force_Z[p, q])
            e = (v - z) / (UG[p, p] * UH[q, q])
            Z[p, q], E[p, q], Vpre[p, q] = int(z), e, v
            C[p:, q] += UG[p, p:] * e
            V[p, q + 1:] += C[p, q] * UH[q, q + 1:]
    return dict(Z=Z, E=E, UG=UG, UH=UH, v=Vpre)


def reverse_cholesky_upper(M) -> np.ndarray:
    """Upper-triangular R with positive diagonal and M = R R^T: the Cholesky factor of M with
    the index order reversed. R is the inverse of the upper factor U of M^-1 (M^-1 = U^T U)."""
    M = np.asarray(M, dtype=np.float64)
    L = np.linalg.cholesky(M[::-1, ::-1])
    return np.ascontiguousarray(L[::-1, ::-1])


def gptq2d_residuals(X, Z, G, H) -> np.ndarray:
    """The scaled residual c = v - z of every decision, in closed form from Z alone.

    Section 2: entry (p, q) receives U_G[i, p] U_H[j, q] e_ij from every earlier entry, so
    X - Z = U_G^T E U_H (the entry's own error included). Hence E = Rg^T (X - Z) Rh with
    Rg = U_G^-1, Rh = U_H^-1 (G = Rg Rg^T, H = Rh Rh^T), and c = e U_G[p,p] U_H[q,q] =
    E[p, q] / (Rg[p,p] Rh[q,q]). The sweep's Z is the Babai point of the Kronecker basis:
    every |c| <= 1/2 (the residual lies in the Gram-Schmidt parallelepiped), and no other
    integer matrix has that property, so this checks a Z of any size."""
    D = np.asarray(X, dtype=np.float64) - np.asarray(Z, dtype=np.float64)
    Rg, Rh = reverse_cholesky_upper(G), reverse_cholesky_upper(H)
    E = Rg.T @ D @ Rh
    return E / np.outer(np.diag(Rg), np.diag(Rh))


def two_sided_loss(X, Z, A, B) -> float:
    """||A (Z - X) B||_F^2."""
    D = np.asarray(Z, dtype=np.float64) - np.asarray(X, dtype=np.float64)
    return float(np.linalg.norm(np.asarray(A) @ D @ np.asarray(B)) ** 2)
