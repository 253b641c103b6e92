"""Lattice basis reduction before Babai, in float64 (oracle; test infrastructure only).

The Lattice Geometry of Neural Network Quantization, section 5.2 ("Use of lattice basis
reduction"): before quantizing, reduce the basis of the (regularised) data lattice with LLL to
a good (short, nearly orthogonal) basis and run GPTQ / Babai on that basis (WITHREDUCTION). The
integer coefficients found in the reduced basis map back through the unimodular basis change
T; the page warns that large entries of T can push the quantized weights out of range
(clipping) and overfit the calibration data.

Readings taken here (the page gives no procedure for the quantization grid):
  * the grid is per channel (one scale s and zero-point z per output row, taken from the
    original weights by the min-max rule): then every row's lattice is s X' with the same
    X' = [X; mu I], so one reduction serves the whole layer. With per-group scales every row
    would have its own lattice;
  * GPTQ visits the columns in their natural order, which is Babai's nearest plane on the
    column-reversed basis (section 3.3: the QL decomposition). The reduction is therefore run
    on the reversed basis and reversed back, so that the Gram-Schmidt lengths GPTQ sees are the
    reduced ones;
  * coefficients in the reduced basis are unconstrained integers; mapped back, codes outside
    [0, maxq] are clipped and counted.

LLL itself: Lenstra, Lenstra and Lovasz (1982), with the Lovasz parameter delta = 3/4, run on
the Gram matrix of the basis with the Gram-Schmidt coefficients kept incrementally (the real
version of H. Cohen, "A Course in Computational Algebraic Number Theory", Algorithm 2.6.3).
"""
from __future__ import annotations

import numpy as np


def lll_gram(G: np.ndarray, delta: float = 0.75, max_swaps: int = 10_000_000):
    """LLL-reduce the basis whose Gram matrix is G (n x n, symmetric positive definite).

    Returns (T, G_red, stats): T is an integer unimodular n x n matrix (as float64 with integer
    values) whose columns are the reduced basis vectors' coordinates in the input basis, so
    that the reduced basis is B T and its Gram matrix G_red = T^T G T; stats holds the number
    of swaps and size reductions. On return, with mu and Bn the Gram-Schmidt coefficients and
    squared lengths of B T: |mu[k, j]| <= 1/2 for j < k (size reduction) and
    Bn[k] >= (delta - mu[k, k-1]^2) Bn[k-1] (the Lovasz condition).
    """
    G = np.array(G, dtype=np.float64)
    n = G.shape[0]
    T = np.eye(n)
    mu = np.zeros((n, n))
    Bn = np.zeros(n)
    stats = {"swaps": 0, "reductions": 0}
    if n == 0:
        return T, G, stats

    def gso_row(k):
        for j in range(k):
            mu[k, j] = (G[k, j] - np.dot(mu[j, :j] * mu[k, :j], Bn[:j])) / Bn[j]
        Bn[k] = G[k, k] - np.dot(mu[k, :k] ** 2, Bn[:k])

    def reduce(k, l):
        q = np.rint(mu[k, l])
        if q == 0.0:
            return
        stats["reductions"] += 1
        # b_k <- b_k - q b_l
        T[:, k] -= q * T[:, l]
        G[k, :] -= q * G[l, :]
        G[:, k] -= q * G[:, l]   # G[k, k] is now g_kk - 2 q g_kl + q^2 g_ll
        mu[k, l] -= q
        mu[k, :l] -= q * mu[l, :l]

    def swap(k, kmax):
        stats["swaps"] += 1
        T[:, [k - 1, k]] = T[:, [k, k - 1]]
        G[[k - 1, k], :] = G[[k, k - 1], :]
        G[:, [k - 1, k]] = G[:, [k, k - 1]]
        mu[[k - 1, k], :k - 1] = mu[[k, k - 1], :k - 1]
        m = mu[k, k - 1]
        B = Bn[k] + m * m * Bn[k - 1]
        mu[k, k - 1] = m * Bn[k - 1] / B
        Bn[k] = Bn[k - 1] * Bn[k] / B
        Bn[k - 1] = B
        for i in range(k + 1, kmax + 1):
            t = mu[i, k]
            mu[i, k] = mu[i, k - 1] - m * t
            mu[i, k - 1] = t + mu[k, k - 1] * mu[i, k]

    Bn[0] = G[0, 0]
    k, kmax = 1, 0
    while k < n:
        if k > kmax:
            kmax = k
            gso_row(k)
        reduce(k, k - 1)
        if Bn[k] < (delta - mu[k, k - 1] ** 2) * Bn[k - 1]:
            swap(k, kmax)
            k = max(1, k - 1)
            if stats["swaps"] > max_swaps:
                raise RuntimeError("LLL did not finish within max_swaps")
        else:
            for l in range(k - 2, -1, -1):
                reduce(k, l)
            k += 1
    return T, G, stats


def gram_schmidt(G: np.ndarray):
    """Gram-Schmidt coefficients mu (unit lower triangular) and squared lengths Bn of the
    basis with Gram matrix G, from the Cholesky factor G = R^T R: mu = (R / diag R)^T."""
    R = np.linalg.cholesky(G).T
    d = np.diag(R)
    return (R / d[:, None]).T, d ** 2


def reduce_for_gptq(G: np.ndarray, delta: float = 0.75):
    """LLL for the column order GPTQ visits: reduce the reversed basis, reverse back.

    Returns (T, G_red, stats) with G_red = T^T G T; GPTQ's sweep on G_red in natural column
    order is Babai's nearest plane on the LLL-reduced basis."""
    P = np.arange(G.shape[0])[::-1]
    Tr, Gr, stats = lll_gram(G[np.ix_(P, P)], delta)
    T = np.zeros_like(Tr)
    T[np.ix_(P, P)] = Tr   # T = P Tr P
    return T, Gr[np.ix_(P, P)], stats


def round_in_basis(Ut: np.ndarray, Gb: np.ndarray, force=None, record_v: bool = False):
    """One-sided adaptive rounding of the rows of Ut (real coordinates) to integers under the
    Gram matrix Gb: GPTQ without a grid (rint, ties to even, no clipping) in natural column
    order, which is Babai's nearest plane on the basis with Gram matrix Gb.

    With ``force`` (integers of the same shape) the decisions are taken from it instead and the
    pre-rounding values along that trajectory are returned as well (a replay of another
    implementation's decisions). Returns C, or (C, V) when record_v or force is given."""
    Gi = np.linalg.inv(Gb)
    U = np.linalg.cholesky(Gi).T                 # Gb^-1 = U^T U, U upper
    Wc = np.array(Ut, dtype=np.float64)
    m, n = Wc.shape
    C = np.zeros((m, n))
    V = np.zeros((m, n))
    for j in range(n):
        v = Wc[:, j].copy()
        c = np.rint(v) if force is None else np.asarray(force[:, j], dtype=np.float64)
        e = (v - c) / U[j, j]
        Wc[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        C[:, j] = c
        V[:, j] = v
    if record_v or force is not None:
        return C, V
    return C


def withreduction(W, H_raw, bits: int, lambda_rel: float, delta: float = 0.75) -> dict:
    """GPTQ with lattice basis reduction (WITHREDUCTION), per-channel grid.

    W: m x n weights; H_raw = 2 X^T X. With lambda = lambda_rel mean(diag H_raw) and the
    regularised Gram G' = X'^T X' = (H_raw + lambda I) / 2 (X' = [X; mu I], mu^2 = lambda / 2):
      s, z per row by the min-max rule on the original row (one group per row);
      u = w / s + z (grid coordinates); T, G_red = reduce_for_gptq(G');
      c' = Babai in the reduced basis on T^-1 u;  c = clip(T c', 0, maxq).
    Returns codes, scales, zeros, the count of clipped codes, the unclipped codes, T and the
    regularised loss per row sum (w - w_hat)^T (H_raw + lambda I) (w - w_hat)."""
    from .gptq import damp, minmax_grid
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    maxq = (1 << bits) - 1
    Hd, lam = damp(np.asarray(H_raw, dtype=np.float64), lambda_rel)
    s, z, _ = minmax_grid(W, maxq)
    U = W / s[:, None] + z[:, None]
    T, Gr, stats = reduce_for_gptq(Hd / 2.0)
    Ti = np.rint(np.linalg.inv(T))
    Cr = round_in_basis(U @ Ti.T, Gr)
    C_raw = Cr @ T.T
    C = np.clip(C_raw, 0, maxq)
    Wq = s[:, None] * (C - z[:, None])
    D = W - Wq
    loss = np.einsum("ij,jk,ik->i", D, Hd, D)
    return dict(codes=C.astype(np.int64), codes_unclipped=C_raw, scales=s, zeros=z.astype(np.int64),
                n_clipped=int((C != C_raw).sum()), T=T, G_red=Gr, lam=lam, loss_rows=loss,
                stats=stats)
