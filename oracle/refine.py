"""OLrC + Bid-Up refinement of a quantized layer in float64 (oracle; test infrastructure only).

GPTQ-intrinsic LoRA summary, section 4 ("Refinement by Bid-Up"): after the intrinsic-LoRA
pass, two steps alternate, each minimising the layer-wise reconstruction error
||X W - X (Q + L R)||_F^2 over part of the variables, so the error never increases:
  * OLrC (optimal low-rank compensation): the best L, R for the fixed quantized Q;
  * Bid-Up: coordinate-wise updates of Q on its fixed quantization grid for fixed L, R.

Readings (the page states the mechanism and the guarantee only):
  * Orientation as everywhere in this package: W is m x n (one neuron per row), the
    dequantized weight is Qhat + R^T L^T with L n x r and R r x m, and the error of row o
    is d_o = w_o - qhat_o - (R^T L^T)_o; the objective is sum_o d_o G d_o^T, G = X^T X.
  * OLrC: with E = W - Qhat, the minimiser over rank-r products makes X (L R) the best
    rank-r approximation of X E^T. Its right singular vectors are the top-r eigenvectors P
    of E G E^T (m x m), so L R = E^T P P^T; this module takes R = P^T and L = E^T P
    (P's columns by decreasing eigenvalue, each with its largest-magnitude entry positive).
  * Bid-Up: one pass over the columns j = 0 .. n-1 in natural order, all rows at once.
    For coordinate j of row o the objective is a 1-D quadratic in its code c with vertex
    v = c_j + (d_o G)_j / (G_jj s) in code units (s, z the row's grid for j's group, kept
    fixed); the new code is clip(rint(v), 0, maxq) (round half to even, as the sweep),
    the nearest grid point to the vertex, hence the best code for that coordinate given
    all others. Coordinates with G_jj = 0 do not enter the objective and are left alone.
  * The refinement loop: `iters` rounds of (OLrC, Bid-Up), starting from the pass's codes
    (the pass's own L, R are replaced by the first OLrC).
"""
from __future__ import annotations

import numpy as np

from .gptq import _group_len


def dequant(codes, scales, zeros, group_size: int) -> np.ndarray:
    """Qhat[o, j] = s[o, g] (c[o, j] - z[o, g]) with g = j // group_size."""
    codes = np.asarray(codes, dtype=np.float64)
    m, n = codes.shape
    gs = _group_len(group_size, n)
    g = np.arange(n) // gs
    s = np.asarray(scales, dtype=np.float64)[:, g]
    z = np.asarray(zeros, dtype=np.float64)[:, g]
    return s * (codes - z)


def data_loss_rows(W, Qhat, L, R, G) -> np.ndarray:
    """Per row d G d^T with d = w - qhat - (R^T L^T) (summed: the reconstruction error)."""
    D = np.asarray(W, dtype=np.float64) - Qhat
    if L is not None and np.size(L):
        D = D - np.asarray(R, dtype=np.float64).T @ np.asarray(L, dtype=np.float64).T
    return np.einsum("ij,jk,ik->i", D, G, D)


def olrc(W, Qhat, G, r: int):
    """Best L (n x r), R (r x m) for fixed Qhat: L R = E^T P P^T, P = top-r eigvecs of E G E^T."""
    E = np.asarray(W, dtype=np.float64) - Qhat
    m, n = E.shape
    if r == 0:
        return np.zeros((n, 0)), np.zeros((0, m)), np.zeros(0)
    B = E @ G @ E.T
    w, Z = np.linalg.eigh(0.5 * (B + B.T))
    idx = np.argsort(w)[::-1][:r]
    P = Z[:, idx].copy()
    for c in range(r):
        i = np.argmax(np.abs(P[:, c]))
        if P[i, c] < 0:
            P[:, c] = -P[:, c]
    return E.T @ P, P.T.copy(), w[idx]


def bidup(W, L, R, codes, scales, zeros, group_size: int, bits: int, G,
          force_codes=None) -> dict:
    """One Bid-Up pass: coordinate descent over the codes on the fixed grid, natural order.

    Returns the new codes, the number of changed codes, the vertices v (m x n, code units)
    at which every decision was taken (for judging another implementation's decisions), and
    the per-row loss after the pass. ``force_codes`` replaces the decisions (replay).
    """
    Wd = np.asarray(W, dtype=np.float64)
    m, n = Wd.shape
    maxq = (1 << bits) - 1
    gs = _group_len(group_size, n)
    c = np.array(codes, dtype=np.int64)
    T = Wd - (np.asarray(R, dtype=np.float64).T @ np.asarray(L, dtype=np.float64).T
              if L is not None and np.size(L) else 0.0)
    D = T - dequant(c, scales, zeros, gs)
    Gd = D @ G                       # g_o = d_o G for every row
    V = np.full((m, n), np.nan)
    changed = 0
    sc = np.asarray(scales, dtype=np.float64)
    for j in range(n):
        gjj = G[j, j]
        if not gjj > 0:
            continue
        s = sc[:, j // gs]
        v = c[:, j] + Gd[:, j] / (gjj * s)
        V[:, j] = v
        cn = np.clip(np.rint(v), 0, maxq).astype(np.int64)
        if force_codes is not None:
            cn = np.asarray(force_codes[:, j], dtype=np.int64)
        delta = s * (cn - c[:, j])   # change of qhat_j; d_j changes by -delta
        changed += int(np.count_nonzero(cn != c[:, j]))
        c[:, j] = cn
        D[:, j] -= delta
        Gd -= np.outer(delta, G[j])
    loss = np.einsum("ij,ij->i", D, Gd)
    return dict(codes=c, changed=changed, v=V, loss_rows=loss)


def refine(W, codes, scales, zeros, G, r: int, bits: int, group_size: int, iters: int) -> dict:
    """`iters` rounds of OLrC then Bid-Up; loss history = [start with the pass's codes and the
    first OLrC's L, R, after Bid-Up 1, after OLrC 2, after Bid-Up 2, ...] (non-increasing)."""
    c = np.array(codes, dtype=np.int64)
    hist = []
    L = R = None
    for it in range(iters):
        Qhat = dequant(c, scales, zeros, group_size)
        L, R, _ = olrc(W, Qhat, G, r)
        hist.append(float(data_loss_rows(W, Qhat, L, R, G).sum()))
        out = bidup(W, L, R, c, scales, zeros, group_size, bits, G)
        c = out["codes"]
        hist.append(float(out["loss_rows"].sum()))
    return dict(codes=c, L=L, R=R, loss_hist=np.array(hist))
