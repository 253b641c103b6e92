"""Plain GPTQ layer pass in float64 (oracle; test infrastructure only).

Orientation: W is (out rows m) x (in columns n); the calibration matrix X is
(tokens k) x (in n). The pages write the layer as XW with W in x out (the
GPTQ-intrinsic LoRA summary, "Problem statement") or as Wx with one neuron per
row (Lattice Geometry of Neural Network Quantization, section 2); this module
stores the transpose of the former, i.e. one neuron per row, and sweeps the
input columns j = 0 .. n-1 in their natural order.
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------------------------------
# Hessian and damping
# ---------------------------------------------------------------------------------------

def hessian(X, chunk: int = 16384) -> np.ndarray:
    """H_raw = 2 X^T X, accumulated in float64 over token chunks.

    GPTQ (encyclopedia article), "Technical approach": the quantizer is driven by
    a second-order proxy of the loss, the Hessian of the layer-wise squared
    error, which for ||XW - XQ||^2 is 2 X^T X. No 1/k averaging is applied:
    with a relative damping the result of the pass does not depend on a
    global scale of H.
    """
    X = np.asarray(X)
    k, n = X.shape
    H = np.zeros((n, n), dtype=np.float64)
    for t0 in range(0, k, chunk):
        Xc = np.asarray(X[t0:t0 + chunk], dtype=np.float64)
        H += Xc.T @ Xc
    return 2.0 * H


def damp(H_raw: np.ndarray, lambda_rel: float):
    """H = H_raw + lambda I with lambda = lambda_rel * mean(diag H_raw).

    Lattice Geometry of Neural Network Quantization, section 3.1: the
    regularised basis [X; mu I] is the lattice form of GPTQ's lambda
    regularisation X^T X + lambda I; it keeps the basis independent (H positive
    definite) even when k < n. Returns (H, lambda).
    """
    lam = float(lambda_rel * np.mean(np.diag(H_raw)))
    return H_raw + lam * np.eye(H_raw.shape[0]), lam


def inverse_cholesky_upper(H: np.ndarray) -> np.ndarray:
    """Upper-triangular U with positive diagonal and H^-1 = U^T U.

    GPTQ-2D, section 2 and section 4 ("Factorization"): the error feedback of
    adaptive rounding is read from a triangular factor of the inverse Gram
    matrix. Computed literally: Cholesky of H, triangular inverse, H^-1, then
    the Cholesky factor of H^-1 written as U^T U.
    """
    L = np.linalg.cholesky(H)            # H = L L^T
    Linv = np.linalg.inv(L)              # lower triangular
    Hinv = Linv.T @ Linv                 # H^-1
    return np.linalg.cholesky(Hinv).T    # H^-1 = (U^T)(U), U upper


# ---------------------------------------------------------------------------------------
# Grid
# ---------------------------------------------------------------------------------------

def minmax_grid(seg: np.ndarray, maxq: int):
    """Asymmetric min-max integer grid of one group, per row.

    GPTQ (encyclopedia article), "Technical approach": weights are split into
    groups and each group has its own scale. The pages fix no further detail;
    the reading taken: the range always contains 0 (xmin = min(0, min w),
    xmax = max(0, max w)); a zero range is widened to [-1, 1]; the step is
    s = (xmax - xmin) / maxq and the integer zero-point z = rint(-xmin / s),
    clipped to [0, maxq]. Returns (s, z, z_real) with z_real = -xmin / s
    before rounding.
    """
    xmin = np.minimum(seg.min(axis=1), 0.0)
    xmax = np.maximum(seg.max(axis=1), 0.0)
    flat = xmax == xmin
    xmin = np.where(flat, -1.0, xmin)
    xmax = np.where(flat, 1.0, xmax)
    s = (xmax - xmin) / maxq
    z_real = -xmin / s
    z = np.clip(np.rint(z_real), 0, maxq)
    return s, z, z_real


# ---------------------------------------------------------------------------------------
# The column sweep
# ---------------------------------------------------------------------------------------

def _group_len(group_size: int, n: int) -> int:
    return group_size if group_size else n


def sweep(W, U, bits: int, group_size: int, n_quant: int | None = None,
          force_codes=None, force_zeros=None, record_v: bool = False) -> dict:
    """Greedy fixed-order column sweep with closed-form error feedback.

    GPTQ (encyclopedia article), "Technical approach": columns are quantized one
    at a time and the remaining weights are updated in closed form (the Optimal
    Brain Quantization update) to compensate the error. GPTQ-2D, section 1
    ("one-sided case"): entries are processed in a fixed order and the rounding
    error is propagated through a triangular feedback matrix.

    For each column j (natural order) and every row at once:
      * at a group start (j % group_size == 0; per-channel: j == 0 only) the
        grid (s, z) is taken from the *current* working weights of the group;
      * v = w_j / s + z, c = clip(rint(v), 0, maxq)  (round half to even: the
        deterministic tie-break GPTQ-2D's Theorem 2 asks for);
      * w_hat = s (c - z); e = (w_j - w_hat) / U_jj;
      * w_{j+1:} -= e * U_{j, j+1:}.

    W: m x N. The first ``n_quant`` columns (default N) are quantized; any
    further columns are never quantized and only receive feedback (this is how
    the intrinsic-LoRA extra coordinates are carried). U: at least n_quant rows
    of an N x N upper factor.

    ``force_codes`` / ``force_zeros`` (m x n_quant, m x groups) replace the
    rounding decisions by given ones; this is the replay used to judge another
    implementation's decisions along its own trajectory.
    """
    Wc = np.array(W, dtype=np.float64)
    m, N = Wc.shape
    n = N if n_quant is None else n_quant
    maxq = (1 << bits) - 1
    gs = _group_len(group_size, n)
    G = -(-n // gs)
    codes = np.zeros((m, n), dtype=np.int64)
    scales = np.zeros((m, G))
    zeros = np.zeros((m, G))
    zeros_real = np.zeros((m, G))
    err = np.zeros((m, n))
    Wq = np.zeros((m, n))
    V = np.zeros((m, n)) if record_v else None
    s = z = None
    for j in range(n):
        if j % gs == 0:
            g = j // gs
            s, z, zr = minmax_grid(Wc[:, j:min(j + gs, n)], maxq)
            if force_zeros is not None:
                z = np.asarray(force_zeros[:, g], dtype=np.float64)
            scales[:, g], zeros[:, g], zeros_real[:, g] = s, z, zr
        w = Wc[:, j].copy()
        v = w / s + z
        c = np.clip(np.rint(v), 0, maxq)
        if force_codes is not None:
            c = np.asarray(force_codes[:, j], dtype=np.float64)
        q = s * (c - z)
        e = (w - q) / U[j, j]
        Wc[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        Wc[:, j] = q
        codes[:, j] = c.astype(np.int64)
        err[:, j] = e
        Wq[:, j] = q
        if record_v:
            V[:, j] = v
    out = dict(codes=codes, scales=scales, zeros=zeros.astype(np.int64), zeros_real=zeros_real,
               err=err, Wq=Wq, extra=Wc[:, n:].copy(), loss_rows=(err ** 2).sum(axis=1))
    if record_v:
        out["v"] = V
    return out


def sweep_blocked(W, U, bits: int, group_size: int, block: int, n_quant: int | None = None) -> dict:
    """The same sweep with the lazy block update.

    GPTQ-2D, section 2 ("blocked implementation"): errors of a block of columns
    are accumulated and flushed to the rest of the matrix with one matrix
    product, as in GPTQ's lazy block update; section 3 (Theorem 1) says any
    processing order that respects the feedback dependencies gives the same
    rounding. Inside a block the feedback is applied column by column to the
    block's own columns; the trailing columns receive Err @ U[block, trailing]
    once per block. Requires that every group start falls on a block start or
    that groups nest inside blocks (block % group_size == 0 or
    group_size % block == 0), so that group statistics see fully updated
    weights.
    """
    Wc = np.array(W, dtype=np.float64)
    m, N = Wc.shape
    n = N if n_quant is None else n_quant
    maxq = (1 << bits) - 1
    gs = _group_len(group_size, n)
    assert block % gs == 0 or gs % block == 0
    G = -(-n // gs)
    codes = np.zeros((m, n), dtype=np.int64)
    scales = np.zeros((m, G))
    zeros = np.zeros((m, G))
    err = np.zeros((m, n))
    Wq = np.zeros((m, n))
    s = z = None
    for b0 in range(0, n, block):
        b1 = min(n, b0 + block)
        for j in range(b0, b1):
            if j % gs == 0:
                g = j // gs
                s, z, _ = minmax_grid(Wc[:, j:min(j + gs, n)], maxq)
                scales[:, g], zeros[:, g] = s, z
            w = Wc[:, j].copy()
            c = np.clip(np.rint(w / s + z), 0, maxq)
            q = s * (c - z)
            e = (w - q) / U[j, j]
            Wc[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            Wc[:, j] = q
            codes[:, j], err[:, j], Wq[:, j] = c, e, q
        Wc[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
    return dict(codes=codes, scales=scales, zeros=zeros.astype(np.int64), err=err, Wq=Wq,
                extra=Wc[:, n:].copy(), loss_rows=(err ** 2).sum(axis=1))


def gptq_layer(W, X=None, bits: int = 4, group_size: int = 128, lambda_rel: float = 0.01,
               H_raw=None, rows=None) -> dict:
    """The whole plain pass: H_raw = 2 X^T X, damping, U, sweep.

    ``rows`` optionally restricts the sweep to a subset of rows (rows are
    independent problems: Lattice Geometry of Neural Network Quantization,
    section 2, "decomposition").
    """
    if H_raw is None:
        H_raw = hessian(X)
    H, lam = damp(H_raw, lambda_rel)
    U = inverse_cholesky_upper(H)
    Wr = np.asarray(W, dtype=np.float64)
    if rows is not None:
        Wr = Wr[rows]
    res = sweep(Wr, U, bits, group_size)
    res.update(H_raw=H_raw, H=H, lam=lam, U=U)
    return res


# ---------------------------------------------------------------------------------------
# Losses and replay
# ---------------------------------------------------------------------------------------

def regularised_loss_rows(W, Wq, H) -> np.ndarray:
    """Per row d^T H d with d = w - w_hat: the damped objective GPTQ minimises."""
    D = np.asarray(W, dtype=np.float64) - np.asarray(Wq, dtype=np.float64)
    return np.einsum("ij,jk,ik->i", D, H, D)


def data_loss_rows(W, Wq, G) -> np.ndarray:
    """Per row ||X (w - w_hat)||^2 = d^T G d with G = X^T X.

    GPTQ-intrinsic LoRA summary, "Problem statement": the layer-wise
    reconstruction error ||XW - X(Q + LR)||_F^2; summing the rows gives it.
    """
    return regularised_loss_rows(W, Wq, G)


def replay(W, U, bits: int, group_size: int, codes, zeros, n_quant: int | None = None) -> dict:
    """Follow another implementation's decisions and judge each of them.

    The sweep is re-run with its codes and zero-points forced to the given
    ones, so the oracle's pre-rounding values v are computed along that
    trajectory. Every decision that differs from the oracle's own rounding of v
    is reported with its distance to the rounding boundary, in grid steps
    (|v - (min(c, c') + 1/2)|, or inf when the two codes are not adjacent).
    The same is done for the zero-points (z_real against the given z).
    Returns counts, distances and the oracle's scales along the trajectory.
    """
    codes = np.asarray(codes)
    zeros = np.asarray(zeros)
    maxq = (1 << bits) - 1
    res = sweep(W, U, bits, group_size, n_quant=n_quant, force_codes=codes,
                force_zeros=zeros, record_v=True)
    v = res["v"]
    own = np.clip(np.rint(v), 0, maxq)
    bad = own != codes
    lo = np.minimum(own, codes)
    dist = np.where(np.abs(own - codes) == 1, np.abs(v - (lo + 0.5)), np.inf)
    zr = res["zeros_real"]
    zown = np.clip(np.rint(zr), 0, maxq)
    zbad = zown != zeros
    zlo = np.minimum(zown, zeros)
    zdist = np.where(np.abs(zown - zeros) == 1, np.abs(zr - (zlo + 0.5)), np.inf)
    return dict(
        n_codes=codes.size,
        n_code_mismatch=int(bad.sum()),
        code_dist=dist[bad],
        n_zero_mismatch=int(zbad.sum()),
        zero_dist=zdist[zbad],
        scales=res["scales"],
        zeros_real=zr,
        err=res["err"],
        Wq=res["Wq"],
        extra=res["extra"],
        loss_rows=res["loss_rows"],
        v=v,
    )
