"""Parity at the full workload sizes, in the launch configuration bench.py times (one
gptq_hessian_accumulate call over all calibration tokens, then the factor and the sweep).

The fp64 oracle computes the whole H (chunked X^T X) and the factor; the sweep, whose cost
is m n^2, is replayed on a sample of rows (rows are independent problems), which is enough to
judge every kernel: each sampled row goes through all 48 panels and all lazy updates.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from gpu_parity import REL_H, REL_LOSS, REL_SCALE, check_replay, np64, rel_fro, unpack

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROWS = np.arange(0, 2048, 64)       # 32 rows spread over the layer


@pytest.fixture(scope="module")
def g():
    import post_weight_quantization_06_b200 as g
    return g


def _oracle_hessian(X):
    H = np.zeros((X.shape[1], X.shape[1]))
    for t0 in range(0, X.shape[0], 16384):
        H += oracle.hessian(X[t0:t0 + 16384].double().cpu().numpy())
    return H


def test_full_mlp_down_2048x6144(g):
    L = datagen.mlp_down(device=DEV)
    out = g.quantize_layer(L.W, L.X, bits=L.bits, group_size=L.group_size,
                           lambda_rel=L.lambda_rel, block_size=L.block_size,
                           chunk_tokens=L.k)
    Href = _oracle_hessian(L.X)
    herr = rel_fro(np64(out["H"]), Href)
    Hd, lam = oracle.damp(Href, L.lambda_rel)
    print(f"{L.name}: H rel err {herr:.2e}, lambda rel err {abs(out['lam'].item() - lam) / lam:.2e}")
    assert herr <= REL_H
    assert abs(out["lam"].item() - lam) / lam < 1e-4
    U = oracle.inverse_cholesky_upper(Hd)
    W = np64(L.W)[ROWS]
    codes = unpack(out["codes"], L.bits, L.n)[ROWS]
    zeros = out["zeros"].cpu().numpy().astype(np.int64)[ROWS]
    scales = np64(out["scales"])[ROWS]
    loss = out["loss"].cpu().numpy()[ROWS]
    check_replay(W, U, L.bits, L.group_size, codes, zeros, scales, loss_gpu=loss, label=L.name)
    free = oracle.sweep(W, U, L.bits, L.group_size)
    lr = abs(loss.sum() - free["loss_rows"].sum()) / free["loss_rows"].sum()
    print(f"{L.name}: loss rel err vs free-running oracle {lr:.2e}")
    assert lr <= REL_LOSS


def test_full_lowrank_il_r64(g):
    L = datagen.lowrank(device=DEV)
    out = g.quantize_layer(L.W, L.X, bits=L.bits, group_size=L.group_size,
                           lambda_rel=L.lambda_rel, block_size=L.block_size, r=L.r,
                           chunk_tokens=L.k)
    Href = _oracle_hessian(L.X)
    assert rel_fro(np64(out["H"]), Href) <= REL_H
    G = Href / 2
    V, _ = oracle.top_singular_directions(G, L.r)
    Lg = np64(out["L"])
    verr = np.abs(Lg - V).max() / np.abs(V).max()
    Ht, lam = oracle.il_hessian(G, V, L.lambda_rel)
    print(f"{L.name}: L max rel err {verr:.2e}, lambda~ rel err {abs(out['lam'].item() - lam) / lam:.2e}")
    assert verr <= REL_SCALE and abs(out["lam"].item() - lam) / lam < 1e-4
    Ut = oracle.eig_qr_factor(Ht)
    n, r = L.n, L.r
    Wt = np.hstack([np64(L.W)[ROWS], np.zeros((len(ROWS), r))])
    codes = unpack(out["codes"], L.bits, n)[ROWS]
    zeros = out["zeros"].cpu().numpy().astype(np.int64)[ROWS]
    scales = np64(out["scales"])[ROWS]
    loss = out["loss"].cpu().numpy()[ROWS]
    Rg = np64(out["R"])[:, ROWS].T
    check_replay(Wt, Ut[:n], L.bits, L.group_size, codes, zeros, scales, loss_gpu=loss,
                 n_quant=n, extra_gpu=Rg, label=L.name)
    free = oracle.sweep(Wt, Ut[:n], L.bits, L.group_size, n_quant=n)
    lr = abs(loss.sum() - free["loss_rows"].sum()) / free["loss_rows"].sum()
    print(f"{L.name}: loss rel err vs free-running oracle {lr:.2e}")
    assert lr <= REL_LOSS
