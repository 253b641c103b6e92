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
ROWS = np.arange(0, 2048, 16)       # 128 rows spread over the layer


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

    # ---- one Bid-Up round (r = 0: no low-rank terms) on the pass's codes, same H
    n = L.n
    ws = g.workspace(g.GPTQ_OP_IL_REFINE, L.m, n, 0, 0, DEV)
    codes1 = out["codes"].clone()
    hist = torch.empty(2, dtype=torch.float64, device=DEV)
    g.gptq_il_refine(L.W, out["H"], 0, L.bits, L.group_size, 1, codes1, out["scales"], out["zeros"],
                     None, None, hist, ws)
    g.gptq_sync_status()
    hist = hist.cpu().numpy()
    Gg = np64(out["H"]) / 2
    c0 = unpack(out["codes"], L.bits, n)[ROWS]
    c1 = unpack(codes1, L.bits, n)[ROWS]
    zr = zeros.astype(np.float64)
    rep = oracle.bidup(W, None, None, c0, scales, zr, L.group_size, L.bits, Gg, force_codes=c1)
    v = rep["v"]
    valid = ~np.isnan(v)
    freec = np.clip(np.rint(np.where(valid, v, 0)), 0, (1 << L.bits) - 1)
    mism = valid & (freec != c1)
    worst = float(np.abs(np.abs(v[mism] - c1[mism]) - 0.5).max()) if mism.any() else 0.0
    agree = 1.0 - mism.sum() / valid.sum()
    print(f"{L.name}: Bid-Up codes agree {agree:.6f} ({int(mism.sum())} differ, worst distance "
          f"{worst:.2e} steps), {int((c1 != c0).sum())} codes changed on the sampled rows; loss "
          f"{hist[0]:.6e} -> {hist[1]:.6e}")
    assert agree >= 0.999 and worst < 1e-3 and hist[1] <= hist[0]
    assert (c1 != c0).sum() > 0


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

    # ---- one OLrC + Bid-Up round on the pass's output (same H as the device used)
    m = L.m
    ws = g.workspace(g.GPTQ_OP_IL_REFINE, m, n, r, 0, DEV)
    codes1 = out["codes"].clone()
    Lr = torch.empty(n, r, device=DEV)
    Rr = torch.empty(r, m, device=DEV)
    hist = torch.empty(2, dtype=torch.float64, device=DEV)
    g.gptq_il_refine(L.W, out["H"], r, L.bits, L.group_size, 1, codes1, out["scales"], out["zeros"],
                     Lr, Rr, hist, ws)
    g.gptq_sync_status()
    hist = hist.cpu().numpy()
    Gg = np64(out["H"]) / 2
    Wd = np64(L.W)
    c0_all = unpack(out["codes"], L.bits, n)
    sc_all = np64(out["scales"])
    zr_all = out["zeros"].cpu().numpy().astype(np.float64)
    Qhat = oracle.dequant(c0_all, sc_all, zr_all, L.group_size)
    Lo, Ro, _ = oracle.olrc(Wd, Qhat, Gg, r)
    LRg = np64(Lr) @ np64(Rr)
    e_lr = rel_fro(LRg, Lo @ Ro)
    D = Wd - Qhat - Ro.T @ Lo.T
    loss_o = float(((D @ Gg) * D).sum())
    l0 = abs(hist[0] - loss_o) / loss_o
    print(f"{L.name}: refine OLrC L R rel err {e_lr:.2e}; loss after OLrC {hist[0]:.6e} "
          f"(oracle {loss_o:.6e}, rel err {l0:.2e}); after Bid-Up {hist[1]:.6e}")
    assert e_lr <= 1e-3 and l0 <= REL_LOSS and hist[1] <= hist[0]
    c1 = unpack(codes1, L.bits, n)[ROWS]
    rep = oracle.bidup(Wd[ROWS], np64(Lr), np64(Rr)[:, ROWS], c0_all[ROWS], sc_all[ROWS],
                       zr_all[ROWS], L.group_size, L.bits, Gg, force_codes=c1)
    v = rep["v"]
    valid = ~np.isnan(v)
    free = np.clip(np.rint(np.where(valid, v, 0)), 0, (1 << L.bits) - 1)
    mism = valid & (free != c1)
    worst = float(np.abs(np.abs(v[mism] - c1[mism]) - 0.5).max()) if mism.any() else 0.0
    agree = 1.0 - mism.sum() / valid.sum()
    print(f"{L.name}: refine Bid-Up codes agree {agree:.6f} ({int(mism.sum())} differ, worst "
          f"distance {worst:.2e} steps), {int((c1 != c0_all[ROWS]).sum())} codes changed on the "
          f"sampled rows")
    assert agree >= 0.999 and worst < 1e-3
