"""Pins of the OLrC + Bid-Up refinement oracle (GPTQ-intrinsic LoRA summary, section 4)."""
import itertools

import numpy as np
import pytest

import oracle


def _layer(seed, m, n, k, r_sig=4, snr=30.0):
    g = np.random.default_rng(seed)
    P, _ = np.linalg.qr(g.standard_normal((n, r_sig)))
    a = np.sqrt(snr * n / np.arange(1, r_sig + 1) / (1.0 / np.arange(1, r_sig + 1)).sum())
    X = (g.standard_normal((k, r_sig)) * a) @ P.T + g.standard_normal((k, n))
    W = g.standard_normal((m, n)) * 0.02
    return W, X


def _start(W, X, r, bits, gs):
    res = oracle.il_layer(W, X, r=r, bits=bits, group_size=gs, lambda_rel=1e-3)
    return res, res["H_raw"] / 2.0


def test_olrc_is_the_truncated_svd_of_the_output_error():
    W, X = _layer(1, 7, 24, 300)
    res, G = _start(W, X, 3, 2, 8)
    Qhat = oracle.dequant(res["codes"], res["scales"], res["zeros"], 8)
    for r in (1, 3, 5):
        L, R, _ = oracle.olrc(W, Qhat, G, r)
        Y = X @ (W - Qhat).T                         # k x m output error
        U_, sv, Vt = np.linalg.svd(Y, full_matrices=False)
        Yr = (U_[:, :r] * sv[:r]) @ Vt[:r]
        assert np.allclose(X @ (L @ R), Yr, rtol=1e-8, atol=1e-10 * np.abs(Y).max())
        loss = oracle.lowrank_loss_rows(W, Qhat, L, R, G).sum()
        assert loss == pytest.approx((sv[r:] ** 2).sum(), rel=1e-9)


def test_olrc_rank_zero_is_empty():
    W, X = _layer(2, 4, 16, 100)
    res, G = _start(W, X, 0, 3, 8)
    Qhat = oracle.dequant(res["codes"], res["scales"], res["zeros"], 8)
    L, R, _ = oracle.olrc(W, Qhat, G, 0)
    assert L.shape == (16, 0) and R.shape == (0, 4)


def _loss_of_row(w_t, codes_row, s_row, z_row, gs, G):
    n = len(codes_row)
    g = np.arange(n) // gs
    d = w_t - s_row[g] * (codes_row - z_row[g])
    return d @ G @ d


def test_every_bidup_decision_is_the_best_code_for_its_coordinate():
    """Replays Bid-Up one coordinate at a time and checks each decision against all codes,
    recomputing the whole objective from scratch (no incremental gradient)."""
    W, X = _layer(3, 3, 12, 120)
    bits, gs, r = 2, 4, 2
    res, G = _start(W, X, r, bits, gs)
    Qhat = oracle.dequant(res["codes"], res["scales"], res["zeros"], gs)
    L, R, _ = oracle.olrc(W, Qhat, G, r)
    out = oracle.bidup(W, L, R, res["codes"], res["scales"], res["zeros"], gs, bits, G)
    T = W - R.T @ L.T
    maxq = (1 << bits) - 1
    for o in range(W.shape[0]):
        c = res["codes"][o].astype(np.int64).copy()
        s, z = res["scales"][o], res["zeros"][o].astype(np.float64)
        for j in range(W.shape[1]):
            best = min(range(maxq + 1),
                       key=lambda q: (_loss_of_row(T[o], np.r_[c[:j], q, c[j + 1:]], s, z, gs, G), q))
            losses = [_loss_of_row(T[o], np.r_[c[:j], q, c[j + 1:]], s, z, gs, G) for q in range(maxq + 1)]
            chosen = out["codes"][o, j]
            assert losses[chosen] <= losses[best] * (1 + 1e-12) + 1e-15
            c[j] = chosen
        assert np.array_equal(c, out["codes"][o])
        assert _loss_of_row(T[o], c, s, z, gs, G) == pytest.approx(out["loss_rows"][o], rel=1e-9)


@pytest.mark.parametrize("r,bits,gs", [(0, 3, 8), (2, 2, 8), (4, 3, 0)])
def test_refinement_loss_never_increases(r, bits, gs):
    W, X = _layer(4, 6, 32, 400)
    res, G = _start(W, X, r, bits, gs)
    out = oracle.refine_loop(W, res["codes"], res["scales"], res["zeros"], G, r, bits, gs, iters=4)
    h = out["loss_hist"]
    assert np.all(np.diff(h) <= 1e-12 * h[0])
    # the pass's own L, R are no better than the first OLrC's
    start = oracle.lowrank_loss_rows(W, oracle.dequant(res["codes"], res["scales"], res["zeros"], gs),
                                     res["L"], res["R"], G).sum()
    assert h[0] <= start * (1 + 1e-12)


def test_bidup_fixed_point_admits_no_single_code_improvement():
    W, X = _layer(5, 2, 10, 80)
    bits, gs, r = 2, 5, 1
    res, G = _start(W, X, r, bits, gs)
    Qhat = oracle.dequant(res["codes"], res["scales"], res["zeros"], gs)
    L, R, _ = oracle.olrc(W, Qhat, G, r)
    c = res["codes"]
    for _ in range(50):
        out = oracle.bidup(W, L, R, c, res["scales"], res["zeros"], gs, bits, G)
        c = out["codes"]
        if out["changed"] == 0:
            break
    assert out["changed"] == 0
    T = W - R.T @ L.T
    for o, j, q in itertools.product(range(2), range(10), range(4)):
        s, z = res["scales"][o], res["zeros"][o].astype(np.float64)
        alt = c[o].copy(); alt[j] = q
        assert _loss_of_row(T[o], alt, s, z, gs, G) >= _loss_of_row(T[o], c[o], s, z, gs, G) * (1 - 1e-12)


def _bidup_variant(W, L, R, codes, scales, zeros, gs, bits, G, sign=1.0, propagate=True):
    """The Bid-Up pass with a planted mistake: the step taken the wrong way (sign = -1) or
    code changes not propagated to the later coordinates' gradients."""
    m, n = W.shape
    maxq = (1 << bits) - 1
    c = codes.astype(np.int64).copy()
    T = W - R.T @ L.T
    g_idx = np.arange(n) // gs
    D = T - scales[:, g_idx] * (c - zeros[:, g_idx])
    Gd = D @ G
    for j in range(n):
        s = scales[:, j // gs]
        cn = np.clip(np.rint(c[:, j] + sign * Gd[:, j] / (G[j, j] * s)), 0, maxq).astype(np.int64)
        delta = s * (cn - c[:, j])
        c[:, j] = cn
        if propagate:
            Gd -= np.outer(delta, G[j])
    return c


def test_planted_mistakes_are_caught():
    """Starting far from optimal (random codes), a wrong-way step raises the loss above the
    correct pass's, and a pass that does not propagate its changes takes decisions that the
    brute-force per-coordinate check rejects."""
    W, X = _layer(6, 4, 16, 160)
    bits, gs, r = 2, 8, 2
    res, G = _start(W, X, r, bits, gs)
    Qhat = oracle.dequant(res["codes"], res["scales"], res["zeros"], gs)
    L, R, _ = oracle.olrc(W, Qhat, G, r)
    rnd = np.random.default_rng(9).integers(0, 4, size=res["codes"].shape)
    sc, zr = res["scales"], res["zeros"].astype(np.float64)
    T = W - R.T @ L.T

    def total(cd):
        return sum(_loss_of_row(T[o], cd[o], sc[o], zr[o], gs, G) for o in range(4))

    good = oracle.bidup(W, L, R, rnd, sc, res["zeros"], gs, bits, G)["codes"]
    assert np.array_equal(good, _bidup_variant(W, L, R, rnd, sc, zr, gs, bits, G))
    wrong_way = _bidup_variant(W, L, R, rnd, sc, zr, gs, bits, G, sign=-1.0)
    assert total(good) < total(rnd) < total(wrong_way)
    stale = _bidup_variant(W, L, R, rnd, sc, zr, gs, bits, G, propagate=False)

    def first_bad_decision(cd):
        for o in range(4):
            cur = rnd[o].copy()
            for j in range(16):
                losses = [_loss_of_row(T[o], np.r_[cur[:j], q, cur[j + 1:]], sc[o], zr[o], gs, G)
                          for q in range(4)]
                if losses[cd[o, j]] > min(losses) * (1 + 1e-12) + 1e-15:
                    return (o, j)
                cur[j] = cd[o, j]
        return None

    assert first_bad_decision(good) is None
    assert first_bad_decision(stale) is not None
