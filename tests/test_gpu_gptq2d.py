"""Two-sided adaptive rounding (GPTQ-2D) on the GPU against the fp64 oracle.

Small and ragged shapes: the device's Z is replayed through the oracle's anti-diagonal sweep
(decisions forced to the device's); every decision the oracle would take differently must sit
within CODE_BAND of a rounding boundary, and the errors agree to 1e-3 of their range.
Full size: the closed form X - Z = U_G^T E U_H gives every decision's residual from Z alone;
all must lie in [-1/2, 1/2] up to CODE_BAND (the Babai point of the Kronecker basis is the
only integer matrix with that property)."""
import os

import numpy as np
import pytest
import torch

import datagen
import oracle
from gpu_parity import CODE_AGREE, CODE_BAND, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def g():
    import post_weight_quantization_06_b200 as lib
    return lib


@pytest.fixture
def band(monkeypatch):
    def set_band(w):
        if w is None:
            monkeypatch.delenv("GPTQ_2D_BAND", raising=False)
        else:
            monkeypatch.setenv("GPTQ_2D_BAND", str(w))
    return set_band


def _judge(P, out, label):
    X, G, H = np64(P.X), np64(P.G), np64(P.H)
    Zg = out["Z"].cpu().numpy().astype(np.int64)
    rep = oracle.gptq2d_antidiagonal(X, G, H, force_Z=Zg)
    free = np.rint(rep["v"]).astype(np.int64)
    mism = free != Zg
    agree = 1.0 - mism.sum() / Zg.size
    dist = np.abs(np.abs(rep["v"][mism] - Zg[mism]) - 0.5) if mism.any() else np.zeros(0)
    worst = float(dist.max()) if dist.size else 0.0
    eg = np64(out["err"])
    erel = float(np.abs(eg - rep["E"]).max() / max(np.abs(rep["E"]).max(), 1e-30))
    print(f"{label}: Z agree {agree:.6f} ({int(mism.sum())}/{Zg.size} differ, worst distance "
          f"{worst:.2e}), err max rel diff {erel:.2e}")
    assert agree >= CODE_AGREE
    assert worst < CODE_BAND
    assert erel <= 1e-3
    return Zg, rep


@pytest.mark.parametrize("m,n,w", [(70, 100, None), (70, 100, 1), (160, 224, 3), (257, 130, 4),
                                   (33, 33, 2), (96, 64, 16)])
def test_2d_round_matches_the_oracle(g, band, m, n, w):
    band(w)
    P = datagen.two_sided(m, n, device=DEV, seed=11 + m)
    out = g.round_2d(P.X, P.G, P.H, with_err=True)
    Zg, rep = _judge(P, out, f"2d {m}x{n} band {w}")
    free = oracle.gptq2d_antidiagonal(np64(P.X), np64(P.G), np64(P.H))["Z"]
    print(f"  free-running oracle Z differs in {int((free != Zg).sum())} entries")


@pytest.mark.parametrize("m,n", [(1, 300), (300, 1), (1, 1), (31, 65)])
def test_2d_round_thin_and_ragged(g, m, n):
    """One row or one column: the problem is the one-sided sweep of a vector."""
    P = datagen.two_sided(m, n, device=DEV, seed=3)
    out = g.round_2d(P.X, P.G, P.H, with_err=True)
    _judge(P, out, f"2d {m}x{n}")


def test_2d_round_with_diagonal_grams_is_rint(g):
    """Orthogonal bases: no feedback reaches another entry, Z = rint(X) exactly."""
    m, n = 50, 90
    gen = torch.Generator(device=DEV).manual_seed(7)
    X = torch.randn(m, n, device=DEV, generator=gen) * 4
    G = torch.diag(torch.rand(m, device=DEV, generator=gen) + 0.5)
    H = torch.diag(torch.rand(n, device=DEV, generator=gen) + 0.5)
    out = g.round_2d(X, G, H, with_err=True)
    assert torch.equal(out["Z"], torch.round(X).to(torch.int32))


def test_2d_round_reports_an_indefinite_gram(g):
    P = datagen.two_sided(40, 64, device=DEV, seed=9)
    H = P.H.clone()
    H[5, 5] = -1.0
    with pytest.raises(g.GptqError) as ex:
        g.round_2d(P.X, P.G, H)
    assert ex.value.status == g.GPTQ_ERR_NOT_PD


def test_2d_round_empty(g):
    for m, n in ((0, 5), (5, 0)):
        X = torch.empty(m, n, device=DEV)
        out = g.round_2d(X, torch.eye(m, device=DEV), torch.eye(n, device=DEV))
        assert out["Z"].shape == (m, n)


def test_2d_round_full_size_residuals(g, band):
    """2048 x 6144 (the mlp_down shape): every decision checked through the closed form."""
    band(None)
    P = datagen.two_sided(device=DEV)
    out = g.round_2d(P.X, P.G, P.H)
    Zg = out["Z"].cpu().numpy()
    c = oracle.gptq2d_residuals(np64(P.X), Zg, np64(P.G), np64(P.H))
    over = np.abs(c) - 0.5
    n_out = int((over > 0).sum())
    print(f"2d full size {P.X.shape[0]}x{P.X.shape[1]}: max |c| {np.abs(c).max():.6f}, "
          f"{n_out}/{c.size} decisions beyond 1/2, worst {max(over.max(), 0):.2e}")
    assert over.max() < CODE_BAND
    assert 1.0 - n_out / c.size >= CODE_AGREE
