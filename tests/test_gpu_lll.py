"""GPTQ with lattice basis reduction on the device (gptq_quantize_layer_reduced) against the fp64
oracle (The Lattice Geometry of Neural Network Quantization, section 5.2).

The oracle gets the device's Hessian (its own error is judged by the Hessian tests). Judged:
  * LLL: the same number of swaps and size reductions and the same largest entry of T, T^-1
    (the device and the oracle take the same decisions);
  * the per-channel grid: scales to 1e-6, zero-points exact (a tie may go either way);
  * the rounding in the reduced basis, replayed: every coefficient that differs from the
    oracle's rounding along the device's own trajectory lies within 1e-3 of a tie;
  * codes = clip(T c') exactly, the count of clipped codes, and the loss for those codes;
  * against the free-running oracle: codes >= 99.9 % equal, loss within 0.5 %.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from gpu_parity import CODE_AGREE, CODE_BAND, REL_LOSS, np64, unpack

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def g():
    import post_weight_quantization_06_b200 as g
    return g


def _case(name):
    if name == "tiny":
        L = datagen.tiny(device=DEV)
    else:
        L = datagen.deit("fc1", device=DEV)
    return L


@pytest.mark.parametrize("name,bits", [("tiny", 4), ("tiny", 2), ("deit_fc1", 2)])
def test_reduced_matches_oracle(g, name, bits):
    L = _case(name)
    n = L.n
    H = torch.zeros(n, n, device=DEV)
    g.gptq_hessian_accumulate(H, L.X)
    out = g.quantize_layer_reduced(L.W, H, bits=bits, lambda_rel=L.lambda_rel)
    Hd = np64(H)
    W = np64(L.W)
    m = W.shape[0]
    maxq = (1 << bits) - 1
    ref = oracle.withreduction(W, Hd, bits, L.lambda_rel)
    stats = out["stats"].cpu().numpy()
    T = ref["T"]
    Ti = np.rint(np.linalg.inv(T))
    print(f"{name} b{bits}: swaps {stats[0]} (oracle {ref['stats']['swaps']}), size reductions "
          f"{stats[1]} (oracle {ref['stats']['reductions']}), max |T| {stats[3]}, clipped {stats[4]}")
    assert stats[0] == ref["stats"]["swaps"] and stats[1] == ref["stats"]["reductions"]
    assert stats[3] == max(np.abs(T).max(), np.abs(Ti).max())
    s = np64(out["scales"])
    z = out["zeros"].cpu().numpy().astype(np.float64)
    assert np.abs(s - ref["scales"]).max() / np.abs(ref["scales"]).max() <= 1e-6
    assert np.array_equal(z, ref["zeros"])
    # the device's decisions in the reduced basis, replayed along their own trajectory
    coef = out["coef"].cpu().numpy().astype(np.float64)
    U = W / s[:, None] + z[:, None]
    _, V = oracle.round_in_basis(U @ Ti.T, ref["G_red"], force=coef)
    own = np.rint(V)
    bad = own != coef
    if bad.any():
        lo = np.minimum(own, coef)[bad]
        dist = np.where(np.abs(own - coef)[bad] == 1, np.abs(V[bad] - (lo + 0.5)), np.inf)
        print(f"{name} b{bits}: {int(bad.sum())} of {bad.size} reduced-basis decisions differ, "
              f"worst {dist.max():.2e} from a tie")
        assert bad.mean() <= 1 - CODE_AGREE and dist.max() < CODE_BAND
    raw = coef @ T.T
    codes = unpack(out["codes"], bits, n)
    assert np.array_equal(codes, np.clip(raw, 0, maxq))
    assert stats[4] == int((np.clip(raw, 0, maxq) != raw).sum())
    D = W - s[:, None] * (codes - z[:, None])
    Hdamp = Hd + ref["lam"] * np.eye(n)
    loss_ref = np.einsum("ij,jk,ik->i", D, Hdamp, D)
    lrel = abs(out["loss"].cpu().numpy().sum() - loss_ref.sum()) / loss_ref.sum()
    assert lrel <= 1e-4
    # against the free-running oracle
    agree = (codes == ref["codes"]).mean()
    lfree = abs(loss_ref.sum() - ref["loss_rows"].sum()) / ref["loss_rows"].sum()
    print(f"{name} b{bits}: codes agree {agree:.6f} with the free-running oracle, loss rel "
          f"{lfree:.2e}; loss with reduction / plain GPTQ per channel: see the bench")
    assert agree >= CODE_AGREE and lfree <= REL_LOSS
