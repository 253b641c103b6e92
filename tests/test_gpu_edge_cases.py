"""The grid's degenerate cases on the device, against the fp64 oracle and closed forms.

The per-group min-max grid (GPTQ encyclopedia article, "Technical approach": each group has its
own scale) has cases that random weights never reach:
  * a flat group (every weight equal to zero, e.g. a pruned neuron): the range is widened to
    [-1, 1], so s = 2 / maxq and z = maxq / 2, a tie that either neighbour settles;
  * one-signed groups: xmin = min(0, min w) pins the range at 0 from below (all positive,
    z = 0) or from above (all negative, z = maxq);
  * constant rows, whose codes all sit at the clamp (maxq or 0);
  * weights exactly half a grid step from two codes: round half to even (the deterministic
    tie-break that GPTQ-2D's Theorem 2 asks for). With a power-of-two scale the device's
    fp32 value v = w / s + z is exact, so both sides see the same tie.
With U = I there is no feedback, so every code has a closed form; the second test runs the
same rows through a real factor and judges the device by replay.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_parity import CODE_BAND, check_replay, np64, unpack

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def g():
    import post_weight_quantization_06_b200 as g
    return g


def _edge_rows(n, gs, rng):
    """Rows of W (fp32, each exactly representable): name -> row."""
    rows = {}
    rows["zero"] = np.zeros(n)
    rows["const_pos"] = np.full(n, 0.3)
    rows["const_neg"] = np.full(n, -0.3)
    # exact half steps with s = 1/16, z = 8 at 4 bits: each group holds the range ends -0.5 and
    # 7/16, the other entries sit at (k + 1/2 - 8) / 16 for k = 0 .. 14
    half = np.empty(n)
    for g0 in range(0, n, gs):
        seg = np.array([(k + 0.5 - 8.0) / 16.0 for k in range(15)])
        vals = np.resize(seg, gs)
        vals[0], vals[1] = -0.5, 7.0 / 16.0
        half[g0:g0 + gs] = vals
    rows["half_steps"] = half
    rows["all_pos"] = np.abs(rng.standard_normal(n)) * 0.02 + 1e-3
    rows["all_neg"] = -np.abs(rng.standard_normal(n)) * 0.02 - 1e-3
    out = rng.standard_normal(n) * 0.02
    out[::37] = 0.5                                   # outliers: most codes crowd the middle
    rows["outliers"] = out
    rows["normal"] = rng.standard_normal(n) * 0.02
    return {k: v.astype(np.float32).astype(np.float64) for k, v in rows.items()}


def _run(g, W, U, bits, gs, B=128):
    m, n = W.shape
    G = n // gs if gs else 1
    codes = torch.empty(m, n * bits // 32, dtype=torch.int32, device=DEV)
    scales = torch.empty(m, G, device=DEV)
    zeros = torch.empty(m, G, dtype=torch.uint8, device=DEV)
    loss = torch.empty(m, dtype=torch.float64, device=DEV)
    g.gptq_quantize_layer(torch.from_numpy(W).float().to(DEV),
                          torch.from_numpy(U).float().to(DEV), bits, gs, B, codes, scales,
                          zeros, loss, g.workspace(g.GPTQ_OP_QUANTIZE, m, n, 0, B))
    g.gptq_sync_status()
    return (unpack(codes, bits, n), zeros.cpu().numpy().astype(np.int64), np64(scales),
            loss.cpu().numpy())


def test_degenerate_groups_without_feedback_have_closed_forms(g):
    n, gs, bits = 256, 128, 4
    rows = _edge_rows(n, gs, np.random.default_rng(5))
    names = list(rows)
    W = np.stack([rows[k] for k in names])
    codes, zeros, scales, loss = _run(g, W, np.eye(n), bits, gs)
    rep = check_replay(W, np.eye(n), bits, gs, codes, zeros, scales, label="edge rows, U = I")
    i = {k: names.index(k) for k in names}
    # flat group: range [-1, 1], s = 2/15; z = 7.5 in exact arithmetic, either neighbour
    assert np.allclose(scales[i["zero"]], 2.0 / 15.0, rtol=1e-6)
    assert set(zeros[i["zero"]]) <= {7, 8}
    assert np.array_equal(codes[i["zero"]], np.repeat(zeros[i["zero"]], gs))
    assert loss[i["zero"]] == 0.0
    # one-signed constant rows: all codes at the clamp
    assert np.all(zeros[i["const_pos"]] == 0) and np.all(codes[i["const_pos"]] == 15)
    assert np.all(zeros[i["const_neg"]] == 15) and np.all(codes[i["const_neg"]] == 0)
    assert np.allclose(scales[i["const_pos"]], 0.3 / 15, rtol=1e-6)
    # one-signed random rows: the range is pinned at zero
    assert np.all(zeros[i["all_pos"]] == 0) and np.all(zeros[i["all_neg"]] == 15)
    # exact ties: s = 1/16, z = 8, every tie k + 1/2 goes to the even neighbour
    hs = i["half_steps"]
    assert np.all(scales[hs] == 1.0 / 16.0) and np.all(zeros[hs] == 8)
    v = W[hs] * 16.0 + 8.0
    even = np.where(np.floor(v) % 2 == 0, np.floor(v), np.floor(v) + 1)
    ties = np.abs(v - np.floor(v) - 0.5) == 0
    assert ties.sum() >= n - 4
    assert np.array_equal(codes[hs][ties], even[ties])
    # the oracle agrees everywhere except possibly the flat group's zero-point tie
    assert rep["n_code_mismatch"] == 0 or rep["code_dist"].max() < CODE_BAND


@pytest.mark.parametrize("bits,gs,wdt", [(4, 128, torch.float32), (3, 0, torch.float32),
                                         (2, 64, torch.bfloat16)])
def test_degenerate_rows_through_a_real_factor(g, bits, gs, wdt):
    """The same rows (each repeated with random scalings, plus rows of plain noise) through
    the factor of a correlated Hessian: feedback now moves later columns, so constant rows
    pick up clamped codes and the outlier rows' neighbours are pushed to the range ends.
    Judged by replay: every differing decision must be within 1e-3 steps of a tie."""
    n, m = 512, 96
    rng = np.random.default_rng(7 + bits)
    base = _edge_rows(n, gs if gs else 128, rng)
    W = []
    for r in range(m):
        k = list(base)[r % len(base)]
        W.append(base[k] * (1.0 if r < len(base) else rng.uniform(0.5, 2.0)))
    W = np.stack(W)
    Wt = torch.from_numpy(W).float().to(DEV).to(wdt)
    W = np64(Wt)
    Q, _ = np.linalg.qr(rng.standard_normal((n, n)))
    X = rng.standard_normal((4 * n, n)) @ ((np.arange(1, n + 1) ** -0.6)[:, None] * Q.T)
    Hd, _ = oracle.damp(oracle.hessian(X), 0.01)
    U32 = np.ascontiguousarray(oracle.inverse_cholesky_upper(Hd).astype(np.float32))
    m_, n_ = W.shape
    G = n // gs if gs else 1
    codes = torch.empty(m_, n * bits // 32, dtype=torch.int32, device=DEV)
    scales = torch.empty(m_, G, device=DEV)
    zeros = torch.empty(m_, G, dtype=torch.uint8, device=DEV)
    loss = torch.empty(m_, dtype=torch.float64, device=DEV)
    g.gptq_quantize_layer(Wt, torch.from_numpy(U32).to(DEV), bits, gs, 128, codes, scales,
                          zeros, loss, g.workspace(g.GPTQ_OP_QUANTIZE, m_, n_, 0, 128))
    g.gptq_sync_status()
    c = unpack(codes, bits, n)
    maxq = (1 << bits) - 1
    clamped = ((c == 0) | (c == maxq)).mean()
    print(f"edge rows b{bits} g{gs}: {clamped:.1%} of codes at 0 or maxq")
    check_replay(W, U32.astype(np.float64), bits, gs, c, zeros.cpu().numpy().astype(np.int64),
                 np64(scales), loss_gpu=loss.cpu().numpy(), label=f"edge rows b{bits} g{gs}")
