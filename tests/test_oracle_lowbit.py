"""Pins of the low-precision L / R oracle (GPTQ-intrinsic LoRA summary, "Main results")."""
import numpy as np
import pytest

import oracle


@pytest.mark.parametrize("bits,gs", [(4, 16), (8, 0), (3, 8)])
def test_every_code_is_the_nearest_grid_point(bits, gs):
    A = np.random.default_rng(bits).standard_normal((7, 48)) * np.exp(np.linspace(-3, 2, 48))
    q = oracle.rtn_quantize(A, bits, gs)
    g = np.arange(48) // (gs if gs else 48)
    maxq = (1 << bits) - 1
    for i in range(7):
        for j in range(48):
            s, z = q["scales"][i, g[j]], q["zeros"][i, g[j]]
            grid = s * (np.arange(maxq + 1) - z)
            best = np.argmin(np.abs(A[i, j] - grid))
            assert abs(A[i, j] - grid[q["codes"][i, j]]) <= abs(A[i, j] - grid[best]) + 1e-15
    inside = (q["codes"] > 0) & (q["codes"] < maxq)
    err = np.abs(A - q["deq"])
    assert np.all(err[inside] <= 0.5 * q["scales"][:, g][inside] * (1 + 1e-12))


def test_requantizing_is_idempotent():
    A = np.random.default_rng(3).standard_normal((5, 32))
    q = oracle.rtn_quantize(A, 4, 16)
    g = np.arange(32) // 16
    v = q["deq"] / q["scales"][:, g] + q["zeros"][:, g]
    assert np.array_equal(np.clip(np.rint(v), 0, 15).astype(np.int64), q["codes"])


def test_grid_of_the_low_rank_factors_matches_the_layer_rule():
    """The factors go through minmax_grid exactly as a layer row does (pinned by the golden
    grid rows); a planted transposition (L quantized as stored, n rows of r) is caught."""
    rng = np.random.default_rng(4)
    L = rng.standard_normal((64, 8))
    R = rng.standard_normal((8, 32))
    out = oracle.quantize_lowrank(L, R, bits_L=4, group_size_L=16, bits_R=8)
    s, z, _ = oracle.minmax_grid(L.T[:, :16], 15)
    assert np.allclose(out["L"]["scales"][:, 0], s) and np.array_equal(out["L"]["zeros"][:, 0], z)
    s2, z2, _ = oracle.minmax_grid(R.T, 255)
    assert np.allclose(out["R"]["scales"][:, 0], s2)
    assert out["L_hat"].shape == L.shape and out["R_hat"].shape == R.shape
    wrong = oracle.rtn_quantize(L, 4, 16)["deq"]   # n rows of r: a different grouping
    assert not np.allclose(wrong, out["L_hat"])
    assert np.abs(out["R_hat"] - R).max() <= 0.5 * out["R"]["scales"].max() * (1 + 1e-12)
    assert np.array_equal(oracle.unpack_codes(out["packed_L"], 4, 64), out["L"]["codes"])
