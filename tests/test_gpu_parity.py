"""CUDA path vs the fp64 oracle, through the C ABI, on seeded synthetic layers.

Stage tests feed each entry point the oracle's own inputs (H, U) so that one kernel family
is judged at a time; end-to-end tests run the whole pass from X and W.
"""
import ctypes

import numpy as np
import pytest
import torch

import datagen
import oracle
from gpu_parity import (CODE_BAND, REL_H, REL_LOSS, REL_SCALE, check_replay, np64, rel_fro,
                        unpack)

pytestmark = pytest.mark.gpu
DEV = "cuda"
EPS32 = 2.0 ** -24


@pytest.fixture(scope="module")
def g():
    import post_weight_quantization_06_b200 as g
    return g


def _rng(seed):
    return np.random.default_rng(seed)


def _spd_from_data(n, k, seed, decay=0.5):
    r = _rng(seed)
    Q, _ = np.linalg.qr(r.standard_normal((n, n)))
    X = r.standard_normal((k, n)) @ ((np.arange(1, n + 1) ** -decay)[:, None] * Q.T)
    return X


# ----------------------------------------------------------------------------- Hessian

def test_hessian_fp32_tiny_workload(g):
    L = datagen.tiny(device=DEV)
    H = torch.zeros(L.n, L.n, device=DEV)
    g.gptq_hessian_accumulate(H, L.X)
    g.gptq_sync_status()
    Href = oracle.hessian(np64(L.X))
    err = rel_fro(np64(H), Href)
    print(f"tiny fp32 H rel err {err:.2e}")
    assert err <= REL_H
    assert torch.equal(H, H.t())


@pytest.mark.parametrize("n,k,chunks", [(200, 1000, 1), (1024, 4096, 2), (384, 33000, 3),
                                        (136, 77, 1), (768, 16384, 1)])
def test_hessian_bf16(g, n, k, chunks):
    X = torch.from_numpy(_spd_from_data(n, k, n + k)).float().to(DEV).to(torch.bfloat16)
    H = torch.zeros(n, n, device=DEV)
    bounds = np.linspace(0, k, chunks + 1).astype(int)
    for a, b in zip(bounds[:-1], bounds[1:]):
        g.gptq_hessian_accumulate(H, X[a:b].contiguous())
    g.gptq_sync_status()
    Href = oracle.hessian(np64(X))
    err = rel_fro(np64(H), Href)
    print(f"bf16 H n={n} k={k}: rel err {err:.2e}")
    assert err <= REL_H
    assert torch.equal(H, H.t())


@pytest.mark.parametrize("n,k", [(512, 20000), (1536, 65536)])
def test_hessian_tensor_core_path_is_tighter_than_fp32_chain(g, n, k, monkeypatch):
    """bf16 X with n % 8 == 0 runs on tcgen05 with two-level chunk sums; the SIMT path
    (forced by GPTQ_FORCE_SIMT_HESSIAN) is a plain fp32 chain. Both against the oracle."""
    X = torch.from_numpy(_spd_from_data(n, k, 3 * n)).float().to(DEV).to(torch.bfloat16)
    Href = oracle.hessian(np64(X))
    H_tc = torch.zeros(n, n, device=DEV)
    g.gptq_hessian_accumulate(H_tc, X)
    g.gptq_sync_status()
    monkeypatch.setenv("GPTQ_FORCE_SIMT_HESSIAN", "1")
    H_simt = torch.zeros(n, n, device=DEV)
    g.gptq_hessian_accumulate(H_simt, X)
    g.gptq_sync_status()
    e_tc, e_simt = rel_fro(np64(H_tc), Href), rel_fro(np64(H_simt), Href)
    print(f"H n={n} k={k}: tensor-core rel err {e_tc:.2e}, SIMT rel err {e_simt:.2e}")
    assert torch.equal(H_tc, H_tc.t())
    assert e_tc <= REL_H and e_tc <= e_simt


@pytest.mark.parametrize("n,k,chunks", [(512, 20000, 2), (1000, 3000, 1), (136, 777, 1)])
def test_hessian_fp32_x_on_tensor_cores(g, n, k, chunks, monkeypatch):
    """fp32 X with n % 4 == 0 runs on the fp32-accurate tensor-core product (tf32 x 3) over the
    upper triangle (n = 136 is small enough to take the SIMT kernel inside it); the forced SIMT
    path is a plain fp32 chain. Both against the oracle, chunks additive."""
    X = torch.from_numpy(_spd_from_data(n, k, 5 * n + k)).float().to(DEV)
    Href = oracle.hessian(np64(X))
    bounds = np.linspace(0, k, chunks + 1).astype(int)
    H_tc = torch.zeros(n, n, device=DEV)
    for a, b in zip(bounds[:-1], bounds[1:]):
        g.gptq_hessian_accumulate(H_tc, X[a:b].contiguous())
    g.gptq_sync_status()
    monkeypatch.setenv("GPTQ_FORCE_SIMT_HESSIAN", "1")
    H_simt = torch.zeros(n, n, device=DEV)
    g.gptq_hessian_accumulate(H_simt, X)
    g.gptq_sync_status()
    e_tc, e_simt = rel_fro(np64(H_tc), Href), rel_fro(np64(H_simt), Href)
    print(f"fp32 X n={n} k={k}: tensor-core rel err {e_tc:.2e}, SIMT rel err {e_simt:.2e}")
    assert torch.equal(H_tc, H_tc.t())
    assert e_tc <= REL_H and e_simt <= REL_H


def test_hessian_bounded_wait_reports_timeout_and_device_stays_usable(g, monkeypatch):
    """A wait that nothing will ever satisfy (test hook) gives up after the limit, reports
    GPTQ_ERR_TIMEOUT through the status word, and the next call works normally."""
    n, k = 256, 4096
    X = torch.from_numpy(_spd_from_data(n, k, 11)).float().to(DEV).to(torch.bfloat16)
    monkeypatch.setenv("GPTQ_TEST_STALL", "1")
    monkeypatch.setenv("GPTQ_WAIT_LIMIT_CYCLES", "2000000")
    H = torch.zeros(n, n, device=DEV)
    g.gptq_hessian_accumulate(H, X)
    st, info = g.gptq_sync_status(raise_on_error=False)
    assert st == g.GPTQ_ERR_TIMEOUT and info in (1, 2, 3, 4, 5, 6, 7)
    monkeypatch.delenv("GPTQ_TEST_STALL")
    monkeypatch.delenv("GPTQ_WAIT_LIMIT_CYCLES")
    H.zero_()
    g.gptq_hessian_accumulate(H, X)
    g.gptq_sync_status()
    assert rel_fro(np64(H), oracle.hessian(np64(X))) <= REL_H


# ----------------------------------------------------------------------------- factor

# n = 1000: the factor's tensor-core updates have widths that are not multiples of 32 (their
# last 32-column slices cross the matrix edge)
@pytest.mark.parametrize("n,k,lam", [(256, 512, 0.01), (300, 2000, 0.01), (1024, 4096, 0.01),
                                     (129, 400, 0.1), (1000, 3000, 0.01)])
def test_prepare_hinv_matches_oracle(g, n, k, lam):
    X = _spd_from_data(n, k, 7 * n)
    H32 = oracle.hessian(X).astype(np.float32)
    Hd, lam_ref = oracle.damp(H32.astype(np.float64), lam)
    Uref = oracle.inverse_cholesky_upper(Hd)
    H = torch.from_numpy(H32).to(DEV)
    U = torch.empty(n, n, device=DEV)
    lam_t = torch.empty(1, device=DEV)
    ws = g.workspace(g.GPTQ_OP_PREPARE_HINV, 0, n)
    g.gptq_prepare_hinv(H, lam, U, lam_t, ws)
    g.gptq_sync_status()
    Ug = np64(U)
    assert abs(lam_t.item() - lam_ref) / lam_ref < 1e-6
    assert np.all(np.tril(Ug, -1) == 0)
    ev = np.linalg.eigvalsh(Hd)
    kappa = ev[-1] / ev[0]
    err = rel_fro(Ug, Uref)
    resid = np.abs(Ug.T @ Ug @ Hd - np.eye(n)).max()
    # fp32 factorization: forward error grows like kappa * unit roundoff (a factor of
    # sqrt(n) covers the accumulation length of the blocked updates)
    bound = kappa * EPS32 * np.sqrt(n)
    print(f"U n={n}: kappa {kappa:.1e}, rel err {err:.2e} (bound {bound:.2e}), "
          f"max|U^T U H - I| {resid:.2e}")
    assert err <= bound
    assert np.allclose(np.diag(Ug), np.diag(Uref), rtol=bound)


def test_prepare_hinv_reports_non_positive_pivot(g):
    n = 200
    h = np.eye(n, dtype=np.float32)
    h[150, 150] = -1.0
    U = torch.empty(n, n, device=DEV)
    lam_t = torch.empty(1, device=DEV)
    ws = g.workspace(g.GPTQ_OP_PREPARE_HINV, 0, n)
    g.gptq_prepare_hinv(torch.from_numpy(h).to(DEV), 0.0, U, lam_t, ws)
    st, info = g.gptq_sync_status(raise_on_error=False)
    assert st == g.GPTQ_ERR_NOT_PD and info == 150
    assert g.gptq_sync_status() == (0, 0)   # cleared


def test_sync_status_flag_returns_device_errors_from_the_call(g):
    """GPTQ_FLAG_SYNC_STATUS: the failing call itself returns GPTQ_ERR_NOT_PD; a clean call
    returns GPTQ_OK; with the flag cleared the error waits for gptq_sync_status again."""
    n = 200
    h = np.eye(n, dtype=np.float32)
    h[150, 150] = -1.0
    bad, good = torch.from_numpy(h).to(DEV), torch.eye(n, device=DEV)
    U = torch.empty(n, n, device=DEV)
    lam_t = torch.empty(1, device=DEV)
    ws = g.workspace(g.GPTQ_OP_PREPARE_HINV, 0, n)
    lib = g._lib
    args = lambda H: (ctypes.c_void_p(H.data_ptr()), n, ctypes.c_float(0.0),
                      ctypes.c_void_p(U.data_ptr()), ctypes.c_void_p(lam_t.data_ptr()),
                      ctypes.c_void_p(ws.data_ptr()), ws.numel(), g._stream())
    try:
        g.gptq_set_flags(g.GPTQ_FLAG_SYNC_STATUS)
        assert lib.gptq_prepare_hinv(*args(bad)) == g.GPTQ_ERR_NOT_PD
        assert lib.gptq_prepare_hinv(*args(good)) == g.GPTQ_OK
        g.gptq_set_flags(g.GPTQ_FLAG_DEBUG_CHECKS)
        assert lib.gptq_prepare_hinv(*args(bad)) == g.GPTQ_ERR_NOT_PD
    finally:
        g.gptq_set_flags(0)
    assert lib.gptq_prepare_hinv(*args(bad)) == g.GPTQ_OK
    st, info = g.gptq_sync_status(raise_on_error=False)
    assert st == g.GPTQ_ERR_NOT_PD and info == 150


def test_prepare_hinv_reports_nonfinite_diagonal(g):
    n = 64
    h = np.eye(n, dtype=np.float32)
    h[5, 5] = np.nan
    U = torch.empty(n, n, device=DEV)
    lam_t = torch.empty(1, device=DEV)
    ws = g.workspace(g.GPTQ_OP_PREPARE_HINV, 0, n)
    g.gptq_prepare_hinv(torch.from_numpy(h).to(DEV), 0.01, U, lam_t, ws)
    st, info = g.gptq_sync_status(raise_on_error=False)
    assert st == g.GPTQ_ERR_NONFINITE and info == 5 * n + 5


# ----------------------------------------------------------------------------- sweep

SWEEP_CASES = [
    # m, n, bits, group, block, W dtype
    (200, 256, 4, 128, 128, torch.float32),
    (96, 512, 3, 32, 128, torch.bfloat16),
    (64, 384, 2, 0, 128, torch.float32),
    (70, 512, 4, 256, 128, torch.float32),
    (50, 256, 3, 64, 64, torch.float32),
    (33, 256, 4, 16, 32, torch.float32),
    (17, 128, 8, 128, 128, torch.float32),
    # odd widths: codes straddle 32-bit words
    (48, 256, 5, 64, 64, torch.float32),
    (40, 512, 6, 128, 128, torch.bfloat16),
    (36, 256, 7, 32, 32, torch.float32),
    # groups shorter than the column loop's 16-column slots: boundaries inside a slot
    (40, 256, 4, 8, 64, torch.float32),
    (24, 128, 3, 4, 32, torch.float32),
    (20, 256, 2, 2, 128, torch.bfloat16),
    # 300 rows: the tensor-core lazy updates' last 32-row slices cross the matrix edge
    (300, 640, 4, 128, 128, torch.float32),
    # several 1024-column outer blocks of the two-level lazy update
    (64, 2560, 3, 128, 128, torch.bfloat16),
    (40, 2048, 4, 0, 128, torch.float32),
    (24, 3072, 2, 96, 32, torch.float32),
]


@pytest.mark.parametrize("m,n,bits,gs,B,wdt", SWEEP_CASES)
def test_quantize_stage_matches_oracle(g, m, n, bits, gs, B, wdt):
    """The sweep alone: the device gets the oracle's U (rounded to fp32) and the replay
    uses the same fp32 values."""
    X = _spd_from_data(n, 4 * n, m + n + bits)
    Hd, _ = oracle.damp(oracle.hessian(X), 0.01)
    U32 = np.ascontiguousarray(oracle.inverse_cholesky_upper(Hd).astype(np.float32))
    W = torch.from_numpy(_rng(m * n).standard_normal((m, n)) * 0.02).float().to(DEV).to(wdt)
    G = n // gs if gs else 1
    codes = torch.empty(m, n * bits // 32, dtype=torch.int32, device=DEV)
    scales = torch.empty(m, G, device=DEV)
    zeros = torch.empty(m, G, dtype=torch.uint8, device=DEV)
    loss = torch.empty(m, dtype=torch.float64, device=DEV)
    ws = g.workspace(g.GPTQ_OP_QUANTIZE, m, n, 0, B)
    g.gptq_quantize_layer(W, torch.from_numpy(U32).to(DEV), bits, gs, B, codes, scales, zeros,
                          loss, ws)
    g.gptq_sync_status()
    rep = check_replay(np64(W), U32.astype(np.float64), bits, gs, unpack(codes, bits, n),
                       zeros.cpu().numpy().astype(np.int64), np64(scales),
                       loss_gpu=loss.cpu().numpy(), label=f"sweep {m}x{n} b{bits} g{gs} B{B}")
    # zero-points as reals, along the same trajectory
    zr = rep["zeros_real"]
    assert np.all(np.abs(zeros.cpu().numpy() - zr) <= 0.5 + CODE_BAND)


def test_quantize_with_unaligned_factor_rows_is_identical(g):
    """U starting 4 bytes past a 16-byte boundary takes the column loop's plain-load path for
    its U blocks; the result must equal the cp.async path's bit for bit."""
    m, n, bits, gs, B = 48, 512, 4, 128, 128
    X = _spd_from_data(n, 4 * n, 7)
    Hd, _ = oracle.damp(oracle.hessian(X), 0.01)
    U32 = torch.from_numpy(np.ascontiguousarray(oracle.inverse_cholesky_upper(Hd).astype(np.float32))).to(DEV)
    buf = torch.empty(n * n + 1, device=DEV)
    Umis = buf[1:].view(n, n)
    Umis.copy_(U32)
    assert Umis.data_ptr() % 16 == 4
    W = torch.from_numpy(_rng(3).standard_normal((m, n)) * 0.02).float().to(DEV)
    outs = []
    for U in (U32, Umis):
        codes = torch.empty(m, n * bits // 32, dtype=torch.int32, device=DEV)
        scales = torch.empty(m, n // gs, device=DEV)
        zeros = torch.empty(m, n // gs, dtype=torch.uint8, device=DEV)
        loss = torch.empty(m, dtype=torch.float64, device=DEV)
        g.gptq_quantize_layer(W, U, bits, gs, B, codes, scales, zeros, loss,
                              g.workspace(g.GPTQ_OP_QUANTIZE, m, n, 0, B))
        g.gptq_sync_status()
        outs.append((codes, scales, zeros, loss))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_quantize_reports_nonfinite_weight(g):
    m, n = 8, 128
    W = torch.zeros(m, n, device=DEV)
    W[3, 17] = float("inf")
    U = torch.eye(n, device=DEV)
    codes = torch.empty(m, n * 4 // 32, dtype=torch.int32, device=DEV)
    scales = torch.empty(m, 1, device=DEV)
    zeros = torch.empty(m, 1, dtype=torch.uint8, device=DEV)
    ws = g.workspace(g.GPTQ_OP_QUANTIZE, m, n, 0, 128)
    g.gptq_quantize_layer(W, U, 4, 128, 128, codes, scales, zeros, None, ws)
    st, info = g.gptq_sync_status(raise_on_error=False)
    assert st == g.GPTQ_ERR_NONFINITE and info == 3 * n + 17


def test_quantize_is_deterministic(g):
    L = datagen.attn(device=DEV, scale=0.25)
    a = g.quantize_layer(L.W, L.X, bits=4, group_size=128, lambda_rel=0.01)
    b = g.quantize_layer(L.W, L.X, bits=4, group_size=128, lambda_rel=0.01)
    for key in ("H", "U", "codes", "scales", "zeros", "loss"):
        assert torch.equal(a[key], b[key]), key


# ----------------------------------------------------------------------------- end to end

def _dequant(codes, scales, zeros, bits, gs, n):
    gl = gs if gs else n
    s = np.repeat(scales, gl, axis=1)[:, :n]
    z = np.repeat(zeros.astype(np.float64), gl, axis=1)[:, :n]
    return s * (codes - z)


def _e2e_plain(g, L, rows=None):
    out = g.quantize_layer(L.W, L.X, bits=L.bits, group_size=L.group_size,
                           lambda_rel=L.lambda_rel, block_size=L.block_size)
    X = np64(L.X)
    Href = oracle.hessian(X)
    del X
    herr = rel_fro(np64(out["H"]), Href)
    print(f"{L.name}: H rel err {herr:.2e}")
    assert herr <= REL_H
    Hd, lam = oracle.damp(Href, L.lambda_rel)
    assert abs(out["lam"].item() - lam) / lam < 1e-4
    U = oracle.inverse_cholesky_upper(Hd)
    W = np64(L.W)
    m, n = W.shape
    rows = np.arange(m) if rows is None else rows
    codes = unpack(out["codes"], L.bits, n)[rows]
    zeros = out["zeros"].cpu().numpy().astype(np.int64)[rows]
    scales = np64(out["scales"])[rows]
    loss = out["loss"].cpu().numpy()[rows]
    check_replay(W[rows], U, L.bits, L.group_size, codes, zeros, scales, loss_gpu=loss,
                 label=L.name)
    free = oracle.sweep(W[rows], U, L.bits, L.group_size)
    lr = abs(loss.sum() - free["loss_rows"].sum()) / free["loss_rows"].sum()
    Wq = _dequant(codes, scales, zeros, L.bits, L.group_size, n)
    dl_gpu = oracle.data_loss_rows(W[rows], Wq, Href / 2).sum()
    dl_ref = oracle.data_loss_rows(W[rows], free["Wq"], Href / 2).sum()
    dr = abs(dl_gpu - dl_ref) / dl_ref
    print(f"{L.name}: regularised loss rel err {lr:.2e}, data loss rel err {dr:.2e}")
    assert lr <= REL_LOSS and dr <= REL_LOSS


def test_e2e_tiny(g):
    _e2e_plain(g, datagen.tiny(device=DEV))


def test_e2e_attn(g):
    _e2e_plain(g, datagen.attn(device=DEV))


def test_e2e_deit_fc1(g):
    _e2e_plain(g, datagen.deit("fc1", device=DEV), rows=np.arange(0, 3072, 6))


def test_e2e_deit_fc2(g):
    _e2e_plain(g, datagen.deit("fc2", device=DEV), rows=np.arange(0, 768, 4))


def test_e2e_mlp_down_quarter(g):
    _e2e_plain(g, datagen.mlp_down(device=DEV, scale=0.25), rows=np.arange(0, 512, 2))


# ----------------------------------------------------------------------------- intrinsic LoRA

def _e2e_il(g, L, rows=None):
    out = g.quantize_layer(L.W, L.X, bits=L.bits, group_size=L.group_size,
                           lambda_rel=L.lambda_rel, block_size=L.block_size, r=L.r)
    X = np64(L.X)
    Href = oracle.hessian(X)
    del X
    assert rel_fro(np64(out["H"]), Href) <= REL_H
    G = Href / 2
    V, _ = oracle.top_singular_directions(G, L.r)
    Lg = np64(out["L"])
    verr = np.abs(Lg - V).max() / np.abs(V).max()
    Ht, lam = oracle.il_hessian(G, V, L.lambda_rel)
    lerr = abs(out["lam"].item() - lam) / lam
    print(f"{L.name}: L max rel err {verr:.2e}, lambda~ rel err {lerr:.2e}")
    assert verr <= REL_SCALE and lerr <= 1e-4
    Ut = oracle.eig_qr_factor(Ht)
    W = np64(L.W)
    m, n = W.shape
    rows = np.arange(m) if rows is None else rows
    Wt = np.hstack([W[rows], np.zeros((len(rows), L.r))])
    codes = unpack(out["codes"], L.bits, n)[rows]
    zeros = out["zeros"].cpu().numpy().astype(np.int64)[rows]
    scales = np64(out["scales"])[rows]
    loss = out["loss"].cpu().numpy()[rows]
    Rg = np64(out["R"])[:, rows].T
    check_replay(Wt, Ut[:n], L.bits, L.group_size, codes, zeros, scales, loss_gpu=loss,
                 n_quant=n, extra_gpu=Rg, label=L.name)
    free = oracle.sweep(Wt, Ut[:n], L.bits, L.group_size, n_quant=n)
    lr = abs(loss.sum() - free["loss_rows"].sum()) / free["loss_rows"].sum()
    print(f"{L.name}: loss rel err vs free-running oracle {lr:.2e}")
    assert lr <= REL_LOSS


def test_il_lowrank_quarter(g):
    _e2e_il(g, datagen.lowrank(device=DEV, scale=0.25), rows=np.arange(0, 512, 2))


def test_il_small_rank(g):
    L = datagen.lowrank(device=DEV, scale=0.125, r=8)
    _e2e_il(g, L)


def test_il_odd_rank(g):
    """r = 5: the augmented rows (n + r floats) are not 16-byte multiples, so every product and
    the column loop take their unaligned paths."""
    _e2e_il(g, datagen.lowrank(device=DEV, scale=0.125, r=5))


def test_il_r0_equals_plain(g):
    L = datagen.attn(device=DEV, scale=0.25)
    a = g.quantize_layer(L.W, L.X, bits=4, group_size=128, lambda_rel=0.01)
    b = g.quantize_layer(L.W, None, H=a["H"], bits=4, group_size=128, lambda_rel=0.01, r=0,
                         intrinsic=True)
    b2 = g.quantize_layer(L.W, None, H=a["H"], bits=4, group_size=128, lambda_rel=0.01, r=0,
                          intrinsic=True)
    for key in ("codes", "scales", "zeros", "loss", "lam"):
        assert torch.equal(a[key], b[key]), key
        assert torch.equal(b[key], b2[key]), key
