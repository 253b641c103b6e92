"""Host-side checks of the C ABI: the library loads, exports what include/gptq.h declares,
and rejects bad arguments before touching the device (no GPU needed)."""
import ctypes
import importlib
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "gptq.h")).read()
    return sorted(set(re.findall(r"GPTQ_API\s+[\w\s\*]+?\b(gptq_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    assert _declared() == sorted([
        "gptq_workspace_size", "gptq_status_string", "gptq_sync_status", "gptq_launch_count",
        "gptq_hessian_accumulate", "gptq_prepare_hinv", "gptq_quantize_layer",
        "gptq_quantize_layer_noalloc", "gptq_il_quantize_layer", "gptq_il_refine",
        "gptq_quantize_lowrank", "gptq_2d_round", "gptq_set_flags", "gptq_get_flags",
        "gptq_kernel_times", "gptq_quantize_layer_reduced"])


def test_library_exports_every_declared_symbol():
    import post_weight_quantization_06_b200 as g
    out = subprocess.run(["nm", "-D", "--defined-only", g.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, re.M))
    for name in _declared():
        assert name in exported, name
    lib = ctypes.CDLL(g.LIB_PATH)
    for name in _declared():
        assert getattr(lib, name) is not None
    assert set(g.EXPORTED) == set(_declared())


def test_library_has_no_dynamic_cuda_runtime_dependency():
    import post_weight_quantization_06_b200 as g
    out = subprocess.run(["ldd", g.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out


def test_status_strings():
    import post_weight_quantization_06_b200 as g
    assert g.status_string(0) == "GPTQ_OK"
    for code in range(-7, 0):
        assert g.status_string(code).startswith("GPTQ_ERR_")
    assert "NOT_CONVERGED" in g.status_string(g.GPTQ_ERR_NOT_CONVERGED)
    assert "unknown" in g.status_string(7)


def test_workspace_sizes():
    import post_weight_quantization_06_b200 as g
    assert g.gptq_workspace_size(g.GPTQ_OP_HESSIAN, 10, 64) == 0
    f = g.gptq_workspace_size(g.GPTQ_OP_PREPARE_HINV, 0, 6144)
    assert f >= 6144 * 6144 * 4
    q = g.gptq_workspace_size(g.GPTQ_OP_QUANTIZE, 2048, 6144, 0, 128)
    assert q >= 2048 * 6144 * 4 + 2048 * 128 * 4
    il0 = g.gptq_workspace_size(g.GPTQ_OP_IL_QUANTIZE, 2048, 6144, 0, 128)
    il = g.gptq_workspace_size(g.GPTQ_OP_IL_QUANTIZE, 2048, 6144, 64, 128)
    assert il > il0 >= q + f
    rf = g.gptq_workspace_size(g.GPTQ_OP_IL_REFINE, 2048, 6144, 64, 0)
    assert rf >= 3 * 2048 * 6144 * 4 + 2048 * 2048 * 4
    assert g.gptq_workspace_size(g.GPTQ_OP_IL_REFINE, 2048, 6144, 0, 0) < rf
    assert g.gptq_workspace_size(99, 1, 1) == 0
    t2 = g.gptq_workspace_size(g.GPTQ_OP_2D_ROUND, 2048, 6144)
    assert t2 >= (2 * 6144 * 6144 + 2048 * 2048 + 4 * 2048 * 6144) * 4
    # ragged shapes are padded to whole 32 x 32 tiles
    assert g.gptq_workspace_size(g.GPTQ_OP_2D_ROUND, 70, 100) >= (2 * 128 * 128 + 96 * 96 + 4 * 96 * 128) * 4
    assert g.gptq_workspace_size(g.GPTQ_OP_2D_ROUND, 0, 100) == 0
    for v in (f, q, il0, il, rf, t2):
        assert v % 256 == 0


def _lib():
    import post_weight_quantization_06_b200 as g
    return g._lib


NULL = None
P = ctypes.c_void_p(256)  # never dereferenced: every case below fails validation first


@pytest.mark.parametrize("args", [
    (NULL, P, 0, 10, 64, NULL),      # H missing
    (P, P, 5, 10, 64, NULL),         # bad dtype
    (P, P, 0, -1, 64, NULL),         # negative k
    (P, P, 0, 10, 0, NULL),          # n = 0
])
def test_hessian_rejects_bad_arguments(args):
    assert _lib().gptq_hessian_accumulate(*args) == -1


def test_hessian_k0_is_a_noop():
    import post_weight_quantization_06_b200 as g
    before = g.gptq_launch_count()
    assert _lib().gptq_hessian_accumulate(P, P, 0, 0, 64, NULL) == 0
    assert g.gptq_launch_count() == before


@pytest.mark.parametrize("kw,expect", [
    (dict(bits=1), -1), (dict(bits=9), -1), (dict(block=96), -1), (dict(n=200), -1),
    (dict(gs=48), -1), (dict(gs=100, n=1000, block=100), -1), (dict(m=0), -1),
    (dict(ws_bytes=16), -6), (dict(ws=None), -6),
])
def test_quantize_rejects_bad_arguments(kw, expect):
    import post_weight_quantization_06_b200 as g
    a = dict(m=64, n=256, bits=4, gs=128, block=128, ws=ctypes.c_void_p(1 << 20), ws_bytes=None)
    a.update(kw)
    ws_bytes = a["ws_bytes"]
    if ws_bytes is None:
        ws_bytes = g.gptq_workspace_size(g.GPTQ_OP_QUANTIZE, max(a["m"], 1), a["n"], 0, a["block"])
    st = _lib().gptq_quantize_layer(P, 1, a["m"], a["n"], P, a["bits"], a["gs"], a["block"],
                                    P, P, P, NULL, a["ws"], ws_bytes, NULL)
    assert st == expect


def test_workspace_alignment_is_checked():
    import post_weight_quantization_06_b200 as g
    need = g.gptq_workspace_size(g.GPTQ_OP_PREPARE_HINV, 0, 64)
    st = _lib().gptq_prepare_hinv(P, 64, ctypes.c_float(0.01), P, P, ctypes.c_void_p((1 << 20) + 64),
                                  need, NULL)
    assert st == -6


@pytest.mark.parametrize("r,L,lam", [(-1, P, 0.01), (129, P, 0.01), (4, NULL, 0.01), (256, P, 0.01),
                                     (4, P, -1.0), (4, P, float("nan"))])
def test_il_rejects_bad_arguments(r, L, lam):
    import post_weight_quantization_06_b200 as g
    need = g.gptq_workspace_size(g.GPTQ_OP_IL_QUANTIZE, 64, 256, max(r, 0), 128)
    st = _lib().gptq_il_quantize_layer(P, 1, 64, 256, P, r, 4, 128, ctypes.c_float(lam), 128,
                                       P, P, P, L, P, P, NULL, ctypes.c_void_p(1 << 20), need, NULL)
    assert st == -1


@pytest.mark.parametrize("m,r,iters,loss,bits", [(64, -1, 1, P, 4), (64, 129, 1, P, 4),
                                                 (64, 64, 1, P, 4), (8, 16, 1, P, 4),
                                                 (64, 4, 0, P, 4), (64, 4, 1, NULL, 4),
                                                 (64, 4, 1, P, 1)])
def test_refine_rejects_bad_arguments(m, r, iters, loss, bits):
    import post_weight_quantization_06_b200 as g
    need = g.gptq_workspace_size(g.GPTQ_OP_IL_REFINE, m, 256, max(r, 0), 0)
    st = _lib().gptq_il_refine(P, 1, m, 256, P, r, bits, 128, iters, P, P, P, P, P, loss,
                               ctypes.c_void_p(1 << 20), need, NULL)
    assert st == -1


def test_refine_rejects_a_small_workspace():
    import post_weight_quantization_06_b200 as g
    need = g.gptq_workspace_size(g.GPTQ_OP_IL_REFINE, 64, 256, 4, 0)
    st = _lib().gptq_il_refine(P, 1, 64, 256, P, 4, 4, 128, 1, P, P, P, P, P, P,
                               ctypes.c_void_p(1 << 20), need - 256, NULL)
    assert st == -6


@pytest.mark.parametrize("n,r,bL,gL,bR", [(256, 0, 4, 128, 8), (256, 129, 4, 128, 8),
                                           (256, 64, 1, 128, 8), (256, 64, 4, 100, 8),
                                           (12, 64, 4, 0, 8), (256, 3, 4, 128, 8),
                                           (256, 64, 4, 128, 9)])
def test_lowrank_quantize_rejects_bad_arguments(n, r, bL, gL, bR):
    st = _lib().gptq_quantize_lowrank(P, P, n, 64, r, bL, gL, bR, P, P, P, P, P, P, NULL)
    assert st == -1


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    import post_weight_quantization_06_b200 as g
    monkeypatch.setattr(g, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        g._load()


@pytest.mark.parametrize("X,m,n,G,H,Z", [(NULL, 8, 8, P, P, P), (P, 8, 8, NULL, P, P),
                                         (P, 8, 8, P, NULL, P), (P, 8, 8, P, P, NULL),
                                         (P, -1, 8, P, P, P), (P, 8, -3, P, P, P),
                                         (P, 65537, 8, P, P, P), (P, 8, 70000, P, P, P)])
def test_2d_round_rejects_bad_arguments(X, m, n, G, H, Z):
    st = _lib().gptq_2d_round(X, m, n, G, H, Z, NULL, ctypes.c_void_p(1 << 20), 1 << 40, NULL)
    assert st == -1


def test_2d_round_checks_the_workspace_and_accepts_empty_input():
    import post_weight_quantization_06_b200 as g
    need = g.gptq_workspace_size(g.GPTQ_OP_2D_ROUND, 40, 70)
    lib = _lib()
    assert lib.gptq_2d_round(P, 40, 70, P, P, P, NULL, ctypes.c_void_p(1 << 20), need - 256, NULL) == -6
    assert lib.gptq_2d_round(P, 40, 70, P, P, P, NULL, ctypes.c_void_p((1 << 20) + 16), need, NULL) == -6
    assert lib.gptq_2d_round(P, 40, 70, P, P, P, NULL, NULL, need, NULL) == -6
    # nothing to round: returns at once, touching no pointer
    assert lib.gptq_2d_round(NULL, 0, 70, NULL, NULL, NULL, NULL, NULL, 0, NULL) == 0
    assert lib.gptq_2d_round(NULL, 40, 0, NULL, NULL, NULL, NULL, NULL, 0, NULL) == 0


def test_flags_round_trip_and_host_errors_stay_synchronous():
    import post_weight_quantization_06_b200 as g
    try:
        g.gptq_set_flags(g.GPTQ_FLAG_SYNC_STATUS | g.GPTQ_FLAG_IL_FP64)
        assert g.gptq_get_flags() == g.GPTQ_FLAG_SYNC_STATUS | g.GPTQ_FLAG_IL_FP64
        # argument errors are returned before anything is enqueued or synchronised
        assert _lib().gptq_hessian_accumulate(NULL, P, 0, 10, 64, NULL) == -1
        assert _lib().gptq_2d_round(P, -1, 5, P, P, P, NULL, NULL, 0, NULL) == -1
    finally:
        g.gptq_set_flags(0)
    assert g.gptq_get_flags() == 0


def test_kernel_times_record_is_empty_and_checks_its_arguments():
    """Nothing launched: every class reads zero (no device call is needed to read an empty
    record); the class count and the stage names agree with the header."""
    import post_weight_quantization_06_b200 as g
    src = open(os.path.join(ROOT, "include", "gptq.h")).read()
    assert f"#define GPTQ_KT_NCLASSES {g.GPTQ_KT_NCLASSES}" in src
    stages = re.findall(r"GPTQ_KT_(\w+) = (\d+)", src)
    names = {int(v): k.lower() for k, v in stages if k != "NSTAGES"}
    assert tuple(names[i] for i in range(len(names))) == g.KT_STAGES
    arr = (g.KernelTime * g.GPTQ_KT_NCLASSES)()
    assert g.gptq_kernel_times(arr, g.GPTQ_KT_NCLASSES) == g.GPTQ_KT_NCLASSES
    assert all(c.launches == 0 and c.ms == 0 and c.flops == 0 for c in arr)
    assert g.gptq_kernel_times(None, 0) == g.GPTQ_KT_NCLASSES
    assert g.gptq_kernel_times(None, 3) == g.GPTQ_ERR_ARG
    assert g.gptq_kernel_times(arr, -1) == g.GPTQ_ERR_ARG
    assert g.kernel_times() == {}


P1 = ctypes.c_void_p(256)


@pytest.mark.parametrize("m,n,bits,lam,wdt", [
    (0, 256, 4, 0.01, 1), (8, 0, 4, 0.01, 1), (8, 2049, 4, 0.01, 1), (8, 256, 1, 0.01, 1),
    (8, 256, 9, 0.01, 1), (8, 100, 4, 0.01, 1), (8, 256, 4, -1.0, 1), (8, 256, 4, 0.01, 7)])
def test_reduced_rejects_bad_arguments(m, n, bits, lam, wdt):
    import post_weight_quantization_06_b200 as g
    before = g.gptq_launch_count()
    st = _lib().gptq_quantize_layer_reduced(P1, wdt, m, n, P1, bits, ctypes.c_float(lam), P1, P1,
                                            P1, NULL, NULL, NULL, ctypes.c_void_p(1 << 20),
                                            1 << 40, NULL)
    assert st == -1
    assert g.gptq_launch_count() == before


def test_reduced_checks_its_workspace():
    import post_weight_quantization_06_b200 as g
    m, n = 64, 256
    need = g.gptq_workspace_size(g.GPTQ_OP_REDUCED, m, n, 0, 0)
    assert need > 0 and g.gptq_workspace_size(g.GPTQ_OP_REDUCED, m, 4096, 0, 0) == 0
    before = g.gptq_launch_count()
    st = _lib().gptq_quantize_layer_reduced(P1, 1, m, n, P1, 4, ctypes.c_float(0.01), P1, P1, P1,
                                            NULL, NULL, NULL, ctypes.c_void_p(1 << 20), need - 1,
                                            NULL)
    assert st == -6
    assert g.gptq_launch_count() == before
