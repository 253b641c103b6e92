"""Python binding of libgptq (the B200 GPTQ / GPTQ-intrinsic-LoRA layer pass).

Argument marshalling only: every step runs in the CUDA kernels of ``libgptq.so``.
PyTorch provides device memory and the current stream. The functions carry the
C-ABI names and raise ``GptqError`` on a non-zero status. There is no fallback:
if the library is missing the import of this module fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgptq.so")

GPTQ_OK, GPTQ_ERR_ARG, GPTQ_ERR_NOT_PD, GPTQ_ERR_NONFINITE = 0, -1, -2, -3
GPTQ_ERR_TIMEOUT, GPTQ_ERR_CUDA, GPTQ_ERR_WORKSPACE = -4, -5, -6
GPTQ_ERR_NOT_CONVERGED = -7
GPTQ_BF16, GPTQ_F32 = 0, 1
GPTQ_OP_HESSIAN, GPTQ_OP_PREPARE_HINV, GPTQ_OP_QUANTIZE, GPTQ_OP_IL_QUANTIZE = 0, 1, 2, 3
GPTQ_OP_IL_REFINE, GPTQ_OP_2D_ROUND, GPTQ_OP_REDUCED = 4, 5, 6
GPTQ_FLAG_SYNC_STATUS, GPTQ_FLAG_DEBUG_CHECKS, GPTQ_FLAG_IL_FP64 = 1, 2, 4
GPTQ_FLAG_KERNEL_TIMES = 8
KT_STAGES = ("other", "factor", "sweep", "il", "refine", "2d")   # gptq_kt_stage order
KT_PATHS = ("tc", "simt")
GPTQ_KT_NCLASSES = len(KT_STAGES) * len(KT_PATHS)

EXPORTED = ("gptq_workspace_size", "gptq_status_string", "gptq_sync_status", "gptq_launch_count",
            "gptq_hessian_accumulate", "gptq_prepare_hinv", "gptq_quantize_layer",
            "gptq_quantize_layer_noalloc", "gptq_il_quantize_layer", "gptq_il_refine",
            "gptq_quantize_lowrank", "gptq_2d_round", "gptq_set_flags", "gptq_get_flags",
            "gptq_kernel_times", "gptq_quantize_layer_reduced")


class KernelTime(ctypes.Structure):
    """gptq_kernel_time: totals of one class of GEMM launches."""
    _fields_ = [("launches", ctypes.c_int64), ("ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class GptqError(RuntimeError):
    def __init__(self, status: int, where: str, info: int = 0):
        self.status, self.info = status, info
        super().__init__(f"{where}: {status_string(status)} (status {status}, info {info})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libgptq.so not built ({LIB_PATH}); run __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    c_i64, c_p, c_sz, c_f = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
    c_int = ctypes.c_int
    sig = {
        "gptq_workspace_size": (c_sz, [c_int, c_i64, c_i64, c_int, c_int]),
        "gptq_status_string": (ctypes.c_char_p, [c_int]),
        "gptq_sync_status": (c_int, [c_p, ctypes.POINTER(c_i64)]),
        "gptq_launch_count": (ctypes.c_uint64, []),
        "gptq_hessian_accumulate": (c_int, [c_p, c_p, c_int, c_i64, c_i64, c_p]),
        "gptq_prepare_hinv": (c_int, [c_p, c_i64, c_f, c_p, c_p, c_p, c_sz, c_p]),
        "gptq_quantize_layer": (c_int, [c_p, c_int, c_i64, c_i64, c_p, c_int, c_int, c_int,
                                        c_p, c_p, c_p, c_p, c_p, c_sz, c_p]),
        "gptq_quantize_layer_noalloc": (c_int, [c_p, c_int, c_i64, c_i64, c_p, c_int, c_int,
                                                c_int, c_p, c_p, c_p, c_p, c_p]),
        "gptq_il_quantize_layer": (c_int, [c_p, c_int, c_i64, c_i64, c_p, c_int, c_int, c_int,
                                           c_f, c_int, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p,
                                           c_sz, c_p]),
        "gptq_il_refine": (c_int, [c_p, c_int, c_i64, c_i64, c_p, c_int, c_int, c_int, c_int,
                                   c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_sz, c_p]),
        "gptq_quantize_lowrank": (c_int, [c_p, c_p, c_i64, c_i64, c_int, c_int, c_int, c_int,
                                          c_p, c_p, c_p, c_p, c_p, c_p, c_p]),
        "gptq_2d_round": (c_int, [c_p, c_i64, c_i64, c_p, c_p, c_p, c_p, c_p, c_sz, c_p]),
        "gptq_set_flags": (None, [ctypes.c_uint]),
        "gptq_get_flags": (ctypes.c_uint, []),
        "gptq_kernel_times": (c_int, [ctypes.POINTER(KernelTime), c_int]),
        "gptq_quantize_layer_reduced": (c_int, [c_p, c_int, c_i64, c_i64, c_p, c_int, c_f, c_p, c_p,
                                                c_p, c_p, c_p, c_p, c_p, c_sz, c_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


def status_string(status: int) -> str:
    return _lib.gptq_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GPTQ_BF16
    if t.dtype == torch.float32:
        return GPTQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _check(st: int, where: str):
    if st != GPTQ_OK:
        raise GptqError(st, where)


def gptq_workspace_size(op: int, m: int, n: int, r: int = 0, block_size: int = 128) -> int:
    return int(_lib.gptq_workspace_size(op, m, n, r, block_size))


def workspace(op: int, m: int, n: int, r: int = 0, block_size: int = 128, device=None):
    """A caller-owned workspace tensor (uint8, 256-byte aligned by the caching allocator)."""
    nbytes = gptq_workspace_size(op, m, n, r, block_size)
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device or "cuda")


def gptq_set_flags(flags: int) -> None:
    _lib.gptq_set_flags(int(flags))


def gptq_get_flags() -> int:
    return int(_lib.gptq_get_flags())


def gptq_kernel_times(out, n_out: int) -> int:
    return int(_lib.gptq_kernel_times(out, int(n_out)))


def kernel_times() -> dict:
    """Reads and clears the GEMM launch record of GPTQ_FLAG_KERNEL_TIMES: {(stage, path):
    {launches, ms, flops, bytes}} for every class with at least one launch."""
    arr = (KernelTime * GPTQ_KT_NCLASSES)()
    st = gptq_kernel_times(arr, GPTQ_KT_NCLASSES)
    if st < 0:
        raise GptqError(st, "gptq_kernel_times")
    out = {}
    for c in range(GPTQ_KT_NCLASSES):
        if arr[c].launches:
            out[(KT_STAGES[c // 2], KT_PATHS[c % 2])] = {
                "launches": int(arr[c].launches), "ms": arr[c].ms, "flops": arr[c].flops,
                "bytes": arr[c].bytes}
    return out


def gptq_launch_count() -> int:
    """Kernels launched by libgptq in this process so far."""
    return int(_lib.gptq_launch_count())


def gptq_sync_status(stream=None, raise_on_error: bool = True):
    """Waits for the stream; returns (status, info) of the device status word and clears it."""
    info = ctypes.c_int64(0)
    st = _lib.gptq_sync_status(_stream(stream), ctypes.byref(info))
    if raise_on_error and st != GPTQ_OK:
        raise GptqError(st, "device status", info.value)
    return st, info.value


def gptq_hessian_accumulate(H: torch.Tensor, X: torch.Tensor, stream=None):
    """H += 2 X^T X (H: n x n fp32; X: k x n bf16/fp32)."""
    _dev(H, "H", torch.float32)
    _dev(X, "X")
    k, n = X.shape
    assert H.shape == (n, n)
    _check(_lib.gptq_hessian_accumulate(_ptr(H), _ptr(X), _dtype_code(X), k, n, _stream(stream)),
           "gptq_hessian_accumulate")


def gptq_prepare_hinv(H: torch.Tensor, lambda_rel: float, U: torch.Tensor, lambda_out: torch.Tensor,
                      ws: torch.Tensor, stream=None):
    _dev(H, "H", torch.float32)
    _dev(U, "U", torch.float32)
    _dev(lambda_out, "lambda_out", torch.float32)
    n = H.shape[0]
    _check(_lib.gptq_prepare_hinv(_ptr(H), n, float(lambda_rel), _ptr(U), _ptr(lambda_out),
                                  _ptr(ws), ws.numel(), _stream(stream)), "gptq_prepare_hinv")


def gptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, bits: int, group_size: int,
                        block_size: int, codes: torch.Tensor, scales: torch.Tensor,
                        zeros: torch.Tensor, loss_out: torch.Tensor | None, ws: torch.Tensor,
                        stream=None):
    _dev(W, "W")
    _dev(U, "U", torch.float32)
    _dev(codes, "codes", torch.int32)
    _dev(scales, "scales", torch.float32)
    _dev(zeros, "zeros", torch.uint8)
    if loss_out is not None:
        _dev(loss_out, "loss_out", torch.float64)
    m, n = W.shape
    _check(_lib.gptq_quantize_layer(_ptr(W), _dtype_code(W), m, n, _ptr(U), bits, group_size,
                                    block_size, _ptr(codes), _ptr(scales), _ptr(zeros),
                                    _ptr(loss_out), _ptr(ws), ws.numel(), _stream(stream)),
           "gptq_quantize_layer")


NOALLOC_SCRATCH_BYTES = 64 << 20


def gptq_quantize_layer_noalloc(W: torch.Tensor, U: torch.Tensor, bits: int, group_size: int,
                                block_size: int, codes: torch.Tensor, scales: torch.Tensor,
                                zeros: torch.Tensor, loss_out: torch.Tensor | None, stream=None):
    """gptq_quantize_layer for callers that cannot provide device scratch memory: the
    library's own fixed device array (NOALLOC_SCRATCH_BYTES) is used instead, shared by every
    call on the device, so overlapping calls must be serialised by the caller."""
    _dev(W, "W")
    _dev(U, "U", torch.float32)
    _dev(codes, "codes", torch.int32)
    _dev(scales, "scales", torch.float32)
    _dev(zeros, "zeros", torch.uint8)
    if loss_out is not None:
        _dev(loss_out, "loss_out", torch.float64)
    m, n = W.shape
    _check(_lib.gptq_quantize_layer_noalloc(_ptr(W), _dtype_code(W), m, n, _ptr(U), bits,
                                            group_size, block_size, _ptr(codes), _ptr(scales),
                                            _ptr(zeros), _ptr(loss_out), _stream(stream)),
           "gptq_quantize_layer_noalloc")


def gptq_il_quantize_layer(W: torch.Tensor, H: torch.Tensor, r: int, bits: int, group_size: int,
                           lambda_rel: float, block_size: int, codes: torch.Tensor,
                           scales: torch.Tensor, zeros: torch.Tensor, L: torch.Tensor | None,
                           R: torch.Tensor | None, lambda_out: torch.Tensor,
                           loss_out: torch.Tensor | None, ws: torch.Tensor, stream=None):
    _dev(W, "W")
    _dev(H, "H", torch.float32)
    _dev(codes, "codes", torch.int32)
    _dev(scales, "scales", torch.float32)
    _dev(zeros, "zeros", torch.uint8)
    _dev(lambda_out, "lambda_out", torch.float32)
    m, n = W.shape
    _check(_lib.gptq_il_quantize_layer(_ptr(W), _dtype_code(W), m, n, _ptr(H), r, bits, group_size,
                                       float(lambda_rel), block_size, _ptr(codes), _ptr(scales),
                                       _ptr(zeros), _ptr(L), _ptr(R), _ptr(lambda_out),
                                       _ptr(loss_out), _ptr(ws), ws.numel(), _stream(stream)),
           "gptq_il_quantize_layer")


def gptq_il_refine(W: torch.Tensor, H: torch.Tensor, r: int, bits: int, group_size: int,
                   iters: int, codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                   L: torch.Tensor | None, R: torch.Tensor | None, loss_hist: torch.Tensor,
                   ws: torch.Tensor, stream=None):
    _dev(W, "W")
    _dev(H, "H", torch.float32)
    _dev(codes, "codes", torch.int32)
    _dev(scales, "scales", torch.float32)
    _dev(zeros, "zeros", torch.uint8)
    _dev(loss_hist, "loss_hist", torch.float64)
    m, n = W.shape
    _check(_lib.gptq_il_refine(_ptr(W), _dtype_code(W), m, n, _ptr(H), r, bits, group_size, iters,
                               _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(L), _ptr(R),
                               _ptr(loss_hist), _ptr(ws), ws.numel(), _stream(stream)),
           "gptq_il_refine")


def gptq_quantize_lowrank(L: torch.Tensor, R: torch.Tensor, bits_L: int, group_size_L: int,
                          bits_R: int, codes_L: torch.Tensor, scales_L: torch.Tensor,
                          zeros_L: torch.Tensor, codes_R: torch.Tensor, scales_R: torch.Tensor,
                          zeros_R: torch.Tensor, stream=None):
    _dev(L, "L", torch.float32)
    _dev(R, "R", torch.float32)
    for t, name, dt in ((codes_L, "codes_L", torch.int32), (scales_L, "scales_L", torch.float32),
                        (zeros_L, "zeros_L", torch.uint8), (codes_R, "codes_R", torch.int32),
                        (scales_R, "scales_R", torch.float32), (zeros_R, "zeros_R", torch.uint8)):
        _dev(t, name, dt)
    n, r = L.shape
    m = R.shape[1]
    _check(_lib.gptq_quantize_lowrank(_ptr(L), _ptr(R), n, m, r, bits_L, group_size_L, bits_R,
                                      _ptr(codes_L), _ptr(scales_L), _ptr(zeros_L), _ptr(codes_R),
                                      _ptr(scales_R), _ptr(zeros_R), _stream(stream)),
           "gptq_quantize_lowrank")


def gptq_2d_round(X: torch.Tensor, G: torch.Tensor, H: torch.Tensor, Z: torch.Tensor,
                  err: torch.Tensor | None, ws: torch.Tensor | None, stream=None):
    m, n = X.shape
    if m and n:
        for t, name in ((X, "X"), (G, "G"), (H, "H")):
            _dev(t, name, torch.float32)
        _dev(Z, "Z", torch.int32)
        if err is not None:
            _dev(err, "err", torch.float32)
        if G.shape != (m, m) or H.shape != (n, n) or Z.shape != (m, n):
            raise ValueError("gptq_2d_round: G must be m x m, H n x n, Z m x n")
    nbytes = 0 if ws is None else ws.numel()
    _check(_lib.gptq_2d_round(_ptr(X), m, n, _ptr(G), _ptr(H), _ptr(Z), _ptr(err), _ptr(ws),
                              nbytes, _stream(stream)), "gptq_2d_round")


def gptq_quantize_layer_reduced(W: torch.Tensor, H: torch.Tensor, bits: int, lambda_rel: float,
                                codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                                loss_out: torch.Tensor | None, coef_out: torch.Tensor | None,
                                stats_out: torch.Tensor | None, ws: torch.Tensor, stream=None):
    _dev(W, "W")
    _dev(H, "H", torch.float32)
    _dev(codes, "codes", torch.int32)
    _dev(scales, "scales", torch.float32)
    _dev(zeros, "zeros", torch.uint8)
    if loss_out is not None:
        _dev(loss_out, "loss_out", torch.float64)
    if coef_out is not None:
        _dev(coef_out, "coef_out", torch.int32)
    if stats_out is not None:
        _dev(stats_out, "stats_out", torch.int64)
    m, n = W.shape
    _check(_lib.gptq_quantize_layer_reduced(_ptr(W), _dtype_code(W), m, n, _ptr(H), bits,
                                            float(lambda_rel), _ptr(codes), _ptr(scales),
                                            _ptr(zeros), _ptr(loss_out), _ptr(coef_out),
                                            _ptr(stats_out), _ptr(ws), ws.numel(), _stream(stream)),
           "gptq_quantize_layer_reduced")


def quantize_layer_reduced(W: torch.Tensor, H: torch.Tensor, *, bits: int, lambda_rel: float = 0.01,
                           check_status: bool = True) -> dict:
    """GPTQ after LLL reduction of the data lattice, per-channel grid, with fresh outputs."""
    dev = W.device
    m, n = W.shape
    out = dict(codes=torch.empty(m, n * bits // 32, dtype=torch.int32, device=dev),
               scales=torch.empty(m, dtype=torch.float32, device=dev),
               zeros=torch.empty(m, dtype=torch.uint8, device=dev),
               loss=torch.empty(m, dtype=torch.float64, device=dev),
               coef=torch.empty(m, n, dtype=torch.int32, device=dev),
               stats=torch.zeros(8, dtype=torch.int64, device=dev))
    ws = workspace(GPTQ_OP_REDUCED, m, n, 0, 0, dev)
    gptq_quantize_layer_reduced(W, H, bits, lambda_rel, out["codes"], out["scales"], out["zeros"],
                                out["loss"], out["coef"], out["stats"], ws)
    if check_status:
        gptq_sync_status()
    return out


def round_2d(X: torch.Tensor, G: torch.Tensor, H: torch.Tensor, *, with_err: bool = False,
             check_status: bool = True) -> dict:
    """Two-sided adaptive rounding of X (m x n) under G (m x m) and H (n x n) with fresh
    outputs: Z (int32) and, if asked, the errors."""
    m, n = X.shape
    dev = X.device
    Z = torch.empty(m, n, dtype=torch.int32, device=dev)
    err = torch.empty(m, n, dtype=torch.float32, device=dev) if with_err else None
    ws = workspace(GPTQ_OP_2D_ROUND, m, n, 0, 0, dev) if m and n else None
    gptq_2d_round(X, G, H, Z, err, ws)
    if check_status:
        gptq_sync_status()
    out = dict(Z=Z)
    if with_err:
        out["err"] = err
    return out


# ------------------------------------------------------------------------------------------
# Convenience: one layer end to end with freshly allocated outputs (still only ABI calls).
# ------------------------------------------------------------------------------------------

def quantize_layer(W: torch.Tensor, X: torch.Tensor | None = None, *, H: torch.Tensor | None = None,
                   bits: int = 4, group_size: int = 128, lambda_rel: float = 0.01,
                   block_size: int = 128, r: int = 0, intrinsic: bool = False,
                   chunk_tokens: int = 16384, check_status: bool = True) -> dict:
    """Accumulate H over X in token chunks (unless H is given), then run the plain pass
    (gptq_prepare_hinv + gptq_quantize_layer) or, when r > 0 or ``intrinsic`` is set, the
    intrinsic-LoRA entry point. Returns a dict of device tensors."""
    dev = W.device
    m, n = W.shape
    if H is None:
        H = torch.zeros(n, n, dtype=torch.float32, device=dev)
        for t0 in range(0, X.shape[0], chunk_tokens):
            gptq_hessian_accumulate(H, X[t0:t0 + chunk_tokens])
    G = n // group_size if group_size else 1
    codes = torch.empty(m, n * bits // 32, dtype=torch.int32, device=dev)
    scales = torch.empty(m, G, dtype=torch.float32, device=dev)
    zeros = torch.empty(m, G, dtype=torch.uint8, device=dev)
    loss = torch.empty(m, dtype=torch.float64, device=dev)
    lam = torch.empty(1, dtype=torch.float32, device=dev)
    out = dict(H=H, codes=codes, scales=scales, zeros=zeros, loss=loss, lam=lam)
    if r == 0 and not intrinsic:
        U = torch.empty(n, n, dtype=torch.float32, device=dev)
        ws = workspace(GPTQ_OP_PREPARE_HINV, m, n, 0, block_size, dev)
        gptq_prepare_hinv(H, lambda_rel, U, lam, ws)
        ws2 = workspace(GPTQ_OP_QUANTIZE, m, n, 0, block_size, dev)
        gptq_quantize_layer(W, U, bits, group_size, block_size, codes, scales, zeros, loss, ws2)
        out["U"] = U
    else:
        L = torch.empty(n, max(r, 1), dtype=torch.float32, device=dev)
        R = torch.empty(max(r, 1), m, dtype=torch.float32, device=dev)
        ws = workspace(GPTQ_OP_IL_QUANTIZE, m, n, r, block_size, dev)
        gptq_il_quantize_layer(W, H, r, bits, group_size, lambda_rel, block_size, codes, scales,
                               zeros, L, R, lam, loss, ws)
        out.update(L=L, R=R)
    if check_status:
        gptq_sync_status()
    return out
