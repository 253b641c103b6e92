"""Low-precision storage of the low-rank factors (oracle; test infrastructure only).

GPTQ-intrinsic LoRA summary, "Main results" (empirical side): quantizing the low-rank
factors L and R to low precision, 4-bit and 8-bit respectively, is often lossless or even
beneficial. The page gives no procedure. Reading taken: round-to-nearest (no error
feedback) onto the same per-group min-max grid the pass uses (`minmax_grid`), with each
factor stored the way the layer's own weights are, one neuron per row:
  * L (n x r, page orientation in x out) is quantized as L^T: r rows of n inputs, grouped
    like the layer (group_size; 0 = one group per row);
  * R (r x m) is quantized as R^T: m rows of r inputs, one group per row.
Codes are packed like the layer's codes (`pack_codes`).
"""
from __future__ import annotations

import numpy as np

from .gptq import _group_len, minmax_grid
from .pack import pack_codes


def rtn_quantize(A, bits: int, group_size: int) -> dict:
    """Round each row of A (rows x cols) to its groups' min-max grids: codes, scales, zeros,
    the dequantized matrix and the pre-rounding values v = a / s + z (for judging ties)."""
    A = np.asarray(A, dtype=np.float64)
    rows, cols = A.shape
    maxq = (1 << bits) - 1
    gs = _group_len(group_size, cols)
    G = -(-cols // gs)
    codes = np.zeros((rows, cols), dtype=np.int64)
    scales = np.zeros((rows, G))
    zeros = np.zeros((rows, G), dtype=np.int64)
    V = np.zeros((rows, cols))
    for g in range(G):
        seg = A[:, g * gs:(g + 1) * gs]
        s, z, _ = minmax_grid(seg, maxq)
        v = seg / s[:, None] + z[:, None]
        V[:, g * gs:(g + 1) * gs] = v
        codes[:, g * gs:(g + 1) * gs] = np.clip(np.rint(v), 0, maxq).astype(np.int64)
        scales[:, g] = s
        zeros[:, g] = z.astype(np.int64)
    gi = np.arange(cols) // gs
    deq = scales[:, gi] * (codes - zeros[:, gi])
    return dict(codes=codes, scales=scales, zeros=zeros, deq=deq, v=V)


def quantize_lowrank(L, R, bits_L: int = 4, group_size_L: int = 128, bits_R: int = 8) -> dict:
    """L^T at bits_L with the layer's grouping, R^T at bits_R one group per row; returns both
    results, their packed codes and the dequantized L_hat (n x r), R_hat (r x m)."""
    qL = rtn_quantize(np.asarray(L, dtype=np.float64).T, bits_L, group_size_L)
    qR = rtn_quantize(np.asarray(R, dtype=np.float64).T, bits_R, 0)
    return dict(L=qL, R=qR, L_hat=qL["deq"].T.copy(), R_hat=qR["deq"].T.copy(),
                packed_L=pack_codes(qL["codes"], bits_L), packed_R=pack_codes(qR["codes"], bits_R))
