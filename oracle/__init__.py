"""fp64 CPU oracle for the GPTQ layer pass and its intrinsic-LoRA variant.

TEST INFRASTRUCTURE ONLY. This package is the slow, plain, obviously correct
statement of what the CUDA path must compute. It is imported only by the test
suite, by ``__graft_entry__.smoke()`` (to check one small run) and by the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``. The product path
never imports, links or calls anything in here, and nothing in here imports
the product package: the two share no code. Inputs reach both from the
``datagen`` module, which holds none of the method's arithmetic.

Everything is float64 NumPy. Every function cites the page and section whose
statement it follows. Where the pages leave a step open, the function says
which reading it takes.

Parity status of each function (what pins it; see tests/test_oracle_*.py):

==============================  ==================================================
hessian                         brute-force triple loop on tiny inputs
damp                            closed form (mean of the diagonal)
inverse_cholesky_upper          U^T U H = I, triangularity, and the Gram-Schmidt
                                lengths of the QL factor of [X; mu I]
minmax_grid                     hand-derived golden rows (tests/golden/grid_*.txt)
sweep (plain)                   Babai nearest plane in data space (exact codes),
                                round-to-nearest when X^T X = I, blocking
                                invariance, brute force on tiny n, exact loss
                                identity
il_* (intrinsic LoRA)           r = 0 equals plain GPTQ bit for bit; literal
                                eig+QR factor equals the Schur-complement route;
                                R equals its closed-form conditional optimum;
                                codes and R equal Babai on the augmented lattice;
                                residual-based error bound
pack_codes                      hand-derived golden words (tests/golden/pack_*.txt)
olrc / bidup / refine_loop      OLrC's X (L R) equals the truncated SVD of X E^T and
(OLrC + Bid-Up refinement)      its loss the dropped singular values; every Bid-Up
                                decision is the brute-force best code for its
                                coordinate; the loss history never increases
rtn_quantize / quantize_lowrank every code is the brute-force nearest grid point;
(4-bit L, 8-bit R)              re-quantizing the dequantized values is idempotent;
                                grid and packing pinned as above
gptq2d_* (two-sided rounding)   anti-diagonal sweep equals the vectorised sweep and
                                Babai nearest plane on the basis B^T (x) A; with
                                B = I it is the one-sided sweep of every column
gptq2d_residuals                closed form X - Z = U_G^T E U_H: equals the sweep's
                                recorded v - z; every |c| <= 1/2 for the sweep's Z
                                and a Z moved by one step breaks it
lll_gram / reduce_for_gptq      the output is size-reduced and meets the Lovasz
(lattice basis reduction)       condition (Gram-Schmidt data from an independent
                                Cholesky), T is unimodular and G_red = T^T G T; the
                                LLL bound |b_1|^2 <= 2^(n-1) lambda_1^2 against brute-
                                force shortest vectors; a diagonal Gram is only
                                permuted
round_in_basis / withreduction  equals a data-space nearest plane on an explicit
                                basis; orthogonal data gives round-to-nearest;
                                Babai's bound sum Bn / 4 in the reduced basis; never
                                better than the brute-force optimum on tiny rows
==============================  ==================================================
"""
from .gptq import (
    hessian,
    damp,
    inverse_cholesky_upper,
    minmax_grid,
    sweep,
    sweep_blocked,
    gptq_layer,
    replay,
    regularised_loss_rows,
    data_loss_rows,
)
from .il import (
    top_singular_directions,
    augmented_gram,
    il_hessian,
    eig_qr_factor,
    schur_factor_rows,
    il_layer,
    il_R_closed_form,
)
from .babai import ql_decomposition, babai_nearest_plane
from .pack import pack_codes, unpack_codes
from .refine import olrc, bidup, dequant, refine as refine_loop
from .refine import data_loss_rows as lowrank_loss_rows
from .lowbit import rtn_quantize, quantize_lowrank
from .lll import lll_gram, gram_schmidt, reduce_for_gptq, round_in_basis, withreduction
from .gptq2d import (adaptive_round_1d, gptq2d_antidiagonal, gptq2d_residuals, gptq2d_vectorized,
                     reverse_cholesky_upper, two_sided_loss)

__all__ = [
    "olrc", "bidup", "dequant", "refine_loop", "lowrank_loss_rows", "rtn_quantize",
    "quantize_lowrank", "adaptive_round_1d", "gptq2d_vectorized", "gptq2d_antidiagonal",
    "two_sided_loss", "gptq2d_residuals", "reverse_cholesky_upper",
    "hessian", "damp", "inverse_cholesky_upper", "minmax_grid", "sweep", "sweep_blocked",
    "gptq_layer", "replay", "regularised_loss_rows", "data_loss_rows",
    "top_singular_directions", "augmented_gram", "il_hessian", "eig_qr_factor",
    "schur_factor_rows", "il_layer", "il_R_closed_form",
    "ql_decomposition", "babai_nearest_plane", "pack_codes", "unpack_codes",
]
