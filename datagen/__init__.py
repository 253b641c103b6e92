"""Seeded synthetic layers and calibration sets for the GPTQ layer pass.

This module only draws random inputs. It holds none of the quantization
arithmetic, so both the CUDA path and the fp64 oracle can be fed from it.

Each recipe stands in for a layer shape and calibration set that the GPTQ /
GPTQ-intrinsic-LoRA pages evaluate on (Qwen3-0.6B / 1.7B projections, DeiT-B
MLP layers); the real weights and calibration text are not available, so the
recipes reproduce their shapes and spectral structure:

* ``tiny``      W 256x256 fp32, X 512x256 fp32 = Z diag(s) U, s_i = i^-0.7
* ``attn``      W 1024x1024 bf16 with 0.1% outliers at 10 sigma,
                X 65536x1024 bf16 ~ N(0, Sigma), power-law spectrum (exp -1)
                plus 8 spiked channels at 50x variance
* ``mlp_down``  W 2048x6144 bf16, X 262144x6144 bf16 = GeLU(correlated Gaussian)
* ``deit``      fc1 3072x768 / fc2 768x3072 fp32, X 50432 rows bf16 ~ N(0, Sigma),
                power-law spectrum (exp -1.2)
* ``lowrank``   W as ``mlp_down``; X = rank-64 signal at 100x the energy of an
                isotropic N(0, 1) noise floor
* ``two_sided`` two-sided rounding problem on the ``mlp_down`` shape: X 2048x6144 fp32
                ~ N(0, 9) (weights in grid steps), G 2048x2048 and H 6144x6144 fp32 Gram
                matrices Q diag(l) Q^T, Q Haar, l a power law (exponent 1, mean 1) + 0.01

Every draw comes from a ``torch.Generator`` seeded from (seed, stream id,
chunk index); calibration rows are produced in chunks of 16384 tokens so the
full-size sets can be generated on the device that will consume them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

CHUNK_TOKENS = 16384

# Stream ids keep the draws for different tensors of one layer independent.
_S_W, _S_BASIS, _S_X, _S_OUTLIER, _S_SPIKE, _S_SIGNAL, _S_G2D, _S_H2D = range(8)


def _gen(seed: int, stream: int, chunk: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 10_007 + chunk) & 0x7FFF_FFFF_FFFF)
    return g


def random_orthogonal(n: int, cols: int, seed: int, stream: int, device) -> torch.Tensor:
    """Haar-distributed n x cols matrix with orthonormal columns (QR of a
    Gaussian, signs fixed so that diag(R) > 0). Returned in fp32."""
    g = _gen(seed, stream, 0, device)
    a = torch.randn(n, cols, generator=g, device=device, dtype=torch.float32)
    q, r = torch.linalg.qr(a.double())
    q = q * torch.sign(torch.diagonal(r)).unsqueeze(0)
    return q.float()


def power_law(n: int, alpha: float, device) -> torch.Tensor:
    """Eigenvalues c * i^-alpha (i = 1..n), c chosen so that they sum to n."""
    i = torch.arange(1, n + 1, device=device, dtype=torch.float64)
    lam = i.pow(-alpha)
    return (lam * (n / lam.sum())).float()


@dataclass
class Layer:
    """One layer to quantize: weights W (out x in) and calibration X (tokens x in)."""
    name: str
    W: torch.Tensor
    X: torch.Tensor
    bits: int
    group_size: int            # 0 = one group per row (per-channel)
    lambda_rel: float
    block_size: int = 128
    r: int = 0                 # intrinsic-LoRA rank (0 = plain GPTQ)
    meta: dict = field(default_factory=dict)

    @property
    def m(self) -> int:
        return self.W.shape[0]

    @property
    def n(self) -> int:
        return self.W.shape[1]

    @property
    def k(self) -> int:
        return self.X.shape[0]


def gaussian_weights(m, n, std, dtype, seed, device) -> torch.Tensor:
    g = _gen(seed, _S_W, 0, device)
    return (torch.randn(m, n, generator=g, device=device) * std).to(dtype)


def _chunked_rows(k, n, seed, device, dtype, make_chunk):
    X = torch.empty(k, n, device=device, dtype=dtype)
    for c, t0 in enumerate(range(0, k, CHUNK_TOKENS)):
        t1 = min(k, t0 + CHUNK_TOKENS)
        g = _gen(seed, _S_X, c, device)
        X[t0:t1] = make_chunk(t1 - t0, g).to(dtype)
    return X


def correlated_gaussian_rows(k, n, alpha, seed, device, dtype, gelu=False,
                             spikes=0, spike_var=50.0) -> torch.Tensor:
    """Rows ~ N(0, U diag(c i^-alpha) U^T), optionally through an exact-erf GeLU,
    optionally with ``spikes`` random channels scaled to ``spike_var`` x variance."""
    U = random_orthogonal(n, n, seed, _S_BASIS, device)
    A = (power_law(n, alpha, device).sqrt().unsqueeze(1) * U.t()).contiguous()  # diag(sqrt l) U^T
    col_scale = torch.ones(n, device=device)
    if spikes:
        g = _gen(seed, _S_SPIKE, 0, device)
        idx = torch.randperm(n, generator=g, device=device)[:spikes]
        col_scale[idx] = math.sqrt(spike_var)

    def chunk(rows, g):
        z = torch.randn(rows, n, generator=g, device=device)
        x = z @ A
        if gelu:
            x = torch.nn.functional.gelu(x)
        return x * col_scale

    return _chunked_rows(k, n, seed, device, dtype, chunk)


def lowrank_plus_noise_rows(k, n, rank, energy_ratio, seed, device, dtype) -> torch.Tensor:
    """X = Z_r diag(a) P^T + E with P (n x rank) Haar, a_i^2 proportional to i^-1
    (distinct), sum_i a_i^2 * k = energy_ratio * E[||E||^2] and E iid N(0, 1)."""
    P = random_orthogonal(n, rank, seed, _S_SIGNAL, device)
    i = torch.arange(1, rank + 1, device=device, dtype=torch.float64)
    a2 = i.reciprocal()
    a2 = a2 * (energy_ratio * n / a2.sum())
    A = (a2.sqrt().unsqueeze(1) * P.double().t()).float()        # rank x n

    def chunk(rows, g):
        zr = torch.randn(rows, rank, generator=g, device=device)
        e = torch.randn(rows, n, generator=g, device=device)
        return zr @ A + e

    return _chunked_rows(k, n, seed, device, dtype, chunk)


# ----------------------------------------------------------------------------------------
# The five layer workloads. ``scale`` shrinks every dimension (for fast parity runs of the
# same recipe); scale=1 gives the full sizes.
# ----------------------------------------------------------------------------------------

def _dim(x, scale, mult=128):
    return max(mult, int(round(x * scale / mult)) * mult)


def tiny(device="cpu", seed=0) -> Layer:
    n, m, k = 256, 256, 512
    U = random_orthogonal(n, n, seed, _S_BASIS, device)
    s = torch.arange(1, n + 1, device=device, dtype=torch.float32).pow(-0.7)
    A = s.unsqueeze(1) * U
    g = _gen(seed, _S_X, 0, device)
    X = (torch.randn(k, n, generator=g, device=device) @ A).float()
    W = gaussian_weights(m, n, 0.02, torch.float32, seed, device)
    return Layer("tiny 256x256, 512 tokens, 4-bit g128", W, X, 4, 128, 0.01)


def attn(device="cpu", seed=1, scale=1.0) -> Layer:
    n = _dim(1024, scale)
    m = n
    k = _dim(65536, scale, 1024)
    W = gaussian_weights(m, n, 0.02, torch.float32, seed, device)
    n_out = int(round(0.001 * m * n))
    g = _gen(seed, _S_OUTLIER, 0, device)
    idx = torch.randperm(m * n, generator=g, device=device)[:n_out]
    sign = torch.randint(0, 2, (n_out,), generator=g, device=device).float() * 2 - 1
    W.view(-1)[idx] = 10 * 0.02 * sign
    X = correlated_gaussian_rows(k, n, 1.0, seed, device, torch.bfloat16, spikes=8)
    return Layer(f"attn {m}x{n}, {k} tokens, 4-bit g128", W.to(torch.bfloat16), X, 4, 128, 0.01,
                 meta={"outliers": n_out})


def mlp_down(device="cpu", seed=2, scale=1.0) -> Layer:
    n = _dim(6144, scale)
    m = _dim(2048, scale)
    k = _dim(262144, scale, 1024)
    W = gaussian_weights(m, n, 0.015, torch.bfloat16, seed, device)
    X = correlated_gaussian_rows(k, n, 1.0, seed, device, torch.bfloat16, gelu=True)
    return Layer(f"mlp_down {m}x{n}, {k} tokens, 3-bit g128", W, X, 3, 128, 0.01)


def deit(which="fc1", device="cpu", seed=3, scale=1.0) -> Layer:
    d, h = _dim(768, scale), _dim(3072, scale)
    k = _dim(50432, scale, 1024) if scale != 1.0 else 50432
    m, n = (h, d) if which == "fc1" else (d, h)
    sub = 0 if which == "fc1" else 1
    W = gaussian_weights(m, n, 0.02, torch.float32, seed * 2 + sub, device)
    X = correlated_gaussian_rows(k, n, 1.2, seed * 2 + sub, device, torch.bfloat16)
    return Layer(f"deit {which} {m}x{n}, {k} tokens, 2-bit per-channel", W, X, 2, 0, 0.01)


def lowrank(device="cpu", seed=4, scale=1.0, r=64) -> Layer:
    n = _dim(6144, scale)
    m = _dim(2048, scale)
    k = _dim(262144, scale, 1024)
    W = gaussian_weights(m, n, 0.015, torch.bfloat16, seed, device)
    X = lowrank_plus_noise_rows(k, n, r, 100.0, seed, device, torch.bfloat16)
    return Layer(f"lowrank IL r={r} {m}x{n}, {k} tokens, 3-bit g128", W, X, 3, 128, 1e-4, r=r)


WORKLOADS = {
    "tiny": tiny,
    "attn": attn,
    "mlp_down": mlp_down,
    "deit_fc1": lambda **kw: deit("fc1", **kw),
    "deit_fc2": lambda **kw: deit("fc2", **kw),
    "lowrank": lowrank,
}


@dataclass
class TwoSided:
    """A two-sided rounding problem: X (m x n) and the Gram matrices G (m x m), H (n x n)."""
    name: str
    X: torch.Tensor
    G: torch.Tensor
    H: torch.Tensor


def spectral_gram(k, alpha, floor, seed, stream, device) -> torch.Tensor:
    """Q diag(l) Q^T in fp32 (symmetrised in fp64), Q Haar, l = power law (mean 1) + floor."""
    Q = random_orthogonal(k, k, seed, stream, device).double()
    lam = power_law(k, alpha, device).double() + floor
    M = (Q * lam) @ Q.t()
    return ((M + M.t()) * 0.5).float().contiguous()


def two_sided(m=2048, n=6144, device="cpu", seed=5, x_std=3.0, alpha=1.0, floor=0.01) -> TwoSided:
    g = _gen(seed, _S_X, 0, device)
    X = torch.randn(m, n, generator=g, device=device) * x_std
    G = spectral_gram(m, alpha, floor, seed, _S_G2D, device)
    H = spectral_gram(n, alpha, floor, seed, _S_H2D, device)
    return TwoSided(f"two-sided {m}x{n}", X.contiguous(), G, H)
