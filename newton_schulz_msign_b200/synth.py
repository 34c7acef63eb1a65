"""Seeded synthetic inputs for the msign workloads.

This module only draws random matrices; it performs none of the method's
arithmetic, so both the CUDA path and the CPU oracle may consume what it
returns.  Every generator is deterministic in its ``seed``.

Workload recipes (readings of the pages' workloads; "N(0, s)" means
standard deviation s):

* ``gaussian``        i.i.d. N(0, std^2) entries, numpy PCG64 stream.
* ``gram_operand``    square X with entries N(0,1)/sqrt(m), for X X^T.
* ``momentum_like``   U diag(sigma) V^T + noise, with U, V Haar-random
  orthogonal (QR of a Gaussian with the sign of R's diagonal folded in),
  sigma_i proportional to i^-0.8 and scaled so the noise-free matrix has
  unit RMS entry, plus N(0, 1e-3^2) noise.  A power-law spectrum is the
  momentum-like singular-value profile the msign workloads are quoted on.
* ``llama3_8b_layer_shapes`` the seven weight shapes of one Llama-3-8B
  decoder layer (q/o 4096x4096, k/v 1024x4096, gate/up 14336x4096,
  down 4096x14336).
"""

from __future__ import annotations

import numpy as np

LLAMA3_8B_LAYER = (
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 14336, 4096),
    ("up_proj", 14336, 4096),
    ("down_proj", 4096, 14336),
)
LLAMA3_8B_LAYERS = 32


def llama3_8b_layer_shapes():
    """(name, rows, cols) of the seven matrices of one decoder layer."""
    return list(LLAMA3_8B_LAYER)


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def gaussian(shape, seed: int, std: float = 1.0) -> np.ndarray:
    """float32 array of i.i.d. N(0, std^2) entries."""
    g = rng(seed).standard_normal(size=shape, dtype=np.float64) * std
    return g.astype(np.float32)


def gram_operand(n: int, m: int, seed: int) -> np.ndarray:
    """n x m float32 matrix with N(0, 1)/sqrt(m) entries."""
    return gaussian((n, m), seed, std=1.0 / np.sqrt(m))


def _haar_orthogonal(k: int, n: int, g: np.random.Generator) -> np.ndarray:
    """k x n (k >= n) matrix with orthonormal columns, Haar distributed."""
    z = g.standard_normal(size=(k, n))
    q, r = np.linalg.qr(z)
    return q * np.sign(np.diag(r))


def momentum_like(rows: int, cols: int, seed: int, exponent: float = 0.8,
                  noise_std: float = 1e-3) -> np.ndarray:
    """float32 rows x cols matrix U diag(sigma) V^T + noise (see module doc)."""
    g = rng(seed)
    r = min(rows, cols)
    U = _haar_orthogonal(rows, r, g)
    V = _haar_orthogonal(cols, r, g)
    sigma = np.arange(1, r + 1, dtype=np.float64) ** (-exponent)
    sigma *= np.sqrt(rows * cols) / np.linalg.norm(sigma)
    S = (U * sigma) @ V.T
    S += g.standard_normal(size=(rows, cols)) * noise_std
    return S.astype(np.float32)


def momentum_like_torch(rows: int, cols: int, seed: int, device, exponent: float = 0.8,
                        noise_std: float = 1e-3):
    """Device-side version of ``momentum_like`` for full-size workloads.

    Same recipe, drawn with a seeded ``torch.Generator`` on ``device`` and
    orthogonalised with the device QR (fp32), so that multi-GB inputs do
    not take minutes of host time.  Returns a float32 tensor on ``device``.
    """
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    r = min(rows, cols)

    def haar(k):
        z = torch.randn(k, r, generator=gen, device=device, dtype=torch.float32)
        q, rr = torch.linalg.qr(z)
        return q * torch.sign(torch.diagonal(rr))

    U = haar(rows)
    V = haar(cols)
    sigma = torch.arange(1, r + 1, device=device, dtype=torch.float64) ** (-exponent)
    sigma = sigma * (float(np.sqrt(rows * cols)) / torch.linalg.norm(sigma))
    S = (U * sigma.to(torch.float32)) @ V.T
    S += torch.randn(rows, cols, generator=gen, device=device, dtype=torch.float32) * noise_std
    return S


def gaussian_torch(shape, seed: int, device, std: float = 1.0, dtype=None):
    """Seeded N(0, std^2) tensor drawn on ``device`` (float32 unless given)."""
    import torch

    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32) * std
    return t if dtype is None else t.to(dtype)
