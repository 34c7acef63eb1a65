"""Mousse on the GPU against the fp64 oracle: the inverse fourth roots of the
Kronecker factors (fp32-accurate coupled Newton iteration) and the
preconditioned direction L^(-1/4) msign(L^(-1/4) G R^(-1/4)) R^(-1/4)."""

import math

import numpy as np
import pytest
import torch

import newton_schulz_msign_b200 as msb
from newton_schulz_msign_b200 import synth
from oracle import ns_oracle as O

from helpers import TOL_BF16, TOL_FP32, rel_fro, to_np

pytestmark = pytest.mark.gpu


def spd(n, seed, cond):
    """Symmetric positive definite n x n with eigenvalues log-spread over [1/cond, 1]."""
    g = np.random.default_rng(seed)
    q, _ = np.linalg.qr(g.standard_normal((n, n)))
    w = np.logspace(-math.log10(cond), 0, n)
    a = (q * w) @ q.T
    return 0.5 * (a + a.T)


def kronecker_factors(shape, seed, steps=3, eps_rel=1e-3):
    """Shampoo statistics of a few Gaussian gradients and a damping eps
    relative to their scale (L and R of the Mousse post)."""
    L = R = None
    for t in range(steps):
        L, R = O.mousse_statistics(synth.gaussian(shape, seed=seed + t).astype(np.float64), L, R)
    eps = eps_rel * max(np.trace(L) / shape[0], np.trace(R) / shape[1])
    return L, R, eps


def root_tolerance(a, eps):
    """Relative Frobenius error allowed for (A + eps I)^(-1/4) computed with
    ~fp32 products: the fp32-path tolerance, or kappa * 2^-20 where the
    conditioning makes that larger, kappa = (lambda_max + eps) / (lambda_min + eps).

    A root is sensitive to its data in proportion to the condition number:
    a product error of relative size u moves an eigenvalue lambda by about
    u lambda_max, i.e. by u kappa relative to the smallest one, and the root
    of that direction (the largest entries of the result) by a quarter of
    that.  The GPU's 3xTF32 tensor-core products carry u of about 2^-22 to
    2^-20 (truncating accumulation over K); plain fp32 numpy runs of the same
    iteration land near 0.1 kappa 2^-24."""
    w = np.linalg.eigvalsh(a.astype(np.float64))
    kappa = (w.max() + eps) / (w.min() + eps)
    return max(TOL_FP32, kappa * 2.0 ** -20)


@pytest.mark.parametrize("n,cond", [(64, 1e2), (300, 1e4), (520, 1e3), (7, 10.0)])
def test_inv_root_matches_eigendecomposition(n, cond):
    A = np.stack([spd(n, seed=n + s, cond=cond) for s in range(2)])
    a = torch.from_numpy(A.astype(np.float32)).cuda()
    X = msb.mousse_inv_root(a, eps=0.0, iters=24)
    msb.sync_status()
    assert torch.equal(X, X.transpose(-1, -2))
    ref = O.spd_inv_root(to_np(a), 4)
    tol = max(root_tolerance(to_np(a)[b], 0.0) for b in range(2))
    assert rel_fro(to_np(X), ref) < tol
    # and the defining property, X^4 (A + eps I) = I, to the same accuracy
    x = to_np(X)[0]
    assert np.linalg.norm(np.linalg.matrix_power(x, 4) @ to_np(a)[0] - np.eye(n)) / np.sqrt(n) < 4 * tol


def test_inv_root_of_damped_rank_deficient_statistics():
    # G G^T of a 200 x 60 gradient has rank 60: only the damping makes it invertible
    G = synth.gaussian((200, 60), seed=3).astype(np.float64)
    L, _ = O.mousse_statistics(G)
    eps = 1e-2 * np.trace(L) / 200
    a = torch.from_numpy(L.astype(np.float32)).cuda()
    X = msb.mousse_inv_root(a, eps=eps, iters=20)
    msb.sync_status()
    assert rel_fro(to_np(X), O.spd_inv_root(to_np(a), 4, eps)) < root_tolerance(to_np(a), eps)


@pytest.mark.parametrize("shape", [(96, 200), (200, 96), (256, 512), (130, 130)])
def test_direction_matches_oracle(shape):
    rows, cols = shape
    L, R, eps = kronecker_factors(shape, seed=rows + cols)
    G = synth.gaussian((2,) + shape, seed=7 * rows + cols)
    g = torch.from_numpy(G).to(torch.bfloat16).cuda()
    Lr = msb.mousse_inv_root(torch.from_numpy(np.stack([L, L]).astype(np.float32)).cuda(), eps=eps, iters=24)
    Rr = msb.mousse_inv_root(torch.from_numpy(np.stack([R, R]).astype(np.float32)).cuda(), eps=eps, iters=24)
    d = msb.mousse_direction(g, Lr, Rr)
    msb.sync_status()
    got = to_np(d)
    assert np.all(np.isfinite(got))
    for b in range(2):
        ref = O.mousse_direction(to_np(g[b]), L.astype(np.float32), R.astype(np.float32), eps=eps)
        assert rel_fro(got[b], ref) < TOL_BF16


def test_direction_with_identity_factors_is_msign():
    g = torch.from_numpy(synth.gaussian((192, 320), seed=9)).to(torch.bfloat16).cuda()
    eye_l = torch.eye(192, device="cuda")[None]
    eye_r = torch.eye(320, device="cuda")[None]
    d = msb.mousse_direction(g[None], eye_l, eye_r)[0]
    msb.sync_status()
    assert rel_fro(to_np(d), O.msign_ns(to_np(g), input_cast="bf16")) < TOL_BF16
    assert rel_fro(to_np(d), to_np(msb.msign_ns(g))) < TOL_BF16


def test_direction_full_size():
    # the 4096 x 4096 workload: roots of damped Shampoo statistics on the GPU,
    # the direction against the fp64 oracle (which takes its own roots)
    n = 4096
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    Gs = [torch.randn(n, n, generator=gen, device="cuda") * 1e-2 for _ in range(2)]
    L = sum(G @ G.T for G in Gs).double()
    R = sum(G.T @ G for G in Gs).double()
    eps = float(1e-3 * torch.trace(L) / n)
    Lf, Rf = L.float(), R.float()
    Lr = msb.mousse_inv_root(Lf[None], eps=eps, iters=22)
    Rr = msb.mousse_inv_root(Rf[None], eps=eps, iters=22)
    g = synth.momentum_like_torch(n, n, seed=12, device="cuda").to(torch.bfloat16)
    d = msb.mousse_direction(g[None], Lr, Rr)[0]
    msb.sync_status()
    ref = O.mousse_direction(to_np(g), to_np(Lf), to_np(Rf), eps=eps)
    assert rel_fro(to_np(d), ref) < TOL_BF16
