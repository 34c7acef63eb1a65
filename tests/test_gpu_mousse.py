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


@pytest.mark.parametrize("n,cond", [(64, 1e2), (300, 1e4), (520, 1e3), (7, 10.0)])
def test_inv_root_matches_eigendecomposition(n, cond):
    A = np.stack([spd(n, seed=n + s, cond=cond) for s in range(2)])
    a = torch.from_numpy(A.astype(np.float32)).cuda()
    X = msb.mousse_inv_root(a, eps=0.0, iters=24)
    msb.sync_status()
    assert torch.equal(X, X.transpose(-1, -2))
    ref = O.spd_inv_root(to_np(a), 4)
    assert rel_fro(to_np(X), ref) < TOL_FP32


def test_inv_root_of_damped_rank_deficient_statistics():
    # G G^T of a 200 x 60 gradient has rank 60: only the damping makes it invertible
    G = synth.gaussian((200, 60), seed=3).astype(np.float64)
    L, _ = O.mousse_statistics(G)
    eps = 1e-2 * np.trace(L) / 200
    a = torch.from_numpy(L.astype(np.float32)).cuda()
    X = msb.mousse_inv_root(a, eps=eps, iters=20)
    msb.sync_status()
    assert rel_fro(to_np(X), O.spd_inv_root(to_np(a), 4, eps)) < TOL_FP32


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
