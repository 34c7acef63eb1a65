"""gram_xxt (A = X X^T) on the GPU against the fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import newton_schulz_msign_b200 as msb
from newton_schulz_msign_b200 import synth
from oracle import ns_oracle as O

from helpers import rel_fro, to_np

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "fp16": torch.float16}


def _x(n, m, dt, seed, batch=None):
    shape = (n, m) if batch is None else (batch, n, m)
    x = synth.gaussian(shape, seed=seed, std=1.0 / np.sqrt(max(m, 1)))
    return torch.from_numpy(x).to(TDT[dt]).cuda()


@pytest.mark.parametrize("n,m", [(128, 64), (256, 256), (300, 200), (7, 129), (1, 8), (513, 1000),
                                 (640, 777), (129, 8), (1000, 72)])
@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_gram_xxt_fp32_out_matches_oracle(n, m, dt):
    x = _x(n, m, dt, seed=n * 7919 + m)
    A = msb.gram_xxt(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = O.gram_xxt(to_np(x))
    # fp32 accumulation of exact products: relative error ~ sqrt(m) * 2^-24
    assert rel_fro(to_np(A), ref) < 1e-5
    assert torch.equal(A, A.transpose(-1, -2))


@pytest.mark.parametrize("n,m", [(8, 200000), (300, 70000)])
def test_gram_xxt_long_inner_dimension(n, m):
    # few tiles over a very long K: the product splits along K and the last
    # part adds the fp32 partials.  The tensor cores' fp32 accumulation
    # truncates instead of rounding, so a sum of m positive products (the
    # diagonal) drifts low by up to about 2^-22 of the running sum per
    # 16-wide MMA step: the bound is (m / 16) * 2^-22, 3e-3 at m = 200000
    # (measured 9.4e-4 there, every diagonal entry below the fp64 value)
    x = _x(n, m, "bf16", seed=n + m)
    A = msb.gram_xxt(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = O.gram_xxt(to_np(x))
    assert rel_fro(to_np(A), ref) < (m / 16) * 2.0 ** -22
    assert torch.equal(A, A.transpose(-1, -2))


@pytest.mark.parametrize("n,m", [(256, 512), (384, 128), (100, 300), (7, 129)])
@pytest.mark.parametrize("dt", ["bf16", "fp16"])
def test_gram_xxt_same_dtype_out(n, m, dt):
    x = _x(n, m, dt, seed=n + 31 * m)
    A = msb.gram_xxt(x)
    torch.cuda.synchronize()
    ref = O.gram_xxt(to_np(x))
    got = to_np(A)
    # one rounding of the fp32 result to the output dtype
    ulp = 2.0 ** -8 if dt == "bf16" else 2.0 ** -11
    assert np.all(np.abs(got - ref) <= ulp * np.abs(ref) + 1e-6 * np.abs(ref).max())
    assert torch.equal(A, A.transpose(-1, -2))


def test_gram_xxt_batched():
    x = _x(200, 300, "bf16", seed=5, batch=3)
    A = msb.gram_xxt(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = O.gram_xxt(to_np(x))
    assert rel_fro(to_np(A), ref) < 1e-5
    assert torch.equal(A, A.transpose(-1, -2))


def test_gram_xxt_zero_and_empty():
    x = torch.zeros(64, 128, dtype=torch.bfloat16, device="cuda")
    A = msb.gram_xxt(x)
    assert torch.count_nonzero(A).item() == 0
    e = torch.zeros(0, 32, dtype=torch.bfloat16, device="cuda")
    assert msb.gram_xxt(e).shape == (0, 0)
    z = torch.zeros(5, 0, dtype=torch.bfloat16, device="cuda")
    A = msb.gram_xxt(z, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert A.shape == (5, 5) and torch.count_nonzero(A).item() == 0


@pytest.mark.parametrize("n", [1024, 2048, 4096, 8192])
def test_gram_xxt_sweep_full_size(n):
    # the square Gram sweep: X n x n bf16 with N(0,1)/sqrt(n) entries, A stored
    # bf16.  Exact symmetry everywhere; sampled rows checked against fp64 dot
    # products of the same bf16 inputs.
    gen = torch.Generator(device="cuda")
    gen.manual_seed(n)
    x = (torch.randn(n, n, generator=gen, device="cuda") / np.sqrt(n)).to(torch.bfloat16)
    A = msb.gram_xxt(x)
    A32 = msb.gram_xxt(x, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(A, A.T)
    assert torch.equal(A32, A32.T)
    rows = np.random.default_rng(n).choice(n, size=48, replace=False)
    X = to_np(x)
    ref = X[rows] @ X.T
    # the tensor core accumulates K = n products in fp32 without rounding each
    # partial sum to nearest; the error grows with K (1.8e-5 measured at
    # K = 8192), far below anything an indexing mistake would produce
    assert rel_fro(to_np(A32[rows]), ref) < 1e-4
    got = to_np(A[rows])
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * np.abs(ref).max())
