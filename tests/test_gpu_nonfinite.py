"""Non-finite and zero inputs on the GPU: every entry point returns normally
(no bounded wait runs out), NaN or Inf in one matrix of a batch reaches that
matrix's output and no other, and a zero matrix maps to zero."""

import numpy as np
import pytest
import torch

import newton_schulz_msign_b200 as msb
from newton_schulz_msign_b200 import synth
from oracle import ns_oracle as O

from helpers import TOL_BF16, TOL_FP32, rel_fro, to_np

pytestmark = pytest.mark.gpu


def poisoned_batch(shape, seed, dtype=torch.bfloat16):
    """A batch of three matrices: 0 clean, 1 with one NaN, 2 with one +Inf."""
    x = torch.from_numpy(synth.gaussian((3,) + shape, seed=seed)).to(dtype).cuda()
    x[1, shape[0] // 3, shape[1] // 2] = float("nan")
    x[2, shape[0] - 1, 0] = float("inf")
    return x


@pytest.mark.parametrize("compute", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("shape", [(96, 200), (300, 140)])
def test_msign_ns_nonfinite_stays_in_its_matrix(compute, shape):
    x = poisoned_batch(shape, seed=shape[0] + shape[1], dtype=torch.float32 if compute == "fp32" else torch.bfloat16)
    y = msb.msign_ns(x, compute=compute)
    msb.sync_status()  # raises on a timed-out wait
    got = to_np(y)
    assert not np.all(np.isfinite(got[1])) and not np.all(np.isfinite(got[2]))
    assert np.all(np.isfinite(got[0]))
    cast = {"bf16": "bf16", "fp16": "fp16", "fp32": None}[compute]
    tol = TOL_FP32 if compute == "fp32" else TOL_BF16
    assert rel_fro(got[0], O.msign_ns(to_np(x[0]), input_cast=cast)) < tol


def test_msign_ns_auto_route_nonfinite():
    # the Gram-NS route (fp16 inside): a NaN input must not leave the matrix
    x = torch.from_numpy(synth.gaussian((2, 512, 4608), seed=5)).to(torch.bfloat16).cuda()
    x[1, 7, 11] = float("nan")
    assert msb.msign_ns_route(2, 512, 4608, method="auto") == "gram"
    y = msb.msign_ns(x, method="auto")
    msb.sync_status()
    got = to_np(y)
    assert np.all(np.isfinite(got[0])) and not np.all(np.isfinite(got[1]))
    assert rel_fro(got[0], O.gram_ns(to_np(x[0]))) < TOL_BF16


def test_gram_xxt_nan_poisons_one_row_and_column():
    x = torch.from_numpy(synth.gaussian((2, 300, 200), seed=8, std=0.07)).to(torch.bfloat16).cuda()
    x[1, 37, 150] = float("nan")
    A = msb.gram_xxt(x, out_dtype=torch.float32)
    msb.sync_status()
    a = to_np(A)
    # batch entry 0 untouched
    assert rel_fro(a[0], O.gram_xxt(to_np(x[0]))) < 1e-5
    # entry 1: row and column 37 are NaN (each holds a product with the NaN),
    # everything else is the exact Gram product of the clean rows
    nan = np.isnan(a[1])
    assert nan[37, :].all() and nan[:, 37].all()
    keep = np.ones(300, dtype=bool)
    keep[37] = False
    assert not nan[np.ix_(keep, keep)].any()
    X = to_np(x[1])[keep]
    assert rel_fro(a[1][np.ix_(keep, keep)], O.gram_xxt(X)) < 1e-5
    assert np.array_equal(np.isnan(a[1]), np.isnan(a[1].T))


def test_gram_ns_nonfinite_stays_in_its_matrix():
    x = poisoned_batch((128, 512), seed=9)
    y = msb.gram_ns(x)
    msb.sync_status()
    got = to_np(y)
    assert np.all(np.isfinite(got[0]))
    assert not np.all(np.isfinite(got[1])) and not np.all(np.isfinite(got[2]))
    assert rel_fro(got[0], O.gram_ns(to_np(x[0]))) < TOL_BF16


def test_muon_step_nan_gradient_stays_in_its_matrix():
    shapes = [(128, 256), (128, 256), (256, 96)]
    W = [synth.gaussian_torch(s, seed=10 + i, device="cuda", std=0.02) for i, s in enumerate(shapes)]
    M = [torch.zeros(s, device="cuda") for s in shapes]
    G = [synth.gaussian_torch(s, seed=20 + i, device="cuda", std=1e-4) for i, s in enumerate(shapes)]
    G[1][3, 4] = float("nan")
    W0 = [w.clone() for w in W]
    msb.muon_step(W, M, G, momentum=0.95, lr=0.02)
    msb.sync_status()
    assert not torch.isfinite(W[1]).all() and not torch.isfinite(M[1]).all()
    for i in (0, 2):
        assert torch.isfinite(W[i]).all() and torch.isfinite(M[i]).all()
        Wr, _, _ = O.muon_step(to_np(W0[i]), np.zeros(shapes[i]), to_np(G[i]), momentum=0.95, lr=0.02)
        assert rel_fro(to_np(W[i]) - to_np(W0[i]), Wr - to_np(W0[i])) < TOL_BF16


@pytest.mark.parametrize("compute,method", [("fp16", "standard"), ("fp32", "standard"), ("bf16", "auto")])
def test_zero_matrix_maps_to_zero(compute, method):
    # the eps of each normalisation keeps 0 / ||0|| at 0 on every path
    shape = (2, 512, 4608) if method == "auto" else (2, 96, 160)
    x = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    y = msb.msign_ns(x, compute=compute, method=method)
    msb.sync_status()
    assert torch.count_nonzero(y).item() == 0
