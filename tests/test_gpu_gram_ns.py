"""gram_ns (Stabilized Gram Newton-Schulz, fp16 inner iteration) on the GPU
against the fp64 oracle of the same algorithm and of standard NS."""

import numpy as np
import pytest
import torch

import newton_schulz_msign_b200 as msb
from newton_schulz_msign_b200 import synth
from oracle import ns_oracle as O

from helpers import TOL_BF16, rel_fro, to_np

pytestmark = pytest.mark.gpu


def run(x_np, restarts=(2,), coeffs=None, dt=torch.bfloat16):
    x = torch.from_numpy(np.ascontiguousarray(x_np, dtype=np.float32)).to(dt).cuda()
    y = msb.gram_ns(x, restart_after=restarts, coeffs=coeffs)
    msb.sync_status()
    X = to_np(x)
    return to_np(y), X


@pytest.mark.parametrize("shape", [(128, 512), (256, 1024), (100, 300), (300, 100), (64, 64), (7, 129),
                                   (1, 40), (384, 2048)])
def test_gram_ns_shapes(shape):
    got, X = run(synth.gaussian(shape, seed=shape[0] + 7 * shape[1]))
    assert rel_fro(got, O.gram_ns(X)) < TOL_BF16
    assert rel_fro(got, O.msign_ns(X)) < TOL_BF16


@pytest.mark.parametrize("shape", [(300, 6000), (520, 9000), (6000, 300)])
def test_gram_ns_split_k(shape):
    # few tiles and a long inner dimension: X X^T runs as several K parts
    # (the last one ragged) whose fp32 partials are summed in a fixed order
    got, X = run(synth.gaussian(shape, seed=shape[0] + shape[1]))
    assert rel_fro(got, O.gram_ns(X)) < TOL_BF16


@pytest.mark.parametrize("restarts", [(), (1,), (2,), (3,), (1, 3), (1, 2, 3, 4)])
def test_gram_ns_restart_schedules(restarts):
    got, X = run(synth.gaussian((192, 768), seed=11), restarts=restarts)
    assert rel_fro(got, O.gram_ns(X, restart_after=restarts)) < TOL_BF16
    assert rel_fro(got, O.msign_ns(X)) < TOL_BF16


@pytest.mark.parametrize("table", ["dion_5step", "su_ours_x3_5step", "youjiacheng_6step"])
def test_gram_ns_coefficient_tables(coeff_tables, table):
    sched = coeff_tables[table]
    got, X = run(synth.gaussian((128, 512), seed=12), coeffs=sched)
    assert rel_fro(got, O.gram_ns(X, sched)) < TOL_BF16


def test_gram_ns_batched_and_fp32_io():
    got, X = run(synth.gaussian((3, 96, 400), seed=13), dt=torch.float32)
    assert rel_fro(got, O.gram_ns(X)) < TOL_BF16


def test_gram_ns_zero_input():
    x = torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda")
    y = msb.gram_ns(x)
    msb.sync_status()
    assert torch.count_nonzero(y).item() == 0


def test_gram_ns_momentum_like():
    got, X = run(synth.momentum_like(256, 2048, seed=14))
    assert rel_fro(got, O.gram_ns(X)) < TOL_BF16
    assert rel_fro(got, O.msign_ns(X)) < TOL_BF16


@pytest.mark.parametrize("n,m", [(1024, 4096), (1024, 16384), (2048, 4096), (2048, 16384)])
def test_gram_ns_wide_full_size(n, m):
    # the wide workload: N(0,1) bf16 X, fp16 Gram iteration, restart after step 2;
    # checked against the oracle of Algorithm 2 and against standard NS
    x = synth.gaussian_torch((n, m), seed=n + m, device="cuda").to(torch.bfloat16)
    y = msb.gram_ns(x)
    msb.sync_status()
    X = to_np(x)
    got = to_np(y)
    assert np.all(np.isfinite(got))
    assert rel_fro(got, O.gram_ns(X)) < TOL_BF16
    assert rel_fro(got, O.msign_ns(X)) < TOL_BF16


def test_gram_ns_in_place():
    x = torch.from_numpy(synth.gaussian((384, 2048), seed=91)).to(torch.bfloat16).cuda()
    ref = msb.gram_ns(x)
    y = x.clone()
    msb.gram_ns(y, y)
    msb.sync_status()
    assert torch.equal(y, ref)
