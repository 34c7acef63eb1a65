"""The seeded input generators follow the stated recipes (CPU only): the
same seed gives the same matrix, the Gaussian draws have the stated spread,
and a momentum-like matrix has the power-law spectrum and unit RMS entry
its recipe names, from numpy on the host and from torch on a device."""

import numpy as np
import torch

from newton_schulz_msign_b200 import synth


def test_same_seed_same_matrix():
    assert np.array_equal(synth.gaussian((7, 9), seed=3), synth.gaussian((7, 9), seed=3))
    assert not np.array_equal(synth.gaussian((7, 9), seed=3), synth.gaussian((7, 9), seed=4))
    assert np.array_equal(synth.momentum_like(40, 60, seed=5), synth.momentum_like(40, 60, seed=5))
    a = synth.momentum_like_torch(40, 60, seed=5, device="cpu")
    assert torch.equal(a, synth.momentum_like_torch(40, 60, seed=5, device="cpu"))


def test_gaussian_spread():
    x = synth.gaussian((400, 500), seed=1, std=0.02)
    assert x.dtype == np.float32
    assert abs(x.mean()) < 1e-3 * 0.02 * 50
    assert abs(x.std() / 0.02 - 1) < 0.01
    g = synth.gram_operand(64, 4096, seed=2)
    assert abs(g.std() * np.sqrt(4096) - 1) < 0.02


def _check_momentum_like(S, rows, cols, noise_std=1e-3):
    r = min(rows, cols)
    s = np.linalg.svd(S.astype(np.float64), compute_uv=False)
    # unit RMS entry (the noise adds noise_std^2 to the mean square)
    assert abs(np.sqrt(np.mean(S.astype(np.float64) ** 2)) - 1) < 1e-3
    # sigma_i proportional to i^-0.8 over the head of the spectrum, where
    # the noise (spectral norm ~ noise_std (sqrt(rows) + sqrt(cols))) is negligible
    i = np.arange(1, r + 1)
    ref = i ** -0.8 * np.sqrt(rows * cols) / np.linalg.norm(i ** -0.8)
    head = slice(0, r // 2)
    np.testing.assert_allclose(s[head], ref[head], rtol=5e-3)
    assert s[-1] < ref[-1] + 4 * noise_std * (np.sqrt(rows) + np.sqrt(cols))


def test_momentum_like_recipe_host():
    _check_momentum_like(synth.momentum_like(120, 300, seed=7), 120, 300)
    _check_momentum_like(synth.momentum_like(300, 120, seed=8), 300, 120)


def test_momentum_like_recipe_device():
    S = synth.momentum_like_torch(120, 300, seed=9, device="cpu")
    assert S.dtype == torch.float32 and tuple(S.shape) == (120, 300)
    _check_momentum_like(S.numpy(), 120, 300)


def test_llama_layer_shapes():
    shapes = synth.llama3_8b_layer_shapes()
    assert [n for n, _, _ in shapes] == ["q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj"]
    params = sum(r * c for _, r, c in shapes) * synth.LLAMA3_8B_LAYERS
    assert abs(params - 6.98e9) / 6.98e9 < 1e-3  # the 32-layer stack's matrix parameters
