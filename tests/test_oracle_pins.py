"""Pins for the fp64 oracle: each check ties it to something other than itself
(closed forms from the SVD, library routines, brute force, special cases with
known answers, and the numbers the pages print).  CPU only."""

import math

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import ns_oracle as O
from newton_schulz_msign_b200 import synth

from conftest import load_golden

JORDAN = [(3.4445, -4.7750, 2.0315)] * 5


# ---------------------------------------------------------------- casts

def test_bf16_rounding_matches_torch():
    x = synth.gaussian((4096,), seed=1, std=3.0)
    x = np.concatenate([x, np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5e-3, 0.0, 6.5e4, 3.3e38],
                                    dtype=np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_to_bf16(x), ref)


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 lies half-way between 1 and 1 + 2^-7: the even neighbour is 1.
    assert O.round_to_bf16(np.float32(1.0 + 2 ** -8)) == 1.0
    # 1 + 3*2^-8 lies half-way between 1 + 2^-7 and 1 + 2^-6: the even one is 1 + 2^-6.
    assert O.round_to_bf16(np.float32(1.0 + 3 * 2 ** -8)) == 1.0 + 2 ** -6


def test_fp16_rounding_matches_torch():
    x = synth.gaussian((4096,), seed=2, std=10.0)
    ref = torch.from_numpy(x).to(torch.float64).to(torch.float16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_to_fp16(x), ref)


# ---------------------------------------------------------------- msign by SVD

def test_msign_svd_is_nearest_orthogonal_matrix():
    # msign = argmin_{O^T O = I} ||M - O||_F for square full-rank M (eq. 3 of the
    # msign post); scipy's orthogonal Procrustes solves min ||I R - M||.
    M = synth.gaussian((24, 24), seed=3).astype(np.float64)
    R, _ = scipy.linalg.orthogonal_procrustes(np.eye(24), M)
    np.testing.assert_allclose(O.msign_svd(M), R, atol=1e-12)


@pytest.mark.parametrize("shape", [(16, 40), (40, 16), (20, 20)])
def test_msign_svd_is_inverse_sqrt_form(shape):
    # msign(M) = (M M^T)^{-1/2} M = M (M^T M)^{-1/2} (eq. 2), via scipy's sqrtm.
    M = synth.gaussian(shape, seed=4).astype(np.float64)
    if shape[0] <= shape[1]:
        ref = np.linalg.solve(np.real(scipy.linalg.sqrtm(M @ M.T)), M)
    else:
        ref = np.linalg.solve(np.real(scipy.linalg.sqrtm(M.T @ M)), M.T).T
    np.testing.assert_allclose(O.msign_svd(M), ref, atol=1e-10)


def test_msign_svd_rank_deficient_keeps_zero_singular_values():
    g = synth.rng(5)
    M = g.standard_normal((12, 3)) @ g.standard_normal((3, 20))  # rank 3
    S = np.linalg.svd(O.msign_svd(M), compute_uv=False)
    np.testing.assert_allclose(S[:3], 1.0, atol=1e-12)
    np.testing.assert_allclose(S[3:], 0.0, atol=1e-12)


# ---------------------------------------------------------------- scalar map

def test_scalar_map_single_step_values_at_one():
    # one quintic step at x = 1 is a + b + c; its slope there is a + 3b + 5c.
    a, b, c = JORDAN[0]
    assert O.ns_scalar(1.0, [JORDAN[0]]) == pytest.approx(0.701, abs=1e-12)
    h = 1e-6
    slope = (O.ns_scalar(1 + h, [JORDAN[0]]) - O.ns_scalar(1 - h, [JORDAN[0]])) / (2 * h)
    assert slope == pytest.approx(a + 3 * b + 5 * c, rel=1e-8)


def test_scalar_map_slope_at_zero_is_a_to_the_T():
    # The composed map phi has phi'(0) = a^5 (coefficient-design post, nil9.net).
    h = 1e-9
    d = O.ns_scalar(h, JORDAN) / h
    assert d == pytest.approx(3.4445 ** 5, rel=1e-6)


@pytest.mark.parametrize("name", ["cubic_1p99", "cubic_bernstein"])
def test_cubic_designs_fix_one(coeff_tables, name):
    # f(1) = a + b = 1 for both cubic designs of the coefficient-design post.
    assert O.ns_scalar(1.0, coeff_tables[name]) == pytest.approx(1.0, abs=1e-12)


def test_scalar_map_is_odd():
    x = np.linspace(-1, 1, 101)
    np.testing.assert_allclose(O.ns_scalar(-x, JORDAN), -O.ns_scalar(x, JORDAN), atol=0)


# ---------------------------------------------------------------- NS matrix iteration

@pytest.mark.parametrize("shape", [(8, 8), (16, 48), (48, 16), (33, 70), (1, 9), (9, 1)])
@pytest.mark.parametrize("table", ["jordan", "youjiacheng_6step", "dion_5step", "su_ours_x3_5step"])
def test_ns_matches_svd_closed_form(coeff_tables, shape, table):
    # The iteration keeps the singular vectors and maps each normalised singular
    # value through the composed scalar polynomial (section 原理分析 of the msign
    # post; Proposition 1 of the Gram-NS post).
    M = synth.gaussian(shape, seed=sum(shape)).astype(np.float64)
    sched = coeff_tables[table]
    got = O.msign_ns(M, sched)
    ref = O.msign_ns_closed_form(M, sched)
    np.testing.assert_allclose(got, ref, atol=1e-11 * max(1.0, np.abs(ref).max()))


def test_ns_batched_equals_per_matrix():
    M = synth.gaussian((3, 10, 14), seed=7).astype(np.float64)
    got = O.msign_ns(M)
    for i in range(3):
        np.testing.assert_allclose(got[i], O.msign_ns(M[i]), atol=1e-14)


def test_ns_batched_tall_transposes_per_matrix():
    M = synth.gaussian((2, 14, 10), seed=8).astype(np.float64)
    got = O.msign_ns(M)
    for i in range(2):
        np.testing.assert_allclose(got[i], O.msign_ns_closed_form(M[i]), atol=1e-12)


def test_ns_zero_input_gives_zero():
    assert np.all(O.msign_ns(np.zeros((6, 9))) == 0.0)


def test_ns_row_vector():
    # a single row has one singular value, ||v||; normalised it is 1, so the
    # output is phi_5(1) v / ||v||.
    v = synth.gaussian((1, 37), seed=9).astype(np.float64)
    got = O.msign_ns(v)
    np.testing.assert_allclose(got, O.ns_scalar(1.0, JORDAN) * v / np.linalg.norm(v), atol=1e-14)
    assert O.ns_scalar(1.0, JORDAN) == pytest.approx(0.6964, abs=5e-5)


def test_ns_orthogonal_input():
    # all n singular values of an orthogonal Q are 1, normalised to 1/sqrt(n).
    n = 16
    Q, _ = np.linalg.qr(synth.gaussian((n, n), seed=10).astype(np.float64))
    np.testing.assert_allclose(O.msign_ns(Q), O.ns_scalar(1 / math.sqrt(n), JORDAN) * Q, atol=1e-13)


def test_ns_diagonal_input_keeps_signs():
    d = np.array([3.0, -1.0, 0.5, -0.01, 0.0])
    got = O.msign_ns(np.diag(d))
    expect = np.sign(d) * O.ns_scalar(np.abs(d) / np.linalg.norm(d), JORDAN)
    np.testing.assert_allclose(got, np.diag(expect), atol=1e-14)


def test_ns_output_band_vs_exact_msign():
    # Jordan's quintic does not converge to 1 (a + b + c != 1), so NS output
    # singular values sit in a band around 1 instead of at 1.  For the 256 x 512
    # Gaussian workload (seed 0) all normalised singular values lie in
    # [0.01, 0.11], where phi_5 is in [0.68, 1.14].
    M = np.random.default_rng(0).standard_normal((256, 512))
    s = np.linalg.svd(O.msign_ns(M), compute_uv=False)
    assert 0.68 < s.min() and s.max() < 1.14
    rel = np.linalg.norm(O.msign_ns(M) - O.msign_svd(M)) / np.linalg.norm(O.msign_svd(M))
    assert 0.05 < rel < 0.3


def test_ns_input_cast_bf16_is_applied_first():
    M = synth.gaussian((12, 20), seed=11)
    np.testing.assert_allclose(O.msign_ns(M, input_cast="bf16"), O.msign_ns(O.round_to_bf16(M)), atol=0)


# ---------------------------------------------------------------- Gram product

def test_gram_xxt_bruteforce():
    X = synth.gaussian((5, 7), seed=12).astype(np.float64)
    np.testing.assert_allclose(O.gram_xxt(X), O.gram_xxt_bruteforce(X), rtol=1e-13, atol=1e-13)


def test_gram_xxt_exactly_symmetric():
    X = synth.gaussian((2, 37, 53), seed=13).astype(np.float64)
    A = O.gram_xxt(X)
    assert np.array_equal(A, np.swapaxes(A, -1, -2))


# ---------------------------------------------------------------- Gram Newton-Schulz

def _closed_form_gram(M, sched, eps=1e-7):
    # same as msign_ns_closed_form but with the ||X||_F + eps normalisation of
    # Algorithms 1 and 2 of the Gram-NS post.
    U, s, Vt = np.linalg.svd(M, full_matrices=False)
    return (U * O.ns_scalar(s / (np.linalg.norm(M) + eps), sched)) @ Vt


def test_theorem1_scalar_identity():
    # q_T x_0 = x_T and r_T = x_T^2 (Theorem 1 of the Gram-NS post).
    x = np.linspace(0.0, 1.0, 1001)
    q, r = O.gram_ns_scalar(x, JORDAN)
    xt = O.ns_scalar(x, JORDAN)
    np.testing.assert_allclose(q * x, xt, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(r, xt ** 2, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("shape", [(12, 30), (30, 12), (16, 16)])
def test_gram_ns_naive_matches_closed_form(shape):
    M = synth.gaussian(shape, seed=14).astype(np.float64)
    np.testing.assert_allclose(O.gram_ns_naive(M), _closed_form_gram(M, JORDAN), atol=1e-11)


@pytest.mark.parametrize("restarts", [(), (2,), (1, 3), (1, 2, 3, 4)])
def test_gram_ns_stabilised_matches_closed_form(restarts):
    M = synth.gaussian((20, 64), seed=15).astype(np.float64)
    got = O.gram_ns(M, JORDAN, restart_after=restarts, cast_fp16=False)
    np.testing.assert_allclose(got, _closed_form_gram(M, JORDAN), atol=1e-11)


def test_gram_ns_unrestarted_equals_naive():
    # the "avoid explicit a_t I" rewriting of Algorithm 2 is the same recursion
    # as Algorithm 1 when no restart happens.
    M = synth.gaussian((10, 26), seed=16).astype(np.float64)
    np.testing.assert_allclose(O.gram_ns(M, JORDAN, restart_after=(), cast_fp16=False),
                               O.gram_ns_naive(M, JORDAN), atol=1e-12)


def test_gram_ns_agrees_with_standard_ns():
    # Gram NS is standard NS in exact arithmetic; only the eps conventions
    # differ (1e-7 on the norm vs 1e-20 under the root).
    M = np.random.default_rng(0).standard_normal((64, 128))
    a = O.gram_ns(M, JORDAN, cast_fp16=False)
    b = O.msign_ns(M, JORDAN)
    assert np.linalg.norm(a - b) / np.linalg.norm(b) < 1e-8


def test_gram_ns_fp16_cast_stays_within_tolerance():
    M = synth.gaussian((64, 256), seed=17)
    a = O.gram_ns(M, JORDAN)
    b = O.msign_ns(M, JORDAN)
    assert np.linalg.norm(a - b) / np.linalg.norm(b) < 2e-2


def test_gram_ns_restart_every_step_reduces_to_standard_steps():
    # with a restart after every step each segment is one step from R = X X^T,
    # Q = I: X <- (a I + b R + c R^2) X, which is one standard NS step.
    M = synth.gaussian((9, 21), seed=18).astype(np.float64)
    X = M / (np.linalg.norm(M) + 1e-7)
    for a, b, c in JORDAN:
        A = X @ X.T
        X = a * X + (b * A + c * A @ A) @ X
    np.testing.assert_allclose(O.gram_ns(M, JORDAN, restart_after=(1, 2, 3, 4), cast_fp16=False), X,
                               atol=1e-13)


# ---------------------------------------------------------------- FLOP accounting

def test_flop_formulas_match_page():
    fig = load_golden("flop_figures.json")
    n = 64
    for alpha in (1, 2, 4, 8):
        m = alpha * n
        typ = O.ns_flops(n, m, 5, symmetric=False)
        assert typ == (fig["standard_typical_T5"]["coef_alpha"] * alpha
                       + fig["standard_typical_T5"]["coef_const"]) * n ** 3
        assert O.ns_flops(n, m, 5, symmetric=True) == 5 * (3 * alpha + 1) * n ** 3
        naive = O.gram_ns_plan(n, m, 5, restart_after=())
        assert len(naive) == fig["naive_gram_T5"]["gemms"]
        assert sum(f for _, f in naive) == (fig["naive_gram_T5"]["coef_const"]
                                           + fig["naive_gram_T5"]["coef_alpha"] * alpha) * n ** 3


def test_flop_savings_match_printed_percentages():
    fig = load_golden("flop_figures.json")
    n, m = 64, 256
    sym, typ = O.ns_flops(n, m, 5, True), O.ns_flops(n, m, 5, False)
    naive, rest = O.gram_ns_flops(n, m, 5, ()), O.gram_ns_flops(n, m, 5, (2,))
    assert round(100 * (1 - naive / sym)) == fig["naive_savings_alpha4"]["vs_symmetric_pct"]
    assert round(100 * (1 - naive / typ)) == fig["naive_savings_alpha4"]["vs_typical_pct"]
    assert round(100 * (1 - rest / sym)) == fig["restarted_savings_alpha4"]["vs_symmetric_pct"]
    assert round(100 * (1 - rest / typ)) == fig["restarted_savings_alpha4"]["vs_typical_pct"]
    # the restart's net cost: +3 m n^2 - 3 n^3
    assert rest - naive == 3 * m * n * n - 3 * n ** 3


# ---------------------------------------------------------------- Muon

@pytest.mark.parametrize("shape", [(12, 20), (20, 12)])
def test_muon_step_closed_form(shape):
    W = synth.gaussian(shape, seed=19, std=0.02).astype(np.float64)
    M = synth.gaussian(shape, seed=20, std=1e-3).astype(np.float64)
    G = synth.gaussian(shape, seed=21, std=1e-4).astype(np.float64)
    W1, M1, Ot = O.muon_step(W, M, G, momentum=0.95, lr=0.02, input_cast=None)
    np.testing.assert_allclose(M1, 0.95 * M + G, atol=0)
    scale = math.sqrt(max(1.0, shape[0] / shape[1]))
    np.testing.assert_allclose(W1, W - 0.02 * scale * O.msign_ns_closed_form(0.95 * M + G), atol=1e-12)


# ---------------------------------------------------------------- improved initial normalisation

@pytest.mark.parametrize("shape", [(40, 90), (90, 40), (64, 64)])
def test_improved_init_closed_form(shape):
    # [P2] section 改进初值: rescaling X0 (and its Gram powers) by
    # n = ||(X0 X0^T)^2||_F^(1/4) at step 0 is the plain iteration on the
    # singular values sigma_i / (||M||_F n), with n^8 = sum (sigma_i/||M||_F)^8;
    # written here through the SVD, independently of the oracle's matrix steps
    M = np.random.default_rng(sum(shape)).standard_normal(shape)
    U, s, Vt = np.linalg.svd(M, full_matrices=False)
    x = s / np.sqrt(np.sum(s ** 2) + 1e-20)
    n = (np.sum(x ** 8) + 1e-20) ** 0.125
    expect = (U * O.ns_scalar(x / n)) @ Vt
    got = O.msign_ns_improved_init(M)
    assert np.allclose(got, expect, rtol=1e-10, atol=1e-12)
    # and it is not the plain iteration
    assert not np.allclose(got, O.msign_ns(M), atol=1e-3)


def test_improved_init_raises_small_singular_values():
    # the page's measurement: on 100 x 100 Gaussian matrices the smallest
    # output singular value mostly more than doubles, and the mean singular
    # value moves closer to 1
    ratios, closer = [], 0
    for seed in range(20):
        M = np.random.default_rng(1000 + seed).standard_normal((100, 100))
        s0 = np.linalg.svd(O.msign_ns(M), compute_uv=False)
        s1 = np.linalg.svd(O.msign_ns_improved_init(M), compute_uv=False)
        ratios.append(s1.min() / s0.min())
        closer += abs(s1.mean() - 1) < abs(s0.mean() - 1)
    assert np.median(ratios) >= 2.0
    assert closer >= 18


def test_improved_init_is_a_rescale_of_the_input():
    # the improved iteration on M equals the plain iteration started from
    # X0 / n -- i.e. msign_ns on M scaled so that its Frobenius normalisation
    # lands on X0 / n -- checked on the batch axis as well
    Ms = np.random.default_rng(7).standard_normal((3, 30, 50))
    got = O.msign_ns_improved_init(Ms)
    for i in range(3):
        X0 = Ms[i] / np.sqrt(np.sum(Ms[i] ** 2) + 1e-20)
        A = X0 @ X0.T
        n = (np.sum((A @ A) ** 2) + 1e-20) ** 0.125
        Y = X0 / n
        for a, b, c in [(3.4445, -4.7750, 2.0315)] * 5:
            Y = a * Y + b * (Y @ Y.T) @ Y + c * (Y @ Y.T) @ (Y @ Y.T) @ Y
        assert np.allclose(got[i], Y, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- Mousse

def _spd(n, seed, cond=1e3):
    """Random symmetric positive definite matrix with eigenvalues spread over
    [1/cond, 1] and its eigendecomposition."""
    g = np.random.default_rng(seed)
    q, _ = np.linalg.qr(g.standard_normal((n, n)))
    w = np.logspace(-math.log10(cond), 0, n)
    return (q * w) @ q.T, w, q


@pytest.mark.parametrize("p", [1, 2, 4])
def test_spd_inv_root_inverts_the_power(p):
    A, _, _ = _spd(24, seed=p)
    X = O.spd_inv_root(A, p, eps=1e-3)
    Ad = A + 1e-3 * np.eye(24)
    # X^p (A + eps I) = I, and X is symmetric positive definite
    np.testing.assert_allclose(np.linalg.matrix_power(X, p) @ Ad, np.eye(24), atol=1e-9)
    np.testing.assert_allclose(X, X.T, atol=1e-12)
    assert np.linalg.eigvalsh(X).min() > 0
    if p == 1:
        np.testing.assert_allclose(X, np.linalg.inv(Ad), rtol=1e-9, atol=1e-9)
    if p == 2:
        np.testing.assert_allclose(X, scipy.linalg.inv(scipy.linalg.sqrtm(Ad)).real, rtol=1e-8, atol=1e-9)


def test_spd_inv_root_of_a_diagonal_is_elementwise():
    d = np.array([4.0, 1.0, 0.0625, 16.0])
    np.testing.assert_allclose(O.spd_inv_root(np.diag(d), 4), np.diag([2 ** -0.5, 1.0, 2.0, 0.5]), rtol=1e-14)
    with pytest.raises(ValueError):
        O.spd_inv_root(np.diag([1.0, 0.0]), 4)


def test_mousse_statistics_are_shampoo_gram_sums():
    g1 = synth.gaussian((5, 7), seed=1).astype(np.float64)
    g2 = synth.gaussian((5, 7), seed=2).astype(np.float64)
    L, R = O.mousse_statistics(g1)
    L, R = O.mousse_statistics(g2, L, R, beta=0.5)
    np.testing.assert_allclose(L, 0.5 * np.einsum("ik,jk->ij", g1, g1) + np.einsum("ik,jk->ij", g2, g2))
    np.testing.assert_allclose(R, 0.5 * np.einsum("ki,kj->ij", g1, g1) + np.einsum("ki,kj->ij", g2, g2))


@pytest.mark.parametrize("shape", [(16, 40), (40, 16), (24, 24)])
def test_mousse_with_identity_factors_is_muon(shape):
    G = synth.gaussian(shape, seed=sum(shape)).astype(np.float64)
    r, c = shape
    np.testing.assert_allclose(O.mousse_direction(G, np.eye(r), np.eye(c)), O.msign_ns(G), atol=1e-12)
    np.testing.assert_allclose(O.mousse_direction(G, np.eye(r), np.eye(c), exact=True), O.msign_svd(G), atol=1e-12)


@pytest.mark.parametrize("shape", [(12, 30), (30, 12)])
def test_mousse_exact_direction_solves_the_constrained_problem(shape):
    # the post's problem: min Tr(G^T dW) s.t. ||P dW Q||_op <= 1 with
    # P = L^(1/4), Q = R^(1/4); its minimum is -||P^-1 G Q^-1||_* (nuclear
    # norm), reached at dW = -D, and P D Q has every singular value 1
    r, c = shape
    G = synth.gaussian(shape, seed=r * c).astype(np.float64)
    L, _, _ = _spd(r, seed=r, cond=50.0)
    R, _, _ = _spd(c, seed=c + 1, cond=20.0)
    D = O.mousse_direction(G, L, R, exact=True)
    P = scipy.linalg.fractional_matrix_power(L, 0.25).real
    Q = scipy.linalg.fractional_matrix_power(R, 0.25).real
    np.testing.assert_allclose(np.linalg.svd(P @ D @ Q, compute_uv=False), 1.0, atol=1e-9)
    Gt = np.linalg.solve(P, G) @ np.linalg.inv(Q)
    nuclear = np.linalg.svd(Gt, compute_uv=False).sum()
    assert abs(np.trace(G.T @ (-D)) + nuclear) < 1e-9 * nuclear
    # no other feasible step does better: random directions scaled onto the
    # constraint's boundary
    g = np.random.default_rng(3)
    for _ in range(20):
        Y = g.standard_normal(shape)
        Y /= np.linalg.norm(Y, 2)
        dW = np.linalg.solve(P, Y) @ np.linalg.inv(Q)
        assert np.trace(G.T @ dW) >= -nuclear - 1e-9


def test_mousse_diagonal_factors_scale_rows_and_columns():
    G = synth.gaussian((10, 14), seed=5).astype(np.float64)
    lr_ = np.linspace(0.5, 4.0, 10)
    lc = np.linspace(0.2, 3.0, 14)
    D = O.mousse_direction(G, np.diag(lr_), np.diag(lc), exact=True)
    pr, pc = lr_ ** -0.25, lc ** -0.25
    ref = pr[:, None] * O.msign_svd(pr[:, None] * G * pc[None, :]) * pc[None, :]
    np.testing.assert_allclose(D, ref, atol=1e-12)
    # and the factors' scale only rescales the direction
    D2 = O.mousse_direction(G, 16.0 * np.diag(lr_), 81.0 * np.diag(lc), exact=True)
    np.testing.assert_allclose(D2, D / (2.0 * 3.0), atol=1e-12)
