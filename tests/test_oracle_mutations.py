"""Planted mistakes in the oracle, each caught by a pin.

A pin is worth what it catches.  Each case copies the source of one oracle
function, changes one expression the way a plausible slip would (a dropped
term, swapped coefficients, a wrong sign, a transposed operand, a wrong
exponent, a skipped step), installs the changed function in the oracle module
for the duration of the test, and runs the pin that guards that function: the
pin must fail.  The mistakes are planted in the oracle only, on the CPU; the
oracle itself is restored after each case."""

import __future__
import inspect

import pytest

from oracle import ns_oracle as O

import test_oracle_pins as P


def plant(monkeypatch, name, old, new):
    """Replace oracle function `name` by its own source with `old` changed to `new`."""
    src = inspect.getsource(getattr(O, name))
    assert src.count(old) == 1, f"{name}: {old!r} is not in its source exactly once"
    code = compile(src.replace(old, new), f"<{name} with a planted mistake>", "exec",
                   flags=__future__.annotations.compiler_flag, dont_inherit=True)
    scope = {}
    exec(code, O.__dict__, scope)  # the changed function sees the oracle's module globals
    monkeypatch.setattr(O, name, scope[name])


def ns_closed_form(tabs, shape=(16, 48)):
    P.test_ns_matches_svd_closed_form(tabs, shape, "jordan")


def gram_closed_form(tabs):
    P.test_gram_ns_stabilised_matches_closed_form((2,))


CASES = [
    # standard NS step ([P2] eq. 6)
    ("quintic: b and c swapped", "_quintic", "a * X + b * P1 + c * P2", "a * X + c * P1 + b * P2", ns_closed_form),
    ("quintic: a X dropped", "_quintic", "a * X + b * P1 + c * P2", "b * P1 + c * P2", ns_closed_form),
    ("quintic: sign of the cubic term", "_quintic", "a * X + b * P1 + c * P2", "a * X - b * P1 + c * P2",
     ns_closed_form),
    ("quintic: second Gram power dropped", "_quintic", "P2 = G @ P1", "P2 = G @ X", ns_closed_form),
    ("quintic: operands in the wrong order", "_quintic", "P1 = G @ X", "P1 = X @ G",
     lambda t: ns_closed_form(t, (8, 8))),
    ("quintic: tall side in the wrong order", "_quintic", "P1 = X @ G", "P1 = G @ X",
     lambda t: ns_closed_form(t, (48, 16))),
    # normalisation and loop ([P2] eq. 4, section 参考实现)
    ("start: squared norm", "_frobenius_start", "np.sqrt(np.sum(X * X, axis=(-2, -1), keepdims=True) + eps)",
     "(np.sum(X * X, axis=(-2, -1), keepdims=True) + eps)", ns_closed_form),
    ("msign_ns: first step skipped", "msign_ns", "for a, b, c in _as_schedule(coeffs):",
     "for a, b, c in _as_schedule(coeffs)[1:]:", ns_closed_form),
    ("msign_ns: input cast not applied", "msign_ns", "X = _apply_input_cast(M, input_cast)",
     "X = np.array(M, dtype=np.float64)", lambda t: P.test_ns_input_cast_bf16_is_applied_first()),
    # the closed forms the pins compare with
    ("scalar map: cube written as square", "ns_scalar", "b * x ** 3", "b * x ** 2", ns_closed_form),
    ("closed form: singular values not normalised", "msign_ns_closed_form", "ns_scalar(s / nrm, coeffs)",
     "ns_scalar(s, coeffs)", ns_closed_form),
    ("svd msign keeps the singular values", "msign_svd", "return U[:, :r] @ Vt[:r, :]",
     "return (U[:, :r] * s[:r]) @ Vt[:r, :]", lambda t: P.test_msign_svd_is_nearest_orthogonal_matrix()),
    # casts
    ("bf16: truncation", "round_to_bf16", "u + np.uint64(0x7FFF) + keep_lsb", "u",
     lambda t: P.test_bf16_rounding_matches_torch()),
    ("bf16: ties away from zero", "round_to_bf16", "np.uint64(0x7FFF) + keep_lsb", "np.uint64(0x8000)",
     lambda t: P.test_bf16_rounding_ties_to_even()),
    # sharper initial normalisation ([P2] section 改进初值)
    ("improved init: fourth root instead of eighth", "msign_ns_improved_init", "** 0.125", "** 0.25",
     lambda t: P.test_improved_init_closed_form((40, 90))),
    ("improved init: multiplies by the bound", "msign_ns_improved_init", "X = X / nu", "X = X * nu",
     lambda t: P.test_improved_init_closed_form((90, 40))),
    # X X^T
    ("gram_xxt: X^T X", "gram_xxt", "A = X @ np.swapaxes(X, -1, -2)", "A = np.swapaxes(X, -1, -2) @ X",
     lambda t: P.test_gram_xxt_bruteforce()),
    ("gram_xxt: lower triangle left empty", "gram_xxt", "np.where(upper, A, np.swapaxes(A, -1, -2))",
     "np.where(upper, A, 0.0)", lambda t: P.test_gram_xxt_bruteforce()),
    # Gram NS ([P3] Algorithms 1 and 2, Theorem 1)
    ("naive Gram NS: R multiplied on one side", "gram_ns_naive", "R = Z @ R @ Z", "R = Z @ R",
     lambda t: P.test_gram_ns_naive_matches_closed_form((12, 30))),
    ("naive Gram NS: Q not accumulated", "gram_ns_naive", "Q = Q @ Z", "Q = Z",
     lambda t: P.test_gram_ns_naive_matches_closed_form((30, 12))),
    ("Gram NS: a Q dropped", "gram_ns", "Q = Q @ Z + a * Q", "Q = Q @ Z", gram_closed_form),
    ("Gram NS: a Z instead of a R", "gram_ns", "RZ = R @ Z + a * R", "RZ = R @ Z + a * Z", gram_closed_form),
    ("Gram NS: sign of a RZ", "gram_ns", "R = Z @ RZ + a * RZ", "R = Z @ RZ - a * RZ", gram_closed_form),
    ("Gram NS: restart product skipped", "gram_ns", "X = Q @ X", "X = X", gram_closed_form),
    ("Theorem 1: r updated by z once", "gram_ns_scalar", "r = r * z * z", "r = r * z",
     lambda t: P.test_theorem1_scalar_identity()),
    # FLOP bookkeeping ([P3] sections 1.2, 2.4, 3.4)
    ("flops: A^2 not halved", "ns_flops", "sym * 2 * n ** 3", "2 * n ** 3",
     lambda t: P.test_flop_formulas_match_page()),
    ("flops: first Q Z of a segment counted", "gram_ns_plan", "if t != s0:", "if True:",
     lambda t: P.test_flop_savings_match_printed_percentages()),
    # Muon ([P3] section 1.1)
    ("muon: scale of the wrong aspect", "muon_step", "max(1.0, rows / cols)", "max(1.0, cols / rows)",
     lambda t: P.test_muon_step_closed_form((20, 12))),
    ("muon: momentum factor dropped", "muon_step", "momentum * np.asarray(M, dtype=np.float64)",
     "np.asarray(M, dtype=np.float64)", lambda t: P.test_muon_step_closed_form((12, 20))),
    # Mousse (the Mousse post, section "Mousse")
    ("inverse root: sign of the exponent", "spd_inv_root", "** (-1.0 / p)", "** (1.0 / p)",
     lambda t: P.test_spd_inv_root_inverts_the_power(4)),
    ("Mousse: right back-projection dropped", "mousse_direction", "return Pi @ O @ Qi", "return Pi @ O",
     lambda t: P.test_mousse_exact_direction_solves_the_constrained_problem((12, 30))),
    ("Mousse: left projection dropped", "mousse_direction", "Gt = Pi @ G @ Qi", "Gt = G @ Qi",
     lambda t: P.test_mousse_exact_direction_solves_the_constrained_problem((30, 12))),
    ("Mousse statistics: decay dropped", "mousse_statistics",
     "L = GG if L is None else beta * np.asarray(L, dtype=np.float64) + GG",
     "L = GG if L is None else np.asarray(L, dtype=np.float64) + GG",
     lambda t: P.test_mousse_statistics_are_shampoo_gram_sums()),
]


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # some planted mistakes overflow
@pytest.mark.parametrize("name,fn,old,new,pin", CASES, ids=[c[0] for c in CASES])
def test_pin_catches_planted_mistake(monkeypatch, coeff_tables, name, fn, old, new, pin):
    pin(coeff_tables)  # the pin passes on the oracle as it is
    plant(monkeypatch, fn, old, new)
    with pytest.raises((AssertionError, ValueError)):
        pin(coeff_tables)
