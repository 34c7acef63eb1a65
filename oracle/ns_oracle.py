"""Plain, slow, fp64 CPU oracle for the Newton-Schulz msign family.

TEST INFRASTRUCTURE ONLY. Nothing in the product package may import this
module. Its only callers are the test-suite, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``.  It shares
no code, constants or tables with the CUDA path; the only thing both sides
consume is the seeded input generator module, which holds none of the
method's arithmetic.

Sources (cited by page title and section/equation):

* [P2] "msign算子的Newton-Schulz迭代（上）" (kexue.fm/archives/10922):
  definition of msign via the SVD (eq. 1-2), the normalised start
  X0 = M/||M||_F and the quintic iteration (eq. 4, 6), Jordan's
  coefficients (eq. 7), the batched reference routine in section
  "参考实现" (cast to bf16, transpose when rows > cols, eps inside the
  square root), the scalar reduction in section "原理分析" and the per-step
  coefficient idea in section "解开约束" (eq. 12).
* [P3] "Gram Newton-Schulz" (zifeng-mai.github.io, 2026/04/05): the muon
  update (section 1.1), FLOP accounting (sections 1.2, 2.4, 3.4),
  Algorithm 1 (Naive Gram Newton-Schulz, section 2.3), Algorithm 2
  (Stabilized Gram Newton-Schulz, section 3.4), Theorem 1 (section 2.2).
* [P5] the Mousse post (anti-entrophic.github.io/posts/10054), section
  "Mousse": the update L^(-1/4) msign(L^(-1/4) G R^(-1/4)) R^(-1/4) with
  Shampoo-style Kronecker factors L and R.

Conventions (readings of the pages where they leave a step open):

* Arithmetic is fp64 throughout.  The only roundings are the explicit
  casts the pages prescribe: the input cast to the compute dtype of [P2]
  "参考实现" (``input_cast='bf16'``) and the fp16 cast of step 2 of
  Algorithm 2 in [P3] section 3.4 (``cast_fp16=True``).
* Orientation: standard NS forms its Gram matrix on the smaller side of X
  (X X^T for rows <= cols, X^T X otherwise), which is why [P2] "参考实现"
  transposes tall inputs; Gram NS works on the wide orientation (n <= m,
  tall inputs transposed and the result transposed back) as [P3]
  Algorithms 1-2 are written for X in R^{n x m} with n <= m.
* Standard NS normalises with sqrt(sum(x^2) + eps), eps = 1e-20 ([P2]
  "参考实现"); Gram NS with ||X||_F + eps, eps = 1e-7 ([P3] Alg. 1 step 1,
  Alg. 2 step 1).
* Coefficients are a list of (a_t, b_t, c_t) triples, one per step; the
  default is Jordan's triple repeated T = 5 times ([P2] eq. 7).

Parity pins: every public function here is checked in
``tests/test_oracle_*.py`` against closed forms, invariants, special cases
and the figures the pages print; none is "parity unpinned".
"""

from __future__ import annotations

import math
from typing import Iterable, Sequence

import numpy as np

# Jordan's quintic coefficients and step count, [P2] eq. (7).
JORDAN_ABC = (3.4445, -4.7750, 2.0315)
JORDAN_STEPS = 5


def jordan_schedule(steps: int = JORDAN_STEPS) -> list[tuple[float, float, float]]:
    """Jordan's constant triple repeated ``steps`` times ([P2] eq. 7)."""
    return [JORDAN_ABC] * steps


# ----------------------------------------------------------------------------
# Casts the pages prescribe (the only non-fp64 roundings in this oracle)
# ----------------------------------------------------------------------------

def round_to_bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 value (ties to even); returns float64.

    bfloat16 keeps the top 16 bits of an IEEE float32.  The input is first
    taken as float32 (the inputs the method receives are float32 or already
    bfloat16-valued), then the low 16 bits are rounded away: add 0x7FFF plus
    the lowest kept bit, and clear the low half.  This is the input rounding
    the routine of [P2] section 参考实现 applies before normalising.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = ((u + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)) << np.uint64(16)
    out = (u & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)
    return out.astype(np.float64).reshape(f.shape)


def round_to_fp16(x) -> np.ndarray:
    """Round to the nearest IEEE half (ties to even); returns float64.

    This is the ``float16(X)`` cast of [P3] Algorithm 2, step 2.
    """
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def _apply_input_cast(x, input_cast):
    if input_cast is None:
        return np.array(x, dtype=np.float64, copy=True)
    if input_cast == "bf16":
        return round_to_bf16(x)
    if input_cast == "fp16":
        return round_to_fp16(x)
    raise ValueError(f"unknown input_cast {input_cast!r}")


def _as_schedule(coeffs) -> list[tuple[float, float, float]]:
    if coeffs is None:
        return jordan_schedule()
    sched = [tuple(float(v) for v in abc) for abc in coeffs]
    for abc in sched:
        if len(abc) != 3:
            raise ValueError("each step needs an (a, b, c) triple")
    return sched


# ----------------------------------------------------------------------------
# Closed forms
# ----------------------------------------------------------------------------

def msign_svd(M) -> np.ndarray:
    """msign(M) = U[:, :r] V[:, :r]^T from the SVD ([P2] eq. 1).

    Every non-zero singular value becomes 1; zero singular values stay 0.
    Rank r is decided with the usual numerical threshold
    max(shape) * eps * sigma_max.
    """
    M = np.asarray(M, dtype=np.float64)
    U, s, Vt = np.linalg.svd(M, full_matrices=False)
    if s.size == 0 or s[0] == 0.0:
        return np.zeros_like(M)
    tol = max(M.shape) * np.finfo(np.float64).eps * s[0]
    r = int(np.sum(s > tol))
    return U[:, :r] @ Vt[:r, :]


def ns_scalar(x, coeffs=None) -> np.ndarray:
    """The scalar map the iteration applies to each singular value.

    x_{t+1} = a_t x_t + b_t x_t^3 + c_t x_t^5  ([P2] section 原理分析 and the
    per-step form of section 解开约束).  Returns x_T for each entry of x.
    """
    x = np.asarray(x, dtype=np.float64).copy()
    for a, b, c in _as_schedule(coeffs):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def msign_ns_closed_form(M, coeffs=None, eps: float = 1e-20) -> np.ndarray:
    """U phi_T(Sigma / ||M||_F) V^T: what T exact NS steps return.

    [P2] section 原理分析 (and [P3] Proposition 1): the iteration keeps the
    singular vectors and maps every normalised singular value through the
    scalar polynomial composed T times.  Uses the same eps convention as
    ``msign_ns`` so the two agree to rounding.
    """
    M = np.asarray(M, dtype=np.float64)
    U, s, Vt = np.linalg.svd(M, full_matrices=False)
    nrm = math.sqrt(float(np.sum(M * M)) + eps)
    return (U * ns_scalar(s / nrm, coeffs)) @ Vt


# ----------------------------------------------------------------------------
# Standard Newton-Schulz msign
# ----------------------------------------------------------------------------

def _gram_side(X):
    """(G, left): the smaller Gram matrix of X and which side it sits on.

    For rows <= cols, G = X X^T (rows x rows) and left = True; otherwise
    G = X^T X (cols x cols) and left = False.  Square matrices take the
    left form."""
    Xt = np.swapaxes(X, -1, -2)
    if X.shape[-2] <= X.shape[-1]:
        return X @ Xt, True
    return Xt @ X, False


def _quintic(X, a, b, c):
    """One step of [P2] eq. 6: X <- a X + b X (X^T X) + c X (X^T X)^2, the
    odd quintic applied to every singular value of X.

    The three terms are formed one by one through the smaller Gram matrix G
    (eq. 6 on the right of X, or the same polynomial written on the left,
    a X + b (X X^T) X + c (X X^T)^2 X, when X is wide): with P1 = G X and
    P2 = G P1 (or X G and P1 G) the step is a X + b P1 + c P2."""
    G, left = _gram_side(X)
    if left:
        P1 = G @ X
        P2 = G @ P1
    else:
        P1 = X @ G
        P2 = P1 @ G
    return a * X + b * P1 + c * P2


def _frobenius_start(X, eps):
    """X0 = X / ||X||_F ([P2] eq. 4), with the routine's guard eps added to
    the sum of squares under the square root."""
    return X / np.sqrt(np.sum(X * X, axis=(-2, -1), keepdims=True) + eps)


def msign_ns(M, coeffs=None, eps: float = 1e-20, input_cast=None) -> np.ndarray:
    """Quintic Newton-Schulz msign, batched over leading dims, in fp64.

    [P2] eq. 4 starts from X0 = M / ||M||_F, which puts every singular value
    in [0, 1]; eq. 6 then applies x -> a x + b x^3 + c x^5 to the singular
    values once per step (one (a, b, c) per step, Jordan's triple by default,
    eq. 7).  The page's routine first rounds the input to the compute dtype
    (``input_cast``; None = no rounding) and guards the norm with eps = 1e-20
    under the square root.  Everything here is fp64; each step is
    ``_quintic`` (which forms the Gram matrix on the smaller side, the
    reason the routine transposes tall inputs).
    """
    X = _apply_input_cast(M, input_cast)
    if X.ndim < 2:
        raise ValueError("msign needs at least a matrix")
    X = _frobenius_start(X, eps)
    for a, b, c in _as_schedule(coeffs):
        X = _quintic(X, a, b, c)
    return np.ascontiguousarray(X)


def msign_ns_improved_init(M, coeffs=None, eps: float = 1e-20, input_cast=None) -> np.ndarray:
    """Standard NS with the sharper initial normalisation of [P2] section
    改进初值, in fp64.

    The Frobenius norm shrinks X0 more than needed.  With G the Gram matrix
    of X0 and sigma its singular values, ||G^2||_F^2 = sum sigma^8, so
    sigma_1 <= (sum sigma^8)^(1/8) = ||G^2||_F^(1/4) <= ||X0||_F = 1.  The
    section therefore divides X0 by nu = ||G^2||_F^(1/4) (eps guards the
    zero matrix: nu = (||G^2||_F^2 + eps)^(1/8)), which keeps sigma_1 <= 1
    while enlarging the small singular values, and then runs the same steps.
    The page reuses the step-0 products (dividing G by nu^2 and G^2 by
    nu^4) to save work; this oracle forms the rescaled X0 and starts over,
    which is the same iteration in exact arithmetic.
    """
    X = _apply_input_cast(M, input_cast)
    if X.ndim < 2:
        raise ValueError("msign needs at least a matrix")
    X = _frobenius_start(X, eps)
    G, _ = _gram_side(X)
    G2 = G @ G
    nu = (np.sum(G2 * G2, axis=(-2, -1), keepdims=True) + eps) ** 0.125
    X = X / nu
    for a, b, c in _as_schedule(coeffs):
        X = _quintic(X, a, b, c)
    return np.ascontiguousarray(X)


# ----------------------------------------------------------------------------
# Gram product
# ----------------------------------------------------------------------------

def gram_xxt(X) -> np.ndarray:
    """A = X X^T, batched over leading dims, fp64 (the symmetric Gram
    product of the flash-muon ``matmul_transpose`` post, nil9.net).
    The result is symmetrised by construction: entry (i, j) and (j, i)
    are the same dot product, so the oracle returns exactly symmetric A."""
    X = np.asarray(X, dtype=np.float64)
    A = X @ np.swapaxes(X, -1, -2)
    upper = np.triu(np.ones(A.shape[-2:], dtype=bool))
    return np.where(upper, A, np.swapaxes(A, -1, -2))


def gram_xxt_bruteforce(X) -> np.ndarray:
    """Triple loop version of X X^T for tiny inputs (a pin for gram_xxt)."""
    X = np.asarray(X, dtype=np.float64)
    n, m = X.shape
    A = np.zeros((n, n))
    for i in range(n):
        for j in range(n):
            acc = 0.0
            for k in range(m):
                acc += X[i, k] * X[j, k]
            A[i, j] = acc
    return A


# ----------------------------------------------------------------------------
# Gram Newton-Schulz ([P3] sections 2.3 and 3.4)
# ----------------------------------------------------------------------------

def _orient(X):
    flip = X.shape[-2] > X.shape[-1]
    return (np.swapaxes(X, -1, -2) if flip else X), flip


def gram_ns_naive(M, coeffs=None, eps: float = 1e-7, input_cast=None) -> np.ndarray:
    """[P3] Algorithm 1 (Naive Gram Newton-Schulz), fp64.

      X <- X / (||X||_F + eps);  R_0 = X X^T;  Q_0 = I;
      for t: Z_t = a_t I + b_t R + c_t R^2;  Q_t = Q_{t-1} Z_t;
             R_t = Z_t R_{t-1} Z_t;
      return Q_T X.
    Wide orientation (n <= m) as in the standard routine.
    """
    X, flip = _orient(_apply_input_cast(M, input_cast))
    X = np.array(X, dtype=np.float64)
    n = X.shape[-2]
    I = np.eye(n)
    X = X / (np.sqrt(np.sum(X * X, axis=(-2, -1), keepdims=True)) + eps)
    R = X @ np.swapaxes(X, -1, -2)
    Q = np.broadcast_to(I, R.shape).copy()
    for a, b, c in _as_schedule(coeffs):
        Z = a * I + b * R + c * (R @ R)
        Q = Q @ Z
        R = Z @ R @ Z
    out = Q @ X
    return np.swapaxes(out, -1, -2) if flip else out


def gram_ns(M, coeffs=None, restart_after: Iterable[int] = (2,), eps: float = 1e-7,
            input_cast=None, cast_fp16: bool = True) -> np.ndarray:
    """[P3] Algorithm 2 (Stabilized Gram Newton-Schulz), fp64 arithmetic.

      1. X <- X / (||X||_F + eps)
      2. X <- float16(X)                     (``cast_fp16``)
      3. for each segment of steps between restarts:
           R <- X X^T ;  Q <- I
           for t in the segment:
             Z  <- b_t R + c_t R^2
             Q  <- Q Z + a_t Q
             RZ <- R Z + a_t R
             R  <- Z RZ + a_t RZ
           X <- Q X                          (the restart)
      4. return X  (= Q X of the last segment)
    ``restart_after`` lists the step numbers after which the Gram matrix is
    recomputed; the page's schedule restarts after step 2 ([P3] section
    3.2).  An empty list gives the unrestarted iteration, and restarting
    after every step reproduces standard NS ([P3] end of section 3.4).
    Every product written in the algorithm is performed, including Q = I Z
    at the first step of a segment; skipping it is a FLOP saving the page
    describes, not a change of result.
    """
    sched = _as_schedule(coeffs)
    T = len(sched)
    cuts = sorted({int(t) for t in restart_after if 0 < int(t) < T})
    bounds = [0] + cuts + [T]
    X, flip = _orient(_apply_input_cast(M, input_cast))
    X = np.array(X, dtype=np.float64)
    n = X.shape[-2]
    I = np.eye(n)
    XT = lambda Y: np.swapaxes(Y, -1, -2)  # noqa: E731
    X = X / (np.sqrt(np.sum(X * X, axis=(-2, -1), keepdims=True)) + eps)
    if cast_fp16:
        X = round_to_fp16(X)
    for s0, s1 in zip(bounds[:-1], bounds[1:]):
        R = X @ XT(X)
        Q = np.broadcast_to(I, R.shape).copy()
        for a, b, c in sched[s0:s1]:
            Z = b * R + c * (R @ R)
            Q = Q @ Z + a * Q
            RZ = R @ Z + a * R
            R = Z @ RZ + a * RZ
        X = Q @ X
    return XT(X) if flip else X


def gram_ns_scalar(x, coeffs=None):
    """[P3] Theorem 1 in scalar form: r_0 = x^2, q_0 = 1,
    z_t = h_t(r_{t-1}) with h_t(y) = a_t + b_t y + c_t y^2 (Lemma 1),
    q_t = q_{t-1} z_t, r_t = r_{t-1} z_t^2.  Returns (q_T, r_T)."""
    x = np.asarray(x, dtype=np.float64)
    r = x * x
    q = np.ones_like(x)
    for a, b, c in _as_schedule(coeffs):
        z = a + b * r + c * r * r
        q = q * z
        r = r * z * z
    return q, r


# ----------------------------------------------------------------------------
# Muon update ([P3] section 1.1, formula lost in extraction; reading below)
# ----------------------------------------------------------------------------

def muon_step(W, M, G, momentum: float = 0.95, lr: float = 0.02, coeffs=None,
              eps: float = 1e-20, input_cast="bf16"):
    """One Muon update of one weight matrix, fp64.

    M <- momentum * M + G;  O = msign_NS(M);  W <- W - lr * sqrt(max(1, rows/cols)) * O.
    The momentum recursion with M_0 = 0 is the one [P3] section 1.1 names
    (mu, eta); the sqrt(max(1, rows/cols)) factor is the spectral scaling
    of the Muon update used by the Llama-shaped workload.  Returns
    (W_new, M_new, O).
    """
    W = np.asarray(W, dtype=np.float64)
    M_new = momentum * np.asarray(M, dtype=np.float64) + np.asarray(G, dtype=np.float64)
    O = msign_ns(M_new, coeffs=coeffs, eps=eps, input_cast=input_cast)
    rows, cols = W.shape[-2], W.shape[-1]
    scale = math.sqrt(max(1.0, rows / cols))
    return W - lr * scale * O, M_new, O


# ----------------------------------------------------------------------------
# Mousse: msign in a space whitened by Shampoo-style Kronecker factors
# (the Mousse post, anti-entrophic.github.io/posts/10054, section "Mousse")
# ----------------------------------------------------------------------------

def spd_inv_root(A, p: int = 4, eps: float = 0.0) -> np.ndarray:
    """(A + eps I)^(-1/p) of a symmetric positive (semi)definite matrix,
    batched over leading dims, from its eigendecomposition in fp64.

    The Mousse post writes its preconditioners as P = L^(1/4) and
    Q = R^(1/4) and uses their inverses; eps is the usual damping that
    keeps a rank-deficient statistic invertible.  Raises ValueError if a
    damped eigenvalue is not positive.
    """
    A = np.asarray(A, dtype=np.float64)
    A = 0.5 * (A + np.swapaxes(A, -1, -2))
    w, V = np.linalg.eigh(A)
    w = w + eps
    if np.any(w <= 0.0):
        raise ValueError("spd_inv_root needs positive damped eigenvalues")
    return (V * w[..., None, :] ** (-1.0 / p)) @ np.swapaxes(V, -1, -2)


def mousse_statistics(G, L=None, R=None, beta: float = 1.0):
    """Shampoo-style Kronecker statistics of a gradient G (rows x cols):
    L <- beta L + G G^T (rows x rows) and R <- beta R + G^T G (cols x cols).

    The post approximates the Hessian by (R kron L)^(1/2) "Shampoo-style"
    and gives no update rule for the two factors; the plainest reading is
    Shampoo's accumulated Gram matrices of the gradient, with beta = 1 a
    running sum and beta < 1 an exponential average.  Returns (L, R)."""
    G = np.asarray(G, dtype=np.float64)
    Gt = np.swapaxes(G, -1, -2)
    GG, GtG = G @ Gt, Gt @ G
    L = GG if L is None else beta * np.asarray(L, dtype=np.float64) + GG
    R = GtG if R is None else beta * np.asarray(R, dtype=np.float64) + GtG
    return L, R


def mousse_direction(G, L, R, coeffs=None, eps: float = 0.0, exact: bool = False) -> np.ndarray:
    """The Mousse direction D = L^(-1/4) msign(L^(-1/4) G R^(-1/4)) R^(-1/4);
    the update is Delta W = -D (times a learning rate).

    From the post: with P = L^(1/4), Q = R^(1/4) the constraint
    ||P Delta W Q||_op <= 1 and Y = P Delta W Q turn min Tr(G^T Delta W)
    into min Tr(G~^T Y) over ||Y||_op <= 1 with G~ = P^-1 G Q^-1, whose
    minimiser is Y = -msign(G~); mapping back gives Delta W =
    -P^-1 msign(G~) Q^-1.  ``exact`` takes msign from the SVD (the
    constrained optimum); otherwise msign is the Newton-Schulz iteration of
    ``msign_ns`` with ``coeffs`` (what an optimizer runs).  L and R are
    damped by eps before their roots are taken.
    """
    G = np.asarray(G, dtype=np.float64)
    Pi = spd_inv_root(L, 4, eps)
    Qi = spd_inv_root(R, 4, eps)
    Gt = Pi @ G @ Qi
    O = msign_svd(Gt) if exact else msign_ns(Gt, coeffs)
    return Pi @ O @ Qi


# ----------------------------------------------------------------------------
# FLOP bookkeeping ([P3] sections 1.2, 2.4, 3.4)
# ----------------------------------------------------------------------------

def ns_flops(n: int, m: int, steps: int = 5, symmetric: bool = True) -> float:
    """FLOPs of standard NS on an n x m matrix (n <= m).

    Per step ([P3] section 1.2): X X^T costs 2 m n^2, A^2 costs 2 n^3 and
    B X costs 2 m n^2.  With symmetric products (only one triangle of the
    two symmetric outputs is needed) the first two halve, giving
    T (3 alpha + 1) n^3 in total ([P3] section 2.4)."""
    sym = 0.5 if symmetric else 1.0
    per = sym * 2 * m * n * n + sym * 2 * n ** 3 + 2 * m * n * n
    return steps * per


def gram_ns_plan(n: int, m: int, steps: int = 5, restart_after: Sequence[int] = (2,)):
    """The list of products a Gram-NS run performs after the savings the
    page lists, with their FLOP cost under the symmetric-GEMM model.

    Per step ([P3] section 2.4): R^2 costs n^3, Q Z costs n^3, Z R Z costs
    2 n^3 (as R Z then Z (R Z)).  Start and end: X X^T costs m n^2 and
    Q X costs 2 m n^2.  Savings: the first Q Z of a segment is Q = Z
    (Q = I), and the last R update of a segment is never used.  A restart
    adds Q X (2 m n^2) and X X^T (m n^2) ([P3] section 3.4).
    Returns a list of (name, flops)."""
    cuts = sorted({int(t) for t in restart_after if 0 < int(t) < steps})
    bounds = [0] + cuts + [steps]
    plan = []
    for s0, s1 in zip(bounds[:-1], bounds[1:]):
        plan.append(("XXt", m * n * n))
        for t in range(s0, s1):
            plan.append((f"R2[{t + 1}]", n ** 3))
            if t != s0:
                plan.append((f"QZ[{t + 1}]", n ** 3))
            if t != s1 - 1:
                plan.append((f"RZ[{t + 1}]", n ** 3))
                plan.append((f"ZRZ[{t + 1}]", n ** 3))
        plan.append(("QX", 2 * m * n * n))
    return plan


def gram_ns_flops(n: int, m: int, steps: int = 5, restart_after: Sequence[int] = (2,)) -> float:
    return float(sum(f for _, f in gram_ns_plan(n, m, steps, restart_after)))
