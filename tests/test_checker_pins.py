"""Pins of the oracle's checker functions and of its multi-step driver.

Every parity assertion goes through ``oracle.rel_fro`` (relative Frobenius error,
the error metric the parity bound is stated in) and ``oracle.orthogonality_error``
(max |P^T P - I|, the bound on the GPU's own P), and the fixed-B workload goes
through ``oracle.run_steps(..., reset_momentum=True)``.  They are pinned here by
values worked out by hand and by closed forms, not by the functions themselves, and
each plausible slip (dividing by the wrong norm, the raw numerator at a zero
reference, P P^T for P^T P, a signed maximum, a dropped identity, a momentum reset
that is ignored or applied after the step) is planted in a copy at the end of this
file and must trip at least one pin.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import dion_oracle as od


# ------------------------------------------------------------------ rel_fro

def pin_rel_fro_hand(rel):
    """||(0,4) - (0,5)|| / ||(0,5)|| = 1/5; the 3-4-5 triangle: ||(3,4)|| = 5."""
    errs = [
        abs(rel(np.array([[0.0, 4.0]]), np.array([[0.0, 5.0]])) - 0.2),
        abs(rel(np.array([[3.0, 4.0]]), np.array([[0.0, 8.0]])) - 5.0 / 8.0),
        # a 2x2 case: difference (1, -2; 2, 0) has norm 3, reference norm 6
        abs(rel(np.array([[3.0, 0.0], [2.0, 4.0]]), np.array([[2.0, 2.0], [0.0, 4.0]]))
            - 3.0 / math.sqrt(24.0)),
    ]
    return max(errs)


def pin_rel_fro_zero_reference(rel):
    """A zero reference gives the absolute norm of the difference, and 0 when both are 0
    (the documented convention: a kernel that returns garbage for a zero reference must
    not read as exact)."""
    return max(abs(rel(np.array([[3.0, 4.0]]), np.zeros((1, 2))) - 5.0),
               abs(rel(np.zeros((2, 3)), np.zeros((2, 3))) - 0.0))


def pin_rel_fro_scale_and_symmetry(rel):
    """rel(c a, c b) = rel(a, b) for c != 0; rel(b + e, b) depends on ||e|| only
    (sign and placement of e do not matter)."""
    rng = np.random.default_rng(31)
    a = rng.standard_normal((5, 4))
    b = rng.standard_normal((5, 4))
    e = np.zeros((5, 4))
    e[2, 1] = 0.25
    e2 = np.zeros((5, 4))
    e2[4, 3] = -0.25
    return max(abs(rel(-3.0 * a, -3.0 * b) - rel(a, b)),
               abs(rel(b + e, b) - rel(b + e2, b)),
               abs(rel(b + e, b) - 0.25 / math.sqrt(float(np.sum(b * b)))))


def pin_rel_fro_brute_force(rel):
    """Against sums of squares taken element by element in Python."""
    rng = np.random.default_rng(32)
    a = rng.standard_normal((3, 4))
    b = rng.standard_normal((3, 4))
    num = den = 0.0
    for i in range(3):
        for j in range(4):
            num += (a[i, j] - b[i, j]) ** 2
            den += b[i, j] ** 2
    return abs(rel(a, b) - math.sqrt(num) / math.sqrt(den))


REL_PINS = [pin_rel_fro_hand, pin_rel_fro_zero_reference, pin_rel_fro_scale_and_symmetry,
            pin_rel_fro_brute_force]


# ------------------------------------------------------------------ orthogonality_error

def pin_orth_err_exact_cases(oe):
    """Orthonormal columns give 0 (a tall 3x2 selection, a rotation); scaling one column
    by 2 makes its diagonal entry 4 - 1 = 3."""
    c, s = math.cos(0.3), math.sin(0.3)
    return max(oe(np.array([[1.0, 0.0], [0.0, 1.0], [0.0, 0.0]])),
               oe(np.array([[c, -s], [s, c]])),
               abs(oe(np.array([[2.0, 0.0], [0.0, 1.0], [0.0, 0.0]])) - 3.0))


def pin_orth_err_off_diagonal(oe):
    """P = (1, 0.1; 0, 1): P^T P = (1, 0.1; 0.1, 1.01), so max |P^T P - I| = 0.1."""
    return abs(oe(np.array([[1.0, 0.1], [0.0, 1.0]])) - 0.1)


def pin_orth_err_shrunk_column(oe):
    """A column of norm 1/2 gives a diagonal entry 1/4 - 1 = -3/4: the error is its
    magnitude 0.75 (the largest signed entry would be 0)."""
    return abs(oe(np.array([[0.5, 0.0], [0.0, 1.0], [0.0, 0.0]])) - 0.75)


def pin_orth_err_wide_gram(oe):
    """For a tall P with orthonormal columns P P^T is a projector, not I: a checker that
    formed P P^T would report 1 where the answer is 0."""
    q = np.linalg.qr(np.random.default_rng(33).standard_normal((7, 3)))[0]
    return oe(q)


ORTH_PINS = [pin_orth_err_exact_cases, pin_orth_err_off_diagonal, pin_orth_err_shrunk_column,
             pin_orth_err_wide_gram]

PIN_TOL = 1e-12


@pytest.mark.parametrize("pin", REL_PINS, ids=lambda p: p.__name__)
def test_rel_fro_meets_pin(pin):
    assert pin(oracle.rel_fro) < PIN_TOL


@pytest.mark.parametrize("pin", ORTH_PINS, ids=lambda p: p.__name__)
def test_orthogonality_error_meets_pin(pin):
    assert pin(oracle.orthogonality_error) < PIN_TOL


# ------------------------------------------------------------------ run_steps

def pin_reset_momentum_full_rank(run):
    """Fixed B at full rank with the momentum reset before every step: each step starts
    from M = 0 and G = B, so M' = mu B after any number of steps (P P^T = I).  Without
    the reset, M after two steps would be mu (mu B + B)."""
    rng = np.random.default_rng(34)
    B = rng.standard_normal((6, 6))
    Q = rng.standard_normal((6, 6))
    Q /= np.linalg.norm(Q, axis=0, keepdims=True)
    X = rng.standard_normal((6, 6))
    M0 = rng.standard_normal((6, 6))          # discarded by the first reset
    _, M, _, _, _ = run(X, M0, Q, [B, B, B], 0.9, 0.05, reset_momentum=True)
    return np.abs(M - 0.9 * B).max()


def pin_no_reset_accumulates(run):
    """Without the reset, at full rank M' = mu (M + G): from M = 0 and three steps of the
    same G, M = (mu + mu^2 + mu^3) G."""
    rng = np.random.default_rng(35)
    G = rng.standard_normal((5, 5))
    Q = rng.standard_normal((5, 5))
    Q /= np.linalg.norm(Q, axis=0, keepdims=True)
    _, M, _, _, _ = run(np.zeros((5, 5)), np.zeros((5, 5)), Q, [G, G, G], 0.5, 0.1)
    return np.abs(M - (0.5 + 0.25 + 0.125) * G).max()


def pin_run_steps_update_norm(run):
    """Each step moves X by exactly lr sqrt(m/n) sqrt(r) in Frobenius norm, so after T
    steps in the same direction (r = 1 on a fixed rank-one B whose Q is already its right
    singular vector) X moves by T lr sqrt(m/n)."""
    m, n = 8, 2
    u = np.zeros(m); u[0] = 1.0
    v = np.array([0.6, 0.8])
    B = 2.0 * np.outer(u, v)
    X, _, _, _, _ = run(np.zeros((m, n)), np.zeros((m, n)), v[:, None], [B, B, B, B], 0.9, 0.1,
                        reset_momentum=True)
    return abs(np.linalg.norm(X) - 4 * 0.1 * math.sqrt(m / n))


RUN_PINS = [pin_reset_momentum_full_rank, pin_no_reset_accumulates, pin_run_steps_update_norm]


@pytest.mark.parametrize("pin", RUN_PINS, ids=lambda p: p.__name__)
def test_run_steps_meets_pin(pin):
    assert pin(oracle.run_steps) < 1e-10


# ------------------------------------------------ planted mistakes must trip a pin

def _rel_mutant(kind):
    def rel(a, ref):
        a, ref = np.asarray(a, np.float64), np.asarray(ref, np.float64)
        num = np.linalg.norm(a - ref)
        if kind == "divide_by_a":
            den = np.linalg.norm(a)
        elif kind == "max_abs":
            num, den = np.abs(a - ref).max(), np.abs(ref).max()
        elif kind == "squared":
            num, den = num ** 2, np.linalg.norm(ref) ** 2
        elif kind == "sum_not_norm":
            num, den = np.abs(np.sum(a - ref)), np.abs(np.sum(ref))
        else:
            den = np.linalg.norm(ref)
        if den == 0:
            if kind == "zero_ref_is_exact":
                return 0.0
            if kind == "zero_ref_is_inf":
                return float("inf") if num else 0.0
            return float(num)
        return float(num / den)
    return rel


REL_MUTANTS = ["divide_by_a", "max_abs", "squared", "sum_not_norm", "zero_ref_is_exact",
               "zero_ref_is_inf"]


@pytest.mark.parametrize("kind", REL_MUTANTS)
def test_planted_rel_fro_mistake_is_caught(kind):
    rel = _rel_mutant(kind)
    with np.errstate(all="ignore"):
        errs = {p.__name__: p(rel) for p in REL_PINS}
    assert any(not (e < PIN_TOL) for e in errs.values()), errs


def _orth_mutant(kind):
    def oe(P):
        P = np.asarray(P, np.float64)
        if kind == "outer_gram":
            return float(np.max(np.abs(P @ P.T - np.eye(P.shape[0]))))
        if kind == "signed_max":
            return float(np.max(P.T @ P - np.eye(P.shape[1])))
        if kind == "no_identity":
            return float(np.max(np.abs(P.T @ P)))
        if kind == "frobenius":
            return float(np.linalg.norm(P.T @ P - np.eye(P.shape[1])))
        if kind == "diagonal_only":
            return float(np.max(np.abs(np.diag(P.T @ P) - 1.0)))
        return float(np.max(np.abs(P.T @ P - np.eye(P.shape[1]))))
    return oe


ORTH_MUTANTS = ["outer_gram", "signed_max", "no_identity", "frobenius", "diagonal_only"]


@pytest.mark.parametrize("kind", ORTH_MUTANTS)
def test_planted_orthogonality_error_mistake_is_caught(kind):
    oe = _orth_mutant(kind)
    errs = {p.__name__: p(oe) for p in ORTH_PINS}
    assert any(not (e < PIN_TOL) for e in errs.values()), errs


def _run_mutant(kind):
    def run(X, M, Q, grads, mu, lr, scale=None, reset_momentum=False):
        X, M, Q = (np.asarray(a, np.float64) for a in (X, M, Q))
        P = R = None
        for G in grads:
            if reset_momentum and kind == "reset_after":
                X, M, Q, P, R = od.dion_step(X, M, G, Q, mu, lr, scale)
                M = np.zeros_like(M)
                continue
            if reset_momentum and kind != "reset_ignored":
                M = np.zeros_like(M)
            X, M, Q, P, R = od.dion_step(X, M, G, Q, mu, lr, scale)
            if kind == "first_step_only":
                break
        return X, M, Q, P, R
    return run


RUN_MUTANTS = ["reset_ignored", "reset_after", "first_step_only"]


@pytest.mark.parametrize("kind", RUN_MUTANTS)
def test_planted_run_steps_mistake_is_caught(kind):
    run = _run_mutant(kind)
    errs = {p.__name__: p(run) for p in RUN_PINS}
    assert any(not (e < 1e-10) for e in errs.values()), errs
