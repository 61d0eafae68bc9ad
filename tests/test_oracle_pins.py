"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

The pages print no worked example of the Dion step, so the oracle is pinned by:
  * hand-worked tiny steps (tests/golden/hand_worked_steps.txt);
  * consequences of the step that hold exactly for orthonormal P and unit-column Q
    (P^T M' = mu R^T, ||X' - X||_F = lr s sqrt(r), M' = mu B at full rank);
  * reductions to textbook routines: Cholesky-QR through SciPy's Cholesky and
    triangular solve, the power method (r = 1) and orthogonal iteration converging
    to the SVD's singular vectors and polar factor (numpy.linalg.svd);
  * exactness on low-rank inputs (the error-feedback residual vanishes).
Each plausible slip in the oracle (a dropped term, a wrong sign, the old Q in the
weight update, a transposed factor, row instead of column normalisation) is planted
in a copy of the step at the end of this file and must trip at least one pin.
"""
import math

import numpy as np
import pytest
import scipy.linalg as sla

import oracle
from oracle import dion_oracle as od

RNG = np.random.default_rng(20260101)


def _unit_cols(a):
    return a / np.linalg.norm(a, axis=0, keepdims=True)


def _rand_state(m, n, r, rng):
    X = rng.standard_normal((m, n))
    M = rng.standard_normal((m, n))
    G = rng.standard_normal((m, n))
    Q = _unit_cols(rng.standard_normal((n, r)))
    return X, M, G, Q


# ---------------------------------------------------------------- pin functions
# Each takes a step function with the oracle's signature and returns the error
# against the pinned value (0 when exact).

def pin_hand_case_a(step):
    M = np.array([[1.0, 0], [0, 1]]); G = np.array([[2.0, 0], [0, 0]])
    Q = np.array([[1.0], [0]]); X = np.array([[1.0, 2], [3, 4]])
    Xn, Mn, Qn, P, R = step(X, M, G, Q, 0.9, 0.1)
    err = max(np.abs(Mn - np.array([[2.7, 0], [0, 1]])).max(),
              np.abs(Xn - np.array([[0.9, 2], [3, 4]])).max(),
              np.abs(Qn - np.array([[1.0], [0]])).max(),
              np.abs(P - np.array([[1.0], [0]])).max(),
              np.abs(R - np.array([[3.0], [0]])).max())
    return err


def pin_hand_case_b(step):
    M = np.array([[1.0, 0], [0, 1]]); G = np.array([[2.0, 0], [0, 0]])
    Q = np.array([[-1.0], [0]]); X = np.array([[1.0, 2], [3, 4]])
    Xn, Mn, Qn, P, R = step(X, M, G, Q, 0.9, 0.1)
    return max(np.abs(Mn - np.array([[2.7, 0], [0, 1]])).max(),
               np.abs(Xn - np.array([[0.9, 2], [3, 4]])).max(),
               np.abs(P - np.array([[-1.0], [0]])).max(),
               np.abs(Qn - np.array([[-1.0], [0]])).max())


def pin_hand_case_c(step):
    B = np.array([[1.0, 2], [0, 1], [2, 0]])
    Q = np.array([[0.6], [0.8]])
    Xn, Mn, Qn, P, R = step(np.zeros((3, 2)), np.zeros((3, 2)), B, Q, 0.5, 0.2)
    p0 = np.array([2.2, 0.8, 1.2]); rr = np.array([4.6, 5.2])
    m_exp = B - 0.5 * np.outer(p0, rr) / 6.92
    q_exp = rr / math.sqrt(48.2)
    x_exp = -0.2 * math.sqrt(1.5) * np.outer(p0, rr) / (math.sqrt(6.92) * math.sqrt(48.2))
    return max(np.abs(Mn - m_exp).max(), np.abs(Qn[:, 0] - q_exp).max(),
               np.abs(Xn - x_exp).max(), np.abs(P[:, 0] - p0 / math.sqrt(6.92)).max(),
               np.abs(R[:, 0] - rr / math.sqrt(6.92)).max())


def pin_hand_case_d(step):
    B = np.array([[2.0, 1], [1, 3]])
    _, Mn, _, P, _ = step(np.zeros((2, 2)), np.zeros((2, 2)), B, np.eye(2), 0.8, 0.1)
    return np.abs(Mn - 0.8 * B).max()


def pin_feedback_projection(step, m=40, n=24, r=6, mu=0.9):
    """P^T M' = mu R^T: holds for orthonormal P whatever B is."""
    X, M, G, Q = _rand_state(m, n, r, np.random.default_rng(1))
    _, Mn, _, P, R = step(X, M, G, Q, mu, 0.05)
    return np.abs(P.T @ Mn - mu * R.T).max() / np.abs(R).max()


def pin_update_norm(step, m=40, n=24, r=6, lr=0.05):
    """||X' - X||_F = lr * sqrt(m/n) * sqrt(r): trace(Q P^T P Q^T) = sum ||q_j||^2 = r."""
    X, M, G, Q = _rand_state(m, n, r, np.random.default_rng(2))
    Xn = step(X, M, G, Q, 0.9, lr)[0]
    return abs(np.linalg.norm(Xn - X) - lr * math.sqrt(m / n) * math.sqrt(r))


def pin_unit_columns(step, m=30, n=50, r=7):
    X, M, G, Q = _rand_state(m, n, r, np.random.default_rng(3))
    Qn = step(X, M, G, Q, 0.9, 0.05)[2]
    return np.abs(np.linalg.norm(Qn, axis=0) - 1.0).max()


def pin_low_rank_g(step, m=36, n=20, k=3, r=5, mu=0.7):
    """M = 0, G of rank k <= r: span(B Q) = col(B), so M' = mu G exactly."""
    rng = np.random.default_rng(4)
    G = rng.standard_normal((m, k)) @ rng.standard_normal((k, n))
    Q = _unit_cols(rng.standard_normal((n, r)))
    Mn = step(np.zeros((m, n)), np.zeros((m, n)), G, Q, mu, 0.1)[1]
    return np.abs(Mn - mu * G).max() / np.abs(G).max()


def pin_low_rank_m(step, m=36, n=20, k=4, r=4, mu=0.6):
    """G = 0, M of rank k <= r: M' = mu M exactly."""
    rng = np.random.default_rng(5)
    M = rng.standard_normal((m, k)) @ rng.standard_normal((k, n))
    Q = _unit_cols(rng.standard_normal((n, r)))
    Mn = step(np.zeros((m, n)), M, np.zeros((m, n)), Q, mu, 0.1)[1]
    return np.abs(Mn - mu * M).max() / np.abs(M).max()


def pin_rank_one_direction(step, m=9, n=6, lr=0.3):
    """B = sigma u v^T, r = 1: the update is exactly -lr s u v^T (new Q, not the old one)."""
    rng = np.random.default_rng(6)
    u = _unit_cols(rng.standard_normal((m, 1)))[:, 0]
    v = _unit_cols(rng.standard_normal((n, 1)))[:, 0]
    B = 2.5 * np.outer(u, v)
    Q = _unit_cols(rng.standard_normal((n, 1)))
    X = rng.standard_normal((m, n))
    Xn = step(X, np.zeros((m, n)), B, Q, 0.9, lr)[0]
    return np.abs((Xn - X) + lr * math.sqrt(m / n) * np.outer(u, v)).max()


def pin_power_method(step, m=12, n=8, steps=200):
    """r = 1 on a fixed B is the power method: P -> u1, Q -> v1 (up to a joint sign)."""
    rng = np.random.default_rng(7)
    U = np.linalg.qr(rng.standard_normal((m, n)))[0]
    V = np.linalg.qr(rng.standard_normal((n, n)))[0]
    sig = np.array([3.0, 1.5, 1.0, 0.8, 0.5, 0.3, 0.2, 0.1])
    B = (U * sig) @ V.T
    u_, s_, vt_ = np.linalg.svd(B)
    Q = _unit_cols(rng.standard_normal((n, 1)))
    X = np.zeros((m, n)); M = np.zeros((m, n))
    for _ in range(steps):
        X, M, Q, P, R = step(X, np.zeros((m, n)), B, Q, 0.9, 0.0)
    return max(np.abs(np.outer(P[:, 0], Q[:, 0]) - np.outer(u_[:, 0], vt_[0])).max(),
               abs(np.linalg.norm(R) - s_[0]))


def pin_polar_limit(step, k=8, steps=80):
    """Full rank on a fixed B with well separated singular values: P Q^T -> U V^T."""
    rng = np.random.default_rng(8)
    U = np.linalg.qr(rng.standard_normal((k, k)))[0]
    V = np.linalg.qr(rng.standard_normal((k, k)))[0]
    B = (U * 2.0 ** -np.arange(k)) @ V.T
    u_, _, vt_ = np.linalg.svd(B)
    Q = _unit_cols(rng.standard_normal((k, k)))
    X = np.zeros((k, k))
    for _ in range(steps):
        X2, _, Q, P, _ = step(X, np.zeros((k, k)), B, Q, 0.9, 1.0)
    return np.abs(P @ Q.T - u_ @ vt_).max()


def pin_zero_gradient(step, m=10, n=6, r=3):
    X = RNG.standard_normal((m, n))
    Q = _unit_cols(RNG.standard_normal((n, r)))
    Xn, Mn, Qn, _, _ = step(X, np.zeros((m, n)), np.zeros((m, n)), Q, 0.9, 0.1)
    return max(np.abs(Xn - X).max(), np.abs(Mn).max(), np.abs(Qn).max())


PINS = [pin_hand_case_a, pin_hand_case_b, pin_hand_case_c, pin_hand_case_d,
        pin_feedback_projection, pin_update_norm, pin_unit_columns, pin_low_rank_g,
        pin_low_rank_m, pin_rank_one_direction, pin_power_method, pin_polar_limit,
        pin_zero_gradient]
TOL = 1e-9


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_meets_pin(pin):
    assert pin(oracle.dion_step) < TOL


# ------------------------------------------------------- orth: two textbook routes

@pytest.mark.parametrize("m,r", [(50, 8), (200, 32), (64, 64)])
def test_orth_equals_cholesky_qr(m, r):
    """Sign-fixed Householder QR == Cholesky-QR (SciPy cholesky + triangular solve)."""
    rng = np.random.default_rng(m * 1000 + r)
    P0 = rng.standard_normal((m, r)) @ np.diag(np.linspace(1, 4, r))
    P, Rf = oracle.orth(P0)
    L = sla.cholesky(P0.T @ P0, lower=True)
    P_chol = sla.solve_triangular(L, P0.T, lower=True).T      # P0 L^-T
    assert np.abs(P - P_chol).max() < 1e-11
    assert np.abs(P.T @ P - np.eye(r)).max() < 1e-12
    assert np.abs(np.tril(Rf, -1)).max() == 0.0 and (np.diag(Rf) > 0).all()
    assert np.abs(P @ Rf - P0).max() < 1e-12 * np.abs(P0).max() * m


def test_orth_rank_deficient_spans_input():
    rng = np.random.default_rng(11)
    P0 = rng.standard_normal((30, 3)) @ rng.standard_normal((3, 6))
    P, _ = oracle.orth(P0)
    assert np.abs(P.T @ P - np.eye(6)).max() < 1e-12
    assert np.abs(P @ (P.T @ P0) - P0).max() < 1e-12


def test_colnorm_unit_and_zero_columns():
    R = np.array([[3.0, 0.0, 1.0], [4.0, 0.0, -1.0]])
    Qn = oracle.colnorm(R)
    assert np.allclose(Qn[:, 0], [0.6, 0.8]) and np.all(Qn[:, 1] == 0)
    assert np.allclose(Qn[:, 2], [2 ** -0.5, -(2 ** -0.5)])


def test_full_rank_fixed_b_momentum_is_mu_b():
    """r = min(m, n): P P^T = I, so M' = mu B at every step (the full-rank closed form)."""
    rng = np.random.default_rng(12)
    B = rng.standard_normal((16, 16))
    Q = _unit_cols(rng.standard_normal((16, 16)))
    X = np.zeros((16, 16))
    for _ in range(3):
        X, Mn, Q, P, R = oracle.dion_step(X, np.zeros((16, 16)), B, Q, 0.95, 0.01)
        assert np.abs(Mn - 0.95 * B).max() < 1e-11


def test_stacked_is_per_matrix():
    rng = np.random.default_rng(13)
    X = rng.standard_normal((3, 12, 8)); M = rng.standard_normal((3, 12, 8))
    G = rng.standard_normal((3, 12, 8)); Q = _unit_cols(rng.standard_normal((8, 4)))
    Qs = np.stack([Q] * 3)
    out = oracle.dion_step_stacked(X, M, G, Qs, 0.9, 0.1)
    one = oracle.dion_step(X[1], M[1], G[1], Q, 0.9, 0.1)
    for a, b in zip(out, one):
        assert np.array_equal(a[1], b)


def test_workload_c1_oracle_invariants():
    """The oracle on the 256x128 r=32 workload keeps every invariant over 10 steps."""
    import workloads as W
    wl = W.WORKLOADS["single_256x128_r32"]
    X = W.weights(wl, 0)[0]; M = W.momentum(wl, 0)[0]; Q = W.right_factor(wl, 0)[0]
    X, M, Q = [t.double().numpy() for t in (X, M, Q)]
    for t in range(wl.steps):
        G = W.gradient(wl, 0, t)[0].double().numpy()
        Xn, Mn, Qn, P, R = oracle.dion_step(X, M, G, Q, wl.mu, wl.lr)
        assert oracle.orthogonality_error(P) < 1e-12
        assert np.abs(np.linalg.norm(Qn, axis=0) - 1).max() < 1e-13
        assert abs(np.linalg.norm(Xn - X) - wl.lr * math.sqrt(2) * math.sqrt(32)) < 1e-12
        assert np.abs(P.T @ Mn - wl.mu * R.T).max() < 1e-10
        X, M, Q = Xn, Mn, Qn


# ----------------------------------------------- planted mistakes must trip a pin

def _mutant(kind):
    def step(X, M, G, Q, mu, lr, scale=None):
        X, M, G, Q = (np.asarray(a, dtype=np.float64) for a in (X, M, G, Q))
        m, n = X.shape
        s = math.sqrt(m / n) if scale is None else scale
        B = M if kind == "drop_g" else (G if kind == "drop_m" else M + G)
        P0 = B @ Q
        if kind == "no_sign_fix":
            P = np.linalg.qr(P0)[0]
        else:
            P = od.orth(P0)[0]
        R = B.T @ P
        if kind == "mu_swapped":
            Mn = B - mu * P @ R.T
        elif kind == "feedback_sign":
            Mn = B + (1 - mu) * P @ R.T
        else:
            Mn = B - (1 - mu) * P @ R.T
        if kind == "row_norm":
            Qn = R / np.linalg.norm(R, axis=1, keepdims=True)
        else:
            Qn = od.colnorm(R)
        if kind == "old_q":
            Xn = X - lr * s * P @ Q.T
        elif kind == "no_scale":
            Xn = X - lr * P @ Qn.T
        elif kind == "inverse_scale":
            Xn = X - lr / s * P @ Qn.T
        elif kind == "update_sign":
            Xn = X + lr * s * P @ Qn.T
        else:
            Xn = X - lr * s * P @ Qn.T
        return Xn, Mn, Qn, P, R
    return step


MUTANTS = ["drop_g", "drop_m", "no_sign_fix", "mu_swapped", "feedback_sign", "row_norm",
           "old_q", "no_scale", "inverse_scale", "update_sign"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistake_is_caught(kind):
    step = _mutant(kind)
    with np.errstate(all="ignore"):
        errs = {p.__name__: p(step) for p in PINS}
    assert any(not (e < TOL) for e in errs.values()), errs
