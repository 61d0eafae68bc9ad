"""Pins of the RMMC oracle (CurvaDion's momentum-change statistic, read as
max |M' - M| / max |M|) against values worked by hand and closed forms of the Dion
step, not against the function itself; each plausible slip is planted in a copy at
the end and must trip a pin."""
import math

import numpy as np
import pytest

import oracle


def pin_hand_values(f):
    """M = (1, -4; 2, 0), M' = (1.5, -3; 2, -1): the change (0.5, 1; 0, -1) has largest
    entry 1, the momentum 4: RMMC = 1/4.  A change of 6 at the largest entry of a
    momentum whose largest entry is -3 gives 2."""
    return max(abs(f(np.array([[1.0, -4.0], [2.0, 0.0]]),
                     np.array([[1.5, -3.0], [2.0, -1.0]])) - 0.25),
               abs(f(np.array([[-3.0, 1.0]]), np.array([[3.0, 1.0]])) - 2.0))


def pin_zero_momentum(f):
    """No scale: +inf when the momentum moved, 0 when it did not."""
    a = f(np.zeros((2, 2)), np.array([[0.0, 1e-30], [0.0, 0.0]]))
    b = f(np.zeros((2, 2)), np.zeros((2, 2)))
    return (0.0 if a == float("inf") else 1.0) + abs(b)


def pin_full_rank_decay(f, mu=0.9):
    """G = 0 at full rank: the Dion step gives M' = mu M exactly (P P^T = I), so the
    change is (mu - 1) M and RMMC = 1 - mu whatever M is."""
    rng = np.random.default_rng(41)
    M = rng.standard_normal((8, 8))
    Q = rng.standard_normal((8, 8))
    Q /= np.linalg.norm(Q, axis=0, keepdims=True)
    _, Mn, _, _, _ = oracle.dion_step(np.zeros((8, 8)), M, np.zeros((8, 8)), Q, mu, 0.1)
    return abs(f(M, Mn) - (1 - mu))


def pin_low_rank_decay(f, mu=0.6):
    """G = 0 and M of rank 3 <= r = 4: again M' = mu M, RMMC = 1 - mu."""
    rng = np.random.default_rng(42)
    M = rng.standard_normal((20, 3)) @ rng.standard_normal((3, 12))
    Q = rng.standard_normal((12, 4))
    Q /= np.linalg.norm(Q, axis=0, keepdims=True)
    _, Mn, _, _, _ = oracle.dion_step(np.zeros((20, 12)), M, np.zeros((20, 12)), Q, mu, 0.1)
    return abs(f(M, Mn) - (1 - mu))


def pin_scale_invariance(f):
    """Scaling both momenta by c != 0 leaves the statistic unchanged."""
    rng = np.random.default_rng(43)
    a, b = rng.standard_normal((5, 7)), rng.standard_normal((5, 7))
    return abs(f(-2.5 * a, -2.5 * b) - f(a, b))


PINS = [pin_hand_values, pin_zero_momentum, pin_full_rank_decay, pin_low_rank_decay,
        pin_scale_invariance]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_rmmc_meets_pin(pin):
    assert pin(oracle.rmmc) < 1e-12


def test_gate_is_strictly_above_the_threshold():
    assert oracle.needs_sync(0.3, 0.2) and not oracle.needs_sync(0.2, 0.2)
    assert oracle.needs_sync(float("inf"), 1e30) and not oracle.needs_sync(0.0, 0.0)


def _mutant(kind):
    def f(M_prev, M_new):
        M_prev, M_new = np.asarray(M_prev, float), np.asarray(M_new, float)
        d = M_new - M_prev
        if kind == "frobenius":
            num, den = np.linalg.norm(d), np.linalg.norm(M_prev)
        elif kind == "relative_to_new":
            num, den = np.abs(d).max(), np.abs(M_new).max()
        elif kind == "signed":
            num, den = d.max(), M_prev.max()
        elif kind == "elementwise":
            with np.errstate(all="ignore"):
                q = np.abs(d) / np.abs(M_prev)
            q[np.isnan(q)] = 0.0
            num, den = q.max(), 1.0
        else:
            num, den = np.abs(d).max(), np.abs(M_prev).max()
        if kind == "zero_is_zero" and den == 0:
            return 0.0
        if den == 0:
            return float("inf") if num > 0 else 0.0
        return float(num / den)
    return f


MUTANTS = ["frobenius", "relative_to_new", "signed", "elementwise", "zero_is_zero"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistake_is_caught(kind):
    f = _mutant(kind)
    with np.errstate(all="ignore"):
        errs = {p.__name__: p(f) for p in PINS}
    assert any(not (e < 1e-12) for e in errs.values()), errs
