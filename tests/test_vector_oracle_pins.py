"""Pins of the fp64 oracle of the vector-parameter step (AdamW, Lion).

Nothing here comes from the oracle itself:
  * hand-worked steps (tests/golden/vector_hand_worked.txt), parsed from the file;
  * closed forms: AdamW's first step from a zero state is lr g / (|g| + eps) per
    element, and with a constant gradient the bias correction makes every step the
    same; a zero gradient leaves only the decoupled decay; Lion's step is exactly lr
    wherever the interpolation is non-zero, and its momentum under a constant
    gradient is (1 - b2^k) g; with b1 = 0 Lion is sign descent on g;
  * a library routine: torch.optim.AdamW (fp64, CPU) from a non-zero state.
Plausible slips (no bias correction, the decay after the step, eps inside the square
root, swapped betas, |g| in place of g^2; Lion's sign of m or of g alone, its momentum
with b1, no decay) are planted in copies below and must each trip a pin.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "vector_hand_worked.txt")
HP_HAND = dict(lr=0.125, b1=0.5, b2=0.75, wd=0.5)


def _golden(rule):
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line.startswith(rule + " "):
            continue
        lhs, rhs = line[len(rule):].split("->")
        rows.append(({k: float(v) for k, v in (f.split("=") for f in lhs.split())},
                     {k: float(v) for k, v in (f.split("=") for f in rhs.split())}))
    return rows


def test_golden_file_has_both_rules():
    assert len(_golden("adamw")) == 2 and len(_golden("lion")) == 4


# ---------------------------------------------------------------- AdamW pins
# Each takes a step function with the signature of oracle.adamw_step and returns the
# error against the pinned value.

def pin_adamw_hand(step):
    err = 0.0
    for a, want in _golden("adamw"):
        x, m, v = step(np.array([a["x"]]), np.array([a["g"]]), np.array([a["m"]]),
                       np.array([a["v"]]), t=int(a["t"]), eps=0.5, **HP_HAND)
        err = max(err, abs(x[0] - want["x"]), abs(m[0] - want["m"]), abs(v[0] - want["v"]))
    return err


def pin_adamw_first_step(step):
    rng = np.random.default_rng(1)
    x0, g = rng.standard_normal(50), rng.standard_normal(50)
    lr, wd, eps = 0.25, 0.5, 0.125
    x, _, _ = step(x0, g, np.zeros(50), np.zeros(50), t=1, lr=lr, b1=0.75, b2=0.875,
                   eps=eps, wd=wd)
    return np.abs(x - (x0 * (1 - lr * wd) - lr * g / (np.abs(g) + eps))).max()


def pin_adamw_constant_gradient(step):
    rng = np.random.default_rng(2)
    x0, g = rng.standard_normal(30), rng.standard_normal(30)
    x, m, v = x0, np.zeros(30), np.zeros(30)
    lr, eps = 0.125, 0.25
    for t in range(1, 7):
        x, m, v = step(x, g, m, v, t=t, lr=lr, b1=0.75, b2=0.5, eps=eps, wd=0.0)
    return np.abs(x - (x0 - 6 * lr * g / (np.abs(g) + eps))).max()


def pin_adamw_zero_gradient(step):
    x0 = np.random.default_rng(3).standard_normal(20)
    x, m, v = step(x0, np.zeros(20), np.zeros(20), np.zeros(20), t=3, lr=0.25, b1=0.5,
                   b2=0.75, eps=0.5, wd=0.5)
    return max(np.abs(x - 0.875 * x0).max(), np.abs(m).max(), np.abs(v).max())


def pin_adamw_torch(step):
    """torch.optim.AdamW in fp64 on the CPU, resumed at step 4 from a non-zero state."""
    rng = np.random.default_rng(4)
    x0, g = rng.standard_normal(40), rng.standard_normal(40)
    m0, v0 = 0.1 * rng.standard_normal(40), 0.01 * rng.random(40)
    lr, b1, b2, eps, wd = 0.125, 0.875, 0.96875, 0.0625, 0.25
    p = torch.nn.Parameter(torch.tensor(x0, dtype=torch.float64))
    opt = torch.optim.AdamW([p], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd,
                            foreach=False)
    p.grad = torch.tensor(g, dtype=torch.float64)
    opt.state[p] = {"step": torch.tensor(3.0, dtype=torch.float64),
                    "exp_avg": torch.tensor(m0, dtype=torch.float64),
                    "exp_avg_sq": torch.tensor(v0, dtype=torch.float64)}
    opt.step()
    x, m, v = step(x0, g, m0, v0, t=4, lr=lr, b1=b1, b2=b2, eps=eps, wd=wd)
    return max(np.abs(x - p.detach().numpy()).max(),
               np.abs(m - opt.state[p]["exp_avg"].numpy()).max(),
               np.abs(v - opt.state[p]["exp_avg_sq"].numpy()).max())


ADAMW_PINS = [pin_adamw_hand, pin_adamw_first_step, pin_adamw_constant_gradient,
              pin_adamw_zero_gradient, pin_adamw_torch]


# ---------------------------------------------------------------- Lion pins

def pin_lion_hand(step):
    err = 0.0
    for a, want in _golden("lion"):
        x, m = step(np.array([a["x"]]), np.array([a["g"]]), np.array([a["m"]]), **HP_HAND)
        err = max(err, abs(x[0] - want["x"]), abs(m[0] - want["m"]))
    return err


def pin_lion_step_is_lr(step):
    rng = np.random.default_rng(5)
    x0, g, m0 = rng.standard_normal(64), rng.standard_normal(64), rng.standard_normal(64)
    m0[:8] = -g[:8]                       # b1 = 0.5: c = 0 exactly on these
    x, _ = step(x0, g, m0, lr=0.25, b1=0.5, b2=0.75, wd=0.0)
    d = np.abs(x - x0)
    return max(np.abs(d[8:] - 0.25).max(), d[:8].max())


def pin_lion_momentum_closed_form(step):
    g = np.random.default_rng(6).standard_normal(16)
    x, m = np.zeros(16), np.zeros(16)
    for _ in range(5):
        x, m = step(x, g, m, lr=0.125, b1=0.5, b2=0.75, wd=0.0)
    return np.abs(m - (1 - 0.75 ** 5) * g).max()


def pin_lion_b1_zero_is_sign_descent(step):
    rng = np.random.default_rng(7)
    x0, g, m0 = rng.standard_normal(32), rng.standard_normal(32), rng.standard_normal(32)
    x, _ = step(x0, g, m0, lr=0.125, b1=0.0, b2=0.75, wd=0.5)
    return np.abs(x - (x0 * (1 - 0.0625) - 0.125 * np.sign(g))).max()


def pin_lion_decay(step):
    x0 = np.random.default_rng(8).standard_normal(12)
    x, _ = step(x0, np.zeros(12), np.zeros(12), lr=0.25, b1=0.5, b2=0.75, wd=0.5)
    return np.abs(x - 0.875 * x0).max()


LION_PINS = [pin_lion_hand, pin_lion_step_is_lr, pin_lion_momentum_closed_form,
             pin_lion_b1_zero_is_sign_descent, pin_lion_decay]
TOL = 1e-12


@pytest.mark.parametrize("pin", ADAMW_PINS, ids=lambda p: p.__name__)
def test_adamw_oracle_meets_pin(pin):
    assert pin(oracle.adamw_step) < TOL


@pytest.mark.parametrize("pin", LION_PINS, ids=lambda p: p.__name__)
def test_lion_oracle_meets_pin(pin):
    assert pin(oracle.lion_step) < TOL


def test_lion_direction_is_taken_in_fp32():
    """b1 = 0.9, m = 1, g = -9: in fp64, 0.9 + 0.1 * (-9) is exactly 0 (sign 0); in fp32
    1 - b1 rounds to 0.100000024 and c = 0.9 - 0.90000021 < 0 (sign -1).  The library
    fixes the decision to fp32, and so must the oracle."""
    assert 0.9 * 1.0 + 0.1 * -9.0 == 0.0      # in fp64 the decision would be sign 0
    s = oracle.lion_direction(np.array([1.0]), np.array([-9.0]), 0.9)[0]
    assert s == -1.0
    assert np.isnan(oracle.lion_direction(np.array([np.nan]), np.array([1.0]), 0.9)[0])
    assert oracle.lion_direction(np.array([0.0]), np.array([0.0]), 0.9)[0] == 0.0


# ----------------------------------------------- planted mistakes must trip a pin

def _adamw_mutant(kind):
    def step(x, g, m, v, *, t, lr, b1, b2, eps, wd):
        x, g, m, v = (np.asarray(a, dtype=np.float64) for a in (x, g, m, v))
        if kind == "swap_betas":
            b1, b2 = b2, b1
        if kind != "decay_after":
            x = x * (1 - lr * wd)
        m = b1 * m + (1 - b1) * g
        v = b2 * v + (1 - b2) * (np.abs(g) if kind == "abs_g" else g * g)
        mh = m if kind == "no_bias_correction" else m / (1 - b1 ** t)
        vh = v if kind == "no_bias_correction" else v / (1 - b2 ** t)
        den = np.sqrt(vh + eps) if kind == "eps_in_sqrt" else np.sqrt(vh) + eps
        xn = x - lr * mh / den
        if kind == "decay_after":
            xn = xn - lr * wd * xn
        return xn, m, v
    return step


def _lion_mutant(kind):
    def step(x, g, m, *, lr, b1, b2, wd):
        x, g, m = (np.asarray(a, dtype=np.float64) for a in (x, g, m))
        c = {"sign_of_m": m, "sign_of_g": g}.get(kind, b1 * m + (1 - b1) * g)
        decay = 1.0 if kind == "no_decay" else 1 - lr * wd
        xn = x * decay - lr * np.sign(c)
        bm = b1 if kind == "momentum_b1" else b2
        return xn, bm * m + (1 - bm) * g
    return step


@pytest.mark.parametrize("kind", ["swap_betas", "decay_after", "abs_g", "no_bias_correction",
                                  "eps_in_sqrt"])
def test_adamw_planted_mistake_is_caught(kind):
    errs = {p.__name__: p(_adamw_mutant(kind)) for p in ADAMW_PINS}
    assert max(errs.values()) > 1e-6, errs


@pytest.mark.parametrize("kind", ["sign_of_m", "sign_of_g", "no_decay", "momentum_b1"])
def test_lion_planted_mistake_is_caught(kind):
    errs = {p.__name__: p(_lion_mutant(kind)) for p in LION_PINS}
    assert max(errs.values()) > 1e-6, errs


def test_vector_step_lists():
    rng = np.random.default_rng(9)
    xs = [rng.standard_normal(k) for k in (3, 5)]
    gs = [rng.standard_normal(k) for k in (3, 5)]
    ms = [np.zeros(k) for k in (3, 5)]
    vs = [np.zeros(k) for k in (3, 5)]
    hp = dict(t=1, lr=0.125, b1=0.5, b2=0.75, eps=0.5, wd=0.0)
    X, M, V = oracle.vector_step("adamw", xs, gs, ms, vs, **hp)
    for i in range(2):
        x, m, v = oracle.adamw_step(xs[i], gs[i], ms[i], vs[i], **hp)
        assert np.array_equal(X[i], x) and np.array_equal(M[i], m) and np.array_equal(V[i], v)
    assert math.isclose(X[0][0], xs[0][0] - 0.125 * gs[0][0] / (abs(gs[0][0]) + 0.5))
