"""fp64 CPU oracle of the vector-parameter step (AdamW, Lion) -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the package's smoke check and the CPU-baseline leg of the
benchmark may import this module.  It shares no code with the CUDA library.

Which parameters: Dion takes only the 2-D weight matrices; biases and
normalisation gains go to AdamW or Lion (rivista.ai, "Dion e la fine del
monopolio di Adam negli optimizer AI distribuiti", paragraph 5).  The article
names the two rules without writing them, so they are taken as published:

AdamW, "Decoupled Weight Decay Regularization" (Loshchilov and Hutter), with
the decoupled decay applied to the weight before the Adam step and the bias
correction of step number t >= 1:

    x <- x (1 - lr wd)
    m <- b1 m + (1 - b1) g
    v <- b2 v + (1 - b2) g^2
    x <- x - lr * (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)

Lion, "Symbolic Discovery of Optimization Algorithms" (Chen et al.):

    c = b1 m + (1 - b1) g
    x <- x (1 - lr wd) - lr sign(c)        sign(0) = 0, sign(NaN) = NaN
    m <- b2 m + (1 - b2) g

Everything is fp64 except c: its sign is a discrete decision, so it is taken
in the arithmetic the library fixes for it -- fp32, with 1 - b1 rounded to
fp32 and each product and the sum rounded to fp32 (no fused multiply-add) --
from the fp32 values of m and g.
"""
from __future__ import annotations

import numpy as np


def adamw_step(x, g, m, v, *, t: int, lr: float, b1: float, b2: float, eps: float, wd: float):
    """One AdamW step of one parameter; returns (x', m', v') as fp64 arrays."""
    if t < 1:
        raise ValueError("the step number t starts at 1")
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    b1, b2, lr, eps, wd = (float(np.float32(a)) for a in (b1, b2, lr, eps, wd))
    x = x * (1.0 - lr * wd)
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    m_hat = m / (1.0 - b1 ** t)
    v_hat = v / (1.0 - b2 ** t)
    x = x - lr * m_hat / (np.sqrt(v_hat) + eps)
    return x, m, v


def lion_direction(m, g, b1: float):
    """sign(b1 m + (1 - b1) g) in the fp32 arithmetic the library fixes for it."""
    m32 = np.asarray(m, dtype=np.float32)
    g32 = np.asarray(g, dtype=np.float32)
    b1_32 = np.float32(b1)
    omb1 = np.float32(1.0) - b1_32
    with np.errstate(invalid="ignore"):
        c = b1_32 * m32 + omb1 * g32      # numpy float32: each operation rounded to fp32
    return np.sign(c).astype(np.float64)  # sign(0) = 0, sign(NaN) = NaN


def lion_step(x, g, m, *, lr: float, b1: float, b2: float, wd: float):
    """One Lion step of one parameter; returns (x', m') as fp64 arrays."""
    s = lion_direction(m, g, b1)
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    b1, b2, lr, wd = (float(np.float32(a)) for a in (b1, b2, lr, wd))
    x = x * (1.0 - lr * wd) - lr * s
    m = b2 * m + (1.0 - b2) * g
    return x, m


def vector_step(rule: str, xs, gs, ms, vs=None, **hp):
    """The step of a list of parameters (each its own arrays); returns new lists."""
    if rule == "adamw":
        out = [adamw_step(x, g, m, v, **hp) for x, g, m, v in zip(xs, gs, ms, vs)]
        return [o[0] for o in out], [o[1] for o in out], [o[2] for o in out]
    if rule == "lion":
        out = [lion_step(x, g, m, **hp) for x, g, m in zip(xs, gs, ms)]
        return [o[0] for o in out], [o[1] for o in out], None
    raise ValueError(f"unknown rule {rule!r}")
