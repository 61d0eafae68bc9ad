"""Parity of the CUDA vector-parameter step (AdamW, Lion) with its fp64 oracle (GPU).

Tolerances.  The kernel keeps x, m, v in fp32 and computes in fp32.  A forward error
bound of that evaluation, per element and step, from the oracle's own intermediates:
x is rounded twice a step (after the decay and after the update, half an ulp of |x|
each) and the fp32 decay factor 1 - lr wd carries half an ulp of 1, so 2^-22 |x'|; the
AdamW move lr m_hat / (sqrt(v_hat) + eps) passes through about eight roundings, each
relative to the sum of the absolute values of its terms (m can cancel), so
2^-19 lr (b1 |m| + (1 - b1) |g|) / (1 - b1^t) / (sqrt(v_hat') + eps).  The bounds add up
over the steps.  m and v: relative Frobenius error <= 1e-5 after a few steps.
Lion's direction is a discrete decision taken in fp32 on both sides from the same fp32
state, so each Lion step is checked from the GPU's own state ("teacher forcing"): a
flipped sign would be an error of 2 lr, far above the bound.
"""
import numpy as np
import pytest
import torch

import oracle
import rank_orthonormalized_optimizer_b200 as dion
import workloads as W

pytestmark = pytest.mark.gpu

# ragged sizes around the float4 and chunk (8192) granularity, and an empty tensor
SIZES = [1, 3, 4, 5, 17, 1023, 4096, 8192, 8195, 3 * 8192 + 7, 0, 100003]


def _state(sizes, seed, device="cuda", unaligned=()):
    """x, g, m, v lists; entries in `unaligned` are views one element into a buffer, so
    their pointers are 4- but not 16-byte aligned."""
    gen = torch.Generator().manual_seed(seed)
    out = {k: [] for k in "xgmv"}
    for i, n in enumerate(sizes):
        for k, scale in (("x", 1.0), ("g", 1e-2), ("m", 1e-2), ("v", 1e-2)):
            t = torch.randn(n, generator=gen, dtype=torch.float32) * scale
            if k == "v":
                t = t * t
            if i in unaligned:
                buf = torch.zeros(n + 1, dtype=torch.float32, device=device)
                buf[1:] = t.to(device)
                out[k].append(buf[1:])
            else:
                out[k].append(t.to(device).contiguous())
    return out


def _np(ts):
    return [t.detach().cpu().double().numpy() for t in ts]


HP = dict(b1=0.9, b2=0.999, eps=1e-8, wd=0.01)


def _adamw_ref(xs, gs, ms, vs, *, t, lr, b1, b2, eps, wd):
    """The oracle's step of a list of parameters and the per-element bound of one fp32
    step (see the module's docstring)."""
    X, M, V = oracle.vector_step("adamw", xs, gs, ms, vs, t=t, lr=lr, b1=b1, b2=b2, eps=eps,
                                 wd=wd)
    bound = []
    for x1, g, m, v1 in zip(X, gs, ms, V):
        terms = (b1 * np.abs(m) + (1 - b1) * np.abs(g)) / (1 - b1 ** t)
        den = np.sqrt(v1 / (1 - b2 ** t)) + eps
        bound.append(2.0 ** -22 * np.abs(x1) + 2.0 ** -19 * lr * terms / den)
    return X, M, V, bound


def _rel(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / nb if nb > 0 else np.linalg.norm(a)


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_adamw_matches_oracle(wd):
    s = _state(SIZES, 11, unaligned=(3, 7))
    xs, gs0, ms, vs = (_np(s[k]) for k in "xgmv")
    lr, b1, b2, eps, T = 1e-3, 0.9, 0.999, 1e-8, 5
    bound = [np.zeros(n) for n in SIZES]
    gen = torch.Generator().manual_seed(12)
    for t in range(1, T + 1):
        grads = [torch.randn(n, generator=gen) * 1e-2 for n in SIZES]
        for dst, src in zip(s["g"], grads):
            dst.copy_(src.to(dst.device))
        nl = dion.vec_step(s["x"], s["g"], s["m"], s["v"], rule="adamw", lr=lr, betas=(b1, b2),
                           eps=eps, weight_decay=wd, step=t)
        assert nl == 1
        xs, ms, vs, b = _adamw_ref(xs, [g.double().numpy() for g in grads], ms, vs, t=t, lr=lr,
                                   b1=b1, b2=b2, eps=eps, wd=wd)
        bound = [a + c for a, c in zip(bound, b)]
    torch.cuda.synchronize()
    for i, n in enumerate(SIZES):
        xg, mg, vg = (_np([s[k][i]])[0] for k in "xmv")
        assert np.all(np.abs(xg - xs[i]) <= bound[i]), i
        if n:
            assert _rel(mg, ms[i]) <= 1e-5 and _rel(vg, vs[i]) <= 1e-5, i
    # the unaligned entries sit one element into their buffers: the guard word is intact
    assert s["x"][3]._base[0].item() == 0.0


@pytest.mark.parametrize("wd", [0.0, 0.25])
def test_lion_matches_oracle_step_by_step(wd):
    s = _state(SIZES, 21, unaligned=(2, 9))
    lr, b1, b2 = 1e-4, 0.9, 0.99
    # exact zeros of c = 0.5 m + 0.5 g in fp32 where m = -g (b1 = 0.5 below)
    s["m"][6][:100] = -s["g"][6][:100]
    gen = torch.Generator().manual_seed(22)
    for step in range(4):
        beta1 = 0.5 if step == 0 else b1
        x0, m0, g0 = (_np(s[k]) for k in "xmg")
        # the oracle decides sign(c) from the same fp32 values the kernel reads
        m32 = [t.detach().cpu().numpy() for t in s["m"]]
        g32 = [t.detach().cpu().numpy() for t in s["g"]]
        nl = dion.vec_step(s["x"], s["g"], s["m"], None, rule="lion", lr=lr, betas=(beta1, b2),
                           weight_decay=wd)
        assert nl == 1
        torch.cuda.synchronize()
        for i, n in enumerate(SIZES):
            if n == 0:
                continue
            xr, mr = oracle.lion_step(x0[i], g32[i].astype(np.float64), m32[i], lr=lr,
                                      b1=beta1, b2=b2, wd=wd)
            xg, mg = _np([s["x"][i]])[0], _np([s["m"][i]])[0]
            assert np.all(np.abs(xg - xr) <= 2.0 ** -22 * np.abs(xr) + 1e-6 * lr), (step, i)
            assert _rel(mg, mr) <= 1e-6, (step, i)
            if step == 0 and i == 6:            # c == 0: only the decay moved x
                assert np.allclose(xg[:100], x0[i][:100] * (1 - lr * wd), rtol=2 ** -22, atol=0)
        for dst in s["g"]:
            dst.copy_(torch.randn(dst.numel(), generator=gen).to(dst.device) * 1e-2)


def test_many_tensors_take_several_launches():
    sizes = [5 + (i % 7) * 300 for i in range(300)] + [0] * 10
    s = _state(sizes, 31)
    xs, gs, ms, vs = (_np(s[k]) for k in "xgmv")
    nl = dion.vec_step(s["x"], s["g"], s["m"], s["v"], rule="adamw", lr=1e-3, step=3)
    assert nl == 3                                    # 300 non-empty tensors, 128 per launch
    xr, mr, vr, bound = _adamw_ref(xs, gs, ms, vs, t=3, lr=1e-3, **HP)
    torch.cuda.synchronize()
    for i in range(len(sizes)):
        xg = _np([s["x"][i]])[0]
        assert np.all(np.abs(xg - xr[i]) <= bound[i]), i


def test_nonfinite_gradient_stays_in_its_element():
    s = _state([4096, 300], 41)
    s["g"][0][17] = float("nan")
    s["g"][1][5] = float("inf")
    xs, gs, ms, vs = (_np(s[k]) for k in "xgmv")
    dion.vec_step(s["x"], s["g"], s["m"], s["v"], rule="adamw", lr=1e-3, step=2)
    torch.cuda.synchronize()
    with np.errstate(invalid="ignore", over="ignore"):
        xr, _, _, bound = _adamw_ref(xs, gs, ms, vs, t=2, lr=1e-3, **HP)
    xg = _np(s["x"])
    assert np.isnan(xg[0][17]) and not np.isfinite(xg[1][5])
    for i, bad in ((0, 17), (1, 5)):
        keep = np.ones(xg[i].size, bool)
        keep[bad] = False
        assert np.all(np.abs(xg[i][keep] - xr[i][keep]) <= bound[i][keep])


def test_norm_gains_workload_both_rules():
    vw = W.VECTOR_WORKLOADS["norms_h4096_l32"]
    state = [W.vector_state(vw, i, 0, "cuda") for i in range(len(vw.sizes))]
    x, g, m, v = (list(t) for t in zip(*state))
    xs, gs, ms, vs = _np(x), _np(g), _np(m), _np(v)
    dion.vec_step(x, g, m, v, rule="adamw", lr=vw.lr, step=1)
    torch.cuda.synchronize()
    xr, mr, vr, bound = _adamw_ref(xs, gs, ms, vs, t=1, lr=vw.lr, **HP)
    for i in range(len(vw.sizes)):
        assert np.all(np.abs(_np([x[i]])[0] - xr[i]) <= bound[i])
    # then a Lion step from the state AdamW left (lr 1e-4, betas 0.9 / 0.99, no decay)
    x0 = _np(x)
    m32 = [t.detach().cpu().numpy() for t in m]
    g32 = [t.detach().cpu().numpy() for t in g]
    dion.vec_step(x, g, m, None, rule="lion")
    torch.cuda.synchronize()
    for i in range(len(vw.sizes)):
        xr, mr = oracle.lion_step(x0[i], g32[i].astype(np.float64), m32[i], lr=1e-4, b1=0.9,
                                  b2=0.99, wd=0.0)
        assert np.all(np.abs(_np([x[i]])[0] - xr) <= 2.0 ** -22 * np.abs(xr) + 1e-10)
        assert _rel(_np([m[i]])[0], mr) <= 1e-6


def test_prepared_plan_over_steps_matches_oracle():
    """A VecStepPlan marshals the pointer table once; three steps through it equal three
    one-off calls' oracle trajectory (the step number is passed per call)."""
    sizes = [4096] * 65 + [7]                        # 66 tensors: one launch of up to 128
    s = _state(sizes, 51)
    xs, gs, ms, vs = (_np(s[k]) for k in "xgmv")
    plan = dion.VecStepPlan(s["x"], s["g"], s["m"], s["v"], rule="adamw", lr=1e-3)
    bound = [np.zeros(n) for n in sizes]
    for t in range(1, 4):
        assert plan.step(t) == 1
        xs, ms, vs, b = _adamw_ref(xs, gs, ms, vs, t=t, lr=1e-3, **HP)
        bound = [a + c for a, c in zip(bound, b)]
    torch.cuda.synchronize()
    for i in range(len(sizes)):
        assert np.all(np.abs(_np([s["x"][i]])[0] - xs[i]) <= bound[i]), i
