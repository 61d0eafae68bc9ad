"""CurvaDion's momentum-change statistic (RMMC) from the fused update (GPU).

The update kernels take max |M' - M| and max |M| of every matrix from the values they
stream anyway; the status kernel divides them and sets DION_MAT_HIGH_RMMC where the
ratio exceeds the threshold.  Checked against the fp64 oracle's RMMC of the same step
(parity tolerances), against the statistic recomputed from the GPU's own M before and
after the step (fp32 rounding only), and against the closed form RMMC = 1 - mu of a
full-rank step on a zero gradient.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_harness import GpuRun
from rank_orthonormalized_optimizer_b200 import MAT_HIGH_RMMC, VIEW_RMMC

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _own_rmmc(before, after):
    d = (after.double() - before.double()).flatten(1).abs().max(dim=1).values
    s = before.double().flatten(1).abs().max(dim=1).values
    return (d / s).cpu().numpy()


@pytest.mark.parametrize("path", ["tensor", "simt"])
@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_rmmc_matches_the_oracle(precision, path):
    wl = W.custom(f"rmmc_{precision}", [(3, 256, 128, 32), (2, 130, 200, 48)],
                  precision=precision, steps=3)
    run = GpuRun(wl, kernel_path=path)
    run.step(1)
    for bi in range(2):     # from M = 0 every moved momentum has no scale: +inf
        assert np.all(np.isinf(run.opt.view(bi, VIEW_RMMC, run.ws).cpu().numpy()))
    run.step(wl.steps - 2)
    before = [m.clone() for m in run.M]
    run.step(1)
    for bi, b in enumerate(wl.buckets):
        got = run.opt.view(bi, VIEW_RMMC, run.ws).double().cpu().numpy()
        own = _own_rmmc(before[bi], run.M[bi])
        assert np.abs(got - own).max() <= 1e-6 * own.max(), (got, own)
        for s in range(b.count):
            X = W.weights(wl, bi, slots=[s])[0].double().numpy()
            M = np.zeros((b.m, b.n))
            Q = W.right_factor(wl, bi, slots=[s])[0].double().numpy()
            for t in range(wl.steps):
                G = W.gradient(wl, bi, t, slots=[s])[0].double().numpy()
                M_prev = M
                X, M, Q, _, _ = oracle.dion_step(X, M, G, Q, wl.mu, wl.lr)
            ref = oracle.rmmc(M_prev, M)
            assert abs(got[s] - ref) <= TOL[precision] * ref, (bi, s, got[s], ref)


def test_zero_gradient_at_full_rank_gives_one_minus_mu():
    """r = m = n: P P^T = I, so a step with G = 0 gives M' = mu M and RMMC = 1 - mu."""
    wl = W.custom("rmmc_decay", [(2, 64, 64, 64), (1, 96, 96, 96)], precision="fp32", steps=2)
    run = GpuRun(wl)
    run.step(1)
    run.step(1, G_override=[torch.zeros_like(x) for x in run.X])
    for bi in range(2):
        got = run.opt.view(bi, VIEW_RMMC, run.ws).cpu().numpy()
        assert np.abs(got - (1 - wl.mu)).max() <= 1e-5, got


def test_gate_bit_marks_the_matrices_above_the_threshold():
    wl = W.custom("rmmc_gate", [(6, 256, 128, 32)], precision="bf16", steps=3)
    probe = GpuRun(wl)
    probe.step(3)
    vals = np.sort(probe.opt.view(0, VIEW_RMMC, probe.ws).cpu().numpy())
    tau = float(0.5 * (vals[2] + vals[3]))          # three matrices above, three below
    run = GpuRun(wl, rmmc_threshold=tau)
    run.step(3)
    got = run.opt.view(0, VIEW_RMMC, run.ws).cpu().numpy()
    st = run.status.cpu().numpy()
    assert np.array_equal((st & MAT_HIGH_RMMC) != 0, got > tau), (st, got, tau)
    assert ((st & MAT_HIGH_RMMC) != 0).sum() == 3
