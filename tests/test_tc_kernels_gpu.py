"""Tensor-core kernels against the SIMT kernels on identical inputs (GPU).

One step through each kernel path from the same state: P isolates B Q (the
orthonormalisation that follows is the same code on both paths), R isolates B^T P,
and M, X isolate the fused update.  Both paths round B, Q, P, R to bf16 and differ by
fp32 accumulation order, ~1e-6 relative in P.  Rounding P to bf16 then flips a
fraction ~delta / 2^-8 of its entries by one bf16 ulp, which moves R, M and dX by about
sqrt(delta * 2^-8) ~ 1e-4 (dX also inherits the flips of the bf16 R and Q).  A wrong
tile, descriptor or swizzle gives errors of order 1.
"""
import numpy as np
import pytest
import torch

import workloads as W
from parity_harness import GpuRun
from rank_orthonormalized_optimizer_b200 import VIEW_R

pytestmark = pytest.mark.gpu

SHAPES = [
    [(3, 256, 128, 32)],
    [(2, 512, 1024, 256)],
    [(2, 1024, 512, 64)],
    [(3, 300, 136, 16), (2, 130, 200, 48)],     # ragged tiles in every direction
    [(1, 1000, 520, 320)],                      # two N tiles, ragged
    [(2, 640, 384, 128)],
]


def _rel(a, b):
    return ((a.double() - b.double()).norm() / b.double().norm().clamp_min(1e-30)).item()


@pytest.mark.parametrize("buckets", SHAPES, ids=lambda b: "_".join("x".join(map(str, s)) for s in b))
def test_tensor_views_match_simt(buckets):
    wl = W.custom("tcv_" + "_".join("x".join(map(str, s)) for s in buckets), buckets,
                  precision="bf16", steps=1)
    a = GpuRun(wl, kernel_path="tensor")
    b = GpuRun(wl, kernel_path="simt")
    a.step(1)
    b.step(1)
    for i, bk in enumerate(wl.buckets):
        pa, pb = a.P(i), b.P(i)
        ra, rb = a.opt.view(i, VIEW_R, a.ws), b.opt.view(i, VIEW_R, b.ws)
        ep, er = _rel(pa, pb), _rel(ra, rb)
        em = _rel(a.M[i], b.M[i])
        ex = _rel(a.X[i] - a.X0[i], b.X[i] - b.X0[i])
        print(bk, f"P {ep:.2e} R {er:.2e} M {em:.2e} dX {ex:.2e}")
        assert ep < 1e-4, ("B Q", ep)
        assert er < 1e-3, ("B^T P", er)
        assert em < 2e-4, ("update M", em)
        assert ex < 2e-3, ("update X", ex)
    assert int(a.status.max()) & 12 == 0


def test_bounded_waits_time_out_cleanly():
    """With a one-poll wait limit the tensor-core kernels give up, report
    DION_MAT_TIMEOUT, and leave the context usable for the next (normal) step."""
    wl = W.custom("timeout", [(4, 512, 4096, 64)], precision="bf16", steps=1)
    run = GpuRun(wl, kernel_path="tensor", max_wait_spins=1)
    run.step(1)
    st = run.status.cpu().numpy()
    assert np.any(st & 8), st
    ok = GpuRun(wl, kernel_path="tensor")
    ok.step(1)
    assert not np.any(ok.status.cpu().numpy() & 8)
    ref = GpuRun(wl, kernel_path="simt")
    ref.step(1)
    assert _rel(ok.M[0], ref.M[0]) < 1e-5
    torch.cuda.synchronize()
