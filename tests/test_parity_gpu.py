"""Parity of the CUDA Dion step with the fp64 oracle on every workload (GPU).

Tolerances (relative Frobenius error per matrix, max over the checked matrices):
  fp32 contractions   X, M and Q <= 1e-4 after the step count of the workload
  bf16-input GEMMs    X and M <= 2e-2; Q <= 2e-2 with its columns weighted by the norms
                      of the R columns they normalise (a bf16 operand perturbs R_j by
                      about 2^-8 ||B||, so the direction of a column of R that is small
                      beside ||B|| -- the last ones at full rank -- is fixed only to
                      2^-8 ||B|| / ||R_j||; weighted, Q's error is R's)
  every matrix        max |P^T P - I| <= 1e-4 on the GPU's own P
The weight change dX = X_T - X_0 is checked too, since X_0 dominates X.  Its bound
has two parts: the operand rounding (bf16 operands carry a relative error up to 2^-8
per product, fp32 ones 2^-23 amplified by the subspace conditioning: fp32 1e-3, bf16
6e-2 over the step count), plus the rounding of the fp32 state X itself, which every
step perturbs by up to half an ulp per element: 3 x 2^-24 ||X_0||_F sqrt(T) / ||dX||_F.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_harness import GpuRun, compare, oracle_slot, update_norm_error

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}
TOL_DX = {"fp32": 1e-3, "bf16": 6e-2}
ORTH_TOL = 1e-4


def _check(rep, precision, dx=True, full_rank=False):
    print(rep)
    assert rep.rel_x <= TOL[precision], rep
    assert rep.rel_m <= TOL[precision], rep
    assert rep.rel_q_w <= TOL[precision], rep
    if precision == "fp32" and not full_rank:
        # below full rank R's columns are the leading directions, none small beside
        # ||B||: Q itself must meet the bound (at full rank the last columns of R are
        # as small as B's smallest singular values, and only the weighted error is due)
        assert rep.rel_q <= TOL[precision], rep
    assert rep.orth_gpu <= ORTH_TOL, rep
    if dx:
        assert rep.rel_dx <= TOL_DX[precision] + 3 * rep.dx_floor, rep
    assert not rep.status_or & (4 | 8), rep      # no non-finite Gram, no timeout


@pytest.mark.parametrize("path", ["tensor", "simt"])
@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_single_256x128_r32(path, precision):
    wl = W.WORKLOADS["single_256x128_r32"]
    run = GpuRun(wl, precision=precision, kernel_path=path)
    rep = compare(run, wl.steps)
    _check(rep, precision)


@pytest.mark.parametrize("path", ["tensor", "simt"])
def test_fullrank_16x1024_polar(path):
    """Full rank on a fixed B: M' = mu B exactly, and the distance of P Q^T to the polar
    factor U V^T follows the oracle's curve over 50 steps."""
    wl = W.WORKLOADS["fullrank_16x1024x1024"]
    run = GpuRun(wl, kernel_path=path)
    checkpoints = [1, 5, 10, 20, 50]
    slots = [0, 15]
    svd = {s: W.fixed_b_svd(wl, 0, s) for s in slots}
    polar = {s: (u @ v.T) for s, (u, _, v) in svd.items()}
    gpu_curve = {s: [] for s in slots}
    done = 0
    for c in checkpoints:
        run.step(c - done)
        done = c
        P = run.P(0)
        for s in slots:
            pq = P[s].double().cpu() @ run.Q[0][s].double().cpu().T
            gpu_curve[s].append((torch.linalg.norm(pq - polar[s]) / torch.linalg.norm(polar[s])).item())
        if c == 10:
            for s in slots:
                B = W.gradient(wl, 0, 0, run.gen, slots=[s])[0].double()
                rel = (torch.linalg.norm(run.M[0][s].double().cpu() - wl.mu * B) /
                       torch.linalg.norm(wl.mu * B)).item()
                assert rel <= TOL["fp32"], rel
    for s in slots:
        X0 = W.weights(wl, 0, run.gen, slots=[s])[0].double().numpy()
        Q = W.right_factor(wl, 0, run.gen, slots=[s])[0].double().numpy()
        B = W.gradient(wl, 0, 0, run.gen, slots=[s])[0].double().numpy()
        X, M = X0, np.zeros_like(B)
        curve, t = [], 0
        for c in checkpoints:
            while t < c:
                X, M, Q, P, R = oracle.dion_step(X, np.zeros_like(B), B, Q, wl.mu, wl.lr)
                t += 1
            curve.append(np.linalg.norm(P @ Q.T - polar[s].numpy()) / np.linalg.norm(polar[s].numpy()))
        print("slot", s, "oracle", np.round(curve, 6), "gpu", np.round(gpu_curve[s], 6))
        assert np.abs(np.array(curve) - np.array(gpu_curve[s])).max() <= 1e-4
        assert oracle.rel_fro(run.X[0][s].double().cpu().numpy(), X) <= TOL["fp32"]
        assert oracle.rel_fro(run.M[0][s].double().cpu().numpy(), M) <= TOL["fp32"]
    assert run.orth_error() <= ORTH_TOL


@pytest.mark.parametrize("path", ["tensor", "simt"])
def test_transformer_h2048_l24(path):
    wl = W.WORKLOADS["transformer_h2048_l24_r256"]
    run = GpuRun(wl, kernel_path=path)
    rep = compare(run, wl.steps, slots_per_bucket=wl.sample_slots)
    _check(rep, "bf16")


def test_transformer_h4096_l32_ff11008():
    """The 7B-like workload at full size (224 matrices, 6.48e9 parameters)."""
    wl = W.WORKLOADS["transformer_h4096_l32_ff11008_r256"]
    run = GpuRun(wl, kernel_path="tensor")
    rep = compare(run, wl.steps, slots_per_bucket=wl.sample_slots)
    _check(rep, "bf16")
    # Gram sums over m = 4096 and 11008 rows: with the tensor cores' biased fp32
    # accumulation left unchunked, max|P^T P - I| grew with m (7.5e-5 at 11008) while
    # the second-pass test, blind to a uniform bias, saw nothing; chunked it is ~5e-6
    assert rep.orth_gpu <= 2e-5, rep


@pytest.mark.parametrize("r", [64, 128, 256, 512, 1024, 2048, 4096, 8192])
def test_square_8x8192_rank_sweep(r):
    """Every rank of the sweep on 8 stacked 8192 x 8192 fp32 matrices, 10 steps, slot 0
    against the oracle (the oracle's 10 steps of one 8192 x 8192 matrix take up to a few
    minutes on the host at r = 8192)."""
    wl = W.WORKLOADS[f"square_8x8192_r{r}"]
    run = GpuRun(wl)
    rep = compare(run, wl.steps, slots_per_bucket=(0,))
    _check(rep, "fp32", full_rank=(r == 8192))


# ------------------------------------------------------------------ edge cases

EDGE = [
    ("ragged", [(3, 200, 136, 16), (2, 130, 72, 48)]),
    ("tall_thin", [(2, 1000, 24, 16)]),
    ("full_rank_square", [(2, 64, 64, 64)]),
    ("wide", [(2, 48, 520, 32)]),
    ("many_small", [(300, 32, 16, 16)]),
    # r > 256: the recursive factorisation, with a last block of 16 (272 = 256 + 16;
    # 784 = 512 + 272) and row counts that are not multiples of the 128-row tiles
    ("recursive_chol", [(2, 600, 560, 272), (2, 1100, 800, 784)]),
    # r <= 256 with m over 512 rows: the Gram adds 512-row K chunks in fp32 (3 chunks,
    # the last ragged; 5 chunks over a 2 x 2 tile grid with r = 144)
    ("chunked_gram", [(3, 1300, 96, 64), (2, 2100, 256, 144)]),
    # with stack_orth, buckets of equal m and r share one orthonormalisation stack: the
    # first and third here (the stack completes after the third bucket's B Q), the
    # second alone
    ("stacked_orth", [(3, 256, 128, 32), (2, 300, 64, 48), (2, 256, 384, 32)]),
    # a stack on the recursive factorisation (r = 272 > 256)
    ("stacked_recursive", [(2, 600, 560, 272), (1, 600, 320, 272)]),
]


@pytest.mark.parametrize("path", ["tensor", "simt"])
@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("name,buckets", EDGE, ids=[e[0] for e in EDGE])
def test_edge_shapes(name, buckets, precision, path):
    wl = W.custom(f"edge_{name}", buckets, precision=precision, steps=4)
    run = GpuRun(wl, kernel_path=path, stack_orth=name.startswith("stacked"))
    X_before = [x.clone() for x in run.X]
    rep = compare(run, 4)
    _check(rep, precision, dx=False)


@pytest.mark.parametrize("mode,bit", [("householder", 1), ("cholqr2", 2), ("cholqr", 0)])
def test_orth_modes(mode, bit):
    wl = W.custom(f"orth_{mode}", [(3, 256, 128, 32), (2, 300, 64, 48)], precision="fp32", steps=5)
    run = GpuRun(wl, orth_mode=mode)
    rep = compare(run, 5)
    _check(rep, "fp32")
    st = run.status.cpu().numpy()
    if bit:
        assert np.all(st & bit), st


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_rank_deficient_large_r_falls_back(precision):
    """r = 320 > 256 (recursive factorisation).  Slot 0 gets B of rank 64 < r: in fp32
    its Gram is singular to working precision, the factorisation fails a pivot or the
    diagonal-ratio test, and the matrix goes to Householder QR (bf16 rounding of B
    makes it full rank with small singular values, so there the route is not fixed).
    Its P is not unique (only col(B) is fixed), so the check is the invariants:
    P^T P = I and B - P P^T B = 0 (to the rounding of B in bf16).  Slot 1 gets a
    full-rank Gaussian B in the same bucket and must match the oracle's step."""
    m, n, r, k = 512, 384, 320, 64
    wl = W.custom("lowrank_r320", [(2, m, n, r)], precision=precision, steps=1)
    run = GpuRun(wl)
    X0, Q0 = run.X[0].clone(), run.Q[0].clone()
    g = torch.Generator().manual_seed(5)
    U = torch.linalg.qr(torch.randn(m, k, generator=g, dtype=torch.float64))[0]
    V = torch.linalg.qr(torch.randn(n, k, generator=g, dtype=torch.float64))[0]
    G = torch.stack([U @ V.T, torch.randn(m, n, generator=g, dtype=torch.float64)]).float()
    run.step(1, G_override=[G.cuda()])
    st = run.status.cpu().numpy()
    assert not st[1] & 1, st
    if precision == "fp32":
        assert st[0] & 1, st
    assert not np.any(st & (4 | 8)), st
    assert run.orth_error() <= ORTH_TOL
    P = run.P(0)[0].double().cpu()
    B = G[0].double()
    res = B - P @ (P.T @ B)
    assert (res.norm() / B.norm()).item() <= (1e-5 if precision == "fp32" else 1e-2)
    X, M, Q, _, _ = oracle.dion_step(X0[1].cpu().numpy(), np.zeros((m, n)), G[1].numpy(),
                                     Q0[1].cpu().numpy(), wl.mu, wl.lr)
    tol = TOL[precision]
    assert oracle.rel_fro(run.X[0][1].double().cpu().numpy(), X) <= tol
    assert oracle.rel_fro(run.M[0][1].double().cpu().numpy(), M) <= tol


def test_shifted_iteration_recovers_qr_of_ill_conditioned_p0():
    """r = 384 > 256 and cond(P0) ~ 1e5: Cholesky-QR fails its diagonal-ratio test and the
    shifted Cholesky-QR iteration (not Householder) produces P.  Whatever route, P must
    be P0's Q factor: P^T P = I, and R = P^T P0 upper triangular with a positive
    diagonal, P0 = P R.  These hold to rounding whatever the conditioning (the entries of
    P itself do not: they move by up to cond(P0) u)."""
    m, n, r = 640, 512, 384
    wl = W.custom("illcond_r384", [(2, m, n, r)], precision="fp32", steps=1)
    run = GpuRun(wl)
    Q0 = run.Q[0].double().cpu()
    g = torch.Generator().manual_seed(11)
    U = torch.linalg.qr(torch.randn(2, m, n, generator=g, dtype=torch.float64))[0]
    V = torch.linalg.qr(torch.randn(2, n, n, generator=g, dtype=torch.float64))[0]
    sig = torch.logspace(0, -5, n, dtype=torch.float64)
    B = (U * sig) @ V.transpose(1, 2)
    run.step(1, G_override=[B.float().cuda()])
    st = run.status.cpu().numpy()
    assert np.all(st & 1) and not np.any(st & (4 | 8)), st
    assert run.orth_error() <= ORTH_TOL
    P = run.P(0).double().cpu()
    P0 = B.float().double() @ Q0
    R = P.transpose(1, 2) @ P0
    for i in range(2):
        scale = torch.linalg.norm(P0[i])
        # both at the level of P's own orthogonality error (<= orth_tol = 2e-5 at exit)
        assert torch.linalg.norm(torch.tril(R[i], -1)) / scale <= 1e-4
        assert torch.all(torch.diagonal(R[i]) > 0)
        assert torch.linalg.norm(P0[i] - P[i] @ torch.triu(R[i])) / scale <= 1e-4


def test_update_norm_is_lr_s_sqrt_r():
    """||X' - X||_F = lr sqrt(m/n) sqrt(r) for orthonormal P and unit-column Q."""
    for precision, tol in (("fp32", 1e-5), ("bf16", 1e-2)):
        wl = W.custom(f"norm_{precision}", [(4, 512, 256, 64), (2, 256, 512, 32)],
                      precision=precision, steps=1)
        run = GpuRun(wl)
        for _ in range(3):
            before = [x.clone() for x in run.X]
            run.step(1)
            assert update_norm_error(run, before) <= tol


def test_zero_gradient_gives_zero_update():
    wl = W.custom("zero", [(2, 128, 64, 16)], precision="fp32", steps=1)
    run = GpuRun(wl)
    X0 = run.X[0].clone()
    run.step(1, G_override=[torch.zeros_like(run.X[0])])
    assert torch.equal(run.X[0], X0)
    assert torch.count_nonzero(run.M[0]) == 0 and torch.count_nonzero(run.Q[0]) == 0
    st = run.status.cpu().numpy()
    assert np.all(st & 16), st            # zero columns reported
    assert not np.any(st & 8)


def test_nonfinite_gradient_is_reported_and_contained():
    wl = W.custom("nan", [(3, 128, 64, 16)], precision="fp32", steps=1)
    run = GpuRun(wl)
    G = W.gradient(wl, 0, 0).cuda()
    G[1, 5, 7] = float("nan")
    X_ok = run.X[0][[0, 2]].clone()
    run.step(1, G_override=[G])
    st = run.status.cpu().numpy()
    assert st[1] & 4 and not (st[0] & 4) and not (st[2] & 4), st
    for s in (0, 2):
        X0, X, M, Q, P, R = oracle_slot(wl, 0, s, 1, "cpu")
        assert oracle.rel_fro(run.X[0][s].double().cpu().numpy(), X) <= TOL["fp32"]


def test_deterministic_and_resumable():
    """Two runs are bitwise equal, and 3 + 3 steps through a saved state equal 6 steps."""
    wl = W.custom("det", [(4, 384, 256, 32), (3, 256, 512, 48)], precision="bf16", steps=6)
    a = GpuRun(wl)
    a.step(6)
    b = GpuRun(wl)
    b.step(6)
    for i in range(2):
        assert torch.equal(a.X[i], b.X[i]) and torch.equal(a.M[i], b.M[i])
        assert torch.equal(a.Q[i], b.Q[i])
    c = GpuRun(wl)
    c.step(3)
    saved = [(x.cpu(), m.cpu(), q.cpu()) for x, m, q in zip(c.X, c.M, c.Q)]
    del c
    d = GpuRun(wl)
    for i, (x, m, q) in enumerate(saved):
        d.X[i].copy_(x); d.M[i].copy_(m); d.Q[i].copy_(q)
    d.t = 3
    d.step(3)
    for i in range(2):
        assert torch.equal(a.X[i], d.X[i]) and torch.equal(a.M[i], d.M[i])


@pytest.mark.parametrize("stack_orth", [False, True])
@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_step_from_host_equals_device_step(precision, stack_orth):
    """The host-gradient entry point uploads the buckets of one orthonormalisation stack
    after another (the largest stack first) and steps a stack as soon as its gradients
    have arrived; over several steps, each overwriting G that the previous step's update
    read, it gives bitwise the device step's state and status.  The buckets are listed
    smallest first, so the upload order is not theirs; r = 272 takes the recursive
    factorisation and the fallback graph."""
    wl = W.custom("from_host", [(2, 256, 128, 32), (3, 600, 560, 272), (4, 1024, 512, 64),
                                (1, 256, 64, 32)],
                  precision=precision, steps=3)
    # with stack_orth the first and last bucket share an orthonormalisation stack
    a = GpuRun(wl, stack_orth=stack_orth)
    b = GpuRun(wl, stack_orth=stack_orth)
    nb = len(wl.buckets)
    host_status = torch.zeros(b.opt.num_matrices, dtype=torch.int32).pin_memory()
    for t in range(3):
        grads = [W.gradient(wl, i, t, "cpu") for i in range(nb)]
        a.step(1, G_override=[g.cuda() for g in grads])
        pinned = [g.pin_memory() for g in grads]
        b.opt.step_from_host(b.X, b.M, b.G, b.Q, pinned, wl.lr, b.ws, b.status, host_status)
        torch.cuda.synchronize()
        for i in range(nb):
            assert torch.equal(a.X[i], b.X[i]) and torch.equal(a.M[i], b.M[i]), (t, i)
            assert torch.equal(a.Q[i], b.Q[i]), (t, i)
            assert torch.equal(b.G[i].cpu(), grads[i])
        assert torch.equal(host_status, a.status.cpu()), t
        assert torch.equal(b.status.cpu(), a.status.cpu()), t


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_stacked_orthonormalisation_is_bucket_by_bucket_bitwise(precision):
    """With stack_orth, buckets of equal m and r share one orthonormalisation stack; every
    matrix is still orthonormalised on its own (its own Gram tiles, its own Cholesky), so
    a bucket's X, M, Q and status are bit for bit those of the same bucket planned alone."""
    shapes = [(3, 256, 128, 32), (2, 256, 384, 32), (2, 600, 560, 272), (1, 600, 320, 272)]
    wl = W.custom(f"stacked_{precision}", shapes, precision=precision, steps=3)
    together = GpuRun(wl, stack_orth=True)
    together.step(3)
    for i, b in enumerate(shapes):
        alone_wl = W.custom(f"stacked_{precision}", [b], precision=precision, steps=3)
        alone = GpuRun(alone_wl)
        # the same inputs: bucket i's seeds under the stacked workload's name and index
        alone.X[0].copy_(W.weights(wl, i, alone.gen).cuda())
        alone.Q[0].copy_(W.right_factor(wl, i, alone.gen).cuda())
        for t in range(3):
            alone.step(1, G_override=[W.gradient(wl, i, t, alone.gen).cuda()])
        assert torch.equal(alone.X[0], together.X[i]), i
        assert torch.equal(alone.M[0], together.M[i]) and torch.equal(alone.Q[0], together.Q[i]), i
        lo = sum(s[0] for s in shapes[:i])
        assert torch.equal(alone.status.cpu(), together.status.cpu()[lo:lo + b[0]]), i


def test_tensor_and_simt_paths_agree():
    wl = W.custom("paths", [(6, 1024, 512, 64), (4, 512, 1024, 128)], precision="bf16", steps=3)
    a = GpuRun(wl, kernel_path="tensor")
    b = GpuRun(wl, kernel_path="simt")
    a.step(3)
    b.step(3)
    for i in range(2):
        dm = (a.M[i] - b.M[i]).norm() / b.M[i].norm()
        dx = ((a.X[i] - a.X0[i]) - (b.X[i] - b.X0[i])).norm() / (b.X[i] - b.X0[i]).norm()
        print(i, dm.item(), dx.item())
        assert dm <= 1e-3 and dx <= 1e-2


def test_launch_count_and_profile():
    wl = W.custom("prof", [(2, 256, 128, 32), (1, 128, 256, 16)], precision="bf16", steps=1)
    run = GpuRun(wl)
    run.opt.profile_enable(True)
    run.step(2)
    prof = run.opt.profile_read()
    assert run.opt.last_launch_count > 0
    # on the tensor path B = M + G is formed inside the B Q kernel (no form_b launch)
    used = [k for k in prof if k != "form_b"]
    assert all(prof[k][0] > 0 and prof[k][1] > 0 for k in used), prof
    assert prof["form_b"][1] == 0, prof
