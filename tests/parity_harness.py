"""Run the CUDA Dion step and the fp64 oracle on the same seeded inputs (test infrastructure).

Inputs come from ``workloads``; the GPU side runs every matrix of every bucket through
the C ABI, the oracle runs the sampled slots one by one.  Matrices are independent, so
a sampled slot's oracle result is its exact reference whatever the bucket size.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

import oracle
import workloads as W
from rank_orthonormalized_optimizer_b200 import VIEW_P, DionB200

SMALL_PARAMS = 64 << 20     # workloads up to this many parameters are drawn on the CPU


@dataclass
class Report:
    rel_x: float = 0.0
    rel_m: float = 0.0
    rel_q: float = 0.0
    rel_q_w: float = 0.0           # Q's error with each column weighted by ||R_j|| (see below)
    rel_dx: float = 0.0
    dx_floor: float = 0.0          # fp32 rounding of the stored X, relative to ||dX||
    orth_gpu: float = 0.0          # max |P^T P - I| over every matrix of the GPU run
    status_or: int = 0
    per_slot: list = field(default_factory=list)

    def __str__(self):
        return (f"rel_F X {self.rel_x:.3e}  M {self.rel_m:.3e}  Q {self.rel_q:.3e} "
                f"(R-weighted {self.rel_q_w:.3e})  "
                f"dX {self.rel_dx:.3e} (fp32 floor {self.dx_floor:.1e})  |P^T P - I| {self.orth_gpu:.3e}  status {self.status_or}")


class GpuRun:
    """State of one workload on the GPU, stepped through the C ABI."""

    def __init__(self, wl: W.Workload, *, precision=None, kernel_path="tensor", orth_mode="auto",
                 gen_device=None, **opts):
        self.wl = wl
        self.gen = gen_device or ("cpu" if wl.params <= SMALL_PARAMS else "cuda")
        self.opt = DionB200([(b.count, b.m, b.n, b.r) for b in wl.buckets], mu=wl.mu,
                            precision=precision or wl.precision, kernel_path=kernel_path,
                            orth_mode=orth_mode, **opts)
        nb = len(wl.buckets)
        self.X = [W.weights(wl, i, self.gen).cuda() for i in range(nb)]
        self.X0 = [x.clone() for x in self.X] if wl.params <= SMALL_PARAMS else None
        self.M = [W.momentum(wl, i, "cuda") for i in range(nb)]
        self.Q = [W.right_factor(wl, i, self.gen).cuda() for i in range(nb)]
        self.G = [torch.empty_like(x) for x in self.X]
        self.ws = self.opt.alloc_workspace()
        self.status = self.opt.alloc_status()
        self.t = 0

    def step(self, steps: int = 1, G_override=None):
        for _ in range(steps):
            for i in range(len(self.wl.buckets)):
                if G_override is not None:
                    self.G[i].copy_(G_override[i])
                else:
                    self.G[i].copy_(W.gradient(self.wl, i, self.t, self.gen))
                if self.wl.grad == "fixed_sqrt_spectrum":
                    self.M[i].zero_()
            self.opt.step(self.X, self.M, self.G, self.Q, self.wl.lr, self.ws, self.status)
            self.t += 1
        torch.cuda.synchronize()

    def P(self, bi):
        return self.opt.view(bi, VIEW_P, self.ws)

    def orth_error(self) -> float:
        worst = 0.0
        for bi, b in enumerate(self.wl.buckets):
            P = self.P(bi)
            for c0 in range(0, b.count, 16):
                p = P[c0:c0 + 16].double()
                g = torch.bmm(p.transpose(1, 2), p)
                g -= torch.eye(b.r, dtype=torch.float64, device=g.device)
                worst = max(worst, g.abs().max().item())
        return worst


def oracle_slot(wl: W.Workload, bi: int, slot: int, steps: int, gen: str):
    """The oracle's X, M, Q after ``steps`` steps of one matrix (fp64), plus its X0."""
    X0 = W.weights(wl, bi, gen, slots=[slot])[0].cpu().double().numpy()
    M = W.momentum(wl, bi, "cpu", slots=[slot])[0].double().numpy()
    Q = W.right_factor(wl, bi, gen, slots=[slot])[0].cpu().double().numpy()
    grads = (W.gradient(wl, bi, t, gen, slots=[slot])[0].cpu().double().numpy()
             for t in range(steps))
    X, M, Q, P, R = oracle.run_steps(X0, M, Q, grads, wl.mu, wl.lr,
                                     reset_momentum=(wl.grad == "fixed_sqrt_spectrum"))
    return X0, X, M, Q, P, R


def rel_q_weighted(q_gpu, Q_ref, R_ref) -> float:
    """||(Q_gpu - Q_ref) D||_F / ||Q_ref D||_F with D = diag(||R_ref[:, j]||).

    Q = colnorm(R): column j is R_j / ||R_j||.  The operands' rounding perturbs R_j by
    about eps ||B|| whatever ||R_j|| is, so the direction of a column whose norm is small
    beside ||B|| (full rank: the last columns) is fixed only to eps ||B|| / ||R_j||.
    Weighting each column's error by the norm of the R column it normalises measures Q
    at the accuracy the arithmetic gives it (it is R's relative error, column directions
    only)."""
    d = np.sqrt(np.sum(R_ref * R_ref, axis=0))
    return float(np.linalg.norm((q_gpu - Q_ref) * d) / max(np.linalg.norm(Q_ref * d), 1e-300))


def compare(run: GpuRun, steps: int, slots_per_bucket=None) -> Report:
    """Step the GPU run ``steps`` times and compare sampled slots with the oracle."""
    run.step(steps)
    rep = Report()
    for bi, b in enumerate(run.wl.buckets):
        if slots_per_bucket is None:
            slots = range(b.count) if b.count <= 4 else sorted({0, b.count - 1})
        else:
            slots = sorted({s % b.count for s in slots_per_bucket})
        for s in slots:
            X0, X, M, Q, P, R = oracle_slot(run.wl, bi, s, steps, run.gen)
            gx = run.X[bi][s].double().cpu().numpy()
            gm = run.M[bi][s].double().cpu().numpy()
            gq = run.Q[bi][s].double().cpu().numpy()
            # X is fp32 state: each step rounds every element by up to half an ulp, a noise
            # floor of about 2^-24 ||X||_F sqrt(steps) in dX that no kernel can remove
            floor = 2.0 ** -24 * np.linalg.norm(X0) * math.sqrt(steps) / max(
                np.linalg.norm(X - X0), 1e-300)
            one = dict(bucket=bi, slot=s, rel_x=oracle.rel_fro(gx, X), rel_m=oracle.rel_fro(gm, M),
                       rel_q=oracle.rel_fro(gq, Q), rel_q_w=rel_q_weighted(gq, Q, R),
                       rel_dx=oracle.rel_fro(gx - X0, X - X0), dx_floor=floor)
            rep.per_slot.append(one)
            rep.rel_x = max(rep.rel_x, one["rel_x"])
            rep.rel_m = max(rep.rel_m, one["rel_m"])
            rep.rel_q = max(rep.rel_q, one["rel_q"])
            rep.rel_q_w = max(rep.rel_q_w, one["rel_q_w"])
            rep.rel_dx = max(rep.rel_dx, one["rel_dx"])
            rep.dx_floor = max(rep.dx_floor, one["dx_floor"])
    rep.orth_gpu = run.orth_error()
    rep.status_or = int(np.bitwise_or.reduce(run.status.cpu().numpy()))
    return rep


def update_norm_error(run: GpuRun, X_before) -> float:
    """max over matrices of | ||X' - X||_F - lr s sqrt(r) | / (lr s sqrt(r))."""
    worst = 0.0
    for bi, b in enumerate(run.wl.buckets):
        want = run.wl.lr * math.sqrt(b.m / b.n) * math.sqrt(b.r)
        d = (run.X[bi].double() - X_before[bi].double()).flatten(1).norm(dim=1)
        worst = max(worst, ((d - want).abs() / want).max().item())
    return worst
