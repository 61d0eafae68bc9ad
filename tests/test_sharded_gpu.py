"""The row-sharded CUDA step, its ranks emulated on one GPU (GPU).

A world of w ranks is w handles of DionB200RowSharded, each with its own workspace
and its own rows of X, M and G.  At every exchange the handles' buffers are summed by
torch on the one stream and the sum is written back into each: each rank's kernels
have finished their part when the sum runs, and no kernel waits on another rank.
Stacked back together, the ranks' rows must match the fp64 oracle's whole-matrix step
within the parity tolerances; every rank must hold the same Q and status bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from parity_harness import oracle_slot, rel_q_weighted
from rank_orthonormalized_optimizer_b200 import VIEW_P, DionB200RowSharded

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}
ORTH_TOL = 1e-4


class Emulated:
    def __init__(self, wl, world, precision, orth_mode="auto"):
        self.wl, self.world = wl, world
        shapes = [(b.count, b.m, b.n, b.r) for b in wl.buckets]
        self.h = [DionB200RowSharded(shapes, k, world, mu=wl.mu, precision=precision,
                                     orth_mode=orth_mode) for k in range(world)]
        nb = len(wl.buckets)
        self.rows = [[h.row_ranges[i] for h in self.h] for i in range(nb)]
        X = [W.weights(wl, i).cuda() for i in range(nb)]
        Q = [W.right_factor(wl, i).cuda() for i in range(nb)]
        self.X = [[X[i][:, r0:r0 + mk].contiguous() for (r0, mk) in self.rows[i]]
                  for i in range(nb)]
        self.M = [[torch.zeros_like(x) for x in xs] for xs in self.X]
        self.Q = [[Q[i].clone() for _ in range(world)] for i in range(nb)]
        self.ws = [h.alloc_workspace() for h in self.h]
        self.st = [h.alloc_status() for h in self.h]
        self.kinds = []
        self.t = 0

    def step(self, G_full=None):
        nb = len(self.wl.buckets)
        G = G_full or [W.gradient(self.wl, i, self.t).cuda() for i in range(nb)]
        Gk = [[G[i][:, r0:r0 + mk].contiguous() for (r0, mk) in self.rows[i]] for i in range(nb)]
        xs = [h.begin([self.X[i][k] for i in range(nb)], [self.M[i][k] for i in range(nb)],
                      [Gk[i][k] for i in range(nb)], [self.Q[i][k] for i in range(nb)],
                      self.wl.lr, self.ws[k], self.st[k])
              for k, h in enumerate(self.h)]
        kinds = []
        while xs[0][1] is not None:
            assert len({x[0] for x in xs}) == 1 and len({x[1].numel() for x in xs}) == 1, xs
            kinds.append(xs[0][0])
            total = xs[0][1].clone()
            for _, buf in xs[1:]:
                total += buf
            for _, buf in xs:
                buf.copy_(total)
            xs = [h.advance() for h in self.h]
        assert all(x[1] is None for x in xs)
        self.kinds.append(kinds)
        self.t += 1

    def whole(self, i):
        """Stacked X, M of bucket i, the Q of rank 0 and the stacked P of the last step."""
        X = torch.cat(self.X[i], dim=1)
        M = torch.cat(self.M[i], dim=1)
        P = torch.cat([h.view(i, VIEW_P, ws) for h, ws in zip(self.h, self.ws)], dim=1)
        return X, M, self.Q[i][0], P


def _same_on_every_rank(em):
    for qs in em.Q:
        assert all(torch.equal(q, qs[0]) for q in qs[1:])
    assert all(torch.equal(s, em.st[0]) for s in em.st[1:])


def _orth_err(P):
    p = P.double()
    g = torch.bmm(p.transpose(1, 2), p) - torch.eye(p.shape[2], dtype=torch.float64,
                                                     device=p.device)
    return g.abs().max().item()


MIXED = [(3, 256, 128, 32),      # r <= 256, fused B Q
         (2, 200, 136, 128),     # m = 200 split 100 / 100 (or 67 / 67 / 66): r above the rows
         (2, 600, 560, 272)]     # r > 256: the recursive factorisation


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_row_shards_match_the_oracle(precision, world):
    wl = W.custom(f"rowshard_{precision}", MIXED, precision=precision, steps=3)
    em = Emulated(wl, world, precision)
    for _ in range(wl.steps):
        em.step()
    torch.cuda.synchronize()
    assert em.kinds[0] == ["gram", "gram2", "r"], em.kinds
    _same_on_every_rank(em)
    assert not np.any(em.st[0].cpu().numpy() & (1 | 4 | 8))
    for i, b in enumerate(wl.buckets):
        X, M, Q, P = em.whole(i)
        assert _orth_err(P) <= ORTH_TOL
        for s in range(b.count):
            X0, Xr, Mr, Qr, _, Rr = oracle_slot(wl, i, s, wl.steps, "cpu")
            q = Q[s].double().cpu().numpy()
            rel = [oracle.rel_fro(X[s].double().cpu().numpy(), Xr),
                   oracle.rel_fro(M[s].double().cpu().numpy(), Mr),
                   # Q as in the whole-matrix parity tests: plain in fp32, its columns
                   # weighted by the norms of R's columns with bf16 operands
                   oracle.rel_fro(q, Qr) if precision == "fp32" else rel_q_weighted(q, Qr, Rr)]
            print(precision, world, i, s, ["%.2e" % v for v in rel])
            assert max(rel) <= TOL[precision], (i, s, rel)


def test_rejected_matrix_takes_the_gathered_householder_qr():
    """Slot 0 gets a gradient of rank 16 < r = 64 (M = 0): its Gram is singular, every
    rank flags it, the bucket's P0 is gathered and Householder QR of the whole P0 gives
    its P.  P is not unique there, so the check is the invariants (P^T P = I, M' = mu G
    since span(P) holds col(G)); slot 1 (Gaussian) must match the oracle."""
    wl = W.custom("rowshard_gather", [(2, 256, 192, 64)], precision="fp32", steps=1)
    em = Emulated(wl, 2, "fp32")
    m, n, r = 256, 192, 64
    g = torch.Generator().manual_seed(21)
    U = torch.linalg.qr(torch.randn(m, 16, generator=g, dtype=torch.float64))[0]
    V = torch.linalg.qr(torch.randn(n, 16, generator=g, dtype=torch.float64))[0]
    G = torch.stack([U @ V.T, torch.randn(m, n, generator=g, dtype=torch.float64)]).float().cuda()
    X0 = torch.cat(em.X[0], dim=1).clone()
    Q0 = em.Q[0][0].clone()
    em.step([G])
    torch.cuda.synchronize()
    assert em.kinds[0] == ["gram", "gram2", "gather", "r"], em.kinds
    _same_on_every_rank(em)
    st = em.st[0].cpu().numpy()
    assert st[0] & 1 and not st[1] & 1 and not np.any(st & (4 | 8)), st
    X, M, Q, P = em.whole(0)
    assert _orth_err(P) <= ORTH_TOL
    assert (M[0] - wl.mu * G[0]).norm() / G[0].norm() <= 1e-5
    Xr, Mr, Qr, _, _ = oracle.dion_step(X0[1].cpu().numpy(), np.zeros((m, n)),
                                        G[1].cpu().numpy(), Q0[1].cpu().numpy(), wl.mu, wl.lr)
    for a, ref in ((X[1], Xr), (M[1], Mr), (Q[1], Qr)):
        assert oracle.rel_fro(a.double().cpu().numpy(), ref) <= TOL["fp32"]


def test_householder_mode_gathers_every_bucket():
    wl = W.custom("rowshard_hh", [(2, 256, 128, 32), (1, 300, 64, 48)], precision="fp32",
                  steps=2)
    em = Emulated(wl, 2, "fp32", orth_mode="householder")
    for _ in range(wl.steps):
        em.step()
    torch.cuda.synchronize()
    assert em.kinds[0] == ["gram", "gram2", "gather", "gather", "r"], em.kinds
    _same_on_every_rank(em)
    assert np.all(em.st[0].cpu().numpy() & 1)
    for i, b in enumerate(wl.buckets):
        X, M, Q, P = em.whole(i)
        for s in range(b.count):
            _, Xr, Mr, Qr, _, _ = oracle_slot(wl, i, s, wl.steps, "cpu")
            for a, ref in ((X, Xr), (M, Mr), (Q, Qr)):
                assert oracle.rel_fro(a[s].double().cpu().numpy(), ref) <= TOL["fp32"]


def test_one_rank_is_the_whole_step():
    """World size 1: the sharded step runs the same kernels on the same rows as
    dion_step_batched, except that the column norms' partial sums come from R itself
    rather than from B^T P's epilogue.  After one step M (which does not depend on the
    new Q) is bit for bit the same; X and Q differ by the rounding of that sum's order,
    which the second step carries on: they must agree within the parity tolerance."""
    from parity_harness import GpuRun
    wl = W.custom("rowshard_one", [(3, 256, 128, 32), (2, 600, 560, 272)], precision="fp32",
                  steps=2)
    em = Emulated(wl, 1, "fp32")
    ref = GpuRun(wl, gen_device="cpu")
    for t in range(2):
        em.step()
        ref.step(1)
        torch.cuda.synchronize()
        for i in range(2):
            X, M, Q, _ = em.whole(i)
            if t == 0:
                assert torch.equal(M, ref.M[i])
            for a, b in ((X - ref.X0[i], ref.X[i] - ref.X0[i]), (M, ref.M[i]), (Q, ref.Q[i])):
                assert ((a - b).norm() / b.norm()).item() <= TOL["fp32"]
