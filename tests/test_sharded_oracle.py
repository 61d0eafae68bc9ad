"""The row-sharded Dion step against the whole-matrix oracle, over gloo (CPU).

Ranks hold row blocks of X, M and G and a replicated Q; the Gram of P0 (r x r) and
R = B^T P (n x r) are summed over ranks by an all-reduce (torch.distributed over gloo,
fp64).  Put back together, the ranks' rows must equal the unsharded oracle's step to
fp64 rounding, over several steps, for an even and an uneven split, at full rank, and
when the Gram is singular (the gathered-QR branch), where only the invariants of the
step are unique.
"""
import os

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle

SEED = 20260305


def _case(name):
    rng = np.random.default_rng(SEED + {"general": 1, "uneven_full_rank": 2,
                                        "rank_deficient": 3}[name])
    if name == "general":
        m, n, r, steps = 50, 24, 6, 3
        G = [rng.standard_normal((m, n)) for _ in range(steps)]
    elif name == "uneven_full_rank":
        m, n, r, steps = 37, 16, 16, 3
        G = [rng.standard_normal((m, n)) for _ in range(steps)]
    else:
        m, n, r, steps = 40, 12, 5, 1
        G = [rng.standard_normal((m, 2)) @ rng.standard_normal((2, n))]
    X = rng.standard_normal((m, n))
    Q = rng.standard_normal((n, r))
    Q /= np.linalg.norm(Q, axis=0, keepdims=True)
    return m, n, r, X, np.zeros((m, n)), Q, G


def _worker(rank, world, port, name, out):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m, n, r, X, M, Q, G = _case(name)
        row0, mk = oracle.row_range(m, world, rank)
        sl = slice(row0, row0 + mk)

        def allreduce(a):
            t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
            dist.all_reduce(t)
            return t.numpy()

        Xk, Mk = X[sl].copy(), M[sl].copy()
        gathered = []
        for g in G:
            Xk, Mk, Q, Pk, R, gth = oracle.dion_step_row_shard(
                Xk, Mk, g[sl], Q, 0.9, 0.05, allreduce, row0=row0, m_full=m)
            gathered.append(gth)
        out.put((rank, row0, Xk, Mk, Q, Pk, gathered))
    finally:
        dist.destroy_process_group()


def _run(name, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() * 7 + world) % 2000
    procs = [ctx.Process(target=_worker, args=(k, world, port, name, q)) for k in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X = np.concatenate([t[2] for t in res])
    M = np.concatenate([t[3] for t in res])
    P = np.concatenate([t[5] for t in res])
    return X, M, [t[4] for t in res], P, [t[6] for t in res]


@pytest.mark.parametrize("name,world", [("general", 2), ("uneven_full_rank", 2),
                                        ("general", 3)])
def test_row_shards_equal_the_whole_step(name, world):
    X, M, Qs, P, gathered = _run(name, world)
    m, n, r, X0, M0, Q0, G = _case(name)
    Xr, Mr, Qr = X0, M0, Q0
    for g in G:
        Xr, Mr, Qr, Pr, _ = oracle.dion_step(Xr, Mr, g, Qr, 0.9, 0.05)
    for Q in Qs:                                  # every rank holds the same Q
        assert oracle.rel_fro(Q, Qr) < 1e-12
    assert oracle.rel_fro(X, Xr) < 1e-12 and oracle.rel_fro(M, Mr) < 1e-12
    assert oracle.rel_fro(X - X0, Xr - X0) < 1e-11
    assert oracle.rel_fro(P, Pr) < 1e-12
    assert not any(any(g) for g in gathered)


def test_singular_gram_takes_the_gathered_qr():
    """G of rank 2 < r = 5 and M = 0: the Gram of P0 is singular, every rank takes the
    gathered QR, and the step keeps its invariants: P^T P = I, span(P) holds col(B), so
    M' = mu G; ||X' - X||_F = lr s sqrt(r)."""
    X, M, Qs, P, gathered = _run("rank_deficient", 2)
    m, n, r, X0, M0, Q0, G = _case("rank_deficient")
    assert all(g == [True] for g in gathered)
    assert oracle.orthogonality_error(P) < 1e-12
    assert np.abs(M - 0.9 * G[0]).max() < 1e-12
    assert abs(np.linalg.norm(X - X0) - 0.05 * np.sqrt(m / n) * np.sqrt(r)) < 1e-12


def test_one_rank_is_the_whole_step():
    """World size 1 (the all-reduce is the identity) is the unsharded step."""
    m, n, r, X0, M0, Q0, G = _case("general")
    Xr, Mr, Qr, Pr, Rr = oracle.dion_step(X0, M0, G[0], Q0, 0.9, 0.05)
    X, M, Q, P, R, gth = oracle.dion_step_row_shard(X0, M0, G[0], Q0, 0.9, 0.05, lambda a: a,
                                                    row0=0, m_full=m)
    assert not gth
    for a, b in ((X, Xr), (M, Mr), (Q, Qr), (P, Pr), (R, Rr)):
        assert oracle.rel_fro(a, b) < 1e-13


def test_row_ranges_cover_the_rows_once():
    for m, world in ((10, 3), (7, 7), (4096, 8), (11008, 3)):
        rows = [oracle.row_range(m, world, k) for k in range(world)]
        assert rows[0][0] == 0
        for (a0, ak), (b0, _) in zip(rows, rows[1:]):
            assert a0 + ak == b0
        assert rows[-1][0] + rows[-1][1] == m
        assert max(k for _, k in rows) - min(k for _, k in rows) <= 1
