"""fp64 CPU oracle of one Dion optimizer step -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the package's smoke check and the CPU-baseline leg of
the benchmark may import this module.  The CUDA library never calls it, and
it shares no code with the CUDA path: the two meet only through the seeded
inputs of ``workloads``.

What one step computes, for a weight X (m x n), its error-feedback momentum
M (m x n), its gradient G (m x n) and the right factor Q (n x r) kept from
the previous step:

  1. B  = M + G
  2. P0 = B Q                          one amortised power-iteration step
  3. P  = orth(P0)                     orthonormal basis of span(P0)
  4. R  = B^T P                        second half of the power step
  5. M' = B - (1 - mu) P R^T           error feedback: keep what rank r missed
  6. Q' = colnorm(R)                   unit columns, the next warm start
  7. X' = X - lr * s * P Q'^T,         s = sqrt(m / n)

Sources (rivista.ai, "Dion e la fine del monopolio di Adam negli optimizer
AI distribuiti" -- the article on "Dion: Distributed Orthonormalized
Updates"):
  * paragraph 2: only the leading r singular directions are orthonormalised,
    not the whole matrix (steps 2-4, 7);
  * paragraph 3: error feedback keeps the difference between the full matrix
    and its low-rank part and feeds it back into later updates (step 5);
  * paragraph 5: Newton-Schulz is replaced by an amortised power iteration
    with QR and Cholesky decompositions (steps 2-4); only 2-D parameters go
    through this step.
The article gives no formulas; the step above is the plainest reading of
its prose and is the one the CUDA library implements.

Step 3 is written as its plain definition: the thin QR factorisation
P0 = P Rfac whose triangular factor has a non-negative diagonal.  For a P0
of full column rank that factor is unique, and it is exactly what
Cholesky-QR (Rfac = chol(P0^T P0)^T, P = P0 Rfac^-1) reaches in exact
arithmetic, so the oracle is agnostic to how the GPU orthonormalises.  It is
computed with LAPACK's Householder QR (numpy.linalg.qr) and the columns'
signs are then fixed so that diag(Rfac) >= 0 (sign(0) taken as +1).

Step 6 divides each column of R by its 2-norm.  A column whose norm is
exactly zero has no direction; it is set to zero (so a zero gradient gives a
zero update), which the pages leave open.

Everything is fp64 NumPy; inputs given in fp32 are widened first.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):            # a torch tensor: take a CPU copy
        a = a.detach().cpu().numpy()
    return np.asarray(a, dtype=np.float64)


def form_b(M, G):
    """Step 1: B = M + G (the momentum buffer plus this step's gradient)."""
    return _f64(M) + _f64(G)


def orth(P0):
    """Step 3: the orthonormal factor P of the thin QR P0 = P Rfac, diag(Rfac) >= 0.

    Returns (P, Rfac).  Paragraph 5 of the Dion article names QR and
    Cholesky decompositions as the orthonormalisation.
    """
    P0 = _f64(P0)
    q, rf = np.linalg.qr(P0, mode="reduced")
    d = np.sign(np.diag(rf))
    d[d == 0] = 1.0
    return q * d[None, :], rf * d[:, None]


def colnorm(R):
    """Step 6: divide every column of R by its Euclidean norm over the n rows.

    A column of norm exactly zero becomes a zero column.
    """
    R = _f64(R)
    norms = np.sqrt(np.sum(R * R, axis=0))
    out = np.zeros_like(R)
    nz = norms > 0
    out[:, nz] = R[:, nz] / norms[nz]
    return out


def default_scale(m: int, n: int) -> float:
    """s = sqrt(m / n): the shape factor applied to the update P Q^T."""
    return float(np.sqrt(m / n))


def dion_step(X, M, G, Q, mu: float, lr: float, scale: float | None = None):
    """One Dion step on one matrix; returns (X', M', Q', P, R), all fp64.

    X, M, G: m x n.  Q: n x r (previous right factor).  ``scale`` defaults to
    sqrt(m / n).
    """
    X, M, G, Q = _f64(X), _f64(M), _f64(G), _f64(Q)
    m, n = X.shape
    if scale is None:
        scale = default_scale(m, n)
    B = form_b(M, G)                                   # step 1
    P0 = B @ Q                                         # step 2
    P, _ = orth(P0)                                    # step 3
    R = B.T @ P                                        # step 4
    M_new = B - (1.0 - mu) * (P @ R.T)                 # step 5
    Q_new = colnorm(R)                                 # step 6
    X_new = X - lr * scale * (P @ Q_new.T)             # step 7
    return X_new, M_new, Q_new, P, R


def dion_step_stacked(X, M, G, Q, mu: float, lr: float, scale: float | None = None):
    """The same step on a stack [k, m, n] of independent matrices (a loop, nothing fused)."""
    outs = [dion_step(X[i], M[i], G[i], Q[i], mu, lr, scale) for i in range(len(X))]
    return tuple(np.stack([o[j] for o in outs]) for j in range(5))


def run_steps(X, M, Q, grads, mu: float, lr: float, scale: float | None = None,
              reset_momentum: bool = False):
    """Run len(grads) steps on one matrix; ``grads`` is a sequence of G's.

    With ``reset_momentum`` the momentum is zeroed before every step (the
    fixed-B experiments pass M = 0 and G = B each step).
    Returns the final (X, M, Q, P, R).
    """
    X, M, Q = _f64(X), _f64(M), _f64(Q)
    P = R = None
    for G in grads:
        if reset_momentum:
            M = np.zeros_like(M)
        X, M, Q, P, R = dion_step(X, M, G, Q, mu, lr, scale)
    return X, M, Q, P, R


def rel_fro(a, ref) -> float:
    """||a - ref||_F / ||ref||_F in fp64 (0 when both are zero)."""
    a, ref = _f64(a), _f64(ref)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(a - ref)
    if den == 0:
        return float(num)
    return float(num / den)


def orthogonality_error(P) -> float:
    """max |P^T P - I| over all entries."""
    P = _f64(P)
    return float(np.max(np.abs(P.T @ P - np.eye(P.shape[1]))))
