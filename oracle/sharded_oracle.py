"""fp64 CPU oracle of the row-sharded Dion step -- TEST INFRASTRUCTURE ONLY.

Only the test suite may import this module.  It shares no code with the CUDA
library.

The Dion article (rivista.ai, "Dion e la fine del monopolio di Adam negli
optimizer AI distribuiti") says the method cuts the data synchronised between
nodes (paragraph 3) and works under data, tensor and fully sharded data
parallelism, FSDP2 included (paragraph 5), without saying how a sharded step is
computed.  The reading taken here is the plainest one the step allows: the rows
of every matrix are split among the ranks (rank k holds rows [row0, row0 + m_k)
of X, M and G), the right factor Q (n x r) is replicated, and the step needs only
sums over ranks of r-sized quantities:

  1. B_k  = M_k + G_k                              local rows
  2. P0_k = B_k Q                                  local rows
  3. W    = sum_k P0_k^T P0_k                      all-reduce of r x r: the Gram of P0
     L    = chol(W);  P_k = P0_k L^-T              Cholesky-QR, every rank the same L
     (when W is not numerically positive definite, the rows of P0 are gathered --
      an all-reduce of the zero-padded m x r P0 -- and P is the thin-QR factor of
      the whole P0, of which each rank keeps its rows)
  4. R    = sum_k B_k^T P_k                        all-reduce of n x r
  5. M_k' = B_k - (1 - mu) P_k R^T                 local rows
  6. Q'   = colnorm(R)                             every rank the same Q'
  7. X_k' = X_k - lr s P_k Q'^T                    local rows, s = sqrt(m / n) of the
                                                   whole matrix
Step 3 gives exactly the factor of the unsharded step: stacking the P_k gives
P0 L^-T, and the Gram of the stacked P0 is W, so P is the Q factor with a
positive triangular diagonal -- what ``dion_oracle.orth`` computes.

``allreduce(a)`` returns the elementwise sum of ``a`` over all ranks (every rank
calls it in the same order with arrays of the same shape).
"""
from __future__ import annotations

import numpy as np

from .dion_oracle import _f64, colnorm, default_scale, orth

#: Cholesky-QR in fp64 keeps P orthonormal to about cond(P0)^2 * 1e-16; beyond a
#: diagonal ratio of 1e6 (cond(P0) of about 1e6) the gathered QR is used instead.
CHOL_DIAG_RATIO = 1e6


def row_range(m: int, world: int, rank: int):
    """Rows [row0, row0 + m_k) of rank ``rank`` when m rows are split as evenly as
    possible, the first m % world ranks taking one row more."""
    base, extra = divmod(m, world)
    row0 = rank * base + min(rank, extra)
    return row0, base + (1 if rank < extra else 0)


def _cholesky_or_none(W):
    try:
        L = np.linalg.cholesky(W)
    except np.linalg.LinAlgError:
        return None
    d = np.diag(L)
    if not np.all(np.isfinite(d)) or d.min() <= 0 or d.max() / d.min() > CHOL_DIAG_RATIO:
        return None
    return L


def dion_step_row_shard(X_k, M_k, G_k, Q, mu: float, lr: float, allreduce, *, row0: int,
                        m_full: int, scale: float | None = None):
    """One Dion step on this rank's rows of one matrix.

    X_k, M_k, G_k: m_k x n (rows row0 .. row0 + m_k of the whole m_full x n matrix).
    Q: n x r, the same on every rank.  Returns (X_k', M_k', Q', P_k, R, gathered), where
    ``gathered`` tells whether step 3 took the gathered QR.
    """
    X_k, M_k, G_k, Q = _f64(X_k), _f64(M_k), _f64(G_k), _f64(Q)
    m_k, n = X_k.shape
    r = Q.shape[1]
    if scale is None:
        scale = default_scale(m_full, n)
    B_k = M_k + G_k                                        # step 1
    P0_k = B_k @ Q                                         # step 2
    W = allreduce(P0_k.T @ P0_k)                           # step 3: Gram of P0
    L = _cholesky_or_none(W)
    gathered = L is None
    if gathered:
        full = np.zeros((m_full, r))
        full[row0:row0 + m_k] = P0_k
        P_full, _ = orth(allreduce(full))
        P_k = P_full[row0:row0 + m_k]
    else:
        P_k = np.linalg.solve(L, P0_k.T).T                 # P0_k L^-T
    R = allreduce(B_k.T @ P_k)                             # step 4
    M_new = B_k - (1.0 - mu) * (P_k @ R.T)                 # step 5
    Q_new = colnorm(R)                                     # step 6
    X_new = X_k - lr * scale * (P_k @ Q_new.T)             # step 7
    return X_new, M_new, Q_new, P_k, R, gathered
