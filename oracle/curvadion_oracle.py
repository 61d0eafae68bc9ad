"""fp64 CPU oracle of the momentum-change statistic of CurvaDion -- TEST
INFRASTRUCTURE ONLY.

Only the test suite may import this module.  It shares no code with the CUDA
library.

The page on "CurvaDion: Curvature-Adaptive Distributed Orthonormalization"
(mlsanity.com, Abstract) says that plain Dion synchronises at every step, that
the need to synchronise changes over training, and that CurvaDion detects the
high-curvature regions that need it with the Relative Maximum Momentum Change
(RMMC), built from the momentum the optimizer already keeps, at O(d) operations
per layer.  The page does not write the statistic down.  The reading taken here
is the plainest one its name and cost allow, per weight matrix (layer), with M
the error-feedback momentum before the step and M' after it:

    RMMC = max_ij |M'_ij - M_ij| / max_ij |M_ij|

the largest entry of the momentum's change relative to the largest entry of the
momentum: one pass over the d entries, no extra state.  A zero momentum has no
scale: the statistic is +inf when the momentum changed and 0 when it did not.
The gate: a matrix needs synchronisation when RMMC > tau, for a threshold tau the
caller chooses (the page gives none).
"""
from __future__ import annotations

import numpy as np

from .dion_oracle import _f64


def rmmc(M_prev, M_new) -> float:
    """max |M_new - M_prev| / max |M_prev| of one matrix (inf / 0 for a zero M_prev)."""
    M_prev, M_new = _f64(M_prev), _f64(M_new)
    num = float(np.max(np.abs(M_new - M_prev))) if M_prev.size else 0.0
    den = float(np.max(np.abs(M_prev))) if M_prev.size else 0.0
    if den == 0.0:
        return float("inf") if num > 0.0 else 0.0
    return num / den


def needs_sync(rmmc_value: float, tau: float) -> bool:
    """CurvaDion's gate: synchronise where the momentum changes faster than tau."""
    return rmmc_value > tau
