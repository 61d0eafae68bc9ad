"""fp64 CPU oracle of the Dion step (test infrastructure; never on the product path)."""
from .dion_oracle import (colnorm, default_scale, dion_step, dion_step_stacked, form_b,
                          orth, orthogonality_error, rel_fro, run_steps)

__all__ = ["colnorm", "default_scale", "dion_step", "dion_step_stacked", "form_b", "orth",
           "orthogonality_error", "rel_fro", "run_steps"]
