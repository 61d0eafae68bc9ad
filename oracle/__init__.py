"""fp64 CPU oracles of the Dion step and of the vector-parameter step (test
infrastructure; never on the product path)."""
from .dion_oracle import (colnorm, default_scale, dion_step, dion_step_stacked, form_b,
                          orth, orthogonality_error, rel_fro, run_steps)
from .vector_oracle import adamw_step, lion_direction, lion_step, vector_step

__all__ = ["colnorm", "default_scale", "dion_step", "dion_step_stacked", "form_b", "orth",
           "orthogonality_error", "rel_fro", "run_steps", "adamw_step", "lion_direction",
           "lion_step", "vector_step"]
