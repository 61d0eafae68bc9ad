"""fp64 CPU oracles of the Dion step (whole and row-sharded), of CurvaDion's
momentum-change statistic and of the vector-parameter step (test infrastructure;
never on the product path)."""
from .curvadion_oracle import needs_sync, rmmc
from .dion_oracle import (colnorm, default_scale, dion_step, dion_step_stacked, form_b,
                          orth, orthogonality_error, rel_fro, run_steps)
from .sharded_oracle import dion_step_row_shard, row_range
from .vector_oracle import adamw_step, lion_direction, lion_step, vector_step

__all__ = ["colnorm", "default_scale", "dion_step", "dion_step_stacked", "form_b", "orth",
           "orthogonality_error", "rel_fro", "run_steps", "dion_step_row_shard", "row_range",
           "rmmc", "needs_sync", "adamw_step", "lion_direction", "lion_step", "vector_step"]
