"""CPU fp64 oracle of the MS-GLA layer forward pass (test infrastructure only)."""
from .msgla_oracle import (pool, logsigmoid, branch_projections, gla_recurrent, hold_index,
                           hold, fusion_weights, head_rmsnorm, layer_forward, state_updates,
                           decode_init, decode_step)
