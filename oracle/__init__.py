"""CPU oracle for RetNet multi-scale retention (test infrastructure only).

Plain, slow, float64 numpy restatement of what the retention hot path
computes.  Only the tests, the smoke check and the benchmark's CPU-baseline
leg may import it; the CUDA library never does, and the two share no code.
"""
from .retention import (  # noqa: F401
    decay_gammas,
    rotation_thetas,
    xpos_rotate,
    decay_mask,
    retention_parallel,
    retention_recurrent,
    retention_chunkwise,
    retention_step,
    groupnorm_swish,
    retention_prefill,
    retention_parallel_backward,
    xpos_rotate_backward,
    retention_prefill_backward,
    linear,
    msr_layer,
)
