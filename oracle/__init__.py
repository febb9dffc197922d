"""Float64 CPU oracle for the MonarchAttention forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only the tests, the smoke check and the CPU-baseline leg of the benchmark do.
It shares no code with the CUDA path; the two meet only through the seeded
input generators.
"""
from .monarch_ref import (  # noqa: F401
    LFactor,
    RFactor,
    dense_logits,
    group_valid,
    groups,
    materialise,
    monarch_attention,
    monarch_attention_backward,
    objective,
    objective_dense,
    output,
    r_update,
    l_update,
    token_mask,
)
