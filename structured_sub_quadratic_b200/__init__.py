"""MonarchAttention forward pass for B200 (sm_100a): C-ABI library + binding.

``api`` binds ``libmonarch_attn.so`` (built by ``_build``); ``inputs`` holds
the seeded synthetic workloads.  Importing the package does not load the
library; the first call through ``api`` does, and raises if it is missing.
"""

__all__ = ["api", "inputs"]
