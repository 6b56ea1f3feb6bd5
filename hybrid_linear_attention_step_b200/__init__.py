"""Decode-time Gated DeltaNet state update with slot indirection, for B200 (sm_100a).

The compute lives in hand-written CUDA behind a C-ABI shared library
(``libgdn_b200.so``, declared in ``include/gdn_step.h``).  ``gdn`` is the thin
ctypes binding with the same entry-point names; ``workloads`` holds the seeded
synthetic inputs.  Import ``hybrid_linear_attention_step_b200.gdn`` to load the
library: it raises if the compiled extension is missing.
"""

__all__ = ["gdn", "workloads", "build"]
