"""B200-native (sm_100a) Gated DeltaNet-2 recurrence: chunked prefill and decode.

The compute lives in ``libgdn2.so`` (CUDA, C ABI declared in ``include/gdn2.h``).
:mod:`delta_rule_linear_gdn_b200.gdn2` is the thin ctypes binding; importing
this package does not load the library, so the seeded input generator
(:mod:`delta_rule_linear_gdn_b200.inputs`) can be used without a GPU.
"""

__all__ = ["gdn2", "inputs"]
