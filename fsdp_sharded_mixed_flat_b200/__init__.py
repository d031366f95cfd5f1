"""B200 (sm_100a) library for the per-rank arithmetic of one ZeRO-3 / FSDP step.

The product is libzero3.so (C ABI in include/zero3.h): a flat-parameter
planner with the per-stage memory ledger, a fused reduce-scatter reduction +
AdamW + bf16-cast kernel, and an all-gather + unflatten kernel.  The Python
binding lives in `fsdp_sharded_mixed_flat_b200.zero3` and is imported on
demand, so that building the library does not need it loaded:

    from fsdp_sharded_mixed_flat_b200 import zero3
"""

__all__ = ["zero3", "build"]
