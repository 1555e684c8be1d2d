"""CPU float64 oracle of the DeepSeek-V4.1-Flash routed-expert FFN layer.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline leg may import this package. The product path (the CUDA library and
its Python binding) never does, and there is no CPU fallback through it.

Parity status: every function here is pinned by tests/test_oracle_*.py against
values fixed by the mathematics or the pages (hand-worked example, closed forms,
brute force, library decoders); none is "parity unpinned".
"""
from . import mx
from .moe import (ExpertSource, MoEResult, Route, clamped_swiglu, dense_reference,
                  expert_forward, hash_route, moe_forward, moe_forward_hashed, moe_forward_partial,
                  permutation_reference, route, silu, softplus, sqrtsoftplus)

__all__ = ["mx", "ExpertSource", "MoEResult", "Route", "clamped_swiglu",
           "dense_reference", "expert_forward", "hash_route", "moe_forward", "moe_forward_hashed", "moe_forward_partial",
           "permutation_reference",
           "route", "silu", "softplus", "sqrtsoftplus"]
