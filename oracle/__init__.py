"""CPU oracle for the streamed decoder-layer training step.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import or execute anything in this package.
The product path (the C-ABI library and its Python binding) never routes
through it; there is no CPU fallback.

The oracle is the plain definition of the computation: the full-activation
forward and backward of a stack of Qwen2.5-style decoder layers in float64,
with no streaming, no recomputation, no tiling and no fusion. Streaming,
double buffering, segmented checkpointing and chunked MLP execution (MegaTrain,
abstract and the blog summary's design points 2-4) change where and when the
work runs, not what it computes, so the oracle does not model them.

Every function is pinned by tests/test_oracle_pins.py against closed forms,
invariants, brute-force loops or finite differences; see each docstring.
"""
from .layer import (  # noqa: F401
    OracleCfg,
    attention_bwd,
    attention_fwd,
    layer_bwd,
    layer_fwd,
    rmsnorm_bwd,
    rmsnorm_fwd,
    rope_apply,
    rope_tables,
    stack_fwd_bwd,
    swiglu_bwd,
    swiglu_fwd,
)
from .optimizer import adamw_step  # noqa: F401
