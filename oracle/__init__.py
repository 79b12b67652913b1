"""fp64 CPU oracle for one streamed-layer training step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls, links or
executes this package: only `tests/`, `__graft_entry__.smoke()` and the
`cpu_baseline` / `--impl reference` legs of `bench.py` use it.

It is a plain, slow, obviously correct restatement of what one training step of
MegaTrain's memory-centric training computes ("MegaTrain: Full Precision
Training of 100B+ Parameter Large Language Models on a Single GPU", abstract:
stream parameters in per layer, compute gradients out, update with Adam on the
host), for a Llama-style pre-norm decoder. Streaming, double buffering and
checkpointed recompute do not change the mathematics (intelligentliving.co,
"Checkpointing, Manual Gradients, and CPU-Side Optimizer Steps": recompute only
trades compute for memory), so the oracle is the plain definition: a full,
unchunked forward that keeps every activation, a hand-written backward, and
AdamW with decoupled weight decay (Kingma & Ba, "Adam: A Method for Stochastic
Optimization", cited by the MegaTrain paper).

Every function here is pinned by tests in `tests/test_oracle_*.py` against
finite differences, closed forms, invariants and library routines that do not
share its code. It shares no code with the CUDA path.
"""
from .model import (  # noqa: F401
    OracleConfig,
    arena_layout,
    arena_floats,
    unpack_arena,
    pack_arena,
    bf16_round,
    rmsnorm_fwd,
    rmsnorm_bwd,
    rope_tables,
    rope_fwd,
    rope_bwd,
    attention_fwd,
    attention_bwd,
    attention_lse,
    silu,
    swiglu_fwd,
    swiglu_bwd,
    layer_fwd,
    layer_bwd,
    softmax_ce,
    head_ce_fwd_bwd,
    train_step_grads,
)
from .adamw import adamw_update  # noqa: F401
