"""Why the end-to-end updated-parameter bar is 5e-3 and not 1e-3, and which
rounding point holds how much of the floor.

The CPU emulation in precision_emulation.py reproduces this path's bf16
rounding points (fp32 arithmetic, the same bf16 weights the oracle uses) for
one step of the tiny workload; the first AdamW step is applied to its
gradients and to the oracle's, and the relative L2 of the two updated masters
is the floor. The first Adam step is ~lr * sign(g): elements whose gradient is
below the arithmetic error flip sign and move by 2 lr, so the floor is
~0.1 sqrt(flip fraction).

Findings pinned here (seeded, deterministic):
- the path as built sits between 1e-3 and the 5e-3 the GPU tests use;
- every rounding point ON ITS OWN (stored activations, stored gradients, the
  attention kernels' P and dS) already puts the floor above 1e-3, so 1e-3
  needs higher precision at all of them at once;
- exact weight-gradient GEMM operands alone (a hi+lo split of X and dY, the
  remedy first proposed for this) move the floor by under 5 %;
- with every rounding point exact the emulation meets the oracle to ~1e-5.
"""
import numpy as np
import pytest

import oracle
import synth
from precision_emulation import Prec, emulated_grads, first_step_floor

HYP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


@pytest.fixture(scope="module")
def tiny():
    shape = synth.WORKLOADS["tiny"]
    c = oracle.OracleConfig(**shape)
    W32 = synth.init_weights(shape, 0)
    Wb = {k: oracle.bf16_round(v) for k, v in W32.items()}
    tok, lab = synth.tokens_labels(c.b, c.s, c.V, 0)
    _, G = oracle.train_step_grads(Wb, tok, lab, c)
    return c, W32, Wb, tok, lab, G


def _floor(tiny, p):
    c, W32, Wb, tok, lab, G = tiny
    return first_step_floor(W32, G, emulated_grads(Wb, tok, lab, c, p), HYP, oracle.adamw_update)


def test_bf16_input_floor_of_first_adam_step(tiny):
    floor, flips, den = _floor(tiny, Prec())
    assert 1e-3 < floor < 5e-3, floor
    # the sign-flip model explains it: each flipped element moves by 2 lr
    c, W32, *_ = tiny
    n = sum(w.size for w in W32.values())
    assert abs(floor - 2 * HYP["lr"] * np.sqrt(flips * n / den)) < 0.2 * floor


def test_each_rounding_point_alone_is_above_the_bar(tiny):
    alone = {
        "stored activations": Prec(fwd_store=True, bwd_store=False, attn_inner=False),
        "stored gradients": Prec(fwd_store=False, bwd_store=True, attn_inner=False),
        "attention P and dS": Prec(fwd_store=False, bwd_store=False, attn_inner=True),
    }
    floors = {k: _floor(tiny, p)[0] for k, p in alone.items()}
    assert all(f > 1e-3 for f in floors.values()), floors


def test_exact_weight_gradient_operands_do_not_help(tiny):
    base = _floor(tiny, Prec())[0]
    dw = _floor(tiny, Prec(dw_exact=True))[0]
    assert abs(dw - base) < 0.05 * base, (base, dw)
    assert dw > 1e-3


def test_all_exact_meets_the_oracle(tiny):
    floor, flips, _ = _floor(tiny, Prec(False, False, False, True))
    assert floor < 1e-4 and flips < 1e-5, (floor, flips)
