"""AdamW with decoupled weight decay, fp64, for the host-side optimizer step.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The MegaTrain pages keep the fp32 master weights and both Adam moments in host
memory and update them on the CPU (intelligentliving.co, "Checkpointing, Manual
Gradients, and CPU-Side Optimizer Steps"; MegaTrain abstract). The update is
Adam (Kingma & Ba, "Adam: A Method for Stochastic Optimization", Algorithm 1)
with the weight decay decoupled from the gradient, applied in this order:
  p <- p (1 - lr wd)
  m <- b1 m + (1 - b1) g
  v <- b2 v + (1 - b2) g^2
  p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
with t counting steps from 1 and the decay applied to every tensor.
"""
from __future__ import annotations

import numpy as np


def adamw_update(p, g, m, v, t: int, lr: float, beta1: float, beta2: float,
                 eps: float, wd: float):
    """Returns the new (p, m, v) as float64 arrays; inputs are not modified."""
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    p = p * (1.0 - lr * wd)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** t)
    vhat = v / (1.0 - beta2 ** t)
    p = p - lr * mhat / (np.sqrt(vhat) + eps)
    return p, m, v
