"""Why the end-to-end updated-parameter bar is 5e-3 and not 1e-3.

Emulates this path's rounding points on the CPU (fp32 arithmetic, bf16 at
every GEMM input, the same bf16 weights the oracle uses) for one step of the
tiny workload, applies the first AdamW step to both gradient sets, and measures
the relative L2 of the updated master against the oracle. The first Adam step
is ~lr * sign(g): elements whose gradient is below the bf16 error flip sign, so
the floor is ~0.1 * sqrt(flip fraction). The measured floor must sit between
1e-3 (the bar bf16 inputs cannot reach) and the 5e-3 the GPU tests use."""
import numpy as np
import torch
import torch.nn.functional as F

import oracle
import synth
from oracle.model import (ATTN_NORM, WQ, WK, WV, WO, MLP_NORM, WGATE, WUP, WDOWN, EMBED, FINAL_NORM, LM_HEAD)


class _RoundBf16(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x):
        return x.to(torch.bfloat16).to(torch.float32)

    @staticmethod
    def backward(ctx, g):
        return g.to(torch.bfloat16).to(torch.float32)


def _emulated_grads(Wb, tok, lab, c):
    r = _RoundBf16.apply
    Wt = {k: torch.tensor(v, dtype=torch.float32, requires_grad=True) for k, v in Wb.items()}
    hd, (b, s) = c.hd, tok.shape
    ang = torch.arange(s, dtype=torch.float64)[:, None] * (c.rope_base ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd))[None]
    cs, sn = torch.cos(ang).float()[None, :, None], torch.sin(ang).float()[None, :, None]

    def rope(x):
        x1, x2 = x[..., :hd // 2], x[..., hd // 2:]
        return torch.cat([x1 * cs - x2 * sn, x2 * cs + x1 * sn], -1)

    x = F.embedding(torch.tensor(tok).long(), Wt[(-1, EMBED)])
    for l in range(c.L):
        w = lambda t: Wt[(l, t)]  # noqa: E731
        u = r(F.rms_norm(x, (c.d,), w(ATTN_NORM), c.norm_eps))
        q = r(rope((u @ w(WQ).T).view(b, s, c.H, hd))).transpose(1, 2)
        k = r(rope((u @ w(WK).T).view(b, s, c.Hkv, hd))).transpose(1, 2)
        v = r((u @ w(WV).T).view(b, s, c.Hkv, hd)).transpose(1, 2)
        o = r(F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True))
        h = x + o.transpose(1, 2).reshape(b, s, -1) @ w(WO).T
        m = r(F.rms_norm(h, (c.d,), w(MLP_NORM), c.norm_eps))
        x = h + r(F.silu(r(m @ w(WGATE).T)) * r(m @ w(WUP).T)) @ w(WDOWN).T
    n = r(F.rms_norm(x, (c.d,), Wt[(-1, FINAL_NORM)], c.norm_eps))
    loss = F.cross_entropy((n @ Wt[(-1, LM_HEAD)].T).reshape(-1, c.V), torch.tensor(lab).reshape(-1).long())
    loss.backward()
    return {k: t.grad.double().numpy() for k, t in Wt.items()}


def test_bf16_input_floor_of_first_adam_step():
    shape = synth.WORKLOADS["tiny"]
    c = oracle.OracleConfig(**shape)
    W32 = synth.init_weights(shape, 0)
    Wb = {k: oracle.bf16_round(v) for k, v in W32.items()}
    tok, lab = synth.tokens_labels(c.b, c.s, c.V, 0)
    _, G = oracle.train_step_grads(Wb, tok, lab, c)
    Ge = _emulated_grads(Wb, tok, lab, c)
    hyp = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)
    num = den = 0.0
    flips = total = 0
    for k, w in W32.items():
        p0 = w.astype(np.float64)
        pe, _, _ = oracle.adamw_update(p0, Ge[k], 0 * p0, 0 * p0, 1, **hyp)
        po, _, _ = oracle.adamw_update(p0, G[k], 0 * p0, 0 * p0, 1, **hyp)
        num += np.sum((pe - po) ** 2)
        den += np.sum(po ** 2)
        flips += np.sum(np.sign(Ge[k]) != np.sign(G[k]))
        total += G[k].size
    floor = np.sqrt(num / den)
    assert 1e-3 < floor < 5e-3, floor
    # the sign-flip model explains it: each flipped element moves by 2 lr
    assert abs(floor - 2 * hyp["lr"] * np.sqrt(flips / den)) < 0.2 * floor
