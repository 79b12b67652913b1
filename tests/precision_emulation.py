"""CPU emulation of where this path rounds to bf16, with each rounding point
switchable, to measure how much of the first-Adam-step floor each one holds.

Test infrastructure (not the oracle, not the product): fp32 torch autograd on
the same bf16 weights the oracle uses, with bf16 rounding placed where the
GPU path rounds:

- fwd_store: activations stored in bf16 between kernels and read by the
  forward and weight-gradient GEMMs (u, q/k/v after RoPE, the attention output,
  w, gate|up, the SwiGLU output, the final-norm output);
- bwd_store: gradients stored in bf16 and read by the input- and
  weight-gradient GEMMs (the gradient of every projection's output, of the
  attention output and of the SwiGLU output, dlogits);
- attn_inner: the attention kernels' own bf16 operands (P for P V and dV,
  dS for dQ and dK);
- dw_exact: the weight-gradient GEMMs read exact fp32 copies of both operands
  instead of the bf16 ones (what a hi+lo split of X and dY on the tensor cores
  computes to ~16 mantissa bits), everything else as chosen above.

The fp32 residual stream, fp32 accumulation, fp32 softmax, fp32 logits and
fp32 RMSNorm statistics are kept, as on the GPU.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.nn.functional as F

from oracle.model import (ATTN_NORM, WQ, WK, WV, WO, MLP_NORM, WGATE, WUP, WDOWN, EMBED, FINAL_NORM, LM_HEAD)


@dataclass(frozen=True)
class Prec:
    fwd_store: bool = True
    bwd_store: bool = True
    attn_inner: bool = True
    dw_exact: bool = False


def _bf(x):
    return x.to(torch.bfloat16).to(torch.float32)


class _R(torch.autograd.Function):
    """Round the value (fwd) and/or the gradient arriving at it (bwd)."""

    @staticmethod
    def forward(ctx, x, fwd, bwd):
        ctx.bwd = bwd
        return _bf(x) if fwd else x.clone()

    @staticmethod
    def backward(ctx, g):
        return (_bf(g) if ctx.bwd else g), None, None


class _Lin(torch.autograd.Function):
    """y = x W^T with the GPU's operand precisions: x read in bf16 when
    rx, the incoming gradient read in bf16 by both backward GEMMs when rg; with
    dw_exact the weight-gradient GEMM reads the exact fp32 x and gradient."""

    @staticmethod
    def forward(ctx, x, W, rx, rg, dw_exact):
        xr = _bf(x) if rx else x
        ctx.save_for_backward(x, xr, W)
        ctx.rg, ctx.dw_exact = rg, dw_exact
        return xr @ W.T

    @staticmethod
    def backward(ctx, gy):
        x, xr, W = ctx.saved_tensors
        gr = _bf(gy) if ctx.rg else gy
        dx = gr @ W
        a, b = (gy, x) if ctx.dw_exact else (gr, xr)
        dW = a.reshape(-1, a.shape[-1]).T @ b.reshape(-1, b.shape[-1])
        return dx, dW, None, None, None


def _attention(q, k, v, p: Prec, scale):
    """Causal attention [b, H, s, hd] with GQA already expanded; P rounded for
    P V / dV and dS rounded for dQ / dK when attn_inner."""
    s = q.shape[-2]
    S = _R.apply((q @ k.transpose(-1, -2)) * scale, False, p.attn_inner)
    mask = torch.ones(s, s, dtype=torch.bool).triu(1)
    P = torch.softmax(S.masked_fill(mask, float("-inf")), dim=-1)
    return _R.apply(P, p.attn_inner, False) @ v


def emulated_grads(Wb: dict, tok: np.ndarray, lab: np.ndarray, c, p: Prec) -> dict:
    """Gradients of the mean next-token CE of the decoder (weights Wb, keyed
    like the oracle's), computed with the rounding points of p."""
    lin = lambda x, W, rx: _Lin.apply(x, W, rx, p.bwd_store, p.dw_exact)  # noqa: E731
    st = lambda x: _R.apply(x, p.fwd_store, False)  # noqa: E731
    Wt = {k: torch.tensor(v, dtype=torch.float32, requires_grad=True) for k, v in Wb.items()}
    hd, (b, s) = c.hd, tok.shape
    rep = c.H // c.Hkv
    ang = torch.arange(s, dtype=torch.float64)[:, None] * \
        (c.rope_base ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd))[None]
    cs, sn = torch.cos(ang).float()[None, :, None], torch.sin(ang).float()[None, :, None]

    def rope(x):
        x1, x2 = x[..., :hd // 2], x[..., hd // 2:]
        return torch.cat([x1 * cs - x2 * sn, x2 * cs + x1 * sn], -1)

    x = F.embedding(torch.tensor(tok).long(), Wt[(-1, EMBED)])
    for l in range(c.L):
        w = lambda t: Wt[(l, t)]  # noqa: E731
        u = F.rms_norm(x, (c.d,), w(ATTN_NORM), c.norm_eps)
        q = st(rope(lin(u, w(WQ), p.fwd_store).view(b, s, c.H, hd))).transpose(1, 2)
        k = st(rope(lin(u, w(WK), p.fwd_store).view(b, s, c.Hkv, hd))).transpose(1, 2)
        v = st(lin(u, w(WV), p.fwd_store).view(b, s, c.Hkv, hd)).transpose(1, 2)
        k, v = k.repeat_interleave(rep, dim=1), v.repeat_interleave(rep, dim=1)
        # the attention output and the SwiGLU output are stored in bf16 (read
        # by the forward GEMM, and by the weight-gradient GEMM unless dw_exact);
        # their gradients (outputs of input-gradient GEMMs) are stored in bf16
        o = _R.apply(_attention(q, k, v, p, 1.0 / np.sqrt(hd)).transpose(1, 2).reshape(b, s, -1), False,
                     p.bwd_store)
        h = x + lin(o, w(WO), p.fwd_store)
        m = F.rms_norm(h, (c.d,), w(MLP_NORM), c.norm_eps)
        gate, up = st(lin(m, w(WGATE), p.fwd_store)), st(lin(m, w(WUP), p.fwd_store))
        act = _R.apply(F.silu(gate) * up, False, p.bwd_store)
        x = h + lin(act, w(WDOWN), p.fwd_store)
    n = F.rms_norm(x, (c.d,), Wt[(-1, FINAL_NORM)], c.norm_eps)
    z = lin(n, Wt[(-1, LM_HEAD)], p.fwd_store)
    loss = F.cross_entropy(z.reshape(-1, c.V), torch.tensor(lab).reshape(-1).long())
    loss.backward()
    return {k: t.grad.double().numpy() for k, t in Wt.items()}


def first_step_floor(W32: dict, G_ref: dict, G: dict, hyp: dict, adamw_update):
    """Relative L2 of the master after the first AdamW step on gradients G
    against the step on G_ref, and the fraction of elements whose gradient
    sign differs."""
    num = den = 0.0
    flips = total = 0
    for k, w in W32.items():
        p0 = w.astype(np.float64)
        pe, _, _ = adamw_update(p0, G[k], 0 * p0, 0 * p0, 1, **hyp)
        po, _, _ = adamw_update(p0, G_ref[k], 0 * p0, 0 * p0, 1, **hyp)
        num += float(np.sum((pe - po) ** 2))
        den += float(np.sum(po ** 2))
        flips += int(np.sum(np.sign(G[k]) != np.sign(G_ref[k])))
        total += G_ref[k].size
    return float(np.sqrt(num / den)), flips / total, den
