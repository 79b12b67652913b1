"""Pins the oracle's whole forward and backward against PyTorch autograd in
fp64 on the CPU, built from library routines only (F.embedding, F.rms_norm,
F.scaled_dot_product_attention with GQA, F.silu, F.cross_entropy) and with
RoPE written as a complex multiplication -- a different formulation from the
oracle's rotate-half arithmetic. The torch model shares no code with the
oracle."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth
from oracle.model import (ATTN_NORM, WQ, WK, WV, WO, MLP_NORM, WGATE, WUP, WDOWN,
                          EMBED, FINAL_NORM, LM_HEAD)


def _torch_step(W, tok, lab, c):
    Wt = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in W.items()}
    hd = c.hd
    b, s = tok.shape
    pos = torch.arange(s, dtype=torch.float64)
    inv = c.rope_base ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    rot = torch.polar(torch.ones(s, hd // 2, dtype=torch.float64), pos[:, None] * inv[None, :])

    def rope(x):  # x [b, s, n, hd]; pair (i, i + hd/2) is one complex number
        z = torch.complex(x[..., : hd // 2], x[..., hd // 2:]) * rot[None, :, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    x = F.embedding(torch.tensor(tok), Wt[(-1, EMBED)])
    for l in range(c.L):
        w = lambda t: Wt[(l, t)]
        u = F.rms_norm(x, (c.d,), w(ATTN_NORM), c.norm_eps)
        q = rope((u @ w(WQ).T).view(b, s, c.H, hd)).transpose(1, 2)
        k = rope((u @ w(WK).T).view(b, s, c.Hkv, hd)).transpose(1, 2)
        v = (u @ w(WV).T).view(b, s, c.Hkv, hd).transpose(1, 2)
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
        h = x + o.transpose(1, 2).reshape(b, s, c.H * hd) @ w(WO).T
        m = F.rms_norm(h, (c.d,), w(MLP_NORM), c.norm_eps)
        x = h + (F.silu(m @ w(WGATE).T) * (m @ w(WUP).T)) @ w(WDOWN).T
    n = F.rms_norm(x, (c.d,), Wt[(-1, FINAL_NORM)], c.norm_eps)
    z = n @ Wt[(-1, EMBED) if c.tied else (-1, LM_HEAD)].T  # tied: one parameter, two uses
    loss = F.cross_entropy(z.reshape(-1, c.V), torch.tensor(lab).reshape(-1).long())
    loss.backward()
    return loss.item(), {k: v.grad.numpy() for k, v in Wt.items()}


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("shape", [
    dict(L=2, d=64, H=4, Hkv=4, F=96, V=80, b=2, s=16),
    dict(L=1, d=48, H=6, Hkv=2, F=72, V=33, b=3, s=11),   # GQA 3:1, ragged sizes
    dict(L=1, d=128, H=2, Hkv=1, F=200, V=70, b=1, s=40),  # head_dim 64, GQA 2:1
])
def test_oracle_matches_torch_autograd(shape):
    c = oracle.OracleConfig(**shape)
    W = {k: v.astype(np.float64) for k, v in synth.init_weights(shape, 5).items()}
    rng = np.random.default_rng(1)
    for k in W:  # non-trivial gains and larger weights so every path matters
        if k[1] in (ATTN_NORM, MLP_NORM, FINAL_NORM):
            W[k] = W[k] + rng.normal(0, 0.2, W[k].shape)
        else:
            W[k] = W[k] * 10
    tok = rng.integers(0, c.V, (c.b, c.s))
    lab = rng.integers(0, c.V, (c.b, c.s))
    loss, G = oracle.train_step_grads(W, tok, lab, c)
    tloss, TG = _torch_step(W, tok, lab, c)
    assert abs(loss - tloss) <= 1e-12 * abs(tloss)
    for k in W:
        assert _rel(G[k], TG[k]) <= 1e-10, (k, _rel(G[k], TG[k]))


def test_tiny_workload_matches_torch():
    cfg = synth.WORKLOADS["tiny"]
    c = oracle.OracleConfig(**cfg)
    W = {k: v.astype(np.float64) for k, v in synth.init_weights(cfg, 0).items()}
    tok, lab = synth.tokens_labels(c.b, c.s, c.V, 0)
    loss, G = oracle.train_step_grads(W, tok, lab, c)
    tloss, TG = _torch_step(W, tok, lab, c)
    assert abs(loss - tloss) <= 1e-12 * abs(tloss)
    for k in W:
        assert _rel(G[k], TG[k]) <= 1e-10, k


def test_tied_embeddings_match_torch():
    """Tied embeddings: torch autograd accumulates both uses of the one table
    parameter; the oracle adds the head's gradient to the gather's."""
    shape = dict(L=2, d=64, H=4, Hkv=2, F=96, V=80, b=2, s=16, tied=True)
    c = oracle.OracleConfig(**shape)
    W = {k: v.astype(np.float64) * (1 if k[1] in (ATTN_NORM, MLP_NORM, FINAL_NORM) else 10)
         for k, v in synth.init_weights(shape, 9).items()}
    assert (-1, LM_HEAD) not in W
    rng = np.random.default_rng(4)
    tok = rng.integers(0, c.V, (c.b, c.s))
    lab = rng.integers(0, c.V, (c.b, c.s))
    loss, G = oracle.train_step_grads(W, tok, lab, c)
    tloss, TG = _torch_step(W, tok, lab, c)
    assert abs(loss - tloss) <= 1e-12 * abs(tloss)
    for k in W:
        assert _rel(G[k], TG[k]) <= 1e-10, k
