"""Shows the oracle's pins have teeth: each plausible mistake planted in the
oracle (a sign, a dropped term, a wrong index, a missing scale) must make the
fp64 torch-autograd comparison fail. Mistakes are planted in the oracle only,
on the CPU, with pytest's monkeypatch."""
import numpy as np
import pytest

import oracle
import oracle.model as M
import synth
from test_oracle_vs_torch import _rel, _torch_step

SHAPE = dict(L=1, d=48, H=6, Hkv=2, F=72, V=33, b=2, s=9)


def _mismatch():
    c = oracle.OracleConfig(**SHAPE)
    W = {k: v.astype(np.float64) * (1 if k[1] in (M.ATTN_NORM, M.MLP_NORM, M.FINAL_NORM) else 10)
         for k, v in synth.init_weights(SHAPE, 5).items()}
    rng = np.random.default_rng(1)
    tok = rng.integers(0, c.V, (c.b, c.s))
    lab = rng.integers(0, c.V, (c.b, c.s))
    loss, G = M.train_step_grads(W, tok, lab, c)
    tloss, TG = _torch_step(W, tok, lab, c)
    worst = max(_rel(G[k], TG[k]) for k in W)
    return max(abs(loss - tloss), worst)


def test_unmutated_oracle_agrees():
    assert _mismatch() < 1e-10


def _rope_bwd_wrong_sign(dy, cos, sin):
    return M.rope_fwd(dy, cos, sin)


def _rms_bwd_dropped_term(x, g, r, dy):
    d = x.shape[-1]
    return r * g * dy, np.sum((dy * x * r).reshape(-1, d), axis=0)


_orig_attn_fwd = M.attention_fwd


def _attn_fwd_wrong_group(q, k, v):
    H, Hkv = q.shape[2], k.shape[2]
    perm = np.array([h % Hkv for h in range(H)])  # tiles instead of grouping
    return _orig_attn_fwd(q, k[:, :, perm], v[:, :, perm])


def _swiglu_bwd_no_chain(gt, up, dact):
    sg = 1 / (1 + np.exp(-gt))
    return dact * up * sg, dact * gt * sg


_orig_attn_bwd = M.attention_bwd


def _attn_bwd_unscaled_dk(q, k, v, P, do):
    dq, dk, dv = _orig_attn_bwd(q, k, v, P, do)
    return dq, dk * np.sqrt(q.shape[-1]), dv


_orig_head = M.head_ce_fwd_bwd


def _head_not_mean(xL, gf, Wh, labels, eps):
    loss, dx, dg, dW = _orig_head(xL, gf, Wh, labels, eps)
    T = xL.shape[0]
    return loss, dx * T, dg * T, dW * T


def _rope_fwd_pairs_adjacent(x, cos, sin):
    x1, x2 = x[..., 0::2], x[..., 1::2]
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


_orig_scores = M._visible_scores


def _scores_see_next_key(q, k, q_offset=0):
    return _orig_scores(q, k, q_offset + 1)  # causal mask off by one: key i + 1 visible to query i


@pytest.mark.parametrize("name,fn", [
    ("rope_bwd", _rope_bwd_wrong_sign),
    ("rmsnorm_bwd", _rms_bwd_dropped_term),
    ("swiglu_bwd", _swiglu_bwd_no_chain),
    ("attention_bwd", _attn_bwd_unscaled_dk),
    ("head_ce_fwd_bwd", _head_not_mean),
    ("rope_fwd", _rope_fwd_pairs_adjacent),
    ("attention_fwd", _attn_fwd_wrong_group),
    ("_visible_scores", _scores_see_next_key),
])
def test_planted_mistake_is_caught(monkeypatch, name, fn):
    monkeypatch.setattr(M, name, fn)
    assert _mismatch() > 1e-6, name
