"""Pins of the oracle's building blocks against closed forms, invariants,
brute force and library routines (each test names the fact it relies on)."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- attention

def _brute_attention(q, k, v):
    """Scalar loops: for each (b, head, i) a numerically safe softmax over
    j <= i, query head h reading KV head h // (H / Hkv)."""
    b, s, H, hd = q.shape
    group = H // k.shape[2]
    o = np.zeros_like(q)
    for bi in range(b):
        for h in range(H):
            g = h // group
            for i in range(s):
                sc = [sum(q[bi, i, h, e] * k[bi, j, g, e] for e in range(hd)) / math.sqrt(hd)
                      for j in range(i + 1)]
                mx = max(sc)
                ex = [math.exp(x - mx) for x in sc]
                z = sum(ex)
                for e in range(hd):
                    o[bi, i, h, e] = sum(ex[j] * v[bi, j, g, e] for j in range(i + 1)) / z
    return o


def test_attention_brute_force_gqa():
    rng = np.random.default_rng(0)
    q = rng.normal(size=(2, 7, 4, 4))
    k = rng.normal(size=(2, 7, 2, 4))
    v = rng.normal(size=(2, 7, 2, 4))
    o, P = oracle.attention_fwd(q, k, v)
    assert np.allclose(o, _brute_attention(q, k, v), rtol=1e-12, atol=1e-12)
    assert np.allclose(P.sum(-1), 1.0)
    assert np.all(np.triu(P[0, 0], 1) == 0)  # nothing above the diagonal


def _brute_attention_rows(q, k, v, q_offset):
    """Scalar loops for query rows at positions q_offset + i against keys
    0 .. s_k - 1: softmax over j <= q_offset + i; also the log-sum-exp."""
    b, r, H, hd = q.shape
    group = H // k.shape[2]
    o = np.zeros_like(q)
    lse = np.zeros((b, H, r))
    for bi in range(b):
        for h in range(H):
            g = h // group
            for i in range(r):
                last = q_offset + i
                sc = [sum(q[bi, i, h, e] * k[bi, j, g, e] for e in range(hd)) / math.sqrt(hd)
                      for j in range(last + 1)]
                mx = max(sc)
                ex = [math.exp(x - mx) for x in sc]
                z = sum(ex)
                lse[bi, h, i] = mx + math.log(z)
                for e in range(hd):
                    o[bi, i, h, e] = sum(ex[j] * v[bi, j, g, e] for j in range(last + 1)) / z
    return o, lse


def test_attention_query_block_brute_force_gqa():
    """A block of query rows at positions q_offset .. against the whole key
    prefix (how the long-context parity tests sample rows) follows the same
    causal rule, checked by scalar loops."""
    rng = np.random.default_rng(5)
    sk, r, off = 11, 3, 6
    q = rng.normal(size=(2, r, 4, 4))
    k = rng.normal(size=(2, sk, 2, 4))
    v = rng.normal(size=(2, sk, 2, 4))
    o, P = oracle.attention_fwd(q, k, v, q_offset=off)
    ro, rlse = _brute_attention_rows(q, k, v, off)
    assert np.allclose(o, ro, rtol=1e-12, atol=1e-12)
    assert np.allclose(oracle.attention_lse(q, k, q_offset=off), rlse, rtol=1e-12, atol=1e-12)
    assert P.shape == (2, 4, r, sk) and np.allclose(P.sum(-1), 1.0)
    for i in range(r):
        assert np.all(P[:, :, i, off + i + 1:] == 0)  # keys after the row's position are invisible


def test_attention_query_block_zero_query_is_prefix_mean():
    rng = np.random.default_rng(6)
    sk, r, off = 12, 4, 8
    q = np.zeros((1, r, 2, 8))
    k = rng.normal(size=(1, sk, 1, 8))
    v = rng.normal(size=(1, sk, 1, 8))
    o, _ = oracle.attention_fwd(q, k, v, q_offset=off)
    for i in range(r):
        assert np.allclose(o[0, i, 0], v[0, :off + i + 1, 0].mean(axis=0))


def test_attention_query_block_backward_central_differences():
    """dq of the block's rows and the block's contribution to dk and dv, for
    L = sum(o * W), against central differences in fp64."""
    rng = np.random.default_rng(7)
    sk, r, off, hd = 7, 3, 4, 4
    q = rng.normal(size=(1, r, 2, hd))
    k = rng.normal(size=(1, sk, 1, hd))
    v = rng.normal(size=(1, sk, 1, hd))
    Wt = rng.normal(size=(1, r, 2, hd))
    o, P = oracle.attention_fwd(q, k, v, q_offset=off)
    dq, dk, dv = oracle.attention_bwd(q, k, v, P, Wt)
    h = 1e-6

    def loss(q_, k_, v_):
        return float(np.sum(oracle.attention_fwd(q_, k_, v_, q_offset=off)[0] * Wt))

    for x, g in ((q, dq), (k, dk), (v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = [xp if a is x else a for a in (q, k, v)]
            argm = [xm if a is x else a for a in (q, k, v)]
            fd[idx] = (loss(*args) - loss(*argm)) / (2 * h)
        assert np.allclose(g, fd, rtol=1e-6, atol=1e-8)


def test_attention_zero_query_is_prefix_mean():
    rng = np.random.default_rng(1)
    s = 9
    q = np.zeros((1, s, 4, 8))
    k = rng.normal(size=(1, s, 2, 8))
    v = rng.normal(size=(1, s, 2, 8))
    o, _ = oracle.attention_fwd(q, k, v)
    for h in range(4):
        pref = np.cumsum(v[0, :, h // 2], axis=0) / np.arange(1, s + 1)[:, None]
        assert np.allclose(o[0, :, h], pref)


def test_attention_single_position_is_v():
    rng = np.random.default_rng(2)
    q, k, v = (rng.normal(size=(3, 1, 2, 4)) for _ in range(3))
    o, _ = oracle.attention_fwd(q, k, v)
    assert np.allclose(o, v)


def test_attention_bwd_equal_keys_give_zero_dq():
    """All keys equal => every score row is constant, P is uniform over j <= i
    and rows of dS sum to 0, so dq = dS k / sqrt(hd) = 0."""
    rng = np.random.default_rng(3)
    s = 6
    q = rng.normal(size=(1, s, 2, 4))
    k = np.broadcast_to(rng.normal(size=(1, 1, 1, 4)), (1, s, 1, 4)).copy()
    v = rng.normal(size=(1, s, 1, 4))
    o, P = oracle.attention_fwd(q, k, v)
    dq, dk, dv = oracle.attention_bwd(q, k, v, P, rng.normal(size=o.shape))
    assert np.abs(dq).max() < 1e-13
    assert np.isfinite(dk).all() and np.isfinite(dv).all()


def test_attention_lse_closed_form_and_consistency():
    """q = 0: every visible score is 0, so lse_i = log(i + 1). In general
    P = exp(S / sqrt(hd) - lse) on visible entries."""
    rng = np.random.default_rng(13)
    s = 7
    q0 = np.zeros((1, s, 2, 4))
    k = rng.normal(size=(1, s, 1, 4))
    assert np.allclose(oracle.attention_lse(q0, k)[0, 0], np.log(np.arange(1, s + 1)))
    q = rng.normal(size=(2, s, 4, 8))
    k = rng.normal(size=(2, s, 2, 8))
    v = rng.normal(size=(2, s, 2, 8))
    _, P = oracle.attention_fwd(q, k, v)
    lse = oracle.attention_lse(q, k)
    kk = np.repeat(k, 2, axis=2)
    S = np.einsum("bihd,bjhd->bhij", q, kk) / np.sqrt(8)
    vis = np.tril(np.ones((s, s), dtype=bool))
    assert np.allclose(np.exp(S - lse[..., None])[:, :, vis], P[:, :, vis])


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(4)
    q = rng.normal(size=(2, 13, 6, 16))
    k = rng.normal(size=(2, 13, 3, 16))
    v = rng.normal(size=(2, 13, 3, 16))
    o, _ = oracle.attention_fwd(q, k, v)
    t = lambda a: torch.tensor(a).transpose(1, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), is_causal=True, enable_gqa=True).transpose(1, 2).numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- RoPE

def test_rope_position_zero_is_identity_and_norm_preserved():
    rng = np.random.default_rng(5)
    cos, sin = oracle.rope_tables(10, 8, 10000.0)
    x = rng.normal(size=(2, 10, 3, 8))
    y = oracle.rope_fwd(x, cos, sin)
    assert np.allclose(y[:, 0], x[:, 0])
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1))
    assert np.allclose(oracle.rope_bwd(y, cos, sin), x)  # orthogonal: transpose inverts


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(6)
    hd = 16
    cos, sin = oracle.rope_tables(40, hd, 10000.0)
    qv, kv = rng.normal(size=hd), rng.normal(size=hd)

    def at(vec, p):
        x = np.zeros((1, 40, 1, hd))
        x[0, p, 0] = vec
        return oracle.rope_fwd(x, cos, sin)[0, p, 0]

    base = at(qv, 7) @ at(kv, 3)
    for shift in (1, 5, 20):
        assert np.isclose(at(qv, 7 + shift) @ at(kv, 3 + shift), base, rtol=1e-10)


def test_rope_frequencies():
    cos, sin = oracle.rope_tables(3, 4, 10000.0)
    # theta_0 = 1, theta_1 = 10000^(-1/2) = 0.01
    assert np.allclose(np.arctan2(sin[1], cos[1]), [1.0, 0.01])
    assert np.allclose(np.arctan2(sin[2], cos[2]), [2.0, 0.02])


# ----------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_input():
    cval, eps = 3.0, 1e-5
    x = np.full((2, 8), cval)
    g = np.linspace(0.5, 2, 8)
    y, _ = oracle.rmsnorm_fwd(x, g, eps)
    assert np.allclose(y, cval / math.sqrt(cval * cval + eps) * g)


def test_rmsnorm_bwd_scale_invariance():
    """With eps = 0, RMSNorm(a x) = RMSNorm(x), so the gradient is orthogonal
    to x: sum_j dx_j x_j = 0."""
    rng = np.random.default_rng(7)
    x = rng.normal(size=(5, 16))
    g = rng.normal(size=16)
    _, r = oracle.rmsnorm_fwd(x, g, 0.0)
    dx, _ = oracle.rmsnorm_bwd(x, g, r, rng.normal(size=(5, 16)))
    assert np.abs(np.sum(dx * x, axis=-1)).max() < 1e-12


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(8)
    x = rng.normal(size=(4, 24))
    g = rng.normal(size=24)
    y, _ = oracle.rmsnorm_fwd(x, g, 1e-5)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (24,), torch.tensor(g), 1e-5).numpy()
    assert np.allclose(y, ref, rtol=1e-13)


# ----------------------------------------------------------------- SwiGLU

def test_silu_special_values_and_torch():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    z = np.linspace(-8, 8, 41)
    assert np.allclose(oracle.silu(z), torch.nn.functional.silu(torch.tensor(z)).numpy())
    dgt, dup = oracle.swiglu_bwd(np.zeros(1), np.ones(1), np.ones(1))
    assert np.isclose(dgt[0], 0.5) and dup[0] == 0.0  # silu'(0) = 1/2, silu(0) = 0


# ----------------------------------------------------------------- cross-entropy

def test_uniform_logits_give_ln_vocab():
    rng = np.random.default_rng(9)
    T, d, V = 12, 8, 37
    xL = rng.normal(size=(T, d))
    labels = rng.integers(0, V, T)
    loss, dxL, dgf, dW = oracle.head_ce_fwd_bwd(xL, np.ones(d), np.zeros((V, d)), labels, 1e-5)
    assert abs(loss - math.log(V)) < 1e-14
    assert np.abs(dxL).max() == 0 and np.abs(dgf).max() == 0
    # dz = (1/V - onehot)/T, so dW = dz^T n has columns summing to zero over V
    assert np.abs(dW.sum(axis=0)).max() < 1e-14
    n, _ = oracle.rmsnorm_fwd(xL, np.ones(d), 1e-5)
    onehot = np.zeros((T, V)); onehot[np.arange(T), labels] = 1
    assert np.allclose(dW, ((1.0 / V - onehot) / T).T @ n)


def test_ce_matches_torch():
    rng = np.random.default_rng(10)
    T, d, V = 10, 6, 15
    xL, Wh, g = rng.normal(size=(T, d)), rng.normal(size=(V, d)), rng.normal(size=d)
    labels = rng.integers(0, V, T)
    loss, *_ = oracle.head_ce_fwd_bwd(xL, g, Wh, labels, 1e-5)
    n, _ = oracle.rmsnorm_fwd(xL, g, 1e-5)
    ref = torch.nn.functional.cross_entropy(torch.tensor(n @ Wh.T), torch.tensor(labels)).item()
    assert abs(loss - ref) < 1e-13


def test_loss_at_init_closed_form():
    """Unit-RMS hidden states times N(0, 0.02^2) head rows give logits of
    variance sigma^2 = 0.0004 d, so E[loss] = ln V + sigma^2 / 2."""
    cfg = synth.WORKLOADS["tiny"]
    c = oracle.OracleConfig(**cfg)
    W = {k: v.astype(np.float64) for k, v in synth.init_weights(cfg, 0).items()}
    tok, lab = synth.tokens_labels(c.b, c.s, c.V, 0)
    loss, _ = oracle.train_step_grads(W, tok, lab, c)
    expect = math.log(c.V) + 0.0004 * c.d / 2
    assert abs(loss - expect) < 0.1, (loss, expect)


# ----------------------------------------------------------------- AdamW

H = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def test_adamw_first_step_closed_form():
    p0, g = np.array([0.02, -0.01, 0.5]), np.array([3e-4, -2e-2, 0.0])
    p, m, v = oracle.adamw_update(p0, g, np.zeros(3), np.zeros(3), 1, **H)
    expect = p0 * (1 - 1e-4) - 1e-3 * g / (np.abs(g) + 1e-8)
    assert np.allclose(p, expect, rtol=0, atol=1e-15)
    assert p[2] == p0[2] * (1 - 1e-4)  # g = 0: decay only
    assert np.allclose(m, 0.1 * g) and np.allclose(v, 0.05 * g * g)


def test_adamw_second_step_closed_form():
    p0, g1, g2 = 0.3, 0.7, -0.2
    p, m, v = oracle.adamw_update(p0, g1, 0.0, 0.0, 1, **H)
    p, m, v = oracle.adamw_update(p, g2, m, v, 2, **H)
    mhat = (0.09 * g1 + 0.1 * g2) / 0.19
    vhat = (0.0475 * g1 ** 2 + 0.05 * g2 ** 2) / 0.0975
    p1 = p0 * (1 - 1e-4) - 1e-3 * g1 / (abs(g1) + 1e-8)
    expect = p1 * (1 - 1e-4) - 1e-3 * mhat / (math.sqrt(vhat) + 1e-8)
    assert abs(p - expect) < 1e-15


def test_adamw_matches_torch():
    rng = np.random.default_rng(11)
    p0 = rng.normal(size=50)
    tp = torch.tensor(p0, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=1e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    p, m, v = p0, np.zeros(50), np.zeros(50)
    for t in range(1, 4):
        g = rng.normal(size=50) * 10 ** rng.uniform(-6, 0, 50)
        tp.grad = torch.tensor(g)
        opt.step()
        p, m, v = oracle.adamw_update(p, g, m, v, t, **H)
    assert np.allclose(p, tp.detach().numpy(), rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------- bf16

def test_bf16_round_matches_torch_rne():
    rng = np.random.default_rng(12)
    x = np.concatenate([
        rng.normal(size=10000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 10000),
        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 3.0e38, 1e-40, 0.0, -0.0,
                  np.inf, -np.inf], dtype=np.float32)])
    ref = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_round(x), ref)
    assert np.isnan(oracle.bf16_round(np.array([np.nan], dtype=np.float32))[0])


# ----------------------------------------------------------------- arena layout

def test_arena_layout_counts_and_alignment():
    for name, cfg in synth.WORKLOADS.items():
        c = oracle.OracleConfig(**cfg)
        layout, total = oracle.arena_layout(c)
        hd = c.d // c.H
        mlp = (3 * c.F * c.d + c.d) * c.E if c.E else 3 * c.F * c.d  # experts: E SwiGLUs and the router
        per_layer = 2 * c.d + c.d * hd * (c.H + 2 * c.Hkv) + c.d * c.H * hd + mlp
        params = 2 * c.V * c.d + c.d + c.L * per_layer
        assert sum(int(np.prod(s)) for *_, s in layout) == params
        assert all(off % 64 == 0 for _, _, off, _ in layout)
        assert params <= total < params + 64 * len(layout)


def test_host_state_sizing_matches_pages():
    """fp32 master + two fp32 Adam moments = 12 bytes per parameter, the
    pages' sizing; 120B parameters then fit in 1.5 TB."""
    gold = json.load(open(os.path.join(GOLDEN, "host_ram_sizing.json")))
    bytes_per_param = 3 * np.dtype(np.float32).itemsize
    assert bytes_per_param == gold["host_state_bytes_per_param"]
    assert gold["largest_model_params"] * bytes_per_param <= gold["largest_model_host_ram_bytes"]


def test_tied_gradient_is_the_untied_pair_summed():
    """With the untied head set equal to the embedding, every gradient is the
    same as in the tied model except the table's, which is the untied
    embedding gradient plus the untied head gradient; the arena loses exactly
    the head tensor."""
    import numpy as np
    import oracle
    import synth
    from oracle.model import EMBED, LM_HEAD
    shape = dict(L=1, d=32, H=2, Hkv=1, F=48, V=40, b=2, s=12)
    untied = oracle.OracleConfig(**shape)
    tied = oracle.OracleConfig(**shape, tied=True)
    W = {k: v.astype(np.float64) for k, v in synth.init_weights({**shape, "tied": True}, 2).items()}
    Wu = dict(W)
    Wu[(-1, LM_HEAD)] = W[(-1, EMBED)].copy()
    tok, lab = synth.tokens_labels(2, 12, 40, 5)
    lt, Gt = oracle.train_step_grads(W, tok, lab, tied)
    lu, Gu = oracle.train_step_grads(Wu, tok, lab, untied)
    assert lt == lu
    for k in Gt:
        want = Gu[k] + (Gu[(-1, LM_HEAD)] if k == (-1, EMBED) else 0)
        assert np.allclose(Gt[k], want, rtol=1e-13, atol=1e-16), k  # same sums, another order
    layout_t, n_t = oracle.arena_layout(tied)
    layout_u, n_u = oracle.arena_layout(untied)
    assert [x[:2] for x in layout_t] == [x[:2] for x in layout_u if x[:2] != (-1, LM_HEAD)]
    assert n_u - n_t == 40 * 32
