"""Pins of the oracle's mixture-of-experts MLP (moe_fwd / moe_bwd and the
whole step with expert layers) against facts that do not come from its code:

- one expert and top-1 routing reduce to the dense SwiGLU MLP (gate = 1);
- with every expert routed (k = E) the output is the softmax-weighted sum of
  all experts, written out token by token;
- permuting the experts (router rows and expert weights alike) changes
  nothing;
- top-k picks the largest logits, ties to the lower index;
- the backward equals central finite differences of the forward (routing
  held fixed, as the perturbations are far smaller than the logit gaps) and
  torch fp64 autograd of an independent restatement;
- the whole training step's gradients with expert layers equal central
  finite differences of its loss.
A planted mistake (a gate applied twice) must fail the autograd comparison."""
import numpy as np
import pytest
import torch

import oracle
from oracle.model import (ATTN_NORM, EMBED, FINAL_NORM, LM_HEAD, MLP_NORM, moe_bwd, moe_fwd, moe_gates,
                          moe_route, swiglu_fwd)


def _experts(rng, E, F, d, scale=0.4):
    return (rng.normal(0, scale, (E, d)), rng.normal(0, scale, (E, F, d)), rng.normal(0, scale, (E, F, d)),
            rng.normal(0, scale, (E, d, F)))


def test_one_expert_top1_is_the_dense_mlp():
    rng = np.random.default_rng(0)
    T, d, F = 7, 12, 10
    w = rng.normal(size=(T, d))
    Wr, Wg, Wu, Wd = _experts(rng, 1, F, d)
    y, _ = moe_fwd(w, Wr, Wg, Wu, Wd, 1)
    dense = swiglu_fwd(w @ Wg[0].T, w @ Wu[0].T) @ Wd[0].T
    assert np.allclose(y, dense, rtol=1e-13, atol=1e-13)


def test_all_experts_routed_is_the_softmax_mixture():
    rng = np.random.default_rng(1)
    T, d, F, E = 5, 8, 6, 4
    w = rng.normal(size=(T, d))
    Wr, Wg, Wu, Wd = _experts(rng, E, F, d)
    y, _ = moe_fwd(w, Wr, Wg, Wu, Wd, E)
    for t in range(T):
        z = [float(w[t] @ Wr[e]) for e in range(E)]
        m = max(z)
        p = [np.exp(v - m) for v in z]
        want = np.zeros(d)
        for e in range(E):
            gt = [float(w[t] @ Wg[e, f]) for f in range(F)]
            up = [float(w[t] @ Wu[e, f]) for f in range(F)]
            act = np.array([g / (1.0 + np.exp(-g)) * u for g, u in zip(gt, up)])
            want += p[e] / sum(p) * (Wd[e] @ act)
        assert np.allclose(y[t], want, rtol=1e-12, atol=1e-12)


def test_expert_permutation_changes_nothing():
    rng = np.random.default_rng(2)
    T, d, F, E, k = 9, 8, 6, 5, 2
    w = rng.normal(size=(T, d))
    Wr, Wg, Wu, Wd = _experts(rng, E, F, d)
    perm = rng.permutation(E)
    y1, _ = moe_fwd(w, Wr, Wg, Wu, Wd, k)
    y2, _ = moe_fwd(w, Wr[perm], Wg[perm], Wu[perm], Wd[perm], k)
    assert np.allclose(y1, y2, rtol=1e-13, atol=1e-13)


def test_topk_picks_the_largest_logits_ties_to_the_lower_index():
    w = np.eye(4)
    Wr = np.array([[1.0, 0, 0, 0], [3.0, 0, 0, 0], [3.0, 0, 0, 0], [2.0, 0, 0, 0]])  # row 0 logits: 1, 3, 3, 2
    _, idx = moe_route(w[:1], Wr, 3)
    assert idx.tolist() == [[1, 2, 3]]
    g = moe_gates(np.array([[0.0, np.log(3.0)]]), np.array([[1, 0]]))
    assert np.allclose(g, [[0.75, 0.25]])


def _fixed_route_loss(w, Wr, Wg, Wu, Wd, k, idx, R):
    y, _ = moe_fwd(w, Wr, Wg, Wu, Wd, k, idx=idx)
    return float(np.sum(R * y))


def test_moe_backward_matches_central_differences():
    rng = np.random.default_rng(3)
    T, d, F, E, k = 8, 6, 5, 4, 2
    w = rng.normal(size=(T, d))
    Wr, Wg, Wu, Wd = _experts(rng, E, F, d)
    R = rng.normal(size=(T, d))  # loss = sum(R * y), so dy = R
    _, cache = moe_fwd(w, Wr, Wg, Wu, Wd, k)
    idx = cache["idx"]
    dw, dWr, dWg, dWu, dWd = moe_bwd(R, Wr, Wg, Wu, Wd, cache)
    h = 1e-6
    for name, arr, grad in (("w", w, dw), ("Wr", Wr, dWr), ("Wg", Wg, dWg), ("Wu", Wu, dWu), ("Wd", Wd, dWd)):
        flat, gflat = arr.reshape(-1), grad.reshape(-1)
        for i in rng.choice(flat.size, size=min(12, flat.size), replace=False):
            old = flat[i]
            flat[i] = old + h
            lp = _fixed_route_loss(w, Wr, Wg, Wu, Wd, k, idx, R)
            flat[i] = old - h
            lm = _fixed_route_loss(w, Wr, Wg, Wu, Wd, k, idx, R)
            flat[i] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - gflat[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, gflat[i])
        # the routing the differences held fixed is the router's own at w
        assert np.array_equal(moe_route(w, Wr, k)[1], idx)


def _torch_moe(w, Wr, Wg, Wu, Wd, idx, double_gate=False):
    """Independent restatement: per routed (token, slot), gate * expert."""
    logits = w @ Wr.T
    sel = torch.gather(logits, 1, idx)
    g = torch.softmax(sel, dim=-1)
    if double_gate:  # a planted mistake
        g = g * g
    y = torch.zeros_like(w)
    for j in range(idx.shape[1]):
        e = idx[:, j]
        gt = torch.einsum("td,tfd->tf", w, Wg[e])
        up = torch.einsum("td,tfd->tf", w, Wu[e])
        act = torch.nn.functional.silu(gt) * up
        y = y + g[:, j:j + 1] * torch.einsum("tf,tdf->td", act, Wd[e])
    return y


@pytest.mark.parametrize("plant", [False, True])
def test_moe_backward_matches_torch_autograd(plant):
    rng = np.random.default_rng(4)
    T, d, F, E, k = 11, 8, 7, 6, 3
    w = rng.normal(size=(T, d))
    Wr, Wg, Wu, Wd = _experts(rng, E, F, d)
    R = rng.normal(size=(T, d))
    y, cache = moe_fwd(w, Wr, Wg, Wu, Wd, k)
    grads = moe_bwd(R, Wr, Wg, Wu, Wd, cache)
    ts = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (w, Wr, Wg, Wu, Wd)]
    yt = _torch_moe(*ts, torch.tensor(cache["idx"]), double_gate=plant)
    (yt * torch.tensor(R)).sum().backward()
    ok = np.allclose(yt.detach().numpy(), y, rtol=1e-12, atol=1e-12) and all(
        np.allclose(t.grad.numpy(), g, rtol=1e-10, atol=1e-12) for t, g in zip(ts, grads))
    assert ok != plant


def _moe_weights(c, seed):
    rng = np.random.default_rng(seed)
    W = {(-1, EMBED): rng.normal(0, 0.5, (c.V, c.d))}
    for l in range(c.L):
        for tid, shape in oracle.model._layer_tensors(c):
            W[(l, tid)] = (1.0 + rng.normal(0, 0.3, shape)) if tid in (ATTN_NORM, MLP_NORM) else rng.normal(0, 0.3, shape)
    W[(-1, FINAL_NORM)] = 1.0 + rng.normal(0, 0.3, (c.d,))
    W[(-1, LM_HEAD)] = rng.normal(0, 0.3, (c.V, c.d))
    return W


def test_step_with_expert_layers_matches_central_differences():
    c = oracle.OracleConfig(L=2, d=16, H=2, Hkv=1, F=12, V=30, b=2, s=6, E=4, topk=2)
    W = _moe_weights(c, 5)
    rng = np.random.default_rng(6)
    tok = rng.integers(0, c.V, (c.b, c.s))
    lab = rng.integers(0, c.V, (c.b, c.s))
    _, G = oracle.train_step_grads(W, tok, lab, c)
    h = 1e-5
    for key in [(0, oracle.model.ROUTER), (1, oracle.model.WGATE), (0, oracle.model.WDOWN), (1, oracle.model.WUP),
                (0, oracle.model.WQ), (-1, EMBED)]:
        flat, gflat = W[key].reshape(-1), G[key].reshape(-1)
        for i in rng.choice(flat.size, size=6, replace=False):
            old = flat[i]
            vals = []
            for kk in (1, -1):
                flat[i] = old + kk * h
                vals.append(oracle.train_step_grads(W, tok, lab, c)[0])
            flat[i] = old
            fd = (vals[0] - vals[1]) / (2 * h)
            assert abs(fd - gflat[i]) <= 2e-6 * max(1.0, abs(fd)) + 1e-9, (key, i, fd, gflat[i])


def test_expert_layer_arena_layout():
    """Expert layers: the three expert matrices stacked [E, ...] under the
    dense ids, the router after them; no dense MLP tensors."""
    c = oracle.OracleConfig(L=1, d=64, H=1, Hkv=1, F=32, V=16, b=1, s=4, E=3, topk=1)
    shapes = {tid: shape for layer, tid, off, shape in oracle.arena_layout(c)[0] if layer == 0}
    assert shapes[oracle.model.WGATE] == (3, 32, 64) and shapes[oracle.model.WUP] == (3, 32, 64)
    assert shapes[oracle.model.WDOWN] == (3, 64, 32) and shapes[oracle.model.ROUTER] == (3, 64)
    assert LM_HEAD not in shapes
