"""Mixture-of-experts layers through mt_train_step, against the oracle.

The GPU computes the router's logits from bf16 operands, the oracle in fp64;
where two logits of a token lie within that rounding the two may choose
different experts, and both choices are correct. So each test first checks
that every choice the GPU made is a valid top-k under the oracle's logits (no
unchosen expert beats a chosen one by more than the rounding), then runs the
oracle with the GPU's routing (mt_get_routing) and compares loss and every
gradient at the bars of the dense step. Head dim 128 with the split attention
backward makes a step bitwise reproducible, which the last test checks."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

SHAPES = {
    "e4k2": dict(L=2, d=256, H=2, Hkv=1, F=128, V=512, b=2, s=64, E=4, topk=2),
    # more experts than routed rows need: several experts get no token
    "sparse": dict(L=2, d=128, H=1, Hkv=1, F=64, V=256, b=1, s=8, E=16, topk=1),
    "ragged": dict(L=3, d=256, H=4, Hkv=2, F=96, V=304, b=3, s=37, E=6, topk=3),
    # one layer, one token: two routed rows, one idle expert
    "one_token": dict(L=1, d=128, H=1, Hkv=1, F=64, V=64, b=1, s=1, E=3, topk=2),
}


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _step(shape, flags=0, nsteps=1):
    from host_memory_streamed_layer_b200 import arena, mt
    cfg = arena.config(shape)
    cfg.flags = flags
    cfg.host_threads = 4
    A = arena.pack(cfg, synth.init_weights(shape, 0))
    ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    out = []
    try:
        for step in range(nsteps):
            tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, step)
            loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
            G = None
            if not flags & mt.MT_FLAG_GRAD_RING:
                G = np.empty_like(A)
                mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
            T = shape["b"] * shape["s"]
            route = {l: mt.mt_get_routing(ctx, l, T, shape["topk"]) for l in range(shape["L"])}
            out.append(dict(loss=loss, G=G, P=A.copy(), route=route))
    finally:
        mt.mt_destroy(ctx)
    return out


def _check_routing(route, logits, k):
    """Each token's chosen experts are distinct, and no unchosen expert's
    oracle logit exceeds the smallest chosen one by more than the rounding of
    a bf16 dot product (relative to the row's scale)."""
    T, E = logits.shape
    assert route.shape == (T, k)
    for t in range(T):
        ch = route[t]
        assert len(set(ch.tolist())) == k and ch.min() >= 0 and ch.max() < E
        rest = np.setdiff1d(np.arange(E), ch)
        tol = 2e-2 * np.max(np.abs(logits[t])) + 1e-6
        if rest.size:
            assert logits[t, rest].max() <= logits[t, ch].min() + tol, (t, logits[t], ch)


@pytest.mark.parametrize("name", list(SHAPES))
def test_expert_step_matches_the_oracle(name):
    shape = SHAPES[name]
    c = oracle.OracleConfig(**shape)
    run = _step(shape)[0]
    tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, 0)
    init = synth.init_weights(shape, 0)
    Wb = {k: oracle.bf16_round(v.astype(np.float32)) for k, v in init.items()}
    logits = {}
    loss, G = oracle.train_step_grads(Wb, tok, lab, c, routing=run["route"], logits_out=logits)
    for l in range(shape["L"]):
        _check_routing(run["route"][l], logits[l], shape["topk"])
    assert abs(run["loss"] - loss) <= 1e-2
    got = oracle.unpack_arena(run["G"], c)
    worst = {k: rel(got[k], G[k]) for k in G if np.linalg.norm(G[k]) > 0}
    assert max(worst.values()) <= 2e-2, sorted(worst.items(), key=lambda kv: -kv[1])[:3]
    # experts no token chose get exactly zero gradient
    for l in range(shape["L"]):
        used = set(run["route"][l].reshape(-1).tolist())
        for e in range(shape["E"]):
            if e not in used:
                for tid in (oracle.model.WGATE, oracle.model.WUP, oracle.model.WDOWN):
                    assert not np.any(got[(l, tid)][e])


def test_expert_step_host_update_is_adamw_on_the_gpu_gradients():
    """The update of expert and router tensors is the host AdamW of the
    gradients the GPU produced (the same routine as the dense tensors)."""
    shape = SHAPES["e4k2"]
    c = oracle.OracleConfig(**shape)
    run = _step(shape)[0]
    init = synth.init_weights(shape, 0)
    P0 = {k: v.astype(np.float64) for k, v in init.items()}
    G = oracle.unpack_arena(run["G"], c)
    P = oracle.unpack_arena(run["P"], c)
    hyp = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)
    for key in [(0, oracle.model.ROUTER), (1, oracle.model.WGATE), (0, oracle.model.WDOWN)]:
        want, _, _ = oracle.adamw_update(P0[key], G[key], np.zeros_like(P0[key]), np.zeros_like(P0[key]), 1, **hyp)
        assert rel(P[key], want) <= 1e-6


def test_expert_steps_are_bitwise_reproducible_and_ring_agrees():
    """With the split attention backward every reduction has a fixed order
    (the routing, the grouped rows, the combine and the router sums too):
    two runs of two steps agree bit for bit, and the gradient ring gives the
    arena run's parameters."""
    from host_memory_streamed_layer_b200 import mt
    shape = SHAPES["e4k2"]
    was = mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_SPLIT)
    try:
        a = _step(shape, nsteps=2)
        b = _step(shape, nsteps=2)
        ring = _step(shape, flags=mt.MT_FLAG_GRAD_RING, nsteps=2)
    finally:
        mt.mt_k_attn_bwd_variant(was)
    for x, y, z in zip(a, b, ring):
        assert x["loss"] == y["loss"] == z["loss"]
        assert np.array_equal(x["G"], y["G"]) and np.array_equal(x["P"], y["P"]) and np.array_equal(x["P"], z["P"])
        for l in x["route"]:
            assert np.array_equal(x["route"][l], y["route"][l])
