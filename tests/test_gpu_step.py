"""End-to-end parity of mt_train_step (through the C ABI) with the oracle.

The oracle runs the same step in fp64 on the bf16-rounded master weights (the
streamed copy the GPU computes with) and updates the fp32 master with AdamW.
Bars (spec tolerances, with the reading for updated parameters derived
in the design notes): loss |d| <= 1e-2; per-tensor gradient relative L2 <=
2e-2; host AdamW on the GPU's own gradients reproduces the updated master to
relative L2 <= 1e-6; the end-to-end updated master is within 5e-3 of the
oracle's (the bf16-input floor of the sign-like first Adam step is ~2.5e-3)."""
import math

import numpy as np
import pytest

import oracle
import synth
from layer_parity import layer_check

pytestmark = pytest.mark.gpu

SHAPES = {
    "tiny": synth.WORKLOADS["tiny"],
    "gqa_ragged": dict(L=3, d=256, H=4, Hkv=2, F=688, V=1024, b=3, s=100),
    "hd128": dict(L=2, d=256, H=2, Hkv=1, F=512, V=520, b=2, s=192),
}
HYP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def _libs():
    from host_memory_streamed_layer_b200 import arena, mt
    return arena, mt


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def run_gpu(shape, nsteps, flags=0, seed=0, init=None):
    arena, mt = _libs()
    cfg = arena.config(shape)
    cfg.flags = flags
    cfg.host_threads = 4
    A = arena.pack(cfg, synth.init_weights(shape, seed) if init is None else init)
    ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    out = []
    try:
        for step in range(nsteps):
            tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], seed, step)
            before = A.copy()
            loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
            G = np.empty_like(A)
            P = np.empty_like(A)
            mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
            mt.mt_get_params(ctx, P.ctypes.data, P.nbytes)
            assert np.array_equal(P, A)  # the caller's arena is the master, updated in place
            out.append(dict(before=before, loss=loss, G=G, P=P, stats=mt.mt_get_stats(ctx)))
    finally:
        mt.mt_destroy(ctx)
    return out


def oracle_steps(shape, nsteps, seed=0):
    """The oracle's own trajectory from the same seeded initial weights."""
    c = oracle.OracleConfig(**shape)
    master = {k: v.astype(np.float64) for k, v in synth.init_weights(shape, seed).items()}
    m = {k: np.zeros_like(v) for k, v in master.items()}
    v2 = {k: np.zeros_like(v) for k, v in master.items()}
    res = []
    for step in range(nsteps):
        tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], seed, step)
        Wb = {k: oracle.bf16_round(w.astype(np.float32)) for k, w in master.items()}
        loss, G = oracle.train_step_grads(Wb, tok, lab, c)
        before = {k: w.copy() for k, w in master.items()}
        for k in master:
            master[k], m[k], v2[k] = oracle.adamw_update(master[k], G[k], m[k], v2[k], step + 1, **HYP)
        res.append(dict(loss=loss, G=G, before=before, P={k: w.copy() for k, w in master.items()}))
    return res


@pytest.mark.parametrize("name", list(SHAPES))
def test_one_step_matches_oracle(name):
    shape = SHAPES[name]
    c = oracle.OracleConfig(**shape)
    g = run_gpu(shape, 1)[0]
    r = oracle_steps(shape, 1)[0]
    assert abs(g["loss"] - r["loss"]) <= 1e-2, (g["loss"], r["loss"])
    G = oracle.unpack_arena(g["G"], c)
    worst = max(rel(G[k], r["G"][k]) for k in r["G"])
    assert worst <= 2e-2, {k: rel(G[k], r["G"][k]) for k in r["G"]}
    # host AdamW on the GPU's own gradients (first step: zero moments)
    before = oracle.unpack_arena(g["before"], c)
    P = oracle.unpack_arena(g["P"], c)
    num = den = 0.0
    for k in before:
        pa, _, _ = oracle.adamw_update(before[k], G[k], 0 * before[k], 0 * before[k], 1, **HYP)
        num += float(np.sum((P[k] - pa) ** 2))
        den += float(np.sum(pa ** 2))
    assert math.sqrt(num / den) <= 1e-6
    # end to end against the oracle's own update
    num = den = 0.0
    for k in before:
        num += float(np.sum((P[k] - r["P"][k]) ** 2))
        den += float(np.sum(r["P"][k] ** 2))
    assert math.sqrt(num / den) <= 5e-3, math.sqrt(num / den)


def test_two_steps_follow_oracle_trajectory():
    shape = SHAPES["tiny"]
    c = oracle.OracleConfig(**shape)
    gs = run_gpu(shape, 2)
    rs = oracle_steps(shape, 2)
    for g, r in zip(gs, rs):
        assert abs(g["loss"] - r["loss"]) <= 1e-2
        G = oracle.unpack_arena(g["G"], c)
        assert max(rel(G[k], r["G"][k]) for k in r["G"]) <= 2e-2


def test_serialized_and_no_update_modes():
    from host_memory_streamed_layer_b200 import mt
    shape = SHAPES["gqa_ragged"]
    c = oracle.OracleConfig(**shape)
    base = run_gpu(shape, 1)[0]
    ser = run_gpu(shape, 1, flags=mt.MT_FLAG_SERIALIZE)[0]
    assert abs(base["loss"] - ser["loss"]) <= 1e-5
    Gb, Gs = oracle.unpack_arena(base["G"], c), oracle.unpack_arena(ser["G"], c)
    assert max(rel(Gs[k], Gb[k]) for k in Gb) <= 1e-3
    nu = run_gpu(shape, 1, flags=mt.MT_FLAG_NO_UPDATE)[0]
    assert np.array_equal(nu["P"], nu["before"])
    Gn = oracle.unpack_arena(nu["G"], c)
    assert max(rel(Gn[k], Gb[k]) for k in Gb) <= 1e-3


@pytest.mark.parametrize("name", ["hd128", "tiny"])
def test_default_steps_are_bitwise_reproducible(name):
    """With the split attention backward (the automatic form, and the only one
    for head dim 64) no reduction of the step depends on timing: the GEMMs
    have no split-K, the normalisation, embedding and loss reductions run in
    a fixed order, and dQ is summed in the query-major kernel. Two pipelined
    runs and a serialized run (one stream) of two steps then give the same
    bits: losses, every gradient and the updated master."""
    arena, mt = _libs()
    shape = SHAPES[name]
    was = mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_AUTO)
    try:
        runs = [run_gpu(shape, 2), run_gpu(shape, 2), run_gpu(shape, 2, flags=mt.MT_FLAG_SERIALIZE)]
    finally:
        mt.mt_k_attn_bwd_variant(was)
    ref = runs[0]
    for other in runs[1:]:
        for a, b in zip(ref, other):
            assert a["loss"] == b["loss"]
            assert np.array_equal(a["G"], b["G"])
            assert np.array_equal(a["P"], b["P"])
    r = oracle_steps(shape, 1)[0]
    assert abs(ref[0]["loss"] - r["loss"]) <= 1e-2


def test_bad_tokens_rejected_before_device_work():
    arena, mt = _libs()
    shape = SHAPES["tiny"]
    cfg = arena.config(shape)
    A = arena.pack(cfg, synth.init_weights(shape, 0))
    A0 = A.copy()
    ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    try:
        tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0)
        tok[0, 3] = shape["V"]
        with pytest.raises(mt.MTError) as e:
            mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
        assert e.value.code == -1
        assert np.array_equal(A, A0)
    finally:
        mt.mt_destroy(ctx)


def test_library_owned_arena_initialisation():
    """NULL arena: the library fills gains with 1 and matrices with N(0, 0.02^2)
    from the seed; the first loss then follows the closed form ln V + sigma^2/2."""
    from host_memory_streamed_layer_b200 import arena, mt
    shape = SHAPES["tiny"]
    cfg = arena.config(shape)
    cfg.seed = 123
    ctx = mt.mt_create(cfg)
    try:
        P = np.empty(mt.mt_arena_bytes(cfg) // 4, dtype=np.float32)
        mt.mt_get_params(ctx, P.ctypes.data, P.nbytes)
        c = oracle.OracleConfig(**shape)
        W = oracle.unpack_arena(P, c)
        assert np.all(W[(0, 0)] == 1.0) and np.all(W[(-1, 101)] == 1.0)
        E = W[(-1, 100)]
        assert abs(E.mean()) < 1e-3 and abs(E.std() - 0.02) < 5e-4
        tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0)
        loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
        assert abs(loss - (math.log(shape["V"]) + 0.0004 * shape["d"] / 2)) < 0.1
    finally:
        mt.mt_destroy(ctx)


def test_chunked_head_matches_oracle(monkeypatch):
    """LM head processed in token chunks (dW_head accumulated across chunks)."""
    monkeypatch.setenv("MT_LOGITS_CHUNK", "128")
    shape = SHAPES["gqa_ragged"]  # T = 300 tokens -> chunks of 128, 128, 44
    c = oracle.OracleConfig(**shape)
    g = run_gpu(shape, 1)[0]
    r = oracle_steps(shape, 1)[0]
    assert abs(g["loss"] - r["loss"]) <= 1e-2
    G = oracle.unpack_arena(g["G"], c)
    assert max(rel(G[k], r["G"][k]) for k in r["G"]) <= 2e-2


def test_checkpoint_resume_continues_the_trajectory():
    """Train two steps in one context; in a second context restore the state
    saved after step 1 and run step 2: same loss and same updated master."""
    from host_memory_streamed_layer_b200 import arena, mt
    shape = SHAPES["tiny"]
    cfg = arena.config(shape)
    A = arena.pack(cfg, synth.init_weights(shape, 0))
    n = A.size
    toks = [synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, k) for k in range(2)]
    ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    try:
        mt.mt_train_step(ctx, toks[0][0].ctypes.data, toks[0][1].ctypes.data)
        P1 = A.copy()
        M1, V1 = np.empty(n, np.float32), np.empty(n, np.float32)
        step = mt.mt_get_opt_state(ctx, M1.ctypes.data, V1.ctypes.data, M1.nbytes)
        loss2 = mt.mt_train_step(ctx, toks[1][0].ctypes.data, toks[1][1].ctypes.data)
        P2 = A.copy()
    finally:
        mt.mt_destroy(ctx)
    assert step == 1 and np.abs(M1).max() > 0 and np.abs(V1).max() > 0
    B = arena.pack(cfg, synth.init_weights(shape, 42))  # different start, overwritten by the restore
    ctx = mt.mt_create(cfg, B.ctypes.data, B.nbytes)
    try:
        mt.mt_set_state(ctx, P1.ctypes.data, M1.ctypes.data, V1.ctypes.data, P1.nbytes, step)
        loss2b = mt.mt_train_step(ctx, toks[1][0].ctypes.data, toks[1][1].ctypes.data)
        P2b = B.copy()
    finally:
        mt.mt_destroy(ctx)
    assert abs(loss2 - loss2b) <= 1e-5
    assert rel(P2b, P2) <= 1e-5


@pytest.mark.parametrize("extra", ["offload", "stash", "offload+stash"])
@pytest.mark.parametrize("name,shape,flags", [
    ("gqa_ragged", SHAPES["gqa_ragged"], 0),
    ("five_layers", dict(L=5, d=256, H=4, Hkv=2, F=688, V=1024, b=2, s=128), 0),
    ("five_layers_ring_defer", dict(L=5, d=256, H=4, Hkv=2, F=688, V=1024, b=2, s=128), 0x8 | 0x10),
    ("long_context", dict(L=4, d=1024, H=8, Hkv=8, F=2816, V=4096, b=1, s=16384), 0x8),
])
def test_offloaded_activations_give_the_resident_result(name, shape, flags, extra):
    """MT_FLAG_OFFLOAD_ACTS: the boundary activations go to host memory in the
    forward and return for each layer's recompute; the copies are exact.
    MT_FLAG_STASH_ATTN: the recompute takes the forward's attention output and
    log-sum-exp instead of running the attention again; the forward is
    deterministic, so they are the recompute's. Either way (and both), two
    steps match the plain run: bit for bit at head dim 128 (the split
    attention backward leaves no order noise), else the first loss to 1e-5,
    every gradient and the updated master to the run-to-run noise of the
    attention's dQ reductions; the first step's loss and gradients match the
    oracle."""
    from host_memory_streamed_layer_b200 import arena, mt
    c = oracle.OracleConfig(**shape)
    runs = {}
    var = (mt.MT_FLAG_OFFLOAD_ACTS if "offload" in extra else 0) | (mt.MT_FLAG_STASH_ATTN if "stash" in extra else 0)
    # Head dim 128 runs the deterministic split attention backward: with no
    # order noise left the two runs must agree bit for bit. (Head dim 64 has
    # only the reduction-based backward.)
    exact = shape["d"] // shape["H"] == 128
    was = mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_SPLIT if exact else mt.ATTN_BWD_AUTO)
    try:
        for off in (0, var):
            cfg = arena.config(shape)
            cfg.flags = flags | off
            cfg.host_threads = 4
            A = arena.pack(cfg, synth.init_weights(shape, 0))
            ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
            out = []
            try:
                for step in range(2):
                    tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, step)
                    loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
                    G = None
                    if not flags & mt.MT_FLAG_GRAD_RING:
                        G = np.empty_like(A)
                        mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
                    out.append((loss, G))
                mt.mt_flush(ctx)
                st = mt.mt_get_stats(ctx)
            finally:
                mt.mt_destroy(ctx)
            runs[off] = (out, A.copy(), st)
    finally:
        mt.mt_k_attn_bwd_variant(was)
    res, off = runs[0], runs[var]
    if exact:
        for (la, Ga), (lb, Gb) in zip(res[0], off[0]):
            assert la == lb and (Ga is None or np.array_equal(Ga, Gb))
        assert np.array_equal(off[1], res[1])
    for step, ((la, Ga), (lb, Gb)) in enumerate(zip(res[0], off[0])):
        # the first forward is deterministic; the second runs on weights that
        # carry the dQ reductions' order noise through one Adam step (at
        # s = 16384 that moves the loss by a few 1e-6 relative)
        assert abs(la - lb) <= (1e-5 if step == 0 else 1e-5 * max(1.0, abs(la)))
        if Ga is not None:
            A_, B_ = oracle.unpack_arena(Ga, c), oracle.unpack_arena(Gb, c)
            assert max(rel(B_[k], A_[k]) for k in A_) <= 1e-4
    # Adam's first steps move each weight by about lr * sign(g): where a
    # gradient lies within the dQ reductions' noise its sign can differ
    # between two runs, so the masters differ by up to 2 lr there (1.4e-3
    # relative seen at s = 16384); the end-to-end bar against the oracle
    assert rel(off[1], res[1]) <= 5e-3
    # the extra link traffic of the offload is accounted for
    T, d, L = shape["b"] * shape["s"], shape["d"], shape["L"]
    moved = 4.0 * (L - 2) * T * d if var & mt.MT_FLAG_OFFLOAD_ACTS else 0.0
    assert off[2]["h2d_bytes"] - res[2]["h2d_bytes"] == pytest.approx(moved)
    # the stash skips exactly the L-1 recomputed attention forwards of a step
    skipped = L - 1 if var & mt.MT_FLAG_STASH_ATTN else 0
    assert res[2]["kernel_launches"] - off[2]["kernel_launches"] == skipped
    if name == "gqa_ragged":
        r = oracle_steps(shape, 1)[0]
        assert abs(off[0][0][0] - r["loss"]) <= 1e-2
        G = oracle.unpack_arena(off[0][0][1], c)
        assert max(rel(G[k], r["G"][k]) for k in r["G"]) <= 2e-2


def _tied_run(shape, flags, nsteps, seed=0):
    from host_memory_streamed_layer_b200 import arena, mt
    cfg = arena.config(shape)
    cfg.flags = flags | mt.MT_FLAG_TIED_EMBED
    cfg.host_threads = 4
    A = arena.pack(cfg, synth.init_weights({**shape, "tied": True}, seed))
    ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    out = []
    try:
        for step in range(nsteps):
            tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], seed, step)
            before = A.copy()
            loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
            G = None
            if not flags & mt.MT_FLAG_GRAD_RING:
                G = np.empty_like(A)
                mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
            mt.mt_flush(ctx)
            out.append(dict(before=before, loss=loss, G=G, P=A.copy()))
    finally:
        mt.mt_destroy(ctx)
    return out


@pytest.mark.parametrize("name", ["tiny", "gqa_ragged", "hd128"])
def test_tied_embeddings_match_oracle(name):
    """MT_FLAG_TIED_EMBED: the head reads the streamed embedding table, and
    the table's gradient is the head's plus the gathered rows'. One step
    against the oracle's tied model: loss, every gradient (no LM-head tensor),
    the host AdamW on the engine's gradients (1e-6) and the end-to-end update
    (the same 5e-3 bar as the untied model)."""
    shape = SHAPES[name]
    c = oracle.OracleConfig(**shape, tied=True)
    g = _tied_run(shape, 0, 1)[0]
    W = {k: oracle.bf16_round(v.astype(np.float32))
         for k, v in oracle.unpack_arena(g["before"], c).items()}
    assert (-1, 102) not in W
    rloss, RG = oracle.train_step_grads(W, *synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, 0), c)
    assert abs(g["loss"] - rloss) <= 1e-2
    G = oracle.unpack_arena(g["G"], c)
    assert max(rel(G[k], RG[k]) for k in RG) <= 2e-2, {k: rel(G[k], RG[k]) for k in RG}
    p, _, _ = oracle.adamw_update(g["before"].astype(np.float64), g["G"].astype(np.float64), 0.0, 0.0, 1, **HYP)
    assert rel(g["P"].astype(np.float64), p) <= 1e-6
    P, before = oracle.unpack_arena(g["P"], c), oracle.unpack_arena(g["before"], c)
    num = den = 0.0
    for k in before:
        po, _, _ = oracle.adamw_update(before[k], RG[k], 0 * before[k], 0 * before[k], 1, **HYP)
        num += float(np.sum((P[k] - po) ** 2))
        den += float(np.sum(po ** 2))
    assert math.sqrt(num / den) <= 5e-3, math.sqrt(num / den)


def test_tied_embeddings_with_ring_and_deferral():
    """Tied embeddings with the gradient ring and deferred updates follow the
    plain tied run for three steps (same losses, same master)."""
    from host_memory_streamed_layer_b200 import mt
    shape = dict(L=5, d=256, H=4, Hkv=2, F=688, V=1024, b=2, s=128)
    base = _tied_run(shape, 0, 3)
    alt = _tied_run(shape, mt.MT_FLAG_GRAD_RING | mt.MT_FLAG_DEFER_UPDATES, 3)
    for a, b in zip(base, alt):
        assert abs(a["loss"] - b["loss"]) <= 1e-4
        assert rel(b["P"], a["P"]) <= 2e-3


def test_bf16_gradient_offload_stays_within_the_bars():
    """MT_FLAG_BF16_GRADS: every gradient is rounded once to bf16 before it
    leaves the GPU (the embedding rows on the host). The gradients the library
    reports are bf16 values, the update is AdamW on exactly those, and the
    loss, gradients and updated master stay within the oracle bars; the cost
    of the extra rounding is measured against the fp32 offload of the same
    step."""
    from host_memory_streamed_layer_b200 import mt
    shape = SHAPES["gqa_ragged"]
    c = oracle.OracleConfig(**shape)
    g16 = run_gpu(shape, 1, flags=mt.MT_FLAG_BF16_GRADS)[0]
    g32 = run_gpu(shape, 1)[0]
    r = oracle_steps(shape, 1)[0]
    assert np.array_equal(g16["G"], oracle.bf16_round(g16["G"]))
    assert abs(g16["loss"] - r["loss"]) <= 1e-2
    G, G32 = oracle.unpack_arena(g16["G"], c), oracle.unpack_arena(g32["G"], c)
    assert max(rel(G[k], r["G"][k]) for k in r["G"]) <= 2e-2
    # the rounding itself: at most half a bf16 ulp per element (2^-9 relative)
    assert max(rel(G[k], G32[k]) for k in G32) <= 5e-3
    p, _, _ = oracle.adamw_update(g16["before"].astype(np.float64), g16["G"].astype(np.float64), 0.0, 0.0, 1, **HYP)
    assert rel(g16["P"].astype(np.float64), p) <= 1e-6
    P, before = oracle.unpack_arena(g16["P"], c), oracle.unpack_arena(g16["before"], c)
    num = sum(float(np.sum((P[k] - r["P"][k]) ** 2)) for k in before)
    den = sum(float(np.sum(r["P"][k] ** 2)) for k in before)
    assert math.sqrt(num / den) <= 5e-3, math.sqrt(num / den)


def test_resume_follows_the_oracle_from_the_restored_state():
    """Checkpoint after step 1 (master, moments, step counter), restore into a
    fresh context and run step 2 there: the loss and gradients are the
    oracle's on the restored master, the update is AdamW at t = 2 from the
    restored moments (relative 1e-6 on the engine's own gradients), and the
    updated master, m and v are within the end-to-end bars of the oracle's
    own step-2 update from the same restored state."""
    from host_memory_streamed_layer_b200 import arena, mt
    shape = SHAPES["gqa_ragged"]
    c = oracle.OracleConfig(**shape)
    cfg = arena.config(shape)
    cfg.host_threads = 4
    A = arena.pack(cfg, synth.init_weights(shape, 0))
    n = A.size
    toks = [synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, k) for k in range(2)]
    ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    try:
        mt.mt_train_step(ctx, toks[0][0].ctypes.data, toks[0][1].ctypes.data)
        P1 = A.copy()
        M1, V1 = np.empty(n, np.float32), np.empty(n, np.float32)
        step = mt.mt_get_opt_state(ctx, M1.ctypes.data, V1.ctypes.data, M1.nbytes)
    finally:
        mt.mt_destroy(ctx)
    assert step == 1
    B = arena.pack(cfg, synth.init_weights(shape, 7))
    ctx = mt.mt_create(cfg, B.ctypes.data, B.nbytes)
    try:
        mt.mt_set_state(ctx, P1.ctypes.data, M1.ctypes.data, V1.ctypes.data, P1.nbytes, step)
        loss2 = mt.mt_train_step(ctx, toks[1][0].ctypes.data, toks[1][1].ctypes.data)
        G2 = np.empty_like(B)
        mt.mt_get_grads(ctx, G2.ctypes.data, G2.nbytes)
        M2, V2 = np.empty(n, np.float32), np.empty(n, np.float32)
        assert mt.mt_get_opt_state(ctx, M2.ctypes.data, V2.ctypes.data, M2.nbytes) == 2
        P2 = B.copy()
    finally:
        mt.mt_destroy(ctx)
    Wb = {k: oracle.bf16_round(w.astype(np.float32)) for k, w in oracle.unpack_arena(P1, c).items()}
    rloss, RG = oracle.train_step_grads(Wb, toks[1][0], toks[1][1], c)
    assert abs(loss2 - rloss) <= 1e-2
    G = oracle.unpack_arena(G2, c)
    assert max(rel(G[k], RG[k]) for k in RG) <= 2e-2
    # the host update from the restored state, on the engine's own gradients
    p, m, v = oracle.adamw_update(P1.astype(np.float64), G2.astype(np.float64), M1.astype(np.float64),
                                  V1.astype(np.float64), 2, **HYP)
    for got, want in ((P2, p), (M2, m), (V2, v)):
        assert rel(got.astype(np.float64), want) <= 1e-6
    # end to end against the oracle's step-2 update from the same restored state
    Pu, Mu, Vu = oracle.unpack_arena(P1, c), oracle.unpack_arena(M1, c), oracle.unpack_arena(V1, c)
    P2d, M2d, V2d = oracle.unpack_arena(P2, c), oracle.unpack_arena(M2, c), oracle.unpack_arena(V2, c)
    num = den = 0.0
    for k in RG:
        po, mo, vo = oracle.adamw_update(Pu[k].astype(np.float64), RG[k], Mu[k].astype(np.float64),
                                         Vu[k].astype(np.float64), 2, **HYP)
        num += float(np.sum((P2d[k] - po) ** 2))
        den += float(np.sum(po ** 2))
        assert rel(M2d[k].astype(np.float64), mo) <= 2e-2, k
        assert rel(V2d[k].astype(np.float64), vo) <= 4e-2, k
    assert math.sqrt(num / den) <= 5e-3, math.sqrt(num / den)


def test_gradient_ring_matches_full_arena_and_oracle():
    """MT_FLAG_GRAD_RING: layer gradients pass through MT_GRAD_RING_SLOTS host
    slots (5 layers > slots, so offloads wait for released slots) and the
    untouched embedding rows take the zero-gradient update. Two steps follow
    the run with the full gradient arena (same tokens and initial master) and
    the first step's update is within the end-to-end bar of the oracle's."""
    from host_memory_streamed_layer_b200 import arena, mt
    shape = dict(L=5, d=256, H=4, Hkv=4, F=688, V=1024, b=2, s=128)
    assert shape["L"] > mt.MT_GRAD_RING_SLOTS
    c = oracle.OracleConfig(**shape)
    full = run_gpu(shape, 2)
    cfg = arena.config(shape)
    cfg.flags = mt.MT_FLAG_GRAD_RING
    cfg.host_threads = 4
    A = arena.pack(cfg, synth.init_weights(shape, 0))
    ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    ring = []
    try:
        for step in range(2):
            tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, step)
            loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
            ring.append(dict(loss=loss, P=A.copy()))
        with pytest.raises(mt.MTError) as e:
            G = np.empty_like(A)
            mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
        assert e.value.code == -2
    finally:
        mt.mt_destroy(ctx)
    for f, r in zip(full, ring):
        assert abs(f["loss"] - r["loss"]) <= 1e-4
        assert rel(r["P"], f["P"]) <= 2e-3
    o = oracle_steps(shape, 1)[0]
    P = oracle.unpack_arena(ring[0]["P"], c)
    num = sum(float(np.sum((P[k] - o["P"][k]) ** 2)) for k in P)
    den = sum(float(np.sum(o["P"][k] ** 2)) for k in P)
    assert abs(ring[0]["loss"] - o["loss"]) <= 1e-2
    assert math.sqrt(num / den) <= 5e-3


@pytest.mark.parametrize("name", ["gqa_ragged", "hd128"])
def test_layer_template_matches_oracle(name):
    """mt_layer_fwd_bwd (the engine's per-layer forward + backward on supplied
    boundary activations) against the oracle's layer, for every layer."""
    from host_memory_streamed_layer_b200 import arena, mt
    shape = SHAPES[name]
    cfg = arena.config(shape)
    init = synth.init_weights(shape, 3)
    A = arena.pack(cfg, init)
    ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    rng = np.random.default_rng(11)
    T, d = shape["b"] * shape["s"], shape["d"]
    try:
        for layer in range(shape["L"]):
            W = {tid: oracle.bf16_round(init[(layer, tid)].astype(np.float32)).astype(np.float64) for tid in range(9)}
            x = rng.normal(size=(T, d)).astype(np.float32)
            dxn = rng.normal(size=(T, d)).astype(np.float32)
            layer_check(mt, ctx, cfg, shape, layer, W, x, dxn, list(range(shape["b"])))
        P = np.empty_like(A)
        mt.mt_get_params(ctx, P.ctypes.data, P.nbytes)
        assert np.array_equal(P, A)  # no optimizer step
    finally:
        mt.mt_destroy(ctx)


def test_step_timeline_is_consistent():
    """mt_get_timeline after a step: 2L-1 weight loads in the order 0..L-1,
    L-2..0; every load's H2D precedes its readiness and every offload follows
    its gradients; the backward offloads run L-1..0; the host ran one job per
    layer plus the head and both embedding jobs, each after its data."""
    from host_memory_streamed_layer_b200 import arena, mt
    shape = dict(L=4, d=256, H=4, Hkv=4, F=688, V=1024, b=2, s=128)
    cfg = arena.config(shape)
    cfg.host_threads = 4
    ctx = mt.mt_create(cfg)
    try:
        tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0)
        for _ in range(2):
            mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
        tl = mt.mt_get_timeline(ctx)
    finally:
        mt.mt_destroy(ctx)
    L = shape["L"]
    assert [x["layer"] for x in tl["loads"]] == list(range(L)) + list(range(L - 2, -1, -1))
    eps = 1e-3
    for ld in tl["loads"]:
        assert 0 - eps <= ld["h2d_start"] <= ld["ready"] + eps
        assert ld["ready"] <= ld["released"] + eps and ld["compute_arrives"] <= ld["released"] + eps
    assert [o["layer"] for o in tl["offload"]] == list(range(L - 1, -1, -1))
    for o in tl["offload"]:
        assert o["grads_ready"] <= o["d2h_start"] + eps <= o["d2h_done"] + 2 * eps
        assert o["d2h_done"] <= tl["phases"]["step_end"] + eps
    ph = tl["phases"]
    assert ph["fwd_end"] <= ph["head_end"] <= ph["bwd_end"] <= ph["step_end"]
    kinds = sorted(j["kind"] for j in tl["jobs"])
    assert kinds == [0] * L + [1, 2, 3]
    assert sorted(j["layer"] for j in tl["jobs"] if j["kind"] == 0) == list(range(L))
    assert all(j["ready_ms"] <= j["done_ms"] for j in tl["jobs"])


def test_head_matches_oracle(monkeypatch):
    """mt_head_fwd_bwd (final norm, LM head in token chunks, CE and its
    backward, as in the step) against the oracle's head."""
    monkeypatch.setenv("MT_LOGITS_CHUNK", "128")  # T = 300: chunks of 128, 128, 44
    from host_memory_streamed_layer_b200 import arena, mt
    from layer_parity import head_check
    shape = SHAPES["gqa_ragged"]
    cfg = arena.config(shape)
    ctx = mt.mt_create(cfg)
    try:
        T = shape["b"] * shape["s"]
        x = np.random.default_rng(5).normal(size=(T, shape["d"])).astype(np.float32)
        _, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 2)
        head_check(mt, ctx, cfg, shape, x, np.ascontiguousarray(lab.reshape(-1)).astype(np.int32))
        with pytest.raises(mt.MTError) as e:
            bad = np.full(T, shape["V"], dtype=np.int32)
            g = np.empty(1 << 22, dtype=np.float32)
            mt.mt_head_fwd_bwd(ctx, x.ctypes.data, bad.ctypes.data, x.ctypes.data, g.ctypes.data, g.nbytes)
        assert e.value.code == -1
    finally:
        mt.mt_destroy(ctx)


def test_deferred_updates_follow_the_undeferred_trajectory(monkeypatch):
    """MT_FLAG_DEFER_UPDATES (2 deferred layers of 6, plus the LM head): three
    steps with no flush between them, so each step's deferred updates run in
    the next step's forward sweep and the weight loads wait for them. Each
    step's loss and gradients match the undeferred run's (stale weights in a
    load would change them), the state after mt_flush is AdamW replayed on the
    engine's own gradients with each step's bias correction (relative 1e-6),
    mt_get_params flushes, the deferred jobs appear in the timeline and finish
    before their layer's forward load starts, and the gradient ring with
    deferral reaches the same master."""
    from host_memory_streamed_layer_b200 import arena, mt
    monkeypatch.setenv("MT_DEFER_LAYERS", "2")
    shape = dict(L=6, d=256, H=4, Hkv=2, F=688, V=1024, b=2, s=128)
    L, nd, n_steps = shape["L"], 2, 3
    toks = [synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, k) for k in range(n_steps)]

    def run(flags, grads):
        cfg = arena.config(shape)
        cfg.flags = flags
        cfg.host_threads = 4
        A = arena.pack(cfg, synth.init_weights(shape, 0))
        P0 = A.copy()
        ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
        losses, Gs = [], []
        try:
            for tok, lab in toks:
                losses.append(mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data))
                if grads:
                    G = np.empty_like(A)
                    mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
                    Gs.append(G)
            tl = mt.mt_get_timeline(ctx)
            P = np.empty_like(A)
            mt.mt_get_params(ctx, P.ctypes.data, P.nbytes)
            assert np.array_equal(P, A)  # the pending updates were applied first
            mt.mt_flush(ctx)  # nothing left: a no-op
            M, V = np.empty_like(A), np.empty_like(A)
            assert mt.mt_get_opt_state(ctx, M.ctypes.data, V.ctypes.data, M.nbytes) == n_steps
        finally:
            mt.mt_destroy(ctx)
        return dict(P0=P0, P=P, M=M, V=V, losses=losses, G=Gs, tl=tl)

    base = run(0, True)
    dfr = run(mt.MT_FLAG_DEFER_UPDATES, True)
    c = oracle.OracleConfig(**shape)
    for k in range(n_steps):
        assert abs(dfr["losses"][k] - base["losses"][k]) <= 1e-5, k
        Gd, Gb = oracle.unpack_arena(dfr["G"][k], c), oracle.unpack_arena(base["G"][k], c)
        assert max(rel(Gd[t], Gb[t]) for t in Gb) <= 1e-3, k
    p, m, v = dfr["P0"].astype(np.float64), 0.0, 0.0
    for k in range(n_steps):
        p, m, v = oracle.adamw_update(p, dfr["G"][k], m, v, k + 1, **HYP)
    for got, want in ((dfr["P"], p), (dfr["M"], m), (dfr["V"], v)):
        assert rel(got.astype(np.float64), want) <= 1e-6
    # timeline of the last step: one check job per layer and for the head, the
    # touched embedding rows, and the previous step's deferred head, layers and
    # untouched embedding rows (those this step gathers first, then the rest)
    jobs = dfr["tl"]["jobs"]
    assert sorted(j["kind"] for j in jobs) == sorted([0] * L + [1, 2, 4, 6, 7] + [5] * nd)
    assert sorted(j["layer"] for j in jobs if j["kind"] == 5) == list(range(L - nd, L))
    loads = dfr["tl"]["loads"]
    for j in jobs:
        if j["kind"] == 5:
            assert j["done_ms"] <= loads[j["layer"]]["h2d_start"] + 1.0
    # gradient ring + deferral: 2 deferred buffers, ring waits from backward index 5
    ring = run(mt.MT_FLAG_DEFER_UPDATES | mt.MT_FLAG_GRAD_RING, False)
    for a, b in zip(ring["losses"], dfr["losses"]):
        assert abs(a - b) <= 1e-4
    assert rel(ring["P"], dfr["P"]) <= 2e-3


@pytest.mark.parametrize("flags", [0, 0x8 | 0x10, 0x40 | 0x100])
def test_poisoned_slots_and_host_stalls_leave_the_steps_unchanged(flags):
    """Race checks without a sanitizer. MT_FLAG_POISON fills each weight slot
    with NaN once the compute stream releases it and each gradient slot before
    a backward writes it: a read before a reload or write completes would turn
    the results into NaN. A host stall injected on the weight stream, then on
    the gradient stream, delays copies without changing what any kernel reads.
    With the split attention backward every reduction has a fixed order, so
    all runs must agree bit for bit (plain, ring + deferral, offload + stash)."""
    arena, mt = _libs()
    shape = dict(SHAPES["hd128"], L=4)  # enough layers for offloaded boundaries and a recompute chain

    def run(extra, stall=None):
        cfg = arena.config(shape)
        cfg.flags = flags | extra
        cfg.host_threads = 4
        A = arena.pack(cfg, synth.init_weights(shape, 0))
        ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
        out = []
        try:
            for step in range(2):
                tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, step)
                if stall is not None:
                    mt.mt_inject_host_stall(ctx, stall[step], 60)
                loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
                mt.mt_flush(ctx)
                G = None
                if not cfg.flags & mt.MT_FLAG_GRAD_RING:
                    G = np.empty_like(A)
                    mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
                out.append((loss, G, A.copy()))
        finally:
            mt.mt_destroy(ctx)
        return out

    was = mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_SPLIT)
    try:
        ref = run(0)
        others = [run(mt.MT_FLAG_POISON), run(0, stall=(0, 2)), run(mt.MT_FLAG_POISON, stall=(2, 0))]
    finally:
        mt.mt_k_attn_bwd_variant(was)
    for other in others:
        for (la, Ga, Pa), (lb, Gb, Pb) in zip(ref, other):
            assert la == lb and np.isfinite(lb)
            assert Ga is None or np.array_equal(Ga, Gb)
            assert np.array_equal(Pa, Pb)
