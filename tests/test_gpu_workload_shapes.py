"""Parity at the shapes of the other workloads, in the launch configuration of
the step: llama-7b (d 4096, 32 heads of 128, FFN 11008, 4 x 4096 tokens),
gqa-14b (d 5120, 40 query heads over 8 KV heads, FFN 13824, vocab 152064,
2 x 4096 tokens) and llama-7b-128k (one sequence of 131072 tokens).

A layer's kernels do not depend on how many layers the model has, so each test
creates a one-layer context with the workload's per-layer shapes (a few GB of
host memory instead of the whole model's). Where the oracle cannot run the
whole shape, the checks use what the method's structure fixes exactly:
- attention: sampled query rows against the oracle on their causal prefix,
  and the last keys' dK and dV, which only the last queries see;
- layer forward and backward: the upstream gradient is nonzero only on a
  prefix of sequence 0, so by causality every weight gradient and the input
  gradient of that prefix depend on the prefix alone (the oracle runs it as a
  sequence of its own), and every other input-gradient row is exactly zero;
- head and cross-entropy: hidden rows are zero outside a block of active
  tokens. A zero row normalises to zero, so its logits are zero (its loss is
  exactly ln V) and it adds nothing to the LM-head or final-gain gradients. Its
  input gradient is eps^(-1/2) g * dn with dn = (mean of the head's rows - the
  row of its label) / T.
These tests carry the `late` marker: they run after the other tests."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = [pytest.mark.gpu, pytest.mark.late]
DEV = "cuda"
HD = 128
NAMES = ["llama-7b", "gqa-14b", "llama-7b-128k"]


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


# ----------------------------------------------------------------- checks
# Each takes the GPU's outputs as numpy arrays, so it can be run on any source
# of them.

def check_attention_rows(Q, K, V, O, LSE, DO, DQ, samples, H, Hkv):
    """Q, O, DO, DQ: [b, s, H, hd]; K, V: [b, s, Hkv, hd] (any array type whose
    slices convert with np.asarray); LSE [b, H, s]. Sampled (bi, h, i): the
    output, log-sum-exp and dq of query row i against the oracle on its prefix."""
    grp = H // Hkv
    for bi, h, i in samples:
        g = h // grp
        q = np.asarray(Q[bi, i:i + 1, h:h + 1], dtype=np.float64)[None]
        k = np.asarray(K[bi, :i + 1, g:g + 1], dtype=np.float64)[None]
        v = np.asarray(V[bi, :i + 1, g:g + 1], dtype=np.float64)[None]
        ro, P = oracle.attention_fwd(q, k, v, q_offset=i)
        got = np.asarray(O[bi, i, h], dtype=np.float64)
        assert np.linalg.norm(got - ro[0, 0, 0]) <= 1e-2 * np.linalg.norm(ro[0, 0, 0]) + 1e-3, (bi, h, i)
        assert abs(float(LSE[bi, h, i]) - oracle.attention_lse(q, k, q_offset=i)[0, 0, 0]) < 1e-3, (bi, h, i)
        do = np.asarray(DO[bi, i:i + 1, h:h + 1], dtype=np.float64)[None]
        rdq, _, _ = oracle.attention_bwd(q, k, v, P, do)
        gq = np.asarray(DQ[bi, i, h], dtype=np.float64)
        assert np.linalg.norm(gq - rdq[0, 0, 0]) <= 2e-2 * np.linalg.norm(rdq[0, 0, 0]) + 1e-3, (bi, h, i)


def check_last_keys(Q, K, V, DO, DK, DV, bi, g, H, Hkv, n=16):
    """dK, dV of the last n keys of sequence bi, KV head g: only the last n
    queries of the group's query heads see them."""
    grp = H // Hkv
    s = K.shape[1]
    q = np.asarray(Q[bi, s - n:, g * grp:(g + 1) * grp], dtype=np.float64)[None]
    k = np.asarray(K[bi, :, g:g + 1], dtype=np.float64)[None]
    v = np.asarray(V[bi, :, g:g + 1], dtype=np.float64)[None]
    do = np.asarray(DO[bi, s - n:, g * grp:(g + 1) * grp], dtype=np.float64)[None]
    _, P = oracle.attention_fwd(q, k, v, q_offset=s - n)
    _, rdk, rdv = oracle.attention_bwd(q, k, v, P, do)
    gk = np.asarray(DK[bi, s - n:, g], dtype=np.float64)
    gv = np.asarray(DV[bi, s - n:, g], dtype=np.float64)
    assert np.linalg.norm(gk - rdk[0, -n:, 0]) <= 2e-2 * np.linalg.norm(rdk[0, -n:, 0])
    assert np.linalg.norm(gv - rdv[0, -n:, 0]) <= 2e-2 * np.linalg.norm(rdv[0, -n:, 0])


def check_layer_prefix(shape, W, x, dxn, xo, dxi, grads, n_pre, tol=2e-2):
    """Sequence 0's first n_pre tokens carry the only nonzero upstream gradient.
    grads: {tensor id: the layer's gradient, shaped like W[tid]}."""
    c = oracle.OracleConfig(**{**shape, "b": 1, "s": n_pre})
    cos, sin = oracle.rope_tables(n_pre, c.hd, c.rope_base)
    x3 = x[:n_pre].astype(np.float64)[None]
    xn, cache = oracle.layer_fwd(x3, W, c, cos, sin)
    dx, G = oracle.layer_bwd(dxn[:n_pre].astype(np.float64)[None], W, cache, c, cos, sin)
    assert rel(xo[:n_pre] - x[:n_pre], (xn - x3)[0]) <= tol
    assert rel(dxi[:n_pre], dx[0]) <= tol
    worst = {tid: rel(grads[tid], G[tid]) for tid in G}
    assert max(worst.values()) <= tol, worst
    assert np.all(dxi[n_pre:] == 0.0)
    assert np.isfinite(xo).all()


def check_head_active(x, labels, gf, Wh, eps, loss, dx, dgf, dW, n_act, tol=2e-2):
    """x is zero outside its first n_act rows. loss, dx [T, d], dgf [d], dW
    [V, d] from the GPU; gf, Wh the bf16 final gain and head as fp64."""
    T, V = x.shape[0], Wh.shape[0]
    w = n_act / T
    l_a, dx_a, dgf_a, dW_a = oracle.head_ce_fwd_bwd(x[:n_act].astype(np.float64), gf, Wh, labels[:n_act], eps)
    assert abs(loss - (w * l_a + (1 - w) * math.log(V))) <= 1e-2, (loss, l_a)
    assert rel(dx[:n_act], w * dx_a) <= tol
    assert rel(dgf, w * dgf_a) <= tol
    assert rel(dW, w * dW_a) <= tol
    rows = np.unique(np.concatenate([np.random.default_rng(0).integers(n_act, T, 62), [n_act, T - 1]]))
    mean_row = Wh.mean(axis=0)
    ref = (mean_row[None] - Wh[labels[rows]]) / T * gf[None] / math.sqrt(eps)
    assert rel(dx[rows], ref) <= tol


# ----------------------------------------------------------------- GPU runs

def _mt():
    from host_memory_streamed_layer_b200 import mt
    return mt


def _one_layer(name):
    return {**synth.WORKLOADS[name], "L": 1}


@pytest.mark.parametrize("name", NAMES)
def test_attention_sampled_at_workload_shape(name):
    """Attention forward and backward on the tensor cores at the workload's
    batch, sequence length and head grouping (5 query heads per KV head at
    14B; 131072 keys at 128k)."""
    mt = _mt()
    sh = synth.WORKLOADS[name]
    B, S, H, Hkv = sh["b"], sh["s"], sh["H"], sh["Hkv"]
    T = B * S
    ld = (H + 2 * Hkv) * HD
    gen = torch.Generator(device=DEV).manual_seed(11)
    qkv = torch.randn(T, ld, device=DEV, generator=gen).to(torch.bfloat16)
    o = torch.empty(T, H * HD, device=DEV, dtype=torch.bfloat16)
    lse = torch.empty(B, H, S, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    p = qkv.data_ptr()
    pk, pv = p + 2 * H * HD, p + 2 * (H + Hkv) * HD
    mt.mt_k_attn_fwd_tc(p, pk, pv, ld, o.data_ptr(), H * HD, lse.data_ptr(), B, S, H, Hkv, HD, 0, err.data_ptr())
    do = torch.randn(T, H * HD, device=DEV, generator=gen).to(torch.bfloat16)
    dvec = torch.empty(B, H, S, device=DEV)
    dqa = torch.empty(T, H * HD, device=DEV)
    dqkv = torch.empty(T, ld, device=DEV, dtype=torch.bfloat16)
    dp = dqkv.data_ptr()
    mt.mt_k_attn_bwd_tc(p, pk, pv, ld, o.data_ptr(), do.data_ptr(), H * HD, lse.data_ptr(), dvec.data_ptr(),
                        dqa.data_ptr(), H * HD, dp, ld, dp + 2 * H * HD, dp + 2 * (H + Hkv) * HD, ld, B, S, H, Hkv,
                        HD, 0, 0, 0, err.data_ptr())
    torch.cuda.synchronize()
    assert err.item() == 0
    del dvec, dqa

    def split(t):  # [T, (H + 2 Hkv) hd] -> q, k, v views on the host
        a = t.view(B, S, H + 2 * Hkv, HD).float().cpu().numpy()
        return a[:, :, :H], a[:, :, H:H + Hkv], a[:, :, H + Hkv:]

    Q, K, V = split(qkv)
    DQ, DK, DV = split(dqkv)
    O = o.view(B, S, H, HD).float().cpu().numpy()
    DO = do.view(B, S, H, HD).float().cpu().numpy()
    LSE = lse.cpu().numpy()
    rng = np.random.default_rng(0)
    samples = [(0, 0, 0), (B - 1, H - 1, S - 1), (0, H // 2, S // 2 + 1)]
    samples += [(int(b), int(h), int(i)) for b, h, i in zip(rng.integers(0, B, 5), rng.integers(0, H, 5),
                                                             rng.integers(0, S, 5))]
    check_attention_rows(Q, K, V, O, LSE, DO, DQ, samples, H, Hkv)
    check_last_keys(Q, K, V, DO, DK, DV, B - 1, Hkv - 1, H, Hkv)


@pytest.mark.parametrize("name", NAMES)
def test_layer_prefix_parity_at_workload_shape(name):
    """mt_layer_fwd_bwd on all b x s tokens of the workload, upstream gradient
    on the first 1000 tokens of sequence 0 only (a ragged 128-row tile)."""
    from host_memory_streamed_layer_b200 import arena
    mt = _mt()
    sh = _one_layer(name)
    T, d = sh["b"] * sh["s"], sh["d"]
    n_pre = 1000
    cfg = arena.config(sh)
    cfg.seed = 5
    cfg.host_threads = 0
    ctx = mt.mt_create(cfg)
    try:
        P = np.empty(mt.mt_arena_bytes(cfg) // 4, dtype=np.float32)
        mt.mt_get_params(ctx, P.ctypes.data, P.nbytes)
        c = oracle.OracleConfig(**sh)
        shapes = {tid: shp for lay, tid, _, shp in oracle.arena_layout(c)[0] if lay == 0}
        W, spans = {}, {}
        for tid in range(9):
            o, k = mt.mt_tensor_offset(cfg, 0, tid)
            spans[tid] = (o, k)
            W[tid] = oracle.bf16_round(P[o:o + k]).astype(np.float64).reshape(shapes[tid])
        del P
        rng = np.random.default_rng(2)
        x = rng.normal(size=(T, d)).astype(np.float32)
        dxn = np.zeros((T, d), dtype=np.float32)
        dxn[:n_pre] = rng.normal(size=(n_pre, d))
        xo, dxi = np.empty_like(x), np.empty_like(x)
        off0 = spans[0][0]
        nblk = mt.mt_tensor_offset(cfg, -1, mt.MT_T_FINAL_NORM)[0] - off0
        g = np.empty(nblk, dtype=np.float32)
        mt.mt_layer_fwd_bwd(ctx, 0, x.ctypes.data, dxn.ctypes.data, xo.ctypes.data, dxi.ctypes.data, g.ctypes.data,
                            g.nbytes)
    finally:
        mt.mt_destroy(ctx)
    grads = {tid: g[o - off0:o - off0 + k].reshape(shapes[tid]) for tid, (o, k) in spans.items()}
    check_layer_prefix(sh, W, x, dxn, xo, dxi, grads, n_pre)


@pytest.mark.parametrize("name", NAMES)
def test_head_parity_at_workload_shape(name):
    """mt_head_fwd_bwd on all b x s tokens of the workload (the LM head in
    token chunks over the full vocabulary), hidden rows nonzero for the first
    1024 tokens only."""
    from host_memory_streamed_layer_b200 import arena
    mt = _mt()
    sh = _one_layer(name)
    T, d, V = sh["b"] * sh["s"], sh["d"], sh["V"]
    n_act = 1024
    cfg = arena.config(sh)
    cfg.seed = 9
    cfg.host_threads = 0
    ctx = mt.mt_create(cfg)
    try:
        fo, _ = mt.mt_tensor_offset(cfg, -1, mt.MT_T_FINAL_NORM)
        ho, hn = mt.mt_tensor_offset(cfg, -1, mt.MT_T_LM_HEAD)
        P = np.empty(mt.mt_arena_bytes(cfg) // 4, dtype=np.float32)
        mt.mt_get_params(ctx, P.ctypes.data, P.nbytes)
        gf = oracle.bf16_round(P[fo:fo + d]).astype(np.float64)
        Wh = oracle.bf16_round(P[ho:ho + hn]).astype(np.float64).reshape(V, d)
        del P
        x = np.zeros((T, d), dtype=np.float32)
        x[:n_act] = np.random.default_rng(3).normal(size=(n_act, d))
        _, lab = synth.tokens_labels(sh["b"], sh["s"], V, 4)
        labels = np.ascontiguousarray(lab.reshape(-1)).astype(np.int32)
        dx = np.empty_like(x)
        g = np.empty(ho + hn - fo, dtype=np.float32)
        loss = mt.mt_head_fwd_bwd(ctx, x.ctypes.data, labels.ctypes.data, dx.ctypes.data, g.ctypes.data, g.nbytes)
    finally:
        mt.mt_destroy(ctx)
    eps = oracle.OracleConfig(**sh).norm_eps
    check_head_active(x, labels, gf, Wh, eps, loss, dx, g[:d], g[ho - fo:].reshape(V, d), n_act)
