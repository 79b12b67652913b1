"""Shared check of one decoder layer run through mt_layer_fwd_bwd against the
oracle's layer forward and backward (used by the GPU parity tests)."""
import numpy as np

import oracle


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def layer_check(mt, ctx, cfg, shape, layer, W, x, dxn, seqs, tol=2e-2):
    """Runs mt_layer_fwd_bwd on x, dxn ([b*s, d] fp32) and compares sequences
    `seqs` with the oracle's layer forward and backward on bf16 weights W."""
    b, s, d = shape["b"], shape["s"], shape["d"]
    c = oracle.OracleConfig(**shape)
    off0, _ = mt.mt_tensor_offset(cfg, layer, mt.MT_T_ATTN_NORM)
    if layer + 1 < shape["L"]:
        nblk = mt.mt_tensor_offset(cfg, layer + 1, mt.MT_T_ATTN_NORM)[0] - off0
    else:
        nblk = mt.mt_tensor_offset(cfg, -1, mt.MT_T_FINAL_NORM)[0] - off0
    xo = np.empty_like(x)
    dxi = np.empty_like(x)
    g = np.empty(nblk, dtype=np.float32)
    mt.mt_layer_fwd_bwd(ctx, layer, x.ctypes.data, dxn.ctypes.data, xo.ctypes.data, dxi.ctypes.data, g.ctypes.data,
                        g.nbytes)
    sel = np.asarray(seqs)
    cos, sin = oracle.rope_tables(s, c.hd, c.rope_base)
    x3 = x.reshape(b, s, d)[sel].astype(np.float64)
    xn, cache = oracle.layer_fwd(x3, W, c, cos, sin)
    dx, G = oracle.layer_bwd(dxn.reshape(b, s, d)[sel].astype(np.float64), W, cache, c, cos, sin)
    # the layer's own contribution (attention + MLP) next to the residual
    assert rel(xo.reshape(b, s, d)[sel] - x3, xn - x3) <= tol
    assert rel(dxi.reshape(b, s, d)[sel], dx) <= tol
    worst = {}
    for tid in range(9):
        o, n = mt.mt_tensor_offset(cfg, layer, tid)
        got = g[o - off0:o - off0 + n].reshape(G[tid].shape)
        worst[tid] = rel(got, G[tid])
    assert max(worst.values()) <= tol, worst
    return xo, dxi, g



def head_check(mt, ctx, cfg, shape, x, labels, chunk=None, tol=2e-2):
    """Runs mt_head_fwd_bwd on x ([b*s, d] fp32) and labels and compares the
    loss, dx_L and the final-gain and LM-head gradients with the oracle's head
    on the bf16 streamed weights, token-chunked (each chunk's mean loss and
    gradients rescaled to the mean over all tokens)."""
    T, d, V = shape["b"] * shape["s"], shape["d"], shape["V"]
    n = mt.mt_arena_bytes(cfg) // 4
    P = np.empty(n, dtype=np.float32)
    mt.mt_get_params(ctx, P.ctypes.data, P.nbytes)
    fo, _ = mt.mt_tensor_offset(cfg, -1, mt.MT_T_FINAL_NORM)
    ho, hn = mt.mt_tensor_offset(cfg, -1, mt.MT_T_LM_HEAD)
    gf = oracle.bf16_round(P[fo:fo + d]).astype(np.float64)
    Wh = oracle.bf16_round(P[ho:ho + hn]).astype(np.float64).reshape(V, d)
    del P
    dx = np.empty_like(x)
    g = np.empty(ho + hn - fo, dtype=np.float32)
    loss = mt.mt_head_fwd_bwd(ctx, x.ctypes.data, labels.ctypes.data, dx.ctypes.data, g.ctypes.data, g.nbytes)
    chunk = chunk or T
    rl, rdx, rdgf, rdW = 0.0, np.empty((T, d)), np.zeros(d), np.zeros((V, d))
    eps = oracle.OracleConfig(**shape).norm_eps
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        w = (t1 - t0) / T
        l_c, dx_c, dgf_c, dW_c = oracle.head_ce_fwd_bwd(x[t0:t1].astype(np.float64), gf, Wh, labels[t0:t1], eps)
        rl += w * l_c
        rdx[t0:t1] = w * dx_c
        rdgf += w * dgf_c
        rdW += w * dW_c
    assert abs(loss - rl) <= 1e-2, (loss, rl)
    assert rel(dx, rdx) <= tol
    assert rel(g[:d], rdgf) <= tol
    assert rel(g[ho - fo:].reshape(V, d), rdW) <= tol
    return loss
