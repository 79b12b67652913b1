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

