"""fp64 forward and backward of the Llama-style decoder trained by MegaTrain.

TEST INFRASTRUCTURE ONLY (see the package docstring). Plain numpy in float64.

Model, in the notation used throughout (weights stored [out, in]):
  x0       = E[tok]                                  embedding gather
  per layer:
    u      = RMSNorm(x) * g1
    q,k,v  = u Wq^T, u Wk^T, u Wv^T ; q,k <- RoPE(q), RoPE(k)
    a      = causal softmax(q k^T / sqrt(hd)) v      per head, GQA grouping
    h      = x + a Wo^T
    w      = RMSNorm(h) * g2
    x'     = h + (silu(w Wg^T) * (w Wu^T)) Wd^T
  n        = RMSNorm(x_L) * gf ;  z = n Whead^T
  loss     = mean_t [ logsumexp(z_t) - z_t[y_t] ]

The MegaTrain pages ("MegaTrain: Full Precision Training of 100B+ Parameter
Large Language Models on a Single GPU", abstract; saify.me, "The memory-centric
design") say which decoder families are trained but not their equations; the
block above is the plain pre-norm Llama reading, and each function names the
reading it takes.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

# Tensor ids of the arena layout (same numbering as the seeded input module,
# restated here so the oracle depends on nothing outside numpy).
ATTN_NORM, WQ, WK, WV, WO, MLP_NORM, WGATE, WUP, WDOWN = range(9)
ROUTER = 9  # mixture-of-experts layers only
EMBED, FINAL_NORM, LM_HEAD = 100, 101, 102

ALIGN_FLOATS = 64  # every tensor of the fp32 arena starts on a 256-byte boundary


@dataclass(frozen=True)
class OracleConfig:
    L: int
    d: int
    H: int
    Hkv: int
    F: int
    V: int
    b: int
    s: int
    norm_eps: float = 1e-5
    rope_base: float = 10000.0
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.95
    adam_eps: float = 1e-8
    wd: float = 0.1
    # Tied embeddings (one of the decoder variants the pages list as
    # supported: saify.me, "Who this is actually for"): the LM head is the
    # embedding table itself, z = n E^T, so E's gradient is the sum of the
    # gather's and the head's; the arena has no separate LM-head tensor.
    tied: bool = False
    # Mixture-of-experts MLP (another of the families the pages list as
    # supported, saify.me, "Who this is actually for", with no routing rule
    # given): E experts of SwiGLU width F per layer and top-k routing, the
    # plainest reading (moe_fwd below). E = 0: the dense SwiGLU MLP.
    E: int = 0
    topk: int = 2

    @property
    def hd(self) -> int:
        return self.d // self.H

    @property
    def layer_tids(self):
        return list(range(10 if self.E else 9))


# ---------------------------------------------------------------------------
# Host arena layout: the flat fp32 master-parameter array the caller owns.
# ---------------------------------------------------------------------------

def _layer_tensors(c: OracleConfig):
    hd = c.hd
    return [
        (ATTN_NORM, (c.d,)),
        (WQ, (c.H * hd, c.d)),
        (WK, (c.Hkv * hd, c.d)),
        (WV, (c.Hkv * hd, c.d)),
        (WO, (c.d, c.H * hd)),
        (MLP_NORM, (c.d,)),
    ] + ([
        (WGATE, (c.F, c.d)),
        (WUP, (c.F, c.d)),
        (WDOWN, (c.d, c.F)),
    ] if not c.E else [
        (WGATE, (c.E, c.F, c.d)),  # expert e's gate rows at [e]
        (WUP, (c.E, c.F, c.d)),
        (WDOWN, (c.E, c.d, c.F)),
        (ROUTER, (c.E, c.d)),
    ])


def arena_layout(c: OracleConfig):
    """List of (layer, tensor id, offset in floats, shape) in arena order:
    embedding, then each layer's nine tensors, then the final norm and the
    untied LM head (none when tied). Offsets are rounded up to 64 floats (256
    bytes)."""
    out = []
    off = 0

    def put(layer, tid, shape):
        nonlocal off
        out.append((layer, tid, off, shape))
        n = int(np.prod(shape))
        off += (n + ALIGN_FLOATS - 1) // ALIGN_FLOATS * ALIGN_FLOATS

    put(-1, EMBED, (c.V, c.d))
    for l in range(c.L):
        for tid, shape in _layer_tensors(c):
            put(l, tid, shape)
    put(-1, FINAL_NORM, (c.d,))
    if not c.tied:
        put(-1, LM_HEAD, (c.V, c.d))
    return out, off


def arena_floats(c: OracleConfig) -> int:
    return arena_layout(c)[1]


def unpack_arena(arena: np.ndarray, c: OracleConfig, dtype=np.float64) -> dict:
    """Views of the arena as a dict keyed by (layer, tensor id), cast to dtype."""
    layout, total = arena_layout(c)
    assert arena.size >= total, (arena.size, total)
    out = {}
    for layer, tid, off, shape in layout:
        n = int(np.prod(shape))
        out[(layer, tid)] = arena[off:off + n].reshape(shape).astype(dtype)
    return out


def pack_arena(tensors: dict, c: OracleConfig) -> np.ndarray:
    """Inverse of unpack_arena (padding left at zero), as fp32."""
    layout, total = arena_layout(c)
    arena = np.zeros(total, dtype=np.float32)
    for layer, tid, off, shape in layout:
        t = np.asarray(tensors[(layer, tid)], dtype=np.float32).reshape(-1)
        arena[off:off + t.size] = t
    return arena


# ---------------------------------------------------------------------------
# bf16 round-to-nearest-even (the streamed copy of the master weights).
# ---------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round fp32 values to the nearest bfloat16 (ties to even), returned as
    float64. bfloat16 keeps the top 16 bits of the IEEE binary32 pattern, so
    the value is the binary32 pattern with the low 16 bits cleared after
    adding half an ulp (0x7fff plus the kept lsb). NaN stays NaN."""
    f = np.asarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    out = (rounded & 0xFFFFFFFF).astype(np.uint32).view(np.float32).astype(np.float64)
    return np.where(np.isnan(f), np.nan, out)


# ---------------------------------------------------------------------------
# RMSNorm. Reading: y = x / sqrt(mean(x^2) + eps) * g, eps inside the root.
# ---------------------------------------------------------------------------

def rmsnorm_fwd(x: np.ndarray, g: np.ndarray, eps: float):
    """Returns (y, r) with r = 1/sqrt(mean(x^2, last axis) + eps)."""
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * g, r


def rmsnorm_bwd(x: np.ndarray, g: np.ndarray, r: np.ndarray, dy: np.ndarray):
    """Gradient of y_i = g_i x_i r with r = (sum_j x_j^2 / d + eps)^(-1/2).
    dr/dx_j = -r^3 x_j / d, hence
      dx_j = r g_j dy_j - (r^3 x_j / d) sum_i g_i dy_i x_i,
      dg_i = sum over rows of dy_i x_i r.
    Returns (dx, dg)."""
    d = x.shape[-1]
    gdy = g * dy
    dot = np.sum(gdy * x, axis=-1, keepdims=True)
    dx = r * gdy - (r ** 3) * x * dot / d
    dg = np.sum((dy * x * r).reshape(-1, d), axis=0)
    return dx, dg


# ---------------------------------------------------------------------------
# RoPE. Reading: rotate-half pairing (i, i + hd/2), theta_i = base^(-2i/hd),
# positions 0..s-1 restarting for every sequence.
# ---------------------------------------------------------------------------

def rope_tables(s: int, hd: int, base: float):
    """cos and sin tables of shape [s, hd/2]: angle[p, i] = p * base^(-2i/hd)."""
    i = np.arange(hd // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / hd)
    ang = np.arange(s, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def rope_fwd(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """x: [b, s, heads, hd]. Rotates each pair (x_i, x_{i+hd/2}) by angle[p, i]:
      x'_i        = x_i cos - x_{i+hd/2} sin
      x'_{i+hd/2} = x_{i+hd/2} cos + x_i sin"""
    half = x.shape[-1] // 2
    c = cos[None, :, None, :]
    s = sin[None, :, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_bwd(dy: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Transpose of the rotation (rotation by -angle)."""
    half = dy.shape[-1] // 2
    c = cos[None, :, None, :]
    s = sin[None, :, None, :]
    d1, d2 = dy[..., :half], dy[..., half:]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


# ---------------------------------------------------------------------------
# Causal attention with grouped KV heads. Reading: scale 1/sqrt(hd), key j is
# visible to query i iff j <= i (same sequence); query head h reads KV head
# floor(h / (H / Hkv)). The query rows may be a block of the sequence: rows at
# positions q_offset .. q_offset + r - 1 against keys 0 .. s_k - 1 (the same
# visibility rule, so a long sequence can be checked a few rows at a time).
# ---------------------------------------------------------------------------

def _heads_first(x):
    """[b, s, heads, hd] -> [b, heads, s, hd] (a view)."""
    return x.transpose(0, 2, 1, 3)


def _visible_scores(q, k, q_offset=0):
    """Scaled scores q_i . k_j / sqrt(hd) per query head, -inf where key j comes
    after query i. q: [b, r, H, hd], row i at position q_offset + i;
    k: [b, s_k, Hkv, hd] from position 0. Returns [b, H, r, s_k]."""
    b, r, H, hd = q.shape
    sk = k.shape[1]
    kk = np.repeat(k, H // k.shape[2], axis=2)  # kv head for query head h is h // group
    S = _heads_first(q) @ _heads_first(kk).transpose(0, 1, 3, 2) / np.sqrt(hd)
    mask = np.arange(sk)[None, :] <= (q_offset + np.arange(r))[:, None]
    return np.where(mask[None, None], S, -np.inf)


def attention_fwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_offset: int = 0):
    """q: [b, r, H, hd] (rows at positions q_offset ..); k, v: [b, s_k, Hkv, hd].
    Returns (o [b,r,H,hd], P [b,H,r,s_k]); r = s_k and q_offset = 0 is the
    whole sequence."""
    H = q.shape[2]
    vv = np.repeat(v, H // v.shape[2], axis=2)
    S = _visible_scores(q, k, q_offset)
    S = S - S.max(axis=-1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=-1, keepdims=True)
    o = _heads_first(P @ _heads_first(vv))
    return o, P


def attention_lse(q: np.ndarray, k: np.ndarray, q_offset: int = 0) -> np.ndarray:
    """Natural log-sum-exp over visible keys of the scaled scores, [b, H, r]:
    lse[b, h, i] = log sum_{j <= q_offset + i} exp(q_i . k_j / sqrt(hd))."""
    S = _visible_scores(q, k, q_offset)
    m = S.max(axis=-1, keepdims=True)
    return m[..., 0] + np.log(np.sum(np.exp(S - m), axis=-1))


def attention_bwd(q, k, v, P, do):
    """Backward of o = P v with P = softmax(q k^T / sqrt(hd)) (causal):
      dP = do v^T ; dv = P^T do ; dS = P * (dP - rowsum(dP * P)) ;
      dq = dS k / sqrt(hd) ; dk = dS^T q / sqrt(hd);
    dk, dv of a KV head sum over the query heads of its group. With a block of
    query rows (P from attention_fwd with q_offset), dk and dv [b, s_k, ...]
    are those rows' contributions."""
    b, r, H, hd = q.shape
    sk = k.shape[1]
    Hkv = k.shape[2]
    group = H // Hkv
    kh = _heads_first(np.repeat(k, group, axis=2))
    vh = _heads_first(np.repeat(v, group, axis=2))
    doh = _heads_first(do)
    dP = doh @ vh.transpose(0, 1, 3, 2)
    dvv = _heads_first(P.transpose(0, 1, 3, 2) @ doh)
    dS = P * (dP - np.sum(dP * P, axis=-1, keepdims=True))
    scale = 1.0 / np.sqrt(hd)
    dq = _heads_first(dS @ kh) * scale
    dkk = _heads_first(dS.transpose(0, 1, 3, 2) @ _heads_first(q)) * scale
    dk = dkk.reshape(b, sk, Hkv, group, hd).sum(axis=3)
    dv = dvv.reshape(b, sk, Hkv, group, hd).sum(axis=3)
    return dq, dk, dv


# ---------------------------------------------------------------------------
# SwiGLU. Reading: act = silu(gate) * up, silu(z) = z * sigmoid(z).
# ---------------------------------------------------------------------------

def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    return z * _sigmoid(z)


def swiglu_fwd(gt, up):
    return silu(gt) * up


def swiglu_bwd(gt, up, dact):
    """d/dz silu(z) = sigmoid(z) (1 + z (1 - sigmoid(z)))."""
    sg = _sigmoid(gt)
    dgt = dact * up * sg * (1.0 + gt * (1.0 - sg))
    dup = dact * gt * sg
    return dgt, dup


# ---------------------------------------------------------------------------
# Mixture-of-experts MLP. Reading (the pages name MoE variants but no rule):
#   logits = w Wr^T                      [T, E]
#   R_t    = the k experts with the largest logits (ties: lower index first)
#   g_t    = softmax of logits_t over R_t (the gates sum to 1)
#   y_t    = sum_{e in R_t} g_te * SwiGLU_e(w_t),
#            SwiGLU_e(w) = (silu(w Wg_e^T) * (w Wu_e^T)) Wd_e^T
# Every routed token is computed (no capacity limit, none dropped) and the
# loss has no auxiliary balancing term: the pages state neither.
# ---------------------------------------------------------------------------

def moe_route(w: np.ndarray, Wr: np.ndarray, k: int):
    """Router of moe_fwd. w: [T, d]. Returns (logits [T, E], idx [T, k] of the
    k largest logits per row, largest first, ties to the lower index)."""
    logits = w @ Wr.T
    idx = np.argsort(-logits, axis=-1, kind="stable")[:, :k]
    return logits, idx


def moe_gates(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Softmax of each row's selected logits: g [T, k]."""
    sel = np.take_along_axis(logits, idx, axis=-1)
    sel = sel - sel.max(axis=-1, keepdims=True)
    e = np.exp(sel)
    return e / e.sum(axis=-1, keepdims=True)


def moe_fwd(w: np.ndarray, Wr, Wg, Wu, Wd, k: int, idx=None):
    """w: [T, d]; Wr [E, d], Wg/Wu [E, F, d], Wd [E, d, F]. idx: a given
    routing (e.g. one a GPU took where two logits were within rounding of
    each other), else the router's. Returns (y [T, d], cache)."""
    logits, r_idx = moe_route(w, Wr, k)
    if idx is None:
        idx = r_idx
    g = moe_gates(logits, idx)
    T, d = w.shape
    E = Wr.shape[0]
    y = np.zeros((T, d))
    ye = np.zeros(idx.shape + (d,))  # each routed token's expert output, before its gate
    parts = {}
    for e in range(E):
        t, j = np.nonzero(idx == e)
        if t.size == 0:
            continue
        we = w[t]
        gt = we @ Wg[e].T
        up = we @ Wu[e].T
        act = swiglu_fwd(gt, up)
        out = act @ Wd[e].T
        ye[t, j] = out
        parts[e] = (t, j, gt, up, act)
    for j in range(idx.shape[1]):  # fixed order over the k slots
        y += g[:, j:j + 1] * ye[:, j]
    return y, dict(w=w, logits=logits, idx=idx, g=g, ye=ye, parts=parts)


def moe_bwd(dy: np.ndarray, Wr, Wg, Wu, Wd, cache: dict):
    """Backward of moe_fwd for a fixed routing. Returns (dw [T, d], dWr, dWg,
    dWu, dWd):
      dg_tj   = dy_t . ye_tj ;  dlogit_te = g_te (dg_te - sum_j g_tj dg_tj), e in R_t
      expert e, over its tokens: dye = g dy ; dWd_e = dye^T act ; dact = dye Wd_e ;
      (dgt, dup) = SwiGLU backward ; dWg_e = dgt^T w ; dWu_e = dup^T w ;
      dw += dgt Wg_e + dup Wu_e ;  router: dWr = dlogit^T w, dw += dlogit Wr."""
    w, logits, idx, g, ye, parts = (cache[k] for k in ("w", "logits", "idx", "g", "ye", "parts"))
    T, d = w.shape
    E = Wr.shape[0]
    dg = np.einsum("td,tjd->tj", dy, ye)
    dsel = g * (dg - np.sum(g * dg, axis=-1, keepdims=True))
    dlogits = np.zeros_like(logits)
    np.put_along_axis(dlogits, idx, dsel, axis=-1)
    dWr = dlogits.T @ w
    dw = dlogits @ Wr
    dWg, dWu, dWd = np.zeros_like(Wg), np.zeros_like(Wu), np.zeros_like(Wd)
    for e, (t, j, gt, up, act) in parts.items():
        dye = g[t, j][:, None] * dy[t]
        dWd[e] = dye.T @ act
        dact = dye @ Wd[e]
        dgt, dup = swiglu_bwd(gt, up, dact)
        dWg[e] = dgt.T @ w[t]
        dWu[e] = dup.T @ w[t]
        np.add.at(dw, t, dgt @ Wg[e] + dup @ Wu[e])
    return dw, dWr, dWg, dWu, dWd


# ---------------------------------------------------------------------------
# One decoder layer.
# ---------------------------------------------------------------------------

def layer_fwd(x: np.ndarray, W: dict, c: OracleConfig, cos, sin, routing=None):
    """x: [b, s, d] -> (x_next, cache). W keys: ATTN_NORM, WQ, ..., WDOWN (and
    ROUTER with experts; routing: a given [b*s, k] expert choice)."""
    b, s, d = x.shape
    hd = c.hd
    u, r1 = rmsnorm_fwd(x, W[ATTN_NORM], c.norm_eps)
    q = (u @ W[WQ].T).reshape(b, s, c.H, hd)
    k = (u @ W[WK].T).reshape(b, s, c.Hkv, hd)
    v = (u @ W[WV].T).reshape(b, s, c.Hkv, hd)
    qr = rope_fwd(q, cos, sin)
    kr = rope_fwd(k, cos, sin)
    o, P = attention_fwd(qr, kr, v)
    a = o.reshape(b, s, c.H * hd)
    h = x + a @ W[WO].T
    w, r2 = rmsnorm_fwd(h, W[MLP_NORM], c.norm_eps)
    cache = dict(x=x, u=u, r1=r1, qr=qr, kr=kr, v=v, P=P, a=a, h=h, w=w, r2=r2)
    if c.E:
        y, cache["moe"] = moe_fwd(w.reshape(b * s, d), W[ROUTER], W[WGATE], W[WUP], W[WDOWN], c.topk,
                                  idx=routing)
        return h + y.reshape(b, s, d), cache
    gt = w @ W[WGATE].T
    up = w @ W[WUP].T
    act = swiglu_fwd(gt, up)
    x_next = h + act @ W[WDOWN].T
    cache.update(gt=gt, up=up, act=act)
    return x_next, cache


def layer_bwd(dxn: np.ndarray, W: dict, cache: dict, c: OracleConfig, cos, sin):
    """Gradient of a layer given dL/dx_next. Returns (dx, dW dict)."""
    b, s, d = dxn.shape
    hd = c.hd
    T = b * s
    x, u, h, w, a = (cache[k] for k in ("x", "u", "h", "w", "a"))
    G = {}
    if c.E:
        dwf, G[ROUTER], G[WGATE], G[WUP], G[WDOWN] = moe_bwd(dxn.reshape(T, d), W[ROUTER], W[WGATE], W[WUP],
                                                             W[WDOWN], cache["moe"])
        dw = dwf.reshape(b, s, d)
    else:
        act = cache["act"]
        # x' = h + act Wd^T
        G[WDOWN] = dxn.reshape(T, d).T @ act.reshape(T, c.F)
        dact = dxn @ W[WDOWN]
        dgt, dup = swiglu_bwd(cache["gt"], cache["up"], dact)
        G[WGATE] = dgt.reshape(T, c.F).T @ w.reshape(T, d)
        G[WUP] = dup.reshape(T, c.F).T @ w.reshape(T, d)
        dw = dgt @ W[WGATE] + dup @ W[WUP]
    dh_norm, G[MLP_NORM] = rmsnorm_bwd(h, W[MLP_NORM], cache["r2"], dw)
    dh = dxn + dh_norm
    # h = x + a Wo^T
    G[WO] = dh.reshape(T, d).T @ a.reshape(T, c.H * hd)
    da = (dh @ W[WO]).reshape(b, s, c.H, hd)
    dqr, dkr, dv = attention_bwd(cache["qr"], cache["kr"], cache["v"], cache["P"], da)
    dq = rope_bwd(dqr, cos, sin).reshape(T, c.H * hd)
    dk = rope_bwd(dkr, cos, sin).reshape(T, c.Hkv * hd)
    dv = dv.reshape(T, c.Hkv * hd)
    uf = u.reshape(T, d)
    G[WQ] = dq.T @ uf
    G[WK] = dk.T @ uf
    G[WV] = dv.T @ uf
    du = (dq @ W[WQ] + dk @ W[WK] + dv @ W[WV]).reshape(b, s, d)
    dx_norm, G[ATTN_NORM] = rmsnorm_bwd(x, W[ATTN_NORM], cache["r1"], du)
    return dh + dx_norm, G


# ---------------------------------------------------------------------------
# Head: final norm, untied LM head, mean next-token cross-entropy.
# ---------------------------------------------------------------------------

def softmax_ce(z, labels):
    """Per-row cross-entropy of logits z [T, V] against integer labels:
      loss_t = logsumexp(z_t) - z_t[y_t];  g_t = softmax(z_t) - onehot(y_t).
    Returns (loss_t [T], g [T, V])."""
    T = z.shape[0]
    zmax = z.max(axis=-1, keepdims=True)
    lse = zmax[:, 0] + np.log(np.sum(np.exp(z - zmax), axis=-1))
    idx = np.arange(T)
    loss_t = lse - z[idx, labels]
    g = np.exp(z - lse[:, None])
    g[idx, labels] -= 1.0
    return loss_t, g


def head_ce_fwd_bwd(xL, gf, Whead, labels, eps):
    """xL: [T, d]; labels: [T] ints. Returns (loss, dxL, dgf, dWhead) with
      z = RMSNorm(xL) gf Whead^T, loss = mean_t(logsumexp(z_t) - z_t[y_t]),
      dz = (softmax(z) - onehot(y)) / T."""
    T = xL.shape[0]
    n, r = rmsnorm_fwd(xL, gf, eps)
    z = n @ Whead.T
    loss_t, g = softmax_ce(z, labels)
    loss = float(np.mean(loss_t))
    dz = g / T
    dWhead = dz.T @ n
    dn = dz @ Whead
    dxL, dgf = rmsnorm_bwd(xL, gf, r, dn)
    return loss, dxL, dgf, dWhead


# ---------------------------------------------------------------------------
# Whole training step (loss and gradients; the update is in adamw.py).
# ---------------------------------------------------------------------------

def train_step_grads(weights: dict, tokens: np.ndarray, labels: np.ndarray,
                     c: OracleConfig, routing=None, logits_out=None):
    """weights: dict (layer, tensor id) -> float64 array, the values the forward
    and backward use. tokens, labels: int [b, s]. routing: optional dict
    layer -> [b*s, k] expert choice (mixture-of-experts layers), else each
    router's own; logits_out: optional dict that receives each expert layer's
    router logits [b*s, E]. Returns (loss, grads dict)."""
    b, s = tokens.shape
    T = b * s
    cos, sin = rope_tables(s, c.hd, c.rope_base)
    E = weights[(-1, EMBED)]
    x = E[tokens]  # [b, s, d]
    caches = []
    for l in range(c.L):
        W = {tid: weights[(l, tid)] for tid in c.layer_tids}
        x, cache = layer_fwd(x, W, c, cos, sin, routing=(routing or {}).get(l))
        caches.append(cache)
        if c.E and logits_out is not None:
            logits_out[l] = cache["moe"]["logits"]
    Whead = E if c.tied else weights[(-1, LM_HEAD)]
    loss, dx, dgf, dWhead = head_ce_fwd_bwd(
        x.reshape(T, c.d), weights[(-1, FINAL_NORM)], Whead, labels.reshape(T), c.norm_eps)
    grads = {(-1, FINAL_NORM): dgf}
    if not c.tied:
        grads[(-1, LM_HEAD)] = dWhead
    dx = dx.reshape(b, s, c.d)
    for l in reversed(range(c.L)):
        W = {tid: weights[(l, tid)] for tid in c.layer_tids}
        dx, G = layer_bwd(dx, W, caches[l], c, cos, sin)
        for tid, g in G.items():
            grads[(l, tid)] = g
    dE = dWhead.copy() if c.tied else np.zeros_like(E)  # tied: the head's share of E's gradient
    np.add.at(dE, tokens.reshape(T), dx.reshape(T, c.d))
    grads[(-1, EMBED)] = dE
    return loss, grads
