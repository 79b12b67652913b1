"""Pins the oracle's hand-written backward against central finite differences
of its own forward in fp64 (the gradient is the derivative of the loss; a
dropped term, wrong sign or transposed operand anywhere in the backward makes
some entry disagree). Small shapes keep it fast; GQA (H != Hkv), an odd FFN
width and several layers are covered."""
import numpy as np
import pytest

import oracle
from oracle.model import (ATTN_NORM, EMBED, FINAL_NORM, LM_HEAD, MLP_NORM)

SMALL = oracle.OracleConfig(L=2, d=32, H=4, Hkv=2, F=40, V=50, b=2, s=8)


def _weights(c, seed):
    rng = np.random.default_rng(seed)
    W = {(-1, EMBED): rng.normal(0, 0.5, (c.V, c.d))}
    for l in range(c.L):
        for tid, shape in oracle.model._layer_tensors(c):
            if tid in (ATTN_NORM, MLP_NORM):
                W[(l, tid)] = 1.0 + rng.normal(0, 0.3, shape)
            else:
                W[(l, tid)] = rng.normal(0, 0.3, shape)
    W[(-1, FINAL_NORM)] = 1.0 + rng.normal(0, 0.3, (c.d,))
    W[(-1, LM_HEAD)] = rng.normal(0, 0.3, (c.V, c.d))
    return W


def _fd5(W, flat, i, h, tok, lab, c):
    """Fourth-order central difference (-f(+2h) + 8f(+h) - 8f(-h) + f(-2h)) / 12h."""
    old = flat[i]
    vals = []
    for k in (2, 1, -1, -2):
        flat[i] = old + k * h
        vals.append(_loss(W, tok, lab, c))
    flat[i] = old
    return (-vals[0] + 8 * vals[1] - 8 * vals[2] + vals[3]) / (12 * h)


def _loss(W, tok, lab, c):
    loss, _ = _forward_only(W, tok, lab, c)
    return loss


def _forward_only(W, tok, lab, c):
    return oracle.train_step_grads(W, tok, lab, c)


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_matches_central_differences(seed):
    c = SMALL
    W = _weights(c, seed)
    rng = np.random.default_rng(100 + seed)
    tok = rng.integers(0, c.V, (c.b, c.s))
    lab = rng.integers(0, c.V, (c.b, c.s))
    # Repeated tokens exercise the embedding scatter-add.
    tok[1, :3] = tok[0, 0]
    _, G = oracle.train_step_grads(W, tok, lab, c)
    h = 1e-4
    checked = 0
    for key in W:
        p = W[key]
        flat = p.reshape(-1)
        n = flat.size
        if key[1] == EMBED:
            # rows that appear in the batch, plus one that does not
            used = np.unique(tok)
            unused = np.setdiff1d(np.arange(c.V), used)[:1]
            rows = np.concatenate([used[:6], unused])
            idx = np.array([r * c.d + j for r in rows for j in rng.choice(c.d, 3, replace=False)])
        elif p.ndim == 1 and key[0] == 0:
            idx = np.arange(n)  # every gain entry of layer 0
        else:
            idx = rng.choice(n, min(16, n), replace=False)
        for i in idx:
            fd = _fd5(W, flat, i, h, tok, lab, c)
            an = G[key].reshape(-1)[i]
            scale = max(abs(fd), 1e-3 * np.abs(G[key]).max(), 1e-9)
            assert abs(fd - an) <= 1e-6 * scale + 1e-10, (key, i, fd, an)
            checked += 1
    assert checked > 200


def test_fd_on_tiny_workload_shape():
    """A few entries per tensor at the tiny workload's own shape (head_dim 64,
    FFN 688) so the shapes the GPU path runs are covered too."""
    import synth
    cfg = synth.WORKLOADS["tiny"]
    c = oracle.OracleConfig(**cfg)
    c = oracle.OracleConfig(**{**cfg, "b": 1, "s": 16, "L": 1})
    W = {k: v.astype(np.float64) for k, v in synth.init_weights(
        {**cfg, "L": 1}, 3).items()}
    rng = np.random.default_rng(7)
    tok = rng.integers(0, c.V, (c.b, c.s))
    lab = rng.integers(0, c.V, (c.b, c.s))
    _, G = oracle.train_step_grads(W, tok, lab, c)
    h = 1e-4
    for key in W:
        flat = W[key].reshape(-1)
        if key[1] == EMBED:
            cand = np.array([tok[0, 0] * c.d + j for j in range(3)])
        else:
            cand = rng.choice(flat.size, 3, replace=False)
        for i in cand:
            fd = _fd5(W, flat, i, h, tok, lab, c)
            an = G[key].reshape(-1)[i]
            scale = max(abs(fd), 1e-2 * np.abs(G[key]).max(), 1e-12)
            assert abs(fd - an) <= 1e-6 * scale, (key, i, fd, an)


def test_tied_embeddings_match_central_differences():
    """Tied embeddings: the LM head is the embedding table, so the derivative
    of the loss with respect to one table entry covers both uses (gather and
    head). Rows the batch does not gather still get the head's share."""
    c = oracle.OracleConfig(L=1, d=32, H=4, Hkv=2, F=40, V=50, b=2, s=8, tied=True)
    W = _weights(c, 3)
    del W[(-1, LM_HEAD)]
    rng = np.random.default_rng(11)
    tok = rng.integers(0, c.V, (c.b, c.s))
    lab = rng.integers(0, c.V, (c.b, c.s))
    tok[1, :3] = tok[0, 0]
    _, G = oracle.train_step_grads(W, tok, lab, c)
    assert (-1, LM_HEAD) not in G
    used = np.unique(tok)
    unused = np.setdiff1d(np.arange(c.V), used)[:4]
    flat = W[(-1, EMBED)].reshape(-1)
    rows = np.concatenate([used[:5], unused])
    h = 1e-4
    for r in rows:
        for j in rng.choice(c.d, 4, replace=False):
            i = r * c.d + j
            fd = _fd5(W, flat, i, h, tok, lab, c)
            an = G[(-1, EMBED)].reshape(-1)[i]
            scale = max(abs(fd), 1e-3 * np.abs(G[(-1, EMBED)]).max(), 1e-9)
            assert abs(fd - an) <= 1e-6 * scale + 1e-10, (r, j, fd, an)
