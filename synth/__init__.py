"""Seeded synthetic inputs for the streamed-layer training step.

This module is shared by the oracle side and the CUDA side of the tests and the
benchmark. It holds no arithmetic of the training method: it only names the
workload shapes, draws token streams and draws initial weights. Every tensor is
drawn from its own counter-keyed PCG64 stream, keyed by (seed, layer, tensor
id), so the order in which a caller asks for tensors does not matter.

Workload shapes are those of the MegaTrain write-ups' model families (a
Llama-style decoder, see "MegaTrain: Full Precision Training of 100B+ Parameter
Large Language Models on a Single GPU", abstract); sizes are the ones this
repository benchmarks.
"""
from __future__ import annotations

import numpy as np

# name -> decoder shape and batch. L layers, d model width, H query heads,
# Hkv key/value heads, F SwiGLU hidden width, V vocabulary, b sequences of s tokens.
WORKLOADS = {
    "tiny": dict(L=2, d=256, H=4, Hkv=4, F=688, V=1024, b=2, s=128),
    "llama-1.3b": dict(L=24, d=2048, H=16, Hkv=16, F=5504, V=32000, b=8, s=2048),
    "llama-7b": dict(L=32, d=4096, H=32, Hkv=32, F=11008, V=32000, b=4, s=4096),
    "gqa-14b": dict(L=40, d=5120, H=40, Hkv=8, F=13824, V=152064, b=2, s=4096),
    "llama-7b-128k": dict(L=32, d=4096, H=32, Hkv=32, F=11008, V=32000, b=1, s=131072),
    # mixture-of-experts decoder: 8 experts of SwiGLU width 1408, top-2 routing
    # (2.2 B parameters, about 0.9 B active per token)
    "moe-8x1408": dict(L=24, d=2048, H=16, Hkv=16, F=1408, V=32000, b=8, s=2048, E=8, topk=2),
}

# Hyper-parameters shared by every workload.
HYPER = dict(norm_eps=1e-5, rope_base=10000.0, lr=1e-3, beta1=0.9, beta2=0.95,
             adam_eps=1e-8, wd=0.1)

# Tensor ids used to key the weight streams. Per decoder layer:
ATTN_NORM, WQ, WK, WV, WO, MLP_NORM, WGATE, WUP, WDOWN = range(9)
ROUTER = 9  # mixture-of-experts layers
# Model-level tensors use layer = -1:
EMBED, FINAL_NORM, LM_HEAD = 100, 101, 102

INIT_STD = 0.02


def _stream(seed: int, layer: int, tid: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(layer) + 8, int(tid)]))


def tokens_labels(b: int, s: int, V: int, seed: int, step: int = 0):
    """Uniform next-token data: draw b x (s+1) ids in [0, V), tokens are the
    first s of each row and labels the last s. Returns two int32 [b, s] arrays."""
    rng = _stream(seed, -2, 1000 + step)
    seq = rng.integers(0, V, size=(b, s + 1), dtype=np.int64)
    return (np.ascontiguousarray(seq[:, :-1], dtype=np.int32),
            np.ascontiguousarray(seq[:, 1:], dtype=np.int32))


def init_tensor(seed: int, layer: int, tid: int, shape) -> np.ndarray:
    """fp32 initial value of one tensor: gains are ones, matrices N(0, 0.02^2)."""
    if tid in (ATTN_NORM, MLP_NORM, FINAL_NORM):
        return np.ones(shape, dtype=np.float32)
    rng = _stream(seed, layer, tid)
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(INIT_STD))


def layer_shapes(d: int, H: int, Hkv: int, F: int, hd: int, E: int = 0):
    """(tensor id, shape) of one decoder layer, weights stored [out, in]; with
    E experts the MLP matrices are stacked per expert and a router follows."""
    mlp = [(WGATE, (F, d)), (WUP, (F, d)), (WDOWN, (d, F))] if not E else \
        [(WGATE, (E, F, d)), (WUP, (E, F, d)), (WDOWN, (E, d, F)), (ROUTER, (E, d))]
    return [
        (ATTN_NORM, (d,)),
        (WQ, (H * hd, d)),
        (WK, (Hkv * hd, d)),
        (WV, (Hkv * hd, d)),
        (WO, (d, H * hd)),
        (MLP_NORM, (d,)),
    ] + mlp


def init_weights(cfg: dict, seed: int) -> dict:
    """All initial tensors of a decoder as a dict keyed by (layer, tensor id)."""
    d, H, Hkv, F, V, L = cfg["d"], cfg["H"], cfg["Hkv"], cfg["F"], cfg["V"], cfg["L"]
    hd = d // H
    out = {(-1, EMBED): init_tensor(seed, -1, EMBED, (V, d))}
    for l in range(L):
        for tid, shape in layer_shapes(d, H, Hkv, F, hd, cfg.get("E", 0)):
            out[(l, tid)] = init_tensor(seed, l, tid, shape)
    out[(-1, FINAL_NORM)] = init_tensor(seed, -1, FINAL_NORM, (d,))
    if not cfg.get("tied", False):  # tied embeddings: the head is the embedding table
        out[(-1, LM_HEAD)] = init_tensor(seed, -1, LM_HEAD, (V, d))
    return out
