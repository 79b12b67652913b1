"""Packing named fp32 tensors into the library's host arena (marshalling only).

Offsets come from the library itself (mt_tensor_offset); the arena is a
256-byte aligned numpy float32 array that the caller owns and hands to
mt_create.
"""
from __future__ import annotations

import numpy as np

from . import mt


def config(shape: dict, **hyper) -> "mt.mt_config":
    cfg = mt.mt_config_default(**{k: shape[k] for k in ("L", "d", "H", "Hkv", "F", "V", "b", "s")})
    if shape.get("E"):
        cfg.E, cfg.topk = shape["E"], shape.get("topk", 2)
    for k, v in hyper.items():
        setattr(cfg, k, v)
    return cfg


def aligned_empty(nfloats: int, align: int = 256) -> np.ndarray:
    raw = np.empty(nfloats * 4 + align, dtype=np.uint8)
    off = (-raw.ctypes.data) % align
    return raw[off:off + nfloats * 4].view(np.float32)


def pack(cfg, tensors: dict) -> np.ndarray:
    """tensors: (layer, tensor id) -> array, layer -1 for the model-level ones."""
    nbytes = mt.mt_arena_bytes(cfg)
    if nbytes == 0:
        raise ValueError("invalid config")
    arena = aligned_empty(nbytes // 4)
    arena[:] = 0
    for (layer, tid), t in tensors.items():
        off, n = mt.mt_tensor_offset(cfg, layer, tid)
        flat = np.asarray(t, dtype=np.float32).reshape(-1)
        if flat.size != n:
            raise ValueError(f"tensor {(layer, tid)}: {flat.size} elements, layout says {n}")
        arena[off:off + n] = flat
    return arena
