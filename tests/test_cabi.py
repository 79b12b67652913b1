"""Host-side checks of the C ABI that need no GPU: the library loads and
exports every function the headers declare, its arena layout agrees with the
oracle's independent reading of the documented layout, configuration errors
are reported, and the host AdamW matches the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _mt():
    from host_memory_streamed_layer_b200 import mt
    return mt


def _declared_functions():
    names = set()
    for h in ("mt.h", "mt_kernels.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(mt_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_function():
    mt = _mt()
    names = _declared_functions()
    assert len(names) >= 20, names
    for n in sorted(names):
        assert hasattr(mt.lib, n), f"libmt.so does not export {n}"


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_layout_agrees_with_oracle(name):
    mt = _mt()
    shape = synth.WORKLOADS[name]
    cfg = mt.mt_config_default(**shape)
    c = oracle.OracleConfig(**shape)
    layout, total = oracle.arena_layout(c)
    assert mt.mt_arena_bytes(cfg) == total * 4
    for layer, tid, off, shp in layout:
        assert mt.mt_tensor_offset(cfg, layer, tid) == (off, int(np.prod(shp)))


def test_host_state_accounting():
    """Moments (8 B/param) + gradient arena (4 B/param) + bf16 copy (2 B/param)
    on top of the caller's 4 B/param master: 12 B/param of optimizer state
    (master + m + v) as the pages size it, plus the streaming buffers."""
    mt = _mt()
    cfg = mt.mt_config_default(**synth.WORKLOADS["llama-1.3b"])
    P = mt.mt_arena_bytes(cfg) // 4
    extra = mt.mt_host_state_bytes(cfg)
    assert 14 * P <= extra <= 14.2 * P


@pytest.mark.parametrize("bad", [dict(d=100), dict(H=3), dict(Hkv=3), dict(F=689), dict(V=1001), dict(L=0),
                                 dict(d=512, H=2), dict(b=0)])
def test_invalid_config_rejected(bad):
    mt = _mt()
    cfg = mt.mt_config_default(**{**synth.WORKLOADS["tiny"], **bad})
    assert mt.mt_arena_bytes(cfg) == 0
    with pytest.raises(mt.MTError) as e:
        mt.mt_create(cfg)
    assert e.value.code == -2  # MT_ERR_CONFIG, found before any device work


def test_bad_struct_size_and_small_arena():
    mt = _mt()
    cfg = mt.mt_config_default(**synth.WORKLOADS["tiny"])
    arena = np.zeros(mt.mt_arena_bytes(cfg) // 4 - 64, dtype=np.float32)
    with pytest.raises(mt.MTError) as e:
        mt.mt_create(cfg, arena.ctypes.data, arena.nbytes)
    assert e.value.code == -3  # MT_ERR_ARENA
    cfg.struct_size = 12
    with pytest.raises(mt.MTError) as e:
        mt.mt_create(cfg)
    assert e.value.code == -1


def test_host_adamw_matches_oracle_over_steps():
    mt = _mt()
    rng = np.random.default_rng(0)
    n = 10007  # ragged against the 16-wide vector loop
    p = (rng.normal(size=n) * 0.02).astype(np.float32)
    m = np.zeros(n, dtype=np.float32)
    v = np.zeros(n, dtype=np.float32)
    pb = np.zeros(n, dtype=np.uint16)
    rp, rm, rv = p.astype(np.float64), np.zeros(n), np.zeros(n)
    hyper = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)
    mscale = np.zeros(n)  # sum of |terms| of the first moment: fp32 error is relative to it
    for t in range(1, 4):
        g = (rng.normal(size=n) * 10.0 ** rng.uniform(-7, 0, n)).astype(np.float32)
        g[:5] = 0.0
        mt.mt_k_adamw_host(p.ctypes.data, g.ctypes.data, m.ctypes.data, v.ctypes.data, pb.ctypes.data, n,
                           hyper["lr"], hyper["beta1"], hyper["beta2"], hyper["eps"], hyper["wd"], t)
        rp, rm, rv = oracle.adamw_update(rp, g, rm, rv, t, **hyper)
        mscale = 0.9 * mscale + 0.1 * np.abs(g)
        assert np.all(np.abs(p - rp) <= 2e-8 + 1e-6 * np.abs(rp)), t
        assert np.all(np.abs(m - rm) <= 1e-6 * mscale + 1e-30), t
        assert np.all(np.abs(v - rv) <= 1e-5 * rv + 1e-30), t
        # the streamed copy is exactly the round-to-nearest-even of the new master
        ref_bits = (oracle.bf16_round(p).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal(pb, ref_bits)


def test_host_adamw_rejects_bad_step():
    mt = _mt()
    x = np.zeros(4, dtype=np.float32)
    with pytest.raises(mt.MTError):
        mt.mt_k_adamw_host(x.ctypes.data, x.ctypes.data, x.ctypes.data, x.ctypes.data, 0, 4, 1e-3, 0.9, 0.95,
                           1e-8, 0.1, 0)
