"""Host-side checks of the C ABI that need no GPU: the library loads and
exports every function the headers declare, its arena layout agrees with the
oracle's independent reading of the documented layout, configuration errors
are reported, and the host AdamW matches the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

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


@pytest.mark.parametrize("name", ["llama-1.3b", "llama-7b", "gqa-14b"])
def test_host_state_with_gradient_ring(name):
    """With the gradient ring the fp32 gradient arena (4 B/param) is replaced by
    MT_GRAD_RING_SLOTS layer-sized slots plus the final-norm + LM-head
    gradient: master + state is then about 14 B/param, which is what lets the
    14B workload (12.57 B parameters) fit a host with under 200 GB of RAM."""
    mt = _mt()
    shape = synth.WORKLOADS[name]
    cfg = mt.mt_config_default(**shape)
    full = mt.mt_host_state_bytes(cfg)
    cfg.flags = mt.MT_FLAG_GRAD_RING
    ring = mt.mt_host_state_bytes(cfg)
    P = mt.mt_arena_bytes(cfg) // 4
    c = oracle.OracleConfig(**shape)
    layout, _ = oracle.arena_layout(c)
    first = {}
    for layer, tid, off, shp in layout:
        first[(layer, tid)] = (off, int(np.prod(shp)))
    # one layer's gradient block: from its first tensor to the next layer's first tensor
    layer_f = first[(1, mt.MT_T_ATTN_NORM)][0] - first[(0, mt.MT_T_ATTN_NORM)][0]
    fn_off = first[(-1, mt.MT_T_FINAL_NORM)][0]
    head_off, head_n = first[(-1, mt.MT_T_LM_HEAD)]
    head_f = head_off + head_n - fn_off
    assert ring == full - 4 * P + 4 * (mt.MT_GRAD_RING_SLOTS * layer_f + head_f)
    # the fixed buffers weigh less as models grow: ~14.9 B/param at 1.3B, ~14.5 at 14B
    assert ring + 4 * P <= (15.0 if P < 5e9 else 14.6) * P


def test_host_state_with_deferred_updates(monkeypatch):
    """MT_FLAG_DEFER_UPDATES with the ring adds one layer-sized gradient buffer
    per deferred layer (MT_DEFER_LAYERS, default 1, clamped to [0, L-1]); the
    full gradient arena already holds every layer's gradient, and with
    MT_FLAG_NO_UPDATE nothing is deferred."""
    mt = _mt()
    shape = dict(L=4, d=256, H=4, Hkv=4, F=688, V=1024, b=2, s=128)
    cfg = mt.mt_config_default(**shape)
    full = mt.mt_host_state_bytes(cfg)
    cfg.flags = mt.MT_FLAG_GRAD_RING
    ring = mt.mt_host_state_bytes(cfg)
    first = [mt.mt_tensor_offset(cfg, layer, mt.MT_T_ATTN_NORM)[0] for layer in (0, 1)]
    layer_bytes = 4 * (first[1] - first[0])
    cfg.flags = mt.MT_FLAG_GRAD_RING | mt.MT_FLAG_DEFER_UPDATES
    monkeypatch.delenv("MT_DEFER_LAYERS", raising=False)
    assert mt.mt_host_state_bytes(cfg) == ring + layer_bytes
    for env, nd in (("0", 0), ("2", 2), ("99", shape["L"] - 1), ("-3", 0)):
        monkeypatch.setenv("MT_DEFER_LAYERS", env)
        assert mt.mt_host_state_bytes(cfg) == ring + nd * layer_bytes, env
    monkeypatch.setenv("MT_DEFER_LAYERS", "2")
    cfg.flags = mt.MT_FLAG_GRAD_RING | mt.MT_FLAG_DEFER_UPDATES | mt.MT_FLAG_NO_UPDATE
    assert mt.mt_host_state_bytes(cfg) == ring
    cfg.flags = mt.MT_FLAG_DEFER_UPDATES
    assert mt.mt_host_state_bytes(cfg) == full


def test_host_adamw_zero_gradient_reads_nothing():
    """g = NULL is the update of a zero gradient: bit-identical to passing
    zeros, and equal to the oracle's AdamW with g = 0 (decay and moment decay
    only)."""
    mt = _mt()
    rng = np.random.default_rng(3)
    n = 4099
    p0 = (rng.normal(size=n) * 0.02).astype(np.float32)
    m0 = (rng.normal(size=n) * 1e-3).astype(np.float32)
    v0 = (np.abs(rng.normal(size=n)) * 1e-6).astype(np.float32)
    hyper = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)
    outs = []
    for g in (None, np.zeros(n, dtype=np.float32)):
        p, m, v = p0.copy(), m0.copy(), v0.copy()
        pb = np.zeros(n, dtype=np.uint16)
        mt.mt_k_adamw_host(p.ctypes.data, 0 if g is None else g.ctypes.data, m.ctypes.data, v.ctypes.data,
                           pb.ctypes.data, n, hyper["lr"], hyper["beta1"], hyper["beta2"], hyper["eps"],
                           hyper["wd"], 3)
        outs.append((p, m, v, pb))
    for a, b in zip(outs[0], outs[1]):
        assert np.array_equal(a, b)
    rp, rm, rv = oracle.adamw_update(p0.astype(np.float64), np.zeros(n), m0.astype(np.float64),
                                     v0.astype(np.float64), 3, **hyper)
    assert np.all(np.abs(outs[0][0] - rp) <= 2e-8 + 1e-6 * np.abs(rp))
    assert np.allclose(outs[0][1], 0.9 * m0.astype(np.float64), rtol=1e-6, atol=0)
    assert np.allclose(outs[0][2], 0.95 * v0.astype(np.float64), rtol=1e-6, atol=0)


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


def test_host_bf16_copy_special_values_match_torch():
    """With lr = 0 and wd = 0 the master is unchanged and the streamed bf16 copy
    is the library's own round-to-nearest-even of it: ties to even and to odd,
    just below and above a tie, a carry into the next exponent, the overflow to
    infinity of float32's largest value, subnormals, signed zeros and
    infinities bit-exact against torch's conversion, NaN kept NaN, in the
    16-wide vector loop and in the scalar tail."""
    mt = _mt()
    bits = [0x3F808000, 0x3F818000, 0x3F807FFF, 0x3F808001, 0x3F7FFFFF, 0x7F7FFFFF, 0xFF7FFFFF, 0x00000001,
            0x000FFFFF, 0x80008000, 0x00000000, 0x80000000, 0x7F800000, 0xFF800000, 0x3F800000, 0xBF818000,
            0x7FC00000, 0xFFC12345, 0x7F800001]
    vals = np.array(bits, dtype=np.uint32).view(np.float32)
    p = np.concatenate([vals, vals, vals[:15]]).copy()  # 53 = 3 x 16 + 5: vector lanes and a scalar tail
    n = p.size
    p0 = p.copy()
    g, m, v = np.zeros(n, np.float32), np.zeros(n, np.float32), np.zeros(n, np.float32)
    pb = np.zeros(n, dtype=np.uint16)
    mt.mt_k_adamw_host(p.ctypes.data, g.ctypes.data, m.ctypes.data, v.ctypes.data, pb.ctypes.data, n,
                       0.0, 0.9, 0.95, 1e-8, 0.0, 1)
    nan = np.isnan(p0)
    assert np.array_equal(p.view(np.uint32)[~nan], p0.view(np.uint32)[~nan]) and np.isnan(p[nan]).all()
    ref = torch.from_numpy(p0).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got_f = (pb.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(pb[~nan], ref[~nan]), [(hex(b), hex(a), hex(r)) for b, a, r in
                                                 zip(p0.view(np.uint32), pb, ref) if a != r]
    assert np.isnan(got_f[nan]).all()


def test_host_adamw_rejects_bad_step():
    mt = _mt()
    x = np.zeros(4, dtype=np.float32)
    with pytest.raises(mt.MTError):
        mt.mt_k_adamw_host(x.ctypes.data, x.ctypes.data, x.ctypes.data, x.ctypes.data, 0, 4, 1e-3, 0.9, 0.95,
                           1e-8, 0.1, 0)


def test_null_context_calls_are_rejected():
    """Every context call given NULL returns MT_ERR_ARG (mt_destroy ignores it)."""
    mt = _mt()
    assert mt.lib.mt_flush(None) == -1
    assert mt.lib.mt_get_params(None, None, 0) == -1
    assert mt.lib.mt_get_grads(None, None, 0) == -1
    assert mt.lib.mt_get_opt_state(None, None, None, 0, None) == -1
    mt.lib.mt_destroy(None)


def _declared_params():
    """Parameter declarations of every function the headers declare."""
    out = {}
    for h in ("mt.h", "mt_kernels.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^([A-Za-z_][\w\s\*]*?)\b(mt_\w+)\s*\(([^)]*)\)\s*;", src, flags=re.M | re.S):
            params = [p.strip() for p in m.group(3).split(",") if p.strip() and p.strip() != "void"]
            out[m.group(2)] = (m.group(1).strip(), params)
    return out


# scalar C types of the headers: (is floating point, bytes)
_C_SCALARS = {"int": (False, 4), "int32_t": (False, 4), "uint32_t": (False, 4), "int64_t": (False, 8),
              "size_t": (False, 8), "float": (True, 4), "double": (True, 8)}


def _kind_of_ctype(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "pointer"
    return (t in (ctypes.c_float, ctypes.c_double), ctypes.sizeof(t))


def _kind_of_param(decl):
    if "*" in decl:
        return "pointer"
    ctype = decl.replace("const ", "").split()[0]
    return _C_SCALARS[ctype]


def test_binding_signatures_match_the_headers():
    """Every function the Python binding declares takes the arguments and
    returns the type of its C declaration: as many arguments, each a pointer
    where the header has one, else a scalar of the same kind (integer or
    floating point) and width; and the binding covers every declared function."""
    mt = _mt()
    decls = _declared_params()
    assert set(decls) == _declared_functions()
    for name, (ret, params) in sorted(decls.items()):
        fn = getattr(mt.lib, name)
        assert fn.argtypes is not None, f"{name} has no ctypes signature"
        if ret == "void":
            assert fn.restype is None, name
        else:
            assert _kind_of_ctype(fn.restype) == _kind_of_param(ret), (name, ret, fn.restype)
        assert len(fn.argtypes) == len(params), (name, len(fn.argtypes), len(params))
        for i, (t, decl) in enumerate(zip(fn.argtypes, params)):
            assert _kind_of_ctype(t) == _kind_of_param(decl), (name, i, decl, t)


@pytest.mark.parametrize("shape", [synth.WORKLOADS["tiny"], dict(L=3, d=320, H=5, Hkv=1, F=712, V=1000, b=1, s=64)])
def test_arena_pack_round_trips_through_the_oracle_layout(shape):
    """arena.pack places every tensor where the oracle's independent reading of
    the layout expects it, 256-byte aligned, with zero padding between
    tensors; a tensor of the wrong size is rejected."""
    from host_memory_streamed_layer_b200 import arena
    cfg = arena.config(shape, lr=2e-3)
    assert abs(cfg.lr - 2e-3) < 1e-9
    W = synth.init_weights(shape, 4)
    A = arena.pack(cfg, W)
    assert A.ctypes.data % 256 == 0 and A.dtype == np.float32
    c = oracle.OracleConfig(**shape)
    U = oracle.unpack_arena(A, c, dtype=np.float32)
    for k, w in W.items():
        assert np.array_equal(U[k], np.asarray(w, dtype=np.float32).reshape(U[k].shape)), k
    used = np.zeros(A.size, dtype=bool)
    for layer, tid, off, shp in oracle.arena_layout(c)[0]:
        used[off:off + int(np.prod(shp))] = True
    assert np.all(A[~used] == 0)
    bad = dict(W)
    k0 = next(iter(bad))
    bad[k0] = np.zeros(np.asarray(bad[k0]).size + 1, dtype=np.float32)
    with pytest.raises(ValueError):
        arena.pack(cfg, bad)


def test_device_bytes_grow_only_by_the_boundary_activations():
    """mt_device_bytes: two bf16 weight slots, two fp32 gradient slots, the head,
    one workspace and the L+1 boundary activations; one more layer adds exactly
    one fp32 [b*s, d] boundary activation and nothing else (the persistent
    state of saify.me, "The memory-centric design")."""
    from host_memory_streamed_layer_b200 import arena, mt
    for base in (dict(d=1024, H=8, Hkv=8, F=2752, V=4096, b=4, s=1024),
                 dict(d=5120, H=40, Hkv=8, F=13824, V=152064, b=2, s=4096)):
        T, d = base["b"] * base["s"], base["d"]
        sizes = [mt.mt_device_bytes(arena.config(dict(base, L=L))) for L in (1, 2, 5, 40)]
        for (La, a), (Lb, b) in zip(zip((1, 2, 5, 40), sizes), zip((2, 5, 40), sizes[1:])):
            assert b - a == (Lb - La) * T * d * 4
        cfg = arena.config(dict(base, L=2))
        P_layer = sum(mt.mt_tensor_offset(cfg, 0, t)[1] for t in range(9))
        assert sizes[1] > 2 * 2 * P_layer + 2 * 4 * P_layer + 3 * T * d * 4
    bad = arena.config(dict(L=2, d=100, H=2, Hkv=2, F=64, V=64, b=1, s=8))
    assert mt.mt_device_bytes(bad) == 0


def test_offloaded_activations_keep_three_device_slots():
    """MT_FLAG_OFFLOAD_ACTS: the device footprint no longer grows with L (three
    boundary slots), and the host state grows by the L-2 offloaded fp32
    [b*s, d] boundary activations."""
    from host_memory_streamed_layer_b200 import arena, mt
    base = dict(d=1024, H=8, Hkv=8, F=2752, V=4096, b=4, s=1024)
    T, d = base["b"] * base["s"], base["d"]
    dev, host = [], []
    for L in (3, 6, 40):
        cfg = arena.config(dict(base, L=L))
        plain_dev, plain_host = mt.mt_device_bytes(cfg), mt.mt_host_state_bytes(cfg)
        cfg.flags = mt.MT_FLAG_OFFLOAD_ACTS
        dev.append(mt.mt_device_bytes(cfg))
        host.append(mt.mt_host_state_bytes(cfg))
        assert plain_dev - dev[-1] == (L + 1 - 3) * T * d * 4
        assert host[-1] - plain_host == (L - 2) * T * d * 4
    assert dev[0] == dev[1] == dev[2]


def test_attention_stash_adds_one_output_and_lse_per_layer():
    """MT_FLAG_STASH_ATTN: the device keeps L attention outputs (bf16 [b*s, H*hd])
    and log-sum-exp blocks (fp32 [b, H, s]) instead of one of each; host state
    is unchanged. Sizes are 256-byte aligned like every other buffer."""
    from host_memory_streamed_layer_b200 import arena, mt
    base = dict(d=1024, H=8, Hkv=2, F=2752, V=4096, b=3, s=1000)
    T, Hd = base["b"] * base["s"], 1024

    def al(n):
        return (n + 255) // 256 * 256
    for L in (1, 4, 32):
        for extra in (0, mt.MT_FLAG_OFFLOAD_ACTS):
            cfg = arena.config(dict(base, L=L))
            cfg.flags = extra
            plain_dev, plain_host = mt.mt_device_bytes(cfg), mt.mt_host_state_bytes(cfg)
            cfg.flags = extra | mt.MT_FLAG_STASH_ATTN
            grow = al(L * T * Hd * 2) - al(T * Hd * 2) + al(L * base["b"] * base["H"] * base["s"] * 4) \
                - al(base["b"] * base["H"] * base["s"] * 4)
            assert mt.mt_device_bytes(cfg) - plain_dev == grow
            assert mt.mt_host_state_bytes(cfg) == plain_host


def test_tied_embeddings_layout():
    """MT_FLAG_TIED_EMBED: the arena loses exactly the LM-head tensor (the
    oracle's tied layout matches the library's offsets), MT_T_LM_HEAD is
    refused, bf16 gradients are refused, and the shard plan's head block is
    the final gain alone."""
    import oracle
    from host_memory_streamed_layer_b200 import arena, mt
    shape = dict(L=3, d=256, H=4, Hkv=2, F=688, V=1000, b=2, s=64)
    cfg = arena.config(shape)
    untied = mt.mt_arena_bytes(cfg)
    cfg.flags = mt.MT_FLAG_TIED_EMBED
    assert untied - mt.mt_arena_bytes(cfg) == 4 * shape["V"] * shape["d"]
    c = oracle.OracleConfig(**shape, tied=True)
    layout, total = oracle.arena_layout(c)
    assert total * 4 == mt.mt_arena_bytes(cfg)
    for layer, tid, off, shp in layout:
        assert mt.mt_tensor_offset(cfg, layer, tid) == (off, int(np.prod(shp)))
    with pytest.raises(mt.MTError):
        mt.mt_tensor_offset(cfg, -1, mt.MT_T_LM_HEAD)
    # sharded: the head block is the final gain alone (the table is split by rows)
    p = mt.mt_shard_plan(cfg, 2, 1)
    assert p["head_elems"] == shape["d"] and p["embed_row_end"] == shape["V"]
    cfg.flags = mt.MT_FLAG_TIED_EMBED | mt.MT_FLAG_BF16_GRADS
    assert mt.mt_arena_bytes(cfg) == 0


def test_expert_layer_layout_matches_the_oracle():
    """Expert layers (E > 0): the library's arena offsets and sizes are the
    oracle's stacked-expert layout, the router exists only with experts, and
    bad expert counts are refused; the bf16 layer block grows by the same
    expert matrices (host state and device footprint follow)."""
    import oracle
    from host_memory_streamed_layer_b200 import arena, mt
    sh = dict(L=3, d=256, H=2, Hkv=1, F=96, V=304, b=2, s=40, E=6, topk=2)
    cfg = arena.config(sh)
    layout, total = oracle.arena_layout(oracle.OracleConfig(**sh))
    assert mt.mt_arena_bytes(cfg) == total * 4
    for layer, tid, off, shape in layout:
        assert mt.mt_tensor_offset(cfg, layer, tid) == (off, int(np.prod(shape)))
    dense = arena.config(dict(sh, E=0))
    with pytest.raises(mt.MTError):
        mt.mt_tensor_offset(dense, 0, mt.MT_T_ROUTER)
    for E, k in ((65, 1), (4, 0), (4, 5), (-1, 1)):
        bad = arena.config(sh)
        bad.E, bad.topk = E, k
        assert mt.mt_arena_bytes(bad) == 0
    per_layer = mt.mt_tensor_offset(cfg, 1, mt.MT_T_ATTN_NORM)[0] - mt.mt_tensor_offset(cfg, 0, mt.MT_T_ATTN_NORM)[0]
    per_dense = (mt.mt_tensor_offset(dense, 1, mt.MT_T_ATTN_NORM)[0]
                 - mt.mt_tensor_offset(dense, 0, mt.MT_T_ATTN_NORM)[0])
    assert per_layer - per_dense == (6 - 1) * 3 * 96 * 256 + 6 * 256
    assert mt.mt_host_state_bytes(cfg) > mt.mt_host_state_bytes(dense)
    assert mt.mt_device_bytes(cfg) > mt.mt_device_bytes(dense)
    # expert layers partition like dense ones: their arena and bf16 offsets agree (d % 128 == 0)
    p = mt.mt_shard_plan(cfg, 2, 1)
    assert p["layer_elems"] == per_layer and p["layer_end"] == per_layer


def test_tensor_core_attention_backward_refusals_without_a_gpu():
    """mt_k_attn_bwd_tc takes head dims 64 and 128 (MT_ERR_CONFIG otherwise)
    and a dQ accumulator it can store four floats at a time (MT_ERR_ARG
    otherwise), both refused before any device work; the form selector takes
    0, 1 and 2 and returns the previous choice."""
    mt = _mt()
    from host_memory_streamed_layer_b200 import arena
    buf = arena.aligned_empty(1 << 16)
    p = buf.ctypes.data
    b, s, H, Hkv = 1, 8, 2, 1

    def call(hd, ldqa):
        ld = (H + 2 * Hkv) * hd
        return mt.mt_k_attn_bwd_tc(p, p, p, ld, p, p, H * hd, p, p, p, ldqa, p, ld, p, p, ld, b, s, H, Hkv, hd)
    for hd in (32, 96, 256):
        with pytest.raises(mt.MTError) as e:
            call(hd, H * hd)
        assert e.value.code == -2  # MT_ERR_CONFIG
    for hd in (64, 128):
        with pytest.raises(mt.MTError) as e:
            call(hd, H * hd + 1)  # ldqa not a multiple of 4
        assert e.value.code == -1  # MT_ERR_ARG
    was = mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_SPLIT)
    try:
        assert mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_FUSED) == mt.ATTN_BWD_SPLIT
        with pytest.raises(mt.MTError) as e:
            mt.mt_k_attn_bwd_variant(3)
        assert e.value.code == -1
        assert mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_AUTO) == mt.ATTN_BWD_FUSED
    finally:
        mt.mt_k_attn_bwd_variant(was)
