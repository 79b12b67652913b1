"""Sharded streaming (mt_create_sharded) through the C ABI.

On one GPU the sharded path runs with world = 1: every load goes through the
own-part H2D copy plus the NCCL all-gather into the padded slot, every
gradient block through the reduce-scatter, the shared finite check and the
own-part offload, and the embedding through the device table and the dense
row-split gradient. Its steps must give the plain engine's results (bit for
bit at head dim 128, where the split attention backward leaves no order
noise; else the first loss exactly, the gradients and the updated master to
the run-to-run noise of the attention's dQ reductions) and the oracle's.
Ranks on several GPUs are
not run here: with one GPU their collectives would be kernels that wait on
one another; the partition those ranks use is checked on CPU in
tests/test_sharded.py, on two gloo ranks.

The CPU tests at the end check what needs no GPU: the NCCL id, the refusals
and the padded device footprint."""
import os

import numpy as np
import pytest

import oracle
import synth

os.environ.setdefault("NCCL_SOCKET_IFNAME", "lo")  # one host: bootstrap over loopback

SHAPES = {
    "gqa_ragged": dict(L=3, d=256, H=4, Hkv=2, F=688, V=1024, b=3, s=100),
    "hd128": dict(L=2, d=256, H=2, Hkv=1, F=512, V=520, b=2, s=192),
    # expert layers: each rank routes its own tokens; the blocks partition as usual
    "experts": dict(L=2, d=256, H=2, Hkv=1, F=128, V=512, b=2, s=64, E=4, topk=2),
}
HYP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _run(shape, flags, nsteps, sharded):
    from host_memory_streamed_layer_b200 import arena, mt
    cfg = arena.config(shape)
    cfg.flags = flags
    cfg.host_threads = 4
    A = arena.pack(cfg, synth.init_weights(shape, 0))
    if sharded:
        ctx = mt.mt_create_sharded(cfg, A.ctypes.data, A.nbytes, 1, 0, mt.mt_shard_id())
    else:
        ctx = mt.mt_create(cfg, A.ctypes.data, A.nbytes)
    out = []
    try:
        for step in range(nsteps):
            tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, step)
            loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
            # deferred updates (the unsharded engine defers the untouched
            # embedding rows too; the sharded one updates its rows densely)
            # are applied before the state is read
            mt.mt_flush(ctx)
            G = None
            if not flags & mt.MT_FLAG_GRAD_RING:
                G = np.empty_like(A)
                mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
            out.append(dict(loss=loss, G=G, P=A.copy(), stats=mt.mt_get_stats(ctx)))
    finally:
        mt.mt_destroy(ctx)
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("flags", [0, "ring", "offload+stash", "defer+bf16+ring", "tied"])
@pytest.mark.parametrize("name", list(SHAPES))
def test_one_rank_sharded_steps_match_the_plain_engine_and_the_oracle(name, flags):
    from host_memory_streamed_layer_b200 import mt
    shape = dict(SHAPES[name], tied=flags == "tied")
    fl = {0: 0, "ring": mt.MT_FLAG_GRAD_RING, "tied": mt.MT_FLAG_TIED_EMBED,
          "offload+stash": mt.MT_FLAG_OFFLOAD_ACTS | mt.MT_FLAG_STASH_ATTN,
          "defer+bf16+ring": mt.MT_FLAG_DEFER_UPDATES | mt.MT_FLAG_BF16_GRADS | mt.MT_FLAG_GRAD_RING}[flags]
    # Head dim 128 runs the deterministic split attention backward: with one
    # rank every collective is a copy (the mean of one is the value) and the
    # dense zero-gradient rows update exactly like the untouched-row form, so
    # the two engines must agree bit for bit.
    exact = shape["d"] // shape["H"] == 128
    was = mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_SPLIT if exact else mt.ATTN_BWD_AUTO)
    try:
        plain = _run(shape, fl, 2, False)
        shard = _run(shape, fl, 2, True)
    finally:
        mt.mt_k_attn_bwd_variant(was)
    c = oracle.OracleConfig(**shape)
    if shape.get("E"):  # the oracle takes the GPU's routing (checked in test_gpu_moe)
        for a, b in zip(plain, shard):
            assert a["loss"] == b["loss"] and np.array_equal(a["P"], b["P"])
            assert a["G"] is None or np.array_equal(a["G"], b["G"])
        return
    if exact:
        for a, b in zip(plain, shard):
            assert a["loss"] == b["loss"] and np.array_equal(a["P"], b["P"])
            assert a["G"] is None or np.array_equal(a["G"], b["G"])
    for step, (a, b) in enumerate(zip(plain, shard)):
        assert abs(a["loss"] - b["loss"]) <= (1e-5 if step == 0 else 1e-5 * max(1.0, abs(a["loss"])))
        if a["G"] is not None:
            Ga, Gb = oracle.unpack_arena(a["G"], c), oracle.unpack_arena(b["G"], c)
            assert max(rel(Gb[k], Ga[k]) for k in Ga) <= 1e-4
        assert rel(b["P"], a["P"]) <= 1e-3
    # the first step against the oracle, as for the plain engine
    tok, lab = synth.tokens_labels(shape["b"], shape["s"], shape["V"], 0, 0)
    init = synth.init_weights(shape, 0)
    Wb = {k: oracle.bf16_round(v.astype(np.float32)) for k, v in init.items()}
    loss, G = oracle.train_step_grads(Wb, tok, lab, c)
    assert abs(shard[0]["loss"] - loss) <= 1e-2
    if shard[0]["G"] is not None:
        Gs = oracle.unpack_arena(shard[0]["G"], c)
        assert max(rel(Gs[k], G[k]) for k in G) <= 2e-2


@pytest.mark.gpu
def test_one_rank_sharded_link_bytes_are_the_own_parts():
    """With world = 1 the own part is everything: H2D carries every layer
    block (its padding excluded), the head block and the whole bf16 embedding
    table (which the sharded path keeps on the device), D2H every gradient."""
    from host_memory_streamed_layer_b200 import arena, mt
    shape = SHAPES["hd128"]
    st = _run(shape, 0, 1, True)[0]["stats"]
    cfg = arena.config(shape)
    p = mt.mt_shard_plan(cfg, 1, 0)
    L, d, V, T = shape["L"], shape["d"], shape["V"], shape["b"] * shape["s"]
    loads = 2 * L - 1
    assert st["h2d_bytes"] == pytest.approx(loads * p["layer_elems"] * 2 + p["head_elems"] * 2 + V * d * 2
                                            + 4 * (5 * T + 1))
    assert st["d2h_bytes"] == pytest.approx(4 * (p["head_elems"] + V * d + L * p["layer_elems"]) + 4 * (L + 4))


def test_shard_id_and_refusals_without_a_gpu():
    """mt_shard_id gives MT_SHARD_ID_BYTES fresh bytes per call; a sharded
    context refuses d % 128 != 0 before it touches a device, and bad ranks."""
    from host_memory_streamed_layer_b200 import arena, mt
    a, b = mt.mt_shard_id(), mt.mt_shard_id()
    assert len(a) == len(b) == mt.MT_SHARD_ID_BYTES and a != b
    shape = SHAPES["hd128"]
    with pytest.raises(mt.MTError) as e:
        mt.mt_create_sharded(arena.config(dict(shape, d=192, H=3, Hkv=3)), 0, 0, 2, 0, a)
    assert e.value.code == -2
    for world, rank in ((2, 2), (0, 0), (2, -1)):
        with pytest.raises(mt.MTError) as e:
            mt.mt_create_sharded(arena.config(shape), 0, 0, world, rank, a)
        assert e.value.code == -1  # MT_ERR_ARG


def test_sharded_device_footprint_pads_slots_and_adds_the_embedding():
    """mt_device_bytes_sharded = mt_device_bytes with the four slots and the
    head blocks padded to world chunks, plus the device embedding table (bf16)
    and its dense fp32 gradient over world * ceil(V / world) rows, and 4 bytes
    more staging per token (the unique ids are staged always)."""
    from host_memory_streamed_layer_b200 import arena, mt

    def al(n):
        return (n + 255) // 256 * 256
    for wl in ("llama-1.3b", "gqa-14b"):
        sh = synth.WORKLOADS[wl]
        cfg = arena.config(sh)
        base = mt.mt_device_bytes(cfg)
        y = mt.mt_shard_plan(cfg, 1, 0)
        d, V = sh["d"], sh["V"]
        head_w = d + V * d  # (d % 128 == 0: the head block has no padding)
        for world in (1, 2, 8):
            p = mt.mt_shard_plan(cfg, world, 0)
            rows = -(-V // world)
            slots = world * p["layer_chunk"]
            hc = world * p["head_chunk"]
            grow = (2 * (al(slots * 2) - al(y["layer_elems"] * 2)) + 2 * (al(slots * 4) - al(y["layer_elems"] * 4))
                    + al(hc * 2) - al(head_w * 2) + al(hc * 4) - al(y["head_elems"] * 4)
                    + al(world * rows * d * 2) + al(world * rows * d * 4))
            assert mt.mt_device_bytes_sharded(cfg, world) - base == grow, (wl, world)
    assert mt.mt_device_bytes_sharded(arena.config(dict(synth.WORKLOADS["tiny"], d=192, H=3, Hkv=3)), 2) == 0
