"""Sharded streaming over several GPUs of one host: the partition and ownership
logic of mt_shard_plan, checked on CPU.

Data-parallel ranks each train their own micro-batch through the same streamed
layers; each rank loads and all-gathers 1/world of every layer, receives 1/world
of the summed gradients (reduce-scatter) and runs the host AdamW on that part
only (intelligentliving.co, "Balancing Reduced Collective Communication with
Weight Streaming Latency", names the all-gather and reduce-scatter these use).

Two gloo ranks on 127.0.0.1 play the GPUs: the oracle gives each rank's
gradients on its own tokens; the collectives run on gloo over the plan's padded
chunks; each rank updates only its own chunk with the oracle's AdamW. The
result must equal one process updating everything with the mean gradient, every
rank's update must touch only its own elements, and the all-gathered bf16
blocks must be the bf16 copy of the whole updated master.
"""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SHAPE = dict(L=2, d=128, H=2, Hkv=1, F=256, V=256, b=1, s=32)  # one rank's micro-batch
HYP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _blocks(mt, cfg):
    """(name, arena offset, elements) of every sharded block: the decoder layer
    blocks and the [final gain | LM head] block."""
    L = cfg.L
    out = []
    for layer in range(L):
        off = mt.mt_tensor_offset(cfg, layer, mt.MT_T_ATTN_NORM)[0]
        end = mt.mt_tensor_offset(cfg, layer, mt.MT_T_WDOWN)
        out.append((f"layer{layer}", off, end[0] + end[1] - off))
    fo = mt.mt_tensor_offset(cfg, -1, mt.MT_T_FINAL_NORM)[0]
    ho, hn = mt.mt_tensor_offset(cfg, -1, mt.MT_T_LM_HEAD)
    out.append(("head", fo, ho + hn - fo))
    return out


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    import oracle
    import synth
    from host_memory_streamed_layer_b200 import arena, mt
    cfg = arena.config(SHAPE)
    plan = mt.mt_shard_plan(cfg, world, rank)
    c = oracle.OracleConfig(**SHAPE)
    init = synth.init_weights(SHAPE, 0)
    P = arena.pack(cfg, init).astype(np.float64)  # this rank's view of the master
    P0 = P.copy()
    Wb = {k: oracle.bf16_round(v.astype(np.float32)) for k, v in init.items()}
    tok, lab = synth.tokens_labels(1, SHAPE["s"], SHAPE["V"], 100 + rank)
    _, G = oracle.train_step_grads(Wb, tok, lab, c)
    Ga = arena.pack(cfg, {k: v.astype(np.float32) for k, v in G.items()}).astype(np.float64)
    touched = np.zeros(P.size, dtype=bool)
    bf16 = {}
    for name, off, n in _blocks(mt, cfg):
        chunk = plan["layer_chunk"] if name != "head" else plan["head_chunk"]
        b, e = (plan["layer_begin"], plan["layer_end"]) if name != "head" else (plan["head_begin"], plan["head_end"])
        # reduce-scatter of the padded block (gloo: an all-reduce, then the
        # rank keeps its own chunk): the mean gradient's own chunk
        g = torch.zeros(world * chunk, dtype=torch.float64)
        g[:n] = torch.from_numpy(Ga[off:off + n])
        dist.all_reduce(g)
        mine = g[rank * chunk:(rank + 1) * chunk].numpy() / world
        lo, hi = off + b, off + e
        p, _, _ = oracle.adamw_update(P[lo:hi], mine[:e - b], 0.0, 0.0, 1, **HYP)
        P[lo:hi] = p
        touched[lo:hi] = True
        # all-gather of the bf16 chunks into the whole streamed block
        piece = torch.zeros(chunk, dtype=torch.float64)
        piece[:e - b] = torch.from_numpy(oracle.bf16_round(p.astype(np.float32)).astype(np.float64))
        got = [torch.zeros(chunk, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, piece)
        bf16[name] = torch.cat(got)[:n].numpy()
    # embedding: rows are owned; the summed gradient of the rows comes from an all-reduce
    eo, en = mt.mt_tensor_offset(cfg, -1, mt.MT_T_EMBED)
    ge = torch.from_numpy(Ga[eo:eo + en].copy())
    dist.all_reduce(ge)
    d = SHAPE["d"]
    lo, hi = eo + plan["embed_row_begin"] * d, eo + plan["embed_row_end"] * d
    p, _, _ = oracle.adamw_update(P[lo:hi], ge.numpy()[lo - eo:hi - eo] / world, 0.0, 0.0, 1, **HYP)
    P[lo:hi] = p
    touched[lo:hi] = True
    untouched_same = bool(np.array_equal(P[~touched], P0[~touched]))
    dist.destroy_process_group()
    q.put((rank, dict(plan=plan, P=P, touched=touched, bf16=bf16, untouched_same=untouched_same)))


def test_shard_plan_partitions_every_block():
    """Chunks are 128-element aligned, cover every element of a block exactly
    once across the ranks, and the embedding rows likewise; d % 128 != 0 and
    bad ranks are refused."""
    import synth
    from host_memory_streamed_layer_b200 import arena, mt
    for wl in ("tiny", "llama-1.3b", "gqa-14b"):
        cfg = arena.config(synth.WORKLOADS[wl])
        for world in (1, 2, 3, 8):
            plans = [mt.mt_shard_plan(cfg, world, r) for r in range(world)]
            for key in ("layer", "head"):
                n, ch = plans[0][f"{key}_elems"], plans[0][f"{key}_chunk"]
                assert ch % 128 == 0 and world * ch >= n > (world - 1) * ch - 128 * world
                # ranks in order tile [0, n) with no gap and no overlap
                edge = 0
                for p in plans:
                    b, e = p[f"{key}_begin"], p[f"{key}_end"]
                    assert b % 128 == 0 and b <= e <= n and b == edge
                    edge = e
                assert edge == n
            edge = 0
            for p in plans:
                assert p["embed_row_begin"] == edge and p["embed_row_end"] >= edge
                edge = p["embed_row_end"]
            assert edge == cfg.V
            if world == 1:
                assert plans[0]["layer_end"] == plans[0]["layer_elems"]
    with pytest.raises(mt.MTError) as e:
        mt.mt_shard_plan(arena.config(dict(L=1, d=192, H=3, Hkv=3, F=256, V=64, b=1, s=8)), 2, 0)
    assert e.value.code == -2
    with pytest.raises(mt.MTError):
        mt.mt_shard_plan(arena.config(synth.WORKLOADS["tiny"]), 2, 2)


def test_sharded_update_equals_the_replicated_one_on_two_gloo_ranks():
    import oracle
    import synth
    from host_memory_streamed_layer_b200 import arena, mt
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # one process, both micro-batches: the data-parallel step's mean gradient
    cfg = arena.config(SHAPE)
    c = oracle.OracleConfig(**SHAPE)
    init = synth.init_weights(SHAPE, 0)
    Wb = {k: oracle.bf16_round(v.astype(np.float32)) for k, v in init.items()}
    Gs = []
    for rank in range(world):
        tok, lab = synth.tokens_labels(1, SHAPE["s"], SHAPE["V"], 100 + rank)
        Gs.append(arena.pack(cfg, {k: v.astype(np.float32)
                                   for k, v in oracle.train_step_grads(Wb, tok, lab, c)[1].items()}).astype(np.float64))
    P0 = arena.pack(cfg, init).astype(np.float64)
    Pref, _, _ = oracle.adamw_update(P0, (Gs[0] + Gs[1]) / world, 0.0, 0.0, 1, **HYP)
    owned = np.zeros(P0.size, dtype=np.int32)
    for rank in range(world):
        r = out[rank]
        assert r["untouched_same"]  # the update touched only the rank's own elements
        t = r["touched"]
        owned += t
        assert np.array_equal(r["P"][t], Pref[t])
        for name, off, n in _blocks(mt, cfg):
            want = oracle.bf16_round(Pref[off:off + n].astype(np.float32)).astype(np.float64)
            assert np.array_equal(r["bf16"][name], want), name
    # every parameter of the arena is updated by exactly one rank
    pad = np.ones(P0.size, dtype=bool)
    for _, off, n in _blocks(mt, cfg):
        pad[off:off + n] = False
    eo, en = mt.mt_tensor_offset(cfg, -1, mt.MT_T_EMBED)
    pad[eo:eo + en] = False
    assert np.all(owned[~pad] == 1) and np.all(owned[pad] == 0)
