"""The bench's phase bound (bench.step_bounds) on made-up rates: which term
binds in each phase, how deferral moves update bytes into the forward phase,
that the whole step's update bytes bound it too, and that the DRAM model only
adds traffic. No GPU: the inputs are plain numbers."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import synth  # noqa: E402

SH = synth.WORKLOADS["llama-1.3b"]
LINK = {"h2d_gbs": 50.0, "d2h_gbs": 50.0}


def params(sh):
    L = sh["L"]
    return L * bench.layer_params(sh) + 2 * bench.head_params(sh) - sh["d"]  # embedding has no final-norm gain


def test_parameter_counts_match_the_arena():
    from host_memory_streamed_layer_b200 import arena, mt
    cfg = arena.config(SH)
    first = [mt.mt_tensor_offset(cfg, layer, mt.MT_T_ATTN_NORM)[0] for layer in (0, 1)]
    n_layer = sum(mt.mt_tensor_offset(cfg, 0, t)[1] for t in range(9))
    assert bench.layer_params(SH) == n_layer <= first[1] - first[0]
    fn = mt.mt_tensor_offset(cfg, -1, mt.MT_T_FINAL_NORM)[1]
    head = mt.mt_tensor_offset(cfg, -1, mt.MT_T_LM_HEAD)[1]
    assert bench.head_params(SH) == fn + head


def test_host_bound_phase_structure():
    n_unique = 12000
    upd = 30.0 * params(SH)
    kw = dict(peak_tflops=1000.0, link=LINK, h2d_bytes=5e9, d2h_bytes=5e9, update_bytes=upd, n_unique=n_unique)
    slow = bench.step_bounds(SH, host_gbs=100.0, **kw)
    untouched = 30.0 * (SH["V"] - n_unique) * SH["d"]
    assert slow["update_bytes_fwd"] == pytest.approx(untouched)
    assert slow["update_bytes_bwd"] == pytest.approx(upd - untouched)
    # a slow host: the backward is the optimizer's bytes at the host rate
    assert slow["bwd"] == pytest.approx((upd - untouched) / 100e9)
    f_fl, b_fl = bench.phase_flops(SH)
    L = SH["L"]
    assert slow["fwd"] == pytest.approx(max(f_fl / 1e15, 5e9 * L / (2 * L - 1) / 50e9))
    assert slow["bound"] == pytest.approx(max(slow["fwd"] + slow["bwd"], upd / 100e9))
    # a fast host: the backward is the GPU's or the D2H's
    fast = bench.step_bounds(SH, host_gbs=1e6, **kw)
    assert fast["bwd"] == pytest.approx(max(b_fl / 1e15, 5e9 / 50e9))
    # deferral moves the LM head and the deferred layers into the forward phase
    d1 = bench.step_bounds(SH, host_gbs=100.0, deferred_layers=1, **kw)
    moved = 30.0 * (bench.head_params(SH) + bench.layer_params(SH))
    assert d1["update_bytes_fwd"] - slow["update_bytes_fwd"] == pytest.approx(moved)
    assert d1["bwd"] == pytest.approx(slow["bwd"] - moved / 100e9)
    assert d1["fwd"] == slow["fwd"]
    # however the updates are split, the step needs all of them at the host rate
    assert d1["bound"] >= upd / 100e9 - 1e-12
    # the DRAM model adds the copies' traffic, so it never undercuts the bound's phases
    for r in (slow, fast, d1):
        assert r["model"] >= r["fwd"] + r["bwd"] - 1e-12
        assert r["dram_fwd"] + r["dram_bwd"] == pytest.approx(upd + 5e9 + 5e9)


def test_step_spread_and_cpu_model():
    stats = [dict(host_step_ms=h, step_ms=d) for h, d in ((320.0, 290.0), (318.0, 288.0), (330.0, 291.0))]
    sp = bench.step_spread(stats)
    assert sp == dict(host_ms_min=318.0, host_ms_median=320.0, device_ms_min=288.0, device_ms_median=290.0)
    assert bench.step_spread([]) == {}
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()


@pytest.mark.parametrize("env", [None, "0", "2", " 3", "2x", "abc", "-4", "99"])
def test_deferred_layer_count_matches_the_library(monkeypatch, env):
    """bench.defer_layers reads MT_DEFER_LAYERS as the library does: its
    host-memory accounting grows by one layer-sized buffer per deferred layer."""
    from host_memory_streamed_layer_b200 import arena, mt
    sh = dict(L=5, d=256, H=4, Hkv=4, F=688, V=1024, b=2, s=128)
    if env is None:
        monkeypatch.delenv("MT_DEFER_LAYERS", raising=False)
    else:
        monkeypatch.setenv("MT_DEFER_LAYERS", env)
    cfg = arena.config(sh)
    cfg.flags = mt.MT_FLAG_GRAD_RING
    ring = mt.mt_host_state_bytes(cfg)
    cfg.flags |= mt.MT_FLAG_DEFER_UPDATES
    layer_bytes = 4 * (mt.mt_tensor_offset(cfg, 1, 0)[0] - mt.mt_tensor_offset(cfg, 0, 0)[0])
    assert mt.mt_host_state_bytes(cfg) - ring == bench.defer_layers(sh) * layer_bytes


def test_attention_stash_removes_the_recomputed_attention_forwards():
    """With MT_FLAG_STASH_ATTN the schedule executes L-1 fewer causal attention
    forwards (2 b s^2 H hd FLOPs each), all in the backward phase; the model
    FLOPs do not change."""
    sh = synth.WORKLOADS["llama-7b-128k"]
    A = 2.0 * sh["b"] * sh["s"] ** 2 * sh["H"] * (sh["d"] // sh["H"])
    f0, b0 = bench.phase_flops(sh)
    f1, b1 = bench.phase_flops(sh, stash=True)
    assert f1 == f0 and b0 - b1 == pytest.approx((sh["L"] - 1) * A)
    m0, e0 = bench.flops_per_step(sh)
    m1, e1 = bench.flops_per_step(sh, stash=True)
    assert m1 == m0 and e0 - e1 == pytest.approx((sh["L"] - 1) * A)
    assert e0 == pytest.approx(f0 + b0)


def test_expert_workload_counts():
    """Expert layers: the bench's parameter count is the arena's, a token's
    MLP FLOPs count topk experts plus the router, and the recompute includes
    the experts' down projections (the gates' gradients need their outputs)."""
    from host_memory_streamed_layer_b200 import arena, mt
    sh = synth.WORKLOADS["moe-8x1408"]
    cfg = arena.config(sh)
    n_layer = sum(mt.mt_tensor_offset(cfg, 0, t)[1] for t in range(10))
    assert bench.layer_params(sh) == n_layer
    d, F, E, k, L, T = sh["d"], sh["F"], sh["E"], sh["topk"], sh["L"], sh["b"] * sh["s"]
    assert bench.mlp_active(sh) == 3 * d * F * k + E * d and bench.recompute_skip(sh) == 0
    dense = {key: v for key, v in sh.items() if key not in ("E", "topk")}
    m1, e1 = bench.flops_per_step(sh)
    m0, e0 = bench.flops_per_step(dense)
    assert m1 - m0 == pytest.approx(L * 6.0 * T * (bench.mlp_active(sh) - 3 * d * F))
    f1, b1 = bench.phase_flops(sh)
    assert e1 == pytest.approx(f1 + b1)
