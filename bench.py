#!/usr/bin/env python
"""Benchmark of one host-memory-streamed training step (MegaTrain's method).

One step = forward over every streamed layer, LM head and cross-entropy,
checkpointed recompute and backward, gradient offload and the host AdamW
update, on a Llama-style decoder whose fp32 master weights and Adam moments
live in host memory. Default workload: the 1.3B decoder (24 layers, d 2048,
16 heads, SwiGLU 5504, vocab 32000) on 8 x 2048 tokens per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   (the fp64 CPU oracle, bounded sample)

Prints one JSON line on rank 0. With N > 1 (torchrun, one process per GPU)
every rank trains an independent replica (the method runs on one GPU; no
collective is on the data path) and `value` is the sum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import platform
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "training tokens/s"
UNIT = "tokens/s"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per GEMM launch of
# a step, averaged over the step's GEMM launches with each shape weighted by its
# launches per step. Taken from single-kernel captures: one launch of every
# GEMM shape of the workload through the kernel micro-benchmark
# (`python -m host_memory_streamed_layer_b200.kernel_bench gemm --workload W
# --iters 1 --warmup 0`, at most a few GB on the device), never from a
# full-size training run. Workloads without a capture report null, and so does
# a workload whose GEMM kernels changed after its capture.
GEMM_TRAFFIC_PER_LAUNCH = {"gqa-14b": 1257.6e6, "llama-1.3b": 497.3e6}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=None, choices=list(synth.WORKLOADS),
                    help="default: the largest workload whose host state fits this host's memory "
                         "(gqa-14b, else llama-7b, else llama-1.3b)")
    ap.add_argument("--impl", default="mt", choices=["mt", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--timeline", default="", metavar="PATH",
                    help="write the last step's copy/compute timeline (Markdown) to PATH")
    ap.add_argument("--grads", default="ring", choices=["ring", "arena"],
                    help="host gradients: ring of layer slots (14 B/param of host memory) or a full arena (18)")
    ap.add_argument("--host-threads", type=int, default=0, help="host optimizer threads per replica (0: cores / N)")
    ap.add_argument("--offload-acts", action="store_true",
                    help="keep the boundary activations in pinned host memory (MT_FLAG_OFFLOAD_ACTS)")
    ap.add_argument("--shard", action="store_true",
                    help="sharded streaming over the N ranks (mt_create_sharded): each loads, offloads and updates "
                         "1/N of the state, all-gather / reduce-scatter over NCCL")
    ap.add_argument("--attn-bwd", default="auto", choices=["auto", "fused", "split"],
                    help="attention backward: dQ by reductions (fused) or the deterministic split")
    ap.add_argument("--stash-attn", action="store_true",
                    help="keep each layer's attention output for its backward (MT_FLAG_STASH_ATTN)")
    ap.add_argument("--grad-dtype", default="fp32", choices=["fp32", "bf16"],
                    help="dtype of the offloaded gradients (bf16: MT_FLAG_BF16_GRADS, a measured variant)")
    ap.add_argument("--no-defer", action="store_true",
                    help="run every update inside its own step (no MT_FLAG_DEFER_UPDATES)")
    return ap.parse_args()


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# Default workloads, largest first: the 14B decoder is the size of the pages'
# only throughput claim (MegaTrain abstract: 1.84x DeepSpeed ZeRO-3 with CPU
# offload when training 14B models).
DEFAULT_ORDER = ("gqa-14b", "llama-7b", "llama-1.3b")


def host_need_bytes(sh, world=1, ring=True, deferred=1):
    """Host bytes of one replica (an estimate of mt_arena_bytes +
    mt_host_state_bytes, used only to choose the default workload): fp32
    master, two fp32 moments and the bf16 streaming copy (14 B/param), the
    gradient ring of MT_GRAD_RING_SLOTS + deferred layer slots (or a full fp32
    gradient arena), the LM-head gradients and the embedding-gradient staging."""
    P = sh["L"] * layer_params(sh) + 2 * sh["V"] * sh["d"] + sh["d"]
    grads = (3 + deferred) * layer_params(sh) * 4 + head_params(sh) * 4 if ring else 4 * P
    return 14 * P + grads + 4 * sh["b"] * sh["s"] * sh["d"]


def available_host_bytes():
    try:
        import psutil
        return psutil.virtual_memory().available
    except Exception:
        return None


def pick_workload(args, avail, world=1):
    """(workload name, note): --workload when given, else the first of
    DEFAULT_ORDER whose host state fits the available host memory."""
    if args.workload:
        return args.workload, "as requested"
    if avail is None:
        avail = available_host_bytes()
    for name in DEFAULT_ORDER:
        if host_ram_fits(host_need_bytes(synth.WORKLOADS[name]), world, avail):
            note = ("the largest benchmark workload" if name == DEFAULT_ORDER[0] else
                    f"the largest benchmark workload whose host state fits this host "
                    f"({(avail or 0) / 1e9:.0f} GB available)")
            return name, note
    return DEFAULT_ORDER[-1], "the smallest benchmark workload (none fits the host's free memory)"


def mlp_active(sh):
    """Matrix parameters a token runs through in one layer's MLP: the dense
    SwiGLU, or topk experts' plus the router."""
    E = sh.get("E", 0)
    return 3 * sh["d"] * sh["F"] * (sh["topk"] if E else 1) + E * sh["d"]


def recompute_skip(sh):
    """Matrix parameters the recompute leaves out: the dense MLP's down
    projection (the backward needs only its input); expert layers recompute
    it (the gates' gradients need the experts' outputs)."""
    return 0 if sh.get("E", 0) else sh["d"] * sh["F"]


def workload_desc(name, sh):
    experts = f", {sh['E']} experts top-{sh['topk']}" if sh.get("E", 0) else ""
    return (f"{name}: {sh['L']} layers, d {sh['d']}, {sh['H']} heads ({sh['Hkv']} kv), SwiGLU {sh['F']}{experts}, "
            f"vocab {sh['V']}, {sh['b']} x {sh['s']} tokens per GPU; fp32 master + AdamW moments in host RAM, "
            f"bf16 weights streamed per layer")


def flops_per_step(sh, stash=False):
    """Model FLOPs (6 N T with causal attention) and the FLOPs this schedule
    executes (forward, recompute without the down projection, and without the
    attention with stash (MT_FLAG_STASH_ATTN), backward, flash-attention
    backward recompute, LM head)."""
    L, d, H, Hkv, F, V, b, s = (sh[k] for k in ("L", "d", "H", "Hkv", "F", "V", "b", "s"))
    hd = d // H
    T = b * s
    Pm = d * (H + 2 * Hkv) * hd + d * H * hd + mlp_active(sh)
    A = 2.0 * b * s * s * H * hd  # causal attention forward (QK^T and PV over the visible half)
    model = L * (6.0 * T * Pm + 3 * A) + 6.0 * T * V * d
    executed = L * (2.0 * T * Pm + A) + (L - 1) * (2.0 * T * (Pm - recompute_skip(sh)) + (0 if stash else A)) \
        + L * (4.0 * T * Pm + 2.5 * A) + 6.0 * T * V * d
    return model, executed


# ---------------------------------------------------------------------------
# Clock sampling during the timed region.
# ---------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the same workload.
# ---------------------------------------------------------------------------
def oracle_sample_plan(sh):
    """Sizes of a bounded oracle sample of one training step of workload sh
    (about 3-8 s of fp64 work on 16 cores): one sequence of s_smp tokens
    through one decoder layer forward + backward, the final norm + LM head +
    cross-entropy forward/backward on t_head tokens over v_head vocabulary
    rows, and AdamW over n_adam parameters. Each part is scaled to the full
    step by the oracle's own operation count: per sequence of s tokens the
    layer costs 6 s P_mat for its matrices plus 12 s^2 H hd for attention (the
    oracle forms the full s x s score matrix), the head 6 T V d, AdamW a
    constant per parameter."""
    hd = sh["d"] // sh["H"]
    pm = sh["d"] * (sh["H"] + 2 * sh["Hkv"]) * hd + sh["d"] * sh["H"] * hd + mlp_active(sh)
    s_smp = min(sh["s"], 2048 if pm < 1e8 and not sh.get("E", 0) else 512)  # (expert layers: slower per token)
    v_head = min(sh["V"], 32000)
    t_head = int(min(sh["b"] * sh["s"], max(64, 0.6e12 / (6.0 * v_head * sh["d"]) // 64 * 64)))
    p_layer = layer_params(sh)
    p_total = sh["L"] * p_layer + 2 * sh["V"] * sh["d"] + sh["d"]
    n_adam = min(p_layer, 1 << 24)

    def layer_ops(s):
        return 6.0 * s * pm + 12.0 * s * s * sh["H"] * hd

    return dict(s_smp=s_smp, t_head=t_head, v_head=v_head, n_adam=n_adam,
                layer_scale=sh["b"] * sh["L"] * layer_ops(sh["s"]) / layer_ops(s_smp),
                head_scale=(sh["b"] * sh["s"] / t_head) * (sh["V"] / v_head),
                adam_scale=p_total / n_adam, p_total=p_total)


class OracleSample:
    """Inputs of the bounded oracle sample, drawn once; run() times the oracle
    on them and returns (extrapolated tokens/s, seconds measured, description)."""

    def __init__(self, sh, seed=0):
        import oracle
        self.o, self.sh, self.plan = oracle, sh, oracle_sample_plan(sh)
        pl = self.plan
        self.c = oracle.OracleConfig(**{**sh, "b": 1, "L": 1, "s": pl["s_smp"]})
        c, hd = self.c, self.c.d // self.c.H
        self.W = {tid: synth.init_tensor(seed, 0, tid, shp).astype(np.float64)
                  for tid, shp in synth.layer_shapes(c.d, c.H, c.Hkv, c.F, hd, c.E)}
        rng = np.random.default_rng(seed)
        self.x = rng.normal(size=(1, c.s, c.d))
        self.dx = rng.normal(size=self.x.shape)
        self.cos, self.sin = oracle.rope_tables(c.s, hd, c.rope_base)
        self.xh = rng.normal(size=(pl["t_head"], c.d))
        self.Wh = synth.init_tensor(seed, -1, synth.LM_HEAD, (pl["v_head"], c.d)).astype(np.float64)
        self.lab = rng.integers(0, pl["v_head"], pl["t_head"])
        n = pl["n_adam"]
        self.p = rng.normal(size=n) * 0.02
        self.g = rng.normal(size=n) * 1e-4

    def run(self):
        o, c, pl, sh = self.o, self.c, self.plan, self.sh
        t0 = time.perf_counter()
        _, cache = o.layer_fwd(self.x, self.W, c, self.cos, self.sin)
        o.layer_bwd(self.dx, self.W, cache, c, self.cos, self.sin)
        t_layer = time.perf_counter() - t0
        t0 = time.perf_counter()
        o.head_ce_fwd_bwd(self.xh, np.ones(c.d), self.Wh, self.lab, c.norm_eps)
        t_head = time.perf_counter() - t0
        t0 = time.perf_counter()
        o.adamw_update(self.p, self.g, np.zeros_like(self.p), np.zeros_like(self.p), 1, c.lr, c.beta1, c.beta2,
                       c.adam_eps, c.wd)
        t_adam = time.perf_counter() - t0
        t_step = pl["layer_scale"] * t_layer + pl["head_scale"] * t_head + pl["adam_scale"] * t_adam
        T = sh["b"] * sh["s"]
        desc = (f"oracle (fp64 numpy), measured: one decoder layer fwd+bwd on one {pl['s_smp']}-token sequence "
                f"{t_layer:.2f}s, final norm + LM head + CE fwd+bwd on {pl['t_head']} tokens x {pl['v_head']} vocab "
                f"rows {t_head:.2f}s, AdamW over {pl['n_adam'] / 1e6:.1f}M params {t_adam:.2f}s; extrapolated by "
                f"the oracle's operation count to {sh['b']} x {sh['s']} tokens, {sh['L']} layers, vocab {sh['V']} "
                f"and AdamW over {pl['p_total'] / 1e9:.3f}B params ({t_step:.0f}s per step)")
        return T / t_step, t_layer + t_head + t_adam, desc, t_step


def oracle_sample_tokens_per_s(sh, seed=0):
    """One bounded oracle sample (see OracleSample): (tokens/s, seconds, description)."""
    v, secs, desc, _ = OracleSample(sh, seed).run()
    return v, secs, desc


def cpu_model() -> str:
    """The host CPU's model name, as the kernel reports it."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def step_spread(stats):
    """Min and median over the timed steps of each step's host wall time
    (the mt_train_step call) and compute-stream time (device events)."""
    out = {}
    for key, name in (("host_step_ms", "host_ms"), ("step_ms", "device_ms")):
        v = [float(st[key]) for st in stats]
        if v:
            out[name + "_min"] = min(v)
            out[name + "_median"] = statistics.median(v)
    return out


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# Reference arm: the oracle as it stands, bounded samples.
# ---------------------------------------------------------------------------
def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores: every step (warm-up
    and timed) is one bounded sample of the workload (OracleSample), whose
    measured time is the line's ms_per_step; value is the full step's tokens/s
    extrapolated from the sample by the oracle's operation count."""
    if rank != 0:
        return
    wname, wnote = pick_workload(args, None)
    sh = synth.WORKLOADS[wname]
    smp = OracleSample(sh)
    for _ in range(args.warmup):
        smp.run()
    vals, secs, full = [], [], []
    desc = ""
    for _ in range(args.steps):
        v, sec, desc, t_full = smp.run()
        vals.append(v)
        secs.append(sec)
        full.append(t_full)
    value = statistics.median(vals)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": statistics.median(secs) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(wname, sh), "workload_choice": wnote, "global_batch": sh["b"],
                   "seq_len": sh["s"], "parallelism": "none (CPU)"},
        "timing": ("ms_per_step is the measured wall time of one bounded sample; value extrapolates the sample "
                   "to the full step"),
        "extrapolated_ms_per_full_step": statistics.median(full) * 1e3,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Link bandwidth (pinned 1 GiB copies, best of 3) measured in the same run.
# ---------------------------------------------------------------------------
def link_bandwidth(torch, dev):
    n = 1 << 30
    h = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    h2 = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(n, dtype=torch.uint8, device=dev)
    d2 = torch.empty(n, dtype=torch.uint8, device=dev)
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def best(fn):
        b = 1e9
        for _ in range(3):
            torch.cuda.synchronize(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            b = min(b, e0.elapsed_time(e1) / 1e3)
        return b

    def h2d():
        d.copy_(h, non_blocking=True)

    def d2h():
        h.copy_(d, non_blocking=True)

    def both():
        cur = torch.cuda.current_stream(dev)
        s1.wait_stream(cur)
        s2.wait_stream(cur)
        with torch.cuda.stream(s1):
            d.copy_(h, non_blocking=True)
        with torch.cuda.stream(s2):
            h2.copy_(d2, non_blocking=True)
        cur.wait_stream(s1)
        cur.wait_stream(s2)

    r = {"h2d_gbs": n / best(h2d) / 1e9, "d2h_gbs": n / best(d2h) / 1e9, "bidir_gbs_each": n / best(both) / 1e9}
    del h, h2, d, d2
    torch.cuda.empty_cache()
    # give the pinned staging buffers back to the OS before the context pins its own
    for fn in (getattr(torch._C, "_host_emptyCache", None), getattr(torch.cuda, "host_empty_cache", None)):
        if fn is not None:
            fn()
            break
    return r


def host_optimizer_bandwidth(mt, threads, n=1 << 28):
    """GB/s (30 B/param accounting) of the library's host AdamW on its own
    worker pool over 4 x 1 GiB fp32 arrays, best of 3: the host-DRAM ceiling
    the optimizer can reach when nothing else uses memory."""
    return mt.mt_host_optimizer_gbs(n, threads)


def write_timeline(tl, path, workload):
    """Markdown timeline of one step: weight loads against the compute stream,
    gradient offloads, and the host optimizer jobs."""
    ph = tl["phases"]
    out = [f"# Step timeline: {workload}, 1 B200", "",
           "Device times in ms from the step's start on the compute stream (CUDA events); host optimizer",
           "times in ms of host clock from the mt_train_step call (the two origins agree to tens of us).", "",
           f"Phases: forward ends {ph['fwd_end']:.2f}, head ends {ph['head_end']:.2f}, backward ends "
           f"{ph['bwd_end']:.2f}, step ends {ph['step_end']:.2f}.", "",
           "## Weight loads (H2D stream) against the compute stream", "",
           "| load | layer | H2D start | weights ready | compute reaches its wait | compute waits | slot released |",
           "|---:|---:|---:|---:|---:|---:|---:|"]
    wait_total = 0.0
    for i, ld in enumerate(tl["loads"]):
        w = max(0.0, ld["ready"] - ld["compute_arrives"])
        wait_total += w
        out.append(f"| {i} | {ld['layer']} | {ld['h2d_start']:.2f} | {ld['ready']:.2f} | {ld['compute_arrives']:.2f} "
                   f"| {w:.3f} | {ld['released']:.2f} |")
    out += ["", f"Compute stream waiting for weights in this step: {wait_total:.3f} ms.", "",
            "## Gradient offloads (D2H stream)", "",
            "| layer | gradients ready | D2H start | D2H done |", "|---:|---:|---:|---:|"]
    for o in tl["offload"]:
        out.append(f"| {o['layer']} | {o['grads_ready']:.2f} | {o['d2h_start']:.2f} | {o['d2h_done']:.2f} |")
    kinds = {0: "layer", 1: "LM head", 2: "embedding (touched rows)", 3: "embedding (untouched rows)",
             4: "LM head, previous step's deferred update", 5: "layer, previous step's deferred update",
             6: "untouched embedding rows, previous step's deferred update",
             7: "previous step's untouched rows that this step gathers (before its GPU work)"}
    deferred = {j["layer"] for j in tl["jobs"] if j["kind"] == 5}
    has_head = any(j["kind"] == 4 for j in tl["jobs"])
    out += ["", "## Host optimizer jobs (host clock)", "",
            "| job | layer | gradients available | update done |", "|---|---:|---:|---:|"]
    for j in tl["jobs"]:
        name = kinds.get(j["kind"], j["kind"])
        if (j["kind"] == 0 and j["layer"] in deferred) or (j["kind"] == 1 and has_head):
            name += " (finite check; update deferred)"
        out.append(f"| {name} | {j['layer'] if j['kind'] in (0, 5) else ''} "
                   f"| {j['ready_ms']:.2f} | {j['done_ms']:.2f} |")
    with open(path, "w") as f:
        f.write("\n".join(out) + "\n")


def step_bounds(sh, *, peak_tflops, link, host_gbs, h2d_bytes, d2h_bytes, update_bytes, n_unique,
                deferred_layers=None, stash=False):
    """Phase bound of this method's dependency structure (seconds).

    The forward sweep and head (GPU compute or weight H2D, whichever is slower)
    must finish before any gradient of the step exists. The backward (GPU
    compute, D2H over the link) then runs alongside the host updates that need
    this step's gradients, whose bytes move at most at host_gbs, the rate the
    library's AdamW reaches alone on this host. The untouched embedding rows
    and, with deferral (deferred_layers not None), the previous step's LM-head
    and last-layer updates run during the forward sweep instead; all of the
    step's update bytes at host_gbs bound the step as well.

    "model" is not a bound: it adds the copies' host DRAM traffic (pinned memory
    is read by every H2D and written by every D2H) to the optimizer's at the
    same rate, and measured steps beat it where DMA and CPU traffic together
    draw more from host DRAM than the CPU alone."""
    f_fl, b_fl = phase_flops(sh, stash)
    L = sh["L"]
    peak = peak_tflops * 1e12
    h2d_fwd = h2d_bytes * L / (2 * L - 1)
    upd_fwd = 30.0 * (sh["V"] - n_unique) * sh["d"]
    if deferred_layers is not None:
        upd_fwd += 30.0 * (head_params(sh) + deferred_layers * layer_params(sh))
    upd_bwd = update_bytes - upd_fwd
    t_d2h = d2h_bytes / (link["d2h_gbs"] * 1e9)
    fwd = max(f_fl / peak, h2d_fwd / (link["h2d_gbs"] * 1e9))
    host_bwd = upd_bwd / (host_gbs * 1e9)
    bwd = max(b_fl / peak, t_d2h, host_bwd)
    dram_fwd = upd_fwd + h2d_fwd
    dram_bwd = upd_bwd + (h2d_bytes - h2d_fwd) + d2h_bytes
    model = max(fwd, dram_fwd / (host_gbs * 1e9)) + max(b_fl / peak, t_d2h, dram_bwd / (host_gbs * 1e9))
    return dict(fwd=fwd, bwd=bwd, host_bwd=host_bwd, bound=max(fwd + bwd, update_bytes / (host_gbs * 1e9)),
                update_bytes=update_bytes, update_bytes_fwd=upd_fwd, update_bytes_bwd=upd_bwd,
                model=model, dram_fwd=dram_fwd, dram_bwd=dram_bwd)


def defer_layers(sh):
    """Deferred layers as the library reads them: MT_DEFER_LAYERS (default 1)
    parsed like strtol (leading integer, else 0), clamped to [0, L-1]."""
    env = os.environ.get("MT_DEFER_LAYERS")
    if env is None:
        n = 1
    else:
        m = re.match(r"\s*([+-]?\d+)", env)
        n = int(m.group(1)) if m else 0
    return min(max(n, 0), sh["L"] - 1)


def layer_params(sh):
    hd = sh["d"] // sh["H"]
    E = sh.get("E", 0)
    mlp = (3 * sh["d"] * sh["F"] + sh["d"]) * E if E else 3 * sh["d"] * sh["F"]
    return sh["d"] * (sh["H"] + 2 * sh["Hkv"]) * hd + sh["d"] * sh["H"] * hd + mlp + 2 * sh["d"]


def head_params(sh):
    return sh["d"] + sh["V"] * sh["d"]


def phase_flops(sh, stash=False):
    """(forward + head FLOPs, backward-phase FLOPs) of the schedule (stash: the
    recompute runs no attention forward)."""
    L, d, H, Hkv, F, V, b, s = (sh[k] for k in ("L", "d", "H", "Hkv", "F", "V", "b", "s"))
    hd = d // H
    T = b * s
    Pm = d * (H + 2 * Hkv) * hd + d * H * hd + mlp_active(sh)
    A = 2.0 * b * s * s * H * hd
    fwd = L * (2.0 * T * Pm + A) + 6.0 * T * V * d
    bwd = (L - 1) * (2.0 * T * (Pm - recompute_skip(sh)) + (0 if stash else A)) + L * (4.0 * T * Pm + 2.5 * A)
    return fwd, bwd


# ---------------------------------------------------------------------------
# Cross-rank helpers: one process per GPU, replicas with no data-path
# collective. NCCL on the GPU run; the CPU tests drive the same code on gloo.
# ---------------------------------------------------------------------------
class Ranks:
    def __init__(self, torch, dist=None, device=None):
        self.torch, self.dist, self.device = torch, dist, device

    def allmax(self, x: float) -> float:
        """Maximum of x over the ranks (the timed region is the slowest rank's)."""
        if self.dist is None:
            return float(x)
        t = self.torch.tensor([float(x)], device=self.device, dtype=self.torch.float64)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def all_ok(self, ok: bool) -> bool:
        """True only if every rank passes ok=True: every rank takes the same branch."""
        return -self.allmax(-1.0 if ok else 0.0) >= 1.0

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()


def host_ram_fits(need_bytes: int, world: int, avail_bytes, margin_bytes: int = 6 << 30) -> bool:
    """Every replica holds its own host state: N replicas fit when N times one
    replica's bytes plus a margin stay under the host's available memory."""
    return avail_bytes is None or need_bytes * world + margin_bytes < avail_bytes


def weak_value(tokens_per_rank_step: int, world: int, steps: int, t_max_s: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank_step * world * steps / t_max_s


# ---------------------------------------------------------------------------
# Main arm.
# ---------------------------------------------------------------------------
def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    from datetime import timedelta
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)

    ranks = Ranks(torch, dist, dev)
    allmax, barrier = ranks.allmax, ranks.barrier

    from host_memory_streamed_layer_b200 import arena, mt
    # every rank takes the same decision (rank 0's host-memory reading)
    avail_r0 = ranks.allmax(float(available_host_bytes() or 0) if rank == 0 else 0.0) or None
    wname, wnote = pick_workload(args, avail_r0, world)
    args.workload = wname
    sh = synth.WORKLOADS[args.workload]
    T = sh["b"] * sh["s"]
    cfg = arena.config(sh)
    cfg.seed = 1234 if args.shard else 1234 + rank  # one model over the ranks, or N replicas
    cfg.device = local
    # Gradients stream through a ring of host slots (14 instead of 18 B/param of
    # host memory): the 14B workload then fits a ~200 GB host, and so do eight
    # 1.3B replicas.
    # The LM head's and the last layer's updates overlap the next forward sweep
    # (MT_FLAG_DEFER_UPDATES), when the host optimizer is otherwise idle.
    cfg.flags = (mt.MT_FLAG_KERNEL_TIMING | (mt.MT_FLAG_GRAD_RING if args.grads == "ring" else 0) |
                 (0 if args.no_defer else mt.MT_FLAG_DEFER_UPDATES) |
                 (mt.MT_FLAG_BF16_GRADS if args.grad_dtype == "bf16" else 0) |
                 (mt.MT_FLAG_OFFLOAD_ACTS if args.offload_acts else 0) |
                 (mt.MT_FLAG_STASH_ATTN if args.stash_attn else 0))
    ncpu = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cfg.host_threads = args.host_threads or max(1, ncpu // world)

    # Host memory: every replica holds its own master, moments, gradients and bf16 copy.
    need = mt.mt_arena_bytes(cfg) + mt.mt_host_state_bytes(cfg)
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = None
    if not ranks.all_ok(host_ram_fits(need, world, avail)):
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": None, "unit": UNIT, "n_gpus": world,
                              "error": f"host RAM: {world} replicas need {need * world / 1e9:.0f} GB, "
                                       f"{(avail or 0) / 1e9:.0f} GB available"}), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return

    link = link_bandwidth(torch, dev) if rank == 0 else None
    host_bw = host_optimizer_bandwidth(mt, cfg.host_threads) if rank == 0 else None
    # independent host-DRAM ceiling: STREAM triad (12 B/element, non-temporal stores)
    triad = mt.mt_host_triad_gbs(1 << 28, cfg.host_threads) if rank == 0 else None
    mt.mt_k_attn_bwd_variant({"auto": mt.ATTN_BWD_AUTO, "fused": mt.ATTN_BWD_FUSED,
                              "split": mt.ATTN_BWD_SPLIT}[args.attn_bwd])
    if args.shard:
        nccl_id = mt.mt_shard_id() if rank == 0 else bytes(mt.MT_SHARD_ID_BYTES)
        if dist is not None:
            box = [nccl_id]
            dist.broadcast_object_list(box, src=0)
            nccl_id = box[0]
        ctx = mt.mt_create_sharded(cfg, 0, 0, world, rank, nccl_id)
    else:
        ctx = mt.mt_create(cfg)
    try:
        n_e2e = max(3, (args.steps + 1) // 2)
        nsteps = args.warmup + args.steps + n_e2e
        toks = []
        for i in range(nsteps):
            t, l = synth.tokens_labels(sh["b"], sh["s"], sh["V"], seed=rank, step=i)
            tt = torch.from_numpy(t).pin_memory()
            ll = torch.from_numpy(l).pin_memory()
            toks.append((tt, ll))
        # distinct token ids of a timed step: the embedding rows that get a gradient
        n_uniq = sum(int(torch.unique(toks[i][0]).numel())
                     for i in range(args.warmup, args.warmup + args.steps)) / args.steps
        for i in range(args.warmup):
            mt.mt_train_step(ctx, toks[i][0].data_ptr(), toks[i][1].data_ptr())
        stream = torch.cuda.ExternalStream(mt.mt_get_stream(ctx), device=dev)

        # -------- timed region: device events on the engine's compute stream --------
        clocks = Clocks(local)
        clocks.start()
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        stats = []
        losses = []
        for i in range(args.warmup, args.warmup + args.steps):
            losses.append(mt.mt_train_step(ctx, toks[i][0].data_ptr(), toks[i][1].data_ptr()))
            stats.append(mt.mt_get_stats(ctx))
        # the last step's deferred updates run inside the timed region (the
        # first timed step already ran the last warm-up step's)
        mt.mt_flush(ctx)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        clk = clocks.stop()
        t_dev = allmax(e0.elapsed_time(e1) / 1e3)

        # -------- end-to-end: host clock around the public call, host buffers --------
        barrier()
        torch.cuda.synchronize(dev)
        w0 = time.perf_counter()
        for i in range(args.warmup + args.steps, nsteps):
            losses.append(mt.mt_train_step(ctx, toks[i][0].data_ptr(), toks[i][1].data_ptr()))
        mt.mt_flush(ctx)
        w1 = time.perf_counter()
        barrier()
        t_e2e = allmax(w1 - w0)
        if args.timeline and rank == 0:
            write_timeline(mt.mt_get_timeline(ctx), args.timeline, args.workload)
    finally:
        mt.mt_destroy(ctx)

    if rank == 0:
        P, ptype = peaks()
        model_f, exec_f = flops_per_step(sh, args.stash_attn)
        K = args.steps
        value = weak_value(T, world, K, t_dev)
        ms = t_dev / K * 1e3
        g_fl = sum(s["gemm_flops"] for s in stats)
        g_ms = sum(s["gemm_ms"] for s in stats)
        g_n = sum(s["gemm_launches"] for s in stats)
        a_fl = sum(s["attn_flops"] for s in stats)
        a_ms = sum(s["attn_ms"] for s in stats)
        achieved = g_fl / (g_ms / 1e3) / 1e12 if g_ms > 0 else None
        peak = P["bf16_tflops_sustained"]
        mean = lambda k: sum(s[k] for s in stats) / len(stats)  # noqa: E731
        h2d_b, d2h_b = mean("h2d_bytes"), mean("d2h_bytes")
        t_compute = exec_f / (peak * 1e12)
        t_h2d = h2d_b / (link["h2d_gbs"] * 1e9)
        t_d2h = d2h_b / (link["d2h_gbs"] * 1e9)
        sb = step_bounds(sh, peak_tflops=peak, link=link, host_gbs=host_bw, h2d_bytes=h2d_b, d2h_bytes=d2h_b,
                         update_bytes=mean("adamw_bytes"), n_unique=n_uniq,
                         deferred_layers=None if args.no_defer else defer_layers(sh), stash=args.stash_attn)
        host_bytes, upd_fwd, upd_bwd = sb["update_bytes"], sb["update_bytes_fwd"], sb["update_bytes_bwd"]
        t_fwd_b, t_bwd_b, t_host_b, t_bound = sb["fwd"], sb["bwd"], sb["host_bwd"], sb["bound"]
        t_model, dram_fwd, dram_bwd = sb["model"], sb["dram_fwd"], sb["dram_bwd"]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (uniform random tokens from seed, N(0,0.02) weights)",
            "config": {"workload": workload_desc(args.workload, sh), "workload_choice": wnote,
                       "global_batch": sh["b"] * world,
                       "seq_len": sh["s"],
                       "parallelism": (f"sharded streaming over {world} rank(s) (NCCL all-gather / reduce-scatter)"
                                       if args.shard else "replicas" if world > 1 else "single GPU"),
                       "l2": "no flush needed: every step streams all weights (>1 GB) through HBM from host",
                       "deferred_updates": (None if args.no_defer else
                                            f"LM head + last {defer_layers(sh)} layer(s) updated during the next "
                                            "forward sweep; the timed region ends after mt_flush"),
                       "boundary_activations": "pinned host memory" if args.offload_acts else "HBM",
                       "attention_recompute": ("none: O and LSE kept per layer (MT_FLAG_STASH_ATTN)"
                                               if args.stash_attn else "in each layer's recompute"),
                       "attention_backward": ("fused: dQ by fp32 reductions" if args.attn_bwd == "fused"
                                              else "split: dK/dV key-major, dQ query-major, deterministic"),
                       "grads": (f"{args.grad_dtype} gradients offloaded; " +
                                 (f"ring of {mt.MT_GRAD_RING_SLOTS} layer slots in pinned host memory"
                                  if args.grads == "ring" else "full gradient arena in pinned host memory"))},
            "model_tflops": model_f * world / (t_dev / K) / 1e12,
            "executed_tflops": exec_f * world / (t_dev / K) / 1e12,
            "roofline": {"bound": "tensor", "kernel": "tcgen05 bf16 GEMM (all projections, fwd/dX/dW)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": (achieved / peak) if achieved else None,
                         "traffic": GEMM_TRAFFIC_PER_LAUNCH.get(args.workload),
                         "peak_kind": f"bf16_tflops_sustained ({ptype})",
                         "launches_per_step": g_n / K, "gemm_ms_per_step": g_ms / K},
            "step_roofline": {"bound_ms": t_bound * 1e3, "frac": t_bound / (t_dev / K),
                              # compute / host-link only (no host-optimizer term)
                              "compute_link_bound_ms": max(t_compute, t_h2d, t_d2h) * 1e3,
                              "compute_link_frac": max(t_compute, t_h2d, t_d2h) / (t_dev / K),
                              "fwd_bound_ms": t_fwd_b * 1e3, "bwd_bound_ms": t_bwd_b * 1e3,
                              "host_bytes": host_bytes, "host_bound_ms": t_host_b * 1e3,
                              "update_bytes_fwd": upd_fwd, "update_bytes_bwd": upd_bwd,
                              "n_unique_tokens": n_uniq,
                              "host_dram_model": {"ms": t_model * 1e3, "ratio": t_model / (t_dev / K),
                                                  "bytes_fwd": dram_fwd, "bytes_bwd": dram_bwd},
                              "host_optimizer_gbs_measured": host_bw,
                              "host_triad_gbs": triad,
                              "host_adamw_frac_of_triad": (mean("adamw_bytes") / max(mean("adamw_ms"), 1e-9) / 1e6
                                                           / triad) if triad else None,
                              "compute_ms": t_compute * 1e3, "h2d_ms": t_h2d * 1e3, "d2h_ms": t_d2h * 1e3,
                              "link_measured": link, "h2d_bytes": h2d_b, "d2h_bytes": d2h_b,
                              "attention_tflops": a_fl / (a_ms / 1e3) / 1e12 if a_ms > 0 else None,
                              "attention_ms_per_step": a_ms / K,
                              "gpu_step_ms": mean("step_ms"), "fwd_ms": mean("fwd_ms"), "head_ms": mean("head_ms"),
                              "bwd_ms": mean("bwd_ms"), "wait_weights_ms": mean("wait_weights_ms"),
                              "host_adamw_ms": mean("adamw_ms"), "host_adamw_gbs": mean("adamw_bytes") /
                              max(mean("adamw_ms"), 1e-9) / 1e6, "host_threads": cfg.host_threads,
                              "host_step_ms": mean("host_step_ms"), "adamw_first_ms": mean("adamw_first_ms"),
                              "adamw_last_ms": mean("adamw_last_ms"), "enqueue_ms": mean("enqueue_ms")},
            "loss": losses[-1],
            "parity": {"loss_abs": 1e-2, "grad_rel_l2": 2e-2, "updated_param_rel_l2": {
                "target": 1e-3, "met": False, "tested": 5e-3,
                "why": "the first Adam step is ~lr*sign(g); bf16 operands put its floor at ~2.5e-3 and every bf16 "
                       "rounding point alone (stored activations, stored gradients, attention P/dS) exceeds 1e-3"}},
            "clocks": clk,
            "e2e": {"value": weak_value(T, world, n_e2e, t_e2e), "unit": UNIT, "h2d_bytes_per_step": 2 * T * 4,
                    "d2h_bytes_per_step": 4, "steps": n_e2e,
                    "timing": "host wall clock around mt_train_step (public C API), pinned host tokens in, loss out"},
            "gpu_launches": int(sum(s["kernel_launches"] for s in stats)),
            "per_step": step_spread(stats),
        }
        if world == 1 and not args.no_cpu_baseline:
            # host-side only, after the GPU work: the bounded sample, repeated
            # until about 10 s of oracle time (at most 10 times), median
            smp, vals, secs, desc = OracleSample(sh), [], 0.0, ""
            while secs < 10.0 and len(vals) < 10:
                v, sec, desc, _ = smp.run()
                vals.append(v)
                secs += sec
            line["cpu_baseline"] = {"value": statistics.median(vals), "unit": UNIT, "cores": blas_threads(),
                                    "cpu_model": cpu_model(), "kind": "oracle", "sample": desc, "seconds": secs,
                                    "repeats": len(vals)}
        print(json.dumps(line), flush=True)
    if dist is not None:
        barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
