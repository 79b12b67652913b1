"""Micro-benchmark of single hot-path kernels through the C ABI.

    python -m host_memory_streamed_layer_b200.kernel_bench gemm [--shape NAME] [--iters N]
    python -m host_memory_streamed_layer_b200.kernel_bench attn [--fwd-only] [--iters N] [--attn-shape B,S,H[,HD]]
    python -m host_memory_streamed_layer_b200.kernel_bench rmsnorm_bwd [--iters N]
    python -m host_memory_streamed_layer_b200.kernel_bench elementwise [--iters N]

Times each launch with CUDA events on the launching stream after warm-up and
prints achieved TFLOP/s (tensor-bound kernels) or GB/s of algorithmic bytes
(memory-bound kernels). With --iters 1 --warmup 0 it launches exactly once,
which is what an ncu capture of one launch wants. Shapes are those of the
llama-1.3b workload (T = 8 x 2048 tokens, d 2048, FFN 5504, 16 heads); for
the GEMMs, --workload NAME takes every GEMM shape of that workload's training
step instead, and each result line carries the shape's launches per step
(so per-shape ncu figures can be weighted into a per-launch step average);
for attention, --attn-shape B,S,H[,HD] sets sequences, length, heads and head
dim (128 unless given; as many KV heads as query heads).
"""
from __future__ import annotations

import argparse
import json

import torch

from . import mt

T, D, F, V, H, HD, B, S = 16384, 2048, 5504, 32000, 16, 128, 8, 2048
GEMMS = {  # name: (M, N, K, form)
    "qkv_fwd": (T, 3 * D, D, "fwd"), "o_fwd": (T, D, D, "fwd"), "gu_fwd": (T, 2 * F, D, "fwd"),
    "down_fwd": (T, D, F, "fwd"), "down_dx": (T, F, D, "dx"), "gu_dx": (T, D, 2 * F, "dx"),
    "qkv_dx": (T, D, 3 * D, "dx"), "o_dx": (T, D, D, "dx"), "down_dw": (D, F, T, "dw"), "gu_dw": (2 * F, D, T, "dw"),
    "qkv_dw": (3 * D, D, T, "dw"), "o_dw": (D, D, T, "dw"), "head_fwd": (T, V, D, "fwd"),
}


def step_gemms(sh):
    """Every GEMM shape of one training step of workload sh, as the engine
    launches them: name -> (M, N, K, form, launches per step). Forward per
    layer; recompute (no down projection) for all layers but the last; the
    backward's input- and weight-gradient products per layer; the LM head per
    token chunk (chunks of at most ~4 GiB of fp32 logits + bf16 dz, multiples
    of 128 tokens)."""
    if sh.get("E", 0):
        raise ValueError("expert layers: their GEMM sizes follow the routing, not the shape")
    L, d, H, Hkv, Fh, Vh, b, s = (sh[k] for k in ("L", "d", "H", "Hkv", "F", "V", "b", "s"))
    hd = d // H
    Tt, Nqkv, Hd = b * s, (H + 2 * Hkv) * hd, H * hd
    tc = min(Tt, (1 << 32) // (Vh * 6))
    if tc < Tt:
        tc = max(128, tc // 128 * 128)
    chunks = [min(tc, Tt - t0) for t0 in range(0, Tt, tc)]
    g = {
        "qkv_fwd": (Tt, Nqkv, d, "fwd", 2 * L - 1), "o_fwd": (Tt, d, Hd, "fwd", 2 * L - 1),
        "gu_fwd": (Tt, 2 * Fh, d, "fwd", 2 * L - 1), "down_fwd": (Tt, d, Fh, "fwd", L),
        "down_dw": (d, Fh, Tt, "dw", L), "down_dx": (Tt, Fh, d, "dx", L), "gu_dw": (2 * Fh, d, Tt, "dw", L),
        "gu_dx": (Tt, d, 2 * Fh, "dx", L), "o_dw": (d, Hd, Tt, "dw", L), "o_dx": (Tt, Hd, d, "dx", L),
        "qkv_dw": (Nqkv, d, Tt, "dw", L), "qkv_dx": (Tt, d, Nqkv, "dx", L),
    }
    for c in sorted(set(chunks)):
        n = chunks.count(c)
        g[f"head_fwd_{c}"] = (c, Vh, d, "fwd32", n)
        g[f"head_dw_{c}"] = (Vh, d, c, "dw", n)
        g[f"head_dx_{c}"] = (c, d, Vh, "dx32", n)
    return g


def timed(fn, iters, warmup):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if iters == 0:
        return 0.0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters / 1e3


def bench_gemm(names, iters, warmup, table=None):
    """Times each named GEMM; `table` maps name -> (M, N, K, form[, launches
    per step]) (default: the 1.3B shapes). Forms: fwd (bf16 out), fwd32 (fp32
    out, the LM head's logits), dx (B MN-major; bf16 out), dx32 (fp32 out),
    dw (both operands MN-major, fp32 out)."""
    table = table or GEMMS
    st = torch.cuda.current_stream().cuda_stream
    out = []
    for name in names:
        M, N, K, form = table[name][:4]
        A = torch.randn(M * K, device="cuda").to(torch.bfloat16)
        Bm = torch.randn(N * K, device="cuda").to(torch.bfloat16)
        f32 = form in ("dw", "fwd32", "dx32")
        C = torch.empty(M * N, device="cuda", dtype=torch.float32 if f32 else torch.bfloat16)
        if form.startswith("fwd"):
            a = (A.data_ptr(), K, 0, Bm.data_ptr(), K, 0)
        elif form.startswith("dx"):
            a = (A.data_ptr(), K, 0, Bm.data_ptr(), N, 1)
        else:
            a = (A.data_ptr(), M, 1, Bm.data_ptr(), N, 1)
        kind = mt.GEMM_OUT_F32 if f32 else mt.GEMM_OUT_BF16
        sec = timed(lambda: mt.mt_k_gemm_bf16(*a, C.data_ptr(), N, kind, 0, 0, M, N, K, st, 0), iters, warmup)
        fl = 2.0 * M * N * K
        r = {"kernel": "gemm", "shape": name, "M": M, "N": N, "K": K, "us": sec * 1e6,
             "tflops": fl / sec / 1e12 if sec else None}
        if len(table[name]) > 4:
            r["launches_per_step"] = table[name][4]
        out.append(r)
        del A, Bm, C
        torch.cuda.empty_cache()
    return out


def bench_attn(iters, warmup, fwd_only, impl="tc", B=B, S=S, H=H, hd=HD):
    st = torch.cuda.current_stream().cuda_stream
    T = B * S
    ld = 3 * H * hd
    qkv = torch.randn(T, ld, device="cuda").to(torch.bfloat16)
    o = torch.empty(T, H * hd, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, H, S, device="cuda")
    p = qkv.data_ptr()
    pk, pv = p + 2 * H * hd, p + 4 * H * hd
    if impl == "tc":
        fwd = lambda: mt.mt_k_attn_fwd_tc(p, pk, pv, ld, o.data_ptr(), H * hd, lse.data_ptr(), B, S, H, H, hd,  # noqa
                                          st)
    else:
        fwd = lambda: mt.mt_k_attn_fwd(p, pk, pv, ld, o.data_ptr(), H * hd, lse.data_ptr(), B, S, H, H, hd, st)  # noqa
    fl = 2.0 * B * H * S * S * hd
    res = [{"kernel": f"attn_fwd_{impl}", "us": 0, "tflops": None}]
    sec = timed(fwd, iters, warmup)
    res[0].update(us=sec * 1e6, tflops=fl / sec / 1e12 if sec else None)
    if not fwd_only:
        fwd()
        do = torch.randn(T, H * hd, device="cuda").to(torch.bfloat16)
        dvec = torch.empty(B, H, S, device="cuda")
        dqa = torch.empty(T, H * hd, device="cuda")
        dqkv = torch.empty(T, ld, device="cuda", dtype=torch.bfloat16)
        dp = dqkv.data_ptr()
        fn = mt.mt_k_attn_bwd_tc if impl == "tc" else mt.mt_k_attn_bwd
        bwd = lambda: fn(p, pk, pv, ld, o.data_ptr(), do.data_ptr(), H * hd, lse.data_ptr(),  # noqa
                         dvec.data_ptr(), dqa.data_ptr(), H * hd, dp, ld, dp + 2 * H * hd,
                         dp + 4 * H * hd, ld, B, S, H, H, hd, 0, 0, st)
        sec = timed(bwd, iters, warmup)
        res.append({"kernel": f"attn_bwd_{impl}", "us": sec * 1e6, "tflops": 2.5 * fl / sec / 1e12 if sec else None})
    return res


def bench_rmsnorm_bwd(iters, warmup):
    st = torch.cuda.current_stream().cuda_stream
    x, dy, dres, dx = (torch.randn(T, D, device="cuda") for _ in range(4))
    g = torch.ones(D, device="cuda", dtype=torch.bfloat16)
    r = torch.ones(T, device="cuda")
    dxb = torch.empty(T, D, device="cuda", dtype=torch.bfloat16)
    part = torch.empty(mt.mt_k_rmsnorm_bwd_partial_floats(T, D), device="cuda")
    dg = torch.empty(D, device="cuda")
    sec = timed(lambda: mt.mt_k_rmsnorm_bwd(x.data_ptr(), g.data_ptr(), r.data_ptr(), dy.data_ptr(), dres.data_ptr(),
                                            dx.data_ptr(), dxb.data_ptr(), part.data_ptr(), dg.data_ptr(), T, D, st),
                iters, warmup)
    byt = 18.0 * T * D
    return [{"kernel": "rmsnorm_bwd", "us": sec * 1e6, "gbs": byt / sec / 1e9 if sec else None}]


def bench_elementwise(iters, warmup):
    """The HBM-bound kernels of the layer at the 1.3B shape, each against its
    algorithmic bytes (every input read once, every output written once)."""
    st = torch.cuda.current_stream().cuda_stream
    dev = "cuda"
    out = []

    def rec(name, fn, nbytes):
        sec = timed(fn, iters, warmup)
        out.append({"kernel": name, "us": sec * 1e6, "bytes": nbytes, "gbs": nbytes / sec / 1e9 if sec else None})

    x = torch.randn(T, D, device=dev)
    g = torch.ones(D, device=dev, dtype=torch.bfloat16)
    y = torch.empty(T, D, device=dev, dtype=torch.bfloat16)
    rstd = torch.empty(T, device=dev)
    rec("rmsnorm_fwd", lambda: mt.mt_k_rmsnorm_fwd(x.data_ptr(), g.data_ptr(), y.data_ptr(), rstd.data_ptr(), T, D,
                                                   1e-5, st), T * (6 * D + 4))
    gu = torch.randn(T, 2 * F, device=dev).to(torch.bfloat16)
    act = torch.empty(T, F, device=dev, dtype=torch.bfloat16)
    rec("swiglu_fwd", lambda: mt.mt_k_swiglu_fwd(gu.data_ptr(), act.data_ptr(), T, F, st), T * 6 * F)
    dact = torch.randn(T, F, device=dev).to(torch.bfloat16)
    dgu = torch.empty(T, 2 * F, device=dev, dtype=torch.bfloat16)
    rec("swiglu_bwd", lambda: mt.mt_k_swiglu_bwd(gu.data_ptr(), dact.data_ptr(), dgu.data_ptr(), T, F, st),
        T * 10 * F)
    del gu, act, dact, dgu
    Tc = 4096
    z = torch.randn(Tc, V, device=dev)
    lab = torch.randint(0, V, (Tc,), device=dev, dtype=torch.int32)
    dz = torch.empty(Tc, V, device=dev, dtype=torch.bfloat16)
    rl = torch.empty(Tc, device=dev)
    rec("softmax_ce", lambda: mt.mt_k_softmax_ce(z.data_ptr(), V, lab.data_ptr(), dz.data_ptr(), V, rl.data_ptr(), Tc,
                                                 V, 1.0 / T, st), Tc * 6 * V)
    del z, dz
    E = torch.randn(V, D, device=dev).to(torch.bfloat16)
    tok = torch.randint(0, V, (T,), device=dev, dtype=torch.int32)
    xe = torch.empty(T, D, device=dev)
    rec("embed_fwd (table in HBM)", lambda: mt.mt_k_embed_fwd(tok.data_ptr(), E.data_ptr(), xe.data_ptr(), T, D, st),
        T * 6 * D)
    out += bench_rmsnorm_bwd(iters, warmup)
    out[-1]["bytes"] = 18.0 * T * D
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("kernel", choices=["gemm", "attn", "rmsnorm_bwd", "elementwise"])
    ap.add_argument("--shape", default="all")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--fwd-only", action="store_true")
    ap.add_argument("--impl", default="tc", choices=["tc", "mma"])
    ap.add_argument("--workload", default=None, help="GEMMs: every shape of this workload's training step")
    ap.add_argument("--attn-shape", default=f"{B},{S},{H}",
                    help="attention: sequences,length,heads[,head dim] (head dim 128 unless given)")
    ap.add_argument("--attn-variant", default="auto", choices=["auto", "one", "pingpong"],
                    help="attention forward kernel (head dim 128): automatic, one or two query tiles per CTA")
    ap.add_argument("--attn-bwd", default="auto", choices=["auto", "fused", "split"],
                    help="attention backward: dQ by reductions (head dim 128), or the deterministic split")
    a = ap.parse_args()
    if a.kernel == "gemm":
        table = None
        if a.workload:
            import synth
            table = step_gemms(synth.WORKLOADS[a.workload])
        names = list(table or GEMMS) if a.shape == "all" else a.shape.split(",")
        res = bench_gemm(names, a.iters, a.warmup, table)
    elif a.kernel == "attn":
        dims = [int(x) for x in a.attn_shape.split(",")]
        ab, as_, ah = dims[:3]
        ahd = dims[3] if len(dims) > 3 else HD
        mt.mt_k_attn_fwd_variant({"auto": mt.ATTN_AUTO, "one": mt.ATTN_ONE_TILE,
                                  "pingpong": mt.ATTN_PINGPONG}[a.attn_variant])
        mt.mt_k_attn_bwd_variant({"auto": mt.ATTN_BWD_AUTO, "fused": mt.ATTN_BWD_FUSED,
                                  "split": mt.ATTN_BWD_SPLIT}[a.attn_bwd])
        res = bench_attn(a.iters, a.warmup, a.fwd_only, a.impl, ab, as_, ah, ahd)
        for r in res:
            r["shape"] = dict(b=ab, s=as_, heads=ah, hd=ahd)
    elif a.kernel == "elementwise":
        res = bench_elementwise(a.iters, a.warmup)
    else:
        res = bench_rmsnorm_bwd(a.iters, a.warmup)
    for r in res:
        print(json.dumps(r))


if __name__ == "__main__":
    main()
