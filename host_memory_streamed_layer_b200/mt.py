"""ctypes binding of libmt.so with the C names (argument marshalling only).

Raises ImportError at import time when libmt.so is missing: there is no
fallback path; build it with `python -m host_memory_streamed_layer_b200.build`.
"""
from __future__ import annotations

import ctypes
import os

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmt.so")
if not os.path.exists(_PATH):
    raise ImportError(f"{_PATH} is not built; run python -m host_memory_streamed_layer_b200.build")
lib = ctypes.CDLL(_PATH)

c_int, c_i64, c_void_p, c_size_t = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t

MT_OK = 0
ERRORS = {-1: "MT_ERR_ARG", -2: "MT_ERR_CONFIG", -3: "MT_ERR_ARENA", -4: "MT_ERR_NOMEM", -5: "MT_ERR_PIN",
          -6: "MT_ERR_CUDA", -7: "MT_ERR_TIMEOUT", -8: "MT_ERR_NONFINITE", -9: "MT_ERR_DEVICE"}

GEMM_OUT_BF16, GEMM_OUT_F32, GEMM_OUT_F32_ADD = 0, 1, 2


class MTError(RuntimeError):
    def __init__(self, code: int, msg: str = ""):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


def _check(rc: int, what: str = "", ctx=None):
    if rc != MT_OK:
        msg = lib.mt_last_error(ctx).decode() if ctx else ""
        raise MTError(rc, f"{what} {msg}".strip())
    return rc


def _sig(name, res, *args):
    fn = getattr(lib, name, None)
    if fn is not None:
        fn.restype = res
        fn.argtypes = list(args)
    return fn


_sig("mt_k_gemm_bf16", c_int, c_void_p, c_i64, c_int, c_void_p, c_i64, c_int, c_void_p, c_i64, c_int,
     c_void_p, c_i64, c_int, c_int, c_int, c_void_p, c_void_p)


def mt_k_gemm_bf16(A, lda, a_mn, B, ldb, b_mn, C, ldc, out_kind, R, ldr, M, N, K, stream=0, dev_err=0):
    return _check(lib.mt_k_gemm_bf16(A, lda, a_mn, B, ldb, b_mn, C, ldc, out_kind, R or None, ldr, M, N, K,
                                     stream or None, dev_err or None), "mt_k_gemm_bf16")


_sig("mt_k_gemm_variant", c_int, c_int)
_sig("mt_k_attn_fwd_variant", c_int, c_int)
_sig("mt_k_attn_bwd_variant", c_int, c_int)
GEMM_AUTO, GEMM_SINGLE, GEMM_PAIR = 0, 1, 2


def mt_k_gemm_variant(variant: int) -> int:
    """Selects the GEMM kernel family for later calls; returns the previous one."""
    rc = lib.mt_k_gemm_variant(variant)
    if rc < 0:
        raise MTError(rc, "mt_k_gemm_variant")
    return rc


ATTN_AUTO, ATTN_ONE_TILE, ATTN_PINGPONG = 0, 1, 2


def mt_k_attn_fwd_variant(variant: int) -> int:
    """Selects the head-dim-128 attention forward kernel for later calls;
    returns the previous choice."""
    rc = lib.mt_k_attn_fwd_variant(variant)
    if rc < 0:
        raise MTError(rc, "mt_k_attn_fwd_variant")
    return rc


ATTN_BWD_AUTO, ATTN_BWD_FUSED, ATTN_BWD_SPLIT = 0, 1, 2


def mt_k_attn_bwd_variant(variant: int) -> int:
    """Selects the tensor-core attention backward form for later calls:
    automatic (the deterministic split), fused dQ reductions (head dim 128;
    head dim 64 always runs split), or split; returns the previous choice."""
    rc = lib.mt_k_attn_bwd_variant(variant)
    if rc < 0:
        raise MTError(rc, "mt_k_attn_bwd_variant")
    return rc


_sig("mt_k_gemm_wait_limit_ns", c_i64, c_i64)
DEV_TIMEOUT_PRODUCER, DEV_TIMEOUT_MMA, DEV_TIMEOUT_EPILOGUE, DEV_TIMEOUT_TEARDOWN = 1, 2, 3, 4
GEMM_WAIT_DEFAULT_NS = 1_000_000_000


def mt_k_gemm_wait_limit_ns(ns: int) -> int:
    """Sets the main-loop wait limit of later single-CTA GEMM launches (ns < 0
    only queries); returns the previous limit."""
    return lib.mt_k_gemm_wait_limit_ns(ns)


c_float, c_f = ctypes.c_float, ctypes.c_float

_sig("mt_k_rmsnorm_fwd", c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_float, c_void_p)
_sig("mt_k_rmsnorm_bwd_partial_floats", c_size_t, c_int, c_int)
_sig("mt_k_rmsnorm_bwd", c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
     c_void_p, c_int, c_int, c_void_p)
_sig("mt_k_rope", c_int, c_void_p, c_i64, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_float, c_void_p)
_sig("mt_k_swiglu_fwd", c_int, c_void_p, c_void_p, c_int, c_int, c_void_p)
_sig("mt_k_swiglu_bwd", c_int, c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p)
_sig("mt_k_embed_fwd", c_int, c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p)
_sig("mt_k_embed_bwd", c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_int, c_void_p)
_sig("mt_k_softmax_ce", c_int, c_void_p, c_i64, c_void_p, c_void_p, c_i64, c_void_p, c_int, c_int, c_float, c_void_p)
_sig("mt_k_attn_fwd", c_int, c_void_p, c_void_p, c_void_p, c_i64, c_void_p, c_i64, c_void_p, c_int, c_int, c_int,
     c_int, c_int, c_void_p)
_sig("mt_k_attn_fwd_tc", c_int, c_void_p, c_void_p, c_void_p, c_i64, c_void_p, c_i64, c_void_p, c_int, c_int,
     c_int, c_int, c_int, c_void_p, c_void_p)
_sig("mt_k_attn_bwd", c_int, c_void_p, c_void_p, c_void_p, c_i64, c_void_p, c_void_p, c_i64, c_void_p, c_void_p,
     c_void_p, c_i64, c_void_p, c_i64, c_void_p, c_void_p, c_i64, c_int, c_int, c_int, c_int, c_int, c_void_p,
     c_void_p, c_void_p)
_sig("mt_k_attn_bwd_tc", c_int, c_void_p, c_void_p, c_void_p, c_i64, c_void_p, c_void_p, c_i64, c_void_p, c_void_p,
     c_void_p, c_i64, c_void_p, c_i64, c_void_p, c_void_p, c_i64, c_int, c_int, c_int, c_int, c_int, c_void_p,
     c_void_p, c_void_p, c_void_p)
_sig("mt_k_gemm_bf16_rope", c_int, c_void_p, c_i64, c_void_p, c_i64, c_void_p, c_i64, c_int, c_int, c_int, c_int,
     c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p)


_sig("mt_k_rmsnorm_bwd_noalloc", c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
     c_void_p, c_int, c_int, c_void_p)


def _p(x):
    return x or None


def mt_k_rmsnorm_fwd(x, g, y, rstd, T, d, eps, stream=0):
    return _check(lib.mt_k_rmsnorm_fwd(x, g, y, _p(rstd), T, d, eps, _p(stream)), "mt_k_rmsnorm_fwd")


def mt_k_rmsnorm_bwd_partial_floats(T, d):
    return lib.mt_k_rmsnorm_bwd_partial_floats(T, d)


def mt_k_rmsnorm_bwd(x, g, rstd, dy, dres, dx, dx_bf16, dg_part, dg, T, d, stream=0):
    return _check(lib.mt_k_rmsnorm_bwd(x, g, rstd, dy, _p(dres), dx, _p(dx_bf16), dg_part, dg, T, d, _p(stream)),
                  "mt_k_rmsnorm_bwd")


def mt_k_rmsnorm_bwd_noalloc(x, g, rstd, dy, dres, dx, dx_bf16, dg, T, d, stream=0):
    return _check(lib.mt_k_rmsnorm_bwd_noalloc(x, g, rstd, dy, _p(dres), dx, _p(dx_bf16), dg, T, d, _p(stream)),
                  "mt_k_rmsnorm_bwd_noalloc")


def mt_k_rope(buf, ld, T, s, nheads, hd, col0, cos_tab, sin_tab, sign, stream=0):
    return _check(lib.mt_k_rope(buf, ld, T, s, nheads, hd, col0, cos_tab, sin_tab, sign, _p(stream)), "mt_k_rope")


def mt_k_swiglu_fwd(gu, act, T, F, stream=0):
    return _check(lib.mt_k_swiglu_fwd(gu, act, T, F, _p(stream)), "mt_k_swiglu_fwd")


def mt_k_swiglu_bwd(gu, dact, dgu, T, F, stream=0):
    return _check(lib.mt_k_swiglu_bwd(gu, dact, dgu, T, F, _p(stream)), "mt_k_swiglu_bwd")


def mt_k_embed_fwd(tok, E, x, T, d, stream=0):
    return _check(lib.mt_k_embed_fwd(tok, E, x, T, d, _p(stream)), "mt_k_embed_fwd")


def mt_k_embed_bwd(offs, pos, n_unique, dx, rows, d, stream=0):
    return _check(lib.mt_k_embed_bwd(offs, pos, n_unique, dx, rows, d, _p(stream)), "mt_k_embed_bwd")


def mt_k_softmax_ce(z, ldz, labels, dz, lddz, row_loss, Tc, V, scale, stream=0):
    return _check(lib.mt_k_softmax_ce(z, ldz, labels, dz, lddz, row_loss, Tc, V, scale, _p(stream)),
                  "mt_k_softmax_ce")


def mt_k_attn_fwd(q, k, v, ldqkv, o, ldo, lse, b, s, H, Hkv, hd, stream=0):
    return _check(lib.mt_k_attn_fwd(q, k, v, ldqkv, o, ldo, lse, b, s, H, Hkv, hd, _p(stream)), "mt_k_attn_fwd")


def mt_k_attn_fwd_tc(q, k, v, ldqkv, o, ldo, lse, b, s, H, Hkv, hd, stream=0, dev_err=0):
    return _check(lib.mt_k_attn_fwd_tc(q, k, v, ldqkv, o, ldo, lse, b, s, H, Hkv, hd, _p(stream), _p(dev_err)),
                  "mt_k_attn_fwd_tc")


def mt_k_attn_bwd(q, k, v, ldqkv, o, dout, ldo, lse, dvec, dq_acc, ldqa, dq, lddq, dk, dv, lddkv, b, s, H, Hkv, hd,
                  cos_tab=0, sin_tab=0, stream=0):
    return _check(lib.mt_k_attn_bwd(q, k, v, ldqkv, o, dout, ldo, lse, dvec, dq_acc, ldqa, dq, lddq, dk, dv, lddkv,
                                    b, s, H, Hkv, hd, _p(cos_tab), _p(sin_tab), _p(stream)), "mt_k_attn_bwd")


def mt_k_attn_bwd_tc(q, k, v, ldqkv, o, dout, ldo, lse, dvec, dq_acc, ldqa, dq, lddq, dk, dv, lddkv, b, s, H, Hkv,
                     hd, cos_tab=0, sin_tab=0, stream=0, dev_err=0):
    return _check(lib.mt_k_attn_bwd_tc(q, k, v, ldqkv, o, dout, ldo, lse, dvec, dq_acc, ldqa, dq, lddq, dk, dv, lddkv,
                                       b, s, H, Hkv, hd, _p(cos_tab), _p(sin_tab), _p(stream), _p(dev_err)),
                  "mt_k_attn_bwd_tc")


def mt_k_gemm_bf16_rope(A, lda, B, ldb, C, ldc, M, N, K, rope_cols, hd, s, cos_tab, sin_tab, stream=0, dev_err=0):
    return _check(lib.mt_k_gemm_bf16_rope(A, lda, B, ldb, C, ldc, M, N, K, rope_cols, hd, s, cos_tab, sin_tab,
                                          _p(stream), _p(dev_err)), "mt_k_gemm_bf16_rope")


# ---------------------------------------------------------------------------
# Engine API (include/mt.h)
# ---------------------------------------------------------------------------
MT_FLAG_SERIALIZE, MT_FLAG_KERNEL_TIMING, MT_FLAG_NO_UPDATE, MT_FLAG_GRAD_RING = 0x1, 0x2, 0x4, 0x8
MT_FLAG_DEFER_UPDATES = 0x10
MT_FLAG_BF16_GRADS = 0x20
MT_FLAG_OFFLOAD_ACTS = 0x40
MT_FLAG_TIED_EMBED = 0x80
MT_FLAG_STASH_ATTN = 0x100
MT_FLAG_POISON = 0x200
MT_GRAD_RING_SLOTS = 3
MT_T_ATTN_NORM, MT_T_WQ, MT_T_WK, MT_T_WV, MT_T_WO, MT_T_MLP_NORM, MT_T_WGATE, MT_T_WUP, MT_T_WDOWN = range(9)
MT_T_ROUTER = 9
MT_T_EMBED, MT_T_FINAL_NORM, MT_T_LM_HEAD = 100, 101, 102


class mt_config(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("L", ctypes.c_int32), ("d", ctypes.c_int32),
                ("H", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("F", ctypes.c_int32), ("V", ctypes.c_int32),
                ("b", ctypes.c_int32), ("s", ctypes.c_int32), ("norm_eps", ctypes.c_float),
                ("rope_base", ctypes.c_float), ("lr", ctypes.c_float), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("adam_eps", ctypes.c_float), ("wd", ctypes.c_float),
                ("seed", ctypes.c_uint64), ("flags", ctypes.c_uint32), ("device", ctypes.c_int32),
                ("host_threads", ctypes.c_int32), ("E", ctypes.c_int32), ("topk", ctypes.c_int32)]


class mt_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_double) for n in (
        "step_ms", "fwd_ms", "head_ms", "bwd_ms", "h2d_bytes", "d2h_bytes", "h2d_ms", "d2h_ms",
        "wait_weights_ms", "adamw_ms", "adamw_bytes", "gemm_flops", "gemm_ms")] + \
        [("gemm_launches", ctypes.c_int64), ("attn_flops", ctypes.c_double), ("attn_ms", ctypes.c_double),
         ("attn_launches", ctypes.c_int64), ("kernel_launches", ctypes.c_int64), ("host_step_ms", ctypes.c_double),
         ("adamw_first_ms", ctypes.c_double), ("adamw_last_ms", ctypes.c_double), ("enqueue_ms", ctypes.c_double)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_cfgp = ctypes.POINTER(mt_config)
_sig("mt_config_default", c_int, _cfgp)
_sig("mt_arena_bytes", c_size_t, _cfgp)
_sig("mt_tensor_offset", c_int, _cfgp, c_int, c_int, ctypes.POINTER(c_size_t), ctypes.POINTER(c_size_t))
_sig("mt_host_state_bytes", c_size_t, _cfgp)
_sig("mt_create", c_int, _cfgp, c_void_p, c_size_t, ctypes.POINTER(c_void_p))
_sig("mt_train_step", c_int, c_void_p, c_void_p, c_void_p, ctypes.POINTER(ctypes.c_float))
_sig("mt_flush", c_int, c_void_p)
_sig("mt_get_grads", c_int, c_void_p, c_void_p, c_size_t)
_sig("mt_get_timeline", c_int, c_void_p, c_void_p, c_size_t, ctypes.POINTER(c_size_t))
_sig("mt_head_fwd_bwd", c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t)
_sig("mt_layer_fwd_bwd", c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t)
_sig("mt_get_params", c_int, c_void_p, c_void_p, c_size_t)
_sig("mt_get_stats", c_int, c_void_p, ctypes.POINTER(mt_stats))
_sig("mt_destroy", None, c_void_p)
_sig("mt_get_stream", c_int, c_void_p, ctypes.POINTER(c_void_p))
_sig("mt_host_optimizer_gbs", ctypes.c_double, c_size_t, c_int)
_sig("mt_host_triad_gbs", ctypes.c_double, c_size_t, c_int)
_sig("mt_get_opt_state", c_int, c_void_p, c_void_p, c_void_p, c_size_t, ctypes.POINTER(ctypes.c_int64))
_sig("mt_set_state", c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, ctypes.c_int64)
_sig("mt_last_error", ctypes.c_char_p, c_void_p)
_sig("mt_device_bytes", c_size_t, _cfgp)
_sig("mt_inject_host_stall", c_int, c_void_p, c_int, c_int)
_sig("mt_k_adamw_host", c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_float, c_float,
     c_float, c_float, c_float, c_int)


def mt_config_default(**shape) -> mt_config:
    cfg = mt_config()
    _check(lib.mt_config_default(ctypes.byref(cfg)), "mt_config_default")
    for k, v in shape.items():
        setattr(cfg, k, v)
    return cfg


def mt_arena_bytes(cfg: mt_config) -> int:
    return lib.mt_arena_bytes(ctypes.byref(cfg))


def mt_tensor_offset(cfg: mt_config, layer: int, tid: int):
    off, n = c_size_t(), c_size_t()
    _check(lib.mt_tensor_offset(ctypes.byref(cfg), layer, tid, ctypes.byref(off), ctypes.byref(n)),
           "mt_tensor_offset")
    return off.value, n.value


def mt_host_state_bytes(cfg: mt_config) -> int:
    return lib.mt_host_state_bytes(ctypes.byref(cfg))


def mt_create(cfg: mt_config, arena_ptr: int = 0, arena_bytes: int = 0) -> int:
    """Returns the context handle (an int). arena_ptr: host address or 0."""
    ctx = c_void_p()
    rc = lib.mt_create(ctypes.byref(cfg), arena_ptr or None, arena_bytes, ctypes.byref(ctx))
    if rc != MT_OK:
        raise MTError(rc, "mt_create " + lib.mt_last_error(None).decode())
    return ctx.value


def mt_train_step(ctx: int, tokens_ptr: int, labels_ptr: int) -> float:
    loss = ctypes.c_float()
    rc = lib.mt_train_step(ctx, tokens_ptr, labels_ptr, ctypes.byref(loss))
    if rc != MT_OK:
        raise MTError(rc, "mt_train_step " + lib.mt_last_error(ctx).decode())
    return loss.value


def mt_flush(ctx: int):
    return _check(lib.mt_flush(ctx), "mt_flush", ctx)


def mt_get_grads(ctx: int, dst_ptr: int, nbytes: int):
    return _check(lib.mt_get_grads(ctx, dst_ptr, nbytes), "mt_get_grads", ctx)


def mt_layer_fwd_bwd(ctx: int, layer: int, x_in: int, dx_out: int, x_out: int, dx_in: int, grads: int,
                     grads_bytes: int):
    return _check(lib.mt_layer_fwd_bwd(ctx, layer, x_in, dx_out, x_out, dx_in, grads, grads_bytes),
                  "mt_layer_fwd_bwd", ctx)


def mt_head_fwd_bwd(ctx: int, x_L: int, labels: int, dx_L: int, grads: int, grads_bytes: int) -> float:
    loss = ctypes.c_float(0.0)
    _check(lib.mt_head_fwd_bwd(ctx, x_L, labels, ctypes.byref(loss), dx_L, grads, grads_bytes),
           "mt_head_fwd_bwd", ctx)
    return loss.value


def mt_get_timeline(ctx: int) -> dict:
    """Timeline of the last step (see include/mt.h), as a dict of lists."""
    n = c_size_t(0)
    _check(lib.mt_get_timeline(ctx, None, 0, ctypes.byref(n)), "mt_get_timeline", ctx)
    buf = (ctypes.c_float * n.value)()
    _check(lib.mt_get_timeline(ctx, buf, n.value, ctypes.byref(n)), "mt_get_timeline", ctx)
    v = list(buf)
    nl, L, nj = int(v[0]), int(v[1]), int(v[2])
    k = 3
    loads = [dict(layer=int(v[k + 5 * i]), h2d_start=v[k + 5 * i + 1], ready=v[k + 5 * i + 2],
                  compute_arrives=v[k + 5 * i + 3], released=v[k + 5 * i + 4]) for i in range(nl)]
    k += 5 * nl
    offload = [dict(layer=int(v[k + 4 * i]), grads_ready=v[k + 4 * i + 1], d2h_start=v[k + 4 * i + 2],
                    d2h_done=v[k + 4 * i + 3]) for i in range(L)]
    k += 4 * L
    phases = dict(fwd_end=v[k], head_end=v[k + 1], bwd_end=v[k + 2], step_end=v[k + 3])
    k += 4
    jobs = [dict(kind=int(v[k + 4 * i]), layer=int(v[k + 4 * i + 1]), ready_ms=v[k + 4 * i + 2],
                 done_ms=v[k + 4 * i + 3]) for i in range(nj)]
    return dict(loads=loads, offload=offload, phases=phases, jobs=jobs)


def mt_get_params(ctx: int, dst_ptr: int, nbytes: int):
    return _check(lib.mt_get_params(ctx, dst_ptr, nbytes), "mt_get_params", ctx)


def mt_get_stats(ctx: int) -> dict:
    st = mt_stats()
    _check(lib.mt_get_stats(ctx, ctypes.byref(st)), "mt_get_stats", ctx)
    return st.as_dict()


def mt_get_stream(ctx: int) -> int:
    st = c_void_p()
    _check(lib.mt_get_stream(ctx, ctypes.byref(st)), "mt_get_stream", ctx)
    return st.value or 0


class mt_shard(ctypes.Structure):
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32)] + \
        [(n, ctypes.c_uint64) for n in ("layer_elems", "layer_chunk", "layer_begin", "layer_end",
                                         "head_elems", "head_chunk", "head_begin", "head_end")] + \
        [("embed_row_begin", ctypes.c_int32), ("embed_row_end", ctypes.c_int32)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_sig("mt_shard_plan", c_int, _cfgp, c_int, c_int, ctypes.POINTER(mt_shard))


def mt_shard_plan(cfg: mt_config, world: int, rank: int) -> dict:
    sp = mt_shard()
    _check(lib.mt_shard_plan(ctypes.byref(cfg), world, rank, ctypes.byref(sp)), "mt_shard_plan")
    return sp.as_dict()


def mt_device_bytes(cfg: mt_config) -> int:
    return lib.mt_device_bytes(ctypes.byref(cfg))


MT_SHARD_ID_BYTES = 128
_sig("mt_shard_id", c_int, c_void_p)
_sig("mt_create_sharded", c_int, _cfgp, c_void_p, c_size_t, c_int, c_int, c_void_p, ctypes.POINTER(c_void_p))
_sig("mt_device_bytes_sharded", c_size_t, _cfgp, c_int)


def mt_shard_id() -> bytes:
    """A fresh NCCL unique id for mt_create_sharded (one rank makes it; every
    rank passes the same bytes)."""
    buf = ctypes.create_string_buffer(MT_SHARD_ID_BYTES)
    rc = lib.mt_shard_id(buf)
    if rc != MT_OK:
        raise MTError(rc, "mt_shard_id " + lib.mt_last_error(None).decode())
    return buf.raw


def mt_create_sharded(cfg: mt_config, arena_ptr: int, arena_bytes: int, world: int, rank: int, nccl_id: bytes) -> int:
    """Context of rank `rank` of a sharded run; returns once every rank joined."""
    if len(nccl_id) != MT_SHARD_ID_BYTES:
        raise ValueError("nccl_id must be MT_SHARD_ID_BYTES bytes")
    ctx = c_void_p()
    buf = ctypes.create_string_buffer(bytes(nccl_id), MT_SHARD_ID_BYTES)
    rc = lib.mt_create_sharded(ctypes.byref(cfg), arena_ptr or None, arena_bytes, world, rank, buf, ctypes.byref(ctx))
    if rc != MT_OK:
        raise MTError(rc, "mt_create_sharded " + lib.mt_last_error(None).decode())
    return ctx.value


def mt_device_bytes_sharded(cfg: mt_config, world: int) -> int:
    return lib.mt_device_bytes_sharded(ctypes.byref(cfg), world)


_sig("mt_get_routing", c_int, c_void_p, c_int, c_void_p, c_size_t)


def mt_get_routing(ctx: int, layer: int, T: int, topk: int):
    """The experts each of the T tokens chose in `layer`'s last forward, [T, topk]."""
    import numpy as np
    out = np.empty((T, topk), dtype=np.int32)
    _check(lib.mt_get_routing(ctx, layer, out.ctypes.data, out.size), "mt_get_routing", ctx)
    return out


def mt_inject_host_stall(ctx: int, stream: int, ms: int):
    """Test aid: a host function sleeping ms milliseconds on one of the
    context's streams (0 prefetch, 1 compute, 2 offload)."""
    return _check(lib.mt_inject_host_stall(ctx, stream, ms), "mt_inject_host_stall", ctx)


def mt_destroy(ctx: int):
    lib.mt_destroy(ctx)


def mt_last_error(ctx: int = 0) -> str:
    return lib.mt_last_error(ctx or None).decode()


def mt_k_adamw_host(p, g, m, v, pb, n, lr, beta1, beta2, eps, wd, t):
    return _check(lib.mt_k_adamw_host(p, g or None, m, v, pb or None, n, lr, beta1, beta2, eps, wd, t),
                  "mt_k_adamw_host")


def mt_host_optimizer_gbs(n: int = 1 << 28, threads: int = 0) -> float:
    r = lib.mt_host_optimizer_gbs(n, threads)
    if r < 0:
        raise MTError(int(r), "mt_host_optimizer_gbs")
    return r


def mt_host_triad_gbs(n: int = 1 << 28, threads: int = 0) -> float:
    r = lib.mt_host_triad_gbs(n, threads)
    if r < 0:
        raise MTError(int(r), "mt_host_triad_gbs")
    return r


def mt_get_opt_state(ctx: int, m_ptr: int, v_ptr: int, nbytes: int) -> int:
    step = ctypes.c_int64()
    _check(lib.mt_get_opt_state(ctx, m_ptr or None, v_ptr or None, nbytes, ctypes.byref(step)), "mt_get_opt_state",
           ctx)
    return step.value


def mt_set_state(ctx: int, params_ptr: int, m_ptr: int, v_ptr: int, nbytes: int, step: int):
    return _check(lib.mt_set_state(ctx, params_ptr or None, m_ptr or None, v_ptr or None, nbytes, step),
                  "mt_set_state", ctx)
