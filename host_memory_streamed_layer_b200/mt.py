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
        msg = lib.mt_last_error(ctx).decode() if hasattr(lib, "mt_last_error") else ""
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
