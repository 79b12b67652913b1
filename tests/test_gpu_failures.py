"""Failure detection of the streamed training step, without faulting the GPU.

The pages promise fewer crashes and out-of-memory errors than offload systems
(intelligentliving.co, "Leveraging Double-Buffered Pipelining and Stateless
Layer Templates") and give no failure model; these tests pin the library's
documented behaviour (include/mt.h):

- a non-finite gradient (a NaN planted in the host master, so the GPU computes
  NaN activations) returns MT_ERR_NONFINITE and skips every update of the step,
  the untouched embedding rows' zero-gradient update included;
- a kernel taking its bounded-wait exit (the GEMM wait limit set to 0, so the
  first wait that finds a stage not ready gives up) reports MT_DEV_TIMEOUT_*,
  the step returns MT_ERR_DEVICE with every update from that point skipped,
  the state deferred from an earlier valid step still lands, and the next step
  on the same context is correct;
- a host-side stall longer than MT_WAIT_LIMIT_S returns MT_ERR_TIMEOUT and
  the context stays usable and destroys cleanly;
- a configuration whose device budget does not fit fails with MT_ERR_NOMEM
  before allocating anything;
- the device footprint is the documented one and grows with the layer count
  only by the boundary activations (saify.me, "The memory-centric design":
  persistent GPU state stays at about one layer's footprint).
"""
import math
import time

import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]  # single-CTA GEMMs only: every product has fewer 256-row tiles than SM pairs
HYP = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def _libs():
    from host_memory_streamed_layer_b200 import arena, mt
    return arena, mt


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def _ctx(shape, flags, init=None, threads=4):
    arena, mt = _libs()
    cfg = arena.config(shape)
    cfg.flags = flags
    cfg.host_threads = threads
    A = arena.pack(cfg, synth.init_weights(shape, 0) if init is None else init)
    return cfg, A, mt.mt_create(cfg, A.ctypes.data, A.nbytes)


def _opt_state(mt, ctx, n):
    M, V = np.empty(n, np.float32), np.empty(n, np.float32)
    step = mt.mt_get_opt_state(ctx, M.ctypes.data, V.ctypes.data, M.nbytes)
    return M, V, step


def test_gemm_wait_limit_zero_takes_the_bounded_exit():
    """One GEMM with the main-loop wait limit at 0: the kernel gives up at its
    first incomplete wait, records an MT_DEV_TIMEOUT_* code, drains its own
    copies and MMAs and returns; the context stays usable and the same GEMM
    with the default limit is exact again."""
    import torch
    _, mt = _libs()
    M, N, K = 128, 128, 8192  # one output tile, 128 k-blocks: the epilogue's first wait cannot be ready
    g = torch.Generator().manual_seed(0)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    C = torch.zeros(M, N, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    prev = mt.mt_k_gemm_wait_limit_ns(0)
    try:
        assert prev == mt.GEMM_WAIT_DEFAULT_NS
        mt.mt_k_gemm_bf16(A.data_ptr(), K, 0, B.data_ptr(), K, 0, C.data_ptr(), N, mt.GEMM_OUT_F32, 0, 0, M, N, K,
                          0, err.data_ptr())
        torch.cuda.synchronize()  # raises if the context were lost
        code = int(err.item())
        assert code in (mt.DEV_TIMEOUT_PRODUCER, mt.DEV_TIMEOUT_MMA, mt.DEV_TIMEOUT_EPILOGUE), code
    finally:
        assert mt.mt_k_gemm_wait_limit_ns(prev) == 0
    assert mt.mt_k_gemm_wait_limit_ns(-1) == mt.GEMM_WAIT_DEFAULT_NS
    err.zero_()
    mt.mt_k_gemm_bf16(A.data_ptr(), K, 0, B.data_ptr(), K, 0, C.data_ptr(), N, mt.GEMM_OUT_F32, 0, 0, M, N, K,
                      0, err.data_ptr())
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = A.double() @ B.double().T
    assert rel(C.double().cpu().numpy(), ref.cpu().numpy()) < 1e-5


@pytest.mark.parametrize("defer", [False, True])
def test_nonfinite_gradient_skips_every_update(defer):
    """A NaN in layer 0's Wq makes every gradient of the step NaN: the step
    returns MT_ERR_NONFINITE and neither the master (untouched embedding rows
    included), nor the moments move."""
    arena, mt = _libs()
    flags = mt.MT_FLAG_DEFER_UPDATES if defer else 0
    cfg, A, ctx = _ctx(TINY, flags)
    try:
        off, n = mt.mt_tensor_offset(cfg, 0, mt.MT_T_WQ)
        bad = A.copy()
        bad[off + 5] = np.nan
        mt.mt_set_state(ctx, bad.ctypes.data, 0, 0, bad.nbytes, 0)
        tok, lab = synth.tokens_labels(TINY["b"], TINY["s"], TINY["V"], 0)
        with pytest.raises(mt.MTError) as e:
            mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
        assert e.value.code == -8
        mt.mt_flush(ctx)  # nothing may be pending from a failed step
        assert np.array_equal(A, bad, equal_nan=True)
        M, V, _ = _opt_state(mt, ctx, A.size)
        assert not M.any() and not V.any()
    finally:
        mt.mt_destroy(ctx)


def test_device_error_skips_updates_and_the_context_recovers():
    """Step 1 is valid (its LM-head, last-layer and untouched-row updates are
    deferred into step 2); step 2 runs with the GEMM wait limit at 0, so its
    kernels take their bounded exit: MT_ERR_DEVICE, none of step 2's updates
    run, and after a flush the state is exactly AdamW of step 1's gradients.
    Step 3, with the default limit, matches the oracle on that state."""
    arena, mt = _libs()
    c = oracle.OracleConfig(**TINY)
    cfg, A, ctx = _ctx(TINY, mt.MT_FLAG_DEFER_UPDATES)
    P0 = A.copy()
    toks = [synth.tokens_labels(TINY["b"], TINY["s"], TINY["V"], 0, k) for k in range(3)]
    try:
        mt.mt_train_step(ctx, toks[0][0].ctypes.data, toks[0][1].ctypes.data)
        G1 = np.empty_like(A)
        mt.mt_get_grads(ctx, G1.ctypes.data, G1.nbytes)
        prev = mt.mt_k_gemm_wait_limit_ns(0)
        try:
            with pytest.raises(mt.MTError) as e:
                mt.mt_train_step(ctx, toks[1][0].ctypes.data, toks[1][1].ctypes.data)
        finally:
            mt.mt_k_gemm_wait_limit_ns(prev)
        assert e.value.code == -9, str(e.value)
        mt.mt_flush(ctx)
        M, V, step = _opt_state(mt, ctx, A.size)
        p, m, v = oracle.adamw_update(P0.astype(np.float64), G1.astype(np.float64), 0.0, 0.0, 1, **HYP)
        assert rel(A.astype(np.float64), p) <= 1e-6
        assert rel(M.astype(np.float64), m) <= 1e-6 and rel(V.astype(np.float64), v) <= 1e-6
        assert step == 2  # the failed step counts: its updates are skipped, as documented
        P2 = A.copy()
        loss3 = mt.mt_train_step(ctx, toks[2][0].ctypes.data, toks[2][1].ctypes.data)
        G3 = np.empty_like(A)
        mt.mt_get_grads(ctx, G3.ctypes.data, G3.nbytes)
    finally:
        mt.mt_destroy(ctx)
    Wb = {k: oracle.bf16_round(w.astype(np.float32)) for k, w in oracle.unpack_arena(P2, c).items()}
    rloss, RG = oracle.train_step_grads(Wb, toks[2][0], toks[2][1], c)
    assert abs(loss3 - rloss) <= 1e-2
    G = oracle.unpack_arena(G3, c)
    assert max(rel(G[k], RG[k]) for k in RG) <= 2e-2


def test_host_stall_times_out_and_the_context_survives(monkeypatch):
    """A 3 s host stall on the gradient-offload stream against a 1 s wait
    limit: MT_ERR_TIMEOUT, no update, and once the stall is over the same
    context trains correctly; mt_destroy returns."""
    monkeypatch.setenv("MT_WAIT_LIMIT_S", "1")
    arena, mt = _libs()
    c = oracle.OracleConfig(**TINY)
    cfg, A, ctx = _ctx(TINY, 0)
    P0 = A.copy()
    tok, lab = synth.tokens_labels(TINY["b"], TINY["s"], TINY["V"], 0)
    try:
        mt.mt_inject_host_stall(ctx, 2, 3000)
        t0 = time.time()
        with pytest.raises(mt.MTError) as e:
            mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
        assert e.value.code == -7, str(e.value)
        assert time.time() - t0 < 30
        assert np.array_equal(A, P0)
        time.sleep(3.5)  # the stall is over
        loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
        with pytest.raises(mt.MTError):
            mt.mt_inject_host_stall(ctx, 3, 10)
    finally:
        t0 = time.time()
        mt.mt_destroy(ctx)
        assert time.time() - t0 < 30
    Wb = {k: oracle.bf16_round(w.astype(np.float32)) for k, w in oracle.unpack_arena(P0, c).items()}
    rloss, _ = oracle.train_step_grads(Wb, tok, lab, c)
    assert abs(loss - rloss) <= 1e-2


def test_oversized_config_fails_before_allocating():
    """b*s so large that the boundary activations alone exceed the device:
    MT_ERR_NOMEM from the budget preflight, with no device memory taken."""
    import torch
    arena, mt = _libs()
    shape = dict(L=8, d=4096, H=32, Hkv=32, F=11008, V=32000, b=16, s=65536)
    cfg = arena.config(shape)
    assert mt.mt_device_bytes(cfg) > 2 * torch.cuda.mem_get_info()[1]
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    with pytest.raises(mt.MTError) as e:
        mt.mt_create(cfg)
    assert e.value.code == -4
    assert "device budget" in str(e.value)
    assert abs(torch.cuda.mem_get_info()[0] - free0) < (64 << 20)


def test_device_footprint_is_the_documented_one_and_flat_in_layers():
    """cudaMemGetInfo across mt_create: the context takes mt_device_bytes(cfg)
    (within allocation granularity), and going from 2 to 6 layers at equal
    shapes adds exactly the four extra boundary activations."""
    import torch
    arena, mt = _libs()
    base = dict(d=1024, H=8, Hkv=8, F=2752, V=4096, b=4, s=1024)
    T, d = base["b"] * base["s"], base["d"]
    warm = mt.mt_create(arena.config(dict(base, L=1)))  # module load, first-use allocations
    mt.mt_destroy(warm)
    deltas = {}
    for L in (2, 6):
        cfg = arena.config(dict(base, L=L))
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        ctx = mt.mt_create(cfg)
        try:
            deltas[L] = free0 - torch.cuda.mem_get_info()[0]
        finally:
            mt.mt_destroy(ctx)
        want = mt.mt_device_bytes(cfg)
        assert abs(deltas[L] - want) <= (32 << 20), (L, deltas[L], want)
    extra = 4 * T * d * 4
    assert abs((deltas[6] - deltas[2]) - extra) <= (4 << 20), (deltas, extra)
    b2 = mt.mt_device_bytes(arena.config(dict(base, L=2)))
    b6 = mt.mt_device_bytes(arena.config(dict(base, L=6)))
    assert b6 - b2 == extra
    # with the boundary activations offloaded the footprint is flat in L
    cfg = arena.config(dict(base, L=6))
    cfg.flags = mt.MT_FLAG_OFFLOAD_ACTS
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    ctx = mt.mt_create(cfg)
    try:
        delta = free0 - torch.cuda.mem_get_info()[0]
    finally:
        mt.mt_destroy(ctx)
    assert abs(delta - mt.mt_device_bytes(cfg)) <= (32 << 20)
    assert abs(delta - deltas[2]) <= (32 << 20)  # three boundary slots, as the resident 2-layer context
