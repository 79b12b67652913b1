"""Parity at the benchmark's full size (llama-1.3b: T = 8 x 2048 tokens, d 2048,
16 heads of 128, FFN 5504, vocab 32000), in the launch configuration the
bench uses.

The oracle cannot run a whole step at this size, so:
- every GEMM shape of the layer (forward, input-gradient and weight-gradient
  forms, and the LM head) is checked on sampled outputs, each recomputed as an
  fp64 dot product of the same bf16 operands;
- attention forward and backward are checked on sampled query rows (the
  oracle's attention on that row's causal prefix) and on the last keys' dK/dV;
- one full training step through mt_train_step is checked against properties
  that hold at any size: the loss at initialisation (ln V + sigma^2 / 2), every
  gradient finite, exactly-zero gradient rows for embedding rows the batch does
  not use, LM-head gradient columns summing to zero over the vocabulary
  (softmax minus one-hot sums to zero per token), and the host update equal to
  the oracle's AdamW applied to the GPU's gradients on sampled entries.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
SH = synth.WORKLOADS["llama-1.3b"]
T, D, F, V, H, HD, B, S = 16384, 2048, 5504, 32000, 16, 128, 8, 2048


def _mt():
    from host_memory_streamed_layer_b200 import mt
    return mt


GEMMS = [("qkv_fwd", T, 3 * D, D, "fwd"), ("o_fwd", T, D, D, "fwd"), ("gu_fwd", T, 2 * F, D, "fwd"),
         ("down_fwd", T, D, F, "fwd"), ("down_dx", T, F, D, "dx"), ("gu_dx", T, D, 2 * F, "dx"),
         ("qkv_dx", T, D, 3 * D, "dx"), ("down_dw", D, F, T, "dw"), ("gu_dw", 2 * F, D, T, "dw"),
         ("qkv_dw", 3 * D, D, T, "dw"), ("o_dw", D, D, T, "dw"), ("head_fwd", 4096, V, D, "fwd"),
         ("head_dx", 4096, D, V, "dx"), ("head_dw", V, D, 4096, "dw")]


@pytest.mark.parametrize("name,M,N,K,form", GEMMS)
def test_gemm_full_shape_sampled(name, M, N, K, form):
    mt = _mt()
    g = torch.Generator(device=DEV).manual_seed(M + N + K)
    A = torch.randn(M, K, device=DEV, generator=g).to(torch.bfloat16)
    Bm = torch.randn(N, K, device=DEV, generator=g).to(torch.bfloat16)
    if form == "fwd":
        Ad, a_mn, lda, Bd, b_mn, ldb = A, 0, K, Bm, 0, K
    elif form == "dx":
        Ad, a_mn, lda, Bd, b_mn, ldb = A, 0, K, Bm.t().contiguous(), 1, N
    else:
        Ad, a_mn, lda, Bd, b_mn, ldb = A.t().contiguous(), 1, M, Bm.t().contiguous(), 1, N
    C = torch.empty(M, N, device=DEV, dtype=torch.float32)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    mt.mt_k_gemm_bf16(Ad.data_ptr(), lda, a_mn, Bd.data_ptr(), ldb, b_mn, C.data_ptr(), N, mt.GEMM_OUT_F32, 0, 0,
                      M, N, K, torch.cuda.current_stream().cuda_stream, err.data_ptr())
    torch.cuda.synchronize()
    assert err.item() == 0
    rng = np.random.default_rng(K)
    rows = rng.integers(0, M, 256)
    cols = rng.integers(0, N, 256)
    rows[:4] = [0, 0, M - 1, M - 1]
    cols[:4] = [0, N - 1, 0, N - 1]
    a = A[torch.tensor(rows, device=DEV)].double().cpu().numpy()
    b = Bm[torch.tensor(cols, device=DEV)].double().cpu().numpy()
    ref = np.sum(a * b, axis=1)
    got = C[torch.tensor(rows, device=DEV), torch.tensor(cols, device=DEV)].double().cpu().numpy()
    bound = np.sum(np.abs(a * b), axis=1) * K * 2.0 ** -23 + 1e-6
    assert np.all(np.abs(got - ref) <= bound), np.max(np.abs(got - ref) / bound)


@pytest.mark.parametrize("impl", ["mma", "tc"])
def test_attention_full_shape_sampled(impl):
    mt = _mt()
    g = torch.Generator(device=DEV).manual_seed(7)
    ld = 3 * H * HD
    qkv = torch.randn(T, ld, device=DEV, generator=g).to(torch.bfloat16)
    o = torch.empty(T, H * HD, device=DEV, dtype=torch.bfloat16)
    lse = torch.empty(B, H, S, device=DEV)
    p = qkv.data_ptr()
    pk, pv = p + 2 * H * HD, p + 4 * H * HD
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    mt.mt_k_attn_fwd_tc(p, pk, pv, ld, o.data_ptr(), H * HD, lse.data_ptr(), B, S, H, H, HD, 0, err.data_ptr())
    do = torch.randn(T, H * HD, device=DEV, generator=g).to(torch.bfloat16)
    dvec = torch.empty(B, H, S, device=DEV)
    dqa = torch.empty(T, H * HD, device=DEV)
    dqkv = torch.empty(T, ld, device=DEV, dtype=torch.bfloat16)
    dp = dqkv.data_ptr()
    bwd = mt.mt_k_attn_bwd if impl == "mma" else mt.mt_k_attn_bwd_tc
    bwd(p, pk, pv, ld, o.data_ptr(), do.data_ptr(), H * HD, lse.data_ptr(), dvec.data_ptr(),
        dqa.data_ptr(), H * HD, dp, ld, dp + 2 * H * HD, dp + 4 * H * HD, ld, B, S, H, H, HD)
    torch.cuda.synchronize()
    assert err.item() == 0
    Q = qkv.view(B, S, 3, H, HD)
    rng = np.random.default_rng(0)
    for bi, h, i in [(0, 0, 0), (7, 15, S - 1), *zip(rng.integers(0, B, 6), rng.integers(0, H, 6),
                                                     rng.integers(0, S, 6))]:
        bi, h, i = int(bi), int(h), int(i)
        q = Q[bi, :i + 1, 0, h].double().cpu().numpy()[None, :, None]
        k = Q[bi, :i + 1, 1, h].double().cpu().numpy()[None, :, None]
        v = Q[bi, :i + 1, 2, h].double().cpu().numpy()[None, :, None]
        ro, P = oracle.attention_fwd(q, k, v)
        got = o[bi * S + i, h * HD:(h + 1) * HD].double().cpu().numpy()
        assert np.linalg.norm(got - ro[0, i, 0]) <= 1e-2 * np.linalg.norm(ro[0, i, 0]) + 1e-3
        assert abs(lse[bi, h, i].item() - oracle.attention_lse(q, k)[0, 0, i]) < 1e-3
        # dq of row i needs only this prefix
        dor = do[bi * S:bi * S + i + 1, h * HD:(h + 1) * HD].double().cpu().numpy()[None, :, None]
        rdq, _, _ = oracle.attention_bwd(q, k, v, P, dor)
        gq = dqkv[bi * S + i, h * HD:(h + 1) * HD].double().cpu().numpy()
        assert np.linalg.norm(gq - rdq[0, i, 0]) <= 2e-2 * np.linalg.norm(rdq[0, i, 0]) + 1e-3
    # dK, dV of the last 16 keys of sequence 3, head 5 (only the last queries see them)
    bi, h = 3, 5
    q = Q[bi, :, 0, h].double().cpu().numpy()[None, :, None]
    k = Q[bi, :, 1, h].double().cpu().numpy()[None, :, None]
    v = Q[bi, :, 2, h].double().cpu().numpy()[None, :, None]
    _, P = oracle.attention_fwd(q, k, v)
    dor = do[bi * S:(bi + 1) * S, h * HD:(h + 1) * HD].double().cpu().numpy()[None, :, None]
    _, rdk, rdv = oracle.attention_bwd(q, k, v, P, dor)
    gk = dqkv[bi * S + S - 16:bi * S + S, (H + h) * HD:(H + h + 1) * HD].double().cpu().numpy()
    gv = dqkv[bi * S + S - 16:bi * S + S, (2 * H + h) * HD:(2 * H + h + 1) * HD].double().cpu().numpy()
    assert np.linalg.norm(gk - rdk[0, -16:, 0]) <= 2e-2 * np.linalg.norm(rdk[0, -16:, 0])
    assert np.linalg.norm(gv - rdv[0, -16:, 0]) <= 2e-2 * np.linalg.norm(rdv[0, -16:, 0])


@pytest.mark.parametrize("impl", ["mma", "tc", "tc_pingpong", "tc_split"])
def test_attention_whole_heads_full_length(impl):
    """Every row of two whole heads at the full 2048-token length, element by
    element (per-row relative L2): o, the log-sum-exp, dq, dk and dv against
    the oracle's attention of the whole sequence. Each query row's last key
    block is the masked diagonal one and its earlier blocks run the mask-free
    instantiation, and each key row is seen by both kinds, so both are covered
    at full length. GQA (4 query heads per KV head) is on, so dk and dv sum
    over a group."""
    mt = _mt()
    Hkv = H // 4
    g = torch.Generator(device=DEV).manual_seed(11)
    ld = (H + 2 * Hkv) * HD
    qkv = torch.randn(T, ld, device=DEV, generator=g).to(torch.bfloat16)
    o = torch.empty(T, H * HD, device=DEV, dtype=torch.bfloat16)
    lse = torch.empty(B, H, S, device=DEV)
    p = qkv.data_ptr()
    pk, pv = p + 2 * H * HD, p + 2 * (H + Hkv) * HD
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    fwd = mt.mt_k_attn_fwd if impl == "mma" else mt.mt_k_attn_fwd_tc
    was = mt.mt_k_attn_fwd_variant(mt.ATTN_PINGPONG if impl == "tc_pingpong" else mt.ATTN_ONE_TILE)
    try:
        fwd(p, pk, pv, ld, o.data_ptr(), H * HD, lse.data_ptr(), B, S, H, Hkv, HD, 0,
            *([] if impl == "mma" else [err.data_ptr()]))
    finally:
        mt.mt_k_attn_fwd_variant(was)
    do = torch.randn(T, H * HD, device=DEV, generator=g).to(torch.bfloat16)
    dvec = torch.empty(B, H, S, device=DEV)
    dqa = torch.empty(T, H * HD, device=DEV)
    dqkv = torch.empty(T, ld, device=DEV, dtype=torch.bfloat16)
    dp = dqkv.data_ptr()
    bwd = mt.mt_k_attn_bwd if impl == "mma" else mt.mt_k_attn_bwd_tc
    kw = {} if impl == "mma" else {"dev_err": err.data_ptr()}
    was = mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_SPLIT if impl == "tc_split" else mt.ATTN_BWD_FUSED)
    try:
        bwd(p, pk, pv, ld, o.data_ptr(), do.data_ptr(), H * HD, lse.data_ptr(), dvec.data_ptr(), dqa.data_ptr(),
            H * HD, dp, ld, dp + 2 * H * HD, dp + 2 * (H + Hkv) * HD, ld, B, S, H, Hkv, HD, **kw)
    finally:
        mt.mt_k_attn_bwd_variant(was)
    torch.cuda.synchronize()
    assert err.item() == 0

    def rows_close(got, ref, tol, floor):
        num = np.linalg.norm(got - ref, axis=-1)
        den = np.linalg.norm(ref, axis=-1)
        assert np.all(num <= tol * den + floor), float(np.max(num / (den + 1e-30)))

    X = qkv.double().cpu().numpy()
    dO = do.double().cpu().numpy()
    G = dqkv.double().cpu().numpy()
    O = o.double().cpu().numpy()
    for bi, kvh in [(2, 1), (6, 3)]:
        rows = slice(bi * S, (bi + 1) * S)
        k = X[rows, (H + kvh) * HD:(H + kvh + 1) * HD][None, :, None]
        v = X[rows, (H + Hkv + kvh) * HD:(H + Hkv + kvh + 1) * HD][None, :, None]
        dk = np.zeros((S, HD))
        dv = np.zeros((S, HD))
        for h in range(kvh * 4, kvh * 4 + 4):
            q = X[rows, h * HD:(h + 1) * HD][None, :, None]
            ro, P = oracle.attention_fwd(q, k, v)
            rows_close(O[rows, h * HD:(h + 1) * HD], ro[0, :, 0], 1e-2, 1e-3)
            assert np.max(np.abs(lse[bi, h].double().cpu().numpy() - oracle.attention_lse(q, k)[0, 0])) < 1e-3
            rdq, rdk, rdv = oracle.attention_bwd(q, k, v, P, dO[rows, h * HD:(h + 1) * HD][None, :, None])
            rows_close(G[rows, h * HD:(h + 1) * HD], rdq[0, :, 0], 2e-2, 1e-3)
            dk += rdk[0, :, 0]
            dv += rdv[0, :, 0]
        rows_close(G[rows, (H + kvh) * HD:(H + kvh + 1) * HD], dk, 2e-2, 1e-3)
        rows_close(G[rows, (H + Hkv + kvh) * HD:(H + Hkv + kvh + 1) * HD], dv, 2e-2, 1e-3)


def test_full_step_properties():
    from host_memory_streamed_layer_b200 import arena, mt
    cfg = arena.config(SH)
    cfg.seed = 99
    ctx = mt.mt_create(cfg)
    try:
        n = mt.mt_arena_bytes(cfg) // 4
        P0 = np.empty(n, dtype=np.float32)
        mt.mt_get_params(ctx, P0.ctypes.data, P0.nbytes)
        tok, lab = synth.tokens_labels(SH["b"], SH["s"], SH["V"], 5)
        loss = mt.mt_train_step(ctx, tok.ctypes.data, lab.ctypes.data)
        G = np.empty(n, dtype=np.float32)
        P1 = np.empty(n, dtype=np.float32)
        mt.mt_get_grads(ctx, G.ctypes.data, G.nbytes)
        mt.mt_get_params(ctx, P1.ctypes.data, P1.nbytes)
        st = mt.mt_get_stats(ctx)
    finally:
        mt.mt_destroy(ctx)
    assert abs(loss - (math.log(V) + 0.0004 * D / 2)) < 0.15, loss
    assert np.isfinite(G).all()
    off_e, n_e = mt.mt_tensor_offset(cfg, -1, mt.MT_T_EMBED)
    gE = G[off_e:off_e + n_e].reshape(V, D)
    used = np.zeros(V, dtype=bool)
    used[np.unique(tok)] = True
    assert np.all(gE[~used] == 0.0) and np.all(np.abs(gE[used]).sum(axis=1) > 0)
    off_h, n_h = mt.mt_tensor_offset(cfg, -1, mt.MT_T_LM_HEAD)
    gW = G[off_h:off_h + n_h].reshape(V, D).astype(np.float64)
    assert np.linalg.norm(gW.sum(axis=0)) <= 1e-3 * np.linalg.norm(gW) * math.sqrt(V)
    for layer in range(SH["L"]):
        for tid in range(9):
            o, k = mt.mt_tensor_offset(cfg, layer, tid)
            assert np.linalg.norm(G[o:o + k]) > 0, (layer, tid)
    rng = np.random.default_rng(1)
    idx = rng.integers(0, n, 200000)
    pa, _, _ = oracle.adamw_update(P0[idx], G[idx], 0, 0, 1, 1e-3, 0.9, 0.95, 1e-8, 0.1)
    assert np.allclose(P1[idx], pa, rtol=0, atol=2e-8 + 1e-6 * np.abs(pa))
    assert st["wait_weights_ms"] < 0.1 * st["step_ms"]  # prefetch keeps the compute stream fed


@pytest.mark.parametrize("layer", [0, SH["L"] - 1])
def test_layer_local_parity_full_shape(layer):
    """Layer-local parity at the full 1.3B shape, in the launch configuration of
    the training step: mt_layer_fwd_bwd runs the engine's layer forward and
    backward on all 8 x 2048 tokens; the upstream gradient is nonzero only for
    sequences 0 and 1, so the other sequences' input gradients are exactly
    zero and every weight gradient is the sum over those two sequences, which
    the oracle recomputes in fp64 (x_{l+1} and dx_l of sequences 0 and 1, all
    nine weight gradients)."""
    from host_memory_streamed_layer_b200 import arena, mt
    from layer_parity import layer_check
    cfg = arena.config(SH)
    cfg.seed = 5
    ctx = mt.mt_create(cfg)
    try:
        n = mt.mt_arena_bytes(cfg) // 4
        P = np.empty(n, dtype=np.float32)
        mt.mt_get_params(ctx, P.ctypes.data, P.nbytes)
        c = oracle.OracleConfig(**SH)
        shapes = {tid: shp for lay, tid, _, shp in oracle.arena_layout(c)[0] if lay == layer}
        W = {}
        for tid in range(9):
            o, k = mt.mt_tensor_offset(cfg, layer, tid)
            W[tid] = oracle.bf16_round(P[o:o + k]).astype(np.float64).reshape(shapes[tid])
        del P
        rng = np.random.default_rng(layer)
        x = rng.normal(size=(T, D)).astype(np.float32)
        dxn = np.zeros((T, D), dtype=np.float32)
        dxn[:2 * S] = rng.normal(size=(2 * S, D)).astype(np.float32)
        xo, dxi, _ = layer_check(mt, ctx, cfg, SH, layer, W, x, dxn, [0, 1])
        assert np.all(dxi[2 * S:] == 0.0)
        assert np.isfinite(xo).all()
    finally:
        mt.mt_destroy(ctx)


def test_head_parity_full_shape():
    """Head + cross-entropy parity at the full 1.3B shape (8 x 2048 tokens,
    vocab 32000) through mt_head_fwd_bwd, against the oracle token-chunked."""
    from host_memory_streamed_layer_b200 import arena, mt
    from layer_parity import head_check
    cfg = arena.config(SH)
    cfg.seed = 9
    ctx = mt.mt_create(cfg)
    try:
        x = np.random.default_rng(3).normal(size=(T, D)).astype(np.float32)
        _, lab = synth.tokens_labels(B, S, V, 4)
        loss = head_check(mt, ctx, cfg, SH, x, np.ascontiguousarray(lab.reshape(-1)).astype(np.int32), chunk=2048)
        assert abs(loss - (math.log(V) + 0.0004 * D / 2)) < 0.15  # unit-RMS inputs: the closed form holds
    finally:
        mt.mt_destroy(ctx)
