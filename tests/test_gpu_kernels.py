"""Parity of each hot-path kernel (through the C ABI) with the oracle, on
seeded inputs that span several tiles and a ragged tail. Inputs are rounded
to bf16 where the kernel reads bf16, and the oracle computes in fp64 on those
same values. Tolerances follow from the output rounding (bf16: 2^-8 relative)
and fp32 arithmetic."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _mt():
    from host_memory_streamed_layer_b200 import mt
    return mt


def bf(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(DEV)


def f32(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(DEV)


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(a, b, floor=1e-300):
    """||a - b|| / ||b||; `floor` bounds the denominator when b is (near) 0."""
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), floor)


def sync():
    torch.cuda.synchronize()


@pytest.mark.parametrize("T,d", [(300, 256), (37, 2048), (5, 5120), (129, 4096)])
def test_rmsnorm_fwd(T, d):
    mt = _mt()
    rng = np.random.default_rng(T + d)
    x = rng.normal(0, 2, (T, d)).astype(np.float32)
    g = bf(1 + 0.1 * rng.normal(size=d))
    y = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    r = torch.empty(T, dtype=torch.float32, device=DEV)
    xd = f32(x)
    mt.mt_k_rmsnorm_fwd(xd.data_ptr(), g.data_ptr(), y.data_ptr(), r.data_ptr(), T, d, 1e-5)
    sync()
    ref, rr = oracle.rmsnorm_fwd(x.astype(np.float64), np64(g), 1e-5)
    assert np.all(np.abs(np64(y) - ref) <= 2 ** -8 * np.abs(ref) + 1e-6)
    assert np.allclose(np64(r), rr[:, 0], rtol=1e-5)


@pytest.mark.parametrize("T,d", [(300, 256), (37, 2048), (1000, 5120)])
def test_rmsnorm_bwd(T, d):
    mt = _mt()
    rng = np.random.default_rng(T * d)
    x = rng.normal(0, 2, (T, d)).astype(np.float32)
    dy = rng.normal(size=(T, d)).astype(np.float32)
    dres = rng.normal(size=(T, d)).astype(np.float32)
    g = bf(1 + 0.1 * rng.normal(size=d))
    _, r = oracle.rmsnorm_fwd(x.astype(np.float64), np64(g), 1e-5)
    dx = torch.empty(T, d, device=DEV)
    dxb = torch.empty(T, d, dtype=torch.bfloat16, device=DEV)
    part = torch.empty(mt.mt_k_rmsnorm_bwd_partial_floats(T, d), device=DEV)
    dg = torch.empty(d, device=DEV)
    # keep every device input referenced until the kernel has run
    xd, rd, dyd, dresd = f32(x), f32(r[:, 0]), f32(dy), f32(dres)
    mt.mt_k_rmsnorm_bwd(xd.data_ptr(), g.data_ptr(), rd.data_ptr(), dyd.data_ptr(), dresd.data_ptr(),
                        dx.data_ptr(), dxb.data_ptr(), part.data_ptr(), dg.data_ptr(), T, d)
    sync()
    rdx, rdg = oracle.rmsnorm_bwd(x.astype(np.float64), np64(g), r.astype(np.float32).astype(np.float64),
                                  dy.astype(np.float64))
    rdx = rdx + dres
    assert np.allclose(np64(dx), rdx, rtol=1e-4, atol=1e-5 * np.abs(rdx).max())
    assert np.all(np.abs(np64(dxb) - np64(dx)) <= 2 ** -8 * np.abs(np64(dx)))
    assert rel_l2(np64(dg), rdg) < 1e-5


@pytest.mark.parametrize("hd,H,Hkv,s,b", [(64, 4, 4, 128, 2), (128, 4, 2, 100, 3), (128, 40, 8, 33, 1)])
def test_rope_fwd_and_inverse(hd, H, Hkv, s, b):
    mt = _mt()
    rng = np.random.default_rng(hd + s)
    T = b * s
    ld = (H + 2 * Hkv) * hd
    buf0 = rng.normal(size=(T, ld)).astype(np.float32)
    buf = bf(buf0)
    orig = np64(buf)
    cos, sin = oracle.rope_tables(s, hd, 10000.0)
    c32, s32 = f32(cos), f32(sin)  # referenced until the end of the test
    mt.mt_k_rope(buf.data_ptr(), ld, T, s, H, hd, 0, c32.data_ptr(), s32.data_ptr(), 1.0)
    mt.mt_k_rope(buf.data_ptr(), ld, T, s, Hkv, hd, H * hd, c32.data_ptr(), s32.data_ptr(), 1.0)
    sync()
    got = np64(buf)
    q = orig[:, :H * hd].reshape(b, s, H, hd)
    k = orig[:, H * hd:(H + Hkv) * hd].reshape(b, s, Hkv, hd)
    rq = oracle.rope_fwd(q, cos, sin).reshape(T, H * hd)
    rk = oracle.rope_fwd(k, cos, sin).reshape(T, Hkv * hd)
    bound_q = 2 ** -8 * (np.abs(q) + np.roll(np.abs(q), hd // 2, axis=-1)).reshape(T, -1) + 1e-6
    bound_k = 2 ** -8 * (np.abs(k) + np.roll(np.abs(k), hd // 2, axis=-1)).reshape(T, -1) + 1e-6
    assert np.all(np.abs(got[:, :H * hd] - rq) <= bound_q)
    assert np.all(np.abs(got[:, H * hd:(H + Hkv) * hd] - rk) <= bound_k)
    assert np.array_equal(got[:, (H + Hkv) * hd:], orig[:, (H + Hkv) * hd:])  # v untouched
    # backward rotation = transpose
    dy = got[:, :H * hd].reshape(b, s, H, hd)
    mt.mt_k_rope(buf.data_ptr(), ld, T, s, H, hd, 0, c32.data_ptr(), s32.data_ptr(), -1.0)
    sync()
    back = np64(buf)[:, :H * hd]
    rb = oracle.rope_bwd(dy, cos, sin).reshape(T, H * hd)
    assert np.all(np.abs(back - rb) <= 2 ** -8 * (np.abs(dy) + np.roll(np.abs(dy), hd // 2, -1)).reshape(T, -1) + 1e-6)


@pytest.mark.parametrize("T,F", [(256, 688), (77, 5504)])
def test_swiglu(T, F):
    mt = _mt()
    rng = np.random.default_rng(F)
    gu = bf(rng.normal(0, 2, (T, 2 * F)))
    act = torch.empty(T, F, dtype=torch.bfloat16, device=DEV)
    mt.mt_k_swiglu_fwd(gu.data_ptr(), act.data_ptr(), T, F)
    dact = bf(rng.normal(size=(T, F)))
    dgu = torch.empty(T, 2 * F, dtype=torch.bfloat16, device=DEV)
    mt.mt_k_swiglu_bwd(gu.data_ptr(), dact.data_ptr(), dgu.data_ptr(), T, F)
    sync()
    g, u = np64(gu)[:, :F], np64(gu)[:, F:]
    ref = oracle.swiglu_fwd(g, u)
    assert np.all(np.abs(np64(act) - ref) <= 2 ** -8 * np.abs(ref) + 1e-6 * np.abs(u) * (1 + np.abs(g)))
    rg, ru = oracle.swiglu_bwd(g, u, np64(dact))
    got = np64(dgu)
    scale_g = np.abs(np64(dact) * u) * (1 + np.abs(g))
    assert np.all(np.abs(got[:, :F] - rg) <= 2 ** -8 * np.abs(rg) + 1e-6 * scale_g)
    assert np.all(np.abs(got[:, F:] - ru) <= 2 ** -8 * np.abs(ru) + 1e-6 * np.abs(np64(dact) * g))


def test_embedding_fwd_exact_and_bwd():
    mt = _mt()
    rng = np.random.default_rng(3)
    V, d, T = 500, 256, 1000
    E = bf(rng.normal(size=(V, d)))
    tok = rng.integers(0, V, T).astype(np.int32)
    tok[:50] = 7  # a heavily repeated token
    tok_d = torch.tensor(tok, device=DEV)
    x = torch.empty(T, d, device=DEV)
    mt.mt_k_embed_fwd(tok_d.data_ptr(), E.data_ptr(), x.data_ptr(), T, d)
    sync()
    assert np.array_equal(np64(x), np64(E)[tok])
    dx = rng.normal(size=(T, d)).astype(np.float32)
    order = np.argsort(tok, kind="stable").astype(np.int32)
    uniq, counts = np.unique(tok, return_counts=True)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = torch.empty(len(uniq), d, device=DEV)
    offs_d, order_d, dx_d = torch.tensor(offs, device=DEV), torch.tensor(order, device=DEV), f32(dx)
    mt.mt_k_embed_bwd(offs_d.data_ptr(), order_d.data_ptr(), len(uniq), dx_d.data_ptr(), rows.data_ptr(), d)
    sync()
    ref = np.zeros((V, d))
    np.add.at(ref, tok, dx.astype(np.float64))
    assert np.allclose(np64(rows), ref[uniq], rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("T,V", [(64, 1024), (9, 32000), (2, 49152), (2, 49160), (3, 152064)])
def test_softmax_ce(T, V):
    mt = _mt()
    rng = np.random.default_rng(V)
    z = (rng.normal(size=(T, V)) * 3).astype(np.float32)
    lab = rng.integers(0, V, T).astype(np.int32)
    dz = torch.empty(T, V, dtype=torch.bfloat16, device=DEV)
    loss = torch.empty(T, device=DEV)
    scale = 1.0 / 777
    zd, labd = f32(z), torch.tensor(lab, device=DEV)
    mt.mt_k_softmax_ce(zd.data_ptr(), V, labd.data_ptr(), dz.data_ptr(), V, loss.data_ptr(), T, V, scale)
    sync()
    rl, rg = oracle.softmax_ce(z.astype(np.float64), lab)
    assert np.allclose(np64(loss), rl, rtol=1e-5, atol=1e-5)
    ref = rg * scale
    assert np.all(np.abs(np64(dz) - ref) <= 2 ** -8 * np.abs(ref) + 1e-7 * scale)


ATTN = [(64, 4, 4, 128, 2), (128, 4, 2, 100, 3), (128, 8, 1, 200, 1), (64, 2, 2, 1, 2), (128, 4, 4, 64, 1),
        (128, 2, 2, 384, 2), (64, 4, 1, 300, 2), (128, 4, 2, 700, 2)]


def _attn_inputs(hd, H, Hkv, s, b, seed):
    rng = np.random.default_rng(seed)
    T = b * s
    ld = (H + 2 * Hkv) * hd
    qkv = bf(rng.normal(size=(T, ld)))
    a = np64(qkv)
    q = a[:, :H * hd].reshape(b, s, H, hd)
    k = a[:, H * hd:(H + Hkv) * hd].reshape(b, s, Hkv, hd)
    v = a[:, (H + Hkv) * hd:].reshape(b, s, Hkv, hd)
    return qkv, q, k, v, ld


@pytest.mark.parametrize("impl", ["mma", "tc", "tc_pingpong"])
@pytest.mark.parametrize("hd,H,Hkv,s,b", ATTN)
def test_attention_fwd(hd, H, Hkv, s, b, impl):
    """tc: the tcgen05 forward with one query tile per CTA; tc_pingpong: two
    tiles per CTA in ping-pong (head dim 128, selected explicitly: the
    automatic choice takes it only above 8192 tokens)."""
    mt = _mt()
    if impl == "tc_pingpong" and hd != 128:
        pytest.skip("the two-tile forward is for head dim 128")
    qkv, q, k, v, ld = _attn_inputs(hd, H, Hkv, s, b, hd + s)
    T = b * s
    o = torch.empty(T, H * hd, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(b, H, s, device=DEV)
    p = qkv.data_ptr()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    if impl == "mma":
        mt.mt_k_attn_fwd(p, p + 2 * H * hd, p + 2 * (H + Hkv) * hd, ld, o.data_ptr(), H * hd, lse.data_ptr(),
                         b, s, H, Hkv, hd)
    else:
        was = mt.mt_k_attn_fwd_variant(mt.ATTN_PINGPONG if impl == "tc_pingpong" else mt.ATTN_ONE_TILE)
        try:
            mt.mt_k_attn_fwd_tc(p, p + 2 * H * hd, p + 2 * (H + Hkv) * hd, ld, o.data_ptr(), H * hd,
                                lse.data_ptr(), b, s, H, Hkv, hd, 0, err.data_ptr())
        finally:
            mt.mt_k_attn_fwd_variant(was)
    sync()
    assert err.item() == 0
    ro, _ = oracle.attention_fwd(q, k, v)
    got = np64(o).reshape(b, s, H, hd)
    assert rel_l2(got, ro) < 4e-3
    assert np.abs(got - ro).max() < 2e-2 * np.abs(v).max()
    assert np.allclose(np64(lse), oracle.attention_lse(q, k), rtol=1e-4, atol=1e-4)


def _bwd_form(mt, impl):
    """The tensor-core backward's form for impl: tc (fused dQ reductions) or
    tc_split (dK/dV key-major, dQ query-major, deterministic)."""
    return mt.ATTN_BWD_SPLIT if impl == "tc_split" else mt.ATTN_BWD_FUSED


@pytest.mark.parametrize("impl", ["mma", "tc", "tc_split"])
@pytest.mark.parametrize("hd,H,Hkv,s,b", ATTN)
def test_attention_bwd(hd, H, Hkv, s, b, impl):
    if impl == "tc" and hd != 128:
        pytest.skip("the fused tensor-core backward is for head_dim 128")
    mt = _mt()
    if impl != "mma":
        was = mt.mt_k_attn_bwd_variant(_bwd_form(mt, impl))
        try:
            _attention_bwd_case(mt, hd, H, Hkv, s, b, impl)
        finally:
            mt.mt_k_attn_bwd_variant(was)
    else:
        _attention_bwd_case(mt, hd, H, Hkv, s, b, impl)


@pytest.mark.parametrize("hd,H,Hkv,s,b", [(128, 8, 2, 1100, 2), (64, 4, 1, 700, 2)])
def test_split_attention_backward_is_bitwise_reproducible(hd, H, Hkv, s, b):
    """The split form sums each dQ element in one fixed order (the query-major
    kernel's key-block loop) and dK, dV in tensor memory: two runs on the same
    inputs give the same bits, at shapes with many key blocks per query
    block and GQA, for both head dims."""
    mt = _mt()
    qkv, q, k, v, ld = _attn_inputs(hd, H, Hkv, s, b, 3)
    T = b * s
    do = bf(np.random.default_rng(4).normal(size=(T, H * hd)))
    o = torch.empty(T, H * hd, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(b, H, s, device=DEV)
    p = qkv.data_ptr()
    pk, pv = p + 2 * H * hd, p + 2 * (H + Hkv) * hd
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    mt.mt_k_attn_fwd_tc(p, pk, pv, ld, o.data_ptr(), H * hd, lse.data_ptr(), b, s, H, Hkv, hd, 0, err.data_ptr())
    outs = []
    was = mt.mt_k_attn_bwd_variant(mt.ATTN_BWD_SPLIT)
    try:
        for _ in range(2):
            dvec = torch.empty(b, H, s, device=DEV)
            dqa = torch.full((T, H * hd), float("nan"), device=DEV)  # every element must be written
            dqkv = torch.zeros(T, ld, dtype=torch.bfloat16, device=DEV)
            dp = dqkv.data_ptr()
            mt.mt_k_attn_bwd_tc(p, pk, pv, ld, o.data_ptr(), do.data_ptr(), H * hd, lse.data_ptr(), dvec.data_ptr(),
                                dqa.data_ptr(), H * hd, dp, ld, dp + 2 * H * hd, dp + 2 * (H + Hkv) * hd, ld, b, s, H,
                                Hkv, hd, dev_err=err.data_ptr())
            sync()
            outs.append((dqkv.cpu().clone(), dqa.cpu().clone()))
    finally:
        mt.mt_k_attn_bwd_variant(was)
    assert err.item() == 0
    assert torch.isfinite(outs[0][1]).all()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    ro, P = oracle.attention_fwd(q, k, v)
    rdq, rdk, rdv = oracle.attention_bwd(q, k, v, P, np64(do).reshape(b, s, H, hd))
    g = outs[0][0].double().numpy()
    assert rel_l2(g[:, :H * hd].reshape(b, s, H, hd), rdq) < 1e-2
    assert rel_l2(g[:, H * hd:(H + Hkv) * hd].reshape(b, s, Hkv, hd), rdk) < 1e-2
    assert rel_l2(g[:, (H + Hkv) * hd:].reshape(b, s, Hkv, hd), rdv) < 1e-2


def _attention_bwd_case(mt, hd, H, Hkv, s, b, impl):
    qkv, q, k, v, ld = _attn_inputs(hd, H, Hkv, s, b, 7 * hd + s)
    T = b * s
    rng = np.random.default_rng(s)
    do = bf(rng.normal(size=(T, H * hd)))
    o = torch.empty(T, H * hd, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(b, H, s, device=DEV)
    p = qkv.data_ptr()
    pk, pv = p + 2 * H * hd, p + 2 * (H + Hkv) * hd
    mt.mt_k_attn_fwd(p, pk, pv, ld, o.data_ptr(), H * hd, lse.data_ptr(), b, s, H, Hkv, hd)
    dvec = torch.empty(b, H, s, device=DEV)
    dqa = torch.empty(T, H * hd, device=DEV)
    dqkv = torch.zeros(T, ld, dtype=torch.bfloat16, device=DEV)
    dp = dqkv.data_ptr()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    bwd = mt.mt_k_attn_bwd if impl == "mma" else mt.mt_k_attn_bwd_tc
    kw = {} if impl == "mma" else {"dev_err": err.data_ptr()}
    bwd(p, pk, pv, ld, o.data_ptr(), do.data_ptr(), H * hd, lse.data_ptr(), dvec.data_ptr(),
        dqa.data_ptr(), H * hd, dp, ld, dp + 2 * H * hd, dp + 2 * (H + Hkv) * hd, ld, b, s, H, Hkv, hd, **kw)
    sync()
    assert err.item() == 0
    ro, P = oracle.attention_fwd(q, k, v)
    rdq, rdk, rdv = oracle.attention_bwd(q, k, v, P, np64(do).reshape(b, s, H, hd))
    g = np64(dqkv)
    # With s = 1 the softmax has a single entry and dq = dk = 0 exactly; the
    # denominator floor is the scale of the gradient that flows into v.
    floor = 1e-3 * np.linalg.norm(rdv)
    assert rel_l2(g[:, :H * hd].reshape(b, s, H, hd), rdq, floor) < 1e-2
    assert rel_l2(g[:, H * hd:(H + Hkv) * hd].reshape(b, s, Hkv, hd), rdk, floor) < 1e-2
    assert rel_l2(g[:, (H + Hkv) * hd:].reshape(b, s, Hkv, hd), rdv) < 1e-2


@pytest.mark.parametrize("hd,H,Hkv,s,b", [(64, 4, 4, 128, 2), (128, 4, 2, 100, 3), (128, 16, 16, 256, 1),
                                         # large enough for the CTA-pair kernel (256- and 128-wide tiles)
                                         (128, 16, 16, 2048, 2), (64, 16, 4, 1024, 4)])
@pytest.mark.parametrize("variant", [0, 1, 2])
def test_qkv_gemm_with_rope_epilogue(hd, H, Hkv, s, b, variant):
    """q, k, v projection with RoPE fused in the epilogue = oracle RoPE of the
    fp64 product (v columns unrotated), rounded once to bf16; through each GEMM
    kernel family (automatic, single-CTA, CTA pairs)."""
    mt = _mt()
    prev = mt.mt_k_gemm_variant(variant)
    try:
        _qkv_rope_case(mt, hd, H, Hkv, s, b)
    finally:
        mt.mt_k_gemm_variant(prev)


def _qkv_rope_case(mt, hd, H, Hkv, s, b):
    rng = np.random.default_rng(hd * s)
    T, d = b * s, 256
    N = (H + 2 * Hkv) * hd
    A = bf(rng.normal(size=(T, d)))
    Bw = bf(rng.normal(size=(N, d)) * 0.05)
    cos, sin = oracle.rope_tables(s, hd, 10000.0)
    c32, s32 = f32(cos), f32(sin)
    C = torch.empty(T, N, dtype=torch.bfloat16, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    mt.mt_k_gemm_bf16_rope(A.data_ptr(), d, Bw.data_ptr(), d, C.data_ptr(), N, T, N, d, (H + Hkv) * hd, hd, s,
                           c32.data_ptr(), s32.data_ptr(), 0, err.data_ptr())
    sync()
    assert err.item() == 0
    prod = np64(A) @ np64(Bw).T
    q = oracle.rope_fwd(prod[:, :H * hd].reshape(b, s, H, hd), cos, sin).reshape(T, -1)
    k = oracle.rope_fwd(prod[:, H * hd:(H + Hkv) * hd].reshape(b, s, Hkv, hd), cos, sin).reshape(T, -1)
    ref = np.concatenate([q, k, prod[:, (H + Hkv) * hd:]], axis=1)
    got = np64(C)
    scale = np.abs(np64(A)) @ np.abs(np64(Bw)).T  # bound of |products| per element
    pair = np.concatenate([scale[:, :H * hd].reshape(T, H, hd), scale[:, H * hd:(H + Hkv) * hd].reshape(T, Hkv, hd)],
                          axis=1)
    pair = (pair + np.roll(pair, hd // 2, axis=-1)).reshape(T, -1)
    bound = 2 ** -8 * np.abs(ref) + 1e-5 * np.concatenate([pair, scale[:, (H + Hkv) * hd:]], axis=1)
    assert np.all(np.abs(got - ref) <= bound)


@pytest.mark.parametrize("impl", ["mma", "tc", "tc_split"])
@pytest.mark.parametrize("hd,H,Hkv,s,b", [(64, 4, 4, 128, 2), (128, 4, 2, 100, 3), (128, 2, 1, 300, 2)])
def test_attention_bwd_returns_pre_rope_gradients(hd, H, Hkv, s, b, impl):
    """With the RoPE tables the backward returns dL/d(pre-RoPE q, k): the
    oracle's attention backward followed by its rope_bwd."""
    if impl == "tc" and hd != 128:
        pytest.skip("the fused tensor-core backward is for head_dim 128")
    mt = _mt()
    was = mt.mt_k_attn_bwd_variant(_bwd_form(mt, impl))
    try:
        _pre_rope_case(mt, hd, H, Hkv, s, b, impl)
    finally:
        mt.mt_k_attn_bwd_variant(was)


def _pre_rope_case(mt, hd, H, Hkv, s, b, impl):
    qkv, q, k, v, ld = _attn_inputs(hd, H, Hkv, s, b, 11 * hd + s)
    T = b * s
    rng = np.random.default_rng(5 * s)
    do = bf(rng.normal(size=(T, H * hd)))
    o = torch.empty(T, H * hd, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(b, H, s, device=DEV)
    p = qkv.data_ptr()
    pk, pv = p + 2 * H * hd, p + 2 * (H + Hkv) * hd
    mt.mt_k_attn_fwd_tc(p, pk, pv, ld, o.data_ptr(), H * hd, lse.data_ptr(), b, s, H, Hkv, hd)
    cos, sin = oracle.rope_tables(s, hd, 10000.0)
    c32, s32 = f32(cos), f32(sin)
    dvec = torch.empty(b, H, s, device=DEV)
    dqa = torch.empty(T, H * hd, device=DEV)
    dqkv = torch.zeros(T, ld, dtype=torch.bfloat16, device=DEV)
    dp = dqkv.data_ptr()
    bwd = mt.mt_k_attn_bwd if impl == "mma" else mt.mt_k_attn_bwd_tc
    bwd(p, pk, pv, ld, o.data_ptr(), do.data_ptr(), H * hd, lse.data_ptr(), dvec.data_ptr(),
        dqa.data_ptr(), H * hd, dp, ld, dp + 2 * H * hd, dp + 2 * (H + Hkv) * hd, ld, b, s, H, Hkv, hd,
        c32.data_ptr(), s32.data_ptr())
    sync()
    _, P = oracle.attention_fwd(q, k, v)
    rdq, rdk, rdv = oracle.attention_bwd(q, k, v, P, np64(do).reshape(b, s, H, hd))
    rdq, rdk = oracle.rope_bwd(rdq, cos, sin), oracle.rope_bwd(rdk, cos, sin)
    g = np64(dqkv)
    assert rel_l2(g[:, :H * hd].reshape(b, s, H, hd), rdq) < 1e-2
    assert rel_l2(g[:, H * hd:(H + Hkv) * hd].reshape(b, s, Hkv, hd), rdk) < 1e-2
    assert rel_l2(g[:, (H + Hkv) * hd:].reshape(b, s, Hkv, hd), rdv) < 1e-2
