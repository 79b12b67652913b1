"""Parity of the tcgen05 GEMM (through the C ABI) with an fp64 CPU product of
the same bf16 inputs, in the three operand forms the layer uses, across
ragged sizes (M, N, K not multiples of the tile), both tile widths of the
single-CTA kernel and both tile widths of the CTA-pair kernel."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _mt():
    from host_memory_streamed_layer_b200 import mt
    return mt


def _ref(A, B):  # fp64 product of the exact bf16 values
    return A.double().cpu() @ B.double().cpu().T


SMALL = [(128, 256, 64), (256, 512, 128), (300, 200, 100), (1000, 768, 688), (64, 48, 40), (257, 1376, 256)]
# Large enough for the CTA-pair kernel (at least one 256-row tile per SM pair
# of a 148-SM part); the last three are ragged in M, N and K and take 256-wide
# pair tiles, 128-wide pair tiles (they quantize into waves better), and
# 128-wide pair tiles because 256-wide ones would not fill every pair.
LARGE = [(4096, 2304, 512), (2048, 4096, 1024), (2200, 5504, 200), (4000, 2344, 328), (2304, 2048, 4160)]
CASES = [(*c, "auto") for c in SMALL] + [(*c, v) for c in LARGE for v in ("auto", "single", "pair")]


@pytest.mark.parametrize("M,N,K,variant", CASES)
@pytest.mark.parametrize("form", ["fwd", "dx", "dw"])
@pytest.mark.parametrize("out", ["bf16", "f32", "f32_add"])
def test_gemm_matches_fp64(M, N, K, variant, form, out):
    """variant: the GEMM kernel family (auto; single-CTA tiles only; CTA-pair
    tiles wherever the problem has one per SM pair)."""
    mt = _mt()
    prev = mt.mt_k_gemm_variant({"auto": mt.GEMM_AUTO, "single": mt.GEMM_SINGLE, "pair": mt.GEMM_PAIR}[variant])
    try:
        _gemm_case(mt, M, N, K, form, out)
    finally:
        mt.mt_k_gemm_variant(prev)


def _gemm_case(mt, M, N, K, form, out):
    g = torch.Generator(device="cpu").manual_seed(M * 7 + N * 3 + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, generator=g).to(torch.bfloat16)
    ref = _ref(A, B)
    dev = torch.device("cuda")
    # Store the operands in the memory order the form uses.
    if form == "fwd":
        Ad, a_mn, lda = A.to(dev).contiguous(), 0, K
        Bd, b_mn, ldb = B.to(dev).contiguous(), 0, K
    elif form == "dx":
        Ad, a_mn, lda = A.to(dev).contiguous(), 0, K
        Bd, b_mn, ldb = B.t().contiguous().to(dev), 1, N  # stored [K, N]
    else:
        Ad, a_mn, lda = A.t().contiguous().to(dev), 1, M  # stored [K, M]
        Bd, b_mn, ldb = B.t().contiguous().to(dev), 1, N
    if (lda % 8) or (ldb % 8) or (N % 8):
        pytest.skip("row pitch must be a multiple of 8 elements")
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    kind = {"bf16": mt.GEMM_OUT_BF16, "f32": mt.GEMM_OUT_F32, "f32_add": mt.GEMM_OUT_F32_ADD}[out]
    C = torch.empty(M, N, dtype=torch.bfloat16 if out == "bf16" else torch.float32, device=dev)
    R = None
    if out == "f32_add":
        R = torch.randn(M, N, generator=g).to(dev)
        C.copy_(R)  # accumulate in place: C = C + A B^T
        ref = ref + R.double().cpu()
    mt.mt_k_gemm_bf16(Ad.data_ptr(), lda, a_mn, Bd.data_ptr(), ldb, b_mn, C.data_ptr(), N, kind,
                      C.data_ptr() if R is not None else 0, N, M, N, K,
                      torch.cuda.current_stream().cuda_stream, err.data_ptr())
    torch.cuda.synchronize()
    assert err.item() == 0
    got = C.double().cpu()
    # fp32 accumulation of K exact bf16 products: error ~ K * 2^-24 * sum|a b|;
    # bf16 output adds one rounding (2^-9 relative).
    bound = (torch.abs(A.double()) @ torch.abs(B.double()).T) * (K * 2.0 ** -23)
    if out == "bf16":
        bound = bound + ref.abs() * 2.0 ** -8
    assert torch.all((got - ref).abs() <= bound + 1e-6), float(((got - ref).abs() - bound).max())


def test_gemm_rejects_misaligned_pitch():
    mt = _mt()
    dev = torch.device("cuda")
    A = torch.zeros(16, 12, dtype=torch.bfloat16, device=dev)
    C = torch.zeros(16, 16, dtype=torch.float32, device=dev)
    with pytest.raises(mt.MTError):
        mt.mt_k_gemm_bf16(A.data_ptr(), 12, 0, A.data_ptr(), 12, 0, C.data_ptr(), 16, mt.GEMM_OUT_F32,
                          0, 0, 16, 16, 12)
