// C-ABI entry points of the individual kernels (declared in mt_kernels.h).
#include "mt_internal.h"
#include "mt_kernels.h"

extern "C" int mt_k_gemm_bf16(const void* A, int64_t lda, int a_mn_major, const void* B, int64_t ldb,
                              int b_mn_major, void* C, int64_t ldc, int out_kind, const float* R, int64_t ldr,
                              int M, int N, int K, void* stream, int32_t* dev_err) {
  if (out_kind < MT_GEMM_OUT_BF16 || out_kind > MT_GEMM_OUT_F32_ADD) return MT_ERR_ARG;
  if (M < 0 || N < 0 || K < 0) return MT_ERR_ARG;
  mt::GemmDesc g{A, lda, a_mn_major != 0, B, ldb, b_mn_major != 0, C, ldc, out_kind, R, ldr, M, N, K};
  return mt::gemm_bf16(g, static_cast<cudaStream_t>(stream), dev_err);
}
