// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "mt.h"

namespace mt {

enum GemmEpi : int { EPI_BF16 = 0, EPI_F32 = 1, EPI_F32_ADD = 2 };

// C[M,N] = A[M,K] * B[N,K]^T (+ R for EPI_F32_ADD; R may alias C).
//   A K-major: element (m,k) at A[m*lda + k];  A MN-major: at A[k*lda + m]
//   B K-major: element (n,k) at B[n*ldb + k];  B MN-major: at B[k*ldb + n]
struct GemmDesc {
  const void* A;
  int64_t lda;
  bool a_mn;
  const void* B;
  int64_t ldb;
  bool b_mn;
  void* C;
  int64_t ldc;
  int epi;
  const float* R;
  int64_t ldr;
  int M, N, K;
};

int gemm_bf16(const GemmDesc& g, cudaStream_t st, int* dev_err);

}  // namespace mt
