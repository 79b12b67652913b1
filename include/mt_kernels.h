/*
 * mt_kernels.h -- the individual hot-path kernels of one streamed decoder
 * layer, exposed through the C ABI so that each can be checked against the
 * oracle and timed on its own. mt_train_step (mt.h) launches the same kernels.
 *
 * Conventions:
 *   - all tensor pointers are DEVICE pointers owned by the caller; nothing is
 *     allocated or freed by these calls;
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream); the call only enqueues work and returns;
 *   - `dev_err` is an optional device int32 the kernels set to a nonzero code
 *     when a bounded wait inside them runs out (the kernel then returns early
 *     and its outputs are undefined); NULL disables the report;
 *   - bf16 tensors are IEEE bfloat16 bit patterns (uint16); row-major unless
 *     stated; every base pointer and row pitch must be 16-byte aligned;
 *   - return MT_OK or a negative MT_ERR_* (mt.h) for bad arguments or a failed
 *     launch; argument errors are found before anything is enqueued.
 */
#ifndef MT_KERNELS_H_
#define MT_KERNELS_H_

#include <stddef.h>
#include <stdint.h>

#include "mt.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Output kinds of mt_k_gemm_bf16. */
#define MT_GEMM_OUT_BF16 0    /* C bf16 = A B^T (round to nearest even) */
#define MT_GEMM_OUT_F32 1     /* C fp32 = A B^T */
#define MT_GEMM_OUT_F32_ADD 2 /* C fp32 = R + A B^T; R fp32, may equal C */

/* Dense product C[M,N] = A[M,K] B[N,K]^T with bf16 inputs and fp32
 * accumulation on the tcgen05 tensor cores: the matmuls a streamed layer runs
 * (MegaTrain abstract; saify.me, "The memory-centric design": "runs the
 * matmuls"), in forward (X W^T), input-gradient (dY W) and weight-gradient
 * (dY^T X) form.
 *   A: a_mn_major = 0: element (m,k) at A[m*lda + k]; = 1: at A[k*lda + m]
 *   B: b_mn_major = 0: element (n,k) at B[n*ldb + k]; = 1: at B[k*ldb + n]
 *   C: element (m,n) at C[m*ldc + n]; R likewise with ldr.
 * lda, ldb, ldc: multiples of 8 elements; ldr: multiple of 4. K may be any
 * positive size (the tail is zero-filled); M, N any size >= 0. */
int mt_k_gemm_bf16(const void* A, int64_t lda, int a_mn_major, const void* B, int64_t ldb, int b_mn_major,
                   void* C, int64_t ldc, int out_kind, const float* R, int64_t ldr, int M, int N, int K,
                   void* stream, int32_t* dev_err);

#ifdef __cplusplus
}
#endif
#endif /* MT_KERNELS_H_ */
