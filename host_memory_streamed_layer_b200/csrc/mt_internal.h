// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mt.h"

namespace mt {

// Status of the launch just made: MT_OK, or MT_ERR_CUDA with the CUDA message
// kept for last_launch_error() (per thread).
int launch_status();
const char* last_launch_error();

enum GemmEpi : int { EPI_BF16 = 0, EPI_F32 = 1, EPI_F32_ADD = 2, EPI_BF16_ROPE = 3 };

// RoPE applied in the epilogue (EPI_BF16_ROPE): columns [0, cols) hold heads of
// width hd whose rotate-half pairs (i, i + hd/2) are rotated by the angle of
// position (row % seq) with fp32 tables cos/sin [seq, hd/2]; other columns are
// stored unrotated.
struct RopeDesc {
  const float* cos;
  const float* sin;
  int cols, hd, seq;
};

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
  RopeDesc rope;
};

int gemm_bf16(const GemmDesc& g, cudaStream_t st, int* dev_err);
// Kernel family for later GEMMs: 0 automatic, 1 single-CTA, 2 CTA pairs; returns the previous one.
int gemm_variant(int v);
// Forward attention kernel for head dim 128 in later calls (0 automatic, 1 one
// query tile per CTA, 2 two tiles in ping-pong); returns the previous choice.
int attention_fwd_variant(int v);
// Main-loop wait limit (ns) of later single-CTA GEMM launches; returns the previous one.
uint64_t gemm_wait_limit_ns(uint64_t ns);

// 2-D bf16 TMA map: inner (contiguous) extent, outer extent, row pitch ld
// (elements), box {64, box_outer}, 128-byte swizzle, zero fill out of bounds.
bool make_tensor_map_2d_bf16(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
                             int box_outer);
// 2-D fp32 TMA map without swizzle, box {box_inner, box_outer}.
bool make_tensor_map_2d_f32(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
                            int box_inner, int box_outer);

// Causal attention with grouped KV heads. q, k, v: column ranges of one bf16
// row per token (pitch ldqkv); o, dout: [T, H*hd] bf16 (pitch ldo); lse, dvec:
// fp32 [b, H, s]; dq_acc: fp32 [T, ldqa] accumulator (zeroed by the call);
// dq, dk, dv: bf16 outputs with pitches lddq / lddkv.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  int64_t ldqkv;
  void* o;
  int64_t ldo;
  float* lse;
  const void* dout;
  float* dvec;
  float* dq_acc;
  int64_t ldqa;
  void* dq;
  int64_t lddq;
  void* dk;
  void* dv;
  int64_t lddkv;
  int b, s, H, Hkv, hd;
  float scale;
  // When set, the backward returns gradients with respect to q and k before
  // RoPE (the transposed rotation is applied to dQ and dK on output).
  const float* rope_cos;
  const float* rope_sin;
};
int attention_fwd(const AttnArgs& a, cudaStream_t st);
int attention_bwd(const AttnArgs& a, cudaStream_t st);
// Forward on the tcgen05 tensor cores (same outputs as attention_fwd).
int attention_fwd_tc(const AttnArgs& a, cudaStream_t st, int* dev_err);
// Backward on the tcgen05 tensor cores for head_dim 64 or 128 (same outputs
// as attention_bwd); _main is the key-major tensor-core kernel alone.
int attention_bwd_tc(const AttnArgs& a, cudaStream_t st, int* dev_err);
int attention_bwd_tc_main(const AttnArgs& a, cudaStream_t st, int* dev_err, bool skip_dq);
// dQ of the tensor-core backward (head dim 64 or 128) by the query-major
// kernel (no reductions).
int attention_bwd_dq_tc(const AttnArgs& a, cudaStream_t st, int* dev_err);
// Backward form in later calls (0 automatic, 1 fused: dQ by reductions
// inside the key-major kernel, head dim 128 only, 2 split: dK/dV by the
// key-major kernel, dQ by the query-major one, deterministic; head dim 64 is
// always split); returns the previous one.
int attention_bwd_variant(int v);
// Kernels one tensor-core backward of head dim hd launches in the current form.
int attention_bwd_kernels(int hd);

// Mixture-of-experts MLP (moe.cu). Router: logits [T, E], the topk experts
// idx [T, k] and their gates [T, k] of the bf16 MLP input w [T, d] and router
// Wr [E, d]. Gather: xe[slot] = w[row_of[slot]]. Combine: out = h + the
// gated expert outputs ye (fp32 rows by slot). Dy: dye[slot] = gate dy (bf16)
// and dgate = dy . ye. Router backward: dlogits, dWr [E, d] and the MLP
// input's gradient dw [T, d] (router term plus the routed rows' dxe).
int launch_moe_router(const void* w, const void* Wr, int T, int d, int E, int k, float* logits, int32_t* idx,
                      float* gate, cudaStream_t st);
int launch_moe_gather(const void* w, const int32_t* row_of, int rows, int d, void* xe, cudaStream_t st);
int launch_moe_combine(const float* h, const float* ye, const int32_t* slot_of, const float* gate, int T, int k,
                       int d, float* out, cudaStream_t st);
int launch_moe_dy(const float* dy, const float* ye, const int32_t* slot_of, const float* gate, int T, int k, int d,
                  void* dye, float* dgate, cudaStream_t st);
int launch_moe_router_bwd(const float* gate, const float* dgate, const int32_t* idx, const void* w, const void* Wr,
                          const float* dxe, const int32_t* slot_of, int T, int k, int d, int E, float* dlogits,
                          float* dWr, float* dw, cudaStream_t st);

int launch_rmsnorm_fwd(const float* x, const void* g, void* y, float* rstd, int T, int d, float eps, cudaStream_t st);
int rmsnorm_bwd_blocks(int T);
int launch_rmsnorm_bwd(const float* x, const void* g, const float* rstd, const float* dy, const float* dres,
                       float* dx, void* dx_bf16, float* dg_part, float* dg, int T, int d, cudaStream_t st);
int launch_rope(void* buf, int64_t ld, int T, int s, int nheads, int hd, int col0, const float* cosb,
                const float* sinb, float sign, cudaStream_t st);
int launch_swiglu_fwd(const void* gu, void* act, int T, int F, cudaStream_t st);
int launch_swiglu_bwd(const void* gu, const void* dact, void* dgu, int T, int F, cudaStream_t st);
int launch_embed_fwd(const int* tok, const void* E, float* x, int T, int d, cudaStream_t st);
int launch_embed_bwd(const int* offs, const int* pos, int n_unique, const float* dx, float* rows, int d,
                     cudaStream_t st);
int launch_softmax_ce(const float* z, int64_t ldz, const int* labels, void* dz, int64_t lddz, float* row_loss,
                      int Tc, int V, float scale, cudaStream_t st);
int launch_sum_all(const float* v, int n, float* out, int accumulate, cudaStream_t st);
int launch_cast_f32_bf16(const float* in, void* out, int64_t n, cudaStream_t st);

}  // namespace mt
