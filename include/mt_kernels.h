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
 * (MegaTrain abstract; saify.me, "The memory-centric design"), in forward
 * (X W^T), input-gradient (dY W) and weight-gradient (dY^T X) form.
 *   A: a_mn_major = 0: element (m,k) at A[m*lda + k]; = 1: at A[k*lda + m]
 *   B: b_mn_major = 0: element (n,k) at B[n*ldb + k]; = 1: at B[k*ldb + n]
 *   C: element (m,n) at C[m*ldc + n]; R likewise with ldr.
 * lda, ldb, ldc: multiples of 8 elements; ldr: multiple of 4. K may be any
 * positive size (the tail is zero-filled); M, N any size >= 0. */
int mt_k_gemm_bf16(const void* A, int64_t lda, int a_mn_major, const void* B, int64_t ldb, int b_mn_major,
                   void* C, int64_t ldc, int out_kind, const float* R, int64_t ldr, int M, int N, int K,
                   void* stream, int32_t* dev_err);

/* RMSNorm forward, one row per token (reading of the Llama block: eps inside
 * the root): y[t] = x[t] / sqrt(mean_j x[t,j]^2 + eps) * g.
 * x fp32 [T,d]; g bf16 [d]; y bf16 [T,d]; rstd fp32 [T] (may be NULL) receives
 * 1/sqrt(mean x^2 + eps). d multiple of 4. */
int mt_k_rmsnorm_fwd(const float* x, const void* g, void* y, float* rstd, int T, int d, float eps, void* stream);

/* Floats of the per-block partial buffer mt_k_rmsnorm_bwd needs for T rows. */
size_t mt_k_rmsnorm_bwd_partial_floats(int T, int d);

/* RMSNorm backward (hand-written gradient, intelligentliving.co "Checkpointing,
 * Manual Gradients, and CPU-Side Optimizer Steps"):
 *   dx[t,j] = dres[t,j] + r g_j dy[t,j] - x[t,j] r^3 (sum_i g_i dy[t,i] x[t,i]) / d
 *   dg[j]   = sum_t dy[t,j] x[t,j] r_t   (fixed summation order)
 * x, dy, dres (may be NULL), dx: fp32 [T,d]; rstd fp32 [T]; g bf16 [d];
 * dx_bf16 (may be NULL) receives a bf16 copy of dx; dg_part: caller scratch of
 * mt_k_rmsnorm_bwd_partial_floats(T,d) floats; dg fp32 [d]. d <= 8192. */
int mt_k_rmsnorm_bwd(const float* x, const void* g, const float* rstd, const float* dy, const float* dres, float* dx,
                     void* dx_bf16, float* dg_part, float* dg, int T, int d, void* stream);

/* RMSNorm backward that allocates nothing and takes no scratch buffer: the
 * same outputs as mt_k_rmsnorm_bwd (dx, optional dx_bf16, dg) for callers that
 * cannot call cudaMalloc at this point -- for example code whose device memory
 * was all handed to another allocator up front, hot loops that cannot absorb
 * the device-wide synchronisation an allocation may cause, or plugin hosts
 * that forbid allocation after start-up. The method's pages have no
 * counterpart: this is a convenience of this library.
 * The partial sums live in one fixed 4 MiB device array inside the library
 * (1M floats, held on every GPU that loads the library until the process
 * exits); the block count is reduced when needed so that blocks x d partials
 * fit. Limits: d <= 8192 and d % 4 == 0, else MT_ERR_ARG. Every call looks
 * up the array's device address (cudaGetSymbolAddress) on the current device
 * and caches nothing, so a device reset between calls is harmless; the first
 * call on a device also loads the library's module there, so make that first
 * call before any stream capture. Each
 * device has its own copy of the array, and every call on that device shares
 * it, which keeps the last call's contents: two calls whose executions overlap
 * on the GPU (for example on two streams with no ordering between them) race
 * on it and give wrong dg. Calls ordered on one stream are safe. */
int mt_k_rmsnorm_bwd_noalloc(const float* x, const void* g, const float* rstd, const float* dy, const float* dres,
                             float* dx, void* dx_bf16, float* dg, int T, int d, void* stream);

/* RoPE in place on nheads bf16 heads of width hd starting at column col0 of a
 * [T, ld] buffer, token t at position t % s; rotate-half pairs (i, i+hd/2)
 * rotated by angle pos * theta_i (cos/sin tables fp32 [s, hd/2]).
 * sign = +1 forward rotation, -1 its transpose (the backward). */
int mt_k_rope(void* buf, int64_t ld, int T, int s, int nheads, int hd, int col0, const float* cos_tab,
              const float* sin_tab, float sign, void* stream);

/* SwiGLU: gu bf16 [T, 2F] = [gate | up]; act bf16 [T,F] = silu(gate) * up.
 * Backward: dgu = [dact * up * s(1 + gate(1-s)) | dact * gate * s], s = sigmoid(gate).
 * F multiple of 8. */
int mt_k_swiglu_fwd(const void* gu, void* act, int T, int F, void* stream);
int mt_k_swiglu_bwd(const void* gu, const void* dact, void* dgu, int T, int F, void* stream);

/* Embedding gather x[t] = E[tok[t]] (bf16 table -> fp32 rows). E may be a
 * device pointer or a mapped pinned-host pointer. d multiple of 8. */
int mt_k_embed_fwd(const int32_t* tok, const void* E, float* x, int T, int d, void* stream);

/* Embedding gradient rows: rows[u] = sum over i in [offs[u], offs[u+1]) of
 * dx[pos[i]] in that order, for n_unique unique tokens. fp32. */
int mt_k_embed_bwd(const int32_t* offs, const int32_t* pos, int n_unique, const float* dx, float* rows, int d,
                   void* stream);

/* Fused softmax cross-entropy over fp32 logits z [Tc, V] (pitch ldz):
 *   row_loss[t] = logsumexp(z[t]) - z[t, labels[t]]
 *   dz[t]       = (softmax(z[t]) - onehot(labels[t])) * scale   (bf16, pitch lddz)
 * V multiple of 4. */
int mt_k_softmax_ce(const float* z, int64_t ldz, const int32_t* labels, void* dz, int64_t lddz, float* row_loss,
                    int Tc, int V, float scale, void* stream);

/* Causal attention forward, scale 1/sqrt(hd), query head h reads KV head
 * h / (H/Hkv). q, k, v: bf16 column ranges of a per-token row (pitch ldqkv),
 * token t = bi*s + i; o bf16 [b*s, H*hd] (pitch ldo); lse fp32 [b,H,s] natural
 * log-sum-exp of the scaled scores. hd 64 or 128. */
int mt_k_attn_fwd(const void* q, const void* k, const void* v, int64_t ldqkv, void* o, int64_t ldo, float* lse,
                  int b, int s, int H, int Hkv, int hd, void* stream);

/* The same causal attention forward (same arguments, outputs and layout) on the
 * tcgen05 tensor cores: 128-query x 128-key tiles, S and P V in tensor memory,
 * TMA loads. Additionally needs q, k, v and o 16-byte aligned. dev_err:
 * optional device int32 set when a bounded wait inside the kernel runs out. */
int mt_k_attn_fwd_tc(const void* q, const void* k, const void* v, int64_t ldqkv, void* o, int64_t ldo, float* lse,
                     int b, int s, int H, int Hkv, int hd, void* stream, int32_t* dev_err);

/* Causal attention backward from o, lse and dout (bf16, pitch ldo):
 * dvec fp32 [b,H,s] and dq_acc fp32 [b*s, ldqa] are caller scratch (dq_acc is
 * zeroed by the call); dq (pitch lddq), dk and dv (pitch lddkv) are bf16
 * outputs laid out like q, k, v. dk, dv of a KV head sum over its query heads.
 * When cos_tab/sin_tab (fp32 [s, hd/2], as for mt_k_rope) are given, q and k
 * are taken to be post-RoPE and dq, dk are returned with respect to the
 * pre-RoPE values (the transposed rotation is applied on output); NULL
 * returns gradients with respect to q and k as given. */
int mt_k_attn_bwd(const void* q, const void* k, const void* v, int64_t ldqkv, const void* o, const void* dout,
                  int64_t ldo, const float* lse, float* dvec, float* dq_acc, int64_t ldqa, void* dq, int64_t lddq,
                  void* dk, void* dv, int64_t lddkv, int b, int s, int H, int Hkv, int hd, const float* cos_tab,
                  const float* sin_tab, void* stream);

/* The same backward (same arguments and outputs as mt_k_attn_bwd) on the
 * tcgen05 tensor cores, head_dim 64 or 128 (MT_ERR_CONFIG otherwise): one CTA
 * per 128-key block accumulates dK and dV in tensor memory over the group's
 * query heads and 128-query blocks; dQ goes through the fp32 accumulator,
 * summed there by the query-major kernel (split form; head_dim 64 always) or
 * by reductions (fused form, head_dim 128; mt_k_attn_bwd_variant).
 * q, k, v, o, dout, dq_acc 16-byte aligned, ldqa a multiple of 4; dev_err as
 * for mt_k_attn_fwd_tc. */
int mt_k_attn_bwd_tc(const void* q, const void* k, const void* v, int64_t ldqkv, const void* o, const void* dout,
                     int64_t ldo, const float* lse, float* dvec, float* dq_acc, int64_t ldqa, void* dq, int64_t lddq,
                     void* dk, void* dv, int64_t lddkv, int b, int s, int H, int Hkv, int hd, const float* cos_tab,
                     const float* sin_tab, void* stream, int32_t* dev_err);

/* Forward projection with RoPE fused into the epilogue: C bf16 [M,N] =
 * rope(A[M,K] B[N,K]^T), both operands K-major as in mt_k_gemm_bf16. Columns
 * [0, rope_cols) are heads of width hd (64 or 128) whose rotate-half pairs are
 * rotated in fp32 by the angle of position (row % s) from the fp32 tables
 * cos_tab/sin_tab [s, hd/2] before the single rounding to bf16; columns from
 * rope_cols on are stored unrotated. N must be a multiple of hd. */
int mt_k_gemm_bf16_rope(const void* A, int64_t lda, const void* B, int64_t ldb, void* C, int64_t ldc, int M, int N,
                        int K, int rope_cols, int hd, int s, const float* cos_tab, const float* sin_tab, void* stream,
                        int32_t* dev_err);

/* Codes a kernel writes into dev_err when one of its bounded waits runs out
 * (the first code recorded wins). */
#define MT_DEV_TIMEOUT_PRODUCER 1 /* the copy producer waited too long for a free stage */
#define MT_DEV_TIMEOUT_MMA 2      /* the MMA issuer waited too long for operands or an accumulator */
#define MT_DEV_TIMEOUT_EPILOGUE 3 /* the epilogue waited too long for a finished accumulator */
#define MT_DEV_TIMEOUT_TEARDOWN 4 /* a wait for the CTA's own copies or MMAs before exit ran out */

/* Limit, in nanoseconds, of each main-loop wait of the single-CTA GEMM kernel
 * for later launches in this process (mt_k_gemm_bf16, mt_k_gemm_bf16_rope and
 * the engine's GEMMs alike); returns the previous limit. ns < 0 only queries.
 * Default 1e9 (1 s). With 0 a wait gives up at its first poll that finds the
 * stage or accumulator not ready, so a test can make a kernel take its
 * bounded-wait exit without any fault: the kernel records an
 * MT_DEV_TIMEOUT_* code in dev_err, lets its own copies and MMAs finish,
 * frees its tensor memory and returns; outputs are then undefined, and the
 * context stays usable. The waits that let a CTA exit safely keep 1 s, and so
 * does every wait of the CTA-pair kernel (used for problems with at least one
 * 256-row tile per SM pair). Host-side only; not thread-safe against
 * concurrent GEMM launches. */
int64_t mt_k_gemm_wait_limit_ns(int64_t ns);

/* Selects the GEMM kernel family for later calls in this process: 0 automatic
 * (the default, or MT_GEMM_VARIANT=auto), 1 single-CTA tiles only (=single),
 * 2 CTA-pair tiles (tcgen05 cta_group::2, 256-row tiles) wherever a problem
 * has at least one pair tile per SM pair (=pair). Both families compute the
 * same product; this exists for measurement and tests. Returns the previous
 * family, or MT_ERR_ARG for another value (nothing changes). No GPU work. */
int mt_k_gemm_variant(int variant);

/* Selects the tcgen05 attention forward kernel for head dim 128 in later calls
 * (mt_k_attn_fwd_tc and the engine): 0 automatic (the default: two query tiles
 * per CTA for s > 8192, one otherwise), 1 one 128-query tile per CTA, 2 two
 * 128-query tiles per CTA in ping-pong, P kept in tensor memory. Both compute
 * the same attention; this exists for measurement and tests. Returns the
 * previous choice, or MT_ERR_ARG for another value (nothing changes). No GPU
 * work. */
int mt_k_attn_fwd_variant(int variant);

/* Selects the form of the tcgen05 attention backward (mt_k_attn_bwd_tc and the
 * engine) in later calls: 0 automatic (the default: split, deterministic and
 * the faster form at every length measured), 1 fused: one key-major
 * kernel computes dK, dV and dQ, adding each key block's dQ into dq_acc with
 * fp32 reductions (their order, and so dQ's last bits, vary from run to run),
 * 2 split: the key-major kernel computes dK and dV only and a query-major
 * kernel sums dQ over the key blocks in tensor memory and writes each element
 * once (deterministic: the same inputs give the same bits; needs dq_acc
 * 16-byte aligned and ldqa a multiple of 4, MT_ERR_ARG before any GPU work
 * otherwise). Returns
 * the previous choice, or MT_ERR_ARG for another value (nothing changes). No
 * GPU work. */
int mt_k_attn_bwd_variant(int variant);

/* Host AdamW over n fp32 elements, in place (HOST pointers, runs on the
 * calling thread; the engine runs the same routine across its worker pool):
 *   p <- p (1 - lr wd); m <- b1 m + (1-b1) g; v <- b2 v + (1-b2) g^2;
 *   p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * and pb[i] <- bf16(p[i]) rounded to nearest even when pb is not NULL
 * (the streamed copy). g may be NULL for a zero gradient (nothing is read:
 * the embedding rows a batch does not touch). t >= 1 counts steps. The update is Adam (Kingma & Ba,
 * cited by the MegaTrain paper) with decoupled decay, on the CPU as MegaTrain
 * does (intelligentliving.co, "Checkpointing, Manual Gradients, and CPU-Side
 * Optimizer Steps"). */
int mt_k_adamw_host(float* p, const float* g, float* m, float* v, uint16_t* pb, size_t n, float lr, float beta1,
                    float beta2, float eps, float wd, int t);

#ifdef __cplusplus
}
#endif
#endif /* MT_KERNELS_H_ */
