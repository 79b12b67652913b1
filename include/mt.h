/*
 * mt.h -- C interface of the host-memory-streamed layer training library.
 *
 * One training step of a Llama-style decoder whose fp32 master weights and
 * AdamW moments live in pinned host memory. Every layer's bf16 weights are
 * streamed to the GPU, run through forward, checkpointed recompute and
 * backward, and its fp32 gradients are streamed back to the host, where AdamW
 * updates the master weights. The method is MegaTrain's memory-centric
 * training: "MegaTrain: Full Precision Training of 100B+ Parameter Large
 * Language Models on a Single GPU" (arXiv 2604.05091), abstract: parameters
 * and optimizer states stay in host memory, the GPU is a transient compute
 * engine, and per layer parameters stream in and gradients stream out, through
 * a pipelined double-buffered engine on several CUDA streams with stateless
 * layer templates.
 *
 * Conventions for every function below:
 *   - return 0 (MT_OK) on success or a negative MT_ERR_* code; nothing aborts
 *     or exits the process; mt_last_error() gives a message for the context;
 *   - argument, configuration and token-range errors are detected on the host
 *     before any device work and leave all state untouched;
 *   - a context is not thread-safe: one caller thread at a time.
 *
 * Environment read by mt_create:
 *   MT_WAIT_LIMIT_S  limit, in seconds, of every host wait on GPU work and of
 *                    a gradient-ring slot (default 600); past it a call
 *                    returns MT_ERR_TIMEOUT;
 *   MT_LOGITS_CHUNK  tokens per LM-head chunk, a multiple of 128 below the
 *                    default (the default keeps fp32 logits + bf16 dz of a
 *                    chunk under ~4 GiB); smaller chunks use less device
 *                    memory and compute the same result;
 *   MT_DEFER_LAYERS  with MT_FLAG_DEFER_UPDATES, how many of the last layers
 *                    have their update deferred (default 1; clamped to
 *                    [0, L-1]; mt_host_state_bytes reads it too);
 *   MT_OVERLAP_THREADS  with MT_FLAG_DEFER_UPDATES, host threads of the
 *                    updates that overlap the forward sweep (deferred ones and
 *                    the untouched embedding rows; default half the pool), so
 *                    that the weight copies keep their share of host memory
 *                    bandwidth.
 * and by the GEMM launcher: MT_GEMM_VARIANT (see mt_kernels.h).
 */
#ifndef MT_H_
#define MT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MT_OK 0
#define MT_ERR_ARG (-1)        /* bad pointer, size or value */
#define MT_ERR_CONFIG (-2)     /* configuration outside what the kernels support */
#define MT_ERR_ARENA (-3)      /* host arena too small or misaligned */
#define MT_ERR_NOMEM (-4)      /* device or host allocation failed, or budget exceeded */
#define MT_ERR_PIN (-5)        /* pinning the host arena failed */
#define MT_ERR_CUDA (-6)       /* a CUDA runtime call failed */
#define MT_ERR_TIMEOUT (-7)    /* a bounded wait (host or device) ran out */
#define MT_ERR_NONFINITE (-8)  /* a gradient was NaN or Inf: remaining updates skipped */
#define MT_ERR_DEVICE (-9)     /* a kernel reported an error through its error word */

/* Flags (mt_config.flags). */
#define MT_FLAG_SERIALIZE 0x1u     /* run copies and kernels on one stream (debug) */
#define MT_FLAG_KERNEL_TIMING 0x2u /* time GEMM / attention launches with events */
#define MT_FLAG_NO_UPDATE 0x4u     /* compute loss and gradients only, skip AdamW */
/* Gradients stream through a ring of MT_GRAD_RING_SLOTS layer-sized pinned
 * host slots (plus one buffer for the final norm and LM head) instead of a
 * full fp32 gradient arena: host memory drops from 18 to about 14 bytes per
 * parameter, and the gradient of every layer is consumed by its AdamW update
 * as it lands. When the optimizer falls that many layers behind the backward,
 * the next gradient offload waits for a slot (bounded by the context's wait
 * limit). mt_get_grads is not available in this mode. */
#define MT_FLAG_GRAD_RING 0x8u
#define MT_GRAD_RING_SLOTS 3
/* Overlap part of each step's host update with the next step's forward sweep,
 * when the host optimizer is otherwise idle. The updates of the final norm and
 * LM head and of the last MT_DEFER_LAYERS decoder layers (environment variable,
 * default 1, at most L-1) are checked for non-finite gradients in their own
 * step as usual; their AdamW update is then run at the start of the next
 * mt_train_step, which waits (bounded by the wait limit) for it before
 * streaming those weights again. Every update still uses its own step's
 * gradient and bias correction and completes before its weights are next
 * read, so the trajectory is that of the undeferred step. Until a pending
 * update has run, the caller's arena holds those tensors' previous values:
 * mt_flush applies pending updates, and so does every call that reads or
 * writes the training state (mt_get_params, mt_get_opt_state, mt_set_state,
 * mt_layer_fwd_bwd, mt_head_fwd_bwd, mt_destroy). With MT_FLAG_GRAD_RING the
 * deferred layers keep their gradients in MT_DEFER_LAYERS extra pinned
 * layer-sized buffers. Ignored with MT_FLAG_NO_UPDATE. */
#define MT_FLAG_DEFER_UPDATES 0x10u
/* Offload gradients in bf16 instead of fp32: after its finite check on the
 * GPU, each layer's (and the LM head's) fp32 gradient is rounded to bf16
 * (nearest even) and only the bf16 copy crosses the link and sits in host
 * memory; the host AdamW widens it exactly and keeps the fp32 master and
 * moments. It halves the gradient bytes over the link (4 -> 2 per parameter)
 * and in host memory, and cuts the optimizer's host DRAM traffic from 30 to
 * 28 bytes per parameter, at the cost of one more rounding of every gradient
 * (relative error <= 2^-9 per element). The embedding-gradient rows cross
 * the link in fp32 and are rounded the same way on the host. mt_get_grads
 * returns the bf16 values widened to fp32, exactly what the update used. A measured
 * link-versus-accuracy variant: the method's own design offloads the
 * gradients in full precision (MegaTrain abstract: full-precision training). */
#define MT_FLAG_BF16_GRADS 0x20u
/* Keep the layer-boundary activations in pinned host memory instead of HBM:
 * during the forward, x_0 .. x_{L-3} (fp32 [b*s, d] each) are copied to host
 * memory on a stream of their own as soon as they are produced, x_{L-2} moves
 * to a third device slot, and in the backward each x_l returns to the device
 * while layer l+1 computes. The device then holds three boundary slots
 * instead of L+1 (mt_device_bytes), which is what lets the context grow
 * (MegaTrain abstract: 7B at 512k tokens on one GH200; saify.me, "Who this is
 * actually for": ultra-long context as a side effect of the layer-wise
 * design), at the cost of 2 (L-2) b s d 4 bytes more over the host link per
 * step and (L-2) b s d 4 bytes of pinned host memory (mt_host_state_bytes).
 * The arithmetic is unchanged: every copy is exact. */
#define MT_FLAG_OFFLOAD_ACTS 0x40u
/* Tied embeddings: the LM head is the embedding table (z = n E^T), one of the
 * decoder variants the pages list as supported (saify.me, "Who this is
 * actually for": "The repo supports many architectures"). The arena has no
 * LM-head tensor (mt_arena_bytes shrinks by V*d floats; mt_tensor_offset
 * refuses MT_T_LM_HEAD); the head streams the bf16 table each step, and the
 * table's gradient is the head's dense V x d gradient plus the gathered rows'.
 * It is updated with one dense AdamW in the step's last host job, after every
 * gradient of the step has been checked. Not with MT_FLAG_BF16_GRADS. */
#define MT_FLAG_TIED_EMBED 0x80u
/* Keep each layer's attention output O (bf16 [b*s, H*hd]) and log-sum-exp
 * (fp32 [b, H, s]) on the device from the forward sweep to the layer's
 * backward, so that the layer's recompute skips the attention forward. The
 * pages' checkpointing keeps some intermediates and recomputes the rest
 * (intelligentliving.co, "Checkpointing, Manual Gradients, and CPU-Side
 * Optimizer Steps"); which ones is a memory-for-time choice, and at long
 * context, where attention dominates the layer, this one saves one of the
 * layer's two attention forwards (about a fifth of its attention work, the
 * backward counting 2.5 forwards). Costs (L-1) (b s H hd 2 + b H s 4) bytes of HBM
 * (mt_device_bytes). The results are unchanged: the attention forward is
 * deterministic, so the kept O and LSE are those a recompute would give. */
#define MT_FLAG_STASH_ATTN 0x100u
/* Debug: fill every device weight slot with NaN (bf16 0xFFFF) as soon as the
 * compute stream releases it and every gradient slot (fp32 0xFFFFFFFF) just
 * before a layer's backward writes it, so that a read of a slot before its
 * reload or write completes (a missing wait) turns the step's results into
 * NaN instead of silently using stale data. Results are otherwise unchanged;
 * costs one memset per load and per backward layer. (Race detection without
 * a sanitizer, which this environment does not offer.) */
#define MT_FLAG_POISON 0x200u

/* Tensor ids inside a decoder layer and for model-level tensors (layer = -1). */
#define MT_T_ATTN_NORM 0
#define MT_T_WQ 1
#define MT_T_WK 2
#define MT_T_WV 3
#define MT_T_WO 4
#define MT_T_MLP_NORM 5
#define MT_T_WGATE 6
#define MT_T_WUP 7
#define MT_T_WDOWN 8
/* Mixture-of-experts layers (E > 0; saify.me, "Who this is actually for",
 * lists MoE variants among the supported families and gives no routing rule,
 * so the plainest reading is taken): WGATE and WUP hold [E, F, d] (expert e's
 * rows at e * F * d), WDOWN [E, d, F], and MT_T_ROUTER the router [E, d].
 * Per token t of the MLP input w: logits = w Wr^T; the topk experts with the
 * largest logits (ties to the lower index); gates = softmax of those logits;
 * output = sum over them of gate * SwiGLU_e(w). Every routed token is
 * computed (no capacity limit) and the loss has no auxiliary term. */
#define MT_T_ROUTER 9
#define MT_T_EMBED 100
#define MT_T_FINAL_NORM 101
#define MT_T_LM_HEAD 102

typedef struct mt_config {
  uint32_t struct_size; /* sizeof(mt_config); lets the layout grow */
  int32_t L;            /* decoder layers */
  int32_t d;            /* model width */
  int32_t H;            /* query heads; head_dim = d / H, 64 or 128 */
  int32_t Hkv;          /* key/value heads, divides H */
  int32_t F;            /* SwiGLU hidden width */
  int32_t V;            /* vocabulary */
  int32_t b;            /* sequences per step */
  int32_t s;            /* tokens per sequence */
  float norm_eps;       /* RMSNorm epsilon, inside the square root */
  float rope_base;      /* RoPE base, theta_i = base^(-2i/head_dim) */
  float lr, beta1, beta2, adam_eps, wd; /* AdamW, decoupled decay on all tensors */
  uint64_t seed;        /* initial weights when the library owns the arena */
  uint32_t flags;       /* MT_FLAG_* */
  int32_t device;       /* CUDA device ordinal */
  int32_t host_threads; /* host AdamW threads; 0 = all cores but one */
  int32_t E;            /* experts per mixture-of-experts MLP; 0 = the dense SwiGLU MLP */
  int32_t topk;         /* experts each token is routed to (1 <= topk <= E) when E > 0 */
} mt_config;

typedef struct mt_ctx mt_ctx;

/* Per-step counters, filled by mt_get_stats for the last mt_train_step. */
typedef struct mt_stats {
  double step_ms;           /* compute-stream time of the step (device events) */
  double fwd_ms, head_ms, bwd_ms; /* compute-stream phases */
  double h2d_bytes, d2h_bytes;    /* bytes moved over the host link */
  double h2d_ms, d2h_ms;          /* copy-stream busy time */
  double wait_weights_ms;   /* compute stream idle waiting for prefetched weights */
  double adamw_ms;          /* host optimizer busy time (wall) */
  double adamw_bytes;       /* host DRAM bytes the optimizer touched */
  double gemm_flops, gemm_ms; int64_t gemm_launches;  /* with MT_FLAG_KERNEL_TIMING */
  double attn_flops, attn_ms; int64_t attn_launches;
  int64_t kernel_launches;  /* kernels this library launched during the step */
  double host_step_ms;      /* wall time of mt_train_step */
  double adamw_first_ms;    /* host optimizer's first update began, ms after the call started */
  double adamw_last_ms;     /* host optimizer's last update ended, ms after the call started */
  double enqueue_ms;        /* host time spent enqueueing the step's GPU work */
} mt_stats;

/* Fills *cfg with the defaults (struct_size set, hyper-parameters of the
 * workloads: eps 1e-5, RoPE base 10000, lr 1e-3, betas (0.9, 0.95), eps 1e-8,
 * wd 0.1). Shapes are left zero. The pages fix none of these values: AdamW is
 * the optimizer of the paper's references (mlsanity.com index, "Builds on":
 * Adam), the rest are the usual Llama-style settings. */
int mt_config_default(mt_config* cfg);

/* Bytes of the fp32 master arena for cfg, the parameters that live in host
 * memory (MegaTrain abstract: parameters and optimizer states are stored in
 * host memory; intelligentliving.co, "Implementing Host Memory Offloading
 * for Persistent Model State"): the embedding [V,d]; per layer the
 * attention-norm gain [d], Wq [H*hd,d], Wk [Hkv*hd,d], Wv [Hkv*hd,d],
 * Wo [d,H*hd], MLP-norm gain [d], Wgate [F,d], Wup [F,d], Wdown [d,F]; then the
 * final-norm gain [d] and the untied LM head [V,d]. Weights are row-major
 * [out, in]; every tensor starts on a 256-byte boundary. 0 for a bad cfg. */
size_t mt_arena_bytes(const mt_config* cfg);

/* Offset (in floats) and element count of one tensor of the arena (the
 * layout of mt_arena_bytes; tensor_id MT_T_*, layer -1 for the embedding,
 * final norm and LM head). MT_ERR_ARG for an unknown tensor or layer. */
int mt_tensor_offset(const mt_config* cfg, int layer, int tensor_id, size_t* offset_floats, size_t* numel);

/* Host bytes the context holds besides the caller's arena (the pages budget
 * ~12 GB of host memory per 1B parameters for the full-precision state:
 * saify.me, "Who this is actually for"; intelligentliving.co, FAQ, minimum
 * RAM): two fp32 Adam moments (8 B/param, with the caller's 4 B/param master
 * the 12), the bf16 streaming copy (2 B/param) and the staging of
 * the embedding-gradient rows, plus the fp32 gradients: the whole gradient
 * arena (4 B/param), or with MT_FLAG_GRAD_RING in cfg->flags the ring of
 * MT_GRAD_RING_SLOTS layer slots and the final-norm + LM-head gradient (and,
 * with MT_FLAG_DEFER_UPDATES too, MT_DEFER_LAYERS more layer slots); with
 * MT_FLAG_BF16_GRADS the gradient buffers are bf16 (2 B per element); with
 * MT_FLAG_OFFLOAD_ACTS also the (L-2) offloaded fp32 [b*s, d] boundary
 * activations. */
size_t mt_host_state_bytes(const mt_config* cfg);

/* Device bytes mt_create allocates for cfg, in one allocation, 0 for a bad
 * cfg: two bf16 layer-weight slots and two fp32 layer-gradient slots (the
 * double-buffered layer pair of saify.me, "The memory-centric design":
 * persistent GPU state stays at about one layer's footprint), the LM head's
 * weights and gradients, the boundary activations x_0..x_L (fp32 [b*s, d]
 * each, the only per-layer state kept: intelligentliving.co, "Checkpointing,
 * Manual Gradients, and CPU-Side Optimizer Steps") and one layer's workspace.
 * Only the boundary activations grow with L (three slots with
 * MT_FLAG_OFFLOAD_ACTS), and with MT_FLAG_STASH_ATTN each layer's attention
 * output and log-sum-exp. No GPU needed. */
size_t mt_device_bytes(const mt_config* cfg);

/* Partition of the training state over `world` GPUs of one host that each
 * train their own micro-batch through the same streamed layers (data-parallel
 * sharded streaming: each GPU loads 1/world of every layer over its host link
 * and all-gathers the rest from its peers, reduce-scatters the fp32 gradients
 * and offloads only its own part, whose host AdamW it runs; the collectives
 * are the all-gather and reduce-scatter that the pages contrast with
 * MegaTrain's single-GPU streaming: intelligentliving.co, "Balancing Reduced
 * Collective Communication with Weight Streaming Latency").
 * A layer block (the floats of one decoder layer, from its attention-norm gain
 * to the end of Wdown) holds every tensor at the same element offset in the
 * fp32 arena and in the bf16 streamed block, so one element range is a rank's
 * share of the weights it loads, of the summed gradients it receives and of
 * the parameters it updates. Ranks own consecutive chunks of
 * layer_chunk = ceil(layer_elems / (world * 128)) * 128 elements (256-byte
 * aligned in bf16; the device slots are padded to world * layer_chunk, the
 * last ranges clipped, possibly empty); the [final-norm gain | LM head] block
 * is split the same way, and the embedding by rows. Requires d % 128 == 0
 * (MT_ERR_CONFIG otherwise); MT_ERR_ARG for world < 1 or rank outside
 * [0, world). Host-side arithmetic only. */
typedef struct mt_shard {
  int32_t world, rank;
  uint64_t layer_elems, layer_chunk, layer_begin, layer_end; /* elements of a layer block; this rank's [begin, end) */
  uint64_t head_elems, head_chunk, head_begin, head_end;     /* elements of the [final gain | head] block */
  int32_t embed_row_begin, embed_row_end;                    /* embedding rows this rank updates */
} mt_shard;
int mt_shard_plan(const mt_config* cfg, int world, int rank, mt_shard* out);

/* Creates a context on cfg->device: the host-resident state and the small,
 * fixed device footprint of MegaTrain's memory-centric design (MegaTrain
 * abstract: GPUs are transient compute engines; saify.me, "The memory-centric
 * design"). host_param_arena: the caller's fp32
 * master weights in the layout of mt_arena_bytes, at least arena_bytes long and
 * 256-byte aligned; the library updates it in place every step and keeps the
 * pointer for the context's lifetime. Only host threads touch it (the GPU reads
 * the bf16 copies), so it need not be pinned. NULL: the library allocates the
 * arena and fills it from cfg->seed (gains 1, matrices N(0, 0.02^2)). The
 * library owns the moments, the gradient buffers, the bf16 copy (pinned) and
 * all device memory. Fails with MT_ERR_NOMEM before allocating if the device
 * budget does not fit. */
int mt_create(const mt_config* cfg, float* host_param_arena, size_t arena_bytes, mt_ctx** out);

/* Bytes of the NCCL unique id that mt_create_sharded takes. */
#define MT_SHARD_ID_BYTES 128
/* Writes a fresh NCCL unique id (MT_SHARD_ID_BYTES bytes) to id_out. One rank
 * calls it and hands the same bytes to every rank (a torch.distributed
 * broadcast, for instance). NCCL is loaded at run time (libnccl.so.2, 2.18 or
 * later); MT_ERR_CUDA if it cannot be loaded or fails, MT_ERR_ARG for NULL. */
int mt_shard_id(void* id_out);

/* mt_create for rank `rank` of `world` GPUs of one host that train
 * data-parallel with sharded streaming (mt_shard_plan; intelligentliving.co,
 * "Balancing Reduced Collective Communication with Weight Streaming
 * Latency", names the all-gather and reduce-scatter used here). Every rank
 * calls it with the same cfg, the same initial arena contents (or NULL and the
 * same cfg->seed) and the id of mt_shard_id; the call returns once all ranks
 * have joined (NCCL's initialisation is collective). Per step, each rank
 *   - copies its own part of every bf16 layer block, of the [final gain | LM
 *     head] block and its own embedding rows over its host link, and
 *     all-gathers the rest from the peers over NVLink into its device slots;
 *   - runs forward and backward on its own tokens (mt_train_step's tokens
 *     and labels are the rank's micro-batch);
 *   - averages every gradient block over the ranks with a reduce-scatter
 *     that leaves it its own part (the embedding gradient as a dense
 *     [V, d] block split by rows), checks that part for NaN/Inf with the
 *     verdict shared by all ranks, offloads only that part and runs the host
 *     AdamW on the matching elements of its arena.
 * So per rank the host link carries 1/world of the weights and gradients and
 * the host optimizer 1/world of the update. The returned loss is the mean over
 * all ranks' tokens. The arena, the moments, mt_get_params / mt_get_grads /
 * mt_get_opt_state hold current values on the rank's own ranges only.
 * Collectives of the H2D stream and of the compute stream use two
 * communicators, so each runs in one program order on every rank.
 * Requires d % 128 == 0; mt_layer_fwd_bwd / mt_head_fwd_bwd refuse a
 * sharded context. Expert layers, deferred updates, bf16 gradients and tied
 * embeddings work as in an unsharded context (each rank routes its own
 * tokens; a tied head reads the device table and its dense gradient joins
 * the rows' before the ranks' mean). world = 1 runs the same path
 * with one rank (the collectives are copies). */
int mt_create_sharded(const mt_config* cfg, float* host_param_arena, size_t arena_bytes, int world, int rank,
                      const void* id, mt_ctx** out);

/* mt_device_bytes of a rank of a sharded context: slots padded to world
 * chunks, plus the device embedding table (bf16) and its dense fp32
 * gradient, [world * ceil(V / world), d] each. 0 for a bad cfg or world. */
size_t mt_device_bytes_sharded(const mt_config* cfg, int world);

/* The experts each token chose in layer `layer`'s forward of the last step
 * (mixture-of-experts layers, MT_T_ROUTER): idx[t * topk + j], t in [0, b*s)
 * sequence-major, j in [0, topk) largest logit first. n counts int32
 * elements (at least b*s*topk). The routing a forward took is the one its
 * backward used, so a test can hand it to an independent model where two
 * logits lie within rounding of each other. MT_ERR_CONFIG without experts,
 * MT_ERR_ARG for a bad layer, NULL or short buffer. Host-side. */
int mt_get_routing(mt_ctx* ctx, int layer, int32_t* idx, size_t n);

/* One training step: tokens and labels are host int32 arrays of b*s ids in
 * [0, V), sequence-major. Runs forward, loss, backward and the host AdamW
 * update (bias correction from step 1), and writes the mean next-token
 * cross-entropy (computed before the update) to *loss_out. Each tensor's
 * gradients are checked on the GPU before its host update (intelligentliving.co,
 * "Checkpointing, Manual Gradients, and CPU-Side Optimizer Steps": updates run
 * on the CPU as the gradients arrive). Returns MT_ERR_NONFINITE if a gradient
 * was not finite, and MT_ERR_DEVICE if a kernel of the step reported a bounded
 * wait that ran out (its outputs are then undefined): in both cases the
 * updates of the tensors not yet updated are skipped and the arena is partly
 * updated; the embedding rows no token of the step touched are updated only
 * after every check of the step has passed. The next step starts afresh (the
 * device error word is cleared at its start). With MT_FLAG_DEFER_UPDATES some
 * of this step's updates are still pending when it returns (see the flag).
 * Every reduction of a step on one GPU runs in a fixed order (the attention
 * backward in its automatic, split form; mt_k_attn_bwd_variant), so the same
 * arena, tokens and labels give the same loss, gradients and parameters bit
 * for bit, pipelined or with MT_FLAG_SERIALIZE (a sharded context adds the
 * NCCL collectives' own summation order). */
int mt_train_step(mt_ctx* ctx, const int32_t* tokens, const int32_t* labels, float* loss_out);

/* Runs the updates that MT_FLAG_DEFER_UPDATES left pending, and returns when
 * the arena, the moments and the bf16 copies hold the state after the last
 * step. A no-op without pending updates. (The host optimizer step of
 * intelligentliving.co, "Checkpointing, Manual Gradients, and CPU-Side
 * Optimizer Steps", moved in time, not changed.) */
int mt_flush(mt_ctx* ctx);

/* Copies the fp32 gradients of the last step (taken before the update), in the
 * arena layout, to dst (bytes >= mt_arena_bytes): the gradients each layer
 * pushed back to host memory (MegaTrain abstract: per layer, gradients stream
 * out; intelligentliving.co, "Quantifying Host Memory Requirements...": the
 * stream immediately pushes gradients back to the host). MT_ERR_CONFIG for a
 * context created with MT_FLAG_GRAD_RING, which keeps no gradient arena. */
int mt_get_grads(mt_ctx* ctx, float* dst, size_t bytes);

/* One decoder layer through the engine's own stateless layer template, with
 * no optimizer step: the layer's current bf16 streamed weights, the forward
 * from x_in = x_l, the backward from dx_out = dL/dx_{l+1}, on the context's
 * compute stream and workspace (the same kernels and launches as in
 * mt_train_step). MegaTrain's per-layer unit of work (MegaTrain abstract:
 * parameters stream in, gradients stream out; intelligentliving.co,
 * "Leveraging Double-Buffered Pipelining and Stateless Layer Templates").
 * x_in, dx_out: HOST fp32 [b*s, d]; writes x_out = x_{l+1} and dx_in = dL/dx_l
 * (HOST fp32 [b*s, d]) and the layer's fp32 gradients into grads, laid out as
 * the layer's block of the arena: grads[i] is the gradient of arena element
 * (offset of the layer's attention-norm gain) + i, for the floats between it
 * and the next layer's attention-norm gain (grads_bytes at least that many
 * times 4). Synchronous; the master arena and the moments are unchanged.
 * MT_ERR_DEVICE if a kernel's bounded wait expired. */
int mt_layer_fwd_bwd(mt_ctx* ctx, int layer, const float* x_in, const float* dx_out, float* x_out, float* dx_in,
                     float* grads, size_t grads_bytes);

/* The head of the step on its own, with no optimizer step: final RMSNorm,
 * LM-head logits, cross-entropy against labels (mean over the b*s tokens)
 * and its backward, through the same kernels, token chunks and launches as
 * mt_train_step, with the current bf16 streamed final gain and head.
 * x_L: HOST fp32 [b*s, d] (the last layer's output); labels: HOST int32
 * [b*s] in [0, V) (MT_ERR_ARG otherwise, checked first). Writes the loss,
 * dx_L = dL/dx_L (HOST fp32 [b*s, d]) and the gradients of the final gain and
 * the LM head into grads, laid out as the arena from the final gain's offset
 * on (grads_bytes at least 4 * (LM head offset + V*d - final gain offset)).
 * Synchronous; the master arena and the moments are unchanged. */
int mt_head_fwd_bwd(mt_ctx* ctx, const float* x_L, const int32_t* labels, float* loss_out, float* dx_L,
                    float* grads, size_t grads_bytes);

/* Copies the current fp32 master weights (after the last update) to dst
 * (bytes >= mt_arena_bytes), applying pending deferred updates first. The
 * master lives in host memory and is the state the host AdamW updates
 * (intelligentliving.co, "Checkpointing, Manual Gradients, and CPU-Side
 * Optimizer Steps": FP32 master weights and optimizer moments live in RAM). */
int mt_get_params(mt_ctx* ctx, float* dst, size_t bytes);

/* Checkpoint: copies the fp32 Adam moments m and v (arena layout, each at
 * least mt_arena_bytes long) and the number of completed steps. The master
 * weights come from mt_get_params. The host arena is the whole training state
 * (MegaTrain keeps parameters and optimizer state in host memory). */
int mt_get_opt_state(mt_ctx* ctx, float* m_dst, float* v_dst, size_t bytes_each, int64_t* step);

/* Resume: replaces the master weights, both moments and the step counter
 * (bias correction continues from step + 1) and rebuilds the bf16 streaming
 * copies. Any pointer may be NULL to keep that part. Nothing runs on the GPU. */
int mt_set_state(mt_ctx* ctx, const float* params, const float* m, const float* v, size_t bytes_each,
                 int64_t step);

/* Fault injection for tests of the host-side waits: enqueues on the
 * context's stream `stream` (0 weight prefetch, 1 compute, 2 gradient
 * offload) a host function that sleeps `ms` milliseconds (0..60000), so that
 * the work queued after it starts late. The GPU itself is untouched: nothing
 * faults, traps or spins on it. With MT_WAIT_LIMIT_S below the stall, the
 * next mt_train_step returns MT_ERR_TIMEOUT with its remaining updates
 * skipped, and the context can still be used or destroyed (mt_destroy waits
 * for the stall to end). The pages give no failure model beyond fewer
 * crashes and out-of-memory errors (intelligentliving.co, "Leveraging
 * Double-Buffered Pipelining and Stateless Layer Templates"). */
int mt_inject_host_stall(mt_ctx* ctx, int stream, int ms);

/* Counters of the last step: the copy/compute overlap and optimizer-latency
 * figures that the pages ask a profile of this method to report
 * (intelligentliving.co, "Limitations of Current Throughput Metrics...":
 * CPU-to-GPU transfer overlap and optimizer update latencies). */
int mt_get_stats(mt_ctx* ctx, mt_stats* out);

/* Timeline of the last step, for seeing the copy/compute overlap of the
 * pipeline (a profiler-free trace). Writes *n_floats; with out == NULL only
 * the size. Layout (floats):
 *   [0] n_loads (2L-1 weight loads), [1] L, [2] n_jobs;
 *   per weight load i: layer, H2D start, weights ready, compute stream
 *     reaches its wait for them, compute stream releases the slot;
 *   per backward layer (order L-1 .. 0): layer, gradients ready on the
 *     compute stream, D2H start, D2H done;
 *   forward end, head end, backward end, step end;
 *   per host optimizer job (execution order): kind (0 layer, 1 LM head,
 *     2 touched embedding rows, 3 untouched embedding rows, 4 LM head and
 *     5 layer deferred from the previous step by MT_FLAG_DEFER_UPDATES,
 *     6 the previous step's untouched embedding rows deferred by the flag,
 *     7 those of them this step's batch gathers, updated before the step's
 *     GPU work is enqueued; with the flag, kinds 0 and 1 of the deferred
 *     tensors only check their gradients), layer (-1 for the others),
 *     gradients available, update finished.
 * Device times are ms from the step's start on the compute stream (CUDA
 * events); host job times are ms of host clock from the mt_train_step call,
 * a separate clock whose origin is within a few tens of microseconds of it. */
int mt_get_timeline(mt_ctx* ctx, float* out, size_t cap_floats, size_t* n_floats);

/* The context's compute stream (one of the several CUDA streams of the
 * pipelined engine, saify.me "Pipelined double buffering") as a cudaStream_t
 * in *stream, so a caller can
 * order or time its own work against the step (for example record CUDA events
 * around a sequence of mt_train_step calls). The stream stays owned by the
 * context. */
int mt_get_stream(mt_ctx* ctx, void** stream);

/* Host-memory ceiling of the optimizer (intelligentliving.co, "Checkpointing,
 * Manual Gradients, and CPU-Side Optimizer Steps": CPU-side updates can
 * become the slow step): runs the library's host AdamW (the
 * same routine, worker pool and chunking the engine uses) over four fp32
 * arrays of n elements with `threads` threads (0 = all cores but one), best
 * of 3 passes, and returns GB/s counted as 30 bytes per element (read p, g,
 * m, v; write p, m, v and the bf16 copy). Allocates and frees its own host
 * buffers, on transparent huge pages where the host allows them, as the
 * engine allocates its host state; no GPU needed. Returns a negative
 * MT_ERR_* on failure. */
double mt_host_optimizer_gbs(size_t n, int threads);

/* Host DRAM ceiling independent of the optimizer: the STREAM triad
 * a[i] = b[i] + s c[i] over three fp32 arrays of n elements with `threads`
 * threads (0 = all cores but one), parallel first touch, non-temporal stores,
 * best of 5 passes, in GB/s counted as 12 bytes per element (two reads, one
 * write). The host AdamW's 30 bytes per parameter are judged against it
 * (intelligentliving.co, "Checkpointing, Manual Gradients, and CPU-Side
 * Optimizer Steps": CPU-side updates can become the slow step). Allocates
 * and frees its own host buffers (huge pages where the host allows, like the
 * engine's host state); no GPU needed. Negative MT_ERR_* on failure. */
double mt_host_triad_gbs(size_t n, int threads);

/* Applies pending deferred updates, waits for the context's streams, frees
 * its device memory and unpins or frees its host memory. NULL is ignored.
 * The caller's arena then holds the final master weights (MegaTrain abstract:
 * the host holds the parameters; the GPU kept only transient state). */
void mt_destroy(mt_ctx* ctx);

/* Message of the last error of ctx (or of the last failed mt_create when ctx
 * is NULL). Valid until the next call on the same context. The pages describe
 * no error interface; this is the library's own (every call reports instead
 * of aborting, so that out-of-memory and stalls surface as codes:
 * intelligentliving.co, "Leveraging Double-Buffered Pipelining and Stateless
 * Layer Templates", on avoiding unpredictable OOM errors). */
const char* mt_last_error(const mt_ctx* ctx);

#ifdef __cplusplus
}
#endif
#endif /* MT_H_ */
