// Pipelined, double-buffered streaming engine for one training step, and the
// C ABI of include/mt.h.
//
// MegaTrain's memory-centric training (MegaTrain abstract; saify.me "The
// memory-centric design", "Pipelined double buffering", "Stateless layer
// templates"): parameters and optimizer state live in host memory; for each
// layer the engine prefetches the layer's bf16 weights into one of two device
// slots, runs the layer's kernels bound to that slot, pushes its fp32 gradients
// back to host memory and lets the host update the layer with AdamW, so that
// persistent device state is two weight slots, two gradient slots, the
// layer-boundary activations and one layer's workspace.
//
// Streams: H2D prefetch, compute, D2H offload, ordered by per-load and
// per-layer events. The weight loads follow the layer order of the step,
// 0 .. L-1 (forward, keeping only boundary activations) then L-2 .. 0
// (backward, recomputing each layer's forward from its kept input); layer L-1
// stays resident across the turn. Load i+2 reuses the slot of load i and waits
// for the compute stream to release it, so layer n+1 arrives while layer n
// computes. A host optimizer thread waits on each layer's offload event and
// updates that layer's master weights, moments and bf16 copy while the GPU
// continues with the layers below.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <sys/mman.h>

#include <algorithm>
#include <iterator>
#include <atomic>
#include <cmath>
#include <chrono>
#include <condition_variable>
#include <deque>
#include <functional>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "host_adamw.h"
#include "layout.h"
#include "mt_internal.h"
#include "nccl_dl.h"

namespace mt {

namespace {

thread_local std::string g_create_error;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

double now_s() {
  return std::chrono::duration<double>(std::chrono::steady_clock::now().time_since_epoch()).count();
}

// Counter-based normal generator for library-owned arenas: splitmix64 of
// (seed, tensor key, index) -> two uniforms -> Box-Muller.
inline uint64_t splitmix64(uint64_t x) {
  x += 0x9e3779b97f4a7c15ull;
  x = (x ^ (x >> 30)) * 0xbf58476d1ce4e5b9ull;
  x = (x ^ (x >> 27)) * 0x94d049bb133111ebull;
  return x ^ (x >> 31);
}
inline float normal_at(uint64_t key, uint64_t i) {
  const uint64_t a = splitmix64(key ^ splitmix64(2 * i));
  const uint64_t b = splitmix64(key ^ splitmix64(2 * i + 1));
  const double u1 = ((a >> 11) + 1.0) * (1.0 / 9007199254740993.0);  // (0, 1]
  const double u2 = (b >> 11) * (1.0 / 9007199254740992.0);
  return (float)(sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2));
}

struct Job {
  // HEAD_PREV / LAYER_PREV: an update deferred from the previous step
  // (MT_FLAG_DEFER_UPDATES), its gradients already checked. EMBED_UNTOUCHED:
  // the zero-gradient update of the embedding rows no token of the step
  // touched, run once every gradient of the step has passed its checks;
  // EMBED_UNTOUCHED_PREV: the same update deferred into the next step.
  enum Kind { LAYER, HEAD, EMBED, EMBED_UNTOUCHED, HEAD_PREV, LAYER_PREV, EMBED_UNTOUCHED_PREV } kind;
  int layer;
  cudaEvent_t ready;         // offload of this job's gradients has completed
  int flag_index;            // index in the finite-flag array
  const uint8_t* g = nullptr;  // LAYER: host gradient of the layer's first element (gsz bytes each)
  bool defer = false;        // HEAD / LAYER: check now, update at the next step
  int step = 0;              // *_PREV: the AdamW step (bias correction) of the update
};

}  // namespace
}  // namespace mt

using namespace mt;

struct mt_ctx {
  mt_config cfg{};
  Layout lay;
  std::string err;
  int device = 0;
  int step = 0;

  // ---- host memory ----
  float* arena = nullptr;  // fp32 master
  bool arena_owned = false;
  float* m = nullptr;  // Adam moments (pageable, on huge pages where the host allows)
  float* v = nullptr;
  // Host buffers from huge_alloc (pointer, mapped bytes), and those of them
  // that are registered (pinned) for DMA: unregistered and unmapped at destroy.
  std::vector<std::pair<void*, size_t>> huge_bufs;
  std::vector<void*> huge_pinned;
  // Host gradients, gsz bytes per element (4: fp32; 2: bf16 with MT_FLAG_BF16_GRADS).
  int gsz = 4;
  uint8_t* grad = nullptr;        // pinned gradient arena (not with MT_FLAG_GRAD_RING)
  uint8_t* ring = nullptr;        // pinned gradient ring of MT_GRAD_RING_SLOTS layer slots
  uint8_t* grad_head = nullptr;   // [final norm | LM head] gradients: inside grad, or own buffer
  bool grad_head_owned = false;   // own pinned buffer (gradient ring, or tied embeddings)
  size_t layer_f = 0;             // floats of one layer's gradient block
  uint16_t* bf_layers = nullptr;  // pinned bf16 layer blocks
  uint16_t* bf_embed = nullptr;   // pinned bf16 embedding (read by the GPU in place)
  uint16_t* bf_head = nullptr;    // pinned bf16 [final norm | LM head] ([final norm] when tied)
  uint16_t* bf_embed_dev = nullptr;  // device alias of bf_embed
  float* emb_rows_h = nullptr;    // pinned embedding-gradient rows [T, d]
  int32_t* stage_i = nullptr;     // pinned: tokens[T] labels[T] offs[T+1] pos[T]
  int32_t* flags_h = nullptr;     // pinned finite flags [L + 2]
  float* misc_h = nullptr;        // pinned: loss sum, device error word
  std::vector<int32_t> uniq, prev_uniq;
  // MT_FLAG_DEFER_UPDATES: the zero-gradient update of the embedding rows that
  // step `untouched_step` did not touch (its touched rows: untouched_of) is
  // pending; `untouched_skip` lists the rows the queued remainder leaves out.
  bool untouched_pending = false;
  int untouched_step = 0;
  std::vector<int32_t> untouched_of, untouched_skip;
  ThreadPool* pool = nullptr;

  // ---- device memory ----
  void* dmem = nullptr;
  size_t dmem_bytes = 0;
  cudaStream_t s_h2d = nullptr, s_comp = nullptr, s_d2h = nullptr;
  uint16_t* wslot[2] = {nullptr, nullptr};
  float* gslot[2] = {nullptr, nullptr};
  uint16_t* gslot16[2] = {nullptr, nullptr};  // MT_FLAG_BF16_GRADS: bf16 copies offloaded instead
  uint16_t* d_head_g16 = nullptr;
  uint16_t* d_head_w = nullptr;  // [gf | Whead] bf16
  float* d_head_g = nullptr;     // [dgf | dWhead] fp32
  float* xb = nullptr;           // boundary activations [(L+1), T, d], or 3 slots with MT_FLAG_OFFLOAD_ACTS
  // MT_FLAG_OFFLOAD_ACTS: x_0 .. x_{L-3} in pinned host memory, moved on their
  // own stream; per boundary l: offloaded (or copied to slot 2), brought back
  float* xh = nullptr;
  cudaStream_t s_act = nullptr;
  std::vector<cudaEvent_t> ev_xready, ev_xout, ev_xin, ev_bwdone;
  uint16_t *u_b, *qkv_b, *ao_b, *w_b, *gu_b, *act_b, *gxb, *dact_b, *dgu_b, *dhb, *dao_b, *dqkv_b, *n_b, *dz_b;
  float *lse, *h_f, *r1, *r2, *gx0, *gx1, *tmp_f, *dh_f, *dvec, *dqacc, *rms_part, *rf, *logits, *rowloss;
  int32_t *d_tok, *d_lab, *d_offs, *d_pos, *d_flags, *d_err;
  float *d_cos, *d_sin, *d_loss;
  int Tc = 0;  // logits chunk (tokens)

  // ---- events ----
  std::vector<cudaEvent_t> ev_wready, ev_compready, ev_h2d_start, ev_slotfree;  // per weight load
  std::vector<cudaEvent_t> ev_gready, ev_d2h_start, ev_gdrained;               // per backward layer
  cudaEvent_t ev_head_h2d_start, ev_head_wready, ev_head_gready, ev_head_d2h_start, ev_head_drained;
  cudaEvent_t ev_emb_ready, ev_emb_d2h_start, ev_emb_drained;
  cudaEvent_t ev_step_start, ev_fwd_end, ev_head_end, ev_bwd_end, ev_step_end;
  std::vector<cudaEvent_t> ev_timing;  // pool for per-kernel timing pairs
  size_t timing_used = 0;
  struct Timed {
    cudaEvent_t a, b;
    double flops;
    int kind;  // 0 gemm, 1 attention
  };
  std::vector<Timed> timed;

  // ---- optimizer thread ----
  std::thread opt_thread;
  std::mutex opt_mu;
  std::condition_variable opt_cv, opt_done_cv;
  std::deque<Job> jobs;
  int jobs_pending = 0;
  int layer_jobs_done = 0;  // LAYER jobs finished this step: ring slots released
  // MT_FLAG_DEFER_UPDATES: checked updates waiting for the next step, which
  // queued ones have not finished (index l for layer l, L for the LM head),
  // the deferred layer count, the pinned gradient buffers of the deferred
  // layers (ring mode) and the threads of the updates that overlap the
  // forward sweep.
  std::vector<Job> deferred;
  std::vector<char> prev_pending;
  int defer_layers = 0;
  uint8_t* defer_g = nullptr;
  int overlap_threads = 0;
  struct JobTime {
    int kind, layer;
    double ready, done;  // host seconds: gradients landed (wait ended), update finished
  };
  std::vector<JobTime> job_times;  // this step's optimizer jobs, in execution order
  bool opt_stop = false;
  int opt_status = MT_OK;
  bool skip_updates = false;
  double adamw_s = 0, adamw_bytes = 0;
  double call_t0 = 0, adamw_first = 0, adamw_last = 0, enqueue_s = 0;
  double wait_limit_s = 600.0;

  mt_stats stats{};
  int64_t launches = 0;
  std::vector<int> load_seq;  // layer of each weight load

  // ---- sharded streaming (mt_create_sharded) ----
  // Two communicators over the same ranks: the H2D stream's all-gathers and
  // the compute stream's reductions, so that each communicator's collectives
  // run on one stream in one program order on every rank.
  const NcclApi* nccl = nullptr;
  ncclComm_t comm_h2d = nullptr, comm_comp = nullptr;
  mt_shard plan{};              // this rank's element ranges (world 1, everything: unsharded)
  uint16_t* d_embed_w = nullptr;  // bf16 embedding table on the device, [world * rows, d]
  float* d_embed_g = nullptr;     // dense embedding gradient, [world * rows, d]
  int32_t* d_uid = nullptr;       // unique token ids of the step, [T]
  float* emb_own_h = nullptr;     // pinned: this rank's rows of the mean embedding gradient
  cudaEvent_t ev_embw = nullptr;  // embedding table all-gathered
  // Floats from the start of d_head_g to the head's table gradient: the
  // layout's gf_pad, or with tied embeddings on a sharded context past the
  // padded [final gain] block that the reduce-scatter covers.
  size_t head_g_split = 0;
  size_t wslot_bytes = 0;  // bytes of a device weight slot (padded when sharded)

  // ---- mixture-of-experts layers (E > 0) ----
  // Routing of layer l, taken in its forward and reused by its recompute:
  // slot_of[t k + j] (the routed row of token t's j-th expert) and row_of[slot]
  // (the token of a routed row) on the device per layer, and each expert's
  // row count on the host (the expert GEMMs' sizes).
  float *moe_logits = nullptr, *moe_gate = nullptr, *moe_dgate = nullptr, *moe_dlogits = nullptr;
  int32_t *moe_idx = nullptr, *moe_slot = nullptr, *moe_row = nullptr;
  uint16_t *xe_b = nullptr, *dye_b = nullptr;
  float *ye = nullptr, *dxe = nullptr;
  int32_t* moe_idx_h = nullptr;    // pinned: per layer the experts each token chose [T k]
  int32_t* moe_route_h = nullptr;  // pinned: per layer slot_of | row_of [2 T k]
  std::vector<std::vector<int>> moe_count;  // [L][E]
  cudaEvent_t ev_route = nullptr;
};

namespace mteng {

int set_err(mt_ctx* c, int code, const std::string& m) {
  if (c)
    c->err = m;
  else
    g_create_error = m;
  return code;
}

#define CK(call)                                                                                  \
  do {                                                                                            \
    cudaError_t e_ = (call);                                                                      \
    if (e_ != cudaSuccess)                                                                        \
      return set_err(c, MT_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_));          \
  } while (0)
#define CKM(call)               \
  do {                          \
    int r_ = (call);            \
    if (r_ != MT_OK) return r_; \
  } while (0)
#define NK(call)                                                                                       \
  do {                                                                                                 \
    ncclResult_t e_ = (c->nccl->call);                                                                 \
    if (e_ != ncclSuccess)                                                                             \
      return set_err(c, MT_ERR_CUDA, std::string("nccl") + #call + ": " + c->nccl->GetErrorString(e_)); \
  } while (0)

// ---------------------------------------------------------------------------
// Sharded streaming: rank r of `world` owns elements [begin, end) of every
// layer block and of the [final gain | LM head] block, and embedding rows
// [row_begin, row_end). Each loads only its own part over the host link and
// all-gathers the rest; the gradients are averaged over the ranks with a
// reduce-scatter that leaves each rank its own part, which it checks,
// offloads and updates. Device blocks are padded to world * chunk elements.
// ---------------------------------------------------------------------------
bool sharded(const mt_ctx* c) { return c->comm_comp != nullptr; }

size_t embed_rows_chunk(const mt_shard& p, int V) { return (size_t)((V + p.world - 1) / p.world); }

// Reduce-scatter (mean over ranks) of a padded fp32 block on the compute
// stream: rank r's chunk ends up at blk + r * chunk. Then the finite check of
// that chunk into flag `idx`, and the flag's maximum over the ranks, so that
// every rank takes the same skip decision.
int reduce_own_chunk(mt_ctx* c, float* blk, size_t chunk, size_t own_begin, size_t own_end, int idx);

// ---------------------------------------------------------------------------
// Kernel wrappers with launch counting and optional event timing.
// ---------------------------------------------------------------------------
cudaEvent_t timing_event(mt_ctx* c) {
  if (c->timing_used == c->ev_timing.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    c->ev_timing.push_back(e);
  }
  return c->ev_timing[c->timing_used++];
}

int gemm(mt_ctx* c, const GemmDesc& g) {
  const bool timing = (c->cfg.flags & MT_FLAG_KERNEL_TIMING) != 0;
  cudaEvent_t a = nullptr, b = nullptr;
  if (timing) {
    a = timing_event(c);
    b = timing_event(c);
    if (a) cudaEventRecord(a, c->s_comp);
  }
  int r = gemm_bf16(g, c->s_comp, c->d_err);
  if (r != MT_OK) return set_err(c, r, "GEMM launch failed");
  c->launches += 1;
  if (timing && a && b) {
    cudaEventRecord(b, c->s_comp);
    c->timed.push_back({a, b, 2.0 * g.M * (double)g.N * g.K, 0});
  }
  return MT_OK;
}

GemmDesc gd_fwd(const void* A, int64_t lda, const void* B, int64_t ldb, void* C, int64_t ldc, int epi,
                const float* R, int M, int N, int K) {
  return GemmDesc{A, lda, false, B, ldb, false, C, ldc, epi, R, ldc, M, N, K, RopeDesc{}};
}
GemmDesc gd_dx(const void* A, int64_t lda, const void* B, int64_t ldb, void* C, int64_t ldc, int epi, int M, int N,
               int K) {
  return GemmDesc{A, lda, false, B, ldb, true, C, ldc, epi, nullptr, 0, M, N, K, RopeDesc{}};
}
GemmDesc gd_dw(const void* A, int64_t lda, const void* B, int64_t ldb, float* C, int64_t ldc, int epi, int M, int N,
               int K) {
  return GemmDesc{A, lda, true, B, ldb, true, C, ldc, epi, epi == EPI_F32_ADD ? C : nullptr, ldc, M, N, K,
                  RopeDesc{}};
}

int attn(mt_ctx* c, AttnArgs& a, bool bwd) {
  const bool timing = (c->cfg.flags & MT_FLAG_KERNEL_TIMING) != 0;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (timing) {
    e0 = timing_event(c);
    e1 = timing_event(c);
    if (e0) cudaEventRecord(e0, c->s_comp);
  }
  int r = bwd ? attention_bwd_tc(a, c->s_comp, c->d_err)
              : attention_fwd_tc(a, c->s_comp, c->d_err);
  if (r != MT_OK) return set_err(c, r, "attention launch failed");
  c->launches += bwd ? attention_bwd_kernels(a.hd) : 1;
  if (timing && e0 && e1) {
    cudaEventRecord(e1, c->s_comp);
    // causal attention: QK^T and PV over the visible half, per query head
    const double fwd = 2.0 * 2.0 * a.b * (double)a.s * a.s / 2.0 * a.H * a.hd;
    c->timed.push_back({e0, e1, bwd ? 2.5 * fwd : fwd, 1});
  }
  return MT_OK;
}

#define KL(expr, n)                                                                              \
  do {                                                                                           \
    int r_ = (expr);                                                                             \
    if (r_ != MT_OK)                                                                             \
      return set_err(c, r_, std::string("launch: ") + #expr + ": " + last_launch_error());       \
    c->launches += (n);                                                                          \
  } while (0)

// ---------------------------------------------------------------------------
// Check of a gradient range before its host update: flag bit 0 is set if any
// value is NaN or Inf, bit 1 if any kernel so far in the step has reported a
// bounded wait that ran out (its outputs, and so these gradients, are then
// undefined even when finite).
// ---------------------------------------------------------------------------
constexpr int32_t kFlagNonFinite = 1, kFlagDeviceError = 2;

__global__ void k_check_finite(const float* __restrict__ g, size_t n, const int32_t* __restrict__ dev_err,
                               int32_t* __restrict__ flag) {
  bool bad = false;
  const size_t n4 = n / 4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(g)[i];
    bad |= !isfinite(v.x) || !isfinite(v.y) || !isfinite(v.z) || !isfinite(v.w);
  }
  if (blockIdx.x == 0 && threadIdx.x < (n & 3)) bad |= !isfinite(g[n4 * 4 + threadIdx.x]);
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(flag, kFlagNonFinite);
  if (blockIdx.x == 0 && threadIdx.x == 0 && *dev_err != 0) atomicOr(flag, kFlagDeviceError);
}

int check_finite(mt_ctx* c, const float* g, size_t n, int idx) {
  CK(cudaMemsetAsync(c->d_flags + idx, 0, sizeof(int32_t), c->s_comp));
  k_check_finite<<<296, 256, 0, c->s_comp>>>(g, n, c->d_err, c->d_flags + idx);
  CK(cudaGetLastError());
  c->launches += 1;
  return MT_OK;
}

int reduce_own_chunk(mt_ctx* c, float* blk, size_t chunk, size_t own_begin, size_t own_end, int idx) {
  NK(ReduceScatter(blk, blk + (size_t)c->plan.rank * chunk, chunk, ncclFloat32, ncclAvg, c->comm_comp, c->s_comp));
  CKM(check_finite(c, blk + own_begin, own_end - own_begin, idx));
  NK(AllReduce(c->d_flags + idx, c->d_flags + idx, 1, ncclInt32, ncclMax, c->comm_comp, c->s_comp));
  return MT_OK;
}

// dst += src over n floats (n a multiple of 4, both 16-byte aligned).
__global__ void k_add_f32(float* __restrict__ dst, const float* __restrict__ src, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 4; i += (size_t)gridDim.x * blockDim.x) {
    float4 a = reinterpret_cast<float4*>(dst)[i];
    const float4 b = reinterpret_cast<const float4*>(src)[i];
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    reinterpret_cast<float4*>(dst)[i] = a;
  }
}

// Rows of the step's unique tokens (row u for token uid[u]) into a zeroed
// dense [rows, d] gradient; d is a multiple of 4.
__global__ void k_scatter_rows(const float* __restrict__ rows, const int32_t* __restrict__ uid, int n,
                               float* __restrict__ dst, int d) {
  const int d4 = d / 4;
  for (int u = blockIdx.x; u < n; u += gridDim.x) {
    const float4* src = reinterpret_cast<const float4*>(rows + (size_t)u * d);
    float4* out = reinterpret_cast<float4*>(dst + (size_t)uid[u] * d);
    for (int i = threadIdx.x; i < d4; i += blockDim.x) out[i] = src[i];
  }
}

// ---------------------------------------------------------------------------
// Boundary activations on the device. Resident: x_l at xb[l]. With
// MT_FLAG_OFFLOAD_ACTS three [T, d] slots: the forward alternates slots 0 and
// 1 (x_l in slot l mod 2, so x_L also follows that rule); in the backward, x_{L-1} is
// still in its forward slot and x_l for l <= L-2 (brought back from host
// memory, x_{L-2} by a device copy) alternates between slot 2 and slot
// (L-1) mod 2, so that x_{l-1} can load while layer l runs.
// ---------------------------------------------------------------------------
bool offload_acts(const mt_ctx* c) { return (c->cfg.flags & MT_FLAG_OFFLOAD_ACTS) != 0; }

float* x_fwd(mt_ctx* c, int l) {
  const size_t n = (size_t)c->lay.sh.T * c->lay.sh.d;
  return c->xb + (offload_acts(c) ? (size_t)(l & 1) : (size_t)l) * n;
}

float* x_bwd(mt_ctx* c, int l) {
  const int L = c->lay.sh.L;
  if (!offload_acts(c) || l == L - 1) return x_fwd(c, l);
  const size_t n = (size_t)c->lay.sh.T * c->lay.sh.d;
  return c->xb + (size_t)(((L - 2 - l) % 2 == 0) ? 2 : ((L - 1) & 1)) * n;
}

// Attention output O [T, H hd] (bf16) and log-sum-exp [b, H, s] of layer l:
// one buffer for every layer, or with MT_FLAG_STASH_ATTN one per layer, kept
// from the forward sweep to the layer's backward, so that the recompute runs
// no attention forward.
bool stash_attn(const mt_ctx* c) { return (c->cfg.flags & MT_FLAG_STASH_ATTN) != 0; }

uint16_t* ao_of(mt_ctx* c, int l) {
  const Shapes& s = c->lay.sh;
  return c->ao_b + (stash_attn(c) ? (size_t)l * s.T * s.Hd : 0);
}

float* lse_of(mt_ctx* c, int l) {
  const Shapes& s = c->lay.sh;
  return c->lse + (stash_attn(c) ? (size_t)l * s.b * s.H * s.s : 0);
}

// ---------------------------------------------------------------------------
// Layer forward from x with the weights of `slot`. With xo the layer output
// goes there; otherwise (recompute) the down projection is skipped, since the
// backward only needs the intermediates, and with MT_FLAG_STASH_ATTN so is the
// attention, whose output the forward sweep kept (the forward is
// deterministic: the kept O and LSE are the ones a recompute would produce).
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Mixture-of-experts MLP of layer l from the bf16 MLP input w_b (expert
// weights in the slot W). Routed rows are grouped by expert, tokens in
// increasing order within an expert, so every expert product is one GEMM on
// a contiguous block of rows. The forward sweep takes the routing: the
// experts each token chose go to the host, which lays out the rows and keeps
// each expert's row count (the GEMMs' sizes); the recompute reruns the router
// (the same choices: the forward is deterministic) and reuses that layout.
// ---------------------------------------------------------------------------
bool wait_event(mt_ctx* c, cudaEvent_t e);

void moe_dispatch(const int32_t* idx, int T, int k, int E, int32_t* slot_of, int32_t* row_of, std::vector<int>& cnt) {
  std::fill(cnt.begin(), cnt.end(), 0);
  const int Tk = T * k;
  for (int p = 0; p < Tk; ++p) cnt[idx[p]]++;
  std::vector<int> next(E, 0);
  for (int e = 1; e < E; ++e) next[e] = next[e - 1] + cnt[e - 1];
  for (int p = 0; p < Tk; ++p) {
    const int sl = next[idx[p]]++;
    slot_of[p] = sl;
    row_of[sl] = p / k;
  }
}

int moe_fwd(mt_ctx* c, int l, const uint16_t* W, float* xo) {
  const Shapes& s = c->lay.sh;
  const Layout& y = c->lay;
  const int T = s.T, d = s.d, F = s.F, E = s.E, k = s.topk, Tk = T * k;
  cudaStream_t st = c->s_comp;
  const uint16_t* Wg = W + y.bf_gu;
  const uint16_t* Wu = Wg + (size_t)E * F * d;
  const uint16_t* Wd = W + y.bf_d;
  int32_t* slot_of = c->moe_slot + (size_t)l * Tk;
  int32_t* row_of = c->moe_row + (size_t)l * Tk;
  KL(launch_moe_router(c->w_b, W + y.bf_r, T, d, E, k, c->moe_logits, c->moe_idx, c->moe_gate, st), 1);
  if (xo) {
    int32_t* ih = c->moe_idx_h + (size_t)l * Tk;
    CK(cudaMemcpyAsync(ih, c->moe_idx, (size_t)Tk * 4, cudaMemcpyDeviceToHost, st));
    CK(cudaEventRecord(c->ev_route, st));
    if (!wait_event(c, c->ev_route)) return set_err(c, MT_ERR_TIMEOUT, "routing did not arrive within the wait limit");
    for (int p = 0; p < Tk; ++p)
      if (ih[p] < 0 || ih[p] >= E) return set_err(c, MT_ERR_DEVICE, "router chose no valid expert");
    int32_t* hs = c->moe_route_h + (size_t)l * 2 * Tk;
    moe_dispatch(ih, T, k, E, hs, hs + Tk, c->moe_count[l]);
    CK(cudaMemcpyAsync(slot_of, hs, (size_t)Tk * 4, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(row_of, hs + Tk, (size_t)Tk * 4, cudaMemcpyHostToDevice, st));
  }
  KL(launch_moe_gather(c->w_b, row_of, Tk, d, c->xe_b, st), 1);
  const std::vector<int>& cnt = c->moe_count[l];
  size_t off = 0;
  for (int e = 0; e < E; ++e) {
    const int n = cnt[e];
    if (n == 0) continue;
    // gate and up of expert e into the [rows, 2F] buffer's two halves
    CKM(gemm(c, gd_fwd(c->xe_b + off * d, d, Wg + (size_t)e * F * d, d, c->gu_b + off * 2 * F, 2 * F, EPI_BF16,
                       nullptr, n, F, d)));
    CKM(gemm(c, gd_fwd(c->xe_b + off * d, d, Wu + (size_t)e * F * d, d, c->gu_b + off * 2 * F + F, 2 * F,
                       EPI_BF16, nullptr, n, F, d)));
    off += n;
  }
  KL(launch_swiglu_fwd(c->gu_b, c->act_b, Tk, F, st), 1);
  off = 0;
  for (int e = 0; e < E; ++e) {
    const int n = cnt[e];
    if (n == 0) continue;
    CKM(gemm(c, gd_fwd(c->act_b + off * F, F, Wd + (size_t)e * d * F, F, c->ye + off * d, d, EPI_F32, nullptr, n, d,
                       F)));
    off += n;
  }
  if (xo) KL(launch_moe_combine(c->h_f, c->ye, slot_of, c->moe_gate, T, k, d, xo, st), 1);
  return MT_OK;
}

// Backward of moe_fwd from gin = dL/d(MLP output): the expert, gate and router
// weight gradients of layer l into Gw (the layer's gradient block at the
// given tensor ids) and dL/dw (fp32) into c->tmp_f. An expert no token chose
// gets zero gradients.
int moe_bwd(mt_ctx* c, int l, const uint16_t* W, const float* gin, const std::function<float*(int)>& G) {
  const Shapes& s = c->lay.sh;
  const Layout& y = c->lay;
  const int T = s.T, d = s.d, F = s.F, E = s.E, k = s.topk, Tk = T * k;
  cudaStream_t st = c->s_comp;
  const uint16_t* Wg = W + y.bf_gu;
  const uint16_t* Wu = Wg + (size_t)E * F * d;
  const uint16_t* Wd = W + y.bf_d;
  const int32_t* slot_of = c->moe_slot + (size_t)l * Tk;
  const std::vector<int>& cnt = c->moe_count[l];
  KL(launch_moe_dy(gin, c->ye, slot_of, c->moe_gate, T, k, d, c->dye_b, c->moe_dgate, st), 1);
  size_t off = 0;
  for (int e = 0; e < E; ++e) {
    const int n = cnt[e];
    float* gWd = G(MT_T_WDOWN) + (size_t)e * d * F;
    if (n == 0) {
      CK(cudaMemsetAsync(gWd, 0, (size_t)d * F * 4, st));
      continue;
    }
    CKM(gemm(c, gd_dw(c->dye_b + off * d, d, c->act_b + off * F, F, gWd, F, EPI_F32, d, F, n)));
    CKM(gemm(c, gd_dx(c->dye_b + off * d, d, Wd + (size_t)e * d * F, F, c->dact_b + off * F, F, EPI_BF16, n, F, d)));
    off += n;
  }
  KL(launch_swiglu_bwd(c->gu_b, c->dact_b, c->dgu_b, Tk, F, st), 1);
  off = 0;
  for (int e = 0; e < E; ++e) {
    const int n = cnt[e];
    float* gWg = G(MT_T_WGATE) + (size_t)e * F * d;
    float* gWu = G(MT_T_WUP) + (size_t)e * F * d;
    if (n == 0) {
      CK(cudaMemsetAsync(gWg, 0, (size_t)F * d * 4, st));
      CK(cudaMemsetAsync(gWu, 0, (size_t)F * d * 4, st));
      continue;
    }
    const uint16_t* dg = c->dgu_b + off * 2 * F;
    CKM(gemm(c, gd_dw(dg, 2 * F, c->xe_b + off * d, d, gWg, d, EPI_F32, F, d, n)));
    CKM(gemm(c, gd_dw(dg + F, 2 * F, c->xe_b + off * d, d, gWu, d, EPI_F32, F, d, n)));
    float* dx = c->dxe + off * d;
    CKM(gemm(c, gd_dx(dg, 2 * F, Wg + (size_t)e * F * d, d, dx, d, EPI_F32, n, d, F)));
    GemmDesc gu = gd_dx(dg + F, 2 * F, Wu + (size_t)e * F * d, d, dx, d, EPI_F32_ADD, n, d, F);
    gu.R = dx;
    gu.ldr = d;
    CKM(gemm(c, gu));
    off += n;
  }
  KL(launch_moe_router_bwd(c->moe_gate, c->moe_dgate, c->moe_idx, c->w_b, W + y.bf_r, c->dxe, slot_of, T, k, d, E,
                           c->moe_dlogits, G(MT_T_ROUTER), c->tmp_f, st),
     3);
  return MT_OK;
}

int layer_fwd(mt_ctx* c, int l, int slot, const float* x, float* xo) {
  const Shapes& s = c->lay.sh;
  const Layout& y = c->lay;
  const uint16_t* W = c->wslot[slot];
  cudaStream_t st = c->s_comp;
  KL(launch_rmsnorm_fwd(x, W + y.bf_g1, c->u_b, c->r1, s.T, s.d, c->cfg.norm_eps, st), 1);
  {
    // q, k, v projection with RoPE on the q and k heads in the epilogue
    GemmDesc g = gd_fwd(c->u_b, s.d, W + y.bf_qkv, s.d, c->qkv_b, s.Nqkv, EPI_BF16_ROPE, nullptr, s.T, s.Nqkv, s.d);
    g.rope = RopeDesc{c->d_cos, c->d_sin, s.Hd + s.Hkv * s.hd, s.hd, s.s};
    CKM(gemm(c, g));
  }
  AttnArgs a{};
  a.q = c->qkv_b;
  a.k = c->qkv_b + s.Hd;
  a.v = c->qkv_b + s.Hd + s.Hkv * s.hd;
  a.ldqkv = s.Nqkv;
  a.o = ao_of(c, l);
  a.ldo = s.Hd;
  a.lse = lse_of(c, l);
  a.b = s.b;
  a.s = s.s;
  a.H = s.H;
  a.Hkv = s.Hkv;
  a.hd = s.hd;
  a.scale = 1.0f / sqrtf((float)s.hd);
  if (xo || !stash_attn(c)) CKM(attn(c, a, false));
  CKM(gemm(c, gd_fwd(ao_of(c, l), s.Hd, W + y.bf_o, s.Hd, c->h_f, s.d, EPI_F32_ADD, x, s.T, s.d, s.Hd)));
  KL(launch_rmsnorm_fwd(c->h_f, W + y.bf_g2, c->w_b, c->r2, s.T, s.d, c->cfg.norm_eps, st), 1);
  if (s.E > 0) return moe_fwd(c, l, W, xo);
  CKM(gemm(c, gd_fwd(c->w_b, s.d, W + y.bf_gu, s.d, c->gu_b, 2 * s.F, EPI_BF16, nullptr, s.T, 2 * s.F, s.d)));
  KL(launch_swiglu_fwd(c->gu_b, c->act_b, s.T, s.F, st), 1);
  if (xo) CKM(gemm(c, gd_fwd(c->act_b, s.F, W + y.bf_d, s.F, xo, s.d, EPI_F32_ADD, c->h_f, s.T, s.d, s.F)));
  return MT_OK;
}

// Layer backward from its input x: gin = dL/dx_{l+1} (fp32), writes gout =
// dL/dx_l and the layer's fp32 gradients into grad slot gs (arena layout of
// the layer).
int layer_bwd(mt_ctx* c, int l, int slot, const float* x, float* gs, const float* gin, float* gout) {
  const Shapes& s = c->lay.sh;
  const Layout& y = c->lay;
  const uint16_t* W = c->wslot[slot];
  const size_t base = y.layer_begin(l);
  auto G = [&](int tid) { return gs + (y.t(l, tid).off - base); };
  cudaStream_t st = c->s_comp;
  const int T = s.T, d = s.d, F = s.F;

  if (s.E > 0) {
    CKM(moe_bwd(c, l, W, gin, G));
  } else {
    KL(launch_cast_f32_bf16(gin, c->gxb, (int64_t)T * d, st), 1);
    // down projection
    CKM(gemm(c, gd_dw(c->gxb, d, c->act_b, F, G(MT_T_WDOWN), F, EPI_F32, d, F, T)));
    CKM(gemm(c, gd_dx(c->gxb, d, W + y.bf_d, F, c->dact_b, F, EPI_BF16, T, F, d)));
    KL(launch_swiglu_bwd(c->gu_b, c->dact_b, c->dgu_b, T, F, st), 1);
    // gate/up projections
    CKM(gemm(c, gd_dw(c->dgu_b, 2 * F, c->w_b, d, G(MT_T_WGATE), d, EPI_F32, 2 * F, d, T)));
    CKM(gemm(c, gd_dx(c->dgu_b, 2 * F, W + y.bf_gu, d, c->tmp_f, d, EPI_F32, T, d, 2 * F)));
  }
  KL(launch_rmsnorm_bwd(c->h_f, W + y.bf_g2, c->r2, c->tmp_f, gin, c->dh_f, c->dhb, c->rms_part, G(MT_T_MLP_NORM),
                        T, d, st),
     2);
  // output projection
  CKM(gemm(c, gd_dw(c->dhb, d, ao_of(c, l), s.Hd, G(MT_T_WO), s.Hd, EPI_F32, d, s.Hd, T)));
  CKM(gemm(c, gd_dx(c->dhb, d, W + y.bf_o, s.Hd, c->dao_b, s.Hd, EPI_BF16, T, s.Hd, d)));
  // attention
  AttnArgs a{};
  a.q = c->qkv_b;
  a.k = c->qkv_b + s.Hd;
  a.v = c->qkv_b + s.Hd + s.Hkv * s.hd;
  a.ldqkv = s.Nqkv;
  a.o = ao_of(c, l);
  a.ldo = s.Hd;
  a.lse = lse_of(c, l);
  a.dout = c->dao_b;
  a.dvec = c->dvec;
  a.dq_acc = c->dqacc;
  a.ldqa = s.Hd;
  a.dq = c->dqkv_b;
  a.lddq = s.Nqkv;
  a.dk = c->dqkv_b + s.Hd;
  a.dv = c->dqkv_b + s.Hd + s.Hkv * s.hd;
  a.lddkv = s.Nqkv;
  a.b = s.b;
  a.s = s.s;
  a.H = s.H;
  a.Hkv = s.Hkv;
  a.hd = s.hd;
  a.scale = 1.0f / sqrtf((float)s.hd);
  a.rope_cos = c->d_cos;  // dq, dk come back with respect to the pre-RoPE projections
  a.rope_sin = c->d_sin;
  CKM(attn(c, a, true));
  // q/k/v projections
  CKM(gemm(c, gd_dw(c->dqkv_b, s.Nqkv, c->u_b, d, G(MT_T_WQ), d, EPI_F32, s.Nqkv, d, T)));
  CKM(gemm(c, gd_dx(c->dqkv_b, s.Nqkv, W + y.bf_qkv, d, c->tmp_f, d, EPI_F32, T, d, s.Nqkv)));
  KL(launch_rmsnorm_bwd(x, W + y.bf_g1, c->r1, c->tmp_f, c->dh_f, gout, nullptr, c->rms_part, G(MT_T_ATTN_NORM), T,
                        d, st),
     2);
  if (sharded(c))
    return reduce_own_chunk(c, gs, c->plan.layer_chunk, c->plan.layer_begin, c->plan.layer_end, l);
  return check_finite(c, gs, y.layer_end(l) - base, l);
}

// Final norm, LM head and cross-entropy, head gradients; writes dL/dx_L to gout.
int head_step(mt_ctx* c, float* gout) {
  const Shapes& s = c->lay.sh;
  const int T = s.T, d = s.d, V = s.V;
  cudaStream_t st = c->s_comp;
  const size_t gf_pad = c->head_g_split;  // floats between dgf and dWhead
  const uint16_t* gf = c->d_head_w;
  // tied embeddings on a sharded context: the head reads the device table
  const uint16_t* Wh = (sharded(c) && c->lay.tied) ? c->d_embed_w : c->d_head_w + align_up(d, 128);
  float* dgf = c->d_head_g;
  float* dWh = c->d_head_g + gf_pad;
  const float* xL = x_fwd(c, s.L);
  KL(launch_rmsnorm_fwd(xL, gf, c->n_b, c->rf, T, d, c->cfg.norm_eps, st), 1);
  for (int t0 = 0; t0 < T; t0 += c->Tc) {
    const int tc = std::min(c->Tc, T - t0);
    const uint16_t* n_c = c->n_b + (size_t)t0 * d;
    CKM(gemm(c, gd_fwd(n_c, d, Wh, d, c->logits, V, EPI_F32, nullptr, tc, V, d)));
    KL(launch_softmax_ce(c->logits, V, c->d_lab + t0, c->dz_b, V, c->rowloss + t0, tc, V, 1.0f / T, st), 1);
    CKM(gemm(c, gd_dw(c->dz_b, V, n_c, d, dWh, d, t0 == 0 ? EPI_F32 : EPI_F32_ADD, V, d, tc)));
    CKM(gemm(c, gd_dx(c->dz_b, V, Wh, d, c->tmp_f + (size_t)t0 * d, d, EPI_F32, tc, d, V)));
  }
  KL(launch_sum_all(c->rowloss, T, c->d_loss, 0, st), 1);
  if (sharded(c)) NK(AllReduce(c->d_loss, c->d_loss, 1, ncclFloat32, ncclAvg, c->comm_comp, st));
  KL(launch_rmsnorm_bwd(xL, gf, c->rf, c->tmp_f, nullptr, gout, nullptr, c->rms_part, dgf, T, d, st), 2);
  if (sharded(c))
    return reduce_own_chunk(c, c->d_head_g, c->plan.head_chunk, c->plan.head_begin, c->plan.head_end, s.L);
  return check_finite(c, c->d_head_g, c->lay.head_block, s.L);
}

// ---------------------------------------------------------------------------
// Optimizer thread.
// ---------------------------------------------------------------------------
bool wait_event(mt_ctx* c, cudaEvent_t e) {
  if (!e) return true;
  const double t0 = now_s();
  while (true) {
    cudaError_t r = cudaEventQuery(e);
    if (r == cudaSuccess) return true;
    if (r != cudaErrorNotReady) return false;
    if (now_s() - t0 > c->wait_limit_s) return false;
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

struct Seg {
  size_t off, n;       // floats in the arena
  uint16_t* bf;        // bf16 destination of element 0
  const float* g;      // fp32 gradient of element 0; both null: zero gradient
  const uint16_t* g16 = nullptr;  // bf16 gradient of element 0 (MT_FLAG_BF16_GRADS)
};

// AdamW step t over the segments. threads > 0 caps the threads that work on
// it (the others of the pool stay idle).
void adamw_segments(mt_ctx* c, const std::vector<Seg>& segs, int t, int threads = 0) {
  // 64K-element pieces handed out dynamically: a worker slowed by other
  // activity on its core (the enqueueing thread, DMA) does not hold the job up.
  const AdamHyper h{c->cfg.lr, c->cfg.beta1, c->cfg.beta2, c->cfg.adam_eps, c->cfg.wd};
  const size_t chunk = 1 << 16;
  struct Task {
    size_t off, n;
    uint16_t* bf;
    const float* g;
    const uint16_t* g16;
  };
  std::vector<Task> tasks;
  double bytes = 0;  // host DRAM bytes: p, m, v read and written, bf16 copy written, gradient read
  for (const Seg& sg : segs) {
    for (size_t i = 0; i < sg.n; i += chunk)
      tasks.push_back({sg.off + i, std::min(chunk, sg.n - i), sg.bf ? sg.bf + i : nullptr, sg.g ? sg.g + i : nullptr,
                       sg.g16 ? sg.g16 + i : nullptr});
    bytes += (26.0 + (sg.g ? 4.0 : sg.g16 ? 2.0 : 0.0)) * sg.n;
  }
  if (tasks.empty()) return;
  const double t0 = now_s();
  if (c->adamw_first == 0) c->adamw_first = t0;
  auto one = [&](size_t i) {
    const Task& k = tasks[i];
    if (k.g16)
      adamw_chunk_bf16g(c->arena + k.off, k.g16, c->m + k.off, c->v + k.off, k.bf, k.n, h, t);
    else
      adamw_chunk(c->arena + k.off, k.g, c->m + k.off, c->v + k.off, k.bf, k.n, h, t);
  };
  if (threads <= 0 || threads >= c->pool->size()) {
    c->pool->run((int)tasks.size(), [&](int i) { one((size_t)i); });
  } else {
    std::atomic<size_t> next{0};
    c->pool->run(threads, [&](int) {
      for (size_t i = next.fetch_add(1); i < tasks.size(); i = next.fetch_add(1)) one(i);
    });
  }
  c->adamw_last = now_s();
  c->adamw_s += c->adamw_last - t0;
  c->adamw_bytes += bytes;
}

void run_job_body(mt_ctx* c, const Job& j);

void run_job(mt_ctx* c, const Job& j) {
  if (!wait_event(c, j.ready)) {
    c->opt_status = MT_ERR_TIMEOUT;
    c->err = "gradient offload did not complete within the wait limit";
    c->skip_updates = true;
    return;
  }
  const double t0 = now_s();
  run_job_body(c, j);
  c->job_times.push_back({(int)j.kind, j.layer, t0, now_s()});
}

// Segment of n arena floats from `off` whose host gradient starts at g
// (gsz bytes per element).
Seg grad_seg(mt_ctx* c, size_t off, size_t n, uint16_t* bf, const uint8_t* g) {
  if (c->gsz == 2) return Seg{off, n, bf, nullptr, reinterpret_cast<const uint16_t*>(g)};
  return Seg{off, n, bf, reinterpret_cast<const float*>(g)};
}

// AdamW segments of decoder layer l (gradient block g) or, for l < 0, of the
// final norm and LM head (gradients in grad_head).
std::vector<Seg> layer_or_head_segs(mt_ctx* c, int l, const uint8_t* g) {
  const Layout& y = c->lay;
  std::vector<Seg> segs;
  if (l >= 0) {
    uint16_t* blk = c->bf_layers + (size_t)l * y.bf_layer;
    for (int tid = 0; tid < kLayerTensors; ++tid) {
      const TRef& r = y.t(l, tid);
      segs.push_back(grad_seg(c, r.off, r.n, blk + y.bf_of(tid), g + (r.off - y.layer_begin(l)) * c->gsz));
    }
  } else {
    segs.push_back(grad_seg(c, y.final_norm.off, y.final_norm.n, c->bf_head, c->grad_head));
    // (tied: the table's update waits for the gathered rows' gradient, in the EMBED job)
    if (!y.tied)
      segs.push_back(grad_seg(c, y.head.off, y.head.n, c->bf_head + align_up(y.sh.d, 128),
                              c->grad_head + y.gf_pad * c->gsz));
  }
  if (!sharded(c)) return segs;
  // Sharded: only this rank's elements [lo, hi) of the block (offsets from the
  // block's first arena float); the other ranks update the rest.
  const size_t base = l >= 0 ? y.layer_begin(l) : y.final_norm.off;
  const size_t lo = base + (l >= 0 ? c->plan.layer_begin : c->plan.head_begin);
  const size_t hi = base + (l >= 0 ? c->plan.layer_end : c->plan.head_end);
  std::vector<Seg> mine;
  for (const Seg& sg : segs) {
    const size_t b = std::max(sg.off, lo), e = std::min(sg.off + sg.n, hi);
    if (b >= e) continue;
    const size_t k = b - sg.off;
    mine.push_back(Seg{b, e - b, sg.bf ? sg.bf + k : nullptr, sg.g ? sg.g + k : nullptr, sg.g16 ? sg.g16 + k : nullptr});
  }
  return mine;
}

// Segments of the zero-gradient update of every embedding row not listed in
// skip (sorted, distinct row ids): the rows no token of a step touched.
std::vector<Seg> untouched_segs(mt_ctx* c, const std::vector<int32_t>& skip) {
  const Layout& y = c->lay;
  const size_t d = y.sh.d;
  std::vector<Seg> segs;
  int32_t next = 0;  // first row of the current untouched run
  for (size_t u = 0; u <= skip.size(); ++u) {
    const int32_t stop = u < skip.size() ? skip[u] : y.sh.V;
    if (stop > next)
      segs.push_back({y.embed.off + (size_t)next * d, (size_t)(stop - next) * d, c->bf_embed + (size_t)next * d,
                      nullptr});
    next = stop + 1;
  }
  return segs;
}

// Records the outcome of a job's gradient checks (flag bits of k_check_finite)
// and returns true while updates may still run this step: after a failed check
// this and every later update of the step are skipped.
bool passes_checks(mt_ctx* c, int32_t flag) {
  if ((flag & kFlagDeviceError) && c->opt_status == MT_OK) {
    c->opt_status = MT_ERR_DEVICE;
    c->err = "a kernel's bounded wait ran out; this and the remaining updates were skipped";
  } else if ((flag & kFlagNonFinite) && c->opt_status == MT_OK) {
    c->opt_status = MT_ERR_NONFINITE;
    c->err = "non-finite gradient; this and the remaining updates were skipped";
  }
  if (flag & (kFlagDeviceError | kFlagNonFinite)) c->skip_updates = true;
  return !c->skip_updates;
}

void run_job_body(mt_ctx* c, const Job& j) {
  const Layout& y = c->lay;
  const Shapes& s = y.sh;
  if (j.kind == Job::HEAD_PREV || j.kind == Job::LAYER_PREV) {
    // Checked in its own step; it belongs to that step's update, so this
    // step's skip state does not apply to it.
    adamw_segments(c, layer_or_head_segs(c, j.kind == Job::HEAD_PREV ? -1 : j.layer, j.g), j.step,
                   c->overlap_threads);
    return;
  }
  if (j.kind == Job::EMBED_UNTOUCHED_PREV) {
    // The rest of the previous step's untouched-row update (that step passed
    // every check): rows this step does not touch either, so neither the GPU
    // nor this step's updates read them meanwhile.
    adamw_segments(c, untouched_segs(c, c->untouched_skip), j.step, c->overlap_threads);
    return;
  }
  if (j.kind == Job::EMBED_UNTOUCHED) {
    // Queued after the step's last checked job: runs only if every check passed.
    if (c->skip_updates || (c->cfg.flags & MT_FLAG_NO_UPDATE)) return;
    adamw_segments(c, untouched_segs(c, c->uniq), c->step);
    return;
  }
  if (j.kind == Job::EMBED && sharded(c)) {
    // This rank's rows of the mean dense gradient, checked on the device (the
    // flag came back with them, its maximum over the ranks): the gradient
    // arena reports them, the update below reads them from the staging rows.
    // With bf16 gradients the rows are rounded once, here on the host, as the
    // unsharded path rounds its gathered rows.
    const size_t d = s.d, rb = (size_t)c->plan.embed_row_begin, re = (size_t)c->plan.embed_row_end;
    const size_t gsz = c->gsz;
    parallel_ranges(*c->pool, (re - rb) * d, [&](size_t b, size_t e) {
      float* src = c->emb_own_h + b;
      if (gsz == 2)
        for (size_t k = 0; k < e - b; ++k) {
          const uint32_t w = (uint32_t)bf16_rne(src[k]) << 16;
          memcpy(src + k, &w, 4);
        }
      if (c->grad && gsz == 4)
        memcpy(reinterpret_cast<float*>(c->grad) + y.embed.off + rb * d + b, src, (e - b) * 4);
      if (c->grad && gsz == 2)
        bf16_round_chunk(src, reinterpret_cast<uint16_t*>(c->grad) + y.embed.off + rb * d + b, e - b);
    });
    // tied: the final gain's gradient came back in the head's own buffer; the
    // gradient arena reports this rank's part of it
    if (y.tied && c->grad && c->plan.head_end > c->plan.head_begin)
      memcpy(c->grad + (y.final_norm.off + c->plan.head_begin) * gsz, c->grad_head + c->plan.head_begin * gsz,
             (c->plan.head_end - c->plan.head_begin) * gsz);
  } else if (j.kind == Job::EMBED) {
    // Touched rows: check this step's gradient rows for NaN/Inf and, with a
    // gradient arena, put last step's touched rows back to zero and scatter
    // this step's rows in (every other row's stored gradient is 0). The update
    // reads them from the staging rows.
    // (tied embeddings: the rows go into the head's dense table gradient below)
    uint8_t* ge = (c->grad && !y.tied) ? c->grad + y.embed.off * c->gsz : nullptr;
    const size_t d = s.d, gsz = c->gsz;
    const int nt = c->pool->size() * 4;
    if (ge) {
      const size_t np = c->prev_uniq.size();
      c->pool->run(nt, [&](int i) {
        for (size_t k = np * i / nt; k < np * (i + 1) / nt; ++k)
          memset(ge + (size_t)c->prev_uniq[k] * d * gsz, 0, d * gsz);
      });
    }
    c->prev_uniq = c->uniq;
    const size_t nu = c->uniq.size();
    std::vector<char> bad(nt, 0);
    c->pool->run(nt, [&](int i) {
      bool b = false;
      for (size_t u = nu * i / nt; u < nu * (i + 1) / nt; ++u) {
        float* src = c->emb_rows_h + u * d;
        if (gsz == 2)  // bf16 gradients: these rows are rounded once too, here on the host
          for (size_t k = 0; k < d; ++k) {
            const uint32_t w = (uint32_t)bf16_rne(src[k]) << 16;
            memcpy(src + k, &w, 4);
          }
        float acc = 0.f;
        for (size_t k = 0; k < d; ++k) acc += src[k] * 0.f;  // NaN or Inf anywhere makes acc NaN
        b |= !(acc == 0.f);
        if (ge && gsz == 4) memcpy(ge + (size_t)c->uniq[u] * d * 4, src, d * 4);
        if (ge && gsz == 2) bf16_round_chunk(src, reinterpret_cast<uint16_t*>(ge + (size_t)c->uniq[u] * d * 2), d);
      }
      bad[i] = b;
    });
    for (char b : bad)
      if (b) c->flags_h[j.flag_index] |= kFlagNonFinite;
    int32_t dev_err = 0;  // device error word as of the embedding backward
    memcpy(&dev_err, c->misc_h + 2, 4);
    if (dev_err != 0) c->flags_h[j.flag_index] |= kFlagDeviceError;
    if (y.tied) {
      // The table's gradient: the head's dense V x d part plus the gathered
      // rows (distinct rows per task, so no two threads add to one row).
      float* gh = reinterpret_cast<float*>(c->grad_head) + y.gf_pad;
      c->pool->run(nt, [&](int i) {
        for (size_t u = nu * i / nt; u < nu * (i + 1) / nt; ++u) {
          float* row = gh + (size_t)c->uniq[u] * d;
          const float* src = c->emb_rows_h + u * d;
          for (size_t k = 0; k < d; ++k) row[k] += src[k];
        }
      });
      if (c->grad) {  // the gradient arena reports the table's and the final gain's gradients
        parallel_ranges(*c->pool, y.embed.n, [&](size_t b, size_t e) {
          memcpy(reinterpret_cast<float*>(c->grad) + y.embed.off + b, gh + b, (e - b) * 4);
        });
        memcpy(reinterpret_cast<float*>(c->grad) + y.final_norm.off, c->grad_head, d * 4);
      }
    }
  }
  if (!passes_checks(c, c->flags_h[j.flag_index])) return;
  if (c->cfg.flags & MT_FLAG_NO_UPDATE) return;
  if (j.defer) {
    // Gradients are finite: the update runs at the start of the next step.
    Job p = j;
    p.kind = j.kind == Job::HEAD ? Job::HEAD_PREV : Job::LAYER_PREV;
    p.ready = nullptr;
    p.defer = false;
    p.step = c->step;
    c->deferred.push_back(p);
    return;
  }
  std::vector<Seg> segs;
  if (j.kind == Job::LAYER || j.kind == Job::HEAD) {
    segs = layer_or_head_segs(c, j.kind == Job::HEAD ? -1 : j.layer, j.g);
  } else if (sharded(c)) {  // EMBED, sharded: this rank's rows, dense (untouched rows have zero gradient)
    const size_t rb = (size_t)c->plan.embed_row_begin, re = (size_t)c->plan.embed_row_end;
    if (re > rb) segs.push_back({y.embed.off + rb * s.d, (re - rb) * s.d, c->bf_embed + rb * s.d, c->emb_own_h});
  } else if (y.tied) {  // EMBED, tied: one dense update of the whole table
    segs.push_back({y.embed.off, y.embed.n, c->bf_embed, reinterpret_cast<const float*>(c->grad_head) + y.gf_pad});
  } else {
    for (size_t u = 0; u < c->uniq.size(); ++u) {
      const size_t r = (size_t)c->uniq[u];
      segs.push_back({y.embed.off + r * s.d, (size_t)s.d, c->bf_embed + r * s.d, c->emb_rows_h + u * s.d});
    }
  }
  adamw_segments(c, segs, c->step);
  if (j.kind == Job::EMBED && (c->cfg.flags & MT_FLAG_DEFER_UPDATES) && !y.tied && !sharded(c)) {
    // The step's last job: every gradient passed its checks, so the
    // zero-gradient update of the rows it did not touch is due. It runs with
    // the next step (or at the next flush), overlapping its GPU work.
    c->untouched_pending = true;
    c->untouched_step = c->step;
    c->untouched_of = c->uniq;
  }
}

void opt_loop(mt_ctx* c) {
  while (true) {
    Job j;
    {
      std::unique_lock<std::mutex> lk(c->opt_mu);
      c->opt_cv.wait(lk, [&] { return c->opt_stop || !c->jobs.empty(); });
      if (c->opt_stop && c->jobs.empty()) return;
      j = c->jobs.front();
      c->jobs.pop_front();
    }
    run_job(c, j);
    {
      std::lock_guard<std::mutex> lk(c->opt_mu);
      --c->jobs_pending;
      if (j.kind == Job::LAYER) ++c->layer_jobs_done;
      if (j.kind == Job::HEAD_PREV) c->prev_pending[c->lay.sh.L] = 0;
      if (j.kind == Job::LAYER_PREV) c->prev_pending[j.layer] = 0;
    }
    c->opt_done_cv.notify_all();
  }
}

void push_job(mt_ctx* c, const Job& j) {
  {
    std::lock_guard<std::mutex> lk(c->opt_mu);
    c->jobs.push_back(j);
    ++c->jobs_pending;
  }
  c->opt_cv.notify_one();
}

void wait_jobs(mt_ctx* c) {
  std::unique_lock<std::mutex> lk(c->opt_mu);
  c->opt_done_cv.wait(lk, [&] { return c->jobs_pending == 0; });
}

// Queues the updates deferred by the last step in the order the forward sweep
// streams their weights again (layers ascending, then the LM head), then the
// rest of the untouched embedding rows, which nothing of the step reads; they
// touch disjoint tensors, so any order gives the same result. Called between
// steps, when the optimizer is idle.
void queue_deferred(mt_ctx* c) {
  if (c->deferred.empty()) return;
  auto key = [](const Job& j) {
    return j.kind == Job::EMBED_UNTOUCHED_PREV ? INT32_MAX : j.kind == Job::HEAD_PREV ? INT32_MAX - 1 : j.layer;
  };
  std::sort(c->deferred.begin(), c->deferred.end(), [&](const Job& a, const Job& b) { return key(a) < key(b); });
  {
    std::lock_guard<std::mutex> lk(c->opt_mu);
    for (const Job& j : c->deferred) {
      c->jobs.push_back(j);
      if (j.kind == Job::HEAD_PREV) c->prev_pending[c->lay.sh.L] = 1;
      if (j.kind == Job::LAYER_PREV) c->prev_pending[j.layer] = 1;
    }
    c->jobs_pending += (int)c->deferred.size();
  }
  c->deferred.clear();
  c->opt_cv.notify_one();
}

// Queues the remainder of a pending untouched-row update: every row outside
// `skip` (sorted, distinct). Called between steps.
void defer_untouched_rest(mt_ctx* c, std::vector<int32_t> skip) {
  c->untouched_skip = std::move(skip);
  Job j{Job::EMBED_UNTOUCHED_PREV, -1, nullptr, 0};
  j.step = c->untouched_step;
  c->deferred.push_back(j);
  c->untouched_pending = false;
}

// Applies pending deferred updates before the state is read or replaced.
void flush_deferred(mt_ctx* c) {
  if (c->untouched_pending) defer_untouched_rest(c, c->untouched_of);
  if (c->deferred.empty()) return;
  queue_deferred(c);
  wait_jobs(c);
}

// Start of a step with a pending untouched-row update from the last step: the
// rows this step's batch gathers (and later updates) get it first, on every
// host thread, before any GPU work of the step is enqueued; the other rows
// follow in the background. Called with the optimizer idle.
void start_untouched_prev(mt_ctx* c) {
  const Layout& y = c->lay;
  const size_t d = y.sh.d;
  const std::vector<int32_t>& was = c->untouched_of;  // touched by the last step
  std::vector<Seg> first;
  std::vector<int32_t> both;
  both.reserve(was.size() + c->uniq.size());
  std::set_union(was.begin(), was.end(), c->uniq.begin(), c->uniq.end(), std::back_inserter(both));
  for (int32_t r : c->uniq)
    if (!std::binary_search(was.begin(), was.end(), r))
      first.push_back({y.embed.off + (size_t)r * d, d, c->bf_embed + (size_t)r * d, nullptr});
  const double t0 = now_s();
  adamw_segments(c, first, c->untouched_step);
  c->job_times.push_back({7, -1, t0, now_s()});
  defer_untouched_rest(c, std::move(both));
}

// Bounded host wait for the deferred update of layer l (l = L: the LM head)
// queued at the start of this step: its weights are about to be streamed again.
int await_deferred(mt_ctx* c, int l) {
  std::unique_lock<std::mutex> lk(c->opt_mu);
  if (!c->opt_done_cv.wait_for(lk, std::chrono::duration<double>(c->wait_limit_s),
                               [&] { return c->prev_pending[l] == 0; }))
    return set_err(c, MT_ERR_TIMEOUT, "a deferred update did not finish within the wait limit");
  return MT_OK;
}

// ---------------------------------------------------------------------------
// Step.
// ---------------------------------------------------------------------------
int issue_load(mt_ctx* c, int i) {
  const Layout& y = c->lay;
  const int slot = i & 1;
  if (i < y.sh.L && i >= y.sh.L - c->defer_layers) CKM(await_deferred(c, i));  // forward load of a deferred layer
  if (i >= 2) CK(cudaStreamWaitEvent(c->s_h2d, c->ev_slotfree[i - 2], 0));
  CK(cudaEventRecord(c->ev_h2d_start[i], c->s_h2d));
  const uint16_t* src = c->bf_layers + (size_t)c->load_seq[i] * y.bf_layer;
  if (sharded(c)) {  // this rank's part over the host link, the rest from the peers
    const mt_shard& p = c->plan;
    if (p.layer_end > p.layer_begin)
      CK(cudaMemcpyAsync(c->wslot[slot] + p.layer_begin, src + p.layer_begin, (p.layer_end - p.layer_begin) * 2,
                         cudaMemcpyHostToDevice, c->s_h2d));
    NK(AllGather(c->wslot[slot] + (size_t)p.rank * p.layer_chunk, c->wslot[slot], p.layer_chunk, ncclBfloat16,
                 c->comm_h2d, c->s_h2d));
  } else {
    CK(cudaMemcpyAsync(c->wslot[slot], src, y.bf_layer * 2, cudaMemcpyHostToDevice, c->s_h2d));
  }
  CK(cudaEventRecord(c->ev_wready[i], c->s_h2d));
  return MT_OK;
}

// [final gain | LM head] bf16 into the device head block; with tied
// embeddings the head part is the streamed embedding table.
int copy_head_weights(mt_ctx* c, cudaStream_t st) {
  const size_t g = align_up(c->lay.sh.d, 128), n = (size_t)c->lay.sh.V * c->lay.sh.d;
  if (sharded(c)) {  // (on the H2D stream: its communicator)
    const mt_shard& p = c->plan;
    if (p.head_end > p.head_begin)
      CK(cudaMemcpyAsync(c->d_head_w + p.head_begin, c->bf_head + p.head_begin, (p.head_end - p.head_begin) * 2,
                         cudaMemcpyHostToDevice, st));
    NK(AllGather(c->d_head_w + (size_t)p.rank * p.head_chunk, c->d_head_w, p.head_chunk, ncclBfloat16, c->comm_h2d,
                 st));
  } else if (c->lay.tied) {
    CK(cudaMemcpyAsync(c->d_head_w, c->bf_head, g * 2, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(c->d_head_w + g, c->bf_embed, n * 2, cudaMemcpyHostToDevice, st));
  } else {
    CK(cudaMemcpyAsync(c->d_head_w, c->bf_head, (g + n) * 2, cudaMemcpyHostToDevice, st));
  }
  return MT_OK;
}

int issue_head_load(mt_ctx* c) {
  CKM(await_deferred(c, c->lay.sh.L));
  CK(cudaEventRecord(c->ev_head_h2d_start, c->s_h2d));
  CKM(copy_head_weights(c, c->s_h2d));
  CK(cudaEventRecord(c->ev_head_wready, c->s_h2d));
  return MT_OK;
}

// Backward index k (layer l = L-1-k): D2H of the layer's gradients into the
// gradient arena or, in ring mode, into deferred-layer buffer k for the first
// defer_layers indices (their update runs at the next step), else into ring
// slot (k - defer_layers) mod MT_GRAD_RING_SLOTS once the update of backward
// index k - MT_GRAD_RING_SLOTS (the slot's previous user) is done: the layer
// jobs finish in backward order, so that is when layer_jobs_done passes it.
int offload_layer(mt_ctx* c, int l, int k) {
  const Layout& y = c->lay;
  const size_t b = y.layer_begin(l), e = y.layer_end(l), gsz = c->gsz;
  const int nd = c->defer_layers;
  uint8_t* dst = c->grad ? c->grad + b * gsz
                 : k < nd ? c->defer_g + (size_t)k * c->layer_f * gsz
                          : c->ring + (size_t)((k - nd) % MT_GRAD_RING_SLOTS) * c->layer_f * gsz;
  if (!c->grad && k >= nd + MT_GRAD_RING_SLOTS) {
    std::unique_lock<std::mutex> lk(c->opt_mu);
    const int need = k - MT_GRAD_RING_SLOTS + 1;
    if (!c->opt_done_cv.wait_for(lk, std::chrono::duration<double>(c->wait_limit_s),
                                 [&] { return c->layer_jobs_done >= need; }))
      return set_err(c, MT_ERR_TIMEOUT, "gradient ring: no slot was released within the wait limit");
  }
  const void* src = c->gslot[k & 1];
  if (gsz == 2) {  // bf16 offload: round the checked fp32 gradients on the GPU (RNE)
    KL(launch_cast_f32_bf16(c->gslot[k & 1], c->gslot16[k & 1], (int64_t)(e - b), c->s_comp), 1);
    src = c->gslot16[k & 1];
  }
  // the part of the block that crosses the link: all of it, or this rank's own
  const size_t ob = sharded(c) ? c->plan.layer_begin : 0;
  const size_t on = sharded(c) ? c->plan.layer_end - c->plan.layer_begin : e - b;
  CK(cudaEventRecord(c->ev_gready[k], c->s_comp));
  CK(cudaStreamWaitEvent(c->s_d2h, c->ev_gready[k], 0));
  CK(cudaEventRecord(c->ev_d2h_start[k], c->s_d2h));
  if (on > 0)
    CK(cudaMemcpyAsync(dst + ob * gsz, static_cast<const uint8_t*>(src) + ob * gsz, on * gsz, cudaMemcpyDeviceToHost,
                       c->s_d2h));
  CK(cudaMemcpyAsync(c->flags_h + l, c->d_flags + l, 4, cudaMemcpyDeviceToHost, c->s_d2h));
  CK(cudaEventRecord(c->ev_gdrained[k], c->s_d2h));
  Job j{Job::LAYER, l, c->ev_gdrained[k], l, dst};
  j.defer = k < nd;
  push_job(c, j);
  return MT_OK;
}

// MT_FLAG_OFFLOAD_ACTS, forward: x_l (just written on the compute stream)
// leaves the slot that x_{l+2} takes: to host memory for l <= L-3, by a device
// copy into slot 2 for l = L-2 (the first layer recomputed). ev_xout[l]: done.
int stash_act(mt_ctx* c, int l) {
  const int L = c->lay.sh.L;
  if (!offload_acts(c) || l > L - 2) return MT_OK;
  const size_t n = (size_t)c->lay.sh.T * c->lay.sh.d;
  CK(cudaEventRecord(c->ev_xready[l], c->s_comp));
  CK(cudaStreamWaitEvent(c->s_act, c->ev_xready[l], 0));
  if (l == L - 2)
    CK(cudaMemcpyAsync(x_bwd(c, l), x_fwd(c, l), n * 4, cudaMemcpyDeviceToDevice, c->s_act));
  else
    CK(cudaMemcpyAsync(c->xh + (size_t)l * n, x_fwd(c, l), n * 4, cudaMemcpyDeviceToHost, c->s_act));
  CK(cudaEventRecord(c->ev_xout[l], c->s_act));
  return MT_OK;
}

// Backward: x_l (l <= L-3) back from host memory into its backward slot, once
// the slot's last user, layer l+2's backward, is done. ev_xin[l]: landed.
int fetch_act(mt_ctx* c, int l) {
  const int L = c->lay.sh.L;
  if (!offload_acts(c) || l < 0 || l > L - 3) return MT_OK;
  const size_t n = (size_t)c->lay.sh.T * c->lay.sh.d;
  CK(cudaStreamWaitEvent(c->s_act, c->ev_bwdone[l + 2], 0));
  CK(cudaMemcpyAsync(x_bwd(c, l), c->xh + (size_t)l * n, n * 4, cudaMemcpyHostToDevice, c->s_act));
  CK(cudaEventRecord(c->ev_xin[l], c->s_act));
  return MT_OK;
}

// MT_FLAG_POISON: gradient slot k & 1 filled with NaN before backward index
// k writes it (its previous contents have drained to the host).
int poison_grad(mt_ctx* c, int k) {
  if (!(c->cfg.flags & MT_FLAG_POISON)) return MT_OK;
  CK(cudaMemsetAsync(c->gslot[k & 1], 0xFF, c->layer_f * 4, c->s_comp));
  return MT_OK;
}

int enqueue_step(mt_ctx* c, int n_unique) {
  const Layout& y = c->lay;
  const Shapes& s = y.sh;
  const int L = s.L, T = s.T, d = s.d;
  const int nloads = (int)c->load_seq.size();
  cudaStream_t sc = c->s_comp;

  CK(cudaEventRecord(c->ev_step_start, sc));
  CK(cudaMemsetAsync(c->d_err, 0, sizeof(int32_t), sc));  // error word of this step's kernels
  CK(cudaMemcpyAsync(c->d_tok, c->stage_i, (size_t)(5 * T + 1) * 4, cudaMemcpyHostToDevice, sc));
  if (sharded(c)) {
    // The embedding table lives on the device: this rank's rows (updated on
    // the host in the last step) over the link, the rest from the peers.
    const mt_shard& p = c->plan;
    const size_t rows = embed_rows_chunk(p, s.V), rb = (size_t)p.embed_row_begin, re = (size_t)p.embed_row_end;
    if (re > rb)
      CK(cudaMemcpyAsync(c->d_embed_w + rb * d, c->bf_embed + rb * d, (re - rb) * d * 2, cudaMemcpyHostToDevice,
                         c->s_h2d));
    NK(AllGather(c->d_embed_w + (size_t)p.rank * rows * d, c->d_embed_w, rows * d, ncclBfloat16, c->comm_h2d,
                 c->s_h2d));
    CK(cudaEventRecord(c->ev_embw, c->s_h2d));
    CK(cudaStreamWaitEvent(sc, c->ev_embw, 0));
  }
  KL(launch_embed_fwd(c->d_tok, sharded(c) ? c->d_embed_w : c->bf_embed_dev, x_fwd(c, 0), T, d, sc), 1);
  CKM(stash_act(c, 0));
  CKM(issue_load(c, 0));
  if (nloads > 1) CKM(issue_load(c, 1));
  if (L == 1) CKM(issue_head_load(c));

  float* gin = c->gx0;
  float* gout = c->gx1;
  for (int i = 0; i < nloads; ++i) {
    const int slot = i & 1;
    CK(cudaEventRecord(c->ev_compready[i], sc));
    CK(cudaStreamWaitEvent(sc, c->ev_wready[i], 0));
    if (i < L) {
      const int l = i;
      // with offloaded activations x_{l+1} takes the slot of x_{l-1}
      if (offload_acts(c) && l >= 1) CK(cudaStreamWaitEvent(sc, c->ev_xout[l - 1], 0));
      CKM(layer_fwd(c, l, slot, x_fwd(c, l), x_fwd(c, l + 1)));
      CKM(stash_act(c, l + 1));
      if (l == L - 1) {
        CK(cudaEventRecord(c->ev_fwd_end, sc));
        CK(cudaStreamWaitEvent(sc, c->ev_head_wready, 0));
        CKM(head_step(c, gin));
        const size_t n = y.head_block;
        const void* hsrc = c->d_head_g;
        if (c->gsz == 2) {
          KL(launch_cast_f32_bf16(c->d_head_g, c->d_head_g16, (int64_t)n, sc), 1);
          hsrc = c->d_head_g16;
        }
        CK(cudaEventRecord(c->ev_head_gready, sc));
        CK(cudaStreamWaitEvent(c->s_d2h, c->ev_head_gready, 0));
        CK(cudaEventRecord(c->ev_head_d2h_start, c->s_d2h));
        const size_t hb = sharded(c) ? c->plan.head_begin : 0, he = sharded(c) ? c->plan.head_end : n;
        if (he > hb)
          CK(cudaMemcpyAsync(c->grad_head + hb * c->gsz, static_cast<const uint8_t*>(hsrc) + hb * c->gsz,
                             (he - hb) * c->gsz, cudaMemcpyDeviceToHost, c->s_d2h));
        CK(cudaMemcpyAsync(c->flags_h + L, c->d_flags + L, 4, cudaMemcpyDeviceToHost, c->s_d2h));
        CK(cudaEventRecord(c->ev_head_drained, c->s_d2h));
        Job hj{Job::HEAD, -1, c->ev_head_drained, L};
        hj.defer = (c->cfg.flags & MT_FLAG_DEFER_UPDATES) && !(c->cfg.flags & MT_FLAG_NO_UPDATE);
        push_job(c, hj);
        CK(cudaEventRecord(c->ev_head_end, sc));
        // backward of the last layer: its intermediates are still in the workspace
        CKM(poison_grad(c, 0));
        CKM(layer_bwd(c, l, slot, x_bwd(c, l), c->gslot[0], gin, gout));
        CKM(offload_layer(c, l, 0));
        std::swap(gin, gout);
        if (offload_acts(c)) {
          CK(cudaEventRecord(c->ev_bwdone[l], sc));
          CKM(fetch_act(c, l - 2));
        }
      }
    } else {
      const int k = i - (L - 1);  // backward index: layer L-1-k
      const int l = L - 1 - k;
      if (k >= 2) CK(cudaStreamWaitEvent(sc, c->ev_gdrained[k - 2], 0));
      CKM(poison_grad(c, k));
      if (offload_acts(c)) CK(cudaStreamWaitEvent(sc, l == L - 2 ? c->ev_xout[l] : c->ev_xin[l], 0));
      CKM(layer_fwd(c, l, slot, x_bwd(c, l), nullptr));
      CKM(layer_bwd(c, l, slot, x_bwd(c, l), c->gslot[k & 1], gin, gout));
      CKM(offload_layer(c, l, k));
      std::swap(gin, gout);
      if (offload_acts(c)) {
        CK(cudaEventRecord(c->ev_bwdone[l], sc));
        CKM(fetch_act(c, l - 2));
      }
    }
    if (c->cfg.flags & MT_FLAG_POISON) CK(cudaMemsetAsync(c->wslot[slot], 0xFF, c->wslot_bytes, sc));
    CK(cudaEventRecord(c->ev_slotfree[i], sc));
    // The head's weights follow the last forward load on the H2D stream, ahead
    // of the first backward load. Issued here, after layer L-2's forward is
    // queued, a wait for its deferred update holds back no forward layer but
    // the last one.
    if (i + 2 == L) CKM(issue_head_load(c));
    if (i + 2 < nloads) CKM(issue_load(c, i + 2));
  }
  CK(cudaEventRecord(c->ev_bwd_end, sc));
  // embedding gradient rows, in token order per unique id
  KL(launch_embed_bwd(c->d_offs, c->d_pos, n_unique, gin, c->tmp_f, d, sc), 1);
  if (sharded(c)) {
    // dense [world * rows, d] gradient, averaged over the ranks by rows
    const mt_shard& p = c->plan;
    const size_t rows = embed_rows_chunk(p, s.V), rb = (size_t)p.embed_row_begin, re = (size_t)p.embed_row_end;
    CK(cudaMemsetAsync(c->d_embed_g, 0, (size_t)p.world * rows * d * 4, sc));
    if (n_unique > 0) {
      k_scatter_rows<<<std::min(n_unique, 1184), 128, 0, sc>>>(c->tmp_f, c->d_uid, n_unique, c->d_embed_g, d);
      CK(cudaGetLastError());
      c->launches += 1;
    }
    if (y.tied) {  // the table's gradient is also the head's: add it before the ranks' mean
      const size_t n = (size_t)s.V * d;
      k_add_f32<<<(unsigned)std::min<size_t>((n / 4 + 255) / 256, 148 * 16), 256, 0, sc>>>(
          c->d_embed_g, c->d_head_g + c->head_g_split, n);
      CK(cudaGetLastError());
      c->launches += 1;
    }
    CKM(reduce_own_chunk(c, c->d_embed_g, rows * d, rb * d, re * d, L + 1));
    CK(cudaEventRecord(c->ev_emb_ready, sc));
    CK(cudaStreamWaitEvent(c->s_d2h, c->ev_emb_ready, 0));
    CK(cudaEventRecord(c->ev_emb_d2h_start, c->s_d2h));
    if (re > rb)
      CK(cudaMemcpyAsync(c->emb_own_h, c->d_embed_g + rb * d, (re - rb) * d * 4, cudaMemcpyDeviceToHost, c->s_d2h));
    CK(cudaMemcpyAsync(c->flags_h + L + 1, c->d_flags + L + 1, 4, cudaMemcpyDeviceToHost, c->s_d2h));
  } else {
    CK(cudaEventRecord(c->ev_emb_ready, sc));
    CK(cudaStreamWaitEvent(c->s_d2h, c->ev_emb_ready, 0));
    CK(cudaEventRecord(c->ev_emb_d2h_start, c->s_d2h));
    CK(cudaMemcpyAsync(c->emb_rows_h, c->tmp_f, (size_t)n_unique * d * 4, cudaMemcpyDeviceToHost, c->s_d2h));
    c->flags_h[L + 1] = 0;  // set by the host's own check of the rows
  }
  CK(cudaMemcpyAsync(c->misc_h + 2, c->d_err, 4, cudaMemcpyDeviceToHost, c->s_d2h));
  CK(cudaEventRecord(c->ev_emb_drained, c->s_d2h));
  push_job(c, Job{Job::EMBED, -1, c->ev_emb_drained, L + 1});
  // Without deferral the untouched rows' update follows the step's last check.
  // (tied embeddings: every row has a head gradient, so the EMBED job updates
  // them all; sharded: the EMBED job's dense rows include them)
  if (!(c->cfg.flags & MT_FLAG_DEFER_UPDATES) && !y.tied && !sharded(c))
    push_job(c, Job{Job::EMBED_UNTOUCHED, -1, nullptr, L + 1});
  CK(cudaMemcpyAsync(c->misc_h, c->d_loss, 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaMemcpyAsync(c->misc_h + 1, c->d_err, 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaEventRecord(c->ev_step_end, sc));
  return MT_OK;
}

float ev_ms(cudaEvent_t a, cudaEvent_t b) {
  float ms = 0.f;
  if (cudaEventElapsedTime(&ms, a, b) != cudaSuccess) return 0.f;
  return ms;
}

void collect_stats(mt_ctx* c) {
  mt_stats& st = c->stats;
  const int L = c->lay.sh.L;
  st.step_ms = ev_ms(c->ev_step_start, c->ev_step_end);
  st.fwd_ms = ev_ms(c->ev_step_start, c->ev_fwd_end);
  st.head_ms = ev_ms(c->ev_fwd_end, c->ev_head_end);
  st.bwd_ms = ev_ms(c->ev_head_end, c->ev_bwd_end);
  double h2d = ev_ms(c->ev_head_h2d_start, c->ev_head_wready), wait = 0;
  for (size_t i = 0; i < c->load_seq.size(); ++i) {
    h2d += ev_ms(c->ev_h2d_start[i], c->ev_wready[i]);
    const float w = ev_ms(c->ev_compready[i], c->ev_wready[i]);
    if (w > 0) wait += w;
  }
  double d2h = ev_ms(c->ev_head_d2h_start, c->ev_head_drained) + ev_ms(c->ev_emb_d2h_start, c->ev_emb_drained);
  for (int k = 0; k < L; ++k) d2h += ev_ms(c->ev_d2h_start[k], c->ev_gdrained[k]);
  st.h2d_ms = h2d;
  st.d2h_ms = d2h;
  st.wait_weights_ms = wait;
  const Layout& y = c->lay;
  const double act_bytes = offload_acts(c) && L >= 3 ? 4.0 * (L - 2) * y.sh.T * y.sh.d : 0.0;
  if (sharded(c)) {  // this rank's parts only; the rest crosses NVLink
    const mt_shard& p = c->plan;
    const double lay = (double)(p.layer_end - p.layer_begin), head = (double)(p.head_end - p.head_begin);
    const double rows = (double)(p.embed_row_end - p.embed_row_begin) * y.sh.d;
    st.h2d_bytes = act_bytes + (double)c->load_seq.size() * lay * 2 + head * 2 + rows * 2 + 4.0 * (5 * y.sh.T + 1);
    st.d2h_bytes = act_bytes + 4.0 * (head + rows + (double)L * lay) + 4.0 * (L + 4);
  } else {
    st.h2d_bytes = act_bytes + (double)c->load_seq.size() * y.bf_layer * 2 +
                   (double)(align_up(y.sh.d, 128) + (size_t)y.sh.V * y.sh.d) * 2 + 4.0 * (5 * y.sh.T + 1) +
                   (double)y.sh.T * y.sh.d * 2;  // embedding rows read in place
    st.d2h_bytes = act_bytes + (double)c->gsz * y.head_block + 4.0 * c->uniq.size() * y.sh.d + 12.0;
    for (int l = 0; l < L; ++l) st.d2h_bytes += (double)c->gsz * (y.layer_end(l) - y.layer_begin(l));
  }
  if (y.sh.E > 0) {  // each layer's expert choices out and its row layout back, once per step
    const double tk = (double)y.sh.T * y.sh.topk;
    st.d2h_bytes += 4.0 * L * tk;
    st.h2d_bytes += 8.0 * L * tk;
  }
  st.adamw_ms = c->adamw_s * 1e3;
  st.adamw_bytes = c->adamw_bytes;
  st.gemm_flops = st.gemm_ms = st.attn_flops = st.attn_ms = 0;
  st.gemm_launches = st.attn_launches = 0;
  for (const auto& t : c->timed) {
    const double ms = ev_ms(t.a, t.b);
    if (t.kind == 0) {
      st.gemm_flops += t.flops;
      st.gemm_ms += ms;
      st.gemm_launches++;
    } else {
      st.attn_flops += t.flops;
      st.attn_ms += ms;
      st.attn_launches++;
    }
  }
  st.kernel_launches = c->launches;
}

// ---------------------------------------------------------------------------
// Create / destroy helpers.
// ---------------------------------------------------------------------------
// Elements of a device weight / gradient slot and of the device head block:
// the blocks themselves, or padded to world * chunk when sharded.
size_t slot_elems(const Layout& y, const mt_shard* p) {
  return p ? (size_t)p->world * p->layer_chunk : y.bf_layer;
}
size_t gslot_elems(const Layout& y, const mt_shard* p) {
  return p ? (size_t)p->world * p->layer_chunk : y.layer_end(0) - y.layer_begin(0);
}
size_t head_w_elems(const Layout& y, const mt_shard* p) {
  return p ? (size_t)p->world * p->head_chunk : align_up(y.sh.d, 128) + (size_t)y.sh.V * y.sh.d;
}
size_t head_g_split(const Layout& y, const mt_shard* p) {
  return (p && y.tied) ? std::max(y.gf_pad, (size_t)p->world * p->head_chunk) : y.gf_pad;
}
size_t head_g_elems(const Layout& y, const mt_shard* p) {
  if (p && y.tied) return head_g_split(y, p) + (size_t)y.sh.V * y.sh.d;  // [gain, padded | table gradient]
  return p ? (size_t)p->world * p->head_chunk : y.head_block;
}

size_t device_bytes(const Layout& y, int Tc, uint32_t flags, const mt_shard* plan = nullptr) {
  const bool g16 = (flags & MT_FLAG_BF16_GRADS) != 0, offload = (flags & MT_FLAG_OFFLOAD_ACTS) != 0;
  const size_t n_attn = (flags & MT_FLAG_STASH_ATTN) ? (size_t)y.sh.L : 1;  // O / LSE buffers
  const Shapes& s = y.sh;
  const size_t T = s.T, d = s.d, F = s.F, V = s.V;
  const size_t A = 256;
  size_t b = 0;
  auto add = [&](size_t bytes) { b += align_up(bytes, A); };
  add(slot_elems(y, plan) * 2);
  add(slot_elems(y, plan) * 2);
  const size_t lay_f = y.layer_end(0) - y.layer_begin(0);
  add(gslot_elems(y, plan) * 4);
  add(gslot_elems(y, plan) * 4);
  add(head_w_elems(y, plan) * 2);                           // head weights (or the tied table)
  add(head_g_elems(y, plan) * 4);                           // head grads
  if (plan) {                                               // embedding table and its dense gradient
    add((size_t)plan->world * embed_rows_chunk(*plan, s.V) * d * 2);
    add((size_t)plan->world * embed_rows_chunk(*plan, s.V) * d * 4);
  }
  if (g16) {                                                // bf16 offload copies
    add(lay_f * 2);
    add(lay_f * 2);
    add(y.head_block * 2);
  }
  add((size_t)(offload ? std::min(s.L + 1, 3) : s.L + 1) * T * d * 4);  // boundary activations
  add(T * d * 2);                                           // u
  add(T * (size_t)s.Nqkv * 2);                              // qkv
  add(n_attn * T * (size_t)s.Hd * 2);                       // attention output
  add(n_attn * s.b * s.H * (size_t)s.s * 4);                // lse
  add(T * d * 4);                                           // h
  add(T * 4);                                               // r1
  add(T * 4);                                               // r2
  add(T * d * 2);                                           // w
  const size_t R = s.E > 0 ? std::max(T, T * (size_t)s.topk) : T;  // MLP rows (routed rows with experts)
  add(R * 2 * F * 2);                                       // gate|up
  add(R * F * 2);                                           // act
  add(T * d * 4);                                           // gx0
  add(T * d * 4);                                           // gx1
  add(T * d * 2);                                           // gxb
  add(R * F * 2);                                           // dact
  add(R * 2 * F * 2);                                       // dgu
  if (s.E > 0) {
    const size_t Tk = T * (size_t)s.topk, E = s.E;
    add(T * E * 4);                  // logits
    add(T * E * 4);                  // dlogits
    add(Tk * 4);                     // idx
    add(Tk * 4);                     // gate
    add(Tk * 4);                     // dgate
    add((size_t)s.L * Tk * 4 * 2);   // slot_of, row_of per layer
    add(Tk * d * 2);                 // xe
    add(Tk * d * 2);                 // dye
    add(Tk * d * 4);                 // ye
    add(Tk * d * 4);                 // dxe
  }
  add(T * d * 4);                                           // tmp_f
  add(T * d * 4);                                           // dh
  add(T * d * 2);                                           // dhb
  add(T * (size_t)s.Hd * 2);                                // dao
  add((size_t)s.b * s.H * s.s * 4);                         // dvec
  add(T * (size_t)s.Hd * 4);                                // dq accumulator
  add(T * (size_t)s.Nqkv * 2);                              // dqkv
  add((size_t)rmsnorm_bwd_blocks((int)T) * d * 4);          // RMSNorm partials
  add(T * d * 2);                                           // n
  add(T * 4);                                               // rf
  add((size_t)Tc * V * 4);                                  // logits
  add((size_t)Tc * V * 2);                                  // dz
  add(T * 4);                                               // row loss
  add((5 * T + 1) * 4);                                     // tokens, labels, offs, pos, unique ids
  add((size_t)(s.L + 2) * 4);                               // flags
  add(4);                                                   // error word
  add((size_t)s.s * (s.hd / 2) * 4 * 2);                    // cos, sin
  add(4);                                                   // loss
  return b + 4096;
}

// Tokens per LM-head chunk: at most ~4 GiB of fp32 logits + bf16 dz, a
// multiple of 128 tokens; MT_LOGITS_CHUNK may ask for smaller chunks.
int logits_chunk(const Shapes& s) {
  int Tc = (int)std::min<int64_t>(s.T, ((int64_t)1 << 32) / ((int64_t)s.V * 6));
  if (Tc < s.T) Tc = std::max(128, Tc / 128 * 128);
  if (const char* e = getenv("MT_LOGITS_CHUNK")) {
    const int want = atoi(e);
    if (want >= 128 && want % 128 == 0 && want < Tc) Tc = want;
  }
  return Tc;
}

constexpr size_t kHugePage = size_t(2) << 20;

// Host memory on transparent huge pages where the host allows them (the
// advice is given before the first touch). The host optimizer streams the
// master, both moments, the gradient and the bf16 copy of every parameter,
// and 2 MB pages cut its TLB misses: the AdamW routine alone measured 160
// GB/s on 4 KB pages and 174 GB/s on 2 MB pages of a B200 host. The range
// starts on a 2 MB boundary and its pages are zero. nullptr if out of memory.
void* huge_alloc(mt_ctx* c, size_t bytes) {
  const size_t len = align_up(std::max<size_t>(bytes, 1), kHugePage);
  void* got = mmap(nullptr, len + kHugePage, PROT_READ | PROT_WRITE, MAP_PRIVATE | MAP_ANONYMOUS, -1, 0);
  if (got == MAP_FAILED) return nullptr;
  uint8_t* raw = static_cast<uint8_t*>(got);
  uint8_t* p = reinterpret_cast<uint8_t*>(align_up(reinterpret_cast<uintptr_t>(raw), kHugePage));
  if (p > raw) munmap(raw, (size_t)(p - raw));
  const size_t tail = (size_t)((raw + len + kHugePage) - (p + len));
  if (tail) munmap(p + len, tail);
  madvise(p, len, MADV_HUGEPAGE);  // advice only: without huge pages the range keeps 4 KB pages
  c->huge_bufs.push_back({p, len});
  return p;
}

// huge_alloc, faulted in by the worker pool and registered (pinned) for the
// copy engines; mapped: also addressable from the device (its alias from
// cudaHostGetDevicePointer). nullptr if the allocation or the pinning fails.
void* huge_alloc_pinned(mt_ctx* c, size_t bytes, bool mapped) {
  uint8_t* p = static_cast<uint8_t*>(huge_alloc(c, bytes));
  if (!p) return nullptr;
  const size_t len = c->huge_bufs.back().second;
  parallel_ranges(*c->pool, len / 4096, [&](size_t b, size_t e) {
    for (size_t i = b; i < e; ++i) p[i * 4096] = 0;
  });
  if (cudaHostRegister(p, len, cudaHostRegisterPortable | (mapped ? cudaHostRegisterMapped : 0)) != cudaSuccess)
    return nullptr;
  c->huge_pinned.push_back(p);
  return p;
}

void free_all(mt_ctx* c) {
  if (!c) return;
  if (c->opt_thread.joinable()) {
    {
      std::lock_guard<std::mutex> lk(c->opt_mu);
      c->opt_stop = true;
    }
    c->opt_cv.notify_all();
    c->opt_thread.join();
  }
  cudaSetDevice(c->device);
  for (cudaStream_t s : {c->s_h2d, c->s_comp, c->s_d2h, c->s_act})
    if (s) cudaStreamSynchronize(s);
  auto kill = [](std::vector<cudaEvent_t>& v) {
    for (auto e : v)
      if (e) cudaEventDestroy(e);
    v.clear();
  };
  kill(c->ev_wready);
  kill(c->ev_compready);
  kill(c->ev_h2d_start);
  kill(c->ev_slotfree);
  kill(c->ev_gready);
  kill(c->ev_d2h_start);
  kill(c->ev_gdrained);
  kill(c->ev_timing);
  kill(c->ev_xready);
  kill(c->ev_xout);
  kill(c->ev_xin);
  kill(c->ev_bwdone);
  for (cudaEvent_t e : {c->ev_head_h2d_start, c->ev_head_wready, c->ev_head_gready, c->ev_head_d2h_start,
                        c->ev_head_drained, c->ev_emb_ready, c->ev_emb_d2h_start, c->ev_emb_drained,
                        c->ev_step_start, c->ev_fwd_end, c->ev_head_end, c->ev_bwd_end, c->ev_step_end})
    if (e) cudaEventDestroy(e);
  if (c->ev_embw) cudaEventDestroy(c->ev_embw);
  if (c->ev_route) cudaEventDestroy(c->ev_route);
  if (c->comm_h2d) c->nccl->CommDestroy(c->comm_h2d);
  if (c->comm_comp) c->nccl->CommDestroy(c->comm_comp);
  // In serialized mode the three handles are one stream: destroy each once.
  if (c->s_comp) cudaStreamDestroy(c->s_comp);
  if (c->s_h2d && c->s_h2d != c->s_comp) cudaStreamDestroy(c->s_h2d);
  if (c->s_d2h && c->s_d2h != c->s_comp && c->s_d2h != c->s_h2d) cudaStreamDestroy(c->s_d2h);
  if (c->s_act && c->s_act != c->s_comp) cudaStreamDestroy(c->s_act);
  if (c->dmem) cudaFree(c->dmem);
  for (void* p : {(void*)c->emb_rows_h, (void*)c->stage_i, (void*)c->flags_h, (void*)c->misc_h, (void*)c->xh,
                  (void*)c->emb_own_h, (void*)c->moe_idx_h, (void*)c->moe_route_h})
    if (p) cudaFreeHost(p);
  for (void* p : c->huge_pinned) cudaHostUnregister(p);
  for (const auto& b : c->huge_bufs) munmap(b.first, b.second);
  delete c->pool;
  delete c;
}

// world == 0: an unsharded context; else rank `rank` of a sharded one whose
// NCCL unique id is `id`.
int create_impl(const mt_config* cfg, float* arena, size_t arena_bytes, mt_ctx** out, int world = 0, int rank = 0,
                const void* id = nullptr) {
  mt_ctx* c = nullptr;
  std::string why;
  int r = validate_config(cfg, &why);
  if (r != MT_OK) return set_err(nullptr, r, why);
  if (!out) return set_err(nullptr, MT_ERR_ARG, "out is NULL");
  *out = nullptr;
  Layout y = make_layout(*cfg);
  const Shapes& s = y.sh;
  mt_shard plan{};
  const NcclApi* nccl = nullptr;
  if (world > 0) {
    if (!id) return set_err(nullptr, MT_ERR_ARG, "sharded context without an NCCL id");
    r = mt_shard_plan(cfg, world, rank, &plan);
    if (r != MT_OK) return set_err(nullptr, r, "no shard plan for this config (d must be a multiple of 128)");
    nccl = nccl_api(&why);
    if (!nccl) return set_err(nullptr, MT_ERR_CUDA, why);
  }
  if (arena) {
    if (arena_bytes < y.total * 4) return set_err(nullptr, MT_ERR_ARENA, "arena smaller than mt_arena_bytes(cfg)");
    if (reinterpret_cast<uintptr_t>(arena) & 255) return set_err(nullptr, MT_ERR_ARENA, "arena not 256-byte aligned");
  }
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || cfg->device < 0 || cfg->device >= ndev)
    return set_err(nullptr, MT_ERR_CUDA, "no such CUDA device");
  if (cudaSetDevice(cfg->device) != cudaSuccess) return set_err(nullptr, MT_ERR_CUDA, "cudaSetDevice failed");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, cfg->device);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, cfg->device);
  if (major != 10 || minor != 0) return set_err(nullptr, MT_ERR_CUDA, "this library runs on sm_100 (B200) only");

  const int Tc = logits_chunk(s);
  const size_t need = device_bytes(y, Tc, cfg->flags, world > 0 ? &plan : nullptr);
  size_t free_b = 0, total_b = 0;
  if (cudaMemGetInfo(&free_b, &total_b) != cudaSuccess) return set_err(nullptr, MT_ERR_CUDA, "cudaMemGetInfo failed");
  if (need + ((size_t)256 << 20) > free_b) {
    char m[160];
    snprintf(m, sizeof m, "device budget: need %.2f GB, %.2f GB free", need / 1e9, free_b / 1e9);
    return set_err(nullptr, MT_ERR_NOMEM, m);
  }

  c = new mt_ctx();
  c->cfg = *cfg;
  c->lay = y;
  c->plan = plan;
  c->head_g_split = head_g_split(y, world > 0 ? &plan : nullptr);
  c->nccl = nccl;
  c->device = cfg->device;
  c->Tc = Tc;
  c->gsz = (cfg->flags & MT_FLAG_BF16_GRADS) ? 2 : 4;
  const size_t gsz = c->gsz;
  int nthreads = cfg->host_threads;
  if (nthreads <= 0) nthreads = std::max(1, (int)std::thread::hardware_concurrency() - 1);
  c->pool = new ThreadPool(nthreads - 1);

  // host memory
  auto fail = [&](int code, const std::string& m) {
    g_create_error = m;
    free_all(c);
    return code;
  };
  if (arena) {
    c->arena = arena;
  } else {
    c->arena = static_cast<float*>(huge_alloc(c, y.total * 4));
    if (!c->arena) return fail(MT_ERR_NOMEM, "arena alloc");
    c->arena_owned = true;
  }
  c->m = static_cast<float*>(huge_alloc(c, y.total * 4));
  c->v = static_cast<float*>(huge_alloc(c, y.total * 4));
  if (!c->m || !c->v) return fail(MT_ERR_NOMEM, "host moment allocation failed");
  const size_t head_bf = align_up(s.d, 128) + (y.tied ? 0 : (size_t)s.V * s.d);  // host bf16 head block
  const size_t head_f = y.head_block;
  c->layer_f = y.layer_end(0) - y.layer_begin(0);
  for (int l = 1; l < s.L; ++l)
    if (y.layer_end(l) - y.layer_begin(l) != c->layer_f) return fail(MT_ERR_CONFIG, "layer blocks differ in size");
  c->defer_layers = defer_layer_count(*cfg);
  c->prev_pending.assign((size_t)s.L + 1, 0);
  c->overlap_threads = std::max(1, c->pool->size() / 2);
  if (const char* e = getenv("MT_OVERLAP_THREADS")) {
    const int n = atoi(e);
    if (n > 0) c->overlap_threads = std::min(n, c->pool->size());
  }
  if (cfg->flags & MT_FLAG_GRAD_RING) {
    c->ring = static_cast<uint8_t*>(huge_alloc_pinned(c, (size_t)MT_GRAD_RING_SLOTS * c->layer_f * gsz, false));
    c->grad_head = c->ring ? static_cast<uint8_t*>(huge_alloc_pinned(c, head_f * gsz, false)) : nullptr;
    if (!c->ring || !c->grad_head) return fail(MT_ERR_PIN, "pinned gradient ring allocation failed");
    if (c->defer_layers > 0 &&
        !(c->defer_g = static_cast<uint8_t*>(huge_alloc_pinned(c, (size_t)c->defer_layers * c->layer_f * gsz, false))))
      return fail(MT_ERR_PIN, "pinned deferred-layer gradient allocation failed");
  } else {
    if (!(c->grad = static_cast<uint8_t*>(huge_alloc_pinned(c, y.total * gsz, false))))
      return fail(MT_ERR_PIN, "pinned gradient arena allocation failed");
    if (y.tied) {  // the arena has no LM-head tensor: the head's gradient block is separate
      if (!(c->grad_head = static_cast<uint8_t*>(huge_alloc_pinned(c, head_f * gsz, false))))
        return fail(MT_ERR_PIN, "pinned head-gradient allocation failed");
    } else {
      c->grad_head = c->grad + y.final_norm.off * gsz;
    }
  }
  c->grad_head_owned = (cfg->flags & MT_FLAG_GRAD_RING) || y.tied;
  c->bf_layers = static_cast<uint16_t*>(huge_alloc_pinned(c, (size_t)s.L * y.bf_layer * 2, false));
  c->bf_embed = c->bf_layers ? static_cast<uint16_t*>(huge_alloc_pinned(c, (size_t)s.V * s.d * 2, true)) : nullptr;
  c->bf_head = c->bf_embed ? static_cast<uint16_t*>(huge_alloc_pinned(c, head_bf * 2, false)) : nullptr;
  if (!c->bf_head ||
      cudaHostAlloc(reinterpret_cast<void**>(&c->emb_rows_h), (size_t)s.T * s.d * 4, cudaHostAllocPortable) !=
          cudaSuccess ||
      cudaHostAlloc(reinterpret_cast<void**>(&c->stage_i), (size_t)(5 * s.T + 1) * 4, cudaHostAllocPortable) !=
          cudaSuccess ||
      cudaHostAlloc(reinterpret_cast<void**>(&c->flags_h), (size_t)(s.L + 2) * 4, cudaHostAllocPortable) !=
          cudaSuccess ||
      cudaHostAlloc(reinterpret_cast<void**>(&c->misc_h), 64, cudaHostAllocPortable) != cudaSuccess)
    return fail(MT_ERR_PIN, "pinned host allocation failed");
  if (cudaHostGetDevicePointer(reinterpret_cast<void**>(&c->bf_embed_dev), c->bf_embed, 0) != cudaSuccess)
    return fail(MT_ERR_PIN, "embedding table not mapped for device access");
  if (world > 0 &&
      cudaHostAlloc(reinterpret_cast<void**>(&c->emb_own_h),
                    std::max<size_t>(1, embed_rows_chunk(plan, s.V)) * s.d * 4, cudaHostAllocPortable) != cudaSuccess)
    return fail(MT_ERR_PIN, "pinned embedding-row allocation failed");
  if (s.E > 0) {
    const size_t Tk = (size_t)s.T * s.topk;
    if (cudaHostAlloc(reinterpret_cast<void**>(&c->moe_idx_h), (size_t)s.L * Tk * 4, cudaHostAllocPortable) !=
            cudaSuccess ||
        cudaHostAlloc(reinterpret_cast<void**>(&c->moe_route_h), (size_t)s.L * Tk * 2 * 4, cudaHostAllocPortable) !=
            cudaSuccess)
      return fail(MT_ERR_PIN, "pinned routing allocation failed");
    c->moe_count.assign(s.L, std::vector<int>(s.E, 0));
  }
  if ((cfg->flags & MT_FLAG_OFFLOAD_ACTS) && s.L >= 3 &&
      cudaHostAlloc(reinterpret_cast<void**>(&c->xh), (size_t)(s.L - 2) * s.T * s.d * 4, cudaHostAllocPortable) !=
          cudaSuccess)
    return fail(MT_ERR_PIN, "pinned boundary-activation allocation failed");
  // Initialise (owned arena from seed), zero moments and gradients (parallel first touch).
  if (c->arena_owned) {
    auto fill = [&](const TRef& r, uint64_t key, bool gain) {
      parallel_ranges(*c->pool, r.n, [&](size_t b, size_t e) {
        for (size_t i = b; i < e; ++i) c->arena[r.off + i] = gain ? 1.f : 0.02f * normal_at(key, i);
      });
    };
    const uint64_t seed = splitmix64(cfg->seed);
    fill(y.embed, seed ^ 0x1000, false);
    for (int l = 0; l < s.L; ++l)
      for (int tid = 0; tid < kLayerTensors; ++tid)
        fill(y.t(l, tid), seed ^ (((uint64_t)(l + 1) << 8) | tid), tid == MT_T_ATTN_NORM || tid == MT_T_MLP_NORM);
    fill(y.final_norm, seed ^ 0x1001, true);
    if (!y.tied) fill(y.head, seed ^ 0x1002, false);
  }
  if (world > 0) {
    // Sharded: the moments are read and written on the rank's own ranges
    // only, so only those pages are touched (the rest stay unbacked).
    std::vector<std::pair<size_t, size_t>> own;
    for (int l = 0; l < s.L; ++l) own.push_back({y.layer_begin(l) + plan.layer_begin, y.layer_begin(l) + plan.layer_end});
    own.push_back({y.final_norm.off + plan.head_begin, y.final_norm.off + plan.head_end});
    own.push_back({y.embed.off + (size_t)plan.embed_row_begin * s.d, y.embed.off + (size_t)plan.embed_row_end * s.d});
    for (const auto& r : own)
      parallel_ranges(*c->pool, r.second - r.first, [&](size_t b, size_t e) {
        memset(c->m + r.first + b, 0, (e - b) * 4);
        memset(c->v + r.first + b, 0, (e - b) * 4);
      });
    if (c->grad)
      parallel_ranges(*c->pool, y.total, [&](size_t b, size_t e) { memset(c->grad + b * gsz, 0, (e - b) * gsz); });
  } else {
    parallel_ranges(*c->pool, y.total, [&](size_t b, size_t e) {
      memset(c->m + b, 0, (e - b) * 4);
      memset(c->v + b, 0, (e - b) * 4);
      if (c->grad) memset(c->grad + b * gsz, 0, (e - b) * gsz);
    });
  }
  if (c->ring) {
    const size_t nr = (size_t)MT_GRAD_RING_SLOTS * c->layer_f;
    parallel_ranges(*c->pool, nr, [&](size_t b, size_t e) { memset(c->ring + b * gsz, 0, (e - b) * gsz); });
    if (c->defer_g)
      parallel_ranges(*c->pool, (size_t)c->defer_layers * c->layer_f,
                      [&](size_t b, size_t e) { memset(c->defer_g + b * gsz, 0, (e - b) * gsz); });
  }
  if (c->grad_head_owned)
    parallel_ranges(*c->pool, head_f, [&](size_t b, size_t e) { memset(c->grad_head + b * gsz, 0, (e - b) * gsz); });
  // bf16 streaming copies
  for (int l = 0; l < s.L; ++l) {
    uint16_t* blk = c->bf_layers + (size_t)l * y.bf_layer;
    memset(blk, 0, y.bf_layer * 2);
    for (int tid = 0; tid < kLayerTensors; ++tid) {
      const TRef& r = y.t(l, tid);
      uint16_t* dst = blk + y.bf_of(tid);
      parallel_ranges(*c->pool, r.n, [&](size_t b, size_t e) { bf16_round_chunk(c->arena + r.off + b, dst + b, e - b); });
    }
  }
  parallel_ranges(*c->pool, y.embed.n,
                  [&](size_t b, size_t e) { bf16_round_chunk(c->arena + y.embed.off + b, c->bf_embed + b, e - b); });
  memset(c->bf_head, 0, head_bf * 2);
  bf16_round_chunk(c->arena + y.final_norm.off, c->bf_head, s.d);
  uint16_t* bhw = c->bf_head + align_up(s.d, 128);
  parallel_ranges(*c->pool, y.head.n,  // (nothing when tied)
                  [&](size_t b, size_t e) { bf16_round_chunk(c->arena + y.head.off + b, bhw + b, e - b); });

  // device memory: one allocation carved into buffers
  c->dmem_bytes = need;
  if (cudaMalloc(&c->dmem, need) != cudaSuccess) return fail(MT_ERR_NOMEM, "device allocation failed");
  uint8_t* p = static_cast<uint8_t*>(c->dmem);
  auto carve = [&](size_t bytes) {
    void* r = p;
    p += align_up(bytes, 256);
    return r;
  };
  const size_t T = s.T, d = s.d, F = s.F, V = s.V;
  const mt_shard* pp = world > 0 ? &plan : nullptr;
  c->wslot_bytes = slot_elems(y, pp) * 2;
  c->wslot[0] = (uint16_t*)carve(slot_elems(y, pp) * 2);
  c->wslot[1] = (uint16_t*)carve(slot_elems(y, pp) * 2);
  const size_t lay_f = y.layer_end(0) - y.layer_begin(0);
  c->gslot[0] = (float*)carve(gslot_elems(y, pp) * 4);
  c->gslot[1] = (float*)carve(gslot_elems(y, pp) * 4);
  c->d_head_w = (uint16_t*)carve(head_w_elems(y, pp) * 2);
  c->d_head_g = (float*)carve(head_g_elems(y, pp) * 4);
  if (pp) {
    const size_t rows = embed_rows_chunk(plan, s.V);
    c->d_embed_w = (uint16_t*)carve((size_t)world * rows * d * 2);
    c->d_embed_g = (float*)carve((size_t)world * rows * d * 4);
  }
  if (gsz == 2) {
    c->gslot16[0] = (uint16_t*)carve(lay_f * 2);
    c->gslot16[1] = (uint16_t*)carve(lay_f * 2);
    c->d_head_g16 = (uint16_t*)carve(y.head_block * 2);
  }
  c->xb = (float*)carve((size_t)((cfg->flags & MT_FLAG_OFFLOAD_ACTS) ? std::min(s.L + 1, 3) : s.L + 1) * T * d * 4);
  c->u_b = (uint16_t*)carve(T * d * 2);
  c->qkv_b = (uint16_t*)carve(T * (size_t)s.Nqkv * 2);
  const size_t n_attn = (cfg->flags & MT_FLAG_STASH_ATTN) ? (size_t)s.L : 1;
  c->ao_b = (uint16_t*)carve(n_attn * T * (size_t)s.Hd * 2);
  c->lse = (float*)carve(n_attn * s.b * s.H * (size_t)s.s * 4);
  c->h_f = (float*)carve(T * d * 4);
  c->r1 = (float*)carve(T * 4);
  c->r2 = (float*)carve(T * 4);
  c->w_b = (uint16_t*)carve(T * d * 2);
  const size_t R = s.E > 0 ? std::max(T, T * (size_t)s.topk) : T;
  c->gu_b = (uint16_t*)carve(R * 2 * F * 2);
  c->act_b = (uint16_t*)carve(R * F * 2);
  c->gx0 = (float*)carve(T * d * 4);
  c->gx1 = (float*)carve(T * d * 4);
  c->gxb = (uint16_t*)carve(T * d * 2);
  c->dact_b = (uint16_t*)carve(R * F * 2);
  c->dgu_b = (uint16_t*)carve(R * 2 * F * 2);
  if (s.E > 0) {
    const size_t Tk = T * (size_t)s.topk, E = s.E;
    c->moe_logits = (float*)carve(T * E * 4);
    c->moe_dlogits = (float*)carve(T * E * 4);
    c->moe_idx = (int32_t*)carve(Tk * 4);
    c->moe_gate = (float*)carve(Tk * 4);
    c->moe_dgate = (float*)carve(Tk * 4);
    c->moe_slot = (int32_t*)carve((size_t)s.L * Tk * 4 * 2);
    c->moe_row = c->moe_slot + (size_t)s.L * Tk;
    c->xe_b = (uint16_t*)carve(Tk * d * 2);
    c->dye_b = (uint16_t*)carve(Tk * d * 2);
    c->ye = (float*)carve(Tk * d * 4);
    c->dxe = (float*)carve(Tk * d * 4);
  }
  c->tmp_f = (float*)carve(T * d * 4);
  c->dh_f = (float*)carve(T * d * 4);
  c->dhb = (uint16_t*)carve(T * d * 2);
  c->dao_b = (uint16_t*)carve(T * (size_t)s.Hd * 2);
  c->dvec = (float*)carve((size_t)s.b * s.H * s.s * 4);
  c->dqacc = (float*)carve(T * (size_t)s.Hd * 4);
  c->dqkv_b = (uint16_t*)carve(T * (size_t)s.Nqkv * 2);
  c->rms_part = (float*)carve((size_t)rmsnorm_bwd_blocks((int)T) * d * 4);
  c->n_b = (uint16_t*)carve(T * d * 2);
  c->rf = (float*)carve(T * 4);
  c->logits = (float*)carve((size_t)Tc * V * 4);
  c->dz_b = (uint16_t*)carve((size_t)Tc * V * 2);
  c->rowloss = (float*)carve(T * 4);
  c->d_tok = (int32_t*)carve((5 * T + 1) * 4);
  c->d_uid = c->d_tok + 4 * T + 1;
  c->d_lab = c->d_tok + T;
  c->d_offs = c->d_tok + 2 * T;
  c->d_pos = c->d_tok + 3 * T + 1;
  c->d_flags = (int32_t*)carve((size_t)(s.L + 2) * 4);
  c->d_err = (int32_t*)carve(4);
  c->d_cos = (float*)carve((size_t)s.s * (s.hd / 2) * 4);
  c->d_sin = (float*)carve((size_t)s.s * (s.hd / 2) * 4);
  c->d_loss = (float*)carve(4);
  if ((size_t)(p - static_cast<uint8_t*>(c->dmem)) > need) return fail(MT_ERR_NOMEM, "device carve overflow");
  if (cudaMemset(c->dmem, 0, need) != cudaSuccess) return fail(MT_ERR_CUDA, "cudaMemset failed");
  {
    std::vector<float> cs((size_t)s.s * (s.hd / 2)), sn(cs.size());
    for (int pos = 0; pos < s.s; ++pos)
      for (int i = 0; i < s.hd / 2; ++i) {
        const double th = pow((double)cfg->rope_base, -2.0 * i / s.hd);
        cs[(size_t)pos * (s.hd / 2) + i] = (float)cos(pos * th);
        sn[(size_t)pos * (s.hd / 2) + i] = (float)sin(pos * th);
      }
    if (cudaMemcpy(c->d_cos, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->d_sin, sn.data(), sn.size() * 4, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(MT_ERR_CUDA, "RoPE tables");
  }

  // streams and events
  if (cfg->flags & MT_FLAG_SERIALIZE) {
    if (cudaStreamCreateWithFlags(&c->s_comp, cudaStreamNonBlocking) != cudaSuccess)
      return fail(MT_ERR_CUDA, "stream");
    c->s_h2d = c->s_d2h = c->s_act = c->s_comp;
  } else {
    if (cudaStreamCreateWithFlags(&c->s_comp, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c->s_h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&c->s_d2h, cudaStreamNonBlocking) != cudaSuccess ||
        ((cfg->flags & MT_FLAG_OFFLOAD_ACTS) && cudaStreamCreateWithFlags(&c->s_act, cudaStreamNonBlocking) != cudaSuccess))
      return fail(MT_ERR_CUDA, "stream");
  }
  // weight loads: 0..L-1 then L-2..0 (layer L-1 stays resident over the turn)
  for (int l = 0; l < s.L; ++l) c->load_seq.push_back(l);
  for (int l = s.L - 2; l >= 0; --l) c->load_seq.push_back(l);
  const int nloads = (int)c->load_seq.size();
  auto mk = [&](std::vector<cudaEvent_t>& v, int n) {
    v.assign(n, nullptr);
    for (auto& e : v)
      if (cudaEventCreate(&e) != cudaSuccess) return false;
    return true;
  };
  bool ok = mk(c->ev_wready, nloads) && mk(c->ev_compready, nloads) && mk(c->ev_h2d_start, nloads) &&
            mk(c->ev_slotfree, nloads) && mk(c->ev_gready, s.L) && mk(c->ev_d2h_start, s.L) &&
            mk(c->ev_gdrained, s.L);
  if (cfg->flags & MT_FLAG_OFFLOAD_ACTS)
    ok = ok && mk(c->ev_xready, s.L + 1) && mk(c->ev_xout, s.L + 1) && mk(c->ev_xin, s.L + 1) &&
         mk(c->ev_bwdone, s.L + 1);
  for (cudaEvent_t* e : {&c->ev_head_h2d_start, &c->ev_head_wready, &c->ev_head_gready, &c->ev_head_d2h_start,
                         &c->ev_head_drained, &c->ev_emb_ready, &c->ev_emb_d2h_start, &c->ev_emb_drained,
                         &c->ev_step_start, &c->ev_fwd_end, &c->ev_head_end, &c->ev_bwd_end, &c->ev_step_end})
    ok = ok && cudaEventCreate(e) == cudaSuccess;
  if (!ok) return fail(MT_ERR_CUDA, "event creation failed");
  if (s.E > 0 && cudaEventCreateWithFlags(&c->ev_route, cudaEventDisableTiming) != cudaSuccess)
    return fail(MT_ERR_CUDA, "event creation failed");
  if (world > 0) {
    // Every rank joins here (NCCL's initialisation is collective); then the
    // table the first step gathers from: the same bf16 copy on every rank.
    if (cudaEventCreate(&c->ev_embw) != cudaSuccess) return fail(MT_ERR_CUDA, "event creation failed");
    ncclUniqueId uid;
    memcpy(&uid, id, sizeof(uid));
    ncclResult_t e = nccl->CommInitRank(&c->comm_comp, world, uid, rank);
    if (e != ncclSuccess) {
      c->comm_comp = nullptr;
      return fail(MT_ERR_CUDA, std::string("ncclCommInitRank: ") + nccl->GetErrorString(e));
    }
    e = nccl->CommSplit(c->comm_comp, 0, rank, &c->comm_h2d, nullptr);
    if (e != ncclSuccess) {
      c->comm_h2d = nullptr;
      return fail(MT_ERR_CUDA, std::string("ncclCommSplit: ") + nccl->GetErrorString(e));
    }
    if (cudaMemcpy(c->d_embed_w, c->bf_embed, (size_t)s.V * s.d * 2, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(MT_ERR_CUDA, "embedding table copy failed");
  }
  if (const char* w = getenv("MT_WAIT_LIMIT_S")) {
    const double lim = atof(w);
    if (lim > 0) c->wait_limit_s = lim;
  }
  c->opt_thread = std::thread(opt_loop, c);
  *out = c;
  return MT_OK;
}

}  // namespace mteng
using namespace mteng;

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
extern "C" int mt_create(const mt_config* cfg, float* host_param_arena, size_t arena_bytes, mt_ctx** out) {
  g_create_error.clear();
  return create_impl(cfg, host_param_arena, arena_bytes, out);
}

extern "C" int mt_shard_id(void* id_out) {
  g_create_error.clear();
  if (!id_out) return set_err(nullptr, MT_ERR_ARG, "id_out is NULL");
  static_assert(sizeof(ncclUniqueId) == MT_SHARD_ID_BYTES, "NCCL unique id size");
  std::string why;
  const NcclApi* nccl = nccl_api(&why);
  if (!nccl) return set_err(nullptr, MT_ERR_CUDA, why);
  ncclUniqueId uid;
  const ncclResult_t e = nccl->GetUniqueId(&uid);
  if (e != ncclSuccess) return set_err(nullptr, MT_ERR_CUDA, std::string("ncclGetUniqueId: ") + nccl->GetErrorString(e));
  memcpy(id_out, &uid, sizeof(uid));
  return MT_OK;
}

extern "C" int mt_create_sharded(const mt_config* cfg, float* host_param_arena, size_t arena_bytes, int world,
                                 int rank, const void* id, mt_ctx** out) {
  g_create_error.clear();
  if (world < 1 || rank < 0 || rank >= world) return set_err(nullptr, MT_ERR_ARG, "rank outside [0, world)");
  return create_impl(cfg, host_param_arena, arena_bytes, out, world, rank, id);
}

extern "C" int mt_get_routing(mt_ctx* c, int layer, int32_t* idx, size_t n) {
  if (!c) return MT_ERR_ARG;
  const Shapes& s = c->lay.sh;
  if (s.E == 0) return set_err(c, MT_ERR_CONFIG, "no expert layers");
  if (layer < 0 || layer >= s.L || !idx) return set_err(c, MT_ERR_ARG, "layer outside [0, L) or NULL");
  const size_t Tk = (size_t)s.T * s.topk;
  if (n < Tk) return set_err(c, MT_ERR_ARG, "idx smaller than b*s*topk");
  memcpy(idx, c->moe_idx_h + (size_t)layer * Tk, Tk * 4);
  return MT_OK;
}

extern "C" size_t mt_device_bytes_sharded(const mt_config* cfg, int world) {
  mt_shard p{};
  if (mt_shard_plan(cfg, world, 0, &p) != MT_OK) return 0;
  const Layout y = make_layout(*cfg);
  return device_bytes(y, logits_chunk(y.sh), cfg->flags, &p);
}

extern "C" int mt_train_step(mt_ctx* c, const int32_t* tokens, const int32_t* labels, float* loss_out) {
  if (!c) return MT_ERR_ARG;
  if (!tokens || !labels || !loss_out) return set_err(c, MT_ERR_ARG, "tokens, labels and loss_out are required");
  const Shapes& s = c->lay.sh;
  const int T = s.T;
  for (int t = 0; t < T; ++t)
    if (tokens[t] < 0 || tokens[t] >= s.V || labels[t] < 0 || labels[t] >= s.V)
      return set_err(c, MT_ERR_ARG, "token or label outside [0, V)");
  CK(cudaSetDevice(c->device));
  // Host staging: tokens, labels and the per-unique-token position lists.
  int32_t* st = c->stage_i;
  memcpy(st, tokens, (size_t)T * 4);
  memcpy(st + T, labels, (size_t)T * 4);
  std::vector<int32_t> count(s.V, 0);
  for (int t = 0; t < T; ++t) count[tokens[t]]++;
  c->uniq.clear();
  std::vector<int32_t> start(s.V, 0);
  int32_t* offs = st + 2 * T;
  int32_t* pos = st + 3 * T + 1;
  int32_t acc = 0;
  for (int v = 0; v < s.V; ++v)
    if (count[v]) {
      offs[c->uniq.size()] = acc;
      start[v] = acc;
      c->uniq.push_back(v);
      acc += count[v];
    }
  const int n_unique = (int)c->uniq.size();
  offs[n_unique] = acc;
  for (int t = 0; t < T; ++t) pos[start[tokens[t]]++] = t;  // increasing t within each token
  int32_t* uid = st + 4 * T + 1;  // the unique ids, for the sharded dense embedding gradient
  for (int u = 0; u < n_unique; ++u) uid[u] = c->uniq[u];

  c->call_t0 = now_s();
  c->adamw_first = c->adamw_last = 0;
  c->step++;
  c->opt_status = MT_OK;
  c->skip_updates = false;
  c->adamw_s = c->adamw_bytes = 0;
  c->timing_used = 0;
  c->timed.clear();
  c->launches = 0;
  c->err.clear();
  {
    std::lock_guard<std::mutex> lk(c->opt_mu);
    c->layer_jobs_done = 0;
  }
  c->job_times.clear();
  if (c->untouched_pending) start_untouched_prev(c);
  queue_deferred(c);  // the last step's deferred updates overlap this forward sweep
  const double te0 = now_s();
  int r = enqueue_step(c, n_unique);
  c->enqueue_s = now_s() - te0;
  if (r != MT_OK) {
    // Let the optimizer finish the jobs already queued and the streams drain.
    c->skip_updates = true;
    wait_jobs(c);
    cudaDeviceSynchronize();
    return r;
  }
  wait_jobs(c);
  if (!wait_event(c, c->ev_step_end)) return set_err(c, MT_ERR_TIMEOUT, "step did not finish within the wait limit");
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_err(c, MT_ERR_CUDA, cudaGetErrorString(e));
  int32_t dev_err;
  memcpy(&dev_err, c->misc_h + 1, 4);
  if (dev_err != 0) {
    char m[160];
    snprintf(m, sizeof m,
             "kernel reported error %d (bounded wait expired); the step's updates from that point on were skipped",
             dev_err);
    return set_err(c, MT_ERR_DEVICE, m);
  }
  *loss_out = c->misc_h[0] / (float)T;
  collect_stats(c);
  c->stats.host_step_ms = (now_s() - c->call_t0) * 1e3;
  c->stats.enqueue_ms = c->enqueue_s * 1e3;
  c->stats.adamw_first_ms = c->adamw_first > 0 ? (c->adamw_first - c->call_t0) * 1e3 : 0;
  c->stats.adamw_last_ms = c->adamw_last > 0 ? (c->adamw_last - c->call_t0) * 1e3 : 0;
  if (c->opt_status != MT_OK) return c->opt_status;
  return MT_OK;
}

extern "C" int mt_layer_fwd_bwd(mt_ctx* c, int l, const float* x_in, const float* dx_out, float* x_out,
                                float* dx_in, float* grads, size_t grads_bytes) {
  if (!c) return MT_ERR_ARG;
  if (!x_in || !dx_out || !x_out || !dx_in || !grads) return set_err(c, MT_ERR_ARG, "NULL argument");
  const Layout& y = c->lay;
  const Shapes& s = y.sh;
  if (l < 0 || l >= s.L) return set_err(c, MT_ERR_ARG, "layer outside [0, L)");
  if (grads_bytes < c->layer_f * 4) return set_err(c, MT_ERR_ARG, "grads smaller than one layer's block");
  if (sharded(c)) return set_err(c, MT_ERR_CONFIG, "single-layer calls are not available on a sharded context");
  flush_deferred(c);
  CK(cudaSetDevice(c->device));
  const size_t n = (size_t)s.T * s.d;
  cudaStream_t sc = c->s_comp;
  c->timing_used = 0;
  c->timed.clear();
  c->err.clear();
  CK(cudaMemsetAsync(c->d_err, 0, sizeof(int32_t), sc));
  // the layer's streamed bf16 weights into slot 0, x_l into its boundary slot
  CK(cudaMemcpyAsync(c->wslot[0], c->bf_layers + (size_t)l * y.bf_layer, y.bf_layer * 2, cudaMemcpyHostToDevice, sc));
  CK(cudaMemcpyAsync(x_fwd(c, l), x_in, n * 4, cudaMemcpyHostToDevice, sc));
  CK(cudaMemcpyAsync(c->gx0, dx_out, n * 4, cudaMemcpyHostToDevice, sc));
  CKM(layer_fwd(c, l, 0, x_fwd(c, l), x_fwd(c, l + 1)));
  CKM(layer_bwd(c, l, 0, x_fwd(c, l), c->gslot[0], c->gx0, c->gx1));
  CK(cudaMemcpyAsync(x_out, x_fwd(c, l + 1), n * 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaMemcpyAsync(dx_in, c->gx1, n * 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaMemcpyAsync(grads, c->gslot[0], c->layer_f * 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaMemcpyAsync(c->misc_h + 1, c->d_err, 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaStreamSynchronize(sc));
  int32_t dev_err;
  memcpy(&dev_err, c->misc_h + 1, 4);
  if (dev_err != 0) return set_err(c, MT_ERR_DEVICE, "kernel reported an error (bounded wait expired)");
  return MT_OK;
}

extern "C" int mt_head_fwd_bwd(mt_ctx* c, const float* x_L, const int32_t* labels, float* loss_out, float* dx_L,
                               float* grads, size_t grads_bytes) {
  if (!c) return MT_ERR_ARG;
  if (!x_L || !labels || !loss_out || !dx_L || !grads) return set_err(c, MT_ERR_ARG, "NULL argument");
  const Layout& y = c->lay;
  const Shapes& s = y.sh;
  const size_t head_f = y.head_block;
  if (grads_bytes < head_f * 4) return set_err(c, MT_ERR_ARG, "grads smaller than the final-norm + head block");
  if (sharded(c)) return set_err(c, MT_ERR_CONFIG, "single-layer calls are not available on a sharded context");
  for (int t = 0; t < s.T; ++t)
    if (labels[t] < 0 || labels[t] >= s.V) return set_err(c, MT_ERR_ARG, "label outside [0, V)");
  flush_deferred(c);
  CK(cudaSetDevice(c->device));
  const size_t n = (size_t)s.T * s.d;
  cudaStream_t sc = c->s_comp;
  c->timing_used = 0;
  c->timed.clear();
  c->err.clear();
  CK(cudaMemsetAsync(c->d_err, 0, sizeof(int32_t), sc));
  CKM(copy_head_weights(c, sc));
  CK(cudaMemcpyAsync(x_fwd(c, s.L), x_L, n * 4, cudaMemcpyHostToDevice, sc));
  CK(cudaMemcpyAsync(c->d_lab, labels, (size_t)s.T * 4, cudaMemcpyHostToDevice, sc));
  CKM(head_step(c, c->gx0));
  CK(cudaMemcpyAsync(c->misc_h, c->d_loss, 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaMemcpyAsync(dx_L, c->gx0, n * 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaMemcpyAsync(grads, c->d_head_g, head_f * 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaMemcpyAsync(c->misc_h + 1, c->d_err, 4, cudaMemcpyDeviceToHost, sc));
  CK(cudaStreamSynchronize(sc));
  int32_t dev_err;
  memcpy(&dev_err, c->misc_h + 1, 4);
  if (dev_err != 0) return set_err(c, MT_ERR_DEVICE, "kernel reported an error (bounded wait expired)");
  *loss_out = c->misc_h[0] / (float)s.T;
  return MT_OK;
}

extern "C" int mt_get_grads(mt_ctx* c, float* dst, size_t bytes) {
  if (!c || !dst) return MT_ERR_ARG;
  if (!c->grad) return set_err(c, MT_ERR_CONFIG, "created with MT_FLAG_GRAD_RING: no gradient arena is kept");
  if (bytes < c->lay.total * 4) return set_err(c, MT_ERR_ARG, "destination smaller than the arena");
  if (c->gsz == 4) {
    memcpy(dst, c->grad, c->lay.total * 4);
  } else {  // bf16 gradients widen exactly to fp32
    const uint16_t* g = reinterpret_cast<const uint16_t*>(c->grad);
    parallel_ranges(*c->pool, c->lay.total, [&](size_t b, size_t e) {
      for (size_t i = b; i < e; ++i) {
        const uint32_t u = (uint32_t)g[i] << 16;
        memcpy(dst + i, &u, 4);
      }
    });
  }
  return MT_OK;
}

extern "C" int mt_get_params(mt_ctx* c, float* dst, size_t bytes) {
  if (!c || !dst) return MT_ERR_ARG;
  if (bytes < c->lay.total * 4) return set_err(c, MT_ERR_ARG, "destination smaller than the arena");
  flush_deferred(c);
  memcpy(dst, c->arena, c->lay.total * 4);
  return MT_OK;
}

extern "C" int mt_get_opt_state(mt_ctx* c, float* m_dst, float* v_dst, size_t bytes_each, int64_t* step) {
  if (!c) return MT_ERR_ARG;
  const size_t need = c->lay.total * 4;
  if ((m_dst || v_dst) && bytes_each < need) return set_err(c, MT_ERR_ARG, "destination smaller than the arena");
  flush_deferred(c);
  if (m_dst) memcpy(m_dst, c->m, need);
  if (v_dst) memcpy(v_dst, c->v, need);
  if (step) *step = c->step;
  return MT_OK;
}

extern "C" int mt_set_state(mt_ctx* c, const float* params, const float* m, const float* v, size_t bytes_each,
                            int64_t step) {
  if (!c) return MT_ERR_ARG;
  const Layout& y = c->lay;
  const Shapes& s = y.sh;
  const size_t need = y.total * 4;
  if ((params || m || v) && bytes_each < need) return set_err(c, MT_ERR_ARG, "source smaller than the arena");
  if (step < 0 || step > (int64_t)1 << 30) return set_err(c, MT_ERR_ARG, "step out of range");
  flush_deferred(c);  // the pending updates belong to the state being replaced
  if (m) memcpy(c->m, m, need);
  if (v) memcpy(c->v, v, need);
  c->step = (int)step;
  if (params) {
    memcpy(c->arena, params, need);
    // rebuild the bf16 streaming copies from the new master
    for (int l = 0; l < s.L; ++l) {
      uint16_t* blk = c->bf_layers + (size_t)l * y.bf_layer;
      for (int tid = 0; tid < kLayerTensors; ++tid) {
        const TRef& r = y.t(l, tid);
        uint16_t* dst = blk + y.bf_of(tid);
        parallel_ranges(*c->pool, r.n,
                        [&](size_t b, size_t e) { bf16_round_chunk(c->arena + r.off + b, dst + b, e - b); });
      }
    }
    parallel_ranges(*c->pool, y.embed.n,
                    [&](size_t b, size_t e) { bf16_round_chunk(c->arena + y.embed.off + b, c->bf_embed + b, e - b); });
    bf16_round_chunk(c->arena + y.final_norm.off, c->bf_head, s.d);
    uint16_t* bhw = c->bf_head + align_up(s.d, 128);
    parallel_ranges(*c->pool, y.head.n,
                    [&](size_t b, size_t e) { bf16_round_chunk(c->arena + y.head.off + b, bhw + b, e - b); });
  }
  return MT_OK;
}

extern "C" int mt_get_stats(mt_ctx* c, mt_stats* out) {
  if (!c || !out) return MT_ERR_ARG;
  *out = c->stats;
  return MT_OK;
}

extern "C" int mt_get_timeline(mt_ctx* c, float* out, size_t cap_floats, size_t* n_floats) {
  if (!c || !n_floats) return MT_ERR_ARG;
  const int L = c->lay.sh.L;
  const size_t nloads = c->load_seq.size();
  const size_t nj = c->job_times.size();
  const size_t need = 3 + 5 * nloads + 4 * (size_t)L + 4 + 4 * nj;
  *n_floats = need;
  if (!out) return MT_OK;
  if (cap_floats < need) return set_err(c, MT_ERR_ARG, "timeline buffer too small");
  if (c->step == 0) return set_err(c, MT_ERR_ARG, "no step has run");
  CK(cudaSetDevice(c->device));
  auto t = [&](cudaEvent_t e) { return ev_ms(c->ev_step_start, e); };
  size_t k = 0;
  out[k++] = (float)nloads;
  out[k++] = (float)L;
  out[k++] = (float)nj;
  for (size_t i = 0; i < nloads; ++i) {
    out[k++] = (float)c->load_seq[i];
    out[k++] = t(c->ev_h2d_start[i]);
    out[k++] = t(c->ev_wready[i]);
    out[k++] = t(c->ev_compready[i]);
    out[k++] = t(c->ev_slotfree[i]);
  }
  for (int b = 0; b < L; ++b) {
    out[k++] = (float)(L - 1 - b);
    out[k++] = t(c->ev_gready[b]);
    out[k++] = t(c->ev_d2h_start[b]);
    out[k++] = t(c->ev_gdrained[b]);
  }
  out[k++] = t(c->ev_fwd_end);
  out[k++] = t(c->ev_head_end);
  out[k++] = t(c->ev_bwd_end);
  out[k++] = t(c->ev_step_end);
  for (const auto& jt : c->job_times) {
    out[k++] = (float)jt.kind;
    out[k++] = (float)jt.layer;
    out[k++] = (float)((jt.ready - c->call_t0) * 1e3);
    out[k++] = (float)((jt.done - c->call_t0) * 1e3);
  }
  return MT_OK;
}

extern "C" int mt_get_stream(mt_ctx* c, void** stream) {
  if (!c || !stream) return MT_ERR_ARG;
  *stream = c->s_comp;
  return MT_OK;
}

extern "C" size_t mt_device_bytes(const mt_config* cfg) {
  if (validate_config(cfg, nullptr) != MT_OK) return 0;
  const Layout y = make_layout(*cfg);
  return device_bytes(y, logits_chunk(y.sh), cfg->flags);
}

namespace {
void CUDART_CB host_sleep(void* ms) {
  std::this_thread::sleep_for(std::chrono::milliseconds((int64_t)(intptr_t)ms));
}
}  // namespace

extern "C" int mt_inject_host_stall(mt_ctx* c, int stream, int ms) {
  if (!c) return MT_ERR_ARG;
  if (stream < 0 || stream > 2 || ms < 0 || ms > 60000)
    return set_err(c, MT_ERR_ARG, "stream must be 0, 1 or 2 and ms in [0, 60000]");
  CK(cudaSetDevice(c->device));
  cudaStream_t st = stream == 0 ? c->s_h2d : stream == 1 ? c->s_comp : c->s_d2h;
  CK(cudaLaunchHostFunc(st, host_sleep, (void*)(intptr_t)ms));
  return MT_OK;
}

extern "C" int mt_flush(mt_ctx* c) {
  if (!c) return MT_ERR_ARG;
  flush_deferred(c);
  return MT_OK;
}

extern "C" void mt_destroy(mt_ctx* c) {
  if (c) flush_deferred(c);
  free_all(c);
}

extern "C" const char* mt_last_error(const mt_ctx* c) { return c ? c->err.c_str() : g_create_error.c_str(); }
