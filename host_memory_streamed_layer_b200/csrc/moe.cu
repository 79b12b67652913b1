// Mixture-of-experts MLP kernels (the family's routing, dispatch and combine;
// the expert products themselves run on the tcgen05 GEMMs of gemm.cu).
//
// Reading (saify.me, "Who this is actually for", lists MoE variants among the
// supported families with no routing rule): per token t of the MLP input w,
//   logits = w Wr^T; R_t = the topk experts with the largest logits (ties to
//   the lower index); gates = softmax of the logits over R_t;
//   y_t = sum_{e in R_t} gate_te * SwiGLU_e(w_t).
// Every routed token is computed (no capacity limit). Routed rows are grouped
// by expert ("slots": expert e's rows are slots [off_e, off_e + n_e), tokens
// in increasing order), so each expert's products are plain GEMMs over a
// contiguous block of rows; every reduction below runs in a fixed order.
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "mt_internal.h"

namespace mt {

namespace {

using bf16 = __nv_bfloat16;

__device__ __forceinline__ float bf(const bf16 v) { return __bfloat162float(v); }

// One warp per token: the E logits (lanes split d, warp sums), then topk
// rounds of a warp argmax (largest value; ties to the lower index), then the
// gates. Lane e holds logit e (and lane e - 32 the logit e for e >= 32).
__global__ void k_moe_router(const bf16* __restrict__ w, const bf16* __restrict__ Wr, int T, int d, int E, int k,
                             float* __restrict__ logits, int32_t* __restrict__ idx, float* __restrict__ gate) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const bf16* wt = w + (int64_t)t * d;
  float lg[2] = {-INFINITY, -INFINITY};
  for (int e = 0; e < E; ++e) {
    const bf16* wr = Wr + (int64_t)e * d;
    float acc = 0.f;
    for (int c = lane * 8; c < d; c += 256) {  // d is a multiple of 64
      const uint4 a = *reinterpret_cast<const uint4*>(wt + c);
      const uint4 b = *reinterpret_cast<const uint4*>(wr + c);
      const bf16* pa = reinterpret_cast<const bf16*>(&a);
      const bf16* pb = reinterpret_cast<const bf16*>(&b);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc = fmaf(bf(pa[i]), bf(pb[i]), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((e & 31) == lane) lg[e >> 5] = acc;
  }
  for (int h = 0; h < 2; ++h) {
    const int e = lane + 32 * h;
    if (e < E) logits[(int64_t)t * E + e] = lg[h];
  }
  // Selection works on a copy where NaN is -inf, so a token whose logits are
  // not finite still gets distinct valid experts (its outputs then carry the
  // NaN on to the gradient checks); taken and absent experts rank below every
  // candidate by index.
  float cand[2];
  int id[2];
  for (int h = 0; h < 2; ++h) {
    const int e = lane + 32 * h;
    cand[h] = (e < E && !isnan(lg[h])) ? lg[h] : -INFINITY;
    id[h] = e < E ? e : (1 << 20) + e;
  }
  float sel_v = 0.f, m = 0.f, sum = 0.f;
  int sel_e = 0;
  for (int j = 0; j < k; ++j) {
    // best of this lane's two, then across the warp
    float v = cand[0];
    int i = id[0];
    if (cand[1] > v || (cand[1] == v && id[1] < i)) {
      v = cand[1];
      i = id[1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
      if (v2 > v || (v2 == v && i2 < i)) {
        v = v2;
        i = i2;
      }
    }
    // i is a valid expert: at most j < k <= E of them are taken
    for (int h = 0; h < 2; ++h)
      if (id[h] == i) {
        cand[h] = -INFINITY;
        id[h] = (1 << 21) + i;
      }
    const float lv = __shfl_sync(0xffffffffu, lg[i >> 5], i & 31);  // the logit itself (NaN stays NaN)
    if (j == 0) m = lv;
    const float p = __expf(lv - m);
    sum += p;
    if (lane == j) {
      sel_e = i;
      sel_v = p;
    }
  }
  if (lane < k) {
    idx[(int64_t)t * k + lane] = sel_e;
    gate[(int64_t)t * k + lane] = sel_v / sum;
  }
}

// Routed rows grouped by expert: xe[slot] = w[row_of[slot]] (bf16 rows of d).
__global__ void k_moe_gather(const bf16* __restrict__ w, const int32_t* __restrict__ row_of, int rows, int d,
                             bf16* __restrict__ xe) {
  const int d8 = d / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)rows * d8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / d8;
    const int c = (int)(i % d8);
    reinterpret_cast<uint4*>(xe + r * d)[c] = reinterpret_cast<const uint4*>(w + (int64_t)row_of[r] * d)[c];
  }
}

// out[t] = h[t] + sum_j gate[t, j] ye[slot_of[t, j]], j in increasing order.
__global__ void k_moe_combine(const float* __restrict__ h, const float* __restrict__ ye,
                              const int32_t* __restrict__ slot_of, const float* __restrict__ gate, int T, int k,
                              int d, float* __restrict__ out) {
  const int d4 = d / 4;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)T * d4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / d4;
    const int c = (int)(i % d4);
    float4 acc = reinterpret_cast<const float4*>(h + t * d)[c];
    for (int j = 0; j < k; ++j) {
      const float g = gate[t * k + j];
      const float4 y = reinterpret_cast<const float4*>(ye + (int64_t)slot_of[t * k + j] * d)[c];
      acc.x = fmaf(g, y.x, acc.x);
      acc.y = fmaf(g, y.y, acc.y);
      acc.z = fmaf(g, y.z, acc.z);
      acc.w = fmaf(g, y.w, acc.w);
    }
    reinterpret_cast<float4*>(out + t * d)[c] = acc;
  }
}

// One warp per routed (t, j): the expert's output gradient dye[slot] =
// bf16(gate_tj dy_t) and the gate's gradient dgate_tj = dy_t . ye[slot].
__global__ void k_moe_dy(const float* __restrict__ dy, const float* __restrict__ ye,
                         const int32_t* __restrict__ slot_of, const float* __restrict__ gate, int T, int k, int d,
                         bf16* __restrict__ dye, float* __restrict__ dgate) {
  const int lane = threadIdx.x & 31;
  const int64_t p = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (p >= (int64_t)T * k) return;
  const int64_t t = p / k;
  const int64_t slot = slot_of[p];
  const float g = gate[p];
  const float* dyt = dy + t * d;
  const float* yr = ye + slot * d;
  bf16* out = dye + slot * d;
  float acc = 0.f;
  for (int c = lane * 4; c < d; c += 128) {
    const float4 a = *reinterpret_cast<const float4*>(dyt + c);
    const float4 y = *reinterpret_cast<const float4*>(yr + c);
    acc = fmaf(a.x, y.x, fmaf(a.y, y.y, fmaf(a.z, y.z, fmaf(a.w, y.w, acc))));
    __nv_bfloat162 lo = __floats2bfloat162_rn(g * a.x, g * a.y), hi = __floats2bfloat162_rn(g * a.z, g * a.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(out + c) = pk;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) dgate[p] = acc;
}

// Thread per token: the logits' gradient through the softmax over the routed
// experts, dlogit_e = g_e (dg_e - sum_j g_j dg_j) for e in R_t, 0 elsewhere.
__global__ void k_moe_router_bwd(const float* __restrict__ gate, const float* __restrict__ dgate,
                                 const int32_t* __restrict__ idx, int T, int k, int E, float* __restrict__ dlogits) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= T) return;
  float s = 0.f;
  for (int j = 0; j < k; ++j) s = fmaf(gate[t * k + j], dgate[t * k + j], s);
  float* row = dlogits + t * E;
  for (int e = 0; e < E; ++e) row[e] = 0.f;
  for (int j = 0; j < k; ++j) row[idx[t * k + j]] = gate[t * k + j] * (dgate[t * k + j] - s);
}

// Router weight gradient dWr[e, c] = sum_t dlogit[t, e] w[t, c], one thread per
// (e, c), tokens in increasing order.
__global__ void k_moe_router_dw(const float* __restrict__ dlogits, const bf16* __restrict__ w, int T, int d, int E,
                                float* __restrict__ dWr) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= (int64_t)E * d) return;
  const int e = (int)(i / d), c = (int)(i % d);
  float acc = 0.f;
  for (int t = 0; t < T; ++t) acc = fmaf(dlogits[(int64_t)t * E + e], bf(w[(int64_t)t * d + c]), acc);
  dWr[i] = acc;
}

// dw[t] = sum_e dlogit[t, e] Wr[e] + sum_j dxe[slot_of[t, j]] (the MLP input's
// gradient: router term, then the routed rows in slot order j).
__global__ void k_moe_dx(const float* __restrict__ dlogits, const bf16* __restrict__ Wr,
                         const float* __restrict__ dxe, const int32_t* __restrict__ slot_of, int T, int k, int d,
                         int E, float* __restrict__ dw) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < (int64_t)T * d;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / d;
    const int c = (int)(i % d);
    float acc = 0.f;
    for (int e = 0; e < E; ++e) acc = fmaf(dlogits[t * E + e], bf(Wr[(int64_t)e * d + c]), acc);
    for (int j = 0; j < k; ++j) acc += dxe[(int64_t)slot_of[t * k + j] * d + c];
    dw[i] = acc;
  }
}

inline int grid_for(int64_t n, int threads) {
  return (int)std::min<int64_t>((n + threads - 1) / threads, 148 * 16);
}

}  // namespace

int launch_moe_router(const void* w, const void* Wr, int T, int d, int E, int k, float* logits, int32_t* idx,
                      float* gate, cudaStream_t st) {
  if (T <= 0) return MT_OK;
  if (E < 1 || E > 64 || k < 1 || k > E || d % 64) return MT_ERR_ARG;
  k_moe_router<<<(T + 7) / 8, 256, 0, st>>>((const bf16*)w, (const bf16*)Wr, T, d, E, k, logits, idx, gate);
  return launch_status();
}

int launch_moe_gather(const void* w, const int32_t* row_of, int rows, int d, void* xe, cudaStream_t st) {
  if (rows <= 0) return MT_OK;
  k_moe_gather<<<grid_for((int64_t)rows * d / 8, 256), 256, 0, st>>>((const bf16*)w, row_of, rows, d, (bf16*)xe);
  return launch_status();
}

int launch_moe_combine(const float* h, const float* ye, const int32_t* slot_of, const float* gate, int T, int k,
                       int d, float* out, cudaStream_t st) {
  if (T <= 0) return MT_OK;
  k_moe_combine<<<grid_for((int64_t)T * d / 4, 256), 256, 0, st>>>(h, ye, slot_of, gate, T, k, d, out);
  return launch_status();
}

int launch_moe_dy(const float* dy, const float* ye, const int32_t* slot_of, const float* gate, int T, int k, int d,
                  void* dye, float* dgate, cudaStream_t st) {
  if (T <= 0) return MT_OK;
  const int64_t pairs = (int64_t)T * k;
  k_moe_dy<<<(int)((pairs + 7) / 8), 256, 0, st>>>(dy, ye, slot_of, gate, T, k, d, (bf16*)dye, dgate);
  return launch_status();
}

int launch_moe_router_bwd(const float* gate, const float* dgate, const int32_t* idx, const void* w, const void* Wr,
                          const float* dxe, const int32_t* slot_of, int T, int k, int d, int E, float* dlogits,
                          float* dWr, float* dw, cudaStream_t st) {
  if (T <= 0) return MT_OK;
  k_moe_router_bwd<<<(T + 255) / 256, 256, 0, st>>>(gate, dgate, idx, T, k, E, dlogits);
  if (cudaGetLastError() != cudaSuccess) return MT_ERR_CUDA;
  k_moe_router_dw<<<(int)(((int64_t)E * d + 127) / 128), 128, 0, st>>>(dlogits, (const bf16*)w, T, d, E, dWr);
  if (cudaGetLastError() != cudaSuccess) return MT_ERR_CUDA;
  k_moe_dx<<<grid_for((int64_t)T * d, 256), 256, 0, st>>>(dlogits, (const bf16*)Wr, dxe, slot_of, T, k, d, E, dw);
  return launch_status();
}

}  // namespace mt
