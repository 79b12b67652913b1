// Memory-bound kernels of the streamed decoder layer (sm_100a): RMSNorm
// forward/backward, RoPE, SwiGLU forward/backward, embedding gather and
// scatter-add, fused softmax cross-entropy, casts and fixed-order reductions.
//
// These are the non-matmul steps of the Llama-style block that MegaTrain streams
// layer by layer (MegaTrain abstract: stream parameters in, compute gradients
// out; intelligentliving.co "Checkpointing, Manual Gradients, and CPU-Side
// Optimizer Steps": hand-written gradients instead of autograd). Every kernel
// reads and writes contiguous rows with 16-byte vector accesses; reductions
// over tokens are done in a fixed order so results are run-to-run identical.
#include "mt_common.cuh"
#include "mt_internal.h"

namespace mt {

namespace {

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ void load_bf16x4(const bf16* p, float (&v)[4]) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
  v[0] = a.x;
  v[1] = a.y;
  v[2] = b.x;
  v[3] = b.y;
}
__device__ __forceinline__ void store_bf16x4(bf16* p, float a, float b, float c, float d) {
  uint2 u;
  u.x = pack_bf16x2(a, b);
  u.y = pack_bf16x2(c, d);
  *reinterpret_cast<uint2*>(p) = u;
}

// Block-wide sum for a block of 256 threads; every thread gets the result.
__device__ __forceinline__ float block_sum_256(float v, float* sh) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) sh[w] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) t += sh[i];
  return t;
}

// ---------------------------------------------------------------------------
// RMSNorm forward: y = x / sqrt(mean(x^2) + eps) * g, one warp per row.
// ---------------------------------------------------------------------------
__global__ void k_rmsnorm_fwd(const float* __restrict__ x, const bf16* __restrict__ g, bf16* __restrict__ y,
                              float* __restrict__ rstd, int T, int d, float eps) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (int64_t)row * d);
  const int n4 = d >> 2;
  float ss = 0.f;
  for (int i = lane; i < n4; i += 32) {
    float4 v = xr[i];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)d + eps);
  bf16* yr = y + (int64_t)row * d;
  for (int i = lane; i < n4; i += 32) {
    float4 v = xr[i];
    float gv[4];
    load_bf16x4(g + 4 * i, gv);
    store_bf16x4(yr + 4 * i, v.x * r * gv[0], v.y * r * gv[1], v.z * r * gv[2], v.w * r * gv[3]);
  }
  if (lane == 0 && rstd) rstd[row] = r;
}

// ---------------------------------------------------------------------------
// RMSNorm backward. For y_j = g_j x_j r, r = (mean x^2 + eps)^-1/2:
//   dx_j = dres_j + r g_j dy_j - x_j r^3 (sum_i g_i dy_i x_i) / d
//   dg_j = sum over rows of dy_j x_j r      (per-block partials, fixed order)
// A block of 256 threads owns a contiguous chunk of rows and takes them R at a
// time; thread t owns the float4 column groups t, t + 256, ... (K4 of them,
// d <= 1024 K4). The R rows' dot products are reduced together, with one
// barrier per group, so that R rows of loads are in flight per block; the
// reduction buffer alternates between two halves so the next group's writes
// cannot race this group's reads. Two blocks fit an SM.
// ---------------------------------------------------------------------------
constexpr int RMS_KMAX = 8;

template <int K4, int R>
__global__ void __launch_bounds__(256, 2) k_rmsnorm_bwd(const float* __restrict__ x, const bf16* __restrict__ g,
                                                        const float* __restrict__ rstd, const float* __restrict__ dy,
                                                        const float* __restrict__ dres, float* __restrict__ dx,
                                                        bf16* __restrict__ dx_bf16, float* __restrict__ dg_part,
                                                        int T, int d, int rows_per_block) {
  __shared__ float red[2][8][R];
  const int n4 = d >> 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float gv[K4][4];
  float acc[K4][4];
#pragma unroll
  for (int k = 0; k < K4; ++k) {
    const int c = threadIdx.x + k * 256;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[k][e] = 0.f;
    if (c < n4) {
      load_bf16x4(g + 4 * c, gv[k]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) gv[k][e] = 0.f;
    }
  }
  const int r0 = blockIdx.x * rows_per_block;
  const int r1 = min(T, r0 + rows_per_block);
  int half = 0;
  for (int row0 = r0; row0 < r1; row0 += R, half ^= 1) {
    float4 xv[R][K4], dv[R][K4];
    float rr[R], dot[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int row = row0 + q;
      const bool ok = row < r1;
      rr[q] = ok ? rstd[row] : 0.f;
      dot[q] = 0.f;
#pragma unroll
      for (int k = 0; k < K4; ++k) {
        const int c = threadIdx.x + k * 256;
        if (ok && c < n4) {
          xv[q][k] = reinterpret_cast<const float4*>(x + (int64_t)row * d)[c];
          dv[q][k] = reinterpret_cast<const float4*>(dy + (int64_t)row * d)[c];
        } else {
          xv[q][k] = make_float4(0.f, 0.f, 0.f, 0.f);
          dv[q][k] = xv[q][k];
        }
      }
    }
#pragma unroll
    for (int q = 0; q < R; ++q) {
#pragma unroll
      for (int k = 0; k < K4; ++k)
        dot[q] += gv[k][0] * dv[q][k].x * xv[q][k].x + gv[k][1] * dv[q][k].y * xv[q][k].y +
                  gv[k][2] * dv[q][k].z * xv[q][k].z + gv[k][3] * dv[q][k].w * xv[q][k].w;
      dot[q] = warp_sum(dot[q]);
    }
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < R; ++q) red[half][warp][q] = dot[q];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int row = row0 + q;
      if (row >= r1) break;
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) tot += red[half][w][q];
      const float r = rr[q];
      const float c3 = r * r * r * tot / (float)d;
#pragma unroll
      for (int k = 0; k < K4; ++k) {
        const int c = threadIdx.x + k * 256;
        if (c < n4) {
          const float4 dq = dv[q][k], xq = xv[q][k];
          float4 o;
          o.x = r * gv[k][0] * dq.x - xq.x * c3;
          o.y = r * gv[k][1] * dq.y - xq.y * c3;
          o.z = r * gv[k][2] * dq.z - xq.z * c3;
          o.w = r * gv[k][3] * dq.w - xq.w * c3;
          if (dres) {
            const float4 s = reinterpret_cast<const float4*>(dres + (int64_t)row * d)[c];
            o.x += s.x;
            o.y += s.y;
            o.z += s.z;
            o.w += s.w;
          }
          reinterpret_cast<float4*>(dx + (int64_t)row * d)[c] = o;
          if (dx_bf16) store_bf16x4(dx_bf16 + (int64_t)row * d + 4 * c, o.x, o.y, o.z, o.w);
          acc[k][0] += dq.x * xq.x * r;
          acc[k][1] += dq.y * xq.y * r;
          acc[k][2] += dq.z * xq.z * r;
          acc[k][3] += dq.w * xq.w * r;
        }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < K4; ++k) {
    const int c = threadIdx.x + k * 256;
    if (c < n4)
      reinterpret_cast<float4*>(dg_part + (int64_t)blockIdx.x * d)[c] =
          make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
  }
}

// Rows in flight per block: as many as keep the loads of a group within ~64
// registers per thread.
template <int K4>
void rmsnorm_bwd_k4(int nb, const float* x, const bf16* g, const float* rstd, const float* dy, const float* dres,
                    float* dx, bf16* dxb, float* part, int T, int d, int rpb, cudaStream_t st) {
  constexpr int R = K4 >= 5 ? 1 : 8 / K4;
  k_rmsnorm_bwd<K4, R><<<nb, 256, 0, st>>>(x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb);
}

void rmsnorm_bwd_kernel(int nb, const float* x, const bf16* g, const float* rstd, const float* dy, const float* dres,
                        float* dx, bf16* dxb, float* part, int T, int d, int rpb, cudaStream_t st) {
  switch (((d >> 2) + 255) / 256) {
    case 1: rmsnorm_bwd_k4<1>(nb, x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb, st); break;
    case 2: rmsnorm_bwd_k4<2>(nb, x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb, st); break;
    case 3: rmsnorm_bwd_k4<3>(nb, x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb, st); break;
    case 4: rmsnorm_bwd_k4<4>(nb, x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb, st); break;
    case 5: rmsnorm_bwd_k4<5>(nb, x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb, st); break;
    case 6: rmsnorm_bwd_k4<6>(nb, x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb, st); break;
    case 7: rmsnorm_bwd_k4<7>(nb, x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb, st); break;
    default: rmsnorm_bwd_k4<8>(nb, x, g, rstd, dy, dres, dx, dxb, part, T, d, rpb, st); break;
  }
}

// out[j] = sum_b part[b, j] in increasing b (fixed order).
__global__ void k_sum_rows(const float* __restrict__ part, int nb, int d, float* __restrict__ out) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= d) return;
  float s = 0.f;
  for (int b = 0; b < nb; ++b) s += part[(int64_t)b * d + j];
  out[j] = s;
}

// ---------------------------------------------------------------------------
// RoPE on bf16 q and k heads in place (rotate-half pairs (i, i + hd/2)).
// sign = +1: forward rotation by angle; -1: its transpose (backward).
// Thread = (token, head, pair i); heads [0, nheads) start at column `col0`.
// ---------------------------------------------------------------------------
__global__ void k_rope(bf16* __restrict__ buf, int64_t ld, int T, int s, int nheads, int hd, int col0,
                       const float* __restrict__ cosb, const float* __restrict__ sinb, float sign) {
  const int half = hd >> 1;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)T * nheads * (half >> 1);
  if (idx >= total) return;
  const int ip = (int)(idx % (half >> 1)) * 2;  // pair index, 2 at a time
  const int64_t th = idx / (half >> 1);
  const int h = (int)(th % nheads);
  const int t = (int)(th / nheads);
  const int pos = t % s;
  bf16* p = buf + (int64_t)t * ld + col0 + h * hd;
  const float2 c = *reinterpret_cast<const float2*>(cosb + (int64_t)pos * half + ip);
  float2 sn = *reinterpret_cast<const float2*>(sinb + (int64_t)pos * half + ip);
  sn.x *= sign;
  sn.y *= sign;
  const float2 a = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(p + ip));
  const float2 b = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(p + ip + half));
  *reinterpret_cast<uint32_t*>(p + ip) = pack_bf16x2(a.x * c.x - b.x * sn.x, a.y * c.y - b.y * sn.y);
  *reinterpret_cast<uint32_t*>(p + ip + half) = pack_bf16x2(b.x * c.x + a.x * sn.x, b.y * c.y + a.y * sn.y);
}

// ---------------------------------------------------------------------------
// SwiGLU. gu row = [gate (F) | up (F)], act = silu(gate) * up.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + expf(-z)); }

__global__ void k_swiglu_fwd(const bf16* __restrict__ gu, bf16* __restrict__ act, int T, int F) {
  const int64_t i8 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // 8 elements per thread
  const int f8 = F >> 3;
  if (i8 >= (int64_t)T * f8) return;
  const int64_t t = i8 / f8;
  const int j = (int)(i8 % f8) * 8;
  const uint4 gv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + j);
  const uint4 uv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + F + j);
  const uint32_t* g32 = reinterpret_cast<const uint32_t*>(&gv);
  const uint32_t* u32 = reinterpret_cast<const uint32_t*>(&uv);
  uint4 o;
  uint32_t* o32 = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 g2 = unpack_bf16x2(g32[e]), u2 = unpack_bf16x2(u32[e]);
    o32[e] = pack_bf16x2(g2.x * sigmoidf_(g2.x) * u2.x, g2.y * sigmoidf_(g2.y) * u2.y);
  }
  *reinterpret_cast<uint4*>(act + t * F + j) = o;
}

// dgate = dact * up * s (1 + gate (1 - s)), dup = dact * gate * s, s = sigmoid(gate).
__global__ void k_swiglu_bwd(const bf16* __restrict__ gu, const bf16* __restrict__ dact, bf16* __restrict__ dgu,
                             int T, int F) {
  const int64_t i8 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int f8 = F >> 3;
  if (i8 >= (int64_t)T * f8) return;
  const int64_t t = i8 / f8;
  const int j = (int)(i8 % f8) * 8;
  const uint4 gv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + j);
  const uint4 uv = *reinterpret_cast<const uint4*>(gu + t * 2 * F + F + j);
  const uint4 dv = *reinterpret_cast<const uint4*>(dact + t * F + j);
  const uint32_t* g32 = reinterpret_cast<const uint32_t*>(&gv);
  const uint32_t* u32 = reinterpret_cast<const uint32_t*>(&uv);
  const uint32_t* d32 = reinterpret_cast<const uint32_t*>(&dv);
  uint4 og, ou;
  uint32_t* og32 = reinterpret_cast<uint32_t*>(&og);
  uint32_t* ou32 = reinterpret_cast<uint32_t*>(&ou);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 g2 = unpack_bf16x2(g32[e]), u2 = unpack_bf16x2(u32[e]), d2 = unpack_bf16x2(d32[e]);
    const float s0 = sigmoidf_(g2.x), s1 = sigmoidf_(g2.y);
    og32[e] = pack_bf16x2(d2.x * u2.x * s0 * (1.f + g2.x * (1.f - s0)), d2.y * u2.y * s1 * (1.f + g2.y * (1.f - s1)));
    ou32[e] = pack_bf16x2(d2.x * g2.x * s0, d2.y * g2.y * s1);
  }
  *reinterpret_cast<uint4*>(dgu + t * 2 * F + j) = og;
  *reinterpret_cast<uint4*>(dgu + t * 2 * F + F + j) = ou;
}

// ---------------------------------------------------------------------------
// Embedding gather: x[t] = E[tok[t]] (bf16 -> fp32), one warp per token.
// E may be a device pointer or a mapped pointer to pinned host memory.
// ---------------------------------------------------------------------------
__global__ void k_embed_fwd(const int* __restrict__ tok, const bf16* __restrict__ E, float* __restrict__ x, int T,
                            int d) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const bf16* er = E + (int64_t)tok[t] * d;
  float* xr = x + (int64_t)t * d;
  for (int j = lane * 8; j < d; j += 256) {
    const uint4 v = *reinterpret_cast<const uint4*>(er + j);
    const uint32_t* v32 = reinterpret_cast<const uint32_t*>(&v);
    float2 a = unpack_bf16x2(v32[0]), b = unpack_bf16x2(v32[1]), c = unpack_bf16x2(v32[2]),
           e = unpack_bf16x2(v32[3]);
    reinterpret_cast<float4*>(xr + j)[0] = make_float4(a.x, a.y, b.x, b.y);
    reinterpret_cast<float4*>(xr + j)[1] = make_float4(c.x, c.y, e.x, e.y);
  }
}

// Embedding backward: for unique token u, dE_rows[u] = sum of dx over its
// positions, in increasing position order (pos[offs[u] .. offs[u+1])).
__global__ void k_embed_bwd(const int* __restrict__ offs, const int* __restrict__ pos, const float* __restrict__ dx,
                            float* __restrict__ rows, int d) {
  const int u = blockIdx.x;
  const int a = offs[u], b = offs[u + 1];
  for (int j = threadIdx.x * 4; j < d; j += blockDim.x * 4) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = a; i < b; ++i) {
      const float4 v = *reinterpret_cast<const float4*>(dx + (int64_t)pos[i] * d + j);
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    *reinterpret_cast<float4*>(rows + (int64_t)u * d + j) = s;
  }
}

// ---------------------------------------------------------------------------
// Fused softmax cross-entropy over fp32 logits z [Tc, V] (row pitch ldz):
//   loss_t = logsumexp(z_t) - z_t[y_t]
//   dz_t   = (softmax(z_t) - onehot(y_t)) * scale      (bf16, pitch lddz)
// One 256-thread block per row; V % 4 == 0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_softmax_ce(const float* __restrict__ z, int64_t ldz,
                                                    const int* __restrict__ labels, bf16* __restrict__ dz,
                                                    int64_t lddz, float* __restrict__ row_loss, int V, float scale) {
  __shared__ float shm[8], shs[8];
  const int row = blockIdx.x;
  const float4* zr = reinterpret_cast<const float4*>(z + (int64_t)row * ldz);
  const int n4 = V >> 2;
  float m = -INFINITY, sum = 0.f;
  for (int i = threadIdx.x; i < n4; i += 256) {
    const float4 v = zr[i];
    const float mx = fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w));
    if (mx > m) {
      sum *= expf(m - mx);
      m = mx;
    }
    sum += expf(v.x - m) + expf(v.y - m) + expf(v.z - m) + expf(v.w - m);
  }
  // combine (m, sum) across the block
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, sum, o);
    const float mn = fmaxf(m, m2);
    sum = (m == -INFINITY ? 0.f : sum * expf(m - mn)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - mn));
    m = mn;
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    shm[w] = m;
    shs[w] = sum;
  }
  __syncthreads();
  float M = shm[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) M = fmaxf(M, shm[i]);
  float S = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) S += shs[i] * expf(shm[i] - M);
  const float lse = M + logf(S);
  const int y = labels[row];
  if (threadIdx.x == 0) row_loss[row] = lse - z[(int64_t)row * ldz + y];
  bf16* dr = dz + (int64_t)row * lddz;
  for (int i = threadIdx.x; i < n4; i += 256) {
    const float4 v = zr[i];
    const int j = 4 * i;
    float p0 = expf(v.x - lse), p1 = expf(v.y - lse), p2 = expf(v.z - lse), p3 = expf(v.w - lse);
    if (y == j) p0 -= 1.f;
    if (y == j + 1) p1 -= 1.f;
    if (y == j + 2) p2 -= 1.f;
    if (y == j + 3) p3 -= 1.f;
    store_bf16x4(dr + j, p0 * scale, p1 * scale, p2 * scale, p3 * scale);
  }
}

// Sum of n floats by one block, fixed order (per-thread strided, then a tree).
__global__ void k_sum_all(const float* __restrict__ v, int n, float* __restrict__ out, int accumulate) {
  __shared__ float sh[8];
  float s = 0.f;
  for (int i = threadIdx.x; i < n; i += 256) s += v[i];
  s = block_sum_256(s, sh);
  if (threadIdx.x == 0) *out = accumulate ? *out + s : s;
}

__global__ void k_cast_f32_bf16(const float* __restrict__ in, bf16* __restrict__ out, int64_t n4) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(in)[i];
  store_bf16x4(out + 4 * i, v.x, v.y, v.z, v.w);
}

inline int nblk(int64_t n, int per) { return (int)((n + per - 1) / per); }

thread_local const char* g_launch_error = "";

}  // namespace

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return MT_OK;
  g_launch_error = cudaGetErrorString(e);
  return MT_ERR_CUDA;
}

const char* last_launch_error() { return g_launch_error; }

// ---------------------------------------------------------------------------
// Launchers (shape checks are the caller's; these only enqueue).
// ---------------------------------------------------------------------------
int launch_rmsnorm_fwd(const float* x, const void* g, void* y, float* rstd, int T, int d, float eps, cudaStream_t st) {
  if (T <= 0) return MT_OK;
  k_rmsnorm_fwd<<<nblk(T, 8), 256, 0, st>>>(x, (const bf16*)g, (bf16*)y, rstd, T, d, eps);
  return launch_status();
}

int rmsnorm_bwd_blocks(int T) { return T < 296 ? (T > 0 ? T : 1) : 296; }

int launch_rmsnorm_bwd(const float* x, const void* g, const float* rstd, const float* dy, const float* dres,
                       float* dx, void* dx_bf16, float* dg_part, float* dg, int T, int d, cudaStream_t st) {
  if (T <= 0) return MT_OK;
  if (d > 256 * 4 * RMS_KMAX) return MT_ERR_CONFIG;
  const int nb = rmsnorm_bwd_blocks(T);
  const int rpb = (T + nb - 1) / nb;
  rmsnorm_bwd_kernel(nb, x, (const bf16*)g, rstd, dy, dres, dx, (bf16*)dx_bf16, dg_part, T, d, rpb, st);
  k_sum_rows<<<nblk(d, 256), 256, 0, st>>>(dg_part, nb, d, dg);
  return launch_status();
}

int launch_rope(void* buf, int64_t ld, int T, int s, int nheads, int hd, int col0, const float* cosb,
                const float* sinb, float sign, cudaStream_t st) {
  const int64_t total = (int64_t)T * nheads * (hd / 4);
  if (total <= 0) return MT_OK;
  k_rope<<<nblk(total, 256), 256, 0, st>>>((bf16*)buf, ld, T, s, nheads, hd, col0, cosb, sinb, sign);
  return launch_status();
}

int launch_swiglu_fwd(const void* gu, void* act, int T, int F, cudaStream_t st) {
  const int64_t n = (int64_t)T * (F / 8);
  if (n <= 0) return MT_OK;
  k_swiglu_fwd<<<nblk(n, 256), 256, 0, st>>>((const bf16*)gu, (bf16*)act, T, F);
  return launch_status();
}

int launch_swiglu_bwd(const void* gu, const void* dact, void* dgu, int T, int F, cudaStream_t st) {
  const int64_t n = (int64_t)T * (F / 8);
  if (n <= 0) return MT_OK;
  k_swiglu_bwd<<<nblk(n, 256), 256, 0, st>>>((const bf16*)gu, (const bf16*)dact, (bf16*)dgu, T, F);
  return launch_status();
}

int launch_embed_fwd(const int* tok, const void* E, float* x, int T, int d, cudaStream_t st) {
  if (T <= 0) return MT_OK;
  k_embed_fwd<<<nblk(T, 8), 256, 0, st>>>(tok, (const bf16*)E, x, T, d);
  return launch_status();
}

int launch_embed_bwd(const int* offs, const int* pos, int n_unique, const float* dx, float* rows, int d,
                     cudaStream_t st) {
  if (n_unique <= 0) return MT_OK;
  k_embed_bwd<<<n_unique, 128, 0, st>>>(offs, pos, dx, rows, d);
  return launch_status();
}

int launch_softmax_ce(const float* z, int64_t ldz, const int* labels, void* dz, int64_t lddz, float* row_loss,
                      int Tc, int V, float scale, cudaStream_t st) {
  if (Tc <= 0) return MT_OK;
  k_softmax_ce<<<Tc, 256, 0, st>>>(z, ldz, labels, (bf16*)dz, lddz, row_loss, V, scale);
  return launch_status();
}

int launch_sum_all(const float* v, int n, float* out, int accumulate, cudaStream_t st) {
  k_sum_all<<<1, 256, 0, st>>>(v, n, out, accumulate);
  return launch_status();
}

int launch_cast_f32_bf16(const float* in, void* out, int64_t n, cudaStream_t st) {
  if (n <= 0) return MT_OK;
  k_cast_f32_bf16<<<nblk(n / 4, 256), 256, 0, st>>>(in, (bf16*)out, n / 4);
  return launch_status();
}

}  // namespace mt

// ---------------------------------------------------------------------------
// RMSNorm backward without any allocation by caller or library.
//
// The per-block partial sums of dg live in this fixed device array instead of
// a caller buffer. Host code must not pass the array's name to a kernel (in
// host code it is only a stand-in for the device symbol): the device address
// is looked up with cudaGetSymbolAddress on every call, with the caller's
// device current. Nothing is cached, so the address stays right after a
// device reset or a context re-creation, which may reload the module at
// another address.
// ---------------------------------------------------------------------------
namespace mt {
namespace {

constexpr int kNoAllocScratchFloats = 1 << 20;  // 4 MiB per device that loads the library
static __device__ __align__(256) float g_rmsnorm_scratch[kNoAllocScratchFloats];

// Address of the scratch array on the current device.
int scratch_address(float** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_rmsnorm_scratch) != cudaSuccess || !p) return MT_ERR_CUDA;
  *out = static_cast<float*>(p);
  return MT_OK;
}

}  // namespace
}  // namespace mt

extern "C" int mt_k_rmsnorm_bwd_noalloc(const float* x, const void* g, const float* rstd, const float* dy,
                                        const float* dres, float* dx, void* dx_bf16, float* dg, int T, int d,
                                        void* stream) {
  using namespace mt;
  if (!x || !g || !rstd || !dy || !dx || !dg || T < 0 || d <= 0 || (d % 4)) return MT_ERR_ARG;
  if (d > 256 * 4 * RMS_KMAX) return MT_ERR_ARG;  // beyond the widest row the kernel (and scratch) supports
  if (T == 0) return MT_OK;
  float* part = nullptr;
  if (scratch_address(&part) != MT_OK) return MT_ERR_CUDA;
  // As many row blocks as the regular entry point uses, capped so that
  // blocks x d partials fit in the fixed scratch array.
  int nb = rmsnorm_bwd_blocks(T);
  const int cap = kNoAllocScratchFloats / d;
  if (nb > cap) nb = cap;
  const int rpb = (T + nb - 1) / nb;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Every block writes its own partial row (zeros when it owns no rows), so
  // stale contents from an earlier call are never read.
  rmsnorm_bwd_kernel(nb, x, (const bf16*)g, rstd, dy, dres, dx, (bf16*)dx_bf16, part, T, d, rpb, st);
  k_sum_rows<<<nblk(d, 256), 256, 0, st>>>(part, nb, d, dg);
  return launch_status();
}
