// Causal flash attention forward and backward with grouped KV heads (sm_100a).
//
// The attention of the streamed decoder layer: a = softmax(q k^T / sqrt(hd) +
// causal mask) v per head, query head h reading KV head h / (H / Hkv). The
// forward keeps only the output and the per-row log-sum-exp; the backward
// recomputes the probabilities from them (the same compute-for-memory trade
// the MegaTrain pages make with activation checkpointing: intelligentliving.co,
// "Checkpointing, Manual Gradients, and CPU-Side Optimizer Steps").
//
// Tiles of 64 queries x 64 keys, bf16 operands through ldmatrix and
// mma.sync.m16n8k16 with fp32 accumulation, online softmax in registers,
// swizzled shared memory, cp.async double buffering of K/V in the forward.
// Backward: one CTA per (64-key block, KV head, sequence) accumulates dK and dV
// in registers over every query head of its group and every query block at or
// after its keys; dQ is accumulated in fp32 with vector atomics.
//
// Layout: q, k, v are column ranges of one bf16 row per token (pitch ldqkv),
// tokens sequence-major (t = b * s + i); LSE and D are fp32 [b, H, s].
#include "mt_common.cuh"
#include "mt_internal.h"

namespace mt {

namespace {

typedef __nv_bfloat16 bf16;
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Element (r, c) of a tile with rows of HD bf16: 16-byte chunks XOR-swizzled by
// the row so that ldmatrix of 8 rows at one chunk column hits 8 bank groups.
template <int HD>
__device__ __forceinline__ int swz(int r, int c) {
  return r * HD + ((((c >> 3) ^ (r & 7))) << 3) + (c & 7);
}
// Rows of 32 bf16 (4 chunks): swizzle by (r / 2) so 8 consecutive rows differ.
__device__ __forceinline__ int swz32(int r, int c) { return r * 32 + ((((c >> 3) ^ ((r >> 1) & 3))) << 3) + (c & 7); }

// Async copy of R rows x HD columns (row pitch ld) into a swizzled tile; rows
// at or beyond rows_valid are zero-filled.
template <int R, int HD, int NT>
__device__ __forceinline__ void load_tile(bf16* sm, const bf16* g, int64_t ld, int rows_valid) {
  constexpr int CH = HD / 8;
  for (int i = threadIdx.x; i < R * CH; i += NT) {
    const int r = i / CH, c = i % CH;
    const bool v = r < rows_valid;
    cp_async16(smem_u32(sm + swz<HD>(r, c * 8)), v ? (const void*)(g + (int64_t)r * ld + c * 8) : (const void*)g, v);
  }
}

// ---------------------------------------------------------------------------
// Forward.
// ---------------------------------------------------------------------------
template <int HD>
__global__ void __launch_bounds__(128) k_flash_fwd(const bf16* __restrict__ Q, const bf16* __restrict__ K,
                                                   const bf16* __restrict__ V, int64_t ldqkv, bf16* __restrict__ O,
                                                   int64_t ldo, float* __restrict__ LSE, int s, int H, int Hkv,
                                                   float scale) {
  constexpr int BQ = 64, BKV = 64;
  extern __shared__ __align__(128) uint8_t smraw[];
  bf16* sQ = reinterpret_cast<bf16*>(smraw);
  bf16* sK = sQ + BQ * HD;
  bf16* sV = sK + 2 * BKV * HD;

  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (H / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int q0 = qb * BQ;
  const int64_t tb = (int64_t)b * s;
  const bf16* Qb = Q + (tb + q0) * ldqkv + h * HD;
  const bf16* Kb = K + tb * ldqkv + kvh * HD;
  const bf16* Vb = V + tb * ldqkv + kvh * HD;
  const int nkv = qb + 1;

  load_tile<BQ, HD, 128>(sQ, Qb, ldqkv, s - q0);
  load_tile<BKV, HD, 128>(sK, Kb, ldqkv, s);
  load_tile<BKV, HD, 128>(sV, Vb, ldqkv, s);
  cp_commit();

  float o[HD / 8][4];
#pragma unroll
  for (int n = 0; n < HD / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  uint32_t qf[HD / 16][4];
  const float sl2 = scale * LOG2E;
  const int mi = lane >> 3;

  for (int j = 0; j < nkv; ++j) {
    if (j + 1 < nkv) {
      const int nb = (j + 1) & 1;
      load_tile<BKV, HD, 128>(sK + nb * BKV * HD, Kb + (int64_t)(j + 1) * BKV * ldqkv, ldqkv, s - (j + 1) * BKV);
      load_tile<BKV, HD, 128>(sV + nb * BKV * HD, Vb + (int64_t)(j + 1) * BKV * ldqkv, ldqkv, s - (j + 1) * BKV);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk)
        ldsm_x4(smem_u32(sQ + swz<HD>(warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8)), qf[kk][0], qf[kk][1],
                qf[kk][2], qf[kk][3]);
    }
    const bf16* ks = sK + (j & 1) * BKV * HD;
    const bf16* vs = sV + (j & 1) * BKV * HD;

    float sc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[n][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(ks + swz<HD>(np * 16 + (lane & 7) + 8 * (mi >> 1), kk * 16 + (mi & 1) * 8)), b0, b1, b2, b3);
        mma16816(sc[2 * np], qf[kk], b0, b1);
        mma16816(sc[2 * np + 1], qf[kk], b2, b3);
      }
    }
    if (j == qb) {  // diagonal block: key index must not exceed query index
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qi = warp * 16 + gq + 8 * (e >> 1);
          const int kj = n * 8 + 2 * tq + (e & 1);
          if (kj > qi) sc[n][e] = -INFINITY;
        }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int n = 0; n < 8; ++n) mx = fmaxf(mx, fmaxf(sc[n][2 * r], sc[n][2 * r + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(mrow[r], mx);
      const float corr = (mrow[r] == -INFINITY) ? 0.f : exp2f((mrow[r] - mnew) * sl2);
      mrow[r] = mnew;
      lrow[r] *= corr;
#pragma unroll
      for (int n = 0; n < HD / 8; ++n) {
        o[n][2 * r] *= corr;
        o[n][2 * r + 1] *= corr;
      }
      const float mb = mnew * sl2;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const float p0 = exp2f(sc[n][2 * r] * sl2 - mb);
        const float p1 = exp2f(sc[n][2 * r + 1] * sl2 - mb);
        sc[n][2 * r] = p0;
        sc[n][2 * r + 1] = p1;
        lrow[r] += p0 + p1;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
      a[1] = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
      a[2] = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      a[3] = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
      for (int np = 0; np < HD / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(vs + swz<HD>(kk * 16 + (lane & 7) + 8 * (mi & 1), np * 16 + (mi >> 1) * 8)), b0, b1, b2,
                  b3);
        mma16816(o[2 * np], a, b0, b1);
        mma16816(o[2 * np + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = lrow[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = 1.f / l;
    const int qi = q0 + warp * 16 + gq + 8 * r;
    if (qi < s) {
      bf16* orow = O + (tb + qi) * ldo + h * HD;
#pragma unroll
      for (int n = 0; n < HD / 8; ++n)
        *reinterpret_cast<uint32_t*>(orow + n * 8 + 2 * tq) = pack_bf16x2(o[n][2 * r] * inv, o[n][2 * r + 1] * inv);
      if (tq == 0) LSE[((int64_t)b * H + h) * s + qi] = mrow[r] * scale + logf(l);
    }
  }
}

// ---------------------------------------------------------------------------
// Backward preprocessing: D[b,h,i] = sum_e dO[t,h,e] O[t,h,e]; one warp per (t,h).
// ---------------------------------------------------------------------------
__global__ void k_attn_bwd_pre(const bf16* __restrict__ O, const bf16* __restrict__ dO, int64_t ldo,
                               float* __restrict__ D, int T, int s, int H, int hd) {
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (int64_t)T * H) return;
  const int64_t t = w / H;
  const int h = (int)(w % H);
  const bf16* o = O + t * ldo + h * hd;
  const bf16* d = dO + t * ldo + h * hd;
  float acc = 0.f;
  for (int e = lane * 2; e < hd; e += 64) {
    const float2 a = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(o + e));
    const float2 c = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(d + e));
    acc += a.x * c.x + a.y * c.y;
  }
  acc = warp_sum(acc);
  if (lane == 0) {
    const int64_t bi = t / s, i = t % s;
    D[(bi * H + h) * s + i] = acc;
  }
}

// ---------------------------------------------------------------------------
// Backward main kernel.
// ---------------------------------------------------------------------------
template <int HD>
__global__ void __launch_bounds__(128) k_flash_bwd(const bf16* __restrict__ Q, const bf16* __restrict__ K,
                                                   const bf16* __restrict__ V, int64_t ldqkv,
                                                   const bf16* __restrict__ dO, int64_t ldo,
                                                   const float* __restrict__ LSE, const float* __restrict__ Dv,
                                                   float* __restrict__ dQacc, int64_t ldqa, bf16* __restrict__ dK,
                                                   bf16* __restrict__ dV, int64_t lddkv, int s, int H, int Hkv,
                                                   float scale, const float* __restrict__ rcos,
                                                   const float* __restrict__ rsin) {
  constexpr int BKV = 64, BQ = 32;
  extern __shared__ __align__(128) uint8_t smraw[];
  bf16* sK = reinterpret_cast<bf16*>(smraw);
  bf16* sV = sK + BKV * HD;
  bf16* sQ = sV + BKV * HD;
  bf16* sdO = sQ + BQ * HD;
  bf16* sdS = sdO + BQ * HD;
  float* sL = reinterpret_cast<float*>(sdS + BKV * BQ);
  float* sD = sL + BQ;

  const int kvb = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int group = H / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3, mi = lane >> 3;
  const int kv0 = kvb * BKV;
  const int64_t tb = (int64_t)b * s;
  const float sl2 = scale * LOG2E;

  load_tile<BKV, HD, 128>(sK, K + (tb + kv0) * ldqkv + kvh * HD, ldqkv, s - kv0);
  load_tile<BKV, HD, 128>(sV, V + (tb + kv0) * ldqkv + kvh * HD, ldqkv, s - kv0);
  cp_commit();

  float dk[HD / 8][4], dv[HD / 8][4];
#pragma unroll
  for (int n = 0; n < HD / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dk[n][e] = 0.f;
      dv[n][e] = 0.f;
    }

  for (int hh = 0; hh < group; ++hh) {
    const int h = kvh * group + hh;
    const float* Lh = LSE + ((int64_t)b * H + h) * s;
    const float* Dh = Dv + ((int64_t)b * H + h) * s;
    for (int q0 = kv0; q0 < s; q0 += BQ) {
      load_tile<BQ, HD, 128>(sQ, Q + (tb + q0) * ldqkv + h * HD, ldqkv, s - q0);
      load_tile<BQ, HD, 128>(sdO, dO + (tb + q0) * ldo + h * HD, ldo, s - q0);
      cp_commit();
      if (threadIdx.x < BQ) {
        const int qi = q0 + threadIdx.x;
        sL[threadIdx.x] = qi < s ? Lh[qi] : 0.f;
        sD[threadIdx.x] = qi < s ? Dh[qi] : 0.f;
      }
      cp_wait<0>();
      __syncthreads();

      // S^T = K Q^T for this warp's 16 keys x 32 queries.
      float st[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        uint32_t ka[4];
        ldsm_x4(smem_u32(sK + swz<HD>(warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8)), ka[0], ka[1], ka[2],
                ka[3]);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(sQ + swz<HD>(np * 16 + (lane & 7) + 8 * (mi >> 1), kk * 16 + (mi & 1) * 8)), b0, b1, b2,
                  b3);
          mma16816(st[2 * np], ka, b0, b1);
          mma16816(st[2 * np + 1], ka, b2, b3);
        }
      }
      // P^T (masked: key <= query, both inside the sequence).
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kj = kv0 + warp * 16 + gq + 8 * (e >> 1);
          const int ql = n * 8 + 2 * tq + (e & 1);
          const int qi = q0 + ql;
          st[n][e] = (kj <= qi && qi < s && kj < s) ? exp2f(st[n][e] * sl2 - sL[ql] * LOG2E) : 0.f;
        }
      // dV += P^T dO
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16x2(st[2 * kk][0], st[2 * kk][1]);
        a[1] = pack_bf16x2(st[2 * kk][2], st[2 * kk][3]);
        a[2] = pack_bf16x2(st[2 * kk + 1][0], st[2 * kk + 1][1]);
        a[3] = pack_bf16x2(st[2 * kk + 1][2], st[2 * kk + 1][3]);
#pragma unroll
        for (int np = 0; np < HD / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(sdO + swz<HD>(kk * 16 + (lane & 7) + 8 * (mi & 1), np * 16 + (mi >> 1) * 8)), b0, b1,
                    b2, b3);
          mma16816(dv[2 * np], a, b0, b1);
          mma16816(dv[2 * np + 1], a, b2, b3);
        }
      }
      // dP^T = V dO^T
      float dp[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dp[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        uint32_t va[4];
        ldsm_x4(smem_u32(sV + swz<HD>(warp * 16 + (lane & 15), kk * 16 + (lane >> 4) * 8)), va[0], va[1], va[2],
                va[3]);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(sdO + swz<HD>(np * 16 + (lane & 7) + 8 * (mi >> 1), kk * 16 + (mi & 1) * 8)), b0, b1, b2,
                  b3);
          mma16816(dp[2 * np], va, b0, b1);
          mma16816(dp[2 * np + 1], va, b2, b3);
        }
      }
      // dS^T = P^T * (dP^T - D)
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dp[n][e] = st[n][e] * (dp[n][e] - sD[n * 8 + 2 * tq + (e & 1)]);
      // dK += dS^T Q, and stage dS^T (bf16) for dQ.
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16x2(dp[2 * kk][0], dp[2 * kk][1]);
        a[1] = pack_bf16x2(dp[2 * kk][2], dp[2 * kk][3]);
        a[2] = pack_bf16x2(dp[2 * kk + 1][0], dp[2 * kk + 1][1]);
        a[3] = pack_bf16x2(dp[2 * kk + 1][2], dp[2 * kk + 1][3]);
        const int r0 = warp * 16 + gq;
        *reinterpret_cast<uint32_t*>(sdS + swz32(r0, kk * 16 + 2 * tq)) = a[0];
        *reinterpret_cast<uint32_t*>(sdS + swz32(r0 + 8, kk * 16 + 2 * tq)) = a[1];
        *reinterpret_cast<uint32_t*>(sdS + swz32(r0, kk * 16 + 8 + 2 * tq)) = a[2];
        *reinterpret_cast<uint32_t*>(sdS + swz32(r0 + 8, kk * 16 + 8 + 2 * tq)) = a[3];
#pragma unroll
        for (int np = 0; np < HD / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(sQ + swz<HD>(kk * 16 + (lane & 7) + 8 * (mi & 1), np * 16 + (mi >> 1) * 8)), b0, b1, b2,
                    b3);
          mma16816(dk[2 * np], a, b0, b1);
          mma16816(dk[2 * np + 1], a, b2, b3);
        }
      }
      __syncthreads();
      // dQ[32 q, HD] += dS K; warp w owns columns [w*HD/4, (w+1)*HD/4).
      constexpr int NT = HD / 32;  // n-tiles of 8 per warp
      float dq[2][NT][4];
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) dq[m][n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < BKV / 16; ++kk) {
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          uint32_t a[4];
          ldsm_x4_t(smem_u32(sdS + swz32(kk * 16 + (lane & 7) + 8 * (mi >> 1), m * 16 + (mi & 1) * 8)), a[0], a[1],
                    a[2], a[3]);
#pragma unroll
          for (int np = 0; np < NT / 2; ++np) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(smem_u32(sK + swz<HD>(kk * 16 + (lane & 7) + 8 * (mi & 1),
                                            warp * (HD / 4) + np * 16 + (mi >> 1) * 8)),
                      b0, b1, b2, b3);
            mma16816(dq[m][2 * np], a, b0, b1);
            mma16816(dq[m][2 * np + 1], a, b2, b3);
          }
        }
      }
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int qi = q0 + m * 16 + gq + 8 * r;
          if (qi < s) {
            float* dst = dQacc + (tb + qi) * ldqa + h * HD + warp * (HD / 4) + 2 * tq;
#pragma unroll
            for (int n = 0; n < NT; ++n)
              atomicAdd(reinterpret_cast<float2*>(dst + n * 8),
                        make_float2(dq[m][n][2 * r] * scale, dq[m][n][2 * r + 1] * scale));
          }
        }
      __syncthreads();
    }
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int kj = kv0 + warp * 16 + gq + 8 * r;
    if (kj < s) {
      bf16* kr = dK + (tb + kj) * lddkv + kvh * HD + 2 * tq;
      bf16* vr = dV + (tb + kj) * lddkv + kvh * HD + 2 * tq;
      if (rcos) {
        // gradient w.r.t. k before RoPE: transposed rotation of the pair
        // (i, i + HD/2); this thread holds both, in n-tiles n and n + HD/16.
        const float* cs = rcos + (int64_t)kj * (HD / 2);
        const float* sn = rsin + (int64_t)kj * (HD / 2);
#pragma unroll
        for (int n = 0; n < HD / 16; ++n) {
          const int i0 = n * 8 + 2 * tq;
          float a[2], bb[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float x1 = dk[n][2 * r + e] * scale, x2 = dk[n + HD / 16][2 * r + e] * scale;
            a[e] = x1 * cs[i0 + e] + x2 * sn[i0 + e];
            bb[e] = x2 * cs[i0 + e] - x1 * sn[i0 + e];
          }
          *reinterpret_cast<uint32_t*>(kr + n * 8) = pack_bf16x2(a[0], a[1]);
          *reinterpret_cast<uint32_t*>(kr + (n + HD / 16) * 8) = pack_bf16x2(bb[0], bb[1]);
        }
      } else {
#pragma unroll
        for (int n = 0; n < HD / 8; ++n)
          *reinterpret_cast<uint32_t*>(kr + n * 8) = pack_bf16x2(dk[n][2 * r] * scale, dk[n][2 * r + 1] * scale);
      }
#pragma unroll
      for (int n = 0; n < HD / 8; ++n)
        *reinterpret_cast<uint32_t*>(vr + n * 8) = pack_bf16x2(dv[n][2 * r], dv[n][2 * r + 1]);
    }
  }
}

// dQ (fp32 [T, H*hd], pitch ldqa) -> bf16 columns of dqkv (pitch ld). With
// RoPE tables the transposed rotation is applied on the way (pairs (i, i+hd/2)
// of each head at position t % s). Thread = 4 consecutive pairs.
__global__ void k_dq_cast(const float* __restrict__ dq, int64_t ldqa, bf16* __restrict__ out, int64_t ld, int T,
                          int H, int hd, int s, const float* __restrict__ rcos, const float* __restrict__ rsin) {
  const int half = hd >> 1;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int per_row = H * (half >> 2);
  if (i >= (int64_t)T * per_row) return;
  const int64_t t = i / per_row;
  const int k = (int)(i % per_row);
  const int h = k / (half >> 2);
  const int c = (k % (half >> 2)) * 4;  // pair index 0..half-1
  const float* src = dq + t * ldqa + h * hd;
  float4 a = *reinterpret_cast<const float4*>(src + c);
  float4 b = *reinterpret_cast<const float4*>(src + c + half);
  if (rcos) {
    const int pos = (int)(t % s);
    const float4 cs = *reinterpret_cast<const float4*>(rcos + (int64_t)pos * half + c);
    const float4 sn = *reinterpret_cast<const float4*>(rsin + (int64_t)pos * half + c);
    const float4 a0 = a, b0 = b;
    a = make_float4(a0.x * cs.x + b0.x * sn.x, a0.y * cs.y + b0.y * sn.y, a0.z * cs.z + b0.z * sn.z,
                    a0.w * cs.w + b0.w * sn.w);
    b = make_float4(b0.x * cs.x - a0.x * sn.x, b0.y * cs.y - a0.y * sn.y, b0.z * cs.z - a0.z * sn.z,
                    b0.w * cs.w - a0.w * sn.w);
  }
  bf16* o = out + t * ld + h * hd;
  *reinterpret_cast<uint2*>(o + c) = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  *reinterpret_cast<uint2*>(o + c + half) = make_uint2(pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

template <int HD>
int fwd_impl(const AttnArgs& a, cudaStream_t st) {
  constexpr int SMEM = (64 * HD + 4 * 64 * HD) * 2;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(k_flash_fwd<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess)
      return MT_ERR_CUDA;
    attr = true;
  }
  dim3 grid((a.s + 63) / 64, a.H, a.b);
  k_flash_fwd<HD><<<grid, 128, SMEM, st>>>((const bf16*)a.q, (const bf16*)a.k, (const bf16*)a.v, a.ldqkv,
                                           (bf16*)a.o, a.ldo, a.lse, a.s, a.H, a.Hkv, a.scale);
  return launch_status();
}

template <int HD>
int bwd_impl(const AttnArgs& a, cudaStream_t st) {
  constexpr int SMEM = (2 * 64 * HD + 2 * 32 * HD + 64 * 32) * 2 + 2 * 32 * 4;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(k_flash_bwd<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess)
      return MT_ERR_CUDA;
    attr = true;
  }
  const int T = a.b * a.s;
  const int64_t nw = (int64_t)T * a.H;
  k_attn_bwd_pre<<<(int)((nw + 7) / 8), 256, 0, st>>>((const bf16*)a.o, (const bf16*)a.dout, a.ldo, a.dvec, T, a.s,
                                                      a.H, HD);
  if (cudaMemsetAsync(a.dq_acc, 0, (size_t)T * a.ldqa * sizeof(float), st) != cudaSuccess) return MT_ERR_CUDA;
  dim3 grid((a.s + 63) / 64, a.Hkv, a.b);
  k_flash_bwd<HD><<<grid, 128, SMEM, st>>>((const bf16*)a.q, (const bf16*)a.k, (const bf16*)a.v, a.ldqkv,
                                           (const bf16*)a.dout, a.ldo, a.lse, a.dvec, a.dq_acc, a.ldqa,
                                           (bf16*)a.dk, (bf16*)a.dv, a.lddkv, a.s, a.H, a.Hkv, a.scale, a.rope_cos,
                                           a.rope_sin);
  const int64_t nthr = (int64_t)T * a.H * (HD / 8);
  k_dq_cast<<<(int)((nthr + 255) / 256), 256, 0, st>>>(a.dq_acc, a.ldqa, (bf16*)a.dq, a.lddq, T, a.H, HD, a.s,
                                                       a.rope_cos, a.rope_sin);
  return launch_status();
}

}  // namespace

int attention_fwd(const AttnArgs& a, cudaStream_t st) {
  if (a.b <= 0 || a.s <= 0) return MT_OK;
  if (a.hd == 64) return fwd_impl<64>(a, st);
  if (a.hd == 128) return fwd_impl<128>(a, st);
  return MT_ERR_CONFIG;
}

namespace {
int g_bwd_variant = 0;
}

int attention_bwd_variant(int v) {
  const int was = g_bwd_variant;
  g_bwd_variant = v;
  return was;
}

int attention_bwd_kernels(int hd) { return (g_bwd_variant == 1 && hd == 128) ? 3 : 4; }

int attention_bwd_tc(const AttnArgs& a, cudaStream_t st, int* err) {
  if (a.b <= 0 || a.s <= 0) return MT_OK;
  if (a.hd != 128 && a.hd != 64) return MT_ERR_CONFIG;
  const int T = a.b * a.s;
  const int64_t nw = (int64_t)T * a.H;
  k_attn_bwd_pre<<<(int)((nw + 7) / 8), 256, 0, st>>>((const bf16*)a.o, (const bf16*)a.dout, a.ldo, a.dvec, T, a.s,
                                                      a.H, a.hd);
  // automatic: the deterministic split form, which is also the faster one at
  // every length measured (B200, 16 or 32 heads of 128: 746 against 832 us at
  // 8 x 2048, 2268 against 2671 at 4 x 4096, 7695 against 8979 at 16384);
  // its query-major kernel stores dq_acc four floats at a time
  const bool aligned = (reinterpret_cast<uintptr_t>(a.dq_acc) & 15) == 0 && a.ldqa % 4 == 0;
  // head dim 64 has the split form only
  if ((g_bwd_variant == 2 || a.hd == 64) && !aligned) return MT_ERR_ARG;
  const bool split = g_bwd_variant == 2 || a.hd == 64 || (g_bwd_variant == 0 && aligned);
  if (split) {  // dK, dV without reductions; dQ written once per element by the query-major kernel
    int r = attention_bwd_tc_main(a, st, err, true);
    if (r == MT_OK) r = attention_bwd_dq_tc(a, st, err);
    if (r != MT_OK) return r;
  } else {
    if (cudaMemsetAsync(a.dq_acc, 0, (size_t)T * a.ldqa * sizeof(float), st) != cudaSuccess) return MT_ERR_CUDA;
    const int r = attention_bwd_tc_main(a, st, err, false);
    if (r != MT_OK) return r;
  }
  const int64_t nthr = (int64_t)T * a.H * (a.hd / 8);
  k_dq_cast<<<(int)((nthr + 255) / 256), 256, 0, st>>>(a.dq_acc, a.ldqa, (bf16*)a.dq, a.lddq, T, a.H, a.hd, a.s,
                                                       a.rope_cos, a.rope_sin);
  return launch_status();
}

int attention_bwd(const AttnArgs& a, cudaStream_t st) {
  if (a.b <= 0 || a.s <= 0) return MT_OK;
  if (a.hd == 64) return bwd_impl<64>(a, st);
  if (a.hd == 128) return bwd_impl<128>(a, st);
  return MT_ERR_CONFIG;
}

}  // namespace mt
