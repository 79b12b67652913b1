// Causal flash-attention forward on the 5th-generation tensor cores (sm_100a).
//
// Same result as the forward in attention.cu (o = softmax(q k^T / sqrt(hd) +
// causal mask) v per query head with grouped KV heads, plus the per-row
// natural log-sum-exp that the backward needs), organised around tcgen05:
//
//   warp 0      TMA producer: Q once, then K_j and V_j per 128-key block into
//               two 2-stage rings (K_j is released when S_j is done, V_j when
//               O_j is done; one 64-column x 128-row, 128-byte-swizzled box
//               shape serves Q, K and V)
//   warp 1      MMA issuer: S_j = Q K_j^T (128 x 128 x hd) into one of two
//               tensor-memory S buffers, then O_j = P_j V_j (128 x hd x 128)
//               into one of two tensor-memory O buffers; S_{j+1} is issued
//               before O_j so the tensor core works while softmax runs
//   warps 2..9  softmax: two warpgroups; in each, thread r owns query row r
//               (its tensor-memory lane). Both read the whole S_j row for the
//               row max; warpgroup g then computes exp2, the partial row sum
//               and the bf16 P for keys [64g, 64g+64) (one 128-byte-swizzled
//               K-major sub-tile of the A operand of the next MMA) and
//               accumulates O columns [g hd/2, (g+1) hd/2) in registers, one
//               block behind, with the online-softmax correction
//
// Every mbarrier wait is bounded (mt_common.cuh); on expiry the kernel records
// an error code, drains its copies and MMAs (bounded) and returns.
#include "mt_common.cuh"
#include "mt_internal.h"

namespace mt {

namespace {

constexpr int FA_BQ = 128;
constexpr int FA_BKV = 128;
constexpr int FA_THREADS = 320;  // producer, MMA, 8 softmax warps

template <int HD>
struct FaCfg {
  static constexpr int Q_BYTES = FA_BQ * HD * 2;
  static constexpr int KV_BYTES = FA_BKV * HD * 2;  // one of K or V
  static constexpr int STAGES = 2;
  static constexpr int P_BYTES = FA_BQ * FA_BKV * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_P = OFF_V + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;    // S buffers at columns 0 and 128
  static constexpr uint32_t O_COL = 256;  // O buffers at 256 and 256 + HD
};

struct FaParams {
  __nv_bfloat16* O;
  int64_t ldo;
  float* LSE;
  int s, H, Hkv;
  float scale;
  int* err;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int HD>
__global__ void __launch_bounds__(FA_THREADS, 1)
    k_flash_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, FaParams p) {
  using C = FaCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sP = smem + C::OFF_P;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bar + 0;
  uint64_t* k_full = bar + 1;    // [2]
  uint64_t* k_empty = bar + 3;   // [2]  (S_j done: K_j free)
  uint64_t* v_full = bar + 5;    // [2]
  uint64_t* v_empty = bar + 7;   // [2]  (O_j done: V_j free)
  uint64_t* s_full = bar + 9;    // [2]
  uint64_t* s_empty = bar + 11;  // [2]
  uint64_t* p_full = bar + 13;   // [2]
  uint64_t* o_full = bar + 15;   // [2]
  uint64_t* o_empty = bar + 17;  // [2]
  uint64_t* drain = bar + 19;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 20);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 21);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (p.H / p.Hkv);
  const int q0 = qb * FA_BQ;
  const int row0 = b * p.s;  // first token of the sequence
  const int nkv = qb + 1;    // key blocks 0..qb (block qb is the diagonal)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);
      mbar_init(&p_full[i], 8);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int k_last[2] = {-1, -1}, v_last[2] = {-1, -1};
      bool ok = true;
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
      for (int c = 0; c < HD / 64; ++c) tma_load_2d(sQ + c * 16384, &tmQ, q_full, h * HD + c * 64, row0 + q0);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int r = row0 + j * FA_BKV;
        if (*abort_flag || !mbar_wait(&k_empty[st], ph ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[st], C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c)
          tma_load_2d(sK + st * C::KV_BYTES + c * 16384, &tmK, &k_full[st], kvh * HD + c * 64, r);
        k_last[st] = (int)ph;
        if (*abort_flag || !mbar_wait(&v_empty[st], ph ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[st], C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < HD / 64; ++c)
          tma_load_2d(sV + st * C::KV_BYTES + c * 16384, &tmV, &v_full[st], kvh * HD + c * 64, r);
        v_last[st] = (int)ph;
      }
      if (!ok) {
        record_error(p.err, DEV_TIMEOUT_PRODUCER);
        *abort_flag = 1;
        // let every issued copy land before the CTA's shared memory goes away
        if (!mbar_wait(q_full, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        for (int s2 = 0; s2 < 2; ++s2) {
          if (k_last[s2] >= 0 && !mbar_wait(&k_full[s2], (uint32_t)k_last[s2])) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
          if (v_last[s2] >= 0 && !mbar_wait(&v_full[s2], (uint32_t)v_last[s2])) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc_s = idesc_bf16_f32(FA_BQ, FA_BKV, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(FA_BQ, HD, false, true);
      const uint32_t aQ = smem_u32(sQ);
      bool ok = mbar_wait(q_full, 0) && !*abort_flag;
      bool issued = false;
      auto issue_pv = [&](int i) -> bool {
        const int pb = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (*abort_flag || !mbar_wait(&v_full[pb], ph) || !mbar_wait(&p_full[pb], ph) ||
            !mbar_wait(&o_empty[pb], ph ^ 1))
          return false;
        tc_fence_after();
        const uint32_t aP = smem_u32(sP + pb * C::P_BYTES);
        const uint32_t bV = smem_u32(sV + (i & 1) * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < FA_BKV / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(aP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(bV + kk * 2048, 16384, 1024);
          umma_bf16(tmem + C::O_COL + pb * HD, ad, bd, idesc_o, kk != 0);
        }
        umma_commit(&o_full[pb]);
        umma_commit(&v_empty[pb]);
        return true;
      };
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (*abort_flag || !mbar_wait(&k_full[st], ph) || !mbar_wait(&s_empty[st], ph ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t bK = smem_u32(sK + st * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(aQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(bK + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          umma_bf16(tmem + C::S_COL + st * FA_BKV, ad, bd, idesc_s, kk != 0);
        }
        issued = true;
        umma_commit(&s_full[st]);
        umma_commit(&k_empty[st]);
        if (j >= 1 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && !issue_pv(nkv - 1)) ok = false;
      if (!ok) {
        record_error(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
        if (issued) {
          umma_commit(drain);
          if (!mbar_wait(drain, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        }
      }
    }
  } else {
    // ---------------- softmax + output (warps 2..9) ----------------
    constexpr int HH = HD / 2;          // O columns per warpgroup
    const int wg = (warp - 2) >> 2;     // 0: keys/O columns in the first half, 1: second half
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row inside the tile == tensor-memory lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale * 1.4426950408889634f;
    float o[HH];
#pragma unroll
    for (int i = 0; i < HH; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f, corr_prev = 0.f;
    bool ok = true;

    auto accumulate_o = [&](int i, float corr) -> bool {
      const int ob = i & 1;
      if (*abort_flag || !mbar_wait(&o_full[ob], (i >> 1) & 1)) return false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < HH / 16; ++c) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + C::O_COL + ob * HD + wg * HH + c * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) o[c * 16 + e] = o[c * 16 + e] * corr + __uint_as_float(v[e]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[ob]);
      return true;
    };

    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      if (*abort_flag || !mbar_wait(&s_full[sb], ph)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool diag = (j == nkv - 1);
      const uint32_t sbase = tmem + lane_base + C::S_COL + sb * FA_BKV;
      // pass 1: row max of the visible scores (whole row)
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < FA_BKV / 16; ++c) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(sbase + c * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x = __uint_as_float(v[e]);
          if (!diag || c * 16 + e <= r) mx = fmaxf(mx, x);
        }
      }
      const float mnew = fmaxf(m, mx);
      const float corr = (m == -INFINITY) ? 0.f : ex2((m - mnew) * sl2);
      const float mb = mnew * sl2;
      // pass 2: this warpgroup's 64 keys -> probabilities, partial row sum,
      // bf16 P into swizzle sub-tile wg of the A operand
      uint8_t* prow = sP + sb * C::P_BYTES + wg * 16384 + r * 128;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(sbase + wg * 64 + c * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 2; ++q) {  // two 16-byte chunks of 8 keys
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int col = wg * 64 + c * 16 + q * 8 + e;
            float p0 = ex2(__uint_as_float(v[q * 8 + e]) * sl2 - mb);
            float p1 = ex2(__uint_as_float(v[q * 8 + e + 1]) * sl2 - mb);
            if (diag && col > r) p0 = 0.f;
            if (diag && col + 1 > r) p1 = 0.f;
            rs += p0 + p1;
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
          const int chunk = c * 2 + q;  // 0..7 inside the 64-key sub-tile
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      l = l * corr + rs;
      m = mnew;
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_empty[sb]);
        mbar_arrive(&p_full[sb]);
      }
      if (j >= 1 && !accumulate_o(j - 1, corr_prev)) {
        ok = false;
        break;
      }
      corr_prev = corr;
    }
    if (ok && !accumulate_o(nkv - 1, corr_prev)) ok = false;
    if (!ok) {
      record_error(p.err, DEV_TIMEOUT_EPILOGUE);
      *abort_flag = 1;
    }
    // Row sum = both warpgroups' partial sums (exchanged through shared memory
    // reused from the Q tile, which every MMA has finished reading by now).
    float* lsum = reinterpret_cast<float*>(sQ);
    if (ok) lsum[wg * FA_BQ + r] = l;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ok) {
      const float lt = l + lsum[(wg ^ 1) * FA_BQ + r];
      const int qi = q0 + r;
      if (qi < p.s) {
        const float inv = 1.f / lt;
        __nv_bfloat16* orow = p.O + (int64_t)(row0 + qi) * p.ldo + h * HD + wg * HH;
#pragma unroll
        for (int c = 0; c < HH / 8; ++c) {
          uint4 w;
          w.x = pack_bf16x2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
          w.y = pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
          w.z = pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
          w.w = pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
          reinterpret_cast<uint4*>(orow)[c] = w;
        }
        if (wg == 0) p.LSE[((int64_t)b * p.H + h) * p.s + qi] = m * p.scale + logf(lt);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// 2-D bf16 map over `cols` columns of a [rows, ld] buffer, box {64, 128}.
bool fa_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t ld) {
  return make_tensor_map_2d_bf16(m, base, cols, rows, ld, 128);
}

template <int HD>
int launch_fa(const AttnArgs& a, cudaStream_t st, int* err) {
  using C = FaCfg<HD>;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(k_flash_fwd_tc<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
      return MT_ERR_CUDA;
    attr = true;
  }
  const int64_t T = (int64_t)a.b * a.s;
  CUtensorMap mq, mk, mv;
  if (!fa_map(&mq, a.q, (int64_t)a.H * HD, T, a.ldqkv) || !fa_map(&mk, a.k, (int64_t)a.Hkv * HD, T, a.ldqkv) ||
      !fa_map(&mv, a.v, (int64_t)a.Hkv * HD, T, a.ldqkv))
    return MT_ERR_ARG;
  FaParams p{(__nv_bfloat16*)a.o, a.ldo, a.lse, a.s, a.H, a.Hkv, a.scale, err};
  dim3 grid((a.s + FA_BQ - 1) / FA_BQ, a.H, a.b);
  k_flash_fwd_tc<HD><<<grid, FA_THREADS, C::SMEM, st>>>(mq, mk, mv, p);
  return launch_status();
}

}  // namespace

int attention_fwd_tc(const AttnArgs& a, cudaStream_t st, int* err) {
  if (a.b <= 0 || a.s <= 0) return MT_OK;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(a.q) || !al16(a.k) || !al16(a.v) || !al16(a.o) || (a.ldqkv % 8) || (a.ldo % 8)) return MT_ERR_ARG;
  if (a.hd == 64) return launch_fa<64>(a, st, err);
  if (a.hd == 128) return launch_fa<128>(a, st, err);
  return MT_ERR_CONFIG;
}

}  // namespace mt
