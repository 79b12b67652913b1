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
//               tensor-memory S buffers, then O += P_j V_j (128 x hd x 128)
//               into the one tensor-memory O accumulator; S_{j+1} is issued
//               before P_j V_j so the tensor core works while softmax runs
//   warps 2..9  softmax: two warpgroups; in each, thread r owns query row r
//               (its tensor-memory lane). Both load the whole S_j row in one
//               batch for the row max; warpgroup g then computes exp2, the
//               partial row sum and the bf16 P for keys [64g, 64g+64) (one
//               128-byte-swizzled K-major sub-tile of the A operand of the
//               next MMA) from the registers it already holds. The running
//               maximum is raised lazily: only when a row's maximum grows by
//               more than 2^8 (in exp2 units) are the row's O columns rescaled
//               in tensor memory (after the previous P V has landed), so the
//               probabilities stay below 256 and, on most blocks, O is never
//               read back until the end
//
// Every mbarrier wait is bounded (mt_common.cuh); on expiry the kernel records
// an error code, drains its copies and MMAs (bounded) and returns.
#include <type_traits>

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
  static constexpr uint32_t O_COL = 256;  // the O accumulator, HD columns
};

// A row's running maximum is raised only when its block maximum exceeds it by
// more than this many units of exp2 (probabilities then stay <= 2^8).
constexpr float kRescaleLog2 = 8.0f;

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

// Bounded wait whose result is the same on every lane of the warp, so that a
// timeout can never split a warp in front of a warp-collective tcgen05.ld.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity));
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
  uint64_t* o_full = bar + 15;   // [2]  P_j V_j (and every earlier MMA) done, j mod 2
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
      // Descriptors of the first k-step of each operand; k-steps, stages and
      // 64-column sub-tiles only move the start-address field (address / 16),
      // so the loops add constants (the MMAs are 64 cycles each).
      const uint64_t dQ0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dP0 = sdesc_sw128(smem_u32(sP), 16, 1024);
      const uint64_t dV0 = sdesc_sw128(smem_u32(sV), 16384, 1024);
      bool ok = mbar_wait(q_full, 0) && !*abort_flag;
      bool issued = false;
      // O += P_i V_i. The softmax warps signal p_full only after any rescale
      // of O that block i needs, so the accumulator is never read and
      // written at once.
      auto issue_pv = [&](int i) -> bool {
        const int pb = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (*abort_flag || !mbar_wait(&v_full[pb], ph) || !mbar_wait(&p_full[pb], ph)) return false;
        tc_fence_after();
        const uint64_t aP = dP0 + ((pb * C::P_BYTES) >> 4), bV = dV0 + (((i & 1) * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < FA_BKV / 16; ++kk)
          umma_bf16(tmem + C::O_COL, aP + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), bV + ((kk * 2048) >> 4),
                    idesc_o, (i | kk) != 0);
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
        const uint64_t bK = dK0 + ((st * C::KV_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t step = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_bf16(tmem + C::S_COL + st * FA_BKV, dQ0 + step, bK + step, idesc_s, kk != 0);
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
    const uint32_t obase = tmem + lane_base + C::O_COL + wg * HH;  // this warpgroup's O columns
    const float sl2 = p.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;  // running (lazily raised) row maximum, this half's row sum
    bool ok = true;

    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(&s_full[sb], ph)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sbase = tmem + lane_base + C::S_COL + sb * FA_BKV;
      // The whole row in one batch: this warpgroup's 64 keys (kept for the
      // exponentials) and the other 64 (for the maximum only).
      uint32_t v[64], w[64];
      tmem_ld_32x32b_x32(sbase + wg * 64, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld_32x32b_x32(sbase + wg * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_ld_32x32b_x32(sbase + (wg ^ 1) * 64, *reinterpret_cast<uint32_t(*)[32]>(w));
      tmem_ld_32x32b_x32(sbase + (wg ^ 1) * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(w + 32));
      tmem_ld_wait();
      // The causal mask only touches the diagonal block (j == nkv - 1, row r
      // sees keys [0, r] of it): the other blocks run an instantiation without
      // any per-element test.
      float rs = 0.f;
      auto block = [&](auto diag_tag) -> bool {
        constexpr bool DIAG = decltype(diag_tag)::value;
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          if (!DIAG || wg * 64 + e <= r) mx = fmaxf(mx, __uint_as_float(v[e]));
          if (!DIAG || (wg ^ 1) * 64 + e <= r) mx = fmaxf(mx, __uint_as_float(w[e]));
        }
        // Lazy maximum: raise it (and rescale O and l) only when the block's
        // maximum exceeds the running one by more than 2^kRescaleLog2.
        const bool raise = (m == -INFINITY) || (mx - m) * sl2 > kRescaleLog2;
        const float corr = (raise && m != -INFINITY) ? ex2((m - mx) * sl2) : 1.f;
        if (raise) m = mx;
        if (j > 0 && __any_sync(0xffffffffu, raise)) {
          // O holds blocks < j scaled by the old maximum: once P_{j-1} V_{j-1}
          // has landed, multiply this warpgroup's columns of the raised rows.
          const int pj = j - 1;
          if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(&o_full[pj & 1], (pj >> 1) & 1)) return false;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < HH / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(obase + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint32_t t8[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) t8[u] = __float_as_uint(__uint_as_float(o[e + u]) * corr);
              tmem_st_32x32b_x8(obase + c * 32 + e, t8);
            }
          }
          tmem_st_wait();
          tc_fence_before();
        }
        l *= corr;
        // The P buffer of this block was last read by P_{j-2} V_{j-2}.
        if (j >= 2) {
          const int pj = j - 2;
          if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(&o_full[pj & 1], (pj >> 1) & 1)) return false;
        }
        // this warpgroup's 64 keys -> probabilities, partial row sum, bf16 P
        // into swizzle sub-tile wg of the A operand
        uint8_t* prow = sP + sb * C::P_BYTES + wg * 16384 + r * 128;
        const float mb = m * sl2;
#pragma unroll
        for (int chunk = 0; chunk < 8; ++chunk) {  // 16-byte chunks of 8 keys
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int k = chunk * 8 + e;
            float p0 = ex2(fmaf(__uint_as_float(v[k]), sl2, -mb));
            float p1 = ex2(fmaf(__uint_as_float(v[k + 1]), sl2, -mb));
            if (DIAG && wg * 64 + k > r) p0 = 0.f;
            if (DIAG && wg * 64 + k + 1 > r) p1 = 0.f;
            rs += p0 + p1;
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        return true;
      };
      if (!(j == nkv - 1 ? block(std::true_type{}) : block(std::false_type{}))) {
        ok = false;
        break;
      }
      l += rs;
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_empty[sb]);
        mbar_arrive(&p_full[sb]);
      }
    }
    // the last P V
    if (ok && (__any_sync(0xffffffffu, *abort_flag) ||
               !mbar_wait_warp(&o_full[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1)))
      ok = false;
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
      tc_fence_after();
      const float lt = l + lsum[(wg ^ 1) * FA_BQ + r];
      const int qi = q0 + r;
      const float inv = 1.f / lt;
      __nv_bfloat16* orow = p.O + (int64_t)(row0 + qi) * p.ldo + h * HD + wg * HH;
#pragma unroll
      for (int c = 0; c < HH / 32; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(obase + c * 32, o);  // warp-collective: every lane loads
        tmem_ld_wait();
        if (qi < p.s) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 t;
            t.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv, __uint_as_float(o[e + 1]) * inv);
            t.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
            t.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
            t.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
            reinterpret_cast<uint4*>(orow + c * 32 + e)[0] = t;
          }
        }
      }
      if (wg == 0 && qi < p.s) p.LSE[((int64_t)b * p.H + h) * p.s + qi] = m * p.scale + logf(lt);
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

// ===========================================================================
// Forward, head_dim 128, two query tiles per CTA in ping-pong.
//
// A CTA takes 256 consecutive queries of one head as tiles A and B (128 rows
// each) and streams the key blocks both need. Each tile has its own softmax
// warpgroup, whose thread r owns row r of the tile for all 128 keys of a
// block, and its own tensor memory: S (128 columns, over which the thread
// writes its bf16 P in place, the A operand of P V) and O (128 columns). While
// one warpgroup turns S into P, the tensor core runs the other tile's
// products, so the MMAs and the softmax of the two tiles overlap:
//   warp 0   TMA producer: Q_A, Q_B once, then K_j and V_j per 128-key block
//            into two-stage rings
//   warp 1   MMA issuer: S_A(0), S_B(0); per block j: O_A += P_A(j) V_j,
//            S_A(j+1) once that P V is done (it reads the S_A columns),
//            O_B += P_B(j) V_j, S_B(j+1)
//   warps 2..5 / 6..9  softmax of tile A / tile B: row max, lazy rescale of O
//            in tensor memory (only when a row's maximum grows by more than
//            2^8 in exp2 units), exp2, row sum, bf16 P into tensor memory
// Tile A needs key blocks 0 .. 2p, tile B 0 .. 2p + 1 (p the CTA's pair of
// tiles); a tile B wholly past the sequence end does nothing. Shared memory:
// Q_A, Q_B, two K and two V stages (192 KB); no P tile.
// ===========================================================================
namespace {

constexpr int PP_THREADS = 320;  // producer, MMA, two softmax warpgroups

struct PpCfg {
  static constexpr int TILE = 128 * 128 * 2;  // 32 KB: 128 rows x 128 bf16 (two 64-column swizzle sub-tiles)
  static constexpr int OFF_QA = 0;
  static constexpr int OFF_QB = TILE;
  static constexpr int OFF_K = 2 * TILE;  // [2]
  static constexpr int OFF_V = 4 * TILE;  // [2]
  static constexpr int OFF_BAR = 6 * TILE;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  // tensor-memory columns of tile t: S (and P over it) and O
  __host__ __device__ static constexpr uint32_t c_s(int t) { return t ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t c_o(int t) { return t ? 384u : 256u; }
};

__global__ void __launch_bounds__(PP_THREADS, 1)
    k_flash_fwd_pp(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, FaParams p) {
  using C = PpCfg;
  constexpr int HD = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ[2] = {smem + C::OFF_QA, smem + C::OFF_QB};
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bar + 0;
  uint64_t* k_full = bar + 1;    // [2]
  uint64_t* k_empty = bar + 3;   // [2]
  uint64_t* v_full = bar + 5;    // [2]
  uint64_t* v_empty = bar + 7;   // [2]
  uint64_t* s_full = bar + 9;    // [2 tiles] S of the tile's current block in tensor memory
  uint64_t* p_full = bar + 11;   // [2 tiles] P written (and any O rescale done), 4 warps each
  uint64_t* pv_done = bar + 13;  // [2 tiles] the tile's P V (and every earlier MMA) done
  uint64_t* drain = bar + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 17);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (p.H / p.Hkv);
  const int q0 = pair * 256;
  const int row0 = b * p.s;
  // key blocks each tile needs (0 for a tile wholly past the sequence end)
  int nkv_t[2];
  nkv_t[0] = 2 * pair + 1;
  nkv_t[1] = (q0 + 128 < p.s) ? 2 * pair + 2 : 0;
  const int nkv = nkv_t[1] > 0 ? nkv_t[1] : nkv_t[0];

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
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
      const int nq = nkv_t[1] > 0 ? 2 : 1;
      mbar_arrive_expect_tx(q_full, nq * C::TILE);
      for (int t = 0; t < nq; ++t)
        for (int c = 0; c < 2; ++c) tma_load_2d(sQ[t] + c * 16384, &tmQ, q_full, h * HD + c * 64, row0 + q0 + 128 * t);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int r = row0 + j * 128;
        if (*abort_flag || !mbar_wait(&k_empty[st], ph ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[st], C::TILE);
        for (int c = 0; c < 2; ++c) tma_load_2d(sK + st * C::TILE + c * 16384, &tmK, &k_full[st], kvh * HD + c * 64, r);
        k_last[st] = (int)ph;
        if (*abort_flag || !mbar_wait(&v_empty[st], ph ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[st], C::TILE);
        for (int c = 0; c < 2; ++c) tma_load_2d(sV + st * C::TILE + c * 16384, &tmV, &v_full[st], kvh * HD + c * 64, r);
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
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);  // S = Q K^T
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, HD, false, true);    // O += P V, P from tensor memory
      const uint64_t dQ0[2] = {sdesc_sw128(smem_u32(sQ[0]), 16, 1024), sdesc_sw128(smem_u32(sQ[1]), 16, 1024)};
      const uint64_t dK0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV0 = sdesc_sw128(smem_u32(sV), 16384, 1024);
      bool ok = mbar_wait(q_full, 0) && !*abort_flag;
      bool issued = false;
      // S_t(j) = Q_t K_j^T; K_j is released once every tile that uses it has its S.
      auto issue_s = [&](int t, int j) -> bool {
        const int st = j & 1;
        if (*abort_flag || !mbar_wait(&k_full[st], (j >> 1) & 1)) return false;
        // the S columns hold P_t(j - 1) until its P V is done
        if (j > 0 && !mbar_wait(&pv_done[t], (j - 1) & 1)) return false;
        tc_fence_after();
        const uint64_t bK = dK0 + ((st * C::TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t step = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_bf16(tmem + C::c_s(t), dQ0[t] + step, bK + step, idesc_s, kk != 0);
        }
        issued = true;
        umma_commit(&s_full[t]);
        const bool last_user = (t == 1) || nkv_t[1] <= j;
        if (last_user) umma_commit(&k_empty[st]);
        return true;
      };
      // O_t += P_t(j) V_j; V_j is released after its last user.
      auto issue_pv = [&](int t, int j) -> bool {
        const int st = j & 1;
        if (*abort_flag || !mbar_wait(&v_full[st], (j >> 1) & 1) || !mbar_wait(&p_full[t], j & 1)) return false;
        tc_fence_after();
        const uint64_t bV = dV0 + ((st * C::TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          umma_bf16_ts(tmem + C::c_o(t), tmem + C::c_s(t) + 8 * kk, bV + ((kk * 2048) >> 4), idesc_o, (j | kk) != 0);
        umma_commit(&pv_done[t]);
        const bool last_user = (t == 1) || nkv_t[1] <= j;
        if (last_user) umma_commit(&v_empty[st]);
        return true;
      };
      if (ok) ok = issue_s(0, 0);
      if (ok && nkv_t[1] > 0) ok = issue_s(1, 0);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j < nkv_t[0] && !issue_pv(0, j)) ok = false;
        if (ok && j + 1 < nkv_t[0] && !issue_s(0, j + 1)) ok = false;
        if (ok && j < nkv_t[1] && !issue_pv(1, j)) ok = false;
        if (ok && j + 1 < nkv_t[1] && !issue_s(1, j + 1)) ok = false;
      }
      if (!ok) {
        record_error(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      if (issued) {  // every MMA issued here completes before tensor memory is freed
        umma_commit(drain);
        if (!mbar_wait(drain, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
      }
    }
  } else {
    // ---------------- softmax of tile t (warps 2..5: A, 6..9: B) ----------------
    const int t = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row of the tile == tensor-memory lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t sbase = tmem + lane_base + C::c_s(t);
    const uint32_t obase = tmem + lane_base + C::c_o(t);
    const int n_t = nkv_t[t];
    const float sl2 = p.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(&s_full[t], j & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // The causal mask touches only the tile's diagonal block (its last one):
      // row r sees keys [0, r] of it; the other blocks need no test. Half a
      // row (64 scores) is held at a time: both halves for the maximum, then
      // the second half's probabilities are packed (32 registers) before the
      // first half is read again, because P over keys [0, 64) overwrites the
      // S columns [0, 32) and P over [64, 128) the columns [32, 64).
      auto block = [&](auto diag_tag) -> bool {
        constexpr bool DIAG = decltype(diag_tag)::value;
        uint32_t v[64];
        float mx = -INFINITY;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          tmem_ld_32x32b_x32(sbase + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(v));
          tmem_ld_32x32b_x32(sbase + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (!DIAG || hf * 64 + e <= r) mx = fmaxf(mx, __uint_as_float(v[e]));
        }
        const bool raise = (m == -INFINITY) || (mx - m) * sl2 > kRescaleLog2;
        const float corr = (raise && m != -INFINITY) ? ex2((m - mx) * sl2) : 1.f;
        if (raise) m = mx;
        if (j > 0 && __any_sync(0xffffffffu, raise)) {
          // O holds blocks < j at the old maximum: once P(j-1) V has landed,
          // rescale the raised rows (the others multiply by 1)
          if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(&pv_done[t], (j - 1) & 1)) return false;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(obase + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint32_t t8[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) t8[u] = __float_as_uint(__uint_as_float(o[e + u]) * corr);
              tmem_st_32x32b_x8(obase + c * 32 + e, t8);
            }
          }
          tmem_st_wait();
        }
        l *= corr;
        const float mb = m * sl2;
        float rs = 0.f;
        // probabilities of keys [64 hf, 64 hf + 64) from v, as bf16 pairs
        auto probs = [&](int hf, uint32_t (&pk)[32]) {
#pragma unroll
          for (int e = 0; e < 64; e += 2) {
            const int k = hf * 64 + e;
            float p0 = ex2(fmaf(__uint_as_float(v[e]), sl2, -mb));
            float p1 = ex2(fmaf(__uint_as_float(v[e + 1]), sl2, -mb));
            if (DIAG && k > r) p0 = 0.f;
            if (DIAG && k + 1 > r) p1 = 0.f;
            rs += p0 + p1;
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
        };
        uint32_t hi[32], lo[32];
        probs(1, hi);  // v still holds keys [64, 128)
        tmem_ld_32x32b_x32(sbase, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld_32x32b_x32(sbase + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_ld_wait();
        probs(0, lo);
        // key k in column k / 2, even k in the low half (the A-operand layout)
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st_32x32b_x8(sbase + c * 8, *reinterpret_cast<const uint32_t(*)[8]>(lo + 8 * c));
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_st_32x32b_x8(sbase + 32 + c * 8, *reinterpret_cast<const uint32_t(*)[8]>(hi + 8 * c));
        l += rs;
        return true;
      };
      if (!(j == n_t - 1 ? block(std::true_type{}) : block(std::false_type{}))) {
        ok = false;
        break;
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok && n_t > 0 &&
        (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(&pv_done[t], (n_t - 1) & 1)))
      ok = false;
    if (!ok) {
      record_error(p.err, DEV_TIMEOUT_EPILOGUE);
      *abort_flag = 1;
    } else if (n_t > 0) {
      tc_fence_after();
      const int qi = q0 + 128 * t + r;
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.O + (int64_t)(row0 + qi) * p.ldo + h * HD;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(obase + c * 32, o);  // warp-collective: every lane loads
        tmem_ld_wait();
        if (qi < p.s) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[e + 0]) * inv, __uint_as_float(o[e + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
            reinterpret_cast<uint4*>(orow + c * 32 + e)[0] = w;
          }
        }
      }
      if (qi < p.s) p.LSE[((int64_t)b * p.H + h) * p.s + qi] = m * p.scale + logf(l);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int launch_fa_pp(const AttnArgs& a, cudaStream_t st, int* err) {
  using C = PpCfg;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(k_flash_fwd_pp, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
      return MT_ERR_CUDA;
    attr = true;
  }
  const int64_t T = (int64_t)a.b * a.s;
  CUtensorMap mq, mk, mv;
  if (!fa_map(&mq, a.q, (int64_t)a.H * 128, T, a.ldqkv) || !fa_map(&mk, a.k, (int64_t)a.Hkv * 128, T, a.ldqkv) ||
      !fa_map(&mv, a.v, (int64_t)a.Hkv * 128, T, a.ldqkv))
    return MT_ERR_ARG;
  FaParams p{(__nv_bfloat16*)a.o, a.ldo, a.lse, a.s, a.H, a.Hkv, a.scale, err};
  dim3 grid((a.s + 255) / 256, a.H, a.b);
  k_flash_fwd_pp<<<grid, PP_THREADS, C::SMEM, st>>>(mq, mk, mv, p);
  return launch_status();
}

}  // namespace

namespace {
int g_fa_variant = 0;  // 0 automatic, 1 one query tile per CTA, 2 two tiles in ping-pong
}

int attention_fwd_variant(int v) {
  const int was = g_fa_variant;
  g_fa_variant = v;
  return was;
}

int attention_fwd_tc(const AttnArgs& a, cudaStream_t st, int* err) {
  if (a.b <= 0 || a.s <= 0) return MT_OK;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(a.q) || !al16(a.k) || !al16(a.v) || !al16(a.o) || (a.ldqkv % 8) || (a.ldo % 8)) return MT_ERR_ARG;
  if (a.hd == 64) return launch_fa<64>(a, st, err);
  // head dim 128: two query tiles per CTA above 8192 tokens (measured on
  // B200, TFLOP/s one tile / two: 562 / 536 at s = 2048, 706 / 685 at 4096,
  // 809 / 807 at 8192, 903 / 939 at 16384, 911 / 972 at 32768; with short rows
  // the pairs' prologue and epilogue are exposed)
  if (a.hd == 128) {
    const int v = g_fa_variant ? g_fa_variant : (a.s > 8192 ? 2 : 1);
    return v == 2 ? launch_fa_pp(a, st, err) : launch_fa<128>(a, st, err);
  }
  return MT_ERR_CONFIG;
}


// ===========================================================================
// Backward on the tcgen05 tensor cores (head_dim 128).
//
// One CTA per (128-key block, KV head, sequence); it loops over every query
// head of the group and every 128-query block at or after its keys:
//   S^T  = K Q^T,   dP^T = V dO^T            (128 keys x 128 queries, TMEM)
//   P^T  = exp(S^T / sqrt(hd) - LSE),  dS^T = P^T (dP^T - D)   (gradient
//          warps, one key row per thread; P^T and dS^T go back into the S^T
//          columns as bf16 pairs, 16 queries' P^T then their dS^T in the 16
//          columns those queries' scores came from, where dV and dK read them
//          as their A operand; dS^T also into a 128-byte-swizzled shared tile)
//   dV  += P^T dO,  dK += dS^T Q              (128 keys x hd, TMEM, A from TMEM)
//   dQ^T = K^T dS^T                            (hd x 128 queries, into the
//          dP^T columns), read out one head column per thread and added to
//          the fp32 dQ accumulator with global reductions from registers
// Every product is N = 128 wide: 64-wide products run the tensor core at
// little more than half rate (55 instead of 32 cycles per 128 x 64 x 16 MMA,
// measured), which bounded the 64-query form of this kernel.
// Tensor memory: dK [0,128), dV [128,256), S^T / P^T|dS^T [256,384),
// dP^T / dQ^T [384,512). Shared memory: K, V, two Q and two dO stages and the
// dS^T tile, 32 KB each (224 KB).
// ===========================================================================
namespace {

constexpr int FB_BKV = 128, FB_BQ = 128, FB_HD = 128;
constexpr int FB_GWARPS = 16;                   // gradient warps: four per tensor-memory lane quarter
constexpr int FB_QW = FB_BQ / (FB_GWARPS / 4);  // queries per gradient warp (32)
constexpr int FB_THREADS = 64 + 32 * FB_GWARPS; // producer, MMA, gradient warps

struct FbCfg {
  static constexpr int TILE = 128 * 128 * 2;  // 32 KB: 128 rows x 128 bf16 as two 64-column sub-tiles
  static constexpr int SUB = 128 * 128;       // 16 KB: one 64-column sub-tile (128 rows x 128 B)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;       // [2] stages
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;  // [2]
  static constexpr int OFF_DST = OFF_DO + 2 * TILE;
  static constexpr int OFF_BAR = OFF_DST + TILE;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  static constexpr uint32_t C_DK = 0, C_DV = 128, C_S = 256, C_DP = 384;
};

struct FbParams {
  const float* LSE;
  const float* Dv;
  float* dQacc;
  int64_t ldqa;
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  int64_t lddkv;
  int s, H, Hkv;
  float scale;
  const float* rcos;
  const float* rsin;
  int* err;
  int vec_lse;  // LSE and D rows start 16-byte aligned: s % 4 == 0 and aligned bases
};

// Start-address step (address / 16) of k-step kk (16 elements of the
// contraction) inside a K-major 128-row tile made of two 64-column sub-tiles.
__device__ __forceinline__ uint32_t km_step(int kk) {
  return (uint32_t)(((kk >> 2) * FbCfg::SUB + (kk & 3) * 32) >> 4);
}

// The CTA's dK and dV (tensor-memory columns C_DK and C_DV, fp32, one key
// row per lane) out to global memory as bf16, by the 16 gradient warps.
template <int HD>
__device__ __forceinline__ void fb_store_dkdv(uint32_t tmem, uint32_t lane_base, int qg, int key, int row0,
                                              int kvh, const FbParams& p) {
  constexpr int HALF = HD / 2;
  using C = FbCfg;
  // tcgen05.ld is warp-collective: every lane loads, only keys inside the
  // sequence store. Warps of query group 0 and 1 write dK (scaled,
  // transposed RoPE; rotate-half pairs (i, i + HD/2) for i in [HD/4 qg, HD/4 (qg + 1))),
  // groups 2 and 3 write dV columns [HD/2 (qg - 2), HD/2 (qg - 1)).
  const bool store = key < p.s;
  if (qg < 2) {
    __nv_bfloat16* kr = p.dK + (int64_t)(row0 + key) * p.lddkv + kvh * HD;
    const float* cs = (p.rcos && store) ? p.rcos + (int64_t)key * (HALF) : nullptr;
    const float* sn = (p.rsin && store) ? p.rsin + (int64_t)key * (HALF) : nullptr;
#pragma unroll
    for (int cc = 0; cc < HD / 64; ++cc) {  // pairs (i, i + HD/2), 16 at a time
      const int c = qg * (HD / 64) + cc;
      uint32_t a[16], bb[16];
      tmem_ld_32x32b_x16(tmem + lane_base + C::C_DK + c * 16, a);
      tmem_ld_32x32b_x16(tmem + lane_base + C::C_DK + HALF + c * 16, bb);
      tmem_ld_wait();
      uint32_t w1[8], w2[8];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        float y1[2], y2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float x1 = __uint_as_float(a[e + u]) * p.scale, x2 = __uint_as_float(bb[e + u]) * p.scale;
          if (cs) {
            const int i = c * 16 + e + u;
            y1[u] = x1 * cs[i] + x2 * sn[i];
            y2[u] = x2 * cs[i] - x1 * sn[i];
          } else {
            y1[u] = x1;
            y2[u] = x2;
          }
        }
        w1[e >> 1] = pack_bf16x2(y1[0], y1[1]);
        w2[e >> 1] = pack_bf16x2(y2[0], y2[1]);
      }
      if (store) {
        reinterpret_cast<uint4*>(kr + c * 16)[0] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
        reinterpret_cast<uint4*>(kr + c * 16)[1] = make_uint4(w1[4], w1[5], w1[6], w1[7]);
        reinterpret_cast<uint4*>(kr + HALF + c * 16)[0] = make_uint4(w2[0], w2[1], w2[2], w2[3]);
        reinterpret_cast<uint4*>(kr + HALF + c * 16)[1] = make_uint4(w2[4], w2[5], w2[6], w2[7]);
      }
    }
  } else {
    __nv_bfloat16* vr = p.dV + (int64_t)(row0 + key) * p.lddkv + kvh * HD;
#pragma unroll
    for (int cc = 0; cc < HD / 32; ++cc) {
      const int c = (qg - 2) * (HD / 32) + cc;
      uint32_t v[16];
      tmem_ld_32x32b_x16(tmem + lane_base + C::C_DV + c * 16, v);
      tmem_ld_wait();
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
      if (store) {
        reinterpret_cast<uint4*>(vr + c * 16)[0] = make_uint4(w[0], w[1], w[2], w[3]);
        reinterpret_cast<uint4*>(vr + c * 16)[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  }
}

__global__ void __launch_bounds__(FB_THREADS, 1)
    k_flash_bwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   FbParams p) {
  using C = FbCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sdO = smem + C::OFF_DO;
  uint8_t* sdSt = smem + C::OFF_DST;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bar + 0;
  uint64_t* q_full = bar + 1;    // [2]
  uint64_t* q_empty = bar + 3;   // [2]
  uint64_t* s_full = bar + 5;    // S^T and dP^T of an iteration ready
  uint64_t* p_full = bar + 6;    // P^T, dS^T written (tensor and shared memory)
  uint64_t* pdone = bar + 7;     // dV, dK of an iteration done (S^T columns free)
  uint64_t* mma_done = bar + 8;  // dQ^T of an iteration done (and the dS^T tile read)
  uint64_t* dq_empty = bar + 9;  // dQ^T read out (dP^T columns free)
  uint64_t* drain = bar + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kvb = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int group = p.H / p.Hkv;
  const int kv0 = kvb * FB_BKV;
  const int row0 = b * p.s;
  const int nqb = (p.s + FB_BQ - 1) / FB_BQ;
  const int qb_first = kv0 / FB_BQ;
  const int per_head = nqb - qb_first;
  const int n_it = group * per_head;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, FB_GWARPS);
    mbar_init(pdone, 1);
    mbar_init(mma_done, 1);
    mbar_init(dq_empty, FB_GWARPS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int q_last[2] = {-1, -1};
      bool ok = true;
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
      for (int c = 0; c < 2; ++c) {
        tma_load_2d(sK + c * C::SUB, &tmK, kv_full, kvh * FB_HD + c * 64, row0 + kv0);
        tma_load_2d(sV + c * C::SUB, &tmV, kv_full, kvh * FB_HD + c * 64, row0 + kv0);
      }
      int h = kvh * group, qb = qb_first;  // head and query block of iteration it
      for (int it = 0; it < n_it; ++it) {
        const int st = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        const int q0 = qb * FB_BQ, hq = h;
        if (++qb == nqb) {
          qb = qb_first;
          ++h;
        }
        if (*abort_flag || !mbar_wait(&q_empty[st], ph ^ 1)) {
          record_error(p.err, 100 + (it & 63));
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&q_full[st], 2 * C::TILE);
        for (int c = 0; c < 2; ++c) {
          tma_load_2d(sQ + st * C::TILE + c * C::SUB, &tmQ, &q_full[st], hq * FB_HD + c * 64, row0 + q0);
          tma_load_2d(sdO + st * C::TILE + c * C::SUB, &tmO, &q_full[st], hq * FB_HD + c * 64, row0 + q0);
        }
        q_last[st] = (int)ph;
      }
      if (!ok) {
        *abort_flag = 1;
        if (!mbar_wait(kv_full, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        for (int s2 = 0; s2 < 2; ++s2)
          if (q_last[s2] >= 0 && !mbar_wait(&q_full[s2], (uint32_t)q_last[s2])) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t id_s = idesc_bf16_f32(FB_BKV, FB_BQ, false, false);  // keys x queries, K = hd
      constexpr uint32_t id_kv = idesc_bf16_f32(FB_BKV, FB_HD, false, true);  // keys x hd, K = queries (A in TMEM)
      constexpr uint32_t id_dq = idesc_bf16_f32(FB_HD, FB_BQ, true, true);    // hd x queries, K = keys
      // Descriptors of the first k-step of each operand form; the loops add
      // start-address steps (address / 16).
      const uint64_t dK_km = sdesc_sw128(smem_u32(sK), 16, 1024), dV_km = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dQ_km = sdesc_sw128(smem_u32(sQ), 16, 1024), dO_km = sdesc_sw128(smem_u32(sdO), 16, 1024);
      const uint64_t dQ_mn = sdesc_sw128(smem_u32(sQ), C::SUB, 1024), dO_mn = sdesc_sw128(smem_u32(sdO), C::SUB, 1024);
      const uint64_t dK_mn = sdesc_sw128(smem_u32(sK), C::SUB, 1024), ddSt_mn = sdesc_sw128(smem_u32(sdSt), C::SUB, 1024);
      constexpr uint32_t kStage = C::TILE >> 4, kMn = 2048 >> 4;  // one stage; 16 rows of a 128-byte-row tile
      bool issued = false;
      bool ok = mbar_wait(kv_full, 0) && !*abort_flag;
      if (!ok) record_error(p.err, 200);
      for (int it = 0; it < n_it && ok; ++it) {
        const int st = it & 1;
        if (*abort_flag || !mbar_wait(&q_full[st], (it >> 1) & 1)) {
          record_error(p.err, 210 + (it & 63));
          ok = false;
          break;
        }
        // S^T columns hold P^T | dS^T of the previous iteration until its dV, dK finish
        if (it > 0 && !mbar_wait(pdone, (it - 1) & 1)) {
          record_error(p.err, 230 + (it & 15));
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < FB_HD / 16; ++kk)
          umma_bf16(tmem + C::C_S, dK_km + km_step(kk), dQ_km + st * kStage + km_step(kk), id_s, kk != 0);
        issued = true;
        // dP^T columns hold dQ^T of the previous iteration until it is read out
        if (it > 0 && !mbar_wait(dq_empty, (it - 1) & 1)) {
          record_error(p.err, 250 + (it & 15));
          ok = false;
          break;
        }
        // dP^T = V dO^T into the dP^T columns
#pragma unroll
        for (int kk = 0; kk < FB_HD / 16; ++kk)
          umma_bf16(tmem + C::C_DP, dV_km + km_step(kk), dO_km + st * kStage + km_step(kk), id_s, kk != 0);
        umma_commit(s_full);
        if (*abort_flag || !mbar_wait(p_full, it & 1)) {
          record_error(p.err, 280 + (it & 15));
          ok = false;
          break;
        }
        tc_fence_after();
        // dV += P^T dO, dK += dS^T Q: K = 128 queries in 8 steps; query step kk
        // (queries [16 kk, 16 kk + 16)) of P^T sits in columns C_S + 16 kk,
        // its dS^T in the next 8 columns
#pragma unroll
        for (int kk = 0; kk < FB_BQ / 16; ++kk) {
          const bool acc = (it > 0) || (kk > 0);
          const uint32_t ap = tmem + C::C_S + 16 * kk;
          umma_bf16_ts(tmem + C::C_DV, ap, dO_mn + st * kStage + kk * kMn, id_kv, acc);
          umma_bf16_ts(tmem + C::C_DK, ap + 8, dQ_mn + st * kStage + kk * kMn, id_kv, acc);
        }
        umma_commit(pdone);
        // dQ^T = K^T dS^T (K = 128 keys in 8 steps) into the dP^T columns
#pragma unroll
        for (int kk = 0; kk < FB_BKV / 16; ++kk)
          umma_bf16(tmem + C::C_DP, dK_mn + kk * kMn, ddSt_mn + kk * kMn, id_dq, kk != 0);
        umma_commit(mma_done);
        umma_commit(&q_empty[st]);
      }
      if (!ok) {
        *abort_flag = 1;
        if (issued) {
          umma_commit(drain);
          if (!mbar_wait(drain, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        }
      }
    }
  } else {
    // ---------------- gradient warps (2 .. 2 + FB_GWARPS) ----------------
    // Warp w owns tensor-memory lane quarter w mod 4 (32 key rows, or 32 head
    // columns of dQ^T) and query columns [32 qg, 32 qg + 32) of each block.
    const int qg = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row == tensor-memory lane (the head column for dQ^T)
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale * 1.4426950408889634f;
    const int key = kv0 + r;
    const bool vec_ok = p.vec_lse != 0;  // LSE / D rows 16-byte aligned
    bool ok = true;

    // dQ^T of an iteration (complete: the caller waited for mma_done): this
    // warp's 32 query columns for head column r, added to the fp32 dQ
    // accumulator with reductions from registers (a warp's 32 lanes are 32
    // consecutive head columns of one query row: 128 coalesced bytes, whole
    // 32-byte sectors; the reductions are bound by L2 sector operations, and
    // a row-per-thread form with 16-byte vector reductions, which touches
    // half-sectors, measured 13-19 % slower).
    auto flush_dq = [&](int hq, int q0) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + lane_base + C::C_DP + qg * FB_QW, v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_empty);
      const int qf = q0 + qg * FB_QW;
      float* dst = p.dQacc + (int64_t)(row0 + qf) * p.ldqa + (int64_t)hq * FB_HD + r;
#pragma unroll
      for (int e = 0; e < FB_QW; ++e)
        if (qf + e < p.s)
          asm volatile("red.global.add.f32 [%0], %1;" ::"l"(dst + (int64_t)e * p.ldqa), "f"(__uint_as_float(v[e]) * p.scale)
                       : "memory");
    };

    int h = kvh * group, qb = qb_first;  // head and query block of iteration it
    int h_prev = h, q0_prev = 0;         // those of iteration it - 1
    for (int it = 0; it < n_it; ++it) {
      const int q0 = qb * FB_BQ, hq = h;
      if (++qb == nqb) {
        qb = qb_first;
        ++h;
      }
      // dQ^T of the previous iteration first: its columns take this iteration's dP^T
      if (it > 0) {
        if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(mma_done, (it - 1) & 1)) {
          record_error(p.err, 400 + (it & 63));
          ok = false;
          break;
        }
        tc_fence_after();
        flush_dq(h_prev, q0_prev);
      }
      const int qc = q0 + qg * FB_QW;  // first query of this warp's columns
      const float* lse = p.LSE + ((int64_t)b * p.H + hq) * p.s + qc;
      const float* dd = p.Dv + ((int64_t)b * p.H + hq) * p.s + qc;
      // Only blocks that touch the diagonal or a sequence end need the mask.
      const bool need_mask = (qc < kv0 + FB_BKV) || (q0 + FB_BQ > p.s) || (kv0 + FB_BKV > p.s);
      if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(s_full, it & 1)) {
        record_error(p.err, 300 + (it & 63));
        ok = false;
        break;
      }
      tc_fence_after();
      // Two halves of 16 queries: S^T, dP^T -> P^T, dS^T (bf16 pairs) back into
      // this warp's own S^T columns (the ones it has just read) and into the
      // shared dS^T tile.
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float lv[16], dvv[16];
        if (!need_mask && vec_ok) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 a4 = __ldg(reinterpret_cast<const float4*>(lse + hf * 16) + i);
            const float4 d4 = __ldg(reinterpret_cast<const float4*>(dd + hf * 16) + i);
            lv[4 * i] = a4.x * 1.4426950408889634f;
            lv[4 * i + 1] = a4.y * 1.4426950408889634f;
            lv[4 * i + 2] = a4.z * 1.4426950408889634f;
            lv[4 * i + 3] = a4.w * 1.4426950408889634f;
            dvv[4 * i] = d4.x;
            dvv[4 * i + 1] = d4.y;
            dvv[4 * i + 2] = d4.z;
            dvv[4 * i + 3] = d4.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const bool in = qc + hf * 16 + i < p.s;
            lv[i] = in ? __ldg(lse + hf * 16 + i) * 1.4426950408889634f : 0.f;
            dvv[i] = in ? __ldg(dd + hf * 16 + i) : 0.f;
          }
        }
        uint32_t sv[16], dv[16];
        tmem_ld_32x32b_x16(tmem + lane_base + C::C_S + qg * FB_QW + hf * 16, sv);
        tmem_ld_32x32b_x16(tmem + lane_base + C::C_DP + qg * FB_QW + hf * 16, dv);
        tmem_ld_wait();
        uint32_t pp[8], ds[8];
        auto grads = [&](auto mask_tag) {
          constexpr bool MASK = decltype(mask_tag)::value;
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float pv[2], dsv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int qi = qc + hf * 16 + e + u;
              const bool vis = !MASK || (key <= qi && qi < p.s && key < p.s);
              const float pr = vis ? ex2(fmaf(__uint_as_float(sv[e + u]), sl2, -lv[e + u])) : 0.f;
              pv[u] = pr;
              dsv[u] = vis ? pr * (__uint_as_float(dv[e + u]) - dvv[e + u]) : 0.f;
            }
            pp[e >> 1] = pack_bf16x2(pv[0], pv[1]);
            ds[e >> 1] = pack_bf16x2(dsv[0], dsv[1]);
          }
        };
        if (need_mask)
          grads(std::true_type{});
        else
          grads(std::false_type{});
        // P^T of queries [32 qg + 16 hf, +16) -> columns C_S + 32 qg + 16 hf, dS^T in the
        // next 8: exactly the 16 columns this half has just read, so no warp
        // overwrites scores another warp (or its own next half) still needs
        tmem_st_32x32b_x8(tmem + lane_base + C::C_S + qg * FB_QW + hf * 16, pp);
        tmem_st_32x32b_x8(tmem + lane_base + C::C_S + qg * FB_QW + hf * 16 + 8, ds);
        // dS^T row r, queries [32 qg + 16 hf, +16): sub-tile qg / 2, 16-byte chunks 4 (qg % 2) + 2 hf, +1
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const int chunk = 4 * (qg & 1) + 2 * hf + c2;
          const int off = (qg >> 1) * C::SUB + r * 128 + ((chunk ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(sdSt + off) = make_uint4(ds[4 * c2], ds[4 * c2 + 1], ds[4 * c2 + 2], ds[4 * c2 + 3]);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      h_prev = hq;
      q0_prev = q0;
    }
    if (ok && n_it > 0) {
      if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(mma_done, (n_it - 1) & 1)) {
        record_error(p.err, 450);
        ok = false;
      } else {
        tc_fence_after();
        flush_dq(h_prev, q0_prev);
      }
    }
    if (!ok) {
      *abort_flag = 1;
    } else if (n_it > 0) {
      fb_store_dkdv<128>(tmem, lane_base, qg, key, row0, kvh, p);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// ===========================================================================
// dK and dV of the backward, key-major and pipelined (head_dim 64 or 128): the
// key-major half of the deterministic split backward (dQ comes from
// k_flash_bwd_dq). Same products as k_flash_bwd_tc without dQ^T, ordered for
// a tensor core whose issue queue is only a few MMAs deep (the issuing thread
// stalls until its MMAs are nearly done, so the issue order is the schedule):
//   dP^T(n) = V dO^T         -> columns C_DP
//   dV     += P^T(n) dO      (A = P^T, written by the gradient warps over the
//                             S^T(n) scores they have read, as soon as their
//                             exponentials are done: it does not wait for dP^T)
//   S^T(n+1) = K Q^T         -> columns C_S (behind dV(n), which read them)
//   dK     += dS^T(n) Q      (A = dS^T, written over the dP^T(n) values; the
//                             gradient warps have had dV(n) and S^T(n+1) to
//                             compute it)
//   dP^T(n+1)                (behind dK(n), which read its columns)
// Tensor memory is reused only behind the products that read it, which the
// tensor core's in-order execution of one thread's MMAs makes safe, so the
// issuing thread waits for nothing but operands: P^T(n), Q(n+1), dS^T(n),
// dO(n+1). The gradient warps compute P^T(n+1) = exp(S^T - LSE) while dK(n)
// and dP^T(n+1) run, and dS^T(n) while dV(n) and S^T(n+1) run. Each warp
// writes a k-step's 16 queries of P^T (or dS^T) as 8 columns of bf16 pairs
// inside the 32 score columns it has read itself: k-step kk at column
// 32 (kk / 2) + 8 (kk % 2) of its buffer.
// Tensor memory: dK [0,hd), dV [128,128+hd), S^T [256,384), dP^T [384,512).
// Shared memory: K, V and two stages of Q and dO, 128 x hd bf16 each (192 KB
// at hd 128); Q and dO of a stage have barriers of their own. Each gradient
// warp also has a 256-byte slot through which its lanes hand the block's LSE
// and D values (fetched one block ahead, one query per lane) to every lane.
// ===========================================================================
namespace {

template <int HD>
struct FkCfg {
  static constexpr int TILE = 128 * HD * 2;  // 128 rows x HD bf16 as HD / 64 sub-tiles of 64 columns
  static constexpr int SUB = FbCfg::SUB;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;       // [2] stages
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;  // [2]
  static constexpr int OFF_BAR = OFF_DO + 2 * TILE;
  static constexpr int OFF_LD = OFF_BAR + 256;  // per gradient warp: 32 LSE' and 32 D values
  static constexpr int SMEM = 1024 + OFF_LD + FB_GWARPS * 64 * 4;
  static constexpr uint32_t C_DK = 0, C_DV = 128, C_S = 256, C_DP = 384;
};

// Column of k-step kk (16 queries) of P^T or dS^T inside its 128-column buffer.
__device__ __forceinline__ uint32_t fk_a_col(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }

template <int HD>
__global__ void __launch_bounds__(FB_THREADS, 1)
    k_flash_bwd_kv(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   FbParams p) {
  using C = FkCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sdO = smem + C::OFF_DO;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bar + 0;
  uint64_t* q_full = bar + 1;    // [2] Q of a stage landed
  uint64_t* o_full = bar + 3;    // [2] dO of a stage landed
  uint64_t* q_empty = bar + 5;   // [2] the stage's last products done
  uint64_t* s_full = bar + 7;    // S^T(n) done
  uint64_t* p_ready = bar + 8;   // P^T(n) written by every gradient warp
  uint64_t* dp_full = bar + 9;   // dP^T(n) done
  uint64_t* ds_ready = bar + 10; // dS^T(n) written by every gradient warp
  uint64_t* kv_done = bar + 11;  // every product done
  uint64_t* drain = bar + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kvb = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int group = p.H / p.Hkv;
  const int kv0 = kvb * FB_BKV;
  const int row0 = b * p.s;
  const int nqb = (p.s + FB_BQ - 1) / FB_BQ;
  const int qb_first = kv0 / FB_BQ;
  const int per_head = nqb - qb_first;
  const int n_it = group * per_head;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_ready, FB_GWARPS);
    mbar_init(dp_full, 1);
    mbar_init(ds_ready, FB_GWARPS);
    mbar_init(kv_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int q_last[2] = {-1, -1};  // parity of the last loads into each stage
      bool ok = true;
      mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
      for (int c = 0; c < HD / 64; ++c) {
        tma_load_2d(sK + c * C::SUB, &tmK, kv_full, kvh * HD + c * 64, row0 + kv0);
        tma_load_2d(sV + c * C::SUB, &tmV, kv_full, kvh * HD + c * 64, row0 + kv0);
      }
      int h = kvh * group, qb = qb_first;  // head and query block of iteration it
      for (int it = 0; it < n_it; ++it) {
        const int st = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        const int q0 = qb * FB_BQ, hq = h;
        if (++qb == nqb) {
          qb = qb_first;
          ++h;
        }
        if (*abort_flag || !mbar_wait(&q_empty[st], ph ^ 1)) {
          record_error(p.err, 100 + (it & 63));
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&q_full[st], C::TILE);
        for (int c = 0; c < HD / 64; ++c)
          tma_load_2d(sQ + st * C::TILE + c * C::SUB, &tmQ, &q_full[st], hq * HD + c * 64, row0 + q0);
        mbar_arrive_expect_tx(&o_full[st], C::TILE);
        for (int c = 0; c < HD / 64; ++c)
          tma_load_2d(sdO + st * C::TILE + c * C::SUB, &tmO, &o_full[st], hq * HD + c * 64, row0 + q0);
        q_last[st] = (int)ph;
      }
      if (!ok) {
        *abort_flag = 1;
        if (!mbar_wait(kv_full, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        for (int s2 = 0; s2 < 2; ++s2)
          if (q_last[s2] >= 0 && (!mbar_wait(&q_full[s2], (uint32_t)q_last[s2]) ||
                                  !mbar_wait(&o_full[s2], (uint32_t)q_last[s2])))
            record_error(p.err, DEV_TIMEOUT_TEARDOWN);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t id_s = idesc_bf16_f32(FB_BKV, FB_BQ, false, false);  // keys x queries, K = hd
      constexpr uint32_t id_kv = idesc_bf16_f32(FB_BKV, HD, false, true);  // keys x hd, K = queries (A in TMEM)
      const uint64_t dK_km = sdesc_sw128(smem_u32(sK), 16, 1024), dV_km = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dQ_km = sdesc_sw128(smem_u32(sQ), 16, 1024), dO_km = sdesc_sw128(smem_u32(sdO), 16, 1024);
      const uint64_t dQ_mn = sdesc_sw128(smem_u32(sQ), C::SUB, 1024), dO_mn = sdesc_sw128(smem_u32(sdO), C::SUB, 1024);
      constexpr uint32_t kStage = C::TILE >> 4, kMn = 2048 >> 4;  // one stage; 16 rows of a 128-byte-row tile
      bool issued = false;
      bool ok = mbar_wait(kv_full, 0) && !*abort_flag;
      if (!ok) record_error(p.err, 200);
      // S^T(n) = K Q^T into the S^T columns, once Q(n) has landed
      auto issue_s = [&](int n) -> bool {
        const int st = n & 1;
        if (*abort_flag || !mbar_wait(&q_full[st], (n >> 1) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          umma_bf16(tmem + C::C_S, dK_km + km_step(kk), dQ_km + st * kStage + km_step(kk), id_s, kk != 0);
        umma_commit(s_full);
        issued = true;
        return true;
      };
      // dP^T(n) = V dO^T into the dP^T columns, once dO(n) has landed
      auto issue_dp = [&](int n) -> bool {
        const int st = n & 1;
        if (*abort_flag || !mbar_wait(&o_full[st], (n >> 1) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          umma_bf16(tmem + C::C_DP, dV_km + km_step(kk), dO_km + st * kStage + km_step(kk), id_s, kk != 0);
        umma_commit(dp_full);
        issued = true;
        return true;
      };
      if (ok && !(issue_s(0) && issue_dp(0))) {
        record_error(p.err, 210);
        ok = false;
      }
      for (int n = 0; n < n_it && ok; ++n) {
        const int st = n & 1;
        const bool acc0 = n > 0;
        // dV += P^T(n) dO(n): K = 128 queries in 8 steps
        if (*abort_flag || !mbar_wait(p_ready, n & 1)) {
          record_error(p.err, 220 + (n & 15));
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < FB_BQ / 16; ++kk)
          umma_bf16_ts(tmem + C::C_DV, tmem + C::C_S + fk_a_col(kk), dO_mn + st * kStage + kk * kMn, id_kv,
                       acc0 || kk > 0);
        if (n + 1 < n_it && !issue_s(n + 1)) {
          record_error(p.err, 240 + (n & 15));
          ok = false;
          break;
        }
        // dK += dS^T(n) Q(n)
        if (*abort_flag || !mbar_wait(ds_ready, n & 1)) {
          record_error(p.err, 260 + (n & 15));
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < FB_BQ / 16; ++kk)
          umma_bf16_ts(tmem + C::C_DK, tmem + C::C_DP + fk_a_col(kk), dQ_mn + st * kStage + kk * kMn, id_kv,
                       acc0 || kk > 0);
        umma_commit(&q_empty[st]);
        if (n + 1 < n_it && !issue_dp(n + 1)) {
          record_error(p.err, 280 + (n & 15));
          ok = false;
          break;
        }
      }
      if (ok) umma_commit(kv_done);
      if (!ok) {
        *abort_flag = 1;
        if (issued) {
          umma_commit(drain);
          if (!mbar_wait(drain, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        }
      }
    }
  } else {
    // ---------------- gradient warps (2 .. 2 + FB_GWARPS) ----------------
    // Warp w owns tensor-memory lane quarter w mod 4 (32 key rows) and query
    // columns [32 qg, 32 qg + 32) of each block (k-steps 2 qg and 2 qg + 1).
    const int qg = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // key row == tensor-memory lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float sl2 = p.scale * 1.4426950408889634f;
    const int key = kv0 + r;
    // LSE' = LSE log2 e and D of this warp's 32 queries: lane i fetches
    // query i's pair one iteration ahead; the warp's shared slot hands them
    // to every lane (broadcast reads)
    float* sld = reinterpret_cast<float*>(smem + C::OFF_LD) + (warp - 2) * 64;
    auto fetch = [&](int hq_, int q0_, float& l, float& d) {
      const int q = q0_ + qg * FB_QW + lane;
      const int64_t i = ((int64_t)b * p.H + hq_) * p.s + q;
      l = q < p.s ? __ldg(p.LSE + i) * 1.4426950408889634f : 0.f;
      d = q < p.s ? __ldg(p.Dv + i) : 0.f;
    };
    const uint32_t s_cols = tmem + lane_base + C::C_S + qg * FB_QW;
    const uint32_t dp_cols = tmem + lane_base + C::C_DP + qg * FB_QW;
    bool ok = true;

    int h = kvh * group, qb = qb_first;  // head and query block of iteration n
    float pl, pd;
    fetch(h, qb * FB_BQ, pl, pd);
    for (int n = 0; n < n_it; ++n) {
      const int q0 = qb * FB_BQ;
      if (++qb == nqb) {
        qb = qb_first;
        ++h;
      }
      __syncwarp();
      sld[lane] = pl;
      sld[32 + lane] = pd;
      __syncwarp();
      if (n + 1 < n_it) fetch(h, qb * FB_BQ, pl, pd);
      const int qc = q0 + qg * FB_QW;  // first query of this warp's columns
      // Only blocks that touch the diagonal or a sequence end need the mask.
      const bool need_mask = (qc < kv0 + FB_BKV) || (q0 + FB_BQ > p.s) || (kv0 + FB_BKV > p.s);
      // P^T(n) = exp2(S^T sl2 - LSE'): this warp's 32 queries of key row r,
      // kept in fp32 for dS^T and written as bf16 pairs over the scores
      float pf[32];
      if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(s_full, n & 1)) {
        record_error(p.err, 300 + (n & 63));
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t sv[32];
        tmem_ld_32x32b_x32(s_cols, sv);
        tmem_ld_wait();
        auto probs = [&](auto mask_tag) {
          constexpr bool MASK = decltype(mask_tag)::value;
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 a4 = reinterpret_cast<const float4*>(sld)[i4];
            const float lv[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int i = 4 * i4 + u, qi = qc + i;
              const bool vis = !MASK || (key <= qi && qi < p.s && key < p.s);
              pf[i] = vis ? ex2(fmaf(__uint_as_float(sv[i]), sl2, -lv[u])) : 0.f;
            }
          }
        };
        if (need_mask)
          probs(std::true_type{});
        else
          probs(std::false_type{});
        uint32_t pp[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pp[e] = pack_bf16x2(pf[2 * e], pf[2 * e + 1]);
        tmem_st_32x32b_x16(s_cols, pp);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_ready);
      }
      // dS^T(n) = P^T (dP^T - D), bf16 pairs over the dP^T values
      if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(dp_full, n & 1)) {
        record_error(p.err, 340 + (n & 63));
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t dv[32], ds[16];
        tmem_ld_32x32b_x32(dp_cols, dv);
        tmem_ld_wait();
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 d4 = reinterpret_cast<const float4*>(sld + 32)[e4];
          const float dvv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int u = 0; u < 4; u += 2) {
            const int e = 4 * e4 + u;
            ds[e >> 1] = pack_bf16x2(pf[e] * (__uint_as_float(dv[e]) - dvv[u]),
                                     pf[e + 1] * (__uint_as_float(dv[e + 1]) - dvv[u + 1]));
          }
        }
        tmem_st_32x32b_x16(dp_cols, ds);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_ready);
      }
    }
    if (ok && (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(kv_done, 0))) {
      record_error(p.err, 451);
      ok = false;
    }
    if (!ok) {
      *abort_flag = 1;
    } else {
      tc_fence_after();
      fb_store_dkdv<HD>(tmem, lane_base, qg, key, row0, kvh, p);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// ===========================================================================
// dQ of the backward, query-major (head_dim 128), deterministic: one CTA per
// (128-query block, query head, sequence) sums dQ over its key blocks
// 0 .. qb in tensor memory and writes each element once, so no reductions
// and one fixed summation order:
//   S = Q K_j^T,  dP = dO V_j^T            (128 queries x 128 keys, TMEM)
//   dS = exp2(S sl2 - LSE') (dP - D)       (8 gradient warps: one query row
//        per thread, 64 keys per warp; bf16 dS written over the S columns it
//        was computed from, the A operand of the next product)
//   dQ += dS K_j                           (128 queries x hd, TMEM, A from TMEM)
// S is double-buffered, so S_{j+1} runs while block j's gradients are
// computed; dP is single (the gradient warps have read it when they signal).
// Tensor memory: S [0,128) and [128,256), dP [256,384), dQ [384,512).
// Shared memory: Q, dO, two K and two V stages (192 KB). dS of keys
// [0, 64) sits in columns [0, 32) of its S buffer and of keys [64, 128) in
// [64, 96): each warp overwrites only scores it has already read.
// ===========================================================================
namespace {

constexpr int FQ_THREADS = 320;  // producer, MMA, 8 gradient warps

template <int HD>
struct FqCfg {
  static constexpr int TILE = 128 * HD * 2;  // 128 rows x HD bf16 as HD / 64 sub-tiles of 64 columns
  static constexpr int SUB = 128 * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = TILE;
  static constexpr int OFF_K = 2 * TILE;  // [2]
  static constexpr int OFF_V = 4 * TILE;  // [2]
  static constexpr int OFF_BAR = 6 * TILE;
  static constexpr int SMEM = 1024 + OFF_BAR + 256;
  static constexpr uint32_t C_S = 0, C_DP = 256, C_DQ = 384;
};

struct FqParams {
  const float* LSE;
  const float* Dv;
  float* dQacc;
  int64_t ldqa;
  int s, H, Hkv;
  float scale;
  int* err;
};

// Tensor-memory column of the A operand (dS) for k-step kk of S buffer sb.
__device__ __forceinline__ uint32_t fq_a_col(int sb, int kk) {
  return FqCfg<128>::C_S + 128u * sb + (kk < 4 ? 8u * kk : 64u + 8u * (kk - 4));
}

template <int HD>
__global__ void __launch_bounds__(FQ_THREADS, 1)
    k_flash_bwd_dq(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO, FqParams p) {
  using C = FqCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sdO = smem + C::OFF_DO;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* qd_full = bar + 0;
  uint64_t* k_full = bar + 1;    // [2]
  uint64_t* v_full = bar + 3;    // [2]
  uint64_t* kv_empty = bar + 5;  // [2] K_j and V_j read by every product of block j
  uint64_t* s_full = bar + 7;    // [2 S buffers] S_j and dP_j in tensor memory
  uint64_t* p_full = bar + 9;    // dS_j written and dP_j read, 8 warps
  uint64_t* dq_full = bar + 10;  // every dQ product done
  uint64_t* drain = bar + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 13);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (p.H / p.Hkv);
  const int q0 = qb * 128;
  const int row0 = b * p.s;
  const int n = qb + 1;  // key blocks 0 .. qb

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
    }
    mbar_init(p_full, 8);
    mbar_init(dq_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
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
      mbar_arrive_expect_tx(qd_full, 2 * C::TILE);
      for (int c = 0; c < HD / 64; ++c) {
        tma_load_2d(sQ + c * C::SUB, &tmQ, qd_full, h * HD + c * 64, row0 + q0);
        tma_load_2d(sdO + c * C::SUB, &tmO, qd_full, h * HD + c * 64, row0 + q0);
      }
      for (int j = 0; j < n; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (*abort_flag || !mbar_wait(&kv_empty[st], ph ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[st], C::TILE);
        for (int c = 0; c < HD / 64; ++c) tma_load_2d(sK + st * C::TILE + c * C::SUB, &tmK, &k_full[st], kvh * HD + c * 64, row0 + j * 128);
        k_last[st] = (int)ph;
        mbar_arrive_expect_tx(&v_full[st], C::TILE);
        for (int c = 0; c < HD / 64; ++c) tma_load_2d(sV + st * C::TILE + c * C::SUB, &tmV, &v_full[st], kvh * HD + c * 64, row0 + j * 128);
        v_last[st] = (int)ph;
      }
      if (!ok) {
        record_error(p.err, DEV_TIMEOUT_PRODUCER);
        *abort_flag = 1;
        // let every issued copy land before the CTA's shared memory goes away
        if (!mbar_wait(qd_full, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        for (int s2 = 0; s2 < 2; ++s2) {
          if (k_last[s2] >= 0 && !mbar_wait(&k_full[s2], (uint32_t)k_last[s2])) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
          if (v_last[s2] >= 0 && !mbar_wait(&v_full[s2], (uint32_t)v_last[s2])) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false, false);   // S, dP: both operands K-major
      constexpr uint32_t id_dq = idesc_bf16_f32(128, HD, false, true);    // dQ += dS K: A in TMEM, K hd-major
      const uint64_t dQd = sdesc_sw128(smem_u32(sQ), 16, 1024), dOd = sdesc_sw128(smem_u32(sdO), 16, 1024);
      const uint64_t dKk = sdesc_sw128(smem_u32(sK), 16, 1024), dVk = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dKm = sdesc_sw128(smem_u32(sK), C::SUB, 1024);
      constexpr uint32_t kStage = C::TILE >> 4, kMn = 2048 >> 4;
      auto km = [](int kk) { return (uint32_t)(((kk >> 2) * C::SUB + (kk & 3) * 32) >> 4); };
      bool ok = mbar_wait(qd_full, 0) && !*abort_flag;
      bool issued = false;
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (*abort_flag || !mbar_wait(&k_full[st], (j >> 1) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          umma_bf16(tmem + C::C_S + 128u * (j & 1), dQd + km(kk), dKk + st * kStage + km(kk), id_s, kk != 0);
        issued = true;
        return true;
      };
      auto issue_dp = [&](int j) -> bool {
        const int st = j & 1;
        if (*abort_flag || !mbar_wait(&v_full[st], (j >> 1) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk)
          umma_bf16(tmem + C::C_DP, dOd + km(kk), dVk + st * kStage + km(kk), id_s, kk != 0);
        umma_commit(&s_full[j & 1]);  // S_j (issued earlier) and dP_j
        return true;
      };
      if (ok) ok = issue_s(0) && issue_dp(0);
      for (int j = 0; j < n && ok; ++j) {
        const int st = j & 1;
        // S buffer (j + 1) & 1 last held dS_{j-1}, read by a dQ product issued before
        if (j + 1 < n && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        if (*abort_flag || !mbar_wait(p_full, j & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          umma_bf16_ts(tmem + C::C_DQ, tmem + fq_a_col(j & 1, kk), dKm + st * kStage + kk * kMn, id_dq, (j | kk) != 0);
        umma_commit(&kv_empty[st]);
        // the gradient warps have read dP_j: dP_{j+1} may take its columns
        if (j + 1 < n && !issue_dp(j + 1)) {
          ok = false;
          break;
        }
      }
      if (ok) umma_commit(dq_full);
      if (!ok) {
        record_error(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      if (issued) {  // every MMA issued here completes before tensor memory is freed
        umma_commit(drain);
        if (!mbar_wait(drain, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
      }
    }
  } else {
    // ---------------- gradient warps (2 .. 9) ----------------
    const int wq = warp - 2;
    const int half = wq >> 2;             // keys [64 half, 64 half + 64) of each block
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;    // query row of the block == tensor-memory lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int qi = q0 + r;
    const float sl2 = p.scale * 1.4426950408889634f;
    const int64_t vi = ((int64_t)b * p.H + h) * p.s + qi;
    const float lse2 = qi < p.s ? __ldg(p.LSE + vi) * 1.4426950408889634f : 0.f;
    const float dr = qi < p.s ? __ldg(p.Dv + vi) : 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(&s_full[j & 1], (j >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sb = tmem + lane_base + C::C_S + 128u * (j & 1) + 64u * half;
      const uint32_t db = tmem + lane_base + C::C_DP + 64u * half;
      // The causal mask touches only the diagonal block (the last): query row
      // r sees keys [0, r] of it.
      auto chunk = [&](int c, auto diag_tag) {
        constexpr bool DIAG = decltype(diag_tag)::value;
        uint32_t sv[32], dv[32], ds[16];
        tmem_ld_32x32b_x32(sb + 32 * c, sv);
        tmem_ld_32x32b_x32(db + 32 * c, dv);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float g[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int kl = 64 * half + 32 * c + e + u;
            const float pr = ex2(fmaf(__uint_as_float(sv[e + u]), sl2, -lse2));
            g[u] = (DIAG && kl > r) ? 0.f : pr * (__uint_as_float(dv[e + u]) - dr);
          }
          ds[e >> 1] = pack_bf16x2(g[0], g[1]);
        }
        // keys [64 half + 32 c, +32) -> columns 64 half + 16 c .. + 16 (key k in column k / 2
        // within the half's 32 columns): scores this warp has already read
        tmem_st_32x32b_x16(sb + 16 * c, ds);
      };
      if (j == n - 1) {
        chunk(0, std::true_type{});
        chunk(1, std::true_type{});
      } else {
        chunk(0, std::false_type{});
        chunk(1, std::false_type{});
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && (__any_sync(0xffffffffu, *abort_flag) || !mbar_wait_warp(dq_full, 0))) ok = false;
    if (!ok) {
      record_error(p.err, DEV_TIMEOUT_EPILOGUE);
      *abort_flag = 1;
    } else {
      tc_fence_after();
      float* dst = p.dQacc + (int64_t)(row0 + qi) * p.ldqa + (int64_t)h * HD + (HD / 2) * half;
#pragma unroll 1
      for (int c = 0; c < HD / 64; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + C::C_DQ + (HD / 2) * half + 32u * c, v);  // warp-collective
        tmem_ld_wait();
        if (qi < p.s) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + 32 * c + e) =
                make_float4(__uint_as_float(v[e]) * p.scale, __uint_as_float(v[e + 1]) * p.scale,
                            __uint_as_float(v[e + 2]) * p.scale, __uint_as_float(v[e + 3]) * p.scale);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// dQ of the tensor-core backward (head dim 64 or 128) by the query-major kernel: writes every
// element of dq_acc's head columns once (scaled, before RoPE's transpose).
// a.dvec must already hold D = rowsum(dO * O).
namespace {
template <int HD>
int launch_bwd_dq(const AttnArgs& a, cudaStream_t st, int* err) {
  using C = FqCfg<HD>;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(k_flash_bwd_dq<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
      return MT_ERR_CUDA;
    attr = true;
  }
  const int64_t T = (int64_t)a.b * a.s;
  CUtensorMap mq, mk, mv, mo;
  if (!make_tensor_map_2d_bf16(&mq, a.q, (int64_t)a.H * HD, T, a.ldqkv, 128) ||
      !make_tensor_map_2d_bf16(&mk, a.k, (int64_t)a.Hkv * HD, T, a.ldqkv, 128) ||
      !make_tensor_map_2d_bf16(&mv, a.v, (int64_t)a.Hkv * HD, T, a.ldqkv, 128) ||
      !make_tensor_map_2d_bf16(&mo, a.dout, (int64_t)a.H * HD, T, a.ldo, 128))
    return MT_ERR_ARG;
  FqParams p{a.lse, a.dvec, a.dq_acc, a.ldqa, a.s, a.H, a.Hkv, a.scale, err};
  dim3 grid((a.s + 127) / 128, a.H, a.b);
  k_flash_bwd_dq<HD><<<grid, FQ_THREADS, C::SMEM, st>>>(mq, mk, mv, mo, p);
  return launch_status();
}
}  // namespace

int attention_bwd_dq_tc(const AttnArgs& a, cudaStream_t st, int* err) {
  if (a.hd != 64 && a.hd != 128) return MT_ERR_CONFIG;
  if ((reinterpret_cast<uintptr_t>(a.dq_acc) & 15) || (a.ldqa % 4)) return MT_ERR_ARG;
  return a.hd == 128 ? launch_bwd_dq<128>(a, st, err) : launch_bwd_dq<64>(a, st, err);
}

// Key-major part of the tensor-core backward. a.dvec must already hold
// D = rowsum(dO * O) and, unless skip_dq, a.dq_acc must be zeroed; the caller
// casts dQ. skip_dq: dK and dV only, by the pipelined key-major kernel (head
// dim 64 or 128; dQ from attention_bwd_dq_tc); otherwise the fused kernel,
// dQ by reductions (head dim 128).
namespace {
// The key-major kernel for head dim HD: the pipelined dK/dV-only one
// (skip_dq), or the fused one with dQ by reductions (HD = 128 only).
template <int HD>
int launch_bwd_key_major(const AttnArgs& a, cudaStream_t st, int* err, bool skip_dq) {
  static bool attr = false;
  if (!attr) {
    if ((HD == 128 && cudaFuncSetAttribute(k_flash_bwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           FbCfg::SMEM) != cudaSuccess) ||
        cudaFuncSetAttribute(k_flash_bwd_kv<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, FkCfg<HD>::SMEM) !=
            cudaSuccess)
      return MT_ERR_CUDA;
    attr = true;
  }
  const int64_t T = (int64_t)a.b * a.s;
  CUtensorMap mq, mk, mv, mo;
  if (!make_tensor_map_2d_bf16(&mq, a.q, (int64_t)a.H * HD, T, a.ldqkv, FB_BQ) ||
      !make_tensor_map_2d_bf16(&mk, a.k, (int64_t)a.Hkv * HD, T, a.ldqkv, FB_BKV) ||
      !make_tensor_map_2d_bf16(&mv, a.v, (int64_t)a.Hkv * HD, T, a.ldqkv, FB_BKV) ||
      !make_tensor_map_2d_bf16(&mo, a.dout, (int64_t)a.H * HD, T, a.ldo, FB_BQ))
    return MT_ERR_ARG;
  const bool vec = (a.s % 4 == 0) && ((reinterpret_cast<uintptr_t>(a.lse) | reinterpret_cast<uintptr_t>(a.dvec)) & 15) == 0;
  FbParams p{a.lse, a.dvec, a.dq_acc, a.ldqa, (__nv_bfloat16*)a.dk, (__nv_bfloat16*)a.dv, a.lddkv, a.s, a.H, a.Hkv,
             a.scale, a.rope_cos, a.rope_sin, err, vec ? 1 : 0};
  dim3 grid((a.s + FB_BKV - 1) / FB_BKV, a.Hkv, a.b);
  if (skip_dq)
    k_flash_bwd_kv<HD><<<grid, FB_THREADS, FkCfg<HD>::SMEM, st>>>(mq, mk, mv, mo, p);
  else
    k_flash_bwd_tc<<<grid, FB_THREADS, FbCfg::SMEM, st>>>(mq, mk, mv, mo, p);
  return launch_status();
}
}  // namespace

int attention_bwd_tc_main(const AttnArgs& a, cudaStream_t st, int* err, bool skip_dq) {
  if (a.hd == 128) return launch_bwd_key_major<128>(a, st, err, skip_dq);
  if (a.hd == 64 && skip_dq) return launch_bwd_key_major<64>(a, st, err, true);
  return MT_ERR_CONFIG;
}

}  // namespace mt
