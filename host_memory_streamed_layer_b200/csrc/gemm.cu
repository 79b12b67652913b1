// Persistent tcgen05 bf16 GEMM for sm_100a: C[M,N] = A[M,K] * B[N,K]^T, fp32
// accumulation in tensor memory, operands staged by TMA (no multicast).
//
// This is the dense contraction of every projection in the streamed decoder
// layer (MegaTrain, "Full Precision Training of 100B+ Parameter Large Language
// Models on a Single GPU", abstract; saify.me, "The memory-centric design":
// each streamed layer's matrix products run on the GPU): the forward products
// u Wqkv^T, a Wo^T, w Wgu^T, act Wd^T, the input-gradient products dY W and
// the weight-gradient products dY^T X of their backward.
//
// Operands may be K-major (the reduction index is contiguous) or MN-major (the
// output index is contiguous), which covers all three products without a
// transpose kernel:
//   forward   Y  = X  W^T : A = X  [T, in]  K-major,  B = W [out, in] K-major
//   input grad dX = dY W   : A = dY [T, out] K-major,  B = W [out, in] MN-major
//   weight grad dW = dY^T X: A = dY [T, out] MN-major, B = X [T, in]  MN-major
//
// Kernel structure (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: fills a ring of shared-memory stages
//   warp 1      MMA issuer: one thread issues tcgen05.mma 128 x BN x 16
//   warps 2..5  epilogue: tcgen05.ld from tensor memory, convert, store
// The accumulator is double-buffered in tensor memory (2 x BN columns) so the
// epilogue of tile i overlaps the main loop of tile i+1.
//
// Large problems run the CTA-pair form of the same kernel (clusters of two
// CTAs, tcgen05.mma.cta_group::2 on 256 x BN tiles): each SM then stages half
// of the B tile, which halves its shared-memory traffic for B and leaves room
// for deeper pipelines. Small problems (fewer 256-row tiles than SM pairs) use
// the single-CTA form.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "mt_common.cuh"
#include "mt_internal.h"

namespace mt {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes: one swizzle row
constexpr int NUM_THREADS = 192;
constexpr int GROUP_M = 16;  // tile raster: 16 M-tiles share a band of N-tiles

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
};

struct Params {
  int M, N, K;
  void* C;
  int64_t ldc;
  const float* R;
  int64_t ldr;
  int epi;
  int* err;
  RopeDesc rope;
  // Limit of the single-CTA kernel's main-loop waits (ns; 0: give up at the
  // first incomplete poll). Waits that let the CTA exit safely use kWaitLimitNs.
  uint64_t wait_ns;
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
  const int per_group = GROUP_M * num_n;
  const int g = tile / per_group;
  const int first_m = g * GROUP_M;
  const int gsize = min(num_m - first_m, GROUP_M);
  const int r = tile - g * per_group;
  mb = first_m + r % gsize;
  nb = r / gsize;
}

// Converts and stores one warp's accumulator rows of an output tile: thread i
// of the warp owns output row `row` (its tensor-memory lane), `tbase` is the
// tensor-memory address of the warp's lanes at the tile's first column and
// `col_base` the tile's first output column; NC columns are stored.
template <int NC>
__device__ __forceinline__ void store_tile_rows(const Params& p, uint32_t tbase, int row, int col_base) {
  const bool row_ok = row < p.M;
  if (p.epi == EPI_BF16_ROPE) {
    // Heads of width hd tile NC exactly; rotate-half pairs live in 32-column
    // chunks a and a + hd/64 of the same head.
    const int hd = p.rope.hd;
    const int pos = row_ok ? row % p.rope.seq : 0;
    const float* cs = p.rope.cos + (int64_t)pos * (hd >> 1);
    const float* sn = p.rope.sin + (int64_t)pos * (hd >> 1);
#pragma unroll 1
    for (int h0 = 0; h0 < NC; h0 += hd) {
#pragma unroll 1
      for (int a = 0; a < hd / 64; ++a) {
        uint32_t x1[32], x2[32];
        tmem_ld_32x32b_x32(tbase + h0 + a * 32, x1);
        tmem_ld_32x32b_x32(tbase + h0 + a * 32 + hd / 2, x2);
        tmem_ld_wait();
        const int c1 = col_base + h0 + a * 32;
        const int c2 = c1 + hd / 2;
        if (!row_ok || c2 >= p.N) continue;  // N is a multiple of hd: the pair is whole or absent
        __nv_bfloat16* o1 = reinterpret_cast<__nv_bfloat16*>(p.C) + (int64_t)row * p.ldc + c1;
        __nv_bfloat16* o2 = o1 + hd / 2;
        const bool rot = c1 < p.rope.cols;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float y1[8], y2[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a1 = __uint_as_float(x1[8 * j + e]), a2 = __uint_as_float(x2[8 * j + e]);
            if (rot) {
              const float cv = cs[a * 32 + 8 * j + e], sv = sn[a * 32 + 8 * j + e];
              y1[e] = a1 * cv - a2 * sv;
              y2[e] = a2 * cv + a1 * sv;
            } else {
              y1[e] = a1;
              y2[e] = a2;
            }
          }
          reinterpret_cast<uint4*>(o1)[j] = make_uint4(pack_bf16x2(y1[0], y1[1]), pack_bf16x2(y1[2], y1[3]),
                                                       pack_bf16x2(y1[4], y1[5]), pack_bf16x2(y1[6], y1[7]));
          reinterpret_cast<uint4*>(o2)[j] = make_uint4(pack_bf16x2(y2[0], y2[1]), pack_bf16x2(y2[2], y2[3]),
                                                       pack_bf16x2(y2[4], y2[5]), pack_bf16x2(y2[6], y2[7]));
        }
      }
    }
  } else {
#pragma unroll 1
    for (int c = 0; c < NC / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tbase + c * 32, r);
      tmem_ld_wait();
      const int col0 = col_base + c * 32;
      if (!row_ok || col0 >= p.N) continue;
      const bool full_cols = col0 + 32 <= p.N;
      if (p.epi == EPI_BF16) {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.C) + (int64_t)row * p.ldc + col0;
        if (full_cols) {
          uint4* o4 = reinterpret_cast<uint4*>(out);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
            w.y = pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
            w.z = pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
            w.w = pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
            o4[j] = w;
          }
        } else {
          const int nv = p.N - col0;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nv) out[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
        }
      } else {
        float* out = reinterpret_cast<float*>(p.C) + (int64_t)row * p.ldc + col0;
        const float* res = (p.epi == EPI_F32_ADD) ? p.R + (int64_t)row * p.ldr + col0 : nullptr;
        if (full_cols) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 v = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                   __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
            if (res) {
              const float4 q = reinterpret_cast<const float4*>(res)[j];
              v.x += q.x;
              v.y += q.y;
              v.z += q.z;
              v.w += q.w;
            }
            reinterpret_cast<float4*>(out)[j] = v;
          }
        } else {
          const int nv = p.N - col0;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nv) out[j] = __uint_as_float(r[j]) + (res ? res[j] : 0.f);
        }
      }
    }
  }
}

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_bf16(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_m = (p.M + BM - 1) / BM;
  const int num_n = (p.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (p.K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;  // stages filled so far (for the teardown)
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, num_m, num_n, mb, nb);
        const int m0 = mb * BM, n0 = nb * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (*abort_flag || !mbar_wait(&empty[stage], phase ^ 1, p.wait_ns)) {
            record_error(p.err, DEV_TIMEOUT_PRODUCER);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          const int k0 = kb * BK;
          if (!A_MN) {
            tma_load_2d(sa, &tmA, &full[stage], k0, m0);
          } else {
#pragma unroll
            for (int i = 0; i < BM / 64; ++i) tma_load_2d(sa + i * 8192, &tmA, &full[stage], m0 + i * 64, k0);
          }
          if (!B_MN) {
            tma_load_2d(sb, &tmB, &full[stage], k0, n0);
          } else {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i) tma_load_2d(sb + i * 8192, &tmB, &full[stage], n0 + i * 64, k0);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (ok) {
        // Producer tail: wait until the MMA has released every stage, so that no
        // commit-arrive on this CTA's barriers is in flight when it exits. If
        // another role gives up meanwhile, the MMA may never release them:
        // drain this CTA's copies instead (below).
        for (int i = 0; i < C::STAGES && ok; ++i) {
          const uint64_t t0 = globaltimer();
          while (!mbar_wait(&empty[stage], phase ^ 1, 0)) {
            if (*abort_flag) {
              ok = false;
              break;
            }
            if (globaltimer() - t0 > kWaitLimitNs) {
              record_error(p.err, DEV_TIMEOUT_TEARDOWN);
              *abort_flag = 1;
              ok = false;
              break;
            }
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // Let every issued copy land before the CTA's shared memory goes away:
        // stage s was last filled by fill number s + STAGES * q (largest below
        // `issued`), in phase q mod 2.
        for (int s = 0; s < C::STAGES && s < issued; ++s) {
          const int q = (issued - 1 - s) / C::STAGES;
          if (!mbar_wait(&full[s], (uint32_t)(q & 1))) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
      // Descriptors of stage 0. Stage s and k-step kk only move the 14-bit
      // start-address field (address / 16; shared memory stays below 256 KB),
      // so the loop adds constants instead of rebuilding descriptors: the
      // issuing thread must keep pace with 128-cycle MMAs.
      const uint32_t s0 = smem_u32(smem);
      const uint64_t a0 = sdesc_sw128(s0, A_MN ? 8192 : 16, 1024);
      const uint64_t b0 = sdesc_sw128(s0 + C::A_BYTES, B_MN ? 8192 : 16, 1024);
      constexpr uint32_t kStage = C::STAGE_BYTES >> 4;
      constexpr uint32_t kAStep = (A_MN ? 2048 : 32) >> 4, kBStep = (B_MN ? 2048 : 32) >> 4;
      const uint32_t full0 = smem_u32(&full[0]), empty0 = smem_u32(&empty[0]);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (*abort_flag || !mbar_wait(&tempty[acc], acc_phase ^ 1, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          // A stalled producer shows up here as a wait that runs out.
          if (!mbar_wait_u32(full0 + 8 * stage, phase, p.wait_ns)) {
            ok = false;
            break;
          }
          // No tcgen05 fence here: the stage's bytes were written by TMA and
          // published through this mbarrier, which orders them for the MMAs'
          // shared-memory reads. A fence per k-block measurably stalled the
          // tensor pipe (a 64-deep k-block took ~690 instead of 512 cycles).
          const uint64_t ad = a0 + stage * kStage, bd = b0 + stage * kStage;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) umma_bf16(d_tmem, ad + kk * kAStep, bd + kk * kBStep, idesc, (kb | kk) != 0);
          issued = true;
          umma_commit_u32(empty0 + 8 * stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok) {
        record_error(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      // Every MMA issued here completes before tensor memory is freed, also
      // when the epilogue gave up on an accumulator it will never read.
      if (issued) {
        umma_commit(drain);
        if (!mbar_wait(drain, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;  // tensor-memory lanes this warp may read
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      // warp-uniform outcome: the tcgen05.ld below is warp-collective
      if (__any_sync(0xffffffffu, *abort_flag) ||
          !__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, p.wait_ns))) {
        record_error(p.err, DEV_TIMEOUT_EPILOGUE);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      int mb, nb;
      tile_coords(tile, num_m, num_n, mb, nb);
      const int row = mb * BM + quarter * 32 + lane;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      store_tile_rows<BN>(p, tbase, row, nb * BN);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair variant: a cluster of two CTAs on two SMs computes a 256 x BN tile
// with tcgen05.mma.cta_group::2. Each CTA stages its own 128 rows of A and
// half of the tile's BN rows of B, so every SM streams half the B operand of
// the single-CTA kernel per flop and the pipeline holds more stages. The
// leader (rank 0) issues the MMAs; both CTAs' copies complete on the leader's
// `full` barriers, the leader's commits release both CTAs' `empty` stages and
// both `tfull` accumulators, and both CTAs' epilogue warps release the
// leader's `tempty`. Each CTA's tensor memory holds its 128 accumulator rows.
// ---------------------------------------------------------------------------
template <int BN>
struct PairCfg {
  static constexpr int TILE_M = 2 * BM;                  // rows of the pair tile
  static constexpr int A_BYTES = BM * BK * 2;            // this CTA's 128 rows of A
  static constexpr int B_BYTES = (BN / 2) * BK * 2;      // this CTA's half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // per CTA
  static constexpr int STAGES = (BN == 256) ? 6 : 8;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
};

template <int BN, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_bf16_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
  using C = PairCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);  // 4 epilogue warps in each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barrier initialisation and the allocation are visible to both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_m = (p.M + C::TILE_M - 1) / C::TILE_M;
  const int num_n = (p.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (p.K + BK - 1) / BK;
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;  // stages filled so far (for the teardown)
      const uint32_t fb0 = mapa_shared(smem_u32(&full[0]), 0);  // the leader's full barriers
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int mb, nb;
        tile_coords(tile, num_m, num_n, mb, nb);
        const int m0 = mb * C::TILE_M + (int)rank * BM;
        const int n0 = nb * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (*abort_flag || !mbar_wait(&empty[stage], phase ^ 1)) {
            record_error(p.err, DEV_TIMEOUT_PRODUCER);
            *abort_flag = 1;
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          const uint32_t fb = fb0 + 8 * stage;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          const int k0 = kb * BK;
          if (!A_MN) {
            tma_load_2d_pair(sa, &tmA, fb, k0, m0);
          } else {
#pragma unroll
            for (int i = 0; i < BM / 64; ++i) tma_load_2d_pair(sa + i * 8192, &tmA, fb, m0 + i * 64, k0);
          }
          if (!B_MN) {
            tma_load_2d_pair(sb, &tmB, fb, k0, n0);
          } else {
#pragma unroll
            for (int i = 0; i < BN / 128; ++i) tma_load_2d_pair(sb + i * 8192, &tmB, fb, n0 + i * 64, k0);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (ok) {
        // Producer tail: wait until the leader's MMA has released every stage of
        // this CTA, so that no commit-arrive from the peer is in flight when this
        // CTA exits.
        for (int i = 0; i < C::STAGES; ++i) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) {
            record_error(p.err, DEV_TIMEOUT_TEARDOWN);
            break;
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      } else if (rank == 0) {
        // The leader's full barriers count both CTAs' bytes: once every armed
        // phase has completed, no copy of either CTA is still in flight.
        for (int s = 0; s < C::STAGES && s < issued; ++s) {
          const int q = (issued - 1 - s) / C::STAGES;
          if (!mbar_wait(&full[s], (uint32_t)(q & 1))) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader only) ----------------
      constexpr uint32_t idesc = idesc_bf16_f32(C::TILE_M, BN, A_MN, B_MN);
      // Stage-0 descriptors plus constant steps (see the single-CTA kernel).
      const uint32_t s0 = smem_u32(smem);
      const uint64_t a0 = sdesc_sw128(s0, A_MN ? 8192 : 16, 1024);
      const uint64_t b0 = sdesc_sw128(s0 + C::A_BYTES, B_MN ? 8192 : 16, 1024);
      constexpr uint32_t kStage = C::STAGE_BYTES >> 4;
      constexpr uint32_t kAStep = (A_MN ? 2048 : 32) >> 4, kBStep = (B_MN ? 2048 : 32) >> 4;
      const uint32_t full0 = smem_u32(&full[0]), empty0 = smem_u32(&empty[0]);
      const uint32_t empty0_peer = mapa_shared(empty0, 1);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        if (*abort_flag || !mbar_wait_cluster(&tempty[acc], acc_phase ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_u32(full0 + 8 * stage, phase)) {
            ok = false;
            break;
          }
          // No tcgen05 fence here: the stage's bytes were written by TMA and
          // published through this mbarrier, which orders them for the MMAs'
          // shared-memory reads. A fence per k-block measurably stalled the
          // tensor pipe (a 64-deep k-block took ~690 instead of 512 cycles).
          const uint64_t ad = a0 + stage * kStage, bd = b0 + stage * kStage;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_pair(d_tmem, ad + kk * kAStep, bd + kk * kBStep, idesc, (kb | kk) != 0);
          issued = true;
          umma_commit_pair(empty0 + 8 * stage);
          umma_commit_pair(empty0_peer + 8 * stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        const uint32_t tb = smem_u32(&tfull[acc]);
        umma_commit_pair(tb);
        umma_commit_pair(mapa_shared(tb, 1));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok) {
        record_error(p.err, DEV_TIMEOUT_MMA);
        *abort_flag = 1;
      }
      if (issued) {
        umma_commit_pair(smem_u32(drain));
        if (!mbar_wait(drain, 0)) record_error(p.err, DEV_TIMEOUT_TEARDOWN);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5 of both CTAs) ----------------
    const int quarter = warp & 3;  // tensor-memory lanes this warp may read
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs) {
      // warp-uniform outcome: the tcgen05.ld below is warp-collective
      if (__any_sync(0xffffffffu, *abort_flag) || !__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase))) {
        record_error(p.err, DEV_TIMEOUT_EPILOGUE);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      int mb, nb;
      tile_coords(tile, num_m, num_n, mb, nb);
      const int row = mb * C::TILE_M + (int)rank * BM + quarter * 32 + lane;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      store_tile_rows<BN>(p, tbase, row, nb * BN);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(&tempty[acc]);
        else
          mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();  // no MMA of the pair and no tensor-memory read is outstanding
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

}  // namespace

// 2-D bf16 tensor map: inner extent `inner` (contiguous), outer extent `outer`,
// row pitch `ld` elements, box {64, box_outer}, 128-byte swizzle, zero fill.
bool make_tensor_map_2d_bf16(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
                             int box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D fp32 TMA map without swizzle: inner extent (contiguous), outer extent,
// row pitch ld (elements), box {box_inner, box_outer}. Used for reductions.
bool make_tensor_map_2d_f32(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
                            int box_inner, int box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 4)};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

int g_num_sms = 0;
// Main-loop wait limit of the single-CTA kernel for later launches (ns).
uint64_t g_wait_ns = kWaitLimitNs;
// Kernel family: 0 automatic, 1 single-CTA only, 2 CTA pairs wherever they fit
// (MT_GEMM_VARIANT = auto | single | pair, read once; for A/B measurements).
int g_variant = -1;

template <int BN, bool A_MN, bool B_MN>
int launch(const GemmDesc& g, cudaStream_t st, int* err) {
  using C = Cfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(k_gemm_bf16<BN, A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return MT_ERR_CUDA;
    attr_set = true;
  }
  CUtensorMap ta, tb;
  bool ok = A_MN ? make_tensor_map_2d_bf16(&ta, g.A, g.M, g.K, g.lda, 64)
              : make_tensor_map_2d_bf16(&ta, g.A, g.K, g.M, g.lda, BM);
  ok = ok && (B_MN ? make_tensor_map_2d_bf16(&tb, g.B, g.N, g.K, g.ldb, 64)
                    : make_tensor_map_2d_bf16(&tb, g.B, g.K, g.N, g.ldb, BN));
  if (!ok) return MT_ERR_ARG;
  Params p{g.M, g.N, g.K, g.C, g.ldc, g.R, g.ldr, g.epi, err, g.rope, g_wait_ns};
  const int tiles = ((g.M + BM - 1) / BM) * ((g.N + BN - 1) / BN);
  const int grid = tiles < g_num_sms ? tiles : g_num_sms;
  k_gemm_bf16<BN, A_MN, B_MN><<<grid, NUM_THREADS, C::SMEM, st>>>(ta, tb, p);
  return launch_status();
}

template <int BN>
int dispatch_major(const GemmDesc& g, cudaStream_t st, int* err) {
  if (!g.a_mn && !g.b_mn) return launch<BN, false, false>(g, st, err);
  if (!g.a_mn && g.b_mn) return launch<BN, false, true>(g, st, err);
  if (g.a_mn && !g.b_mn) return launch<BN, true, false>(g, st, err);
  return launch<BN, true, true>(g, st, err);
}

template <int BN, bool A_MN, bool B_MN>
int launch_pair(const GemmDesc& g, int max_pairs, cudaStream_t st, int* err) {
  using C = PairCfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(k_gemm_bf16_pair<BN, A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM) != cudaSuccess)
      return MT_ERR_CUDA;
    attr_set = true;
  }
  CUtensorMap ta, tb;
  bool ok = A_MN ? make_tensor_map_2d_bf16(&ta, g.A, g.M, g.K, g.lda, 64)
                 : make_tensor_map_2d_bf16(&ta, g.A, g.K, g.M, g.lda, BM);
  ok = ok && (B_MN ? make_tensor_map_2d_bf16(&tb, g.B, g.N, g.K, g.ldb, 64)
                   : make_tensor_map_2d_bf16(&tb, g.B, g.K, g.N, g.ldb, BN / 2));
  if (!ok) return MT_ERR_ARG;
  // The pair kernel keeps the fixed limit: its two producers would have to
  // agree on the last stage filled before a shorter wait could unwind it.
  Params p{g.M, g.N, g.K, g.C, g.ldc, g.R, g.ldr, g.epi, err, g.rope, kWaitLimitNs};
  const int tiles = ((g.M + C::TILE_M - 1) / C::TILE_M) * ((g.N + BN - 1) / BN);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Pairs that can be resident at once (a GPC with an odd number of free SMs
  // leaves one SM out of the pairing).
  static int resident = 0;
  if (resident == 0) {
    cfg.gridDim = dim3(2 * max_pairs, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&resident, k_gemm_bf16_pair<BN, A_MN, B_MN>, &cfg) != cudaSuccess ||
        resident <= 0) {
      cudaGetLastError();
      resident = max_pairs;
    }
  }
  const int cap = resident < max_pairs ? resident : max_pairs;
  const int pairs = tiles < cap ? tiles : cap;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cudaLaunchKernelEx(&cfg, k_gemm_bf16_pair<BN, A_MN, B_MN>, ta, tb, p);
  return launch_status();
}

template <int BN>
int dispatch_pair(const GemmDesc& g, int max_pairs, cudaStream_t st, int* err) {
  if (!g.a_mn && !g.b_mn) return launch_pair<BN, false, false>(g, max_pairs, st, err);
  if (!g.a_mn && g.b_mn) return launch_pair<BN, false, true>(g, max_pairs, st, err);
  if (g.a_mn && !g.b_mn) return launch_pair<BN, true, false>(g, max_pairs, st, err);
  return launch_pair<BN, true, true>(g, max_pairs, st, err);
}

// Automatic choice of the pair kernel. Measured on the decoder layer's shapes
// (B200): pairs are 2-8 % faster than single-CTA tiles for every product whose
// A operand is K-major (forward and input-gradient products, LM head). For the
// weight gradients (both operands MN-major) 256-wide pair tiles tie or win
// (q,k,v and gate|up), while 128-wide pair tiles lose by 20-30 % (down and O
// projections): those stay on single-CTA tiles.
bool use_pair_auto(const GemmDesc& g, bool pair_tile_256) { return !g.a_mn || pair_tile_256; }

// Fraction of the pairs' time spent on real tiles when `tiles` tiles are dealt
// round-robin to `pairs` persistent pairs.
double wave_efficiency(int tiles, int pairs) {
  const int waves = (tiles + pairs - 1) / pairs;
  return (double)tiles / ((double)waves * pairs);
}

}  // namespace

int gemm_bf16(const GemmDesc& g, cudaStream_t st, int* err) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return (g.M == 0 || g.N == 0) ? MT_OK : MT_ERR_ARG;
  if (!g.A || !g.B || !g.C) return MT_ERR_ARG;
  if (g.epi == EPI_F32_ADD && !g.R) return MT_ERR_ARG;
  if (g.epi == EPI_BF16_ROPE) {
    const RopeDesc& r = g.rope;
    if (!r.cos || !r.sin || (r.hd != 64 && r.hd != 128) || r.seq <= 0 || (g.N % r.hd) || r.cols < 0) return MT_ERR_ARG;
  }
  // TMA: 16-byte aligned base and row pitch; 16-byte aligned epilogue stores.
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(g.A) || !al16(g.B) || !al16(g.C) || (g.R && !al16(g.R))) return MT_ERR_ARG;
  if ((g.lda % 8) || (g.ldb % 8) || (g.ldc % 8) || (g.R && (g.ldr % 4))) return MT_ERR_ARG;
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) return MT_ERR_CUDA;
  }
  if (g_variant < 0) {
    const char* e = getenv("MT_GEMM_VARIANT");
    g_variant = (e && !strcmp(e, "single")) ? 1 : (e && !strcmp(e, "pair")) ? 2 : 0;
  }
  // CTA pairs (256-row tiles) when the pair tiles fill every SM pair at least
  // once; the pair tile's width is 256 unless 128 quantizes into waves clearly
  // better. Small problems use the single-CTA kernel.
  const int max_pairs = g_num_sms / 2;
  const int tm = (g.M + 2 * BM - 1) / (2 * BM);
  const int t256 = tm * ((g.N + 255) / 256), t128 = tm * ((g.N + 127) / 128);
  const bool fits256 = g.N > 128 && t256 >= max_pairs;
  const bool prefer256 = fits256 && wave_efficiency(t128, max_pairs) <= wave_efficiency(t256, max_pairs) + 0.08;
  const bool pair_ok = g_variant == 2 || (g_variant == 0 && use_pair_auto(g, prefer256));
  if (pair_ok && fits256) {
    if (!prefer256) return dispatch_pair<128>(g, max_pairs, st, err);
    return dispatch_pair<256>(g, max_pairs, st, err);
  }
  if (pair_ok && t128 >= max_pairs) return dispatch_pair<128>(g, max_pairs, st, err);
  const int tiles256 = ((g.M + BM - 1) / BM) * ((g.N + 255) / 256);
  if (g.N > 128 && tiles256 >= g_num_sms) return dispatch_major<256>(g, st, err);
  return dispatch_major<128>(g, st, err);
}

uint64_t gemm_wait_limit_ns(uint64_t ns) {
  const uint64_t prev = g_wait_ns;
  g_wait_ns = ns;
  return prev;
}

int gemm_variant(int v) {
  const int prev = g_variant < 0 ? 0 : g_variant;
  if (v >= 0 && v <= 2) g_variant = v;
  return prev;
}

}  // namespace mt
