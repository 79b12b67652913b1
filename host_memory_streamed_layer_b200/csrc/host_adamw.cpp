// Host AdamW (AVX-512 with a portable fallback) and the worker pool.
#include "host_adamw.h"

#include "mt.h"
#include "mt_kernels.h"

#include <algorithm>

#include <immintrin.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>
#include <sys/mman.h>

#include <chrono>
#include <thread>

namespace mt {

uint16_t bf16_rne(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);  // quiet NaN
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

namespace {

inline float bf16_to_f32(uint16_t h) {
  const uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// G is the gradient's element type: float, or uint16_t holding bf16 bits.
template <typename G>
void adamw_scalar(float* p, const G* g, float* m, float* v, uint16_t* pb, size_t n, float decay, float b1,
                  float b2, float step, float inv_sqrt_bc2, float eps) {
  const float c1 = 1.f - b1, c2 = 1.f - b2;
  for (size_t i = 0; i < n; ++i) {
    float gi = 0.f;
    if (g) {
      if constexpr (sizeof(G) == 2)
        gi = bf16_to_f32(g[i]);
      else
        gi = g[i];
    }
    const float mi = b1 * m[i] + c1 * gi;
    const float vi = b2 * v[i] + c2 * gi * gi;
    const float pi = p[i] * decay - step * mi / (sqrtf(vi) * inv_sqrt_bc2 + eps);
    m[i] = mi;
    v[i] = vi;
    p[i] = pi;
    if (pb) pb[i] = bf16_rne(pi);
  }
}

__attribute__((target("avx512f,avx512bw"))) inline __m256i bf16x16_rne(__m512 x) {
  const __m512i u = _mm512_castps_si512(x);
  const __m512i lsb = _mm512_and_si512(_mm512_srli_epi32(u, 16), _mm512_set1_epi32(1));
  __m512i r = _mm512_add_epi32(u, _mm512_add_epi32(lsb, _mm512_set1_epi32(0x7fff)));
  r = _mm512_srli_epi32(r, 16);
  // NaN -> quiet NaN with the same sign and top payload bits
  const __mmask16 nan = _mm512_cmp_ps_mask(x, x, _CMP_UNORD_Q);
  const __m512i qn = _mm512_or_si512(_mm512_srli_epi32(u, 16), _mm512_set1_epi32(0x40));
  r = _mm512_mask_mov_epi32(r, nan, qn);
  return _mm512_cvtepi32_epi16(r);
}

// The bf16 copy is only written (the next step's H2D reads it), so it is
// stored with non-temporal stores when 32-byte aligned: no read-for-ownership.
// HAS_G = false is the update of a zero gradient (embedding rows no token of
// the batch touches): the moments only decay and no gradient is read; the
// result is bit-identical to reading zeros (b m + 0 rounds like b m).
// G = uint16_t reads a bf16 gradient (exactly widened to fp32).
// p, m and v keep ordinary stores: their lines were just read, and streaming
// them out with non-temporal stores measured slower on the B200 hosts' DRAM.
template <bool HAS_G, typename G = float>
__attribute__((target("avx512f,avx512bw"))) void adamw_avx512(float* p, const G* g, float* m, float* v,
                                                              uint16_t* pb, size_t n, float decay, float b1, float b2,
                                                              float step, float inv_sqrt_bc2, float eps) {
  const bool nt = pb && ((reinterpret_cast<uintptr_t>(pb) & 31) == 0);
  const __m512 vb1 = _mm512_set1_ps(b1), vc1 = _mm512_set1_ps(1.f - b1);
  const __m512 vb2 = _mm512_set1_ps(b2), vc2 = _mm512_set1_ps(1.f - b2);
  const __m512 vdec = _mm512_set1_ps(decay), vstep = _mm512_set1_ps(step);
  const __m512 vibc2 = _mm512_set1_ps(inv_sqrt_bc2), veps = _mm512_set1_ps(eps);
  size_t i = 0;
  for (; i + 16 <= n; i += 16) {
    __m512 mi, vi;
    if (HAS_G) {
      __m512 gi;
      if constexpr (sizeof(G) == 2)
        gi = _mm512_castsi512_ps(_mm512_slli_epi32(
            _mm512_cvtepu16_epi32(_mm256_loadu_si256(reinterpret_cast<const __m256i*>(g + i))), 16));
      else
        gi = _mm512_loadu_ps(reinterpret_cast<const float*>(g) + i);
      mi = _mm512_fmadd_ps(vb1, _mm512_loadu_ps(m + i), _mm512_mul_ps(vc1, gi));
      vi = _mm512_fmadd_ps(vb2, _mm512_loadu_ps(v + i), _mm512_mul_ps(vc2, _mm512_mul_ps(gi, gi)));
    } else {
      mi = _mm512_mul_ps(vb1, _mm512_loadu_ps(m + i));
      vi = _mm512_mul_ps(vb2, _mm512_loadu_ps(v + i));
    }
    const __m512 den = _mm512_fmadd_ps(_mm512_sqrt_ps(vi), vibc2, veps);
    const __m512 pi = _mm512_sub_ps(_mm512_mul_ps(_mm512_loadu_ps(p + i), vdec),
                                    _mm512_div_ps(_mm512_mul_ps(vstep, mi), den));
    _mm512_storeu_ps(m + i, mi);
    _mm512_storeu_ps(v + i, vi);
    _mm512_storeu_ps(p + i, pi);
    if (nt)
      _mm256_stream_si256(reinterpret_cast<__m256i*>(pb + i), bf16x16_rne(pi));
    else if (pb)
      _mm256_storeu_si256(reinterpret_cast<__m256i*>(pb + i), bf16x16_rne(pi));
  }
  if (nt) _mm_sfence();
  if (i < n)
    adamw_scalar<G>(p + i, HAS_G ? g + i : nullptr, m + i, v + i, pb ? pb + i : nullptr, n - i, decay, b1, b2, step,
                    inv_sqrt_bc2, eps);
}

__attribute__((target("avx512f,avx512bw"))) void round_avx512(const float* x, uint16_t* out, size_t n) {
  size_t i = 0;
  for (; i + 16 <= n; i += 16)
    _mm256_storeu_si256(reinterpret_cast<__m256i*>(out + i), bf16x16_rne(_mm512_loadu_ps(x + i)));
  for (; i < n; ++i) out[i] = bf16_rne(x[i]);
}

bool detect_avx512() {
  __builtin_cpu_init();
  return __builtin_cpu_supports("avx512f") && __builtin_cpu_supports("avx512bw");
}

}  // namespace

bool adamw_uses_avx512() {
  static const bool yes = detect_avx512();
  return yes;
}

void adamw_chunk(float* p, const float* g, float* m, float* v, uint16_t* pb, size_t n, const AdamHyper& h, int t) {
  const double bc1 = 1.0 - pow((double)h.beta1, t);
  const double bc2 = 1.0 - pow((double)h.beta2, t);
  const float decay = 1.f - h.lr * h.wd;
  const float step = (float)(h.lr / bc1);
  const float inv_sqrt_bc2 = (float)(1.0 / sqrt(bc2));
  if (adamw_uses_avx512() && g)
    adamw_avx512<true>(p, g, m, v, pb, n, decay, h.beta1, h.beta2, step, inv_sqrt_bc2, h.eps);
  else if (adamw_uses_avx512())
    adamw_avx512<false>(p, (const float*)nullptr, m, v, pb, n, decay, h.beta1, h.beta2, step, inv_sqrt_bc2, h.eps);
  else
    adamw_scalar<float>(p, g, m, v, pb, n, decay, h.beta1, h.beta2, step, inv_sqrt_bc2, h.eps);
}

void adamw_chunk_bf16g(float* p, const uint16_t* g, float* m, float* v, uint16_t* pb, size_t n, const AdamHyper& h,
                       int t) {
  if (!g) return adamw_chunk(p, nullptr, m, v, pb, n, h, t);
  const double bc1 = 1.0 - pow((double)h.beta1, t);
  const double bc2 = 1.0 - pow((double)h.beta2, t);
  const float decay = 1.f - h.lr * h.wd;
  const float step = (float)(h.lr / bc1);
  const float inv_sqrt_bc2 = (float)(1.0 / sqrt(bc2));
  if (adamw_uses_avx512())
    adamw_avx512<true, uint16_t>(p, g, m, v, pb, n, decay, h.beta1, h.beta2, step, inv_sqrt_bc2, h.eps);
  else
    adamw_scalar<uint16_t>(p, g, m, v, pb, n, decay, h.beta1, h.beta2, step, inv_sqrt_bc2, h.eps);
}

void bf16_round_chunk(const float* x, uint16_t* out, size_t n) {
  if (adamw_uses_avx512()) {
    round_avx512(x, out, n);
  } else {
    for (size_t i = 0; i < n; ++i) out[i] = bf16_rne(x[i]);
  }
}

// ---------------------------------------------------------------------------
ThreadPool::ThreadPool(int workers) {
  for (int i = 0; i < workers; ++i) workers_.emplace_back([this] { loop(); });
}

ThreadPool::~ThreadPool() {
  {
    std::lock_guard<std::mutex> lk(mu_);
    stop_ = true;
  }
  cv_.notify_all();
  for (auto& w : workers_) w.join();
}

void ThreadPool::loop() {
  uint64_t seen = 0;
  while (true) {
    const std::function<void(int)>* fn;
    int n;
    {
      std::unique_lock<std::mutex> lk(mu_);
      cv_.wait(lk, [&] { return stop_ || gen_ != seen; });
      if (stop_) return;
      seen = gen_;
      fn = fn_;
      n = n_;
      ++active_;
    }
    int done = 0;
    if (fn)
      for (int i = next_.fetch_add(1); i < n; i = next_.fetch_add(1)) {
        (*fn)(i);
        ++done;
      }
    {
      std::lock_guard<std::mutex> lk(mu_);
      finished_ += done;
      --active_;
    }
    done_cv_.notify_all();
  }
}

void ThreadPool::run(int n, const std::function<void(int)>& fn) {
  if (n <= 0) return;
  {
    std::lock_guard<std::mutex> lk(mu_);
    fn_ = &fn;
    n_ = n;
    finished_ = 0;
    next_.store(0);
    ++gen_;
  }
  cv_.notify_all();
  int done = 0;
  for (int i = next_.fetch_add(1); i < n; i = next_.fetch_add(1)) {
    fn(i);
    ++done;
  }
  std::unique_lock<std::mutex> lk(mu_);
  finished_ += done;
  // Every task has run and no worker still holds this call's function.
  done_cv_.wait(lk, [&] { return finished_ >= n && active_ == 0; });
  fn_ = nullptr;
  n_ = 0;
}

void parallel_ranges(ThreadPool& pool, size_t n, const std::function<void(size_t, size_t)>& body) {
  if (n == 0) return;
  const size_t min_chunk = 1 << 16;
  size_t tasks = (size_t)pool.size() * 4;
  size_t chunk = (n + tasks - 1) / tasks;
  if (chunk < min_chunk) chunk = min_chunk;
  chunk = (chunk + 63) & ~size_t(63);
  const int nt = (int)((n + chunk - 1) / chunk);
  pool.run(nt, [&](int i) {
    const size_t b = (size_t)i * chunk;
    const size_t e = b + chunk < n ? b + chunk : n;
    body(b, e);
  });
}

}  // namespace mt

extern "C" int mt_k_adamw_host(float* p, const float* g, float* m, float* v, uint16_t* pb, size_t n, float lr,
                               float beta1, float beta2, float eps, float wd, int t) {
  if ((!p || !m || !v) && n) return MT_ERR_ARG;
  if (t < 1 || !(eps > 0) || !(beta1 >= 0 && beta1 < 1) || !(beta2 >= 0 && beta2 < 1)) return MT_ERR_ARG;
  mt::adamw_chunk(p, g, m, v, pb, n, mt::AdamHyper{lr, beta1, beta2, eps, wd}, t);
  return MT_OK;
}

namespace {
// STREAM triad a[i] = b[i] + s c[i] over fp32 arrays, non-temporal stores (no
// read-for-ownership of a): 12 bytes of DRAM traffic per element.
__attribute__((target("avx512f"))) void triad_avx512(float* a, const float* b, const float* c, size_t n, float s) {
  const __m512 vs = _mm512_set1_ps(s);
  size_t i = 0;
  for (; i + 16 <= n; i += 16)
    _mm512_stream_ps(a + i, _mm512_fmadd_ps(vs, _mm512_loadu_ps(c + i), _mm512_loadu_ps(b + i)));
  _mm_sfence();
  for (; i < n; ++i) a[i] = b[i] + s * c[i];
}
}  // namespace

namespace {
// Probe buffers allocated as the engine allocates its host state: anonymous
// mappings advised onto transparent huge pages before their first touch.
struct ProbeBuf {
  void* p = nullptr;
  size_t len = 0;
  explicit ProbeBuf(size_t bytes) {
    len = (bytes + (size_t(2) << 20) - 1) & ~((size_t(2) << 20) - 1);
    void* got = mmap(nullptr, len, PROT_READ | PROT_WRITE, MAP_PRIVATE | MAP_ANONYMOUS, -1, 0);
    if (got == MAP_FAILED) return;
    madvise(got, len, MADV_HUGEPAGE);
    p = got;
  }
  ~ProbeBuf() {
    if (p) munmap(p, len);
  }
  ProbeBuf(const ProbeBuf&) = delete;
  ProbeBuf& operator=(const ProbeBuf&) = delete;
};
}  // namespace

extern "C" double mt_host_triad_gbs(size_t n, int threads) {
  if (n < (1u << 16)) return MT_ERR_ARG;
  if (threads <= 0) threads = std::max(1, (int)std::thread::hardware_concurrency() - 1);
  ProbeBuf b0(n * 4), b1(n * 4), b2(n * 4);
  float* a[3] = {static_cast<float*>(b0.p), static_cast<float*>(b1.p), static_cast<float*>(b2.p)};
  double best = 0;
  if (a[0] && a[1] && a[2]) {
    mt::ThreadPool pool(threads - 1);
    const size_t chunk = 1 << 16;  // multiple of 16 floats: every chunk starts 64-byte aligned
    const int tasks = (int)((n + chunk - 1) / chunk);
    pool.run(tasks, [&](int i) {  // parallel first touch
      const size_t b = (size_t)i * chunk, m = std::min(chunk, n - b);
      for (int k = 0; k < 3; ++k)
        for (size_t j = 0; j < m; ++j) a[k][b + j] = 1.0f;
    });
    const bool avx = mt::adamw_uses_avx512();
    for (int rep = 0; rep < 5; ++rep) {
      const auto t0 = std::chrono::steady_clock::now();
      pool.run(tasks, [&](int i) {
        const size_t b = (size_t)i * chunk, m = std::min(chunk, n - b);
        if (avx) {
          triad_avx512(a[0] + b, a[1] + b, a[2] + b, m, 0.5f);
        } else {
          for (size_t j = 0; j < m; ++j) a[0][b + j] = a[1][b + j] + 0.5f * a[2][b + j];
        }
      });
      const double sec = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
      best = std::max(best, 12.0 * n / sec / 1e9);
    }
  }
  return best > 0 ? best : MT_ERR_NOMEM;
}

extern "C" double mt_host_optimizer_gbs(size_t n, int threads) {
  if (n < (1u << 16)) return MT_ERR_ARG;
  if (threads <= 0) threads = std::max(1, (int)std::thread::hardware_concurrency() - 1);
  ProbeBuf b0(n * 4), b1(n * 4), b2(n * 4), b3(n * 4), b4(n * 2);
  float* a[4] = {static_cast<float*>(b0.p), static_cast<float*>(b1.p), static_cast<float*>(b2.p),
                 static_cast<float*>(b3.p)};
  uint16_t* pb = static_cast<uint16_t*>(b4.p);
  double best = 0;
  if (a[0] && a[1] && a[2] && a[3] && pb) {
    mt::ThreadPool pool(threads - 1);
    const size_t chunk = 1 << 16;
    const int tasks = (int)((n + chunk - 1) / chunk);
    pool.run(tasks, [&](int i) {  // parallel first touch
      const size_t b = (size_t)i * chunk, m = std::min(chunk, n - b);
      for (int k = 0; k < 4; ++k)
        for (size_t j = 0; j < m; ++j) a[k][b + j] = 1e-3f;
      memset(pb + b, 0, m * 2);
    });
    const mt::AdamHyper h{1e-3f, 0.9f, 0.95f, 1e-8f, 0.1f};
    for (int rep = 0; rep < 3; ++rep) {
      const auto t0 = std::chrono::steady_clock::now();
      pool.run(tasks, [&](int i) {
        const size_t b = (size_t)i * chunk, m = std::min(chunk, n - b);
        mt::adamw_chunk(a[0] + b, a[1] + b, a[2] + b, a[3] + b, pb + b, m, h, 1);
      });
      const double sec = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
      best = std::max(best, 30.0 * n / sec / 1e9);
    }
  }
  return best > 0 ? best : MT_ERR_NOMEM;
}
