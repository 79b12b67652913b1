// C-ABI entry points of the individual kernels (declared in mt_kernels.h).
#include "mt_internal.h"
#include "mt_kernels.h"

extern "C" int mt_k_gemm_bf16(const void* A, int64_t lda, int a_mn_major, const void* B, int64_t ldb,
                              int b_mn_major, void* C, int64_t ldc, int out_kind, const float* R, int64_t ldr,
                              int M, int N, int K, void* stream, int32_t* dev_err) {
  if (out_kind < MT_GEMM_OUT_BF16 || out_kind > MT_GEMM_OUT_F32_ADD) return MT_ERR_ARG;
  if (M < 0 || N < 0 || K < 0) return MT_ERR_ARG;
  mt::GemmDesc g{A, lda, a_mn_major != 0, B, ldb, b_mn_major != 0, C, ldc, out_kind, R, ldr, M, N, K, mt::RopeDesc{}};
  return mt::gemm_bf16(g, static_cast<cudaStream_t>(stream), dev_err);
}

extern "C" int64_t mt_k_gemm_wait_limit_ns(int64_t ns) {
  if (ns < 0) {
    const uint64_t cur = mt::gemm_wait_limit_ns(0);
    mt::gemm_wait_limit_ns(cur);
    return (int64_t)cur;
  }
  return (int64_t)mt::gemm_wait_limit_ns((uint64_t)ns);
}

extern "C" int mt_k_gemm_variant(int variant) {
  if (variant < 0 || variant > 2) return MT_ERR_ARG;
  return mt::gemm_variant(variant);
}

extern "C" int mt_k_attn_fwd_variant(int variant) {
  if (variant < 0 || variant > 2) return MT_ERR_ARG;
  return mt::attention_fwd_variant(variant);
}

extern "C" int mt_k_attn_bwd_variant(int variant) {
  if (variant < 0 || variant > 2) return MT_ERR_ARG;
  return mt::attention_bwd_variant(variant);
}

#include <cmath>

namespace {
inline cudaStream_t S(void* p) { return static_cast<cudaStream_t>(p); }
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
}  // namespace

extern "C" int mt_k_rmsnorm_fwd(const float* x, const void* g, void* y, float* rstd, int T, int d, float eps,
                                void* stream) {
  if (!x || !g || !y || T < 0 || d <= 0 || (d % 4)) return MT_ERR_ARG;
  return mt::launch_rmsnorm_fwd(x, g, y, rstd, T, d, eps, S(stream));
}

extern "C" size_t mt_k_rmsnorm_bwd_partial_floats(int T, int d) {
  return (size_t)mt::rmsnorm_bwd_blocks(T) * (size_t)d;
}

extern "C" int mt_k_rmsnorm_bwd(const float* x, const void* g, const float* rstd, const float* dy, const float* dres,
                                float* dx, void* dx_bf16, float* dg_part, float* dg, int T, int d, void* stream) {
  if (!x || !g || !rstd || !dy || !dx || !dg_part || !dg || T < 0 || d <= 0 || (d % 4) || d > 8192)
    return MT_ERR_ARG;
  return mt::launch_rmsnorm_bwd(x, g, rstd, dy, dres, dx, dx_bf16, dg_part, dg, T, d, S(stream));
}

extern "C" int mt_k_rope(void* buf, int64_t ld, int T, int s, int nheads, int hd, int col0, const float* cos_tab,
                         const float* sin_tab, float sign, void* stream) {
  if (!buf || !cos_tab || !sin_tab || T < 0 || s <= 0 || nheads < 0 || hd <= 0 || (hd % 4) || (col0 % 2) ||
      (ld % 2))
    return MT_ERR_ARG;
  return mt::launch_rope(buf, ld, T, s, nheads, hd, col0, cos_tab, sin_tab, sign, S(stream));
}

extern "C" int mt_k_swiglu_fwd(const void* gu, void* act, int T, int F, void* stream) {
  if (!gu || !act || T < 0 || F <= 0 || (F % 8) || !al16(gu) || !al16(act)) return MT_ERR_ARG;
  return mt::launch_swiglu_fwd(gu, act, T, F, S(stream));
}

extern "C" int mt_k_swiglu_bwd(const void* gu, const void* dact, void* dgu, int T, int F, void* stream) {
  if (!gu || !dact || !dgu || T < 0 || F <= 0 || (F % 8) || !al16(gu) || !al16(dact) || !al16(dgu))
    return MT_ERR_ARG;
  return mt::launch_swiglu_bwd(gu, dact, dgu, T, F, S(stream));
}

extern "C" int mt_k_embed_fwd(const int32_t* tok, const void* E, float* x, int T, int d, void* stream) {
  if (!tok || !E || !x || T < 0 || d <= 0 || (d % 8) || !al16(E) || !al16(x)) return MT_ERR_ARG;
  return mt::launch_embed_fwd(tok, E, x, T, d, S(stream));
}

extern "C" int mt_k_embed_bwd(const int32_t* offs, const int32_t* pos, int n_unique, const float* dx, float* rows,
                              int d, void* stream) {
  if (!offs || !pos || !dx || !rows || n_unique < 0 || d <= 0 || (d % 4)) return MT_ERR_ARG;
  return mt::launch_embed_bwd(offs, pos, n_unique, dx, rows, d, S(stream));
}

extern "C" int mt_k_softmax_ce(const float* z, int64_t ldz, const int32_t* labels, void* dz, int64_t lddz,
                               float* row_loss, int Tc, int V, float scale, void* stream) {
  if (!z || !labels || !dz || !row_loss || Tc < 0 || V <= 0 || (V % 4) || (ldz % 4) || (lddz % 4))
    return MT_ERR_ARG;
  return mt::launch_softmax_ce(z, ldz, labels, dz, lddz, row_loss, Tc, V, scale, S(stream));
}

extern "C" int mt_k_attn_fwd(const void* q, const void* k, const void* v, int64_t ldqkv, void* o, int64_t ldo,
                             float* lse, int b, int s, int H, int Hkv, int hd, void* stream) {
  if (!q || !k || !v || !o || !lse || b < 0 || s < 0 || H <= 0 || Hkv <= 0 || (H % Hkv)) return MT_ERR_ARG;
  if (hd != 64 && hd != 128) return MT_ERR_CONFIG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || (ldqkv % 8) || (ldo % 8)) return MT_ERR_ARG;
  mt::AttnArgs a{};
  a.q = q; a.k = k; a.v = v; a.ldqkv = ldqkv; a.o = o; a.ldo = ldo; a.lse = lse;
  a.b = b; a.s = s; a.H = H; a.Hkv = Hkv; a.hd = hd; a.scale = 1.0f / std::sqrt((float)hd);
  return mt::attention_fwd(a, S(stream));
}

extern "C" int mt_k_attn_bwd(const void* q, const void* k, const void* v, int64_t ldqkv, const void* o,
                             const void* dout, int64_t ldo, const float* lse, float* dvec, float* dq_acc,
                             int64_t ldqa, void* dq, int64_t lddq, void* dk, void* dv, int64_t lddkv, int b, int s,
                             int H, int Hkv, int hd, const float* cos_tab, const float* sin_tab, void* stream) {
  if ((cos_tab == nullptr) != (sin_tab == nullptr)) return MT_ERR_ARG;
  if (!q || !k || !v || !o || !dout || !lse || !dvec || !dq_acc || !dq || !dk || !dv) return MT_ERR_ARG;
  if (b < 0 || s < 0 || H <= 0 || Hkv <= 0 || (H % Hkv)) return MT_ERR_ARG;
  if (hd != 64 && hd != 128) return MT_ERR_CONFIG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || !al16(dout) || !al16(dq_acc) || (ldqkv % 8) || (ldo % 8) ||
      (ldqa % 4) || (lddq % 4) || (lddkv % 2) || ldqa < (int64_t)H * hd)
    return MT_ERR_ARG;
  mt::AttnArgs a{};
  a.q = q; a.k = k; a.v = v; a.ldqkv = ldqkv; a.o = const_cast<void*>(o); a.ldo = ldo; a.lse = const_cast<float*>(lse);
  a.dout = dout; a.dvec = dvec; a.dq_acc = dq_acc; a.ldqa = ldqa; a.dq = dq; a.lddq = lddq; a.dk = dk; a.dv = dv;
  a.lddkv = lddkv; a.b = b; a.s = s; a.H = H; a.Hkv = Hkv; a.hd = hd; a.scale = 1.0f / std::sqrt((float)hd);
  a.rope_cos = cos_tab; a.rope_sin = sin_tab;
  return mt::attention_bwd(a, S(stream));
}

extern "C" int mt_k_attn_fwd_tc(const void* q, const void* k, const void* v, int64_t ldqkv, void* o, int64_t ldo,
                                float* lse, int b, int s, int H, int Hkv, int hd, void* stream, int32_t* dev_err) {
  if (!q || !k || !v || !o || !lse || b < 0 || s < 0 || H <= 0 || Hkv <= 0 || (H % Hkv)) return MT_ERR_ARG;
  if (hd != 64 && hd != 128) return MT_ERR_CONFIG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || (ldqkv % 8) || (ldo % 8)) return MT_ERR_ARG;
  mt::AttnArgs a{};
  a.q = q; a.k = k; a.v = v; a.ldqkv = ldqkv; a.o = o; a.ldo = ldo; a.lse = lse;
  a.b = b; a.s = s; a.H = H; a.Hkv = Hkv; a.hd = hd; a.scale = 1.0f / std::sqrt((float)hd);
  return mt::attention_fwd_tc(a, S(stream), dev_err);
}

extern "C" int mt_k_gemm_bf16_rope(const void* A, int64_t lda, const void* B, int64_t ldb, void* C, int64_t ldc, int M,
                                   int N, int K, int rope_cols, int hd, int s, const float* cos_tab,
                                   const float* sin_tab, void* stream, int32_t* dev_err) {
  if (M < 0 || N < 0 || K < 0 || !cos_tab || !sin_tab) return MT_ERR_ARG;
  mt::GemmDesc g{A, lda, false, B, ldb, false, C, ldc, mt::EPI_BF16_ROPE, nullptr, 0, M, N, K,
                 mt::RopeDesc{cos_tab, sin_tab, rope_cols, hd, s}};
  return mt::gemm_bf16(g, static_cast<cudaStream_t>(stream), dev_err);
}

extern "C" int mt_k_attn_bwd_tc(const void* q, const void* k, const void* v, int64_t ldqkv, const void* o,
                                const void* dout, int64_t ldo, const float* lse, float* dvec, float* dq_acc,
                                int64_t ldqa, void* dq, int64_t lddq, void* dk, void* dv, int64_t lddkv, int b, int s,
                                int H, int Hkv, int hd, const float* cos_tab, const float* sin_tab, void* stream,
                                int32_t* dev_err) {
  if ((cos_tab == nullptr) != (sin_tab == nullptr)) return MT_ERR_ARG;
  if (!q || !k || !v || !o || !dout || !lse || !dvec || !dq_acc || !dq || !dk || !dv) return MT_ERR_ARG;
  if (b < 0 || s < 0 || H <= 0 || Hkv <= 0 || (H % Hkv)) return MT_ERR_ARG;
  if (hd != 128 && hd != 64) return MT_ERR_CONFIG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || !al16(dout) || !al16(dq_acc) || (ldqkv % 8) || (ldo % 8) ||
      (ldqa % 4) || (lddq % 4) || (lddkv % 8) || ldqa < (int64_t)H * hd)
    return MT_ERR_ARG;
  mt::AttnArgs a{};
  a.q = q; a.k = k; a.v = v; a.ldqkv = ldqkv; a.o = const_cast<void*>(o); a.ldo = ldo; a.lse = const_cast<float*>(lse);
  a.dout = dout; a.dvec = dvec; a.dq_acc = dq_acc; a.ldqa = ldqa; a.dq = dq; a.lddq = lddq; a.dk = dk; a.dv = dv;
  a.lddkv = lddkv; a.b = b; a.s = s; a.H = H; a.Hkv = Hkv; a.hd = hd; a.scale = 1.0f / std::sqrt((float)hd);
  a.rope_cos = cos_tab; a.rope_sin = sin_tab;
  return mt::attention_bwd_tc(a, S(stream), dev_err);
}
