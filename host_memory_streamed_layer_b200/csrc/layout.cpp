// Configuration checks and the arena / layer-block layouts (see layout.h).
#include "layout.h"

#include <stdlib.h>
#include <string.h>

#include <algorithm>

namespace mt {

namespace {
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
}  // namespace

int validate_config(const mt_config* c, std::string* why) {
  auto fail = [&](int code, const char* m) {
    if (why) *why = m;
    return code;
  };
  if (!c) return fail(MT_ERR_ARG, "config is NULL");
  if (c->struct_size != sizeof(mt_config)) return fail(MT_ERR_ARG, "mt_config.struct_size != sizeof(mt_config)");
  if (c->L < 1 || c->d < 1 || c->H < 1 || c->Hkv < 1 || c->F < 1 || c->V < 1 || c->b < 1 || c->s < 1)
    return fail(MT_ERR_CONFIG, "every shape must be positive");
  if (c->d % 64) return fail(MT_ERR_CONFIG, "d must be a multiple of 64");
  if (c->d > 8192) return fail(MT_ERR_CONFIG, "d must be at most 8192");
  if (c->d % c->H) return fail(MT_ERR_CONFIG, "d must be a multiple of H");
  const int hd = c->d / c->H;
  if (hd != 64 && hd != 128) return fail(MT_ERR_CONFIG, "head_dim d/H must be 64 or 128");
  if (c->H % c->Hkv) return fail(MT_ERR_CONFIG, "H must be a multiple of Hkv");
  if (c->F % 8) return fail(MT_ERR_CONFIG, "F must be a multiple of 8");
  if (c->V % 8) return fail(MT_ERR_CONFIG, "V must be a multiple of 8");
  if ((int64_t)c->b * c->s > (int64_t)1 << 30) return fail(MT_ERR_CONFIG, "b*s too large");
  if (!(c->norm_eps > 0) || !(c->rope_base > 1) || !(c->lr >= 0) || !(c->beta1 >= 0 && c->beta1 < 1) ||
      !(c->beta2 >= 0 && c->beta2 < 1) || !(c->adam_eps > 0) || !(c->wd >= 0))
    return fail(MT_ERR_CONFIG, "hyper-parameter out of range");
  if (c->host_threads < 0) return fail(MT_ERR_CONFIG, "host_threads must be >= 0");
  if (c->E < 0 || c->E > 64) return fail(MT_ERR_CONFIG, "E (experts) must be in [0, 64]");
  if (c->E > 0 && (c->topk < 1 || c->topk > c->E)) return fail(MT_ERR_CONFIG, "topk must be in [1, E]");
  if ((c->flags & MT_FLAG_TIED_EMBED) && (c->flags & MT_FLAG_BF16_GRADS))
    return fail(MT_ERR_CONFIG, "tied embeddings take their gradients in fp32 (no MT_FLAG_BF16_GRADS)");
  return MT_OK;
}

Layout make_layout(const mt_config& c) {
  Layout y;
  Shapes& s = y.sh;
  s.L = c.L;
  s.d = c.d;
  s.H = c.H;
  s.Hkv = c.Hkv;
  s.F = c.F;
  s.V = c.V;
  s.b = c.b;
  s.s = c.s;
  s.hd = c.d / c.H;
  s.T = c.b * c.s;
  s.Nqkv = (c.H + 2 * c.Hkv) * s.hd;
  s.Hd = c.H * s.hd;
  s.E = c.E;
  s.topk = c.E > 0 ? c.topk : 0;
  const size_t Ee = c.E > 0 ? (size_t)c.E : 1;  // expert blocks of the MLP tensors
  size_t off = 0;
  auto put = [&](size_t n) {
    TRef r{off, n};
    off += round_up(n, 64);
    return r;
  };
  const size_t d = c.d, F = c.F, V = c.V;
  y.embed = put(V * d);
  y.layer.resize((size_t)c.L * kLayerTensors);
  for (int l = 0; l < c.L; ++l) {
    TRef* t = &y.layer[(size_t)l * kLayerTensors];
    t[MT_T_ATTN_NORM] = put(d);
    t[MT_T_WQ] = put((size_t)s.Hd * d);
    t[MT_T_WK] = put((size_t)c.Hkv * s.hd * d);
    t[MT_T_WV] = put((size_t)c.Hkv * s.hd * d);
    t[MT_T_WO] = put(d * (size_t)s.Hd);
    t[MT_T_MLP_NORM] = put(d);
    t[MT_T_WGATE] = put(Ee * F * d);
    t[MT_T_WUP] = put(Ee * F * d);
    t[MT_T_WDOWN] = put(Ee * d * F);
    t[MT_T_ROUTER] = put(c.E > 0 ? (size_t)c.E * d : 0);
  }
  y.final_norm = put(d);
  y.tied = (c.flags & MT_FLAG_TIED_EMBED) != 0;
  if (y.tied)
    y.head = TRef{off, 0};
  else
    y.head = put(V * d);
  y.total = off;
  y.gf_pad = round_up(d, 64);
  y.head_block = y.gf_pad + V * d;
  // bf16 block (128 elements = 256 bytes alignment)
  size_t b = 0;
  auto bput = [&](size_t n) {
    size_t r = b;
    b += round_up(n, 128);
    return r;
  };
  y.bf_g1 = bput(d);
  y.bf_qkv = bput((size_t)s.Nqkv * d);
  y.bf_o = bput(d * (size_t)s.Hd);
  y.bf_g2 = bput(d);
  y.bf_gu = bput(2 * Ee * F * d);
  y.bf_d = bput(Ee * d * F);
  y.bf_r = bput(c.E > 0 ? (size_t)c.E * d : 0);
  y.bf_layer = b;
  return y;
}

size_t Layout::bf_of(int tid) const {
  const size_t d = sh.d;
  switch (tid) {
    case MT_T_ATTN_NORM: return bf_g1;
    case MT_T_WQ: return bf_qkv;
    case MT_T_WK: return bf_qkv + (size_t)sh.Hd * d;
    case MT_T_WV: return bf_qkv + (size_t)(sh.Hd + sh.Hkv * sh.hd) * d;
    case MT_T_WO: return bf_o;
    case MT_T_MLP_NORM: return bf_g2;
    case MT_T_WGATE: return bf_gu;
    case MT_T_WUP: return bf_gu + (size_t)(sh.E > 0 ? sh.E : 1) * sh.F * d;
    case MT_T_WDOWN: return bf_d;
    case MT_T_ROUTER: return bf_r;
  }
  return 0;
}

}  // namespace mt

extern "C" int mt_config_default(mt_config* cfg) {
  if (!cfg) return MT_ERR_ARG;
  memset(cfg, 0, sizeof(*cfg));
  cfg->struct_size = sizeof(mt_config);
  cfg->norm_eps = 1e-5f;
  cfg->rope_base = 10000.f;
  cfg->lr = 1e-3f;
  cfg->beta1 = 0.9f;
  cfg->beta2 = 0.95f;
  cfg->adam_eps = 1e-8f;
  cfg->wd = 0.1f;
  return MT_OK;
}

extern "C" size_t mt_arena_bytes(const mt_config* cfg) {
  if (mt::validate_config(cfg, nullptr) != MT_OK) return 0;
  return mt::make_layout(*cfg).total * sizeof(float);
}

extern "C" int mt_tensor_offset(const mt_config* cfg, int layer, int tid, size_t* offset_floats, size_t* numel) {
  if (mt::validate_config(cfg, nullptr) != MT_OK) return MT_ERR_CONFIG;
  mt::Layout y = mt::make_layout(*cfg);
  mt::TRef r;
  if (layer == -1) {
    if (tid == MT_T_EMBED)
      r = y.embed;
    else if (tid == MT_T_FINAL_NORM)
      r = y.final_norm;
    else if (tid == MT_T_LM_HEAD && !y.tied)
      r = y.head;
    else
      return MT_ERR_ARG;
  } else {
    if (layer < 0 || layer >= cfg->L || tid < 0 || tid >= mt::kLayerTensors) return MT_ERR_ARG;
    if (tid == MT_T_ROUTER && cfg->E == 0) return MT_ERR_ARG;  // dense MLP: no router
    r = y.t(layer, tid);
  }
  if (offset_floats) *offset_floats = r.off;
  if (numel) *numel = r.n;
  return MT_OK;
}

int mt::defer_layer_count(const mt_config& cfg) {
  if (!(cfg.flags & MT_FLAG_DEFER_UPDATES) || (cfg.flags & MT_FLAG_NO_UPDATE)) return 0;
  long n = 1;
  if (const char* e = getenv("MT_DEFER_LAYERS")) n = strtol(e, nullptr, 10);
  return (int)std::min<long>(std::max<long>(n, 0), std::max(cfg.L - 1, 0));
}

extern "C" size_t mt_host_state_bytes(const mt_config* cfg) {
  if (mt::validate_config(cfg, nullptr) != MT_OK) return 0;
  mt::Layout y = mt::make_layout(*cfg);
  const size_t P = y.total;
  const size_t bf = (size_t)y.sh.L * y.bf_layer + (y.tied ? 1 : 2) * (size_t)y.sh.V * y.sh.d + y.sh.d + 256;
  const size_t common = P * 4 * 2 + bf * 2 + (size_t)y.sh.T * y.sh.d * 4;  // m, v; bf16 copy; embedding staging
  const size_t gsz = (cfg->flags & MT_FLAG_BF16_GRADS) ? 2 : 4;           // bytes per host gradient element
  const size_t acts = ((cfg->flags & MT_FLAG_OFFLOAD_ACTS) && y.sh.L >= 3)  // x_0 .. x_{L-3}, fp32
                          ? (size_t)(y.sh.L - 2) * y.sh.T * y.sh.d * 4
                          : 0;
  const size_t head_own = y.tied ? y.head_block * 4 : 0;                  // tied: the head's gradient block
  if (!(cfg->flags & MT_FLAG_GRAD_RING)) return acts + common + P * gsz + head_own;  // whole gradient arena
  const size_t layer_f = y.layer_end(0) - y.layer_begin(0);
  return acts + common + ((size_t)(MT_GRAD_RING_SLOTS + mt::defer_layer_count(*cfg)) * layer_f + y.head_block) * gsz;
}

extern "C" int mt_shard_plan(const mt_config* cfg, int world, int rank, mt_shard* out) {
  if (!out || world < 1 || world > 1024 || rank < 0 || rank >= world) return MT_ERR_ARG;
  if (mt::validate_config(cfg, nullptr) != MT_OK) return MT_ERR_CONFIG;
  if (cfg->d % 128) return MT_ERR_CONFIG;  // fp32 and bf16 block offsets coincide only then
  const mt::Layout y = mt::make_layout(*cfg);
  const size_t lb = y.layer_begin(0), le = y.layer_end(0);
  // The fp32 arena block of a layer and its bf16 streamed block must hold
  // every tensor at the same element offset, so that one element range is one
  // rank's share of the weights, of the gradients and of the update alike.
  if (le - lb != y.bf_layer) return MT_ERR_CONFIG;
  for (int tid = 0; tid < mt::kLayerTensors; ++tid)
    if (y.t(0, tid).off - lb != y.bf_of(tid)) return MT_ERR_CONFIG;
  const size_t head_elems = y.head.off + y.head.n - y.final_norm.off;
  if (y.head.off - y.final_norm.off != (size_t)((cfg->d + 127) / 128 * 128)) return MT_ERR_CONFIG;
  auto chunk = [&](size_t n) { return (n + (size_t)world * 128 - 1) / ((size_t)world * 128) * 128; };
  auto part = [&](size_t n, size_t c, uint64_t* b, uint64_t* e) {
    *b = std::min(n, (size_t)rank * c);
    *e = std::min(n, (size_t)(rank + 1) * c);
  };
  memset(out, 0, sizeof(*out));
  out->world = world;
  out->rank = rank;
  out->layer_elems = le - lb;
  out->layer_chunk = chunk(le - lb);
  part(le - lb, out->layer_chunk, &out->layer_begin, &out->layer_end);
  out->head_elems = head_elems;
  out->head_chunk = chunk(head_elems);
  part(head_elems, out->head_chunk, &out->head_begin, &out->head_end);
  const int rows = (cfg->V + world - 1) / world;
  out->embed_row_begin = std::min(cfg->V, rank * rows);
  out->embed_row_end = std::min(cfg->V, (rank + 1) * rows);
  return MT_OK;
}
