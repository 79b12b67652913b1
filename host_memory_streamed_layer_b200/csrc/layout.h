// Host and device layouts of the streamed model.
//
// fp32 master arena (caller-visible, also the layout of the gradient arena):
//   embedding [V,d]; per layer: attention-norm gain [d], Wq [H hd, d],
//   Wk [Hkv hd, d], Wv [Hkv hd, d], Wo [d, H hd], MLP-norm gain [d],
//   Wgate [F,d], Wup [F,d], Wdown [d,F] (with E experts: [E,F,d], [E,F,d],
//   [E,d,F], then the router [E,d]); final-norm gain [d]; LM head [V,d].
//   Row-major [out, in], every tensor on a 256-byte boundary. With d a
//   multiple of 64 no padding is needed, so Wq|Wk|Wv and Wgate|Wup are
//   adjacent and one layer is one contiguous range.
// bf16 layer block (host mirror and device weight slot), per layer:
//   g1 [d] | Wqkv [(H+2Hkv) hd, d] | Wo [d, H hd] | g2 [d] | Wgu [2F, d] | Wd [d, F]
//   each part on a 256-byte boundary; with E experts Wgu holds every
//   expert's gate rows [E F, d] then every expert's up rows, Wd [E d, F], and
//   the router [E, d] follows.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "mt.h"

namespace mt {

constexpr int kLayerTensors = 10;  // MT_T_ATTN_NORM .. MT_T_WDOWN, MT_T_ROUTER (empty without experts)

struct TRef {
  size_t off = 0;  // elements
  size_t n = 0;    // elements
};

struct Shapes {
  int L, d, H, Hkv, F, V, b, s, hd, T, Nqkv, Hd;  // Hd = H * hd
  int E = 0, topk = 0;                            // experts (0: dense MLP), experts per token
};

struct Layout {
  Shapes sh{};
  // fp32 arena, in floats (head.n == 0 with tied embeddings: the table is the head)
  TRef embed, final_norm, head;
  bool tied = false;
  // [final-norm gain | LM head] gradient block (device and host buffers, also
  // when tied): the gain padded to gf_pad floats, then V*d
  size_t gf_pad = 0, head_block = 0;
  std::vector<TRef> layer;  // L * kLayerTensors
  size_t total = 0;
  size_t layer_begin(int l) const { return layer[(size_t)l * kLayerTensors].off; }
  size_t layer_end(int l) const {
    const TRef& t = layer[(size_t)l * kLayerTensors + kLayerTensors - 1];
    return t.off + t.n;
  }
  const TRef& t(int l, int tid) const { return layer[(size_t)l * kLayerTensors + tid]; }
  // bf16 layer block, in elements
  size_t bf_g1 = 0, bf_qkv = 0, bf_o = 0, bf_g2 = 0, bf_gu = 0, bf_d = 0, bf_r = 0, bf_layer = 0;
  // bf16 offset of arena tensor tid inside the layer block
  size_t bf_of(int tid) const;
};

// Validates cfg (MT_OK or MT_ERR_CONFIG / MT_ERR_ARG with a message).
int validate_config(const mt_config* cfg, std::string* why);
Layout make_layout(const mt_config& cfg);

// Layers whose update MT_FLAG_DEFER_UPDATES defers to the next step: 0 without
// the flag or with MT_FLAG_NO_UPDATE, else MT_DEFER_LAYERS (default 1) clamped
// to [0, L-1].
int defer_layer_count(const mt_config& cfg);

}  // namespace mt
