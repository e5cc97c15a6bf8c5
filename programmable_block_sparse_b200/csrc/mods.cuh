// The fixed menu of mask and score rules as device functions.
//
// mask_mod kinds and the logical query position follow "flexattention-score-
// mod-block-mask" (charlestar.github.io) sections "A call example pinned to one
// version" (window 0 <= p_i - p_j < W), "Packing" (same document) and "At
// decode, q_idx = 0 is not position 0" (q = q_idx + offset); "Attention
// expressions" (docs.tensorcad.dev) "Examples" (prefix-LM, sinks, chunked,
// ALiBi, Gemma 2 cap); "Causal Mask" (quant67.com) section 4 (bottom-right
// alignment when the query is shorter than the keys).
#pragma once

#include <stdint.h>

#include "../../include/flexattn.h"

namespace fa {

struct MaskParams {
  int kind, window, n_sink, prefix, chunk, doc_batch;
  const int* doc_id;
  const int* kv_len;
};

struct ScoreParams {
  int kind;
  float cap;
  int slope_heads;
  int pos_batch;
  const int* pos;
};

// Valid KV length of sequence b, clamped to [0, S].
__device__ __forceinline__ int seq_len_b(const MaskParams& m, int b, int S) {
  if (m.kv_len == nullptr) return S;
  int n = __ldg(m.kv_len + b);
  return n < 0 ? 0 : (n > S ? S : n);
}

// Logical query position of row i: bottom-right aligned against S_b keys.
__device__ __forceinline__ int query_pos(int i, int L, int S_b) { return i + (S_b - L); }

// M(b, q, kv): visibility of key kv for the query at logical position q.
// The caller guarantees 0 <= kv; keys at or beyond S_b are invisible.
__device__ __forceinline__ bool mask_visible(const MaskParams& m, int b, int q, int kv, int S_b, int S) {
  if (kv >= S_b) return false;
  switch (m.kind) {
    case FA_MASK_NONE:
      return true;
    case FA_MASK_CAUSAL:
      return kv <= q;
    case FA_MASK_SLIDING_WINDOW:
      return kv <= q && (q - kv < m.window || kv < m.n_sink);
    case FA_MASK_DOCUMENT: {
      if (kv > q) return false;  // here 0 <= kv <= q < S
      const int* d = m.doc_id + static_cast<int64_t>(m.doc_batch > 1 ? b : 0) * S;
      return __ldg(d + q) == __ldg(d + kv);
    }
    case FA_MASK_PREFIX_LM:
      return kv <= q || kv < m.prefix;
    case FA_MASK_CHUNKED:
      return kv <= q && (q / m.chunk) == (kv / m.chunk);  // both >= 0 when kv <= q
    default:
      return false;
  }
}

// The keys visible to the query at logical position q form at most two
// inclusive spans [a0, a1] and [b0, b1] (empty when the low end exceeds the
// high end), already clipped to [0, S_b - 1].  For DOCUMENT this is only the
// causal bound [0, q]: the same-document test is applied per key on top.
struct KeySpans {
  int a0, a1, b0, b1;
};

__device__ __forceinline__ KeySpans visible_spans(const MaskParams& m, int q, int S_b) {
  const int last = S_b - 1;
  KeySpans r{1, 0, 1, 0};
  switch (m.kind) {
    case FA_MASK_NONE:
      r.a0 = 0;
      r.a1 = last;
      break;
    case FA_MASK_CAUSAL:
    case FA_MASK_DOCUMENT:
      r.a0 = 0;
      r.a1 = min(q, last);
      break;
    case FA_MASK_SLIDING_WINDOW:
      r.a0 = max(q - m.window + 1, 0);
      r.a1 = min(q, last);
      r.b0 = 0;
      r.b1 = min(min(m.n_sink - 1, q), last);
      break;
    case FA_MASK_PREFIX_LM:
      r.a0 = 0;
      r.a1 = min(max(q, m.prefix - 1), last);
      break;
    case FA_MASK_CHUNKED:
      if (q >= 0) {
        r.a0 = (q / m.chunk) * m.chunk;
        r.a1 = min(q, last);
      }
      break;
    default:
      break;
  }
  return r;
}

// slope_h = 2^(-8 (h + 1) / H).
__device__ __forceinline__ float distance_slope(int h, int H) {
  return exp2f(-8.0f * static_cast<float>(h + 1) / static_cast<float>(H));
}

__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int pos_at(const ScoreParams& s, int b, int t, int S) {
  t = t < 0 ? 0 : (t >= S ? S - 1 : t);
  return __ldg(s.pos + static_cast<int64_t>(s.pos_batch > 1 ? b : 0) * S + t);
}

// g(x, b, h, q, kv) for the scaled score x.  kPrecise selects tanhf (fp32
// path) over the hardware tanh approximation (bf16 path).
template <bool kPrecise>
__device__ __forceinline__ float score_apply(const ScoreParams& s, float x, int b, int q, int kv, int S, float slope) {
  switch (s.kind) {
    case FA_SCORE_NONE:
      return x;
    case FA_SCORE_SOFTCAP:
      return s.cap * (kPrecise ? tanhf(x / s.cap) : tanh_fast(x * (1.0f / s.cap)));
    case FA_SCORE_ALIBI:
      return x - slope * static_cast<float>(q - kv);
    case FA_SCORE_CAP_THEN_BIAS: {
      float capped = s.cap * (kPrecise ? tanhf(x / s.cap) : tanh_fast(x * (1.0f / s.cap)));
      int d = (s.pos != nullptr) ? (pos_at(s, b, kv, S) - pos_at(s, b, q, S)) : (kv - q);
      return capped + slope * static_cast<float>(d);
    }
    default:
      return x;
  }
}

}  // namespace fa
