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

// A composed rule (FA_MASK_PROGRAM) as the host rewrote it: an AND of
// clauses, each an OR of literals (a predicate, possibly negated).
constexpr int kMaxClauses = 8;
constexpr int kMaxLits = 4;
constexpr int kLitNeg = 0x100;  // flag in MaskLit::op: the predicate negated

struct MaskLit {
  int op;        // FA_PROG_* predicate, | kLitNeg when negated
  int arg;
  uint32_t pat;  // FA_PROG_STRIDE with arg < 32: bits 0, arg, 2 arg, ... of a word
};

struct MaskParams {
  int kind, window, n_sink, prefix, chunk, doc_batch;
  const int* doc_id;
  const int* kv_len;
  int n_clauses;
  int clause_len[kMaxClauses];
  MaskLit lit[kMaxClauses][kMaxLits];
  int reads_head;  // a literal reads the query head
  int reads_doc;   // a literal reads document ids
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

// floor(a / b) and a mod b in [0, b), for b >= 1 and any a.
__device__ __forceinline__ int floor_div(int a, int b) {
  const int q = a / b;
  return (a % b != 0 && a < 0) ? q - 1 : q;
}
__device__ __forceinline__ int mod_pos(int a, int b) {
  const int r = a % b;
  return r < 0 ? r + b : r;
}

// One predicate of a composed rule for one pair (query position q, key kv,
// query head h); 0 <= kv < S.
__device__ __forceinline__ bool prog_pred(const MaskParams& m, int op, int arg, int b, int h, int q, int kv, int S) {
  switch (op) {
    case FA_PROG_TRUE:
      return true;
    case FA_PROG_CAUSAL:
      return kv <= q;
    case FA_PROG_DISTANCE_BELOW:
      return q - kv < arg;
    case FA_PROG_KEY_BELOW:
      return kv < arg;
    case FA_PROG_SAME_CHUNK:
      return floor_div(q, arg) == floor_div(kv, arg);
    case FA_PROG_SAME_DOCUMENT: {
      if (q < 0 || q >= S) return false;
      const int* d = m.doc_id + static_cast<int64_t>(m.doc_batch > 1 ? b : 0) * S;
      return __ldg(d + q) == __ldg(d + kv);
    }
    case FA_PROG_STRIDE:
      return mod_pos(q - kv, arg) == 0;
    case FA_PROG_HEAD_BELOW:
      return h < arg;
    default:
      return false;
  }
}

// The composed rule for one pair: AND over clauses of OR over literals.
__device__ __forceinline__ bool program_visible(const MaskParams& m, int b, int h, int q, int kv, int S) {
  bool res = true;
#pragma unroll
  for (int c = 0; c < kMaxClauses; ++c) {
    if (c >= m.n_clauses) break;
    bool cl = false;
#pragma unroll
    for (int l = 0; l < kMaxLits; ++l) {
      if (l >= m.clause_len[c]) break;
      const MaskLit lt = m.lit[c][l];
      cl = cl || (prog_pred(m, lt.op & 0xff, lt.arg, b, h, q, kv, S) != ((lt.op & kLitNeg) != 0));
    }
    res = res && cl;
  }
  return res;
}

// Bits [lo, hi] of a 32-bit word (positions relative to the word's first
// key); empty when hi < lo, clipped to [0, 31].
__device__ __forceinline__ uint32_t span_bits(int lo, int hi) {
  lo = max(lo, 0);
  hi = min(hi, 31);
  if (hi < lo) return 0u;
  const uint32_t upto = hi == 31 ? 0xFFFFFFFFu : ((2u << hi) - 1u);
  return upto & ~((1u << lo) - 1u);
}

// One predicate over the 32 keys base .. base + 31 for query q of head h:
// bit i says whether it holds for key base + i.  same_doc holds the
// same-document bits, which the caller computes from staged ids.
__device__ __forceinline__ uint32_t prog_pred_bits(const MaskLit& lt, int h, int q, int base, uint32_t same_doc) {
  const int op = lt.op & 0xff, arg = lt.arg;
  switch (op) {
    case FA_PROG_TRUE:
      return 0xFFFFFFFFu;
    case FA_PROG_CAUSAL:
      return span_bits(-1, q - base);
    case FA_PROG_DISTANCE_BELOW:  // kv > q - arg
      return span_bits(q - arg + 1 - base, 31);
    case FA_PROG_KEY_BELOW:
      return span_bits(-1, arg - 1 - base);
    case FA_PROG_SAME_CHUNK: {
      const int c0 = floor_div(q, arg) * arg;
      return span_bits(c0 - base, c0 + arg - 1 - base);
    }
    case FA_PROG_SAME_DOCUMENT:
      return same_doc;
    case FA_PROG_STRIDE: {  // keys base + i with i = q - base (mod arg)
      const int r = mod_pos(q - base, arg);
      return arg < 32 ? (lt.pat << r) : (r < 32 ? (1u << r) : 0u);
    }
    case FA_PROG_HEAD_BELOW:
      return h < arg ? 0xFFFFFFFFu : 0u;
    default:
      return 0u;
  }
}

// The composed rule over the 32 keys base .. base + 31 (keys >= S_b are the
// caller's to clear).
__device__ __forceinline__ uint32_t program_bits(const MaskParams& m, int h, int q, int base, uint32_t same_doc) {
  uint32_t res = 0xFFFFFFFFu;
#pragma unroll
  for (int c = 0; c < kMaxClauses; ++c) {
    if (c >= m.n_clauses) break;
    uint32_t cl = 0u;
#pragma unroll
    for (int l = 0; l < kMaxLits; ++l) {
      if (l >= m.clause_len[c]) break;
      const MaskLit lt = m.lit[c][l];
      const uint32_t v = prog_pred_bits(lt, h, q, base, same_doc);
      cl |= (lt.op & kLitNeg) ? ~v : v;
    }
    res &= cl;
  }
  return res;
}

// Verdict of one predicate over a whole box of query positions [q0, q1] and
// keys [k0, k1] (head h): 0 false everywhere, 1 true everywhere, 2 mixed or
// not decidable from the bounds (the caller then looks at the cells).
__device__ __forceinline__ int prog_pred_box(const MaskLit& lt, int h, int q0, int q1, int k0, int k1) {
  const int op = lt.op & 0xff, arg = lt.arg;
  switch (op) {
    case FA_PROG_TRUE:
      return 1;
    case FA_PROG_CAUSAL:
      return k1 <= q0 ? 1 : (k0 > q1 ? 0 : 2);
    case FA_PROG_DISTANCE_BELOW:
      return q1 - k0 < arg ? 1 : (q0 - k1 >= arg ? 0 : 2);
    case FA_PROG_KEY_BELOW:
      return k1 < arg ? 1 : (k0 >= arg ? 0 : 2);
    case FA_PROG_SAME_CHUNK: {
      const int a0 = floor_div(q0, arg), a1 = floor_div(q1, arg);
      const int b0 = floor_div(k0, arg), b1 = floor_div(k1, arg);
      if (a0 == a1 && b0 == b1 && a0 == b0) return 1;
      return (a1 < b0 || b1 < a0) ? 0 : 2;
    }
    case FA_PROG_STRIDE: {
      if (arg == 1) return 1;
      const int dmin = q0 - k1, dmax = q1 - k0;
      if (dmax - dmin + 1 >= arg) return 2;  // holds for some pairs, fails for others
      const int first = dmin + mod_pos(-dmin, arg);  // smallest multiple of arg >= dmin
      if (first > dmax) return 0;
      return dmin == dmax ? 1 : 2;
    }
    case FA_PROG_HEAD_BELOW:
      return h < arg ? 1 : 0;
    default:  // FA_PROG_SAME_DOCUMENT reads data: decided per cell
      return 2;
  }
}

// The composed rule over a box, in three-valued logic (0 / 1 / 2 as above).
__device__ __forceinline__ int program_box(const MaskParams& m, int h, int q0, int q1, int k0, int k1) {
  int res = 1;
#pragma unroll
  for (int c = 0; c < kMaxClauses; ++c) {
    if (c >= m.n_clauses) break;
    int cl = 0;
#pragma unroll
    for (int l = 0; l < kMaxLits; ++l) {
      if (l >= m.clause_len[c]) break;
      const MaskLit lt = m.lit[c][l];
      int v = prog_pred_box(lt, h, q0, q1, k0, k1);
      if (lt.op & kLitNeg) v = v == 2 ? 2 : 1 - v;
      cl = (cl == 1 || v == 1) ? 1 : ((cl == 2 || v == 2) ? 2 : 0);
    }
    res = (res == 0 || cl == 0) ? 0 : ((res == 2 || cl == 2) ? 2 : 1);
  }
  return res;
}

// The transposed view, for the backward pass over key rows: one predicate
// over the 32 queries at logical positions qbase .. qbase + 31 for key kv.
__device__ __forceinline__ uint32_t prog_pred_bits_q(const MaskLit& lt, int h, int kv, int qbase, uint32_t same_doc) {
  const int op = lt.op & 0xff, arg = lt.arg;
  switch (op) {
    case FA_PROG_TRUE:
      return 0xFFFFFFFFu;
    case FA_PROG_CAUSAL:  // q >= kv
      return span_bits(kv - qbase, 31);
    case FA_PROG_DISTANCE_BELOW:  // q < kv + arg
      return span_bits(-1, kv + arg - 1 - qbase);
    case FA_PROG_KEY_BELOW:
      return kv < arg ? 0xFFFFFFFFu : 0u;
    case FA_PROG_SAME_CHUNK: {
      const int c0 = floor_div(kv, arg) * arg;
      return span_bits(c0 - qbase, c0 + arg - 1 - qbase);
    }
    case FA_PROG_SAME_DOCUMENT:
      return same_doc;
    case FA_PROG_STRIDE: {  // queries qbase + i with i = kv - qbase (mod arg)
      const int r = mod_pos(kv - qbase, arg);
      return arg < 32 ? (lt.pat << r) : (r < 32 ? (1u << r) : 0u);
    }
    case FA_PROG_HEAD_BELOW:
      return h < arg ? 0xFFFFFFFFu : 0u;
    default:
      return 0u;
  }
}

__device__ __forceinline__ uint32_t program_bits_q(const MaskParams& m, int h, int kv, int qbase, uint32_t same_doc) {
  uint32_t res = 0xFFFFFFFFu;
#pragma unroll
  for (int c = 0; c < kMaxClauses; ++c) {
    if (c >= m.n_clauses) break;
    uint32_t cl = 0u;
#pragma unroll
    for (int l = 0; l < kMaxLits; ++l) {
      if (l >= m.clause_len[c]) break;
      const MaskLit lt = m.lit[c][l];
      const uint32_t v = prog_pred_bits_q(lt, h, kv, qbase, same_doc);
      cl |= (lt.op & kLitNeg) ? ~v : v;
    }
    res &= cl;
  }
  return res;
}

// Fixed rules over the 32 queries qbase .. qbase + 31 for key kv (kv < S_b;
// the caller clears queries outside the valid rows and applies same_doc for
// the document rule).
__device__ __forceinline__ uint32_t fixed_bits_q(const MaskParams& m, int kv, int qbase) {
  switch (m.kind) {
    case FA_MASK_NONE:
      return 0xFFFFFFFFu;
    case FA_MASK_CAUSAL:
    case FA_MASK_DOCUMENT:
      return span_bits(kv - qbase, 31);
    case FA_MASK_SLIDING_WINDOW:
      return kv < m.n_sink ? span_bits(kv - qbase, 31) : span_bits(kv - qbase, kv + m.window - 1 - qbase);
    case FA_MASK_PREFIX_LM:
      return kv < m.prefix ? 0xFFFFFFFFu : span_bits(kv - qbase, 31);
    case FA_MASK_CHUNKED: {
      const int c0 = (kv / m.chunk) * m.chunk;  // kv >= 0
      return span_bits(kv - qbase, c0 + m.chunk - 1 - qbase);
    }
    default:
      return 0u;
  }
}

// M(b, h, q, kv): visibility of key kv for the query at logical position q
// of query head h.  The caller guarantees 0 <= kv; keys at or beyond S_b are
// invisible.
__device__ __forceinline__ bool mask_visible(const MaskParams& m, int b, int h, int q, int kv, int S_b, int S) {
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
    case FA_MASK_PROGRAM:
      return program_visible(m, b, h, q, kv, S);
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
