// Tensor-core prefill kernel for sm_100a: the FlexAttention forward pass over the
// tiles a BlockMask lists, with S = Q K^T and O += P V on tcgen05 (UMMA) and the
// accumulators in tensor memory.
//
// Definition ("flexattention-score-mod-block-mask", charlestar.github.io):
// section "What one connection goes through" (scaled score, score rule, mask to
// -inf, softmax-weighted values); section "mask_mod defines legal connections,
// BlockMask defines block work" (empty tiles skipped, full tiles without the
// element mask but with the score rule, partial tiles with both, score rule
// first); section "The compiler plugs local rules into the attention template"
// (online softmax and tiling without materialising the score matrix).
//
// A work item is two adjacent 128-row query tiles (A = 2p, B = 2p + 1) of one
// (batch, query head).  The kernel is persistent, one CTA per SM, through
// cluster launch control: a CTA that finishes an item takes over the launch
// of the next CTA that has not started, longest items first.  The two
// tiles' BlockMask lists are merged in key order and every K/V tile of the
// union is loaded once for both:
//   warp 0       TMA producer: Q_A, Q_B, then K_u, V_u of every union tile u
//                into NS-stage rings (128 x 64 bf16 boxes, 128-byte swizzle).
//   warp 1       TMEM allocator and MMA issuer (one elected thread):
//                S_X = Q_X K_u^T (SS form, both K-major), O_X += P_X V_u (TS
//                form: P from TMEM, V MN-major), for X in {A, B} and u in the
//                tile's own list.
//   warps 2-5    softmax group of tile A, warps 6-9 of tile B (warp % 4 picks
//                the TMEM lane quadrant); one query
//                row per thread (TMEM lane): S row -> score rule -> element mask
//                (partial / edge tiles) -> running max -> P = 2^(t - m) as bf16
//                into TMEM over the S columns it has read -> running sum;
//                finally O / l and lse.  The two groups alternate on the tensor
//                core: while one computes its softmax the other's MMAs run.
// TMEM columns of tile X in {0, 1}: at head dim 128, S/P at 256 X (P as bf16
// pairs over the first 64 S columns, once read) and O at 256 X + 128; the
// MMA thread issues PV_X(u) before QK_X(next), and the commit that signals
// S_X(next) also covers PV_X(u), so a softmax group that sees its S ready may
// read and rescale O_X and overwrite P_X without further waits.  At head dim
// 64, S at 256 X, P at 256 X + 128 and O at 256 X + 192 have columns of their
// own: QK_X(next) is issued as soon as the group has read S (s_free), ahead
// of PV_X(u), and the group waits for that PV (o_done) only before it writes
// P or rescales O.
// PV runs in two halves: the group signals p_half once P of keys 0-63 is in
// TMEM and p_full once all of P is, so the first four PV MMAs overlap the
// second half of the softmax.
// The running max only moves (and O rescales) when it grows by more than 2^8;
// P then stays below 2^8 and the final O / l ratio is exact.
//
// Barrier phases and ring positions run on across items.  The next item's Q
// is loaded once the current item's last QK has completed, and its first QKs
// are issued as soon as the current item's last PVs are, so the next S is
// computed while the softmax groups write the current item's output.
//
// Every mbarrier wait is bounded; on a timeout the CTA records FA_ERR_TIMEOUT
// in the status word, stops issuing work, drains its own copies and MMAs
// (again with bounded waits), frees its TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "fastmath.cuh"
#include "launch.h"
#include "mods.cuh"

namespace fa {

namespace {

constexpr int kThreads = 320;
constexpr int kTile = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Start of the running maximum: finite and below any real score (log2
// units), so that tiles without a visible key for a row give P = 2^-inf = 0
// with no test of the maximum, and the first visible key always moves it.
constexpr float kNoKeyMax = -1.0e30f;
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int kBoxes = D / 64;             // 64-column boxes per tile row
  static constexpr int kTileBytes = kTile * D * 2;  // one Q/K/V tile
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kSmemBytes = kTileBytes * (2 + 2 * kStages) + 1024;
};

enum : uint32_t { kInA = 1, kFullA = 2, kInB = 4, kFullB = 8 };
constexpr int kInfoFull = 1 << 30;  // class bit in the published tile info

struct Barriers {
  uint4 clc_resp[2];              // answers of the launch-control requests (16-byte aligned)
  uint64_t clc_full[2];           // answer r has landed in clc_resp[r & 1]
  uint64_t clc_empty[2];          // the MMA thread and the 8 softmax warps have read it
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2];
  uint64_t p_half[2];  // the first 64 keys' P is written: their PV may start
  uint64_t s_free[2], o_done[2];  // head dim 64 only: S read out / PV finished
  uint64_t q_empty;               // the item's last QK is done: Q may be reloaded
  uint64_t o_final[2];            // per group: the item's last PV is done
  uint64_t mma_done;              // every MMA of the CTA has completed
  int info[2][2];  // per group, ring of 2: tile index | kFullA-style class bit
  uint32_t tmem_base;
  int abort;
};

// Walks the union of the two query tiles' full and partial lists in
// descending key order (for causal-like rules the nearest, highest-scoring
// keys come first, so the running max rarely has to move afterwards).
struct UnionIter {
  // lists 0 / 1: full / partial of tile A; 2 / 3: full / partial of tile B
  const int* lst[4];
  int j[4];  // index of each list's head, counting down
  int c[4];  // head values (-1 once a list is exhausted), loaded a step ahead
             // so that next() does not wait on global-memory latency

  __device__ void init(const FwdArgs& a, int64_t row_a, bool has_b) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int64_t row = row_a + t;
      const bool on = t == 0 || has_b;
      lst[2 * t] = a.bm.full_kv_indices + row * a.bm.Nb;
      lst[2 * t + 1] = a.bm.kv_indices + row * a.bm.Nb;
      j[2 * t] = (on ? __ldg(a.bm.full_kv_num_blocks + row) : 0) - 1;
      j[2 * t + 1] = (on ? __ldg(a.bm.kv_num_blocks + row) : 0) - 1;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = j[i] >= 0 ? __ldg(lst[i] + j[i]) : -1;
  }
  template <int I>
  __device__ __forceinline__ void advance() {
    --j[I];
    c[I] = j[I] >= 0 ? __ldg(lst[I] + j[I]) : -1;
  }
  __device__ bool next(int& n, uint32_t& flags) {
    n = max(max(c[0], c[1]), max(c[2], c[3]));
    if (n < 0) return false;
    flags = 0;
    if (c[0] == n) {
      flags |= kInA | kFullA;
      advance<0>();
    } else if (c[1] == n) {
      flags |= kInA;
      advance<1>();
    }
    if (c[2] == n) {
      flags |= kInB | kFullB;
      advance<2>();
    } else if (c[3] == n) {
      flags |= kInB;
      advance<3>();
    }
    return true;
  }
};

// Work items.  A work item is a pair of adjacent query tiles of one (batch,
// query head), one per CTA of the launch grid (head, batch, pair), with the
// pair counted down in z: CTAs start in linear order (x fastest, z slowest),
// so every (batch, head)'s last pairs -- under causal-like rules the longest
// lists of key tiles -- come first and the short ones fill in at the end.
// The kernel is persistent through cluster launch control: a running CTA
// takes its own item, then repeatedly cancels the launch of the next CTA
// that has not started and does that CTA's item, keeping its TMEM, barriers
// and pipelines.  Items thus go, longest first, to whichever SM frees up.
struct Item {
  int h, b, mtA, mtB;
  bool has_b;
  int hk, S_b;
  int64_t row_a;  // the block mask's list row of tile A
};

__device__ __forceinline__ Item item_of(const FwdArgs& a, int x, int y, int z) {
  Item it;
  const int pair = static_cast<int>(gridDim.z) - 1 - z;
  it.h = x;
  it.b = y;
  it.mtA = 2 * pair;
  it.mtB = 2 * pair + 1;
  it.has_b = it.mtB < a.bm.Mb;
  it.hk = it.h / a.G;
  it.S_b = seq_len_b(a.mask, it.b, a.S);
  const int bmb = a.bm.B > 1 ? it.b : 0, bmh = a.bm.H > 1 ? it.h : 0;
  it.row_a = (static_cast<int64_t>(bmb) * a.bm.H + bmh) * a.bm.Mb + it.mtA;
  return it;
}

// Rarely run paths, kept out of line so the softmax loop stays compact in the
// instruction cache: a composed mask rule's bits for one 32-key word, and the
// hardware tanh of 64 columns (for a half whose arguments exceed the
// polynomial's range).
__device__ __noinline__ uint32_t program_word(const MaskParams* m, int h, int q, int base, uint32_t same, int S_b) {
  return program_bits(*m, h, q, base, same) & span_bits(-1, S_b - 1 - base);
}
// In place in TMEM: the 64 columns at taddr become tanh(column * c_in).
__device__ __noinline__ void tanh_hw_tmem(uint32_t taddr, float c_in) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t r[16];
    tmem_ld16(taddr + 16 * c, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float y;
      asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(__uint_as_float(r[i]) * c_in));
      r[i] = __float_as_uint(y);
    }
    tmem_st16(taddr + 16 * c, r);
  }
  tmem_wait_st();
}

// The same-document bits of a tile's four 32-key words for the calling row
// (document id `mine`; `none` clears them): lane l reads the ids of keys
// 32 w + l from the staged row, and each distinct document among the warp's
// rows takes one round of ballots (one or two rounds on a packed batch).
// Called by all 32 lanes of a warp.
__device__ __noinline__ uint4 doc_words(const int* keys_doc, int mine, bool none) {
  const int lane = threadIdx.x & 31;
  int kd[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) kd[w] = keys_doc[32 * w + lane];
  uint4 r = make_uint4(0u, 0u, 0u, 0u);
  uint32_t pending = 0xFFFFFFFFu;
  while (pending) {
    const int d = __shfl_sync(0xffffffffu, mine, __ffs(pending) - 1);
    const uint32_t m0 = __ballot_sync(0xffffffffu, kd[0] == d), m1 = __ballot_sync(0xffffffffu, kd[1] == d);
    const uint32_t m2 = __ballot_sync(0xffffffffu, kd[2] == d), m3 = __ballot_sync(0xffffffffu, kd[3] == d);
    const bool take = mine == d;
    if (take) r = make_uint4(m0, m1, m2, m3);
    pending &= ~__ballot_sync(0xffffffffu, take);
  }
  return none ? make_uint4(0u, 0u, 0u, 0u) : r;
}

// Softmax and epilogue of one 128-row query tile; runs on one warpgroup.
// gbase counts the group's tiles of earlier work items and nfin the items in
// which it had tiles (the phases of its barriers run on across items);
// returns false once a wait gave up.
template <int D, int SCORE>
__device__ __forceinline__ bool softmax_group(const FwdArgs& a, Barriers& bars, float (*s_pos)[kTile],
                                              int (*s_doc)[kTile], int X, int mt, int h, int b, int S_b,
                                              int64_t row_a, bool has_b, uint32_t tbase, int& gbase, int& nfin) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;
  const int grow = mt * kTile + r;
  const bool row_ok = grow < a.L;
  const int qpos = query_pos(grow, a.L, S_b);
  const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
  // head dim 64: S, P and O each have their own columns (S at 256 X, P at
  // 256 X + 128, O at 256 X + 192), so the next tile's S can be computed
  // while this tile's P is still being written.  Head dim 128: P overwrites
  // the S columns it has read and O sits at 256 X + 128.
  constexpr bool kSepP = D == 64;
  const uint32_t col_s = 256u * X, col_o = 256u * X + (kSepP ? 192u : 128u);
  const uint32_t col_p = kSepP ? 256u * X + 128u : col_s;
  volatile int* abort = &bars.abort;
  const int Hs = a.score.slope_heads > 0 ? a.score.slope_heads : a.Hq;
  const float slope2 = distance_slope(h, Hs) * kLog2e;
  float c_in, c_out;
  if constexpr (SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_CAP_THEN_BIAS) {
    c_in = a.scale / a.score.cap;
    c_out = a.score.cap * kLog2e;
  } else {
    c_in = 0.0f;
    c_out = a.scale * kLog2e;
  }
  const bool has_pos = SCORE == FA_SCORE_CAP_THEN_BIAS && a.score.pos != nullptr;
  const float pq_scaled = has_pos ? slope2 * static_cast<float>(pos_at(a.score, b, qpos, a.S)) : 0.0f;
  const bool is_prog = a.mask.kind == FA_MASK_PROGRAM;
  // document ids are staged for the document rule and for composed rules
  // that compare documents
  const bool is_doc = a.mask.kind == FA_MASK_DOCUMENT || (is_prog && a.mask.reads_doc);
  const int* doc_row = is_doc ? a.mask.doc_id + static_cast<int64_t>(a.mask.doc_batch > 1 ? b : 0) * a.S : nullptr;
  const int my_doc = (is_doc && row_ok && qpos >= 0) ? __ldg(doc_row + qpos) : -1;
  const KeySpans spans = visible_spans(a.mask, qpos, S_b);
  float m_ref = kNoKeyMax, l_sum = 0.0f;
  float m_true = -INFINITY;  // exact row maximum (log2 units), for max_scores
  bool alive = true;
  int cnt = 0;

  const int64_t row_x = row_a + X;
  const bool x_on = X == 0 || has_b;
  const int total = x_on ? __ldg(a.bm.full_kv_num_blocks + row_x) + __ldg(a.bm.kv_num_blocks + row_x) : 0;
  // the four warps of the group stage key-side values for each other when
  // the rules read positions or document ids (the same for every tile)
  const bool group_stage = has_pos || is_doc;
  // A warp leaves this loop only at its top, together with its whole group
  // when the group stages key-side values (the barrier below): a wait that
  // gives up inside a tile marks the warp dead, it skips the rest of the tile
  // and votes false at the next barrier.
  for (; cnt < total; ++cnt) {
    const int g = gbase + cnt;  // the group's tile count over all items so far
    // a warp-uniform result: the lanes leave the loop together or not at all
    bool ok = alive && __all_sync(0xffffffffu, mbar_wait(&bars.s_full[X], g & 1, abort, a.status, a.wait_cycles));
    const int info = ok ? bars.info[X][g & 1] : 0;
    const int n = info & (kInfoFull - 1);
    const bool full = (info & kInfoFull) != 0;
    const int kv0 = n * kTile;
    const bool edge = kv0 + kTile > S_b;
    const bool stage_doc = is_doc && (!full || edge);  // the same for every row of the tile
    if (group_stage) {
      // this tile's key-side values into smem (double-buffered by g & 1);
      // every warp of the group reaches the barrier on every tile, and it
      // also tells each warp whether all four got their S, so that on a
      // timeout the group leaves together and no warp waits for another
      if (ok) {
        const int kv = kv0 + r;
        if (has_pos) s_pos[g & 1][r] = slope2 * static_cast<float>(pos_at(a.score, b, kv, a.S));
        if (stage_doc) s_doc[g & 1][r] = kv < a.S ? __ldg(doc_row + kv) : -2;
      }
      ok = named_bar_and(1 + X, 128, ok);
    }
    if (!ok) {
      alive = false;
      break;
    }
    tc_fence_after();

    // pass 1, per 64-column half: score rule on every cell, element mask on
    // partial tiles / ragged edges / rows past L, row max.  The transformed
    // scores t = g log2(e) go back to TMEM for pass 2 already shifted by
    // m_fold (the running maximum, or 0 before the first visible key), so
    // that pass 2 subtracts nothing unless the maximum moves.  Arithmetic in
    // f32x2 pairs; maxima as trees of three-input maxima.
    const bool need_mask = !full || edge || !row_ok;
    // same-document bits of the tile's four 32-key words for this row
    uint4 doc_bits = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
    if (stage_doc) doc_bits = doc_words(s_doc[g & 1], my_doc, qpos < 0);  // the same for every row of the tile
    const float m_fold = (m_ref == kNoKeyMax) ? 0.0f : m_ref;
    float mx = -INFINITY;  // maximum of t - m_fold over this tile
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      float t[64];
      const int c0 = 64 * half;
      tmem_load64(tbase + lane_base + col_s + c0, t);
      float2* t2 = reinterpret_cast<float2*>(t);
      if constexpr (SCORE == FA_SCORE_NONE) {
#pragma unroll
        for (int i = 0; i < 32; ++i) t2[i] = fma2(t2[i], splat2(c_out), splat2(-m_fold));
      } else if constexpr (SCORE == FA_SCORE_ALIBI) {
        // bias of column c: slope2 (kv0 + c0 + c - q) - m_fold
        const float2 b0 = splat2(slope2 * static_cast<float>(kv0 + c0 - qpos) - m_fold);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 col = make_float2(static_cast<float>(2 * i), static_cast<float>(2 * i + 1));
          t2[i] = fma2(t2[i], splat2(c_out), fma2(splat2(slope2), col, b0));
        }
      } else {
        // soft-cap on the FMA pipe: c tanh(s / c) with tanh's odd series,
        // exact enough for |s / c| <= kTanhPolyMax; a half whose largest
        // argument is beyond that is redone with the hardware tanh
        float2* th = t2;  // tanh(s / c), computed in place
        float umax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float2 u0, u1;
          th[i] = tanh_poly2(mul2(t2[i], splat2(c_in)), u0);
          th[i + 1] = tanh_poly2(mul2(t2[i + 1], splat2(c_in)), u1);
          umax = max3f(umax, fmaxf(u0.x, u0.y), fmaxf(u1.x, u1.y));
        }
        if (__any_sync(0xffffffffu, !(umax <= kTanhPolyMax * kTanhPolyMax))) {
          // rare: reload the raw scores (still in TMEM) for the hardware tanh
          tanh_hw_tmem(tbase + lane_base + col_s + c0, c_in);
          tmem_load64(tbase + lane_base + col_s + c0, t);
        }
        if constexpr (SCORE == FA_SCORE_SOFTCAP) {
#pragma unroll
          for (int i = 0; i < 32; ++i) t2[i] = fma2(th[i], splat2(c_out), splat2(-m_fold));
        } else if (has_pos) {
          // bias of column c: slope2 (p[kv] - p[q]) - m_fold, p[kv] staged in smem
          const float2* pk = reinterpret_cast<const float2*>(s_pos[g & 1] + c0);
          const float2 b0 = splat2(-pq_scaled - m_fold);
#pragma unroll
          for (int i = 0; i < 32; ++i) t2[i] = fma2(th[i], splat2(c_out), add2(pk[i], b0));
        } else {
          const float2 b0 = splat2(slope2 * static_cast<float>(kv0 + c0 - qpos) - m_fold);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 col = make_float2(static_cast<float>(2 * i), static_cast<float>(2 * i + 1));
            t2[i] = fma2(th[i], splat2(c_out), fma2(splat2(slope2), col, b0));
          }
        }
      }
      if (need_mask) {
        uint32_t bits[2];
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int base = kv0 + c0 + 32 * w;
          // same-document bits of the word's keys (half is a rolled loop: a
          // select, not an index, keeps doc_bits in registers)
          const uint32_t same = half == 0 ? (w == 0 ? doc_bits.x : doc_bits.y) : (w == 0 ? doc_bits.z : doc_bits.w);
          if (is_prog) {
            bits[w] = row_ok ? program_word(&a.mask, h, qpos, base, same, S_b) : 0u;
          } else {
            bits[w] = row_ok ? ((span_bits(spans.a0 - base, spans.a1 - base) |
                                 span_bits(spans.b0 - base, spans.b1 - base)) & same)
                             : 0u;
          }
        }
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (!((bits[c >> 5] >> (c & 31)) & 1u)) t[c] = -INFINITY;
      }
      mx = fmaxf(mx, max64(t));
      tmem_store64(tbase + lane_base + col_s + c0, t);
    }
    tmem_wait_st();
    mx += m_fold;  // the tile's true maximum (log2 units), -inf without a visible key
    m_true = fmaxf(m_true, mx);

    // running max: move it (and rescale O) only when it grows past 2^8.  O_X
    // holds the sum through this group's previous tile once that PV is done:
    // at head dim 128 the commit behind s_full covered it; at head dim 64 the
    // o_done barrier says so.  No MMA writes O_X until P_X is signalled.
    const bool grow_max = mx > m_ref + kRescaleThreshold;
    const float m_new = grow_max ? mx : m_ref;
    // O_X holds a sum only after the group's first tile (its first PV
    // overwrites whatever the columns held)
    const bool rescale = grow_max && cnt > 0;
    // the first tile of an item needs no wait: the previous item's last PV
    // was covered by that item's o_final
    bool pv_done = !kSepP || cnt == 0;
    auto wait_pv = [&]() {
      // the previous tile's PV reads P and writes O; with separate S columns
      // the S of this tile may have landed before that PV finished
      if (!pv_done) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.o_done[X], (g - 1) & 1, abort, a.status, a.wait_cycles))) alive = false;
        tc_fence_after();
        pv_done = true;
      }
    };
    if (__any_sync(0xffffffffu, rescale)) {
      wait_pv();
      const float f = rescale ? ex2_approx(m_ref - m_new) : 1.0f;
      if (alive) {
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t rr[16];
          tmem_ld16(tbase + lane_base + col_o + c * 16, rr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
          tmem_st16(tbase + lane_base + col_o + c * 16, rr);
        }
      }
      l_sum *= f;
    }
    m_ref = m_new;
    // TMEM holds t - m_fold; P = 2^(t - m_ref) needs a further shift only
    // when the maximum moved (or before the first visible key)
    const float delta = m_ref - m_fold;
    const bool shift = __any_sync(0xffffffffu, delta != 0.0f);

    // pass 2, per half: P = 2^(t - m) as bf16 pairs, 64 columns in all
    // (head dim 128: over the first 64 S columns; half h writes columns
    // [32 h, 32 h + 32), all of which pass 2 has read)
    float psum = 0.0f;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      float t[64];
      tmem_load64(tbase + lane_base + col_s + 64 * half, t);
      if (kSepP && half == 1) {
        // all of S is in registers now: the next tile's QK may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_free[X]);
      }
      if (shift) {
        float2* t2 = reinterpret_cast<float2*>(t);
#pragma unroll
        for (int i = 0; i < 32; ++i) t2[i] = add2(t2[i], splat2(-delta));
      }
#pragma unroll
      for (int c = 0; c < 64; ++c) t[c] = ex2_approx(t[c]);
      if (half == 0) wait_pv();
      if (!alive) break;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(t[32 * g + 2 * i], t[32 * g + 2 * i + 1]);
        tmem_st16(tbase + lane_base + col_p + 32 * half + 16 * g, pk);
      }
      // this half of P is in TMEM: signal the MMA thread first (half 0 lets
      // the first half of PV run while the second half of P is computed),
      // then add up the row sum, which nothing waits for
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(half == 0 ? &bars.p_half[X] : &bars.p_full[X]);
      psum += sum64(t);
    }
    if (!alive) {
      tmem_wait_st();
      continue;  // leave at the next tile's vote, with the group
    }
    l_sum += psum;
  }

  // ------------------------------------------------------------- epilogue
  gbase += cnt;
  if (alive && cnt > 0) {
    alive = mbar_wait(&bars.o_final[X], nfin & 1, abort, a.status, a.wait_cycles);
    ++nfin;
    tc_fence_after();
  }
  // TMEM loads are warp-collective: every lane takes part, rows past L
  // included; only the stores depend on the row.
  if (__all_sync(0xffffffffu, alive)) {
    // a row without a visible key has l_sum = 0: out 0 and lse -inf, unless
    // the caller promised there is none (rows_safe), which drops this guard
    const bool live = (a.rows_safe || l_sum > 0.0f) && cnt > 0;
    const float inv = live ? 1.0f / l_sum : 0.0f;
    const int64_t orow_off = b * a.o_stride[0] + h * a.o_stride[1] + static_cast<int64_t>(row_ok ? grow : 0) * a.o_stride[2];
    const int64_t rid = (static_cast<int64_t>(b) * a.Hq + h) * a.L + grow;
    if (row_ok && a.lse) a.lse[rid] = live ? (m_ref + log2f(l_sum)) * kLn2 : -INFINITY;
    if (row_ok && a.max_scores) a.max_scores[rid] = m_true * kLn2;
    // O comes out of TMEM 64 columns per wait (four loads in flight)
#pragma unroll
    for (int cb = 0; cb < D / 64; ++cb) {
      float o64[64];
      if (cnt > 0) {
        tmem_load64(tbase + lane_base + col_o + cb * 64, o64);
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) o64[i] = 0.0f;
      }
#pragma unroll
      for (int c = 4 * cb; c < 4 * cb + 4; ++c) {
        const uint32_t* rr = reinterpret_cast<const uint32_t*>(o64) + 16 * (c - 4 * cb);
        if (row_ok) {
          if (a.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow_off + c * 16);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = live ? make_float4(__uint_as_float(rr[4 * i]) * inv, __uint_as_float(rr[4 * i + 1]) * inv,
                                          __uint_as_float(rr[4 * i + 2]) * inv, __uint_as_float(rr[4 * i + 3]) * inv)
                            : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          } else {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pk[i] = live ? pack_bf16x2(__uint_as_float(rr[2 * i]) * inv, __uint_as_float(rr[2 * i + 1]) * inv) : 0u;
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow_off + c * 16);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
    }
  }
  return alive;
}

template <int D, int SCORE>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ FwdArgs a, const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Barriers bars;
  __shared__ float s_pos[2][2][kTile];  // per group: slope * position of the tile's keys
  __shared__ int s_doc[2][2][kTile];    // per group: document ids of the tile's keys
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;  // Q_A, Q_B
  uint8_t* sK = sQ + 2 * C::kTileBytes;
  uint8_t* sV = sK + NS * C::kTileBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &bars.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 2);  // the QK commit + the MMA thread's tile-info arrive
      mbar_init(&bars.p_full[i], 4);
      mbar_init(&bars.p_half[i], 4);
      mbar_init(&bars.s_free[i], 4);
      mbar_init(&bars.o_done[i], 1);
      mbar_init(&bars.o_final[i], 1);
    }
    mbar_init(&bars.mma_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.clc_full[i], 1);   // the producer's arrive with the 16-byte expectation
      mbar_init(&bars.clc_empty[i], 9);  // the MMA thread + 8 softmax warps
    }
    bars.abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    // One ring position u per union tile, counted over all of the CTA's
    // items; Q of the next item is loaded as soon as the current item's last
    // QK has completed (q_empty), while its last tiles are still in flight.
    // This thread also makes the launch-control requests: request r, made
    // just before the last tile of item r is loaded (a few tiles before the
    // item ends, so that the next item goes to the SM that frees up first),
    // names item r + 1.
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      int u = 0, nq = 0, issued_k = 0, issued_v = 0, requests = 0;
      bool ok = true;
      int cx = blockIdx.x, cy = blockIdx.y, cz = blockIdx.z;
      for (int r = 0; ok && !*abort; ++r) {
        const Item itm = item_of(a, cx, cy, cz);
        UnionIter it;
        it.init(a, itm.row_a, itm.has_b);
        int n;
        uint32_t flags;
        bool any = it.next(n, flags);  // false: no tile for either query tile
        if (any && nq > 0 && !mbar_wait(&bars.q_empty, (nq - 1) & 1, abort, a.status, a.wait_cycles)) break;
        if (any) {
          mbar_expect_tx(&bars.q_full, (itm.has_b ? 2 : 1) * C::kTileBytes);
          for (int c = 0; c < C::kBoxes; ++c) {
            tma_load_4d(sQ + c * (kTile * 128), &map_q, &bars.q_full, c * 64, itm.mtA * kTile, itm.h, itm.b);
            if (itm.has_b)
              tma_load_4d(sQ + C::kTileBytes + c * (kTile * 128), &map_q, &bars.q_full, c * 64, itm.mtB * kTile, itm.h,
                          itm.b);
          }
          ++nq;
        }
        // request r, into answer slot r & 1 once its previous answer is read,
        // is made just before the item's last tile is loaded
        bool requested = false;
        auto request = [&]() -> bool {
          if (r >= 2 && !mbar_wait(&bars.clc_empty[r & 1], ((r >> 1) - 1) & 1, abort, a.status, a.wait_cycles))
            return false;
          mbar_expect_tx(&bars.clc_full[r & 1], 16);
          clc_try_cancel(&bars.clc_resp[r & 1], &bars.clc_full[r & 1]);
          requests = r + 1;
          requested = true;
          return true;
        };
        for (; any; ++u) {
          int n_nxt = 0;
          uint32_t f_nxt = 0;
          const bool have_nxt = it.next(n_nxt, f_nxt);
          const int s = u % NS;
          const uint32_t round = u / NS;
          if (*abort || (!have_nxt && !request()) ||
              (u >= NS && !mbar_wait(&bars.k_empty[s], (round - 1) & 1, abort, a.status, a.wait_cycles))) {
            ok = false;
            break;
          }
          // a paged pool is read in two 64-key boxes per tile, each from its
          // own page (the swizzle follows the smem address, so the halves
          // land exactly as one 128-row box would)
          int pg0 = itm.b, pg1 = itm.b, row0 = n * kTile, row1 = n * kTile + 64;
          if (a.page_table) {
            pg0 = cache_page(a.page_table, a.pages_per_seq, a.page_size, a.num_pages, a.status, itm.b, n * kTile);
            pg1 = cache_page(a.page_table, a.pages_per_seq, a.page_size, a.num_pages, a.status, itm.b, n * kTile + 64);
            row0 = (n * kTile) % a.page_size;
            row1 = (n * kTile + 64) % a.page_size;
          }
          mbar_expect_tx(&bars.k_full[s], C::kTileBytes);
          for (int c = 0; c < C::kBoxes; ++c) {
            uint8_t* dst = sK + s * C::kTileBytes + c * (kTile * 128);
            if (a.page_table) {
              tma_load_4d(dst, &map_k, &bars.k_full[s], c * 64, row0, itm.hk, pg0);
              tma_load_4d(dst + 64 * 128, &map_k, &bars.k_full[s], c * 64, row1, itm.hk, pg1);
            } else {
              tma_load_4d(dst, &map_k, &bars.k_full[s], c * 64, n * kTile, itm.hk, itm.b);
            }
          }
          issued_k = u + 1;
          if (u >= NS && !mbar_wait(&bars.v_empty[s], (round - 1) & 1, abort, a.status, a.wait_cycles)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&bars.v_full[s], C::kTileBytes);
          for (int c = 0; c < C::kBoxes; ++c) {
            uint8_t* dst = sV + s * C::kTileBytes + c * (kTile * 128);
            if (a.page_table) {
              tma_load_4d(dst, &map_v, &bars.v_full[s], c * 64, row0, itm.hk, pg0);
              tma_load_4d(dst + 64 * 128, &map_v, &bars.v_full[s], c * 64, row1, itm.hk, pg1);
            } else {
              tma_load_4d(dst, &map_v, &bars.v_full[s], c * 64, n * kTile, itm.hk, itm.b);
            }
          }
          issued_v = u + 1;
          n = n_nxt;
          flags = f_nxt;
          any = have_nxt;
        }
        if (!ok) break;
        if (!requested && !request()) break;  // an item without tiles
        // the next item, if request r cancelled a CTA
        if (!mbar_wait(&bars.clc_full[r & 1], (r >> 1) & 1, abort, a.status, a.wait_cycles)) break;
        if (!clc_query(&bars.clc_resp[r & 1], cx, cy, cz)) break;
      }
      // Drain on every path: each copy and request this thread issued lands
      // before it leaves, so the CTA never exits with one in flight, even
      // when another warp gives up after this loop has ended.  Only the last
      // request, the last Q and the last NS of each ring can be pending
      // (earlier ones were waited on before reuse); on the normal path they
      // have landed already.
      volatile int never = 0;
      if (requests > 0) mbar_wait(&bars.clc_full[(requests - 1) & 1], ((requests - 1) >> 1) & 1, &never, nullptr);
      if (nq > 0) mbar_wait(&bars.q_full, (nq - 1) & 1, &never, nullptr);
      for (int j = (issued_k > NS ? issued_k - NS : 0); j < issued_k; ++j)
        mbar_wait(&bars.k_full[j % NS], (j / NS) & 1, &never, nullptr);
      for (int j = (issued_v > NS ? issued_v - NS : 0); j < issued_v; ++j)
        mbar_wait(&bars.v_full[j % NS], (j / NS) & 1, &never, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, D, 0, 1);
      // Base smem descriptors, built once; per-MMA descriptors only add the
      // (address >> 4) offset of the K step or stage to the start-address
      // field, which keeps the issue path short.
      const uint64_t dq0 = umma_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk0 = umma_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = umma_desc_sw128(smem_u32(sV), kTile * 128, 1024);
      constexpr uint32_t kTileStep = C::kTileBytes >> 4;
      // counters over all of the CTA's items: ring position, P tiles consumed,
      // QK tiles issued and S tiles read out per group, Q tiles loaded
      int u = 0, nq = 0;
      int pcnt[2] = {0, 0}, qcnt[2] = {0, 0}, freed[2] = {0, 0};
      bool acc[2] = {false, false};
      auto issue_qk = [&](int X, int s, int n, uint32_t flags) {
        // publish the tile index and class for the softmax group (released by
        // this thread's arrive; the phase completes with the MMA commit below)
        bars.info[X][qcnt[X] & 1] = n | ((flags & (X == 0 ? kFullA : kFullB)) ? kInfoFull : 0);
        ++qcnt[X];
        mbar_arrive(&bars.s_full[X]);
        const uint64_t dq = dq0 + X * kTileStep, dk = dk0 + s * kTileStep;
        const uint32_t d_tmem = tbase + 256u * X;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * (kTile * 128) + (kk & 3) * 32) >> 4;
          umma_ss(d_tmem, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars.s_full[X]);
      };
      // O_X += P_X V (the item's first PV of a group overwrites O_X); head
      // dim 64 has P and O in columns of their own and signals o_done
      auto issue_pv = [&](int X, int s) -> bool {
        const uint64_t dv = dv0 + s * kTileStep;
        const uint32_t o_tmem = tbase + 256u * X + (D == 64 ? 192u : 128u);
        const uint32_t p_tmem = tbase + 256u * X + (D == 64 ? 128u : 0u);
        const uint32_t acc0 = acc[X] ? 1u : 0u;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          // keys 64 hf .. 64 hf + 63 once their P is written
          if (!mbar_wait(hf == 0 ? &bars.p_half[X] : &bars.p_full[X], pcnt[X] & 1, abort, a.status, a.wait_cycles)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * hf; kk < 4 * hf + 4; ++kk)
            umma_ts(o_tmem, p_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_pv, kk > 0 ? 1u : acc0);
        }
        if (D == 64) umma_commit(&bars.o_done[X]);
        acc[X] = true;
        ++pcnt[X];
        return true;
      };
      // head dim 64: a group's QK waits until its softmax has read the
      // previous S (s_free), possibly of the previous item
      auto qk_after_free = [&](int X, int s, int n, uint32_t flags) -> bool {
        if (D == 64 && qcnt[X] > 0) {
          if (!mbar_wait(&bars.s_free[X], freed[X] & 1, abort, a.status, a.wait_cycles)) return false;
          ++freed[X];
          tc_fence_after();
        }
        issue_qk(X, s, n, flags);
        return true;
      };
      bool ok = true;
      int cx = blockIdx.x, cy = blockIdx.y, cz = blockIdx.z;
      for (int r = 0; ok && !*abort; ++r) {
        const Item itm = item_of(a, cx, cy, cz);
        UnionIter it;
        it.init(a, itm.row_a, itm.has_b);
        int n_cur, n_nxt = 0;
        uint32_t f_cur, f_nxt = 0;
        bool have_cur = it.next(n_cur, f_cur);  // false: no tile for either query tile
        acc[0] = acc[1] = false;
        if (have_cur) {
          ok = mbar_wait(&bars.q_full, nq & 1, abort, a.status, a.wait_cycles);
          ++nq;
          if (ok) ok = mbar_wait(&bars.k_full[u % NS], (u / NS) & 1, abort, a.status, a.wait_cycles);
          tc_fence_after();
          if (ok && (f_cur & kInA)) ok = qk_after_free(0, u % NS, n_cur, f_cur);
          if (ok && (f_cur & kInB)) ok = qk_after_free(1, u % NS, n_cur, f_cur);
          if (ok) umma_commit(&bars.k_empty[u % NS]);
        }
        for (; ok && have_cur; ++u) {
          const int s = u % NS, s1 = (u + 1) % NS;
          const bool have_nxt = it.next(n_nxt, f_nxt);
          // every QK of the item is issued: Q may be reloaded once they are done
          if (!have_nxt) umma_commit(&bars.q_empty);
          bool k_ready = false, v_ready = false;
          if constexpr (D == 64) {
            // S, P and O in separate columns: the next tile's QK of a group
            // goes in as soon as its softmax has read S, ahead of this
            // tile's PV, so the next S is ready when the softmax needs it.
            for (int X = 0; X < 2 && ok; ++X) {
              const uint32_t in_x = X == 0 ? kInA : kInB;
              if (have_nxt && (f_nxt & in_x)) {
                if (!k_ready) {
                  ok = mbar_wait(&bars.k_full[s1], ((u + 1) / NS) & 1, abort, a.status, a.wait_cycles);
                  tc_fence_after();
                  k_ready = true;
                }
                if (ok) ok = qk_after_free(X, s1, n_nxt, f_nxt);
              }
              if (ok && (f_cur & in_x)) {
                if (!v_ready) {
                  ok = mbar_wait(&bars.v_full[s], (u / NS) & 1, abort, a.status, a.wait_cycles);
                  tc_fence_after();
                  v_ready = true;
                }
                if (ok) ok = issue_pv(X, s);
              }
            }
          } else {
            // P_X shares the S columns: PV_X of this tile, then QK_X of the next
            ok = mbar_wait(&bars.v_full[s], (u / NS) & 1, abort, a.status, a.wait_cycles);
            tc_fence_after();
            for (int X = 0; X < 2 && ok; ++X) {
              const uint32_t in_x = X == 0 ? kInA : kInB;
              if (f_cur & in_x) ok = issue_pv(X, s);
              if (ok && have_nxt && (f_nxt & in_x)) {
                if (!k_ready) {
                  ok = mbar_wait(&bars.k_full[s1], ((u + 1) / NS) & 1, abort, a.status, a.wait_cycles);
                  tc_fence_after();
                  k_ready = true;
                }
                if (ok) issue_qk(X, s1, n_nxt, f_nxt);
              }
            }
          }
          if (!ok) break;
          // every union tile is some group's tile, and so is the next one
          umma_commit(&bars.v_empty[s]);
          if (have_nxt) {
            // K_{u+1} is listed for neither group's next QK only if a group
            // skips it; it still has to be consumed before its slot is reused
            if (!k_ready && !mbar_wait(&bars.k_full[s1], ((u + 1) / NS) & 1, abort, a.status, a.wait_cycles)) {
              ok = false;
              break;
            }
            umma_commit(&bars.k_empty[s1]);
          }
          have_cur = have_nxt;
          n_cur = n_nxt;
          f_cur = f_nxt;
        }
        // the item's O of each group with tiles is complete once these land
        if (!ok) break;
        if (acc[0]) umma_commit(&bars.o_final[0]);
        if (acc[1]) umma_commit(&bars.o_final[1]);
        // the next item, if request r cancelled a CTA
        if (!mbar_wait(&bars.clc_full[r & 1], (r >> 1) & 1, abort, a.status, a.wait_cycles)) break;
        const bool more = clc_query(&bars.clc_resp[r & 1], cx, cy, cz);
        mbar_arrive(&bars.clc_empty[r & 1]);
        if (!more) break;
      }
      // every MMA issued above completes before TMEM is released
      umma_commit(&bars.mma_done);
      volatile int never = 0;
      mbar_wait(&bars.mma_done, 0, &never, nullptr);
    }
  } else {
    // -------------------------------------------------------------- softmax
    // warps 2-5: tile A, warps 6-9: tile B; warp % 4 is the TMEM lane quadrant.
    // The group's four warps agree at each item whether to go on (a warp
    // that gave up inside an item leaves with its group).
    const int X = (warp - 2) >> 2;
    int gbase = 0, nfin = 0;
    bool go = true;
    int cx = blockIdx.x, cy = blockIdx.y, cz = blockIdx.z;
    for (int r = 0; named_bar_and(1 + X, 128, go); ++r) {
      const Item itm = item_of(a, cx, cy, cz);
      const bool alive = softmax_group<D, SCORE>(a, bars, s_pos[X], s_doc[X], X, X == 0 ? itm.mtA : itm.mtB, itm.h,
                                                 itm.b, itm.S_b, itm.row_a, itm.has_b, tbase, gbase, nfin);
      // the next item, if request r cancelled a CTA (the answer is the same
      // for all four warps, so they go on or stop together)
      bool more = false;
      if (alive && __all_sync(0xffffffffu, mbar_wait(&bars.clc_full[r & 1], (r >> 1) & 1, abort, a.status, a.wait_cycles))) {
        more = clc_query(&bars.clc_resp[r & 1], cx, cy, cz);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.clc_empty[r & 1]);
      }
      go = alive && more;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

template <int D, int SCORE>
cudaError_t launch_one(const FwdArgs& a, const Sm100Maps& maps, cudaStream_t stream) {
  auto kern = fwd_sm100_kernel<D, SCORE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  // one CTA per work item; the CTAs that start first (one per SM: shared
  // memory and TMEM allow no second) take over the launches of the rest
  dim3 grid(a.Hq, a.B, (a.bm.Mb + 1) / 2);
  kern<<<grid, kThreads, Cfg<D>::kSmemBytes, stream>>>(a, maps.q, maps.k, maps.v);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const FwdArgs& a, const Sm100Maps& maps, cudaStream_t stream) {
  switch (a.score.kind) {
    case FA_SCORE_NONE: return launch_one<D, FA_SCORE_NONE>(a, maps, stream);
    case FA_SCORE_SOFTCAP: return launch_one<D, FA_SCORE_SOFTCAP>(a, maps, stream);
    case FA_SCORE_ALIBI: return launch_one<D, FA_SCORE_ALIBI>(a, maps, stream);
    default: return launch_one<D, FA_SCORE_CAP_THEN_BIAS>(a, maps, stream);
  }
}

}  // namespace

cudaError_t launch_fwd_sm100(const FwdArgs& a, const Sm100Maps& maps, cudaStream_t stream) {
  return a.E == 64 ? launch_d<64>(a, maps, stream) : launch_d<128>(a, maps, stream);
}

}  // namespace fa
