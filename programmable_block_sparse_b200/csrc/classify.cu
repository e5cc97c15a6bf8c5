// BlockMask construction on the GPU: classify every (b, m, n) tile as empty,
// full or partial and write the ordered index lists.
//
// What is computed follows "PyTorch Flex Attention complete guide" (2kiu.com)
// sections 3.1 (a block counts as sparse only when every element in it is
// masked), 3.2 (ordered per-row index lists) and 4.1 (dense mask, per-block
// reduction, full blocks kept apart from partial ones), and the tile classes of
// "flexattention-score-mod-block-mask" (charlestar.github.io), section
// "mask_mod defines legal connections, BlockMask defines block work".
//
// How: no dense (L, S) temporary.  One CTA per (b, m) row of tiles (and per
// head for a rule that reads the head); each warp classifies whole tiles.
// For the interval-shaped rules (none, causal, sliding window with sinks,
// prefix-LM, chunked) every query row sees a union of at most two key
// intervals, so a tile is classified from per-row
// intersection counts (BM work per tile instead of BM x BN).  The document
// rule counts the same way over runs of equal document id (see
// classify_tile_document).  A composed rule (FA_MASK_PROGRAM) is decided per
// tile by three-valued logic over the tile's bounds, exact where it says all
// or nothing, and otherwise by evaluating the tile's cells 32 keys at a time;
// when it reads the query head, every head row is classified for its head.
#include "common.cuh"
#include "launch.h"
#include "mods.cuh"

namespace fa {

namespace {

// threads per CTA: 16 warps for composed rules, 32 for the other families,
// so that a row of tiles is taken in few rounds (a tile's classification is
// a chain of dependent loads)
constexpr int kClassifyThreads = 512;
constexpr int kClassifyThreadsWide = 1024;
enum : uint8_t { kEmpty = 0, kPartial = 1, kFull = 2 };

// |[lo, hi] intersect [c0, c1]| for inclusive bounds.
__device__ __forceinline__ int overlap(int lo, int hi, int c0, int c1) {
  int a = lo > c0 ? lo : c0;
  int b = hi < c1 ? hi : c1;
  return b >= a ? b - a + 1 : 0;
}

// Number of visible keys in [c0, c1] (inclusive, c1 < S) for logical query q:
// |A| + |B| - |A and B| over the two visible spans.
__device__ __forceinline__ int visible_count(const MaskParams& m, int q, int c0, int c1, int S_b) {
  const KeySpans sp = visible_spans(m, q, S_b);
  return overlap(sp.a0, sp.a1, c0, c1) + overlap(sp.b0, sp.b1, c0, c1) -
         overlap(max(sp.a0, sp.b0), min(sp.a1, sp.b1), c0, c1);
}

__device__ uint8_t classify_tile_intervals(const MaskParams& m, int r0, int r1, int c0, int c1, int L, int S_b) {
  const int lane = threadIdx.x & 31;
  const int width = c1 - c0 + 1;
  bool all_full = true, any_vis = false;
  for (int r = r0 + lane; r <= r1; r += 32) {
    int n = visible_count(m, query_pos(r, L, S_b), c0, c1, S_b);
    all_full &= (n == width);
    any_vis |= (n > 0);
  }
  all_full = __all_sync(0xffffffffu, all_full);
  any_vis = __any_sync(0xffffffffu, any_vis);
  return all_full ? kFull : (any_vis ? kPartial : kEmpty);
}

// Document rule: key kv is visible to query q when kv <= q, kv < S_b and
// doc[kv] == doc[q].  The tile's columns [c0, chi] (chi = last in-range key)
// are cut into runs of equal document id (at most BN <= 128 of them, found
// with ballots and written to this warp's slice of shared memory); a row's
// visible count is the summed overlap of [c0, min(q, chi)] with the runs whose
// id equals doc[q].  Exact for any id layout; a packed batch of documents has
// one or two runs per tile, so a tile costs about BM / 32 steps per lane.
__device__ uint8_t classify_tile_document(const MaskParams& m, int b, int r0, int r1, int c0, int c1, int L, int S,
                                          int S_b, int* run_a, int* run_id) {
  const int lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  const int* d = m.doc_id + static_cast<int64_t>(m.doc_batch > 1 ? b : 0) * S;
  const int chi = min(c1, S_b - 1);
  int nr = 0;
  int prev_last = 0;
  for (int base = c0; base <= chi; base += 32) {
    const int c = base + lane;
    const bool valid = c <= chi;
    const int v = valid ? __ldg(d + c) : 0;
    int prev = __shfl_up_sync(full, v, 1);
    if (lane == 0) prev = prev_last;
    const bool start = valid && (c == c0 || v != prev);
    const unsigned bal = __ballot_sync(full, start);
    if (start) {
      const int idx = nr + __popc(bal & ((1u << lane) - 1u));
      run_a[idx] = c;
      run_id[idx] = v;
    }
    nr += __popc(bal);
    prev_last = __shfl_sync(full, v, 31);
  }
  if (lane == 0) run_a[nr] = chi + 1;
  __syncwarp();
  const int width = c1 - c0 + 1;
  bool all_full = true, any_vis = false;
  for (int r = r0 + lane; r <= r1; r += 32) {
    const int q = query_pos(r, L, S_b);
    const int hi = min(q, chi);
    int cnt = 0;
    if (hi >= c0) {
      const int dq = __ldg(d + q);
      for (int k = 0; k < nr; ++k) {
        const int a = run_a[k];
        if (a > hi) break;
        if (run_id[k] == dq) cnt += min(run_a[k + 1] - 1, hi) - a + 1;
      }
    }
    all_full &= (cnt == width);
    any_vis |= (cnt > 0);
  }
  all_full = __all_sync(full, all_full);
  any_vis = __any_sync(full, any_vis);
  __syncwarp();  // run_a / run_id are rewritten for the warp's next tile
  return all_full ? kFull : (any_vis ? kPartial : kEmpty);
}

// Composed rule: rows [r0, r1] x keys [c0, c1] (inclusive, in range) of head
// h.  Keys >= S_b are invisible; the caller has handled c0 >= S_b.
__device__ uint8_t classify_tile_program(const MaskParams& m, int b, int h, int r0, int r1, int c0, int c1, int L,
                                         int S, int S_b, int* doc_keys) {
  const int lane = threadIdx.x & 31;
  const unsigned full = 0xffffffffu;
  const int chi = min(c1, S_b - 1);  // last key that can be visible
  const int v = program_box(m, h, query_pos(r0, L, S_b), query_pos(r1, L, S_b), c0, chi);
  if (v == 0) return kEmpty;
  if (v == 1) return chi == c1 ? kFull : kPartial;
  // mixed or undecided: count visible keys row by row, 32 keys per word
  const int* d = m.reads_doc ? m.doc_id + static_cast<int64_t>(m.doc_batch > 1 ? b : 0) * S : nullptr;
  if (d) {
    for (int c = c0 + lane; c <= c1; c += 32) doc_keys[c - c0] = __ldg(d + c);
    __syncwarp();
  }
  const int width = c1 - c0 + 1;
  bool all_full = true, any_vis = false;
  for (int r = r0 + lane; r <= r1; r += 32) {
    const int q = query_pos(r, L, S_b);
    const int dq = (d && q >= 0 && q < S) ? __ldg(d + q) : 0;
    int cnt = 0;
    for (int base = c0; base <= c1; base += 32) {
      uint32_t same = 0xFFFFFFFFu;
      if (d) {
        same = 0u;
        const int nk = min(32, c1 - base + 1);
        for (int i = 0; i < nk; ++i) same |= (doc_keys[base - c0 + i] == dq ? 1u : 0u) << i;
        if (q < 0 || q >= S) same = 0u;
      }
      const uint32_t bits = program_bits(m, h, q, base, same) & span_bits(-1, chi - base) & span_bits(-1, c1 - base);
      cnt += __popc(bits);
    }
    all_full &= (cnt == width);
    any_vis |= (cnt > 0);
  }
  all_full = __all_sync(full, all_full);
  any_vis = __any_sync(full, any_vis);
  __syncwarp();  // doc_keys is rewritten for the warp's next tile
  return all_full ? kFull : (any_vis ? kPartial : kEmpty);
}

// One instantiation per family of rules, so that each launch carries only the
// code its rule needs (the kernel runs once per call, its instructions are
// fetched cold): kIntervals for the interval-shaped rules, kDocument,
// kProgram for composed rules.
enum RuleFamily { kIntervals = 0, kDocument = 1, kProgram = 2 };

template <int FAMILY>
__global__ void __launch_bounds__(FAMILY == kProgram ? kClassifyThreads : kClassifyThreadsWide)
    classify_kernel(ClassifyArgs a) {
  constexpr int kWarps = (FAMILY == kProgram ? kClassifyThreads : kClassifyThreadsWide) / 32;
  extern __shared__ uint8_t cls[];
  __shared__ int s_run_a[FAMILY == kDocument ? kWarps : 1][129];
  __shared__ int s_run_id[FAMILY == kIntervals ? 1 : kWarps][128];
  const int mt = blockIdx.x;
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int S_b = seq_len_b(a.mask, b, a.S);
  const int r0 = mt * a.BM;
  const int r1 = min(a.L, r0 + a.BM) - 1;          // inclusive
  const int q_hi = query_pos(r1, a.L, S_b);         // largest logical query position
  const bool causal_family = a.mask.kind == FA_MASK_CAUSAL || a.mask.kind == FA_MASK_SLIDING_WINDOW ||
                             a.mask.kind == FA_MASK_DOCUMENT || a.mask.kind == FA_MASK_CHUNKED;

  // a rule that reads the query head is classified for each head row (one
  // CTA per head: blockIdx.z); any other is classified once and its lists
  // written to every head row
  const bool per_head = a.mask.kind == FA_MASK_PROGRAM && a.mask.reads_head && a.H > 1;
  __shared__ int s_counts[2];
  {
    const int hc = per_head ? static_cast<int>(blockIdx.z) : 0;
    for (int n = warp; n < a.Nb; n += nwarps) {
      const int c0 = n * a.BN;
      const int c1 = min(a.S, c0 + a.BN) - 1;        // inclusive
      uint8_t k;
      if (c0 >= S_b || (causal_family && c0 > q_hi)) {
        k = kEmpty;
      } else if constexpr (FAMILY == kDocument) {
        k = classify_tile_document(a.mask, b, r0, r1, c0, c1, a.L, a.S, S_b, s_run_a[warp], s_run_id[warp]);
      } else if constexpr (FAMILY == kProgram) {
        k = classify_tile_program(a.mask, b, hc, r0, r1, c0, c1, a.L, a.S, S_b, s_run_id[warp]);
      } else {
        k = classify_tile_intervals(a.mask, r0, r1, c0, c1, a.L, S_b);
      }
      if (lane == 0) cls[n] = k;
    }
    __syncthreads();

    // Ordered lists: warp 0 scans the classes 32 tiles at a time.
    const int h_lo = per_head ? hc : 0, h_hi = per_head ? hc + 1 : a.H;
    if (warp == 0) {
      int nfull = 0, npart = 0;
      for (int base = 0; base < a.Nb; base += 32) {
        const int n = base + lane;
        const uint8_t k = n < a.Nb ? cls[n] : kEmpty;
        const unsigned fb = __ballot_sync(0xffffffffu, k == kFull);
        const unsigned pb = __ballot_sync(0xffffffffu, k == kPartial);
        const unsigned below = (1u << lane) - 1u;
        for (int h = h_lo; h < h_hi; ++h) {
          const int64_t row = (static_cast<int64_t>(b) * a.H + h) * a.Mb + mt;
          if (k == kFull) a.full_kv_indices[row * a.Nb + nfull + __popc(fb & below)] = n;
          if (k == kPartial) a.kv_indices[row * a.Nb + npart + __popc(pb & below)] = n;
        }
        nfull += __popc(fb);
        npart += __popc(pb);
      }
      if (lane == 0) {
        s_counts[0] = nfull;
        s_counts[1] = npart;
        for (int h = h_lo; h < h_hi; ++h) {
          const int64_t row = (static_cast<int64_t>(b) * a.H + h) * a.Mb + mt;
          a.full_kv_num_blocks[row] = nfull;
          a.kv_num_blocks[row] = npart;
        }
      }
    }
    __syncthreads();
    const int nfull = s_counts[0], npart = s_counts[1];
    for (int h = h_lo; h < h_hi; ++h) {
      const int64_t row = (static_cast<int64_t>(b) * a.H + h) * a.Mb + mt;
      for (int i = threadIdx.x; i < a.Nb; i += blockDim.x) {
        if (i >= nfull) a.full_kv_indices[row * a.Nb + i] = 0;
        if (i >= npart) a.kv_indices[row * a.Nb + i] = 0;
      }
    }
  }
}

}  // namespace

cudaError_t launch_classify(const ClassifyArgs& a, cudaStream_t stream) {
  const bool per_head = a.mask.kind == FA_MASK_PROGRAM && a.mask.reads_head && a.H > 1;
  dim3 grid(a.Mb, a.B, per_head ? a.H : 1);
  size_t smem = (static_cast<size_t>(a.Nb) + 15) & ~static_cast<size_t>(15);
  auto kern = a.mask.kind == FA_MASK_DOCUMENT  ? classify_kernel<kDocument>
              : a.mask.kind == FA_MASK_PROGRAM ? classify_kernel<kProgram>
                                               : classify_kernel<kIntervals>;
  // static shared memory: 33 KB in the document family, 9 KB in the composed
  if (smem + (a.mask.kind == FA_MASK_DOCUMENT ? 33 * 1024 : 9 * 1024) > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  kern<<<grid, a.mask.kind == FA_MASK_PROGRAM ? kClassifyThreads : kClassifyThreadsWide, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fa
