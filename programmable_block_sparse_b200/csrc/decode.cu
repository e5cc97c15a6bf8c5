// Split-KV decode for short queries against long KV caches, and the
// log-sum-exp combination of its partial results.
//
// The computation is the forward definition of "flexattention-score-mod-
// block-mask" (charlestar.github.io), "What one connection goes through", with
// logical query positions q = i + (S_b - L) ("At decode, q_idx = 0 is not
// position 0"; bottom-right alignment, "Causal Mask" (quant67.com) section 4).
// Only the tiles the BlockMask lists are read.  A decode step streams the whole
// valid cache once, so the kernels are built around HBM bandwidth.  Both
// take, per CTA, the query rows of up to 16 (query head, position) pairs that
// share one KV head (GQA: the group's heads reuse every K/V byte it loads)
// against a contiguous run of the row's listed tiles; the grid is (split,
// KV head x head chunk, batch).
//
//   decode_tc_kernel (head dim 128, tiles of 128 keys): tcgen05 products with
//             the keys on the 128-row M side and the query rows as N = 16,
//             S^T and O^T in TMEM, P through shared memory; one thread per
//             key runs the score rule, mask and softmax (see below).
//   decode_kernel (head dim 64, or tiles of 64 keys): warp 0 streams 64-key
//             K / V sub-tiles by TMA; warps 1-4 each take 16 of every 64 keys
//             with mma.sync m16n8k16 and merge (max, sum, O) through shared
//             memory at the end.
//   output    one split: out and lse directly.  Several splits: normalised O,
//             lse and the row maximum per split into the workspace, then
//             combine_kernel merges them: lse = ln sum_s e^{lse_s},
//             o = sum_s e^{lse_s - lse} o_s, max_scores = max_s m_s.
//   abort     when a bounded wait gives up, the CTA stops issuing work,
//             writes nothing, and drains its own copies and MMAs.
#include <math.h>

#include "common.cuh"
#include "fastmath.cuh"
#include "launch.h"
#include "mods.cuh"

namespace fa {

namespace {

constexpr int kDecThreads = 160;
constexpr int kSub = 64;        // keys per pipeline stage
constexpr int kStagesDec = 3;
constexpr int kRows = 16;       // query rows per CTA (one m16 fragment)
constexpr float kLog2eD = 1.4426950408889634f;
constexpr float kLn2D = 0.6931471805599453f;
constexpr float kRescaleThresholdD = 8.0f;  // log2 units
// Start of the running maximum: finite and below any real score (log2
// units), so that keys hidden from a row give P = 2^-inf = 0 with no test of
// the maximum, and the first visible key always moves it.
constexpr float kNoKeyMaxD = -1.0e30f;

template <int D>
struct DecCfg {
  static constexpr int kBoxBytes = kSub * 128;            // 64 keys x 64 columns of bf16
  static constexpr int kTileBytes = kSub * D * 2;         // one K or V sub-tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kSmemBytes = kStagesDec * kStageBytes + 1024;
};

struct DecBars {
  uint64_t full[kStagesDec], empty[kStagesDec];
  int abort;
};

__device__ __forceinline__ float ex2f_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of (row, 8-element chunk) inside a 128-byte-swizzled box of
// 64 rows x 64 bf16, as written by TMA.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ int list_tile(const FwdArgs& a, int64_t brow, int nfull, int j) {
  return j < nfull ? __ldg(a.bm.full_kv_indices + brow * a.bm.Nb + j)
                   : __ldg(a.bm.kv_indices + brow * a.bm.Nb + (j - nfull));
}

template <int D, int SCORE>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_kernel(const FwdArgs a, const DecodePlan p, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, float* ws_o, float* ws_lse, float* ws_max) {
  using C = DecCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ DecBars bars;
  __shared__ float s_m[4][kRows], s_l[4][kRows], s_t[4][kRows];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int head_chunks = (a.G + p.heads_per_cta - 1) / p.heads_per_cta;
  const int hk = blockIdx.y / head_chunks, hc = blockIdx.y % head_chunks;
  const int b = blockIdx.z;
  const int S_b = seq_len_b(a.mask, b, a.S);
  const int bmb = a.bm.B > 1 ? b : 0;
  // a per-head block mask (a head-dependent rule) gives each CTA one query
  // head (the plan sets heads_per_cta = 1), whose row it reads
  const int bmh = a.bm.H > 1 ? hk * a.G + hc * p.heads_per_cta : 0;
  const int64_t brow = (static_cast<int64_t>(bmb) * a.bm.H + bmh) * a.bm.Mb;  // tile row 0
  const int nfull = __ldg(a.bm.full_kv_num_blocks + brow);
  const int ntiles = nfull + __ldg(a.bm.kv_num_blocks + brow);
  const int t0 = split * p.tiles_per_split;
  const int t1 = min(ntiles, t0 + p.tiles_per_split);
  const int subs_per_tile = a.bm.BN / kSub;
  const int nsub = t1 > t0 ? (t1 - t0) * subs_per_tile : 0;
  volatile int* abort = &bars.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesDec; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 4);
    }
    bars.abort = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // rows of this CTA: row rho -> (query head, position)
  auto row_head = [&](int rho) { return hk * a.G + hc * p.heads_per_cta + rho / a.L; };
  auto row_valid = [&](int rho) {
    const int g = hc * p.heads_per_cta + rho / a.L;
    return rho < p.rows_per_cta && rho / a.L < p.heads_per_cta && g < a.G;
  };

  if (warp == 0) {
    if (lane == 0 && nsub > 0) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      int issued = 0;
      for (int u = 0; u < nsub && !*abort; ++u) {
        const int s = u % kStagesDec;
        if (u >= kStagesDec && !mbar_wait(&bars.empty[s], ((u / kStagesDec) - 1) & 1, abort, a.status, a.wait_cycles)) break;
        const int n = list_tile(a, brow, nfull, t0 + u / subs_per_tile);
        const int kv0 = n * a.bm.BN + (u % subs_per_tile) * kSub;
        // dense cache: rows kv0.. of (b, hk); paged: the 64 keys sit in one page
        int row = kv0, outer = b;
        if (a.page_table) {
          outer = cache_page(a.page_table, a.pages_per_seq, a.page_size, a.num_pages, a.status, b, kv0);
          row = kv0 % a.page_size;
        }
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_expect_tx(&bars.full[s], C::kStageBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(st + c * C::kBoxBytes, &map_k, &bars.full[s], c * 64, row, hk, outer);
          tma_load_4d(st + C::kTileBytes + c * C::kBoxBytes, &map_v, &bars.full[s], c * 64, row, hk, outer);
        }
        issued = u + 1;
      }
      // Every copy issued lands before this thread leaves, on every path: a
      // consumer may give up after the loop above has ended, and the CTA must
      // not exit with copies still in flight.  Only the last kStagesDec can
      // be pending (each earlier slot was waited free before its reuse), and
      // on the normal path they have landed already.
      volatile int never = 0;
      for (int u = (issued > kStagesDec ? issued - kStagesDec : 0); u < issued; ++u)
        mbar_wait(&bars.full[u % kStagesDec], (u / kStagesDec) & 1, &never, nullptr);
    }
  } else {
    const int cw = warp - 1;            // consumer warp: keys [16 cw, 16 cw + 16) of each stage
    const int r_lo = lane >> 2;          // fragment rows r_lo and r_lo + 8
    const int quad = lane & 3;
    // Q as A fragments, straight from global memory
    uint32_t qa[D / 16][4];
    {
      const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int rho = r_lo + 8 * half;
        const bool ok = row_valid(rho);
        const __nv_bfloat16* qrow =
            ok ? qb + b * a.q_stride[0] + row_head(rho) * a.q_stride[1] + (rho % a.L) * a.q_stride[2] : qb;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int e = 16 * ks + 2 * quad;
          qa[ks][half] = ok ? *reinterpret_cast<const uint32_t*>(qrow + e) : 0u;
          qa[ks][half + 2] = ok ? *reinterpret_cast<const uint32_t*>(qrow + e + 8) : 0u;
        }
      }
    }
    // per-row constants for the two fragment rows
    int qpos[2], hq[2];
    bool rok[2];
    float slope2[2];
    const int Hs = a.score.slope_heads > 0 ? a.score.slope_heads : a.Hq;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int rho = r_lo + 8 * half;
      rok[half] = row_valid(rho);
      hq[half] = rok[half] ? row_head(rho) : 0;
      qpos[half] = query_pos(rho % a.L, a.L, S_b);
      slope2[half] = distance_slope(hq[half], Hs);
    }
    // score rule constants in log2 units (SCORE is fixed at compile time)
    const float c_in = (SCORE == FA_SCORE_SOFTCAP) ? a.scale / a.score.cap : 0.0f;
    const float c_out = (SCORE == FA_SCORE_SOFTCAP) ? a.score.cap * kLog2eD : a.scale * kLog2eD;
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_run[2] = {kNoKeyMaxD, kNoKeyMaxD}, l_run[2] = {0.0f, 0.0f};
    float m_true[2] = {-INFINITY, -INFINITY};  // exact row maxima (log2 units), for max_scores

    for (int u = 0; u < nsub; ++u) {
      const int s = u % kStagesDec;
      // a warp-uniform result: the lanes leave the loop together or not at all
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.full[s], (u / kStagesDec) & 1, abort, a.status, a.wait_cycles)))
        break;
      const int j = t0 + u / subs_per_tile;
      const bool full = j < nfull;
      const int n = list_tile(a, brow, nfull, j);
      const int kv0 = n * a.bm.BN + (u % subs_per_tile) * kSub;
      const uint32_t sk = smem_u32(smem + s * C::kStageBytes);
      const uint32_t sv = sk + C::kTileBytes;
      // S = Q K^T for keys kv0 + 16 cw + [0, 16)
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int key = 16 * cw + 8 * (mi >> 1) + rr;
        const int e = 16 * ks + 8 * (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(sk + (e >> 6) * C::kBoxBytes + swz(key, (e & 63) >> 3), b0, b1, b2, b3);
        mma_bf16_16816(sc[0], qa[ks], b0, b1);
        mma_bf16_16816(sc[1], qa[ks], b2, b3);
      }
      // score rule, element mask, online softmax (log2 units)
      const bool need_mask = !full || (kv0 + kSub > S_b);
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int half = e >> 1;
          const int kv = kv0 + 16 * cw + 8 * nt + 2 * quad + (e & 1);
          float g;
          if constexpr (SCORE == FA_SCORE_NONE) {
            g = sc[nt][e] * c_out;
          } else if constexpr (SCORE == FA_SCORE_SOFTCAP) {
            g = c_out * tanh_fast(sc[nt][e] * c_in);
          } else if constexpr (SCORE == FA_SCORE_ALIBI) {
            g = fmaf(sc[nt][e], c_out, -slope2[half] * kLog2eD * static_cast<float>(qpos[half] - kv));
          } else {
            g = score_apply<false>(a.score, sc[nt][e] * a.scale, b, qpos[half], kv, a.S, slope2[half]) * kLog2eD;
          }
          const bool vis = rok[half] && (!need_mask || mask_visible(a.mask, b, hq[half], qpos[half], kv, S_b, a.S));
          g = vis ? g : -INFINITY;
          sc[nt][e] = g;
          mx[half] = fmaxf(mx[half], g);
        }
      }
      // The running max moves (and O, l rescale) only when a row's max grows
      // by more than 2^8 or on its first visible key; P then stays below 2^8
      // and O / l is unchanged.  The four lanes of a row share its max, so
      // they decide alike.
      bool grow[2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        mx[half] = fmaxf(mx[half], __shfl_xor_sync(0xffffffffu, mx[half], 1));
        mx[half] = fmaxf(mx[half], __shfl_xor_sync(0xffffffffu, mx[half], 2));
        m_true[half] = fmaxf(m_true[half], mx[half]);
        grow[half] = mx[half] > m_run[half] + kRescaleThresholdD;
      }
      if (__any_sync(0xffffffffu, grow[0] || grow[1])) {
        float alpha[2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          alpha[half] = grow[half] ? ex2f_approx(m_run[half] - mx[half]) : 1.0f;
          if (grow[half]) m_run[half] = mx[half];
          l_run[half] *= alpha[half];
        }
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          o[i][0] *= alpha[0];
          o[i][1] *= alpha[0];
          o[i][2] *= alpha[1];
          o[i][3] *= alpha[1];
        }
      }
      float ps[2] = {0.0f, 0.0f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sc[nt][e] = ex2f_approx(sc[nt][e] - m_run[e >> 1]);
          ps[e >> 1] += sc[nt][e];
        }
#pragma unroll
      for (int half = 0; half < 2; ++half) l_run[half] += ps[half];
      uint32_t pa[4];
      pa[0] = pack_bf16x2(sc[0][0], sc[0][1]);
      pa[1] = pack_bf16x2(sc[0][2], sc[0][3]);
      pa[2] = pack_bf16x2(sc[1][0], sc[1][1]);
      pa[3] = pack_bf16x2(sc[1][2], sc[1][3]);
      // O += P V over the same 16 keys
#pragma unroll
      for (int et = 0; et < D / 16; ++et) {
        const int key = 16 * cw + 8 * (mi & 1) + rr;
        const int ev = 16 * et + 8 * (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(sv + (ev >> 6) * C::kBoxBytes + swz(key, (ev & 63) >> 3), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * et], pa, b0, b1);
        mma_bf16_16816(o[2 * et + 1], pa, b2, b3);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.empty[s]);
    }
    // row sums across the quad
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      l_run[half] += __shfl_xor_sync(0xffffffffu, l_run[half], 1);
      l_run[half] += __shfl_xor_sync(0xffffffffu, l_run[half], 2);
    }
    if (quad == 0) {
      s_m[cw][r_lo] = m_run[0];
      s_m[cw][r_lo + 8] = m_run[1];
      s_l[cw][r_lo] = l_run[0];
      s_l[cw][r_lo + 8] = l_run[1];
      s_t[cw][r_lo] = m_true[0];
      s_t[cw][r_lo + 8] = m_true[1];
    }
    named_bar_sync(1, 128);
    // Every consumer is past its loop.  A consumer that left it early did so
    // because a wait gave up, and *abort was set before that; the producer
    // sets it only while some stage is still unconsumed.  So *abort is now
    // final for this CTA: on an abort, copies may still be landing in the
    // stage buffers the merge below reuses, so write nothing.
    if (*abort) return;
    // merge the four warps: scale each warp's O by 2^(m_w - m) and add in smem
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int rho = r_lo + 8 * half;
      float m = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) m = fmaxf(m, s_m[w][rho]);
      const float f = ex2f_approx(m_run[half] - m);
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o[i][2 * half] *= f;
        o[i][2 * half + 1] *= f;
      }
    }
    // the stage buffers are idle now (every stage was consumed): reuse them
    float* s_o = reinterpret_cast<float*>(smem);  // [kRows][D]
    for (int i = threadIdx.x - 32; i < kRows * D; i += 128) s_o[i] = 0.0f;
    named_bar_sync(1, 128);
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      const int col = 8 * i + 2 * quad;
      atomicAdd(&s_o[r_lo * D + col], o[i][0]);
      atomicAdd(&s_o[r_lo * D + col + 1], o[i][1]);
      atomicAdd(&s_o[(r_lo + 8) * D + col], o[i][2]);
      atomicAdd(&s_o[(r_lo + 8) * D + col + 1], o[i][3]);
    }
    named_bar_sync(1, 128);
    // write: warp cw handles rows 4 cw .. 4 cw + 3, lanes across columns
    for (int rho = 4 * cw; rho < 4 * cw + 4; ++rho) {
      if (!row_valid(rho)) continue;
      const int hqr = row_head(rho), i = rho % a.L;
      float m = -INFINITY, l = 0.0f;
      for (int w = 0; w < 4; ++w) m = fmaxf(m, s_m[w][rho]);
      for (int w = 0; w < 4; ++w) l += s_l[w][rho] * ex2f_approx(s_m[w][rho] - m);
      float top = -INFINITY;
      for (int w = 0; w < 4; ++w) top = fmaxf(top, s_t[w][rho]);
      // a row without a visible key has l = 0: out 0 and lse -inf, unless the
      // caller promised there is none (rows_safe), which drops this guard
      const bool live = a.rows_safe || l > 0.0f;
      const float inv = live ? 1.0f / l : 0.0f;
      const float lse = live ? (m + log2f(l)) * kLn2D : -INFINITY;
      const int64_t row_id = (static_cast<int64_t>(b) * a.Hq + hqr) * a.L + i;
      if (p.splits == 1) {
        const int64_t off = b * a.o_stride[0] + hqr * a.o_stride[1] + i * a.o_stride[2];
        if (a.out_f32) {
          float* orow = static_cast<float*>(a.out) + off;
          for (int c = lane; c < D; c += 32) orow[c] = s_o[rho * D + c] * inv;
        } else {
          __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + off;
          for (int c = lane; c < D; c += 32) orow[c] = __float2bfloat16_rn(s_o[rho * D + c] * inv);
        }
        if (lane == 0 && a.lse) a.lse[row_id] = lse;
        if (lane == 0 && a.max_scores) a.max_scores[row_id] = top * kLn2D;
      } else {
        float* wrow = ws_o + (row_id * p.splits + split) * D;
        for (int c = lane; c < D; c += 32) wrow[c] = s_o[rho * D + c] * inv;
        if (lane == 0) ws_lse[row_id * p.splits + split] = lse;
        if (lane == 0) ws_max[row_id * p.splits + split] = top;
      }
    }
  }
}

// One warp per (b, h, i) row: merge the per-split (o_s, lse_s).
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const FwdArgs a, const DecodePlan p, const float* ws_o,
                                                      const float* ws_lse, const float* ws_max) {
  const int64_t row_id = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(a.B) * a.Hq * a.L;
  if (row_id >= rows) return;
  const int i = static_cast<int>(row_id % a.L);
  const int h = static_cast<int>((row_id / a.L) % a.Hq);
  const int b = static_cast<int>(row_id / (static_cast<int64_t>(a.L) * a.Hq));
  const float* lrow = ws_lse + row_id * p.splits;
  const float* trow = ws_max + row_id * p.splits;
  float m = -INFINITY, top = -INFINITY;
  for (int s = lane; s < p.splits; s += 32) {
    m = fmaxf(m, lrow[s]);
    top = fmaxf(top, trow[s]);
  }
  for (int off = 16; off > 0; off >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, off));
  }
  float acc[D / 32];
#pragma unroll
  for (int c = 0; c < D / 32; ++c) acc[c] = 0.0f;
  float tot = 0.0f;
  if (a.rows_safe || m != -INFINITY) {
    for (int s = 0; s < p.splits; ++s) {
      const float ls = lrow[s];
      if (!a.rows_safe && ls == -INFINITY) continue;
      const float w = expf(ls - m);
      tot += w;
      const float* orow = ws_o + (row_id * p.splits + s) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) acc[c] = fmaf(w, orow[lane + 32 * c], acc[c]);
    }
  }
  const bool live = a.rows_safe || tot > 0.0f;
  const float inv = live ? 1.0f / tot : 0.0f;
  const int64_t off = b * a.o_stride[0] + h * a.o_stride[1] + i * a.o_stride[2];
  if (a.out_f32) {
    float* out = static_cast<float*>(a.out) + off;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) out[lane + 32 * c] = acc[c] * inv;
  } else {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + off;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) out[lane + 32 * c] = __float2bfloat16_rn(acc[c] * inv);
  }
  if (lane == 0 && a.lse) a.lse[row_id] = live ? m + logf(tot) : -INFINITY;
  if (lane == 0 && a.max_scores) a.max_scores[row_id] = top * kLn2D;
}

// ---------------------------------------------------------------------------
// Tensor-core split-KV decode (tcgen05), for head dim 128 and block masks
// whose tiles are multiples of 128 keys.  A CTA's query rows (at most 16) are the N side of
// both products and the 128 keys of a tile the M side, so the 128-row UMMA
// tile carries no padding rows:
//   S^T (128 keys x 16 rows)  = K_tile (128 x E) Q^T              (SS form)
//   O^T (Ev x 16 rows)       += V_tile^T (Ev x 128) P^T (128 x 16) (SS form;
//                               V read as an MN-major A operand, P from smem)
// Each softmax thread owns one key of the tile (one TMEM lane of S^T) and
// the 16 row scores of that key.  The running maximum of a row is the same
// in every thread; it moves only when some score passes it by more than 2^8
// (one OR-vote per tile finds out), and only then are the row maxima reduced
// over the keys and O^T rescaled in TMEM.  Row sums stay per key thread and
// are reduced once, at the end.
//   warp 0      TMA producer: K and V tiles (64-key boxes, 128-byte swizzle)
//               into a ring of single K or V tiles.
//   warp 1      TMEM allocation; one thread issues QK of tile j, then PV of
//               tile j - 1, so the next S is computed while the softmax runs.
//   warps 2-5   softmax (warp % 4 is the TMEM lane quadrant), epilogue.
// ---------------------------------------------------------------------------
constexpr int kTcThreads = 192;
constexpr int kTcKeys = 128;      // keys per tile: the UMMA M of both products
constexpr int kTcRows = 16;       // query rows: the UMMA N
constexpr int kTcTmemCols = 64;   // S^T buffers at columns 0 and 16, O^T at 32
constexpr int kTcMaxRing = 3;

template <int D>
struct TcCfg {
  static_assert(D == 128, "V^T as the 128-row A operand needs Ev = 128");
  static constexpr int kEntryBytes = kTcKeys * D * 2;     // one K or V tile
  static constexpr int kRing = 3;                         // 96 KB: two CTAs per SM
  static constexpr int kRingBytes = kRing * kEntryBytes;
  static constexpr int kQBytes = (D / 64) * kTcRows * 128;
  static constexpr int kPBufBytes = 2 * kTcRows * 128;    // 128 keys of P as two 64-key boxes
  static constexpr int kSmemBytes = kRingBytes + kQBytes + 2 * kPBufBytes + 1024;
};

struct TcBars {
  uint64_t full[kTcMaxRing], empty[kTcMaxRing];
  uint64_t s_full[2], s_free[2], p_full[2], p_free[2], o_final;
  uint32_t tmem_base;
  int abort;
};

// Reduce-scatter of 16 values per lane over a warp (max or sum): afterwards
// lane l holds the reduction over all 32 lanes of value (l >> 1) & 15.
// Sixteen shuffles instead of 5 x 16 for a full butterfly per value.
template <bool kMax>
__device__ __forceinline__ float warp_reduce16(const float (&v)[16], int lane) {
  auto op = [](float x, float y) { return kMax ? fmaxf(x, y) : x + y; };
  float a8[8], a4[4], a2[2];
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4, h2 = lane & 2;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    a8[i] = op(h16 ? v[8 + i] : v[i], __shfl_xor_sync(0xffffffffu, h16 ? v[i] : v[8 + i], 16));
#pragma unroll
  for (int i = 0; i < 4; ++i)
    a4[i] = op(h8 ? a8[4 + i] : a8[i], __shfl_xor_sync(0xffffffffu, h8 ? a8[i] : a8[4 + i], 8));
#pragma unroll
  for (int i = 0; i < 2; ++i)
    a2[i] = op(h4 ? a4[2 + i] : a4[i], __shfl_xor_sync(0xffffffffu, h4 ? a4[i] : a4[2 + i], 4));
  const float a1 = op(h2 ? a2[1] : a2[0], __shfl_xor_sync(0xffffffffu, h2 ? a2[0] : a2[1], 2));
  return op(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
}

// The sequence with the given rank when sequences are ordered by the length
// of their list of key tiles, longest first (ties by index), for up to 32
// sequences with lists of their own; otherwise the batch order.  Called by
// every lane of a warp.
__device__ __forceinline__ int sequence_of_rank(const FwdArgs& a, int rank) {
  if (a.B > 32 || a.bm.B == 1) return rank;
  const int lane = threadIdx.x & 31;
  int cnt = -1;
  if (lane < a.B) {
    const int64_t row = static_cast<int64_t>(lane) * a.bm.H * a.bm.Mb;  // head row 0, query tile 0
    cnt = __ldg(a.bm.full_kv_num_blocks + row) + __ldg(a.bm.kv_num_blocks + row);
  }
  int r = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int cj = __shfl_sync(0xffffffffu, cnt, j);
    r += (cj > cnt || (cj == cnt && j < lane)) ? 1 : 0;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, lane < a.B && r == rank);
  return hit ? __ffs(hit) - 1 : rank;
}

template <int D, int SCORE>
__global__ void __launch_bounds__(kTcThreads, 2)
    decode_tc_kernel(const __grid_constant__ FwdArgs a, const DecodePlan p,
                     const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                     float* ws_o, float* ws_lse, float* ws_max) {
  using C = TcCfg<D>;
  constexpr int R = C::kRing;
  extern __shared__ uint8_t smem_raw[];
  __shared__ TcBars bars;
  __shared__ float s_red[2][4][kTcRows];
  __shared__ int s_qpos[kTcRows], s_head[kTcRows], s_pq[kTcRows];
  __shared__ float s_slope[kTcRows];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem;
  uint8_t* sQ = smem + C::kRingBytes;
  uint8_t* sP = sQ + C::kQBytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (KV head x head chunk, split, rank): CTAs start in linear order, so
  // the sequences are taken from the longest list of tiles to the shortest,
  // and each sequence's tiles are cut into p.splits equal chunks: the longest
  // chunks start first and the last CTAs to start are the shortest
  const int split = blockIdx.y;
  const int head_chunks = (a.G + p.heads_per_cta - 1) / p.heads_per_cta;
  const int hk = blockIdx.x / head_chunks, hc = blockIdx.x % head_chunks;
  const int b = sequence_of_rank(a, static_cast<int>(blockIdx.z));
  const int S_b = seq_len_b(a.mask, b, a.S);
  const int bmb = a.bm.B > 1 ? b : 0;
  const int bmh = a.bm.H > 1 ? hk * a.G + hc * p.heads_per_cta : 0;  // per-head lists: one head per CTA
  const int64_t brow = (static_cast<int64_t>(bmb) * a.bm.H + bmh) * a.bm.Mb;
  const int nfull = __ldg(a.bm.full_kv_num_blocks + brow);
  const int ntiles = nfull + __ldg(a.bm.kv_num_blocks + brow);
  const int chunk = (ntiles + p.splits - 1) / p.splits;  // this sequence's tiles per split
  const int t0 = split * chunk;
  const int t1 = min(ntiles, t0 + chunk);
  const int subs = a.bm.BN / kTcKeys;  // 128-key tiles per listed block
  const int nsub = t1 > t0 ? (t1 - t0) * subs : 0;
  volatile int* abort = &bars.abort;
  const bool has_pos = SCORE == FA_SCORE_CAP_THEN_BIAS && a.score.pos != nullptr;

  auto row_valid = [&](int r) {
    const int g = hc * p.heads_per_cta + r / a.L;
    return r < p.rows_per_cta && r / a.L < p.heads_per_cta && g < a.G;
  };
  auto row_head = [&](int r) { return hk * a.G + hc * p.heads_per_cta + r / a.L; };

  // Rows and outer coordinates (batch, or page of a paged pool) of the two
  // 64-key boxes of tile j; the producer reads them one tile ahead, so the
  // list and page-table loads are not on its issue path.
  auto tile_addr = [&](int j, int (&row)[2], int (&outer)[2]) {
    const int n = list_tile(a, brow, nfull, t0 + j / subs);
    const int kv0 = n * a.bm.BN + (j % subs) * kTcKeys;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      // a paged cache keeps each 64-key box in one page
      row[h2] = kv0 + 64 * h2;
      outer[h2] = b;
      if (a.page_table) {
        outer[h2] = cache_page(a.page_table, a.pages_per_seq, a.page_size, a.num_pages, a.status, b, row[h2]);
        row[h2] = row[h2] % a.page_size;
      }
    }
  };
  int row_c[2], outer_c[2], row_n[2], outer_n[2];  // tile of copy u, and the next tile
  // K (u even) or V (u odd) of tile u / 2 into ring entry u % R
  auto issue_load = [&](int u) {
    if (u == 0) {
      tile_addr(0, row_c, outer_c);
      if (nsub > 1) tile_addr(1, row_n, outer_n);
    } else if ((u & 1) == 0) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        row_c[h2] = row_n[h2];
        outer_c[h2] = outer_n[h2];
      }
      if ((u >> 1) + 1 < nsub) tile_addr((u >> 1) + 1, row_n, outer_n);
    }
    const int e = u % R;
    const CUtensorMap* map = (u & 1) ? &map_v : &map_k;
    uint8_t* dst = sKV + e * C::kEntryBytes;
    mbar_expect_tx(&bars.full[e], C::kEntryBytes);
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2)
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tma_load_4d(dst + c * (kTcKeys * 128) + h2 * (64 * 128), map, &bars.full[e], c * 64, row_c[h2], hk,
                    outer_c[h2]);
  };
  // The first R copies need no free entry: thread 0 (the producer) issues
  // them right after initialising the barriers, so they are in flight while
  // the CTA stages Q and allocates TMEM.
  const int first_loads = min(R, 2 * nsub);
  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_free[i], 4);
      mbar_init(&bars.p_full[i], 4);
      mbar_init(&bars.p_free[i], 1);
    }
    mbar_init(&bars.o_final, 1);
    bars.abort = 0;
    mbar_fence_init();
    if (nsub > 0) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
    }
    for (int u = 0; u < first_loads; ++u) issue_load(u);
  }
  if (threadIdx.x < kTcRows) {
    const int r = threadIdx.x;
    const int Hs = a.score.slope_heads > 0 ? a.score.slope_heads : a.Hq;
    const bool ok = row_valid(r);
    s_qpos[r] = query_pos(r % a.L, a.L, S_b);
    s_head[r] = ok ? row_head(r) : -1;
    s_slope[r] = distance_slope(ok ? row_head(r) : 0, Hs);
    s_pq[r] = has_pos ? pos_at(a.score, b, s_qpos[r], a.S) : 0;
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, kTcTmemCols);
  if (warp >= 2) {
    // Q rows into shared memory, 128-byte swizzled K-major (the layout TMA
    // writes for a box of 64 columns); rows past the CTA's are zero
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q);
    for (int idx = threadIdx.x - 64; idx < kTcRows * (D / 8); idx += 128) {
      const int r = idx / (D / 8), ch = idx % (D / 8);
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (row_valid(r))
        val = *reinterpret_cast<const uint4*>(qb + b * a.q_stride[0] + row_head(r) * a.q_stride[1] +
                                              (r % a.L) * a.q_stride[2] + ch * 8);
      *reinterpret_cast<uint4*>(sQ + (ch >> 3) * (kTcRows * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                                (((ch & 7) ^ (r & 7)) << 4)) = val;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0 && nsub > 0) {
      int issued = first_loads;
      for (int u = first_loads; u < 2 * nsub && !*abort; ++u) {
        if (!mbar_wait(&bars.empty[u % R], ((u / R) - 1) & 1, abort, a.status, a.wait_cycles)) break;
        issue_load(u);
        issued = u + 1;
      }
      // every copy issued lands before this thread leaves (only the last R
      // can be pending: earlier entries were waited free before reuse)
      volatile int never = 0;
      for (int u = (issued > R ? issued - R : 0); u < issued; ++u)
        mbar_wait(&bars.full[u % R], (u / R) & 1, &never, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kTcKeys, kTcRows, 0, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(kTcKeys, kTcRows, 1, 0);
      const uint64_t dk0 = umma_desc_sw128(smem_u32(sKV), 16, 1024);
      // V^T: M runs along a row of V; its two 64-column blocks are
      // kTcKeys * 128 bytes apart
      const uint64_t dv0 = umma_desc_sw128(smem_u32(sKV), kTcKeys * 128, 1024);
      const uint64_t dq0 = umma_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dp0 = umma_desc_sw128(smem_u32(sP), 16, 1024);
      auto issue_qk = [&](int j) {
        const int e = (2 * j) % R, sb = j & 1;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t aoff =
              static_cast<uint32_t>(e * C::kEntryBytes + (kk >> 2) * (kTcKeys * 128) + (kk & 3) * 32) >> 4;
          const uint32_t boff = static_cast<uint32_t>((kk >> 2) * (kTcRows * 128) + (kk & 3) * 32) >> 4;
          umma_ss(tbase + 16 * sb, dk0 + aoff, dq0 + boff, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars.s_full[sb]);
        umma_commit(&bars.empty[e]);  // K_j may be overwritten once QK_j is done
      };
      auto issue_pv = [&](int j) {
        const int e = (2 * j + 1) % R, pb = j & 1;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTcKeys / 16; ++kk) {
          const uint32_t aoff = static_cast<uint32_t>(e * C::kEntryBytes + kk * 16 * 128) >> 4;
          const uint32_t boff =
              static_cast<uint32_t>(pb * C::kPBufBytes + (kk >> 2) * (kTcRows * 128) + (kk & 3) * 32) >> 4;
          umma_ss(tbase + 32, dv0 + aoff, dp0 + boff, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars.p_free[pb]);
        umma_commit(&bars.empty[e]);  // and V_j once PV_j is done
      };
      // Issue whichever product is ready first: QK of tile jq once K_jq has
      // landed and its S buffer is free (the softmax has read S_{jq-2}), PV
      // of tile jp once P_jp is written.  A PV never waits behind the next
      // tile's K copy, so V's ring entry, and with it the next load, is freed
      // as early as possible.  The loop gives up (timeout) when nothing has
      // become ready for the wait budget.
      // A parity test tells apart only two consecutive phases of a barrier.
      // K_jq's ring entry last held V_{jq-2}; QK_jq is tested only once PV of
      // tile jq-2 has been issued, that is once V_{jq-2} was seen in place,
      // so the entry's barrier is never two phases behind the tested one.
      // (V_jp's entry last held K_{jp-1}, seen before QK_{jp-1}; P and S
      // buffers were likewise seen one use earlier.)
      int jq = 0, jp = 0;
      long long idle_from = clock64();
      while (jp < nsub) {
        bool progressed = false;
        if (jq < nsub && jp >= jq - 1 && mbar_test(&bars.full[(2 * jq) % R], ((2 * jq) / R) & 1) &&
            (jq < 2 || mbar_test(&bars.s_free[jq & 1], ((jq - 2) >> 1) & 1))) {
          issue_qk(jq++);
          progressed = true;
        }
        if (jp < jq && mbar_test(&bars.p_full[jp & 1], (jp >> 1) & 1) &&
            mbar_test(&bars.full[(2 * jp + 1) % R], ((2 * jp + 1) / R) & 1)) {
          issue_pv(jp++);
          progressed = true;
        }
        if (progressed) {
          idle_from = clock64();
        } else if (*abort) {
          break;
        } else if (clock64() - idle_from > a.wait_cycles) {
          record_error(a.status, FA_ERR_TIMEOUT);
          *abort = 1;
          break;
        }
      }
      // every MMA issued above completes before the epilogue or TMEM release
      umma_commit(&bars.o_final);
      volatile int never = 0;
      mbar_wait(&bars.o_final, 0, &never, nullptr);
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int qd = warp & 3;
    const int kk = qd * 32 + lane;  // this thread's key of the tile; its TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    constexpr bool kCapped = SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_CAP_THEN_BIAS;
    const float c_in = kCapped ? a.scale / a.score.cap : 0.0f;
    const float c_out = kCapped ? a.score.cap * kLog2eD : a.scale * kLog2eD;
    const bool want_max = a.max_scores != nullptr;
    float m_run[kTcRows], l_part[kTcRows], tm[kTcRows];
    float sl2[kTcRows], sq2[kTcRows];  // ALiBi in log2 units: slope and slope * q per row
#pragma unroll
    for (int r = 0; r < kTcRows; ++r) {
      m_run[r] = kNoKeyMaxD;
      l_part[r] = 0.0f;
      tm[r] = -INFINITY;
      sl2[r] = s_slope[r] * kLog2eD;
      sq2[r] = sl2[r] * static_cast<float>(s_qpos[r]);
    }
    bool alive = true;
    for (int j = 0; j < nsub; ++j) {
      const int sb = j & 1;
      const int jt = t0 + j / subs;
      const int n = list_tile(a, brow, nfull, jt);
      bool ok = alive && __all_sync(0xffffffffu, mbar_wait(&bars.s_full[sb], (j >> 1) & 1, abort, a.status,
                                                           a.wait_cycles));
      float t[kTcRows];
      bool grow = false;
      if (ok) {
        uint32_t sr[kTcRows];
        tc_fence_after();
        tmem_ld16(tbase + lane_base + 16 * sb, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_free[sb]);  // QK of tile j + 2 may overwrite it
        const int kv0 = n * a.bm.BN + (j % subs) * kTcKeys;
        const int kv = kv0 + kk;
        if constexpr (SCORE == FA_SCORE_NONE) {
#pragma unroll
          for (int r = 0; r < kTcRows; ++r) t[r] = __uint_as_float(sr[r]) * c_out;
        } else if constexpr (SCORE == FA_SCORE_ALIBI) {
          const float kvf = static_cast<float>(kv);
#pragma unroll
          for (int r = 0; r < kTcRows; ++r) t[r] = fmaf(__uint_as_float(sr[r]), c_out, fmaf(sl2[r], kvf, -sq2[r]));
        } else {
          // tanh on the FMA pipe (odd series, |y| <= kTanhPolyMax), the
          // hardware tanh for the rare larger arguments
          float th[kTcRows];
          bool big = false;
#pragma unroll
          for (int i = 0; i < kTcRows / 2; ++i) {
            float2 u2;
            const float2 y = make_float2(__uint_as_float(sr[2 * i]) * c_in, __uint_as_float(sr[2 * i + 1]) * c_in);
            const float2 v2 = tanh_poly2(y, u2);
            th[2 * i] = v2.x;
            th[2 * i + 1] = v2.y;
            big |= fmaxf(u2.x, u2.y) > kTanhPolyMax * kTanhPolyMax;
          }
          if (__any_sync(0xffffffffu, big)) {
#pragma unroll
            for (int r = 0; r < kTcRows; ++r) {
              const float y = __uint_as_float(sr[r]) * c_in;
              if (fabsf(y) > kTanhPolyMax) th[r] = tanh_fast(y);
            }
          }
          if constexpr (SCORE == FA_SCORE_SOFTCAP) {
#pragma unroll
            for (int r = 0; r < kTcRows; ++r) t[r] = th[r] * c_out;
          } else {
            const int pk = has_pos ? pos_at(a.score, b, kv, a.S) : kv;
#pragma unroll
            for (int r = 0; r < kTcRows; ++r) {
              const int d = has_pos ? pk - s_pq[r] : kv - s_qpos[r];
              t[r] = fmaf(th[r], c_out, sl2[r] * static_cast<float>(d));
            }
          }
        }
        // element mask on listed-partial tiles and at the end of the sequence
        if (jt >= nfull || kv0 + kTcKeys > S_b) {
#pragma unroll
          for (int r = 0; r < kTcRows; ++r)
            if (s_head[r] < 0 || !mask_visible(a.mask, b, s_head[r], s_qpos[r], kv, S_b, a.S)) t[r] = -INFINITY;
        }
#pragma unroll
        for (int r = 0; r < kTcRows; ++r) grow |= t[r] > m_run[r] + kRescaleThresholdD;
      }
      // one vote per tile: everything as usual, or a wait gave up, or some
      // row's maximum moves
      if (named_bar_or(1, 128, !ok || grow)) {
        if (named_bar_or(1, 128, !ok)) {
          alive = false;
          break;
        }
        // the tile's row maxima over its 128 keys
        const float v = warp_reduce16<true>(t, lane);
        if ((lane & 1) == 0) s_red[0][qd][(lane >> 1) & 15] = v;
        named_bar_sync(1, 128);
        float alpha[kTcRows];
#pragma unroll
        for (int r = 0; r < kTcRows; ++r) {
          const float tmax = fmaxf(fmaxf(s_red[0][0][r], s_red[0][1][r]), fmaxf(s_red[0][2][r], s_red[0][3][r]));
          const float mn = fmaxf(m_run[r], tmax);
          alpha[r] = ex2_approx(m_run[r] - mn);
          m_run[r] = mn;
          l_part[r] *= alpha[r];
        }
        named_bar_sync(1, 128);  // s_red is read by all before its next use
        if (j > 0) {
          // O^T holds tiles 0 .. j-1: once the last of them is in, rescale
          const int jp = j - 1;
          alive = __all_sync(0xffffffffu, mbar_wait(&bars.p_free[jp & 1], (jp >> 1) & 1, abort, a.status,
                                                    a.wait_cycles));
          if (alive) {
            tc_fence_after();
            uint32_t o[kTcRows];
            tmem_ld16(tbase + lane_base + 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int r = 0; r < kTcRows; ++r) o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha[r]);
            tmem_st16(tbase + lane_base + 32, o);
            tmem_wait_st();
          }
        }
      }
      // P of this tile into buffer j & 1, free once PV of tile j - 2 is done
      if (alive && j >= 2)
        alive = __all_sync(0xffffffffu, mbar_wait(&bars.p_free[sb], ((j - 2) >> 1) & 1, abort, a.status,
                                                  a.wait_cycles));
      if (alive) {
        uint8_t* pbuf = sP + sb * C::kPBufBytes + (kk >> 6) * (kTcRows * 128) + (kk & 7) * 2;
        const int chunk = (kk & 63) >> 3;
#pragma unroll
        for (int r = 0; r < kTcRows; ++r) {
          const float pr = ex2_approx(t[r] - m_run[r]);
          l_part[r] += pr;
          if (want_max) tm[r] = fmaxf(tm[r], t[r]);
          *reinterpret_cast<__nv_bfloat16*>(pbuf + (r >> 3) * 1024 + (r & 7) * 128 + ((chunk ^ (r & 7)) << 4)) =
              __float2bfloat16_rn(pr);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[sb]);
      }
    }
    // every softmax thread arrives here together (the loop is left only
    // through the vote, or at its end)
    bool fin = alive;
    if (fin && nsub > 0) fin = mbar_wait(&bars.o_final, 0, abort, a.status, a.wait_cycles);
    fin = named_bar_and(1, 128, fin && !*abort);
    if (fin) {
      tc_fence_after();
      uint32_t o[kTcRows];
#pragma unroll
      for (int r = 0; r < kTcRows; ++r) o[r] = 0u;
      if (nsub > 0) {
        tmem_ld16(tbase + lane_base + 32, o);
        tmem_wait_ld();
      }
      // row sums and maxima over the 128 keys' partials
      const float vs = warp_reduce16<false>(l_part, lane);
      const float vm = warp_reduce16<true>(tm, lane);
      if ((lane & 1) == 0) {
        s_red[0][qd][(lane >> 1) & 15] = vs;
        s_red[1][qd][(lane >> 1) & 15] = vm;
      }
      named_bar_sync(1, 128);
      const int ev = kk;
#pragma unroll
      for (int r = 0; r < kTcRows; ++r) {
        const int hq = s_head[r];
        if (hq < 0) continue;
        const float l = (s_red[0][0][r] + s_red[0][1][r]) + (s_red[0][2][r] + s_red[0][3][r]);
        const float top = fmaxf(fmaxf(s_red[1][0][r], s_red[1][1][r]), fmaxf(s_red[1][2][r], s_red[1][3][r]));
        // a row without a visible key has l = 0: out 0 and lse -inf, unless
        // the caller promised there is none (rows_safe)
        const bool live = a.rows_safe || l > 0.0f;
        const float inv = live ? 1.0f / l : 0.0f;
        const float lse = live ? (m_run[r] + log2f(l)) * kLn2D : -INFINITY;
        const int i = r % a.L;
        const int64_t row_id = (static_cast<int64_t>(b) * a.Hq + hq) * a.L + i;
        const float val = __uint_as_float(o[r]) * inv;
        if (p.splits == 1) {
          if (ev < D) {
            const int64_t off = b * a.o_stride[0] + hq * a.o_stride[1] + i * a.o_stride[2] + ev;
            if (a.out_f32)
              static_cast<float*>(a.out)[off] = val;
            else
              static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(val);
          }
          if (ev == 0 && a.lse) a.lse[row_id] = lse;
          if (ev == 0 && a.max_scores) a.max_scores[row_id] = top * kLn2D;
        } else {
          if (ev < D) ws_o[(row_id * p.splits + split) * D + ev] = val;
          if (ev == 0) ws_lse[row_id * p.splits + split] = lse;
          if (ev == 0) ws_max[row_id * p.splits + split] = top;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTcTmemCols);
}

template <int D>
cudaError_t launch_decode_d(const FwdArgs& a, const DecodePlan& p, const Sm100Maps& maps, void* workspace,
                            cudaStream_t stream) {
  const int head_chunks = (a.G + p.heads_per_cta - 1) / p.heads_per_cta;
  float* ws_o = static_cast<float*>(workspace);
  const int64_t row_splits = static_cast<int64_t>(a.B) * a.Hq * a.L * p.splits;
  float* ws_lse = ws_o ? ws_o + row_splits * D : nullptr;
  float* ws_max = ws_o ? ws_lse + row_splits : nullptr;
  dim3 grid(p.splits, a.Hkv * head_chunks, a.B);
  cudaError_t e;
  if (D == 128 && a.bm.BN % kTcKeys == 0) {
    // head dim 128, tiles of whole 128-key multiples: the tensor-core kernel
    constexpr int DT = 128;
    auto kern = a.score.kind == FA_SCORE_NONE      ? decode_tc_kernel<DT, FA_SCORE_NONE>
                : a.score.kind == FA_SCORE_SOFTCAP ? decode_tc_kernel<DT, FA_SCORE_SOFTCAP>
                : a.score.kind == FA_SCORE_ALIBI   ? decode_tc_kernel<DT, FA_SCORE_ALIBI>
                                                   : decode_tc_kernel<DT, FA_SCORE_CAP_THEN_BIAS>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<DT>::kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid_tc(a.Hkv * head_chunks, p.splits, a.B);
    kern<<<grid_tc, kTcThreads, TcCfg<DT>::kSmemBytes, stream>>>(a, p, maps.k, maps.v, ws_o, ws_lse, ws_max);
  } else {
    auto kern = a.score.kind == FA_SCORE_NONE      ? decode_kernel<D, FA_SCORE_NONE>
                : a.score.kind == FA_SCORE_SOFTCAP ? decode_kernel<D, FA_SCORE_SOFTCAP>
                : a.score.kind == FA_SCORE_ALIBI   ? decode_kernel<D, FA_SCORE_ALIBI>
                                                   : decode_kernel<D, FA_SCORE_CAP_THEN_BIAS>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg<D>::kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kDecThreads, DecCfg<D>::kSmemBytes, stream>>>(a, p, maps.k, maps.v, ws_o, ws_lse, ws_max);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || p.splits == 1) return e;
  const int64_t rows = static_cast<int64_t>(a.B) * a.Hq * a.L;
  combine_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(a, p, ws_o, ws_lse, ws_max);
  return cudaGetLastError();
}

}  // namespace

int plan_decode(const FwdArgs& a, int split_kv, int num_sms, DecodePlan* p) {
  p->heads_per_cta = a.G < kRows / a.L ? a.G : kRows / a.L;
  if (a.bm.H > 1) p->heads_per_cta = 1;  // per-head tile lists: one query head per CTA
  p->rows_per_cta = p->heads_per_cta * a.L;
  const int head_chunks = (a.G + p->heads_per_cta - 1) / p->heads_per_cta;
  const int units = a.B * a.Hkv * head_chunks;
  const int Nb = a.bm.Nb;
  int splits;
  if (split_kv > 1) {
    splits = split_kv < Nb ? split_kv : Nb;
  } else {
    // about eight CTAs' worth of work per SM over the longest row of tiles;
    // five for the tensor-core kernel (two CTAs per SM, a longer start-up
    // per CTA, and long runs dispatched first): measured on the 32-sequence
    // decode workload, 3 splits in that order beat 5 by 7%
    const bool tc = a.E == 128 && a.bm.BN % kTcKeys == 0;
    const int target = (tc ? 5 : 8) * num_sms;
    splits = (target + units - 1) / units;
    splits = splits < 1 ? 1 : (splits > Nb ? Nb : splits);
  }
  splits = splits > 65535 ? 65535 : splits;  // a grid dimension
  p->tiles_per_split = (Nb + splits - 1) / splits;
  p->splits = (Nb + p->tiles_per_split - 1) / p->tiles_per_split;
  // per (row, split): Ev partial outputs, the partial lse and the row maximum
  p->workspace_bytes = p->splits > 1 ? static_cast<size_t>(a.B) * a.Hq * a.L * p->splits * (a.Ev + 2) * sizeof(float)
                                     : 0;
  return 0;
}

cudaError_t launch_decode(const FwdArgs& a, const DecodePlan& p, const Sm100Maps& maps, void* workspace,
                          cudaStream_t stream) {
  return a.E == 64 ? launch_decode_d<64>(a, p, maps, workspace, stream)
                   : launch_decode_d<128>(a, p, maps, workspace, stream);
}

}  // namespace fa
