// Split-KV decode for short queries against long KV caches, and the
// log-sum-exp combination of its partial results.
//
// The computation is the forward definition of "flexattention-score-mod-
// block-mask" (charlestar.github.io), "What one connection goes through", with
// logical query positions q = i + (S_b - L) ("At decode, q_idx = 0 is not
// position 0"; bottom-right alignment, "Causal Mask" (quant67.com) section 4).
// Only the tiles the BlockMask lists are read.  A decode step streams the whole
// valid cache once, so the kernel is built around HBM bandwidth:
//
//   grid      (split, KV head x head chunk, batch); one CTA takes the query rows
//             of up to 16 (query head, position) pairs that share one KV head
//             (GQA: the group's heads reuse every K/V byte it loads) and a
//             contiguous run of the row's listed tiles.
//   warp 0    TMA producer: 64-key K and V sub-tiles (128-byte swizzle) into a
//             3-stage ring.
//   warps 1-4 consumers: each takes 16 of every 64 keys; S = Q K^T and O += P V
//             with mma.sync m16n8k16 (bf16 in, fp32 accumulate; at most 16 rows
//             make the 128-row tcgen05 tile a poor fit and the step is bound by
//             HBM, not the tensor pipe); score rule, element mask and online
//             softmax in registers.  The four warps' (max, sum, O) are merged
//             through shared memory at the end.
//   output    one split: out and lse directly.  Several splits: normalised O,
//             lse and the row maximum per split into the workspace, then
//             combine_kernel merges them: lse = ln sum_s e^{lse_s},
//             o = sum_s e^{lse_s - lse} o_s, max_scores = max_s m_s.
//   abort     when a bounded wait gives up, the consumers skip the merge (it
//             reuses the stage buffers, which copies in flight may still
//             fill) and write nothing; the producer drains its own copies.
#include <math.h>

#include "common.cuh"
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

template <int D>
cudaError_t launch_decode_d(const FwdArgs& a, const DecodePlan& p, const Sm100Maps& maps, void* workspace,
                            cudaStream_t stream) {
  const int head_chunks = (a.G + p.heads_per_cta - 1) / p.heads_per_cta;
  float* ws_o = static_cast<float*>(workspace);
  const int64_t row_splits = static_cast<int64_t>(a.B) * a.Hq * a.L * p.splits;
  float* ws_lse = ws_o ? ws_o + row_splits * D : nullptr;
  float* ws_max = ws_o ? ws_lse + row_splits : nullptr;
  auto kern = a.score.kind == FA_SCORE_NONE      ? decode_kernel<D, FA_SCORE_NONE>
              : a.score.kind == FA_SCORE_SOFTCAP ? decode_kernel<D, FA_SCORE_SOFTCAP>
              : a.score.kind == FA_SCORE_ALIBI   ? decode_kernel<D, FA_SCORE_ALIBI>
                                                 : decode_kernel<D, FA_SCORE_CAP_THEN_BIAS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.splits, a.Hkv * head_chunks, a.B);
  kern<<<grid, kDecThreads, DecCfg<D>::kSmemBytes, stream>>>(a, p, maps.k, maps.v, ws_o, ws_lse, ws_max);
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
    // about eight CTAs' worth of work per SM over the longest row of tiles
    const int target = 8 * num_sms;
    splits = (target + units - 1) / units;
    splits = splits < 1 ? 1 : (splits > Nb ? Nb : splits);
  }
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
