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
// One CTA computes one 128-row query tile of one (batch, query head):
//   warp 0      TMA producer: Q once, then K_j and V_j for every listed tile j
//               into NS-stage rings (128 x 64 bf16 boxes, 128-byte swizzle).
//   warp 1      TMEM allocator and MMA issuer (one elected thread):
//               S[j%2] = Q K_j^T (SS form, both K-major), then
//               O += P[j%2] V_j (TS form: P from TMEM, V MN-major in smem).
//   warps 2-5   softmax warpgroup, one query row per thread (TMEM lane):
//               load S_j, apply the score rule and (partial / edge tiles) the
//               element mask, update the running max, write P_j = 2^(t - m) as
//               bf16 into TMEM, keep the running sum; finally O / l and lse.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+D) P0 [384,448) P1 [448,512).
// The running max is only moved (and O rescaled) when it grows by more than
// 2^8, so most tiles skip the O rescale; P then stays below 2^8, exact in the
// final O / l ratio.
//
// Every mbarrier wait is bounded; on a timeout the CTA records FA_ERR_TIMEOUT
// in the status word, stops issuing work, drains its own copies and MMAs
// (again with bounded waits), frees its TMEM and exits.
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "mods.cuh"

namespace fa {

namespace {

constexpr int kThreads = 192;
constexpr int kTile = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256, kColP0 = 384;

template <int D>
struct Cfg {
  static constexpr int kBoxes = D / 64;                  // 64-column boxes per tile row
  static constexpr int kTileBytes = kTile * D * 2;       // one Q/K/V tile
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kSmemBytes = kTileBytes * (1 + 2 * kStages) + 1024;
};

struct Barriers {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int tile_at(const FwdArgs& a, int64_t brow, int nfull, int j, bool* is_full) {
  *is_full = j < nfull;
  return *is_full ? __ldg(a.bm.full_kv_indices + brow * a.bm.Nb + j)
                  : __ldg(a.bm.kv_indices + brow * a.bm.Nb + (j - nfull));
}

// Bits [lo, hi] of a 32-bit word (positions relative to the word's first column).
__device__ __forceinline__ uint32_t span_bits(int lo, int hi) {
  lo = max(lo, 0);
  hi = min(hi, 31);
  if (hi < lo) return 0u;
  const uint32_t upto = hi == 31 ? 0xFFFFFFFFu : ((2u << hi) - 1u);
  return upto & ~((1u << lo) - 1u);
}

// One TMEM row of 128 fp32 columns into registers: eight loads in flight, one
// wait.  The empty asm statements after the wait carry the registers as
// read-write operands so no use of them is scheduled before the wait.
__device__ __forceinline__ void tmem_load_row128(uint32_t taddr, float (&t)[128]) {
  uint32_t* u = reinterpret_cast<uint32_t*>(t);
#pragma unroll
  for (int c = 0; c < 8; ++c) tmem_ld16(taddr + c * 16, *reinterpret_cast<uint32_t(*)[16]>(u + c * 16));
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t* x = u + c * 16;
    asm volatile("" : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]),
                 "+r"(x[7]), "+r"(x[8]), "+r"(x[9]), "+r"(x[10]), "+r"(x[11]), "+r"(x[12]), "+r"(x[13]),
                 "+r"(x[14]), "+r"(x[15]));
  }
}

// Score rule in log2 units for one element; `d` = kv - q as a float.
template <int SCORE>
__device__ __forceinline__ float score_log2(float s, float c_in, float c_out, float slope2, float dist) {
  if constexpr (SCORE == FA_SCORE_NONE) {
    return s * c_out;
  } else if constexpr (SCORE == FA_SCORE_SOFTCAP) {
    return c_out * tanh_fast(s * c_in);
  } else if constexpr (SCORE == FA_SCORE_ALIBI) {
    return fmaf(s, c_out, slope2 * dist);
  } else {
    return fmaf(c_out, tanh_fast(s * c_in), slope2 * dist);
  }
}

template <int D, int SCORE>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_sm100_kernel(const FwdArgs a, const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Barriers bars;
  __shared__ float s_pos[2][kTile];  // slope * position of the tile's keys (score with positions)
  __shared__ int s_doc[2][kTile];    // document ids of the tile's keys (partial document tiles)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::kTileBytes;
  uint8_t* sV = sK + NS * C::kTileBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = gridDim.x - 1 - blockIdx.x;  // longest rows of tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / a.G;
  const int S_b = seq_len_b(a.mask, b, a.S);
  const int bmb = a.bm.B > 1 ? b : 0, bmh = a.bm.H > 1 ? h : 0;
  const int64_t brow = (static_cast<int64_t>(bmb) * a.bm.H + bmh) * a.bm.Mb + mt;
  const int nfull = __ldg(a.bm.full_kv_num_blocks + brow);
  const int ntiles = nfull + __ldg(a.bm.kv_num_blocks + brow);
  volatile int* abort = &bars.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_free[i], 4);
      mbar_init(&bars.p_full[i], 4);
      mbar_init(&bars.pv_done[i], 1);
    }
    mbar_init(&bars.drain, 1);
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
    if (lane == 0 && ntiles > 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      mbar_expect_tx(&bars.q_full, C::kTileBytes);
      for (int c = 0; c < C::kBoxes; ++c)
        tma_load_4d(sQ + c * (kTile * 128), &map_q, &bars.q_full, c * 64, mt * kTile, h, b);
      int issued = 0;
      for (int j = 0; j < ntiles && !*abort; ++j) {
        bool full;
        const int n = tile_at(a, brow, nfull, j, &full);
        const int s = j % NS;
        const uint32_t round = j / NS;
        if (j >= NS && !mbar_wait(&bars.k_empty[s], (round - 1) & 1, abort, a.status)) break;
        mbar_expect_tx(&bars.k_full[s], C::kTileBytes);
        for (int c = 0; c < C::kBoxes; ++c)
          tma_load_4d(sK + s * C::kTileBytes + c * (kTile * 128), &map_k, &bars.k_full[s], c * 64, n * kTile, hk, b);
        if (j >= NS && !mbar_wait(&bars.v_empty[s], (round - 1) & 1, abort, a.status)) {
          issued = j + 1;  // K_j is in flight
          break;
        }
        mbar_expect_tx(&bars.v_full[s], C::kTileBytes);
        for (int c = 0; c < C::kBoxes; ++c)
          tma_load_4d(sV + s * C::kTileBytes + c * (kTile * 128), &map_v, &bars.v_full[s], c * 64, n * kTile, hk, b);
        issued = j + 1;
      }
      if (*abort) {
        // Drain: let every copy this thread issued land before the CTA exits.
        volatile int never = 0;
        mbar_wait(&bars.q_full, 0, &never, nullptr);
        for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j) {
          mbar_wait(&bars.k_full[j % NS], (j / NS) & 1, &never, nullptr);
          mbar_wait(&bars.v_full[j % NS], (j / NS) & 1, &never, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc_bf16(128, D, 0, 1);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = mbar_wait(&bars.q_full, 0, abort, a.status);
      auto issue_pv = [&](int t) -> bool {
        const int s = t % NS;
        if (!mbar_wait(&bars.v_full[s], (t / NS) & 1, abort, a.status)) return false;
        if (!mbar_wait(&bars.p_full[t & 1], (t >> 1) & 1, abort, a.status)) return false;
        tc_fence_after();
        const uint32_t p_tmem = tbase + kColP0 + 64 * (t & 1);
        const uint32_t vs = v_addr + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint64_t bdesc = umma_desc_sw128(vs + kk * 16 * 128, kTile * 128, 1024);
          umma_ts(tbase + kColO, p_tmem + kk * 8, bdesc, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars.pv_done[t & 1]);
        umma_commit(&bars.v_empty[s]);
        return true;
      };
      for (int j = 0; ok && j < ntiles; ++j) {
        const int s = j % NS;
        if (!mbar_wait(&bars.k_full[s], (j / NS) & 1, abort, a.status)) break;
        if (j >= 2 && !mbar_wait(&bars.s_free[j & 1], ((j - 2) >> 1) & 1, abort, a.status)) break;
        tc_fence_after();
        const uint32_t ks = k_addr + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kTile * 128) + (kk & 3) * 32;
          umma_ss(tbase + kColS0 + 128 * (j & 1), umma_desc_sw128(q_addr + off, 16, 1024),
                  umma_desc_sw128(ks + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars.s_full[j & 1]);
        umma_commit(&bars.k_empty[s]);
        if (j >= 1 && !issue_pv(j - 1)) break;
      }
      if (!*abort) issue_pv(ntiles - 1);
      // All MMAs this thread issued complete before TMEM is released.
      umma_commit(&bars.drain);
      volatile int never = 0;
      mbar_wait(&bars.drain, 0, &never, nullptr);
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int grow = mt * kTile + r;
    const bool row_ok = grow < a.L;
    const int qpos = query_pos(grow, a.L, S_b);
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
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
    const bool is_doc = a.mask.kind == FA_MASK_DOCUMENT;
    const int* doc_row = is_doc ? a.mask.doc_id + static_cast<int64_t>(a.mask.doc_batch > 1 ? b : 0) * a.S : nullptr;
    const int my_doc = (is_doc && row_ok && qpos >= 0) ? __ldg(doc_row + qpos) : -1;
    const KeySpans spans = visible_spans(a.mask, qpos, S_b);
    float m_ref = -INFINITY, l_sum = 0.0f;
    bool alive = true;

    for (int j = 0; j < ntiles; ++j) {
      bool full;
      const int n = tile_at(a, brow, nfull, j, &full);
      const int kv0 = n * kTile;
      const bool edge = kv0 + kTile > S_b;
      const bool stage_doc = is_doc && (!full || edge);  // the same for every row of the tile
      if (has_pos || stage_doc) {
        // stage this tile's key-side values in smem (double-buffered by j & 1)
        const int kv = kv0 + r;
        if (has_pos) s_pos[j & 1][r] = slope2 * static_cast<float>(pos_at(a.score, b, kv, a.S));
        if (stage_doc) s_doc[j & 1][r] = kv < a.S ? __ldg(doc_row + kv) : -2;
        named_bar_sync(1, 128);
      }
      if (!mbar_wait(&bars.s_full[j & 1], (j >> 1) & 1, abort, a.status)) {
        alive = false;
        break;
      }
      tc_fence_after();
      float t[kTile];
      tmem_load_row128(tbase + lane_base + kColS0 + 128 * (j & 1), t);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.s_free[j & 1]);

      // score rule on every cell (log2 units)
      if constexpr (SCORE == FA_SCORE_NONE) {
#pragma unroll
        for (int c = 0; c < kTile; ++c) t[c] *= c_out;
      } else if constexpr (SCORE == FA_SCORE_SOFTCAP) {
#pragma unroll
        for (int c = 0; c < kTile; ++c) t[c] = c_out * tanh_fast(t[c] * c_in);
      } else if constexpr (SCORE == FA_SCORE_ALIBI) {
        const float bias0 = slope2 * static_cast<float>(kv0 - qpos);
#pragma unroll
        for (int c = 0; c < kTile; ++c) t[c] = fmaf(t[c], c_out, fmaf(slope2, static_cast<float>(c), bias0));
      } else {
        if (has_pos) {
          const float* pk = s_pos[j & 1];
#pragma unroll
          for (int c = 0; c < kTile; ++c) t[c] = fmaf(c_out, tanh_fast(t[c] * c_in), pk[c] - pq_scaled);
        } else {
          const float bias0 = slope2 * static_cast<float>(kv0 - qpos);
#pragma unroll
          for (int c = 0; c < kTile; ++c)
            t[c] = fmaf(c_out, tanh_fast(t[c] * c_in), fmaf(slope2, static_cast<float>(c), bias0));
        }
      }

      // element mask on partial tiles, ragged edges and rows past L
      if (!full || edge || !row_ok) {
        uint32_t bits[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int base = kv0 + 32 * w;
          bits[w] = row_ok ? (span_bits(spans.a0 - base, spans.a1 - base) | span_bits(spans.b0 - base, spans.b1 - base))
                           : 0u;
        }
        if (stage_doc) {
          const int* dk = s_doc[j & 1];
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t same = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) same |= (dk[32 * w + i] == my_doc ? 1u : 0u) << i;
            bits[w] &= same;
          }
        }
#pragma unroll
        for (int c = 0; c < kTile; ++c)
          if (!((bits[c >> 5] >> (c & 31)) & 1u)) t[c] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kTile; ++c) mx = fmaxf(mx, t[c]);

      // running max: move it (and rescale O) only when it grows past 2^8
      const bool grow_max = mx > m_ref + kRescaleThreshold;
      const float m_new = grow_max ? mx : m_ref;
      const bool rescale = grow_max && m_ref != -INFINITY;
      if (__any_sync(0xffffffffu, rescale) && j > 0) {
        // O holds the sum through tile j-1: wait for that PV, then scale in place
        if (!mbar_wait(&bars.pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, abort, a.status)) {
          alive = false;
          break;
        }
        tc_fence_after();
        const float f = rescale ? ex2_approx(m_ref - m_new) : 1.0f;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          uint32_t rr[16];
          tmem_ld16(tbase + lane_base + kColO + c * 16, rr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * f);
          tmem_st16(tbase + lane_base + kColO + c * 16, rr);
        }
        tmem_wait_st();
        l_sum *= f;
      }
      m_ref = m_new;
      const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
      float psum = 0.0f;
#pragma unroll
      for (int c = 0; c < kTile; ++c) {
        t[c] = ex2_approx(t[c] - m_use);
        psum += t[c];
      }
      l_sum += psum;

      // P_j goes to TMEM buffer j%2 once PV_{j-2} has consumed it
      if (j >= 2 && !mbar_wait(&bars.pv_done[j & 1], ((j - 2) >> 1) & 1, abort, a.status)) {
        alive = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < kTile / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(t[c * 32 + 2 * i], t[c * 32 + 2 * i + 1]);
        tmem_st16(tbase + lane_base + kColP0 + 64 * (j & 1) + c * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[j & 1]);
    }

    // ------------------------------------------------------------ epilogue
    if (alive && ntiles > 0) {
      alive = mbar_wait(&bars.pv_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, abort, a.status);
      tc_fence_after();
    }
    // TMEM loads are warp-collective: every lane takes part, rows past L
    // included; only the stores depend on the row.
    if (__all_sync(0xffffffffu, alive)) {
      const bool live = l_sum > 0.0f && ntiles > 0;
      const float inv = live ? 1.0f / l_sum : 0.0f;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.out) + b * a.o_stride[0] + h * a.o_stride[1] +
                            static_cast<int64_t>(row_ok ? grow : 0) * a.o_stride[2];
      if (row_ok && a.lse)
        a.lse[(static_cast<int64_t>(b) * a.Hq + h) * a.L + grow] = live ? (m_ref + log2f(l_sum)) * kLn2 : -INFINITY;
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t rr[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) rr[i] = 0u;
        if (ntiles > 0) {
          tmem_ld16(tbase + lane_base + kColO + c * 16, rr);
          tmem_wait_ld();
        }
        if (row_ok) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = live ? pack_bf16x2(__uint_as_float(rr[2 * i]) * inv, __uint_as_float(rr[2 * i + 1]) * inv) : 0u;
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 16);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
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
  dim3 grid(a.bm.Mb, a.Hq, a.B);
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
