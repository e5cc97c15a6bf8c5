// Backward pass of the FlexAttention forward for sm_100a: the gradients of
// sum(out * dout) with respect to q, k and v, recomputing P from the forward's
// log-sum-exp ("flexattention-score-mod-block-mask" runs the loss's backward
// through flex_attention; the forward definition is "What one connection goes
// through").  With s = scale q k^T, g the score rule, P = exp(g - lse) on
// visible cells (0 elsewhere), D = rowsum(dout * out):
//   dv = P^T dout,   dP = dout v^T,   dS = P (dP - D) dg/ds,
//   dq = scale dS k, dk = scale dS^T q,
// dg/ds = 1 - tanh(s / cap)^2 under a soft-cap, else 1.
//
// Two kernels, each gradient written once in a fixed order (deterministic; the
// guide's WRITE_DQ and dQ write order):
//   bwd_dkdv_kernel  one CTA per (batch, KV head, key tile); it walks the
//                    key tile's query-side list (the guide's from_kv_blocks
//                    lists) for each query head of the KV head's group:
//                    S^T = K Q^T and dP^T = V dout^T on tcgen05 (SS), then
//                    per key row P^T and dS^T, then dV += P^T dout and
//                    dK += dS^T Q (TS, P^T and dS^T from TMEM), accumulated
//                    in TMEM over the whole walk.
//   bwd_dq_kernel    one CTA per (batch, query head, query tile); it walks
//                    the key-side list: S = Q K^T, dP = dout V^T, then per
//                    query row dS, then dQ += dS K (TS).
// Warp roles as in the prefill kernel: warp 0 TMA producer, warp 1 TMEM
// allocator and MMA issuer (one thread), warps 2-9 the rows, one TMEM lane
// (row) per thread and two warps per row, each taking half of the columns.
// TMEM: S at column 0, dP at 128 (P / dS written as bf16 pairs over the
// columns already read), then the accumulators.  Every mbarrier wait is
// bounded; a timeout records FA_ERR_TIMEOUT, the producer drains its copies,
// the MMA thread its MMAs, and the CTA exits.
#include <math.h>

#include "common.cuh"
#include "fastmath.cuh"
#include "launch.h"
#include "mods.cuh"

namespace fa {

namespace {

constexpr int kBwdThreads = 320;
// Rows of a tile take two warps each (warps 2-9; warp % 4 is the TMEM lane
// quadrant): math group 0 takes columns 0-63, group 1 columns 64-127, so two
// warps per SM sub-partition hide each other's latencies.
constexpr int kMathThreads = 256;
// TMEM column of the bf16 pairs for keys (or queries) 16 kk .. 16 kk + 15:
// chunk j = kk / 2 of 32 columns writes its pairs over the first half of its
// own S columns, which only its own thread has read.
__device__ __forceinline__ uint32_t pair_col(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }
constexpr int kBT = 128;  // tile rows and columns
constexpr float kLog2eB = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr int kBoxes = D / 64;
  static constexpr int kTileBytes = kBT * D * 2;
  static constexpr int kStages = D == 64 ? 4 : 2;
  // two resident tiles + a ring of two tiles per stage
  static constexpr int kSmemBytes = kTileBytes * (2 + 2 * kStages) + 1024;
};

struct BwdBars {
  uint64_t fixed_full;                 // the two tiles loaded once
  uint64_t full[4], empty[4];          // the ring (both tiles of a stage)
  uint64_t s_full[2], p_full[2], o_final;  // per half of the tile's columns
  int info[2];                         // tile index | class bit
  int info_h[2];                       // query head (dK / dV kernel)
  uint32_t tmem_base;
  int abort;
};
constexpr int kInfoFullB = 1 << 30;

// tanh accurate to a few fp32 ulps: the odd series below 0.3 in magnitude
// (tanh_poly2, error under 1.5e-6 relative), else 1 - 2 / (e^{2|y|} + 1)
// with its sign.  The gradients sum P and dg/ds = 1 - tanh^2 over many cells
// whose products partly cancel, so the hardware tanh's relative error of
// about 2^-11 would show in them.
__device__ __forceinline__ float tanh_big(float y) {
  const float e = ex2_approx(2.0f * kLog2eB * fminf(fabsf(y), 15.0f));  // tanh(15) is 1 in fp32
  return copysignf(1.0f - __fdividef(2.0f, e + 1.0f), y);
}
// tanh(s c_in) of 32 raw scores: the series on the FMA pipe; the exponential
// form only for arguments beyond kTanhPolyMax, and only when some lane of
// the warp has one, so the common case issues no MUFU operation for it.
__device__ __forceinline__ void tanh32(const uint32_t (&sr)[32], float c_in, float (&th)[32]) {
  float umax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    float2 u;
    const float2 v =
        tanh_poly2(make_float2(__uint_as_float(sr[i]) * c_in, __uint_as_float(sr[i + 1]) * c_in), u);
    th[i] = v.x;
    th[i + 1] = v.y;
    umax = max3f(umax, u.x, u.y);
  }
  if (__any_sync(0xffffffffu, !(umax <= kTanhPolyMax * kTanhPolyMax))) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float y = __uint_as_float(sr[i]) * c_in;
      if (!(fabsf(y) <= kTanhPolyMax)) th[i] = tanh_big(y);
    }
  }
}

// Ties 16 registers written by tcgen05.ld to a point after tcgen05.wait::ld,
// so that no use of them is scheduled before the wait.
__device__ __forceinline__ void hold16(uint32_t (&x)[16]) {
  asm volatile("" : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]), "+r"(x[7]),
               "+r"(x[8]), "+r"(x[9]), "+r"(x[10]), "+r"(x[11]), "+r"(x[12]), "+r"(x[13]), "+r"(x[14]), "+r"(x[15]));
}

// Writes 16 fp32 accumulator columns of a row, times `mul`, as fp32 or bf16
// with 16-byte stores (the gradient tensors are 16-byte aligned).
__device__ __forceinline__ void store16(void* base, int64_t off, bool f32, const uint32_t* rr, float mul) {
  if (f32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(base) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_float4(__uint_as_float(rr[4 * i]) * mul, __uint_as_float(rr[4 * i + 1]) * mul,
                           __uint_as_float(rr[4 * i + 2]) * mul, __uint_as_float(rr[4 * i + 3]) * mul);
  } else {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * mul, __uint_as_float(rr[2 * i + 1]) * mul);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + off);
    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  }
}

// Loads tiles into smem boxes of 64 columns x 128 rows (128-byte swizzle).
template <int D>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int row, int h, int b) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) tma_load_4d(dst + c * (kBT * 128), map, bar, c * 64, row, h, b);
}

// ---------------------------------------------------------------------------
// dQ: one query tile, walking its key-side list
// ---------------------------------------------------------------------------
template <int D, int SCORE>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ BwdArgs a, const __grid_constant__ CUtensorMap map_q,
                  const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_do) {
  using C = BCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ BwdBars bars;
  __shared__ __align__(16) float s_pos[2][kBT];
  __shared__ int s_doc[2][kBT];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = sQ + C::kTileBytes;
  uint8_t* sK = sDO + C::kTileBytes;             // NS stages
  uint8_t* sV = sK + NS * C::kTileBytes;         // NS stages
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, b = blockIdx.y;
  const int mt = gridDim.z - 1 - blockIdx.z;     // longest rows of tiles first
  const int hk = h / a.G;
  const int S_b = seq_len_b(a.mask, b, a.S);
  const int bmb = a.bm.B > 1 ? b : 0, bmh = a.bm.H > 1 ? h : 0;
  const int64_t brow = (static_cast<int64_t>(bmb) * a.bm.H + bmh) * a.bm.Mb + mt;
  const int nfull = __ldg(a.bm.full_kv_num_blocks + brow);
  const int total = nfull + __ldg(a.bm.kv_num_blocks + brow);
  volatile int* abort = &bars.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars.fixed_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 2);  // the MMA thread's arrive (tile info) + the commit
      mbar_init(&bars.p_full[i], 8);  // every math warp
    }
    mbar_init(&bars.o_final, 1);
    bars.abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars.tmem_base;
  auto list_n = [&](int j) {
    return j < nfull ? __ldg(a.bm.full_kv_indices + brow * a.bm.Nb + j)
                     : __ldg(a.bm.kv_indices + brow * a.bm.Nb + (j - nfull));
  };

  if (warp == 0) {
    if (lane == 0 && total > 0) {
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      mbar_expect_tx(&bars.fixed_full, 2 * C::kTileBytes);
      load_tile<D>(sQ, &map_q, &bars.fixed_full, mt * kBT, h, b);
      load_tile<D>(sDO, &map_do, &bars.fixed_full, mt * kBT, h, b);
      int issued = 0;
      for (int u = 0; u < total && !*abort; ++u) {
        const int s = u % NS;
        if (u >= NS && !mbar_wait(&bars.empty[s], ((u / NS) - 1) & 1, abort, a.status, a.wait_cycles)) break;
        const int n = list_n(u);
        mbar_expect_tx(&bars.full[s], 2 * C::kTileBytes);
        load_tile<D>(sK + s * C::kTileBytes, &map_k, &bars.full[s], n * kBT, hk, b);
        load_tile<D>(sV + s * C::kTileBytes, &map_v, &bars.full[s], n * kBT, hk, b);
        issued = u + 1;
      }
      // every copy lands before this thread leaves, on every path
      volatile int never = 0;
      mbar_wait(&bars.fixed_full, 0, &never, nullptr);
      for (int u = (issued > NS ? issued - NS : 0); u < issued; ++u)
        mbar_wait(&bars.full[u % NS], (u / NS) & 1, &never, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, 64, 0, 0);  // one half of the keys
      constexpr uint32_t idesc_dq = umma_idesc_bf16(128, D, 0, 1);
      const uint64_t dq0 = umma_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t ddo0 = umma_desc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dk0 = umma_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = umma_desc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dkmn0 = umma_desc_sw128(smem_u32(sK), kBT * 128, 1024);  // K as an MN-major B operand
      constexpr uint32_t kStep = C::kTileBytes >> 4;
      bool ok = total > 0 && mbar_wait(&bars.fixed_full, 0, abort, a.status, a.wait_cycles);
      for (int u = 0; ok && u < total; ++u) {
        const int s = u % NS;
        if (!mbar_wait(&bars.full[s], (u / NS) & 1, abort, a.status, a.wait_cycles)) break;
        tc_fence_after();
        const int n = list_n(u);
        bars.info[u & 1] = n | (u < nfull ? kInfoFullB : 0);
        // S and dP in two halves of 64 keys each (columns 64 hf ..), so the
        // rows' math on the first half overlaps the products of the second,
        // and dQ over the first half overlaps the math on the second
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * (kBT * 128) + (kk & 3) * 32) >> 4;
            const uint32_t koff = s * kStep + off + ((hf * 64 * 128) >> 4);  // key rows 64 hf ..
            umma_ss(tbase + 64 * hf, dq0 + off, dk0 + koff, idesc_s, kk > 0 ? 1u : 0u);
            umma_ss(tbase + 128 + 64 * hf, ddo0 + off, dv0 + koff, idesc_s, kk > 0 ? 1u : 0u);
          }
          mbar_arrive(&bars.s_full[hf]);
          umma_commit(&bars.s_full[hf]);
        }
        bool half_ok = true;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!(half_ok = mbar_wait(&bars.p_full[hf], u & 1, abort, a.status, a.wait_cycles))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * hf; kk < 4 * hf + 4; ++kk)
            umma_ts(tbase + 256, tbase + pair_col(kk), dkmn0 + s * kStep + ((kk * 16 * 128) >> 4), idesc_dq,
                    (u > 0 || kk > 0) ? 1u : 0u);
        }
        if (!half_ok) break;
        umma_commit(&bars.empty[s]);
      }
      umma_commit(&bars.o_final);
      volatile int never = 0;
      mbar_wait(&bars.o_final, 0, &never, nullptr);
    }
  } else {
    // ------------------------------------------------------------ rows
    const int quad = warp & 3;
    const int jg = (warp - 2) >> 2;  // math group: chunk jg of each 64-column half
    const int r = quad * 32 + lane;
    const int grow = mt * kBT + r;
    const bool row_ok = grow < a.L;
    const int qpos = query_pos(grow, a.L, S_b);
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int Hs = a.score.slope_heads > 0 ? a.score.slope_heads : a.Hq;
    const float slope2 = distance_slope(h, Hs) * kLog2eB;
    constexpr bool kCapped = SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_CAP_THEN_BIAS;
    const float c_in = kCapped ? a.scale / a.score.cap : 0.0f;
    const float c_out = kCapped ? a.score.cap * kLog2eB : a.scale * kLog2eB;
    const bool has_pos = SCORE == FA_SCORE_CAP_THEN_BIAS && a.score.pos != nullptr;
    const float pq_scaled = has_pos ? slope2 * static_cast<float>(pos_at(a.score, b, qpos, a.S)) : 0.0f;
    const bool is_prog = a.mask.kind == FA_MASK_PROGRAM;
    const bool is_doc = a.mask.kind == FA_MASK_DOCUMENT || (is_prog && a.mask.reads_doc);
    const int* doc_row = is_doc ? a.mask.doc_id + static_cast<int64_t>(a.mask.doc_batch > 1 ? b : 0) * a.S : nullptr;
    const int my_doc = (is_doc && row_ok && qpos >= 0) ? __ldg(doc_row + qpos) : 0;
    const KeySpans spans = visible_spans(a.mask, qpos, S_b);
    const int64_t rid = (static_cast<int64_t>(b) * a.Hq + h) * a.L + (row_ok ? grow : 0);
    const float lse_row = row_ok ? a.lse[rid] : -INFINITY;
    const float lse2 = lse_row == -INFINITY ? INFINITY : lse_row * kLog2eB;  // P = 0 on a row without keys
    const float dsum = row_ok ? a.dsum[rid] : 0.0f;
    const bool group_stage = has_pos || is_doc;
    bool alive = true;
    int cnt = 0;
    for (; cnt < total; ++cnt) {
      bool ok = alive && __all_sync(0xffffffffu, mbar_wait(&bars.s_full[0], cnt & 1, abort, a.status, a.wait_cycles));
      const int info = ok ? bars.info[cnt & 1] : 0;
      const int n = info & (kInfoFullB - 1);
      const bool full = (info & kInfoFullB) != 0;
      const int kv0 = n * kBT;
      const bool edge = kv0 + kBT > S_b;
      const bool stage_doc = is_doc && (!full || edge);
      if (group_stage) {
        if (ok && jg == 0) {
          const int kv = kv0 + r;
          if (has_pos) s_pos[cnt & 1][r] = slope2 * static_cast<float>(pos_at(a.score, b, kv, a.S));
          if (stage_doc) s_doc[cnt & 1][r] = kv < a.S ? __ldg(doc_row + kv) : 0;
        }
        ok = named_bar_and(1, kMathThreads, ok);
      }
      if (!ok) {
        alive = false;
        break;
      }
      tc_fence_after();
      const bool need_mask = !full || edge || !row_ok;
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        if (hf == 1) {
          // the second half's products land on their own barrier
          if (!__all_sync(0xffffffffu, mbar_wait(&bars.s_full[1], cnt & 1, abort, a.status, a.wait_cycles))) {
            alive = false;
            break;
          }
          tc_fence_after();
        }
        const int j = 2 * hf + jg;  // this warp's 32-column chunk of the half
        uint32_t sr[32], dp[32];
        tmem_ld16(tbase + lane_base + 32 * j, *reinterpret_cast<uint32_t(*)[16]>(sr));
        tmem_ld16(tbase + lane_base + 32 * j + 16, *reinterpret_cast<uint32_t(*)[16]>(sr + 16));
        tmem_ld16(tbase + lane_base + 128 + 32 * j, *reinterpret_cast<uint32_t(*)[16]>(dp));
        tmem_ld16(tbase + lane_base + 128 + 32 * j + 16, *reinterpret_cast<uint32_t(*)[16]>(dp + 16));
        tmem_wait_ld();
        const int base = kv0 + 32 * j;
        uint32_t bits = 0xFFFFFFFFu;
        if (need_mask) {
          uint32_t same = 0xFFFFFFFFu;
          if (stage_doc) {
            same = 0u;
#pragma unroll
            for (int i = 0; i < 32; ++i) same |= (s_doc[cnt & 1][32 * j + i] == my_doc ? 1u : 0u) << i;
            if (qpos < 0) same = 0u;
          }
          if (is_prog) {
            bits = program_bits(a.mask, h, qpos, base, same) & span_bits(-1, S_b - 1 - base);
          } else {
            bits = (span_bits(spans.a0 - base, spans.a1 - base) | span_bits(spans.b0 - base, spans.b1 - base)) & same;
          }
          if (!row_ok) bits = 0u;
        }
        const float bias0 = (SCORE == FA_SCORE_ALIBI || (SCORE == FA_SCORE_CAP_THEN_BIAS && !has_pos))
                                ? slope2 * static_cast<float>(base - qpos) : 0.0f;
        float th[32];
        if constexpr (kCapped) tanh32(sr, c_in, th);
        // two columns per step in f32x2 arithmetic
        const float* spos = s_pos[cnt & 1] + 32 * j;
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 col = make_float2(static_cast<float>(i), static_cast<float>(i + 1));
          float2 bias = splat2(0.0f);
          if constexpr (SCORE == FA_SCORE_ALIBI) bias = fma2(splat2(slope2), col, splat2(bias0));
          if constexpr (SCORE == FA_SCORE_CAP_THEN_BIAS)
            bias = has_pos ? add2(*reinterpret_cast<const float2*>(spos + i), splat2(-pq_scaled))
                           : fma2(splat2(slope2), col, splat2(bias0));
          float2 t, gp = splat2(1.0f);
          if constexpr (kCapped) {
            const float2 th2 = make_float2(th[i], th[i + 1]);
            t = fma2(th2, splat2(c_out), bias);
            gp = fma2(make_float2(-th2.x, -th2.y), th2, splat2(1.0f));
          } else {
            t = fma2(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), splat2(c_out), bias);
          }
          const float2 e = add2(t, splat2(-lse2));
          const float2 p = make_float2(((bits >> i) & 1u) ? ex2_approx(e.x) : 0.0f,
                                       ((bits >> (i + 1)) & 1u) ? ex2_approx(e.y) : 0.0f);
          float2 ds = mul2(p, add2(make_float2(__uint_as_float(dp[i]), __uint_as_float(dp[i + 1])), splat2(-dsum)));
          if constexpr (kCapped) ds = mul2(ds, gp);
          pk[i >> 1] = pack_bf16x2(ds.x, ds.y);
        }
        // dS of these 32 keys as bf16 pairs over S columns already read
        tmem_st16(tbase + lane_base + 32 * j, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[hf]);
      }
    }
    // epilogue: dq = scale dQ (zero for a row of tiles with no listed key tile)
    if (alive && cnt > 0) {
      alive = mbar_wait(&bars.o_final, 0, abort, a.status, a.wait_cycles);
      tc_fence_after();
    }
    if (__all_sync(0xffffffffu, alive)) {
      const int64_t off = b * a.dq_stride[0] + h * a.dq_stride[1] + static_cast<int64_t>(row_ok ? grow : 0) * a.dq_stride[2];
      // this group's D / 2 columns of dQ, all loads in flight before one wait
      constexpr int kChunks = D / 32;
      uint32_t rr[kChunks][16];
      if (total > 0) {
#pragma unroll
        for (int i = 0; i < kChunks; ++i) tmem_ld16(tbase + lane_base + 256 + (jg * kChunks + i) * 16, rr[i]);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < kChunks; ++i) hold16(rr[i]);
      } else {
#pragma unroll
        for (int i = 0; i < kChunks; ++i)
#pragma unroll
          for (int e = 0; e < 16; ++e) rr[i][e] = 0u;
      }
      if (row_ok) {
#pragma unroll
        for (int i = 0; i < kChunks; ++i) store16(a.dq, off + (jg * kChunks + i) * 16, a.dq_f32, rr[i], a.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}

// ---------------------------------------------------------------------------
// dK, dV: one key tile, walking its query-side lists for every query head of
// its KV head
// ---------------------------------------------------------------------------
struct QWalk {
  // steps: for g in [0, G): the full list, then the partial list, of row
  // (b, head hk G + g, n) of the query-side lists
  const BwdArgs* a;
  int b, hk, n, g, j, nfull, ntot;
  int64_t row;
  __device__ void head(int gg) {
    g = gg;
    j = 0;
    nfull = ntot = 0;
    if (g >= a->G) return;
    const int h = hk * a->G + g;
    const int qb = a->qB > 1 ? b : 0, qh = a->qH > 1 ? h : 0;
    row = (static_cast<int64_t>(qb) * a->qH + qh) * a->bm.Nb + n;
    nfull = __ldg(a->full_q_num_blocks + row);
    ntot = nfull + __ldg(a->q_num_blocks + row);
  }
  __device__ void init(const BwdArgs* aa, int bb, int hh, int nn) {
    a = aa;
    b = bb;
    hk = hh;
    n = nn;
    head(0);
    while (g < a->G && j >= ntot) head(g + 1);
  }
  // next step: (query tile m, full?, head offset g); false when done
  __device__ bool next(int& m, bool& full, int& gg) {
    if (g >= a->G) return false;
    full = j < nfull;
    m = full ? __ldg(a->full_q_indices + row * a->bm.Mb + j) : __ldg(a->q_indices + row * a->bm.Mb + (j - nfull));
    gg = g;
    ++j;
    while (g < a->G && j >= ntot) head(g + 1);
    return true;
  }
};

template <int D, int SCORE>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ BwdArgs a, const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                    const __grid_constant__ CUtensorMap map_do) {
  using C = BCfg<D>;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ BwdBars bars;
  __shared__ __align__(16) float s_lse[2][kBT];
  __shared__ __align__(16) float s_dsum[2][kBT];
  __shared__ __align__(16) float s_pq[2][kBT];
  __shared__ int s_doc[2][kBT];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + C::kTileBytes;
  uint8_t* sQ = sV + C::kTileBytes;               // NS stages
  uint8_t* sDO = sQ + NS * C::kTileBytes;         // NS stages
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hk = blockIdx.x, b = blockIdx.y, n = blockIdx.z;
  const int S_b = seq_len_b(a.mask, b, a.S);
  volatile int* abort = &bars.abort;
  // number of steps: sum over the group's heads of the list lengths
  int total = 0;
  for (int g = 0; g < a.G; ++g) {
    const int h = hk * a.G + g;
    const int64_t row = (static_cast<int64_t>(a.qB > 1 ? b : 0) * a.qH + (a.qH > 1 ? h : 0)) * a.bm.Nb + n;
    total += __ldg(a.full_q_num_blocks + row) + __ldg(a.q_num_blocks + row);
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars.fixed_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 2);  // the MMA thread's arrive (tile info) + the commit
      mbar_init(&bars.p_full[i], 8);  // every math warp
    }
    mbar_init(&bars.o_final, 1);
    bars.abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars.tmem_base;

  if (warp == 0) {
    if (lane == 0 && total > 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_do);
      mbar_expect_tx(&bars.fixed_full, 2 * C::kTileBytes);
      load_tile<D>(sK, &map_k, &bars.fixed_full, n * kBT, hk, b);
      load_tile<D>(sV, &map_v, &bars.fixed_full, n * kBT, hk, b);
      QWalk w;
      w.init(&a, b, hk, n);
      int issued = 0, m, g;
      bool f;
      for (int u = 0; !*abort && w.next(m, f, g); ++u) {
        const int s = u % NS;
        if (u >= NS && !mbar_wait(&bars.empty[s], ((u / NS) - 1) & 1, abort, a.status, a.wait_cycles)) break;
        const int h = hk * a.G + g;
        mbar_expect_tx(&bars.full[s], 2 * C::kTileBytes);
        load_tile<D>(sQ + s * C::kTileBytes, &map_q, &bars.full[s], m * kBT, h, b);
        load_tile<D>(sDO + s * C::kTileBytes, &map_do, &bars.full[s], m * kBT, h, b);
        issued = u + 1;
      }
      volatile int never = 0;
      mbar_wait(&bars.fixed_full, 0, &never, nullptr);
      for (int u = (issued > NS ? issued - NS : 0); u < issued; ++u)
        mbar_wait(&bars.full[u % NS], (u / NS) & 1, &never, nullptr);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(128, 64, 0, 0);  // one half of the queries
      constexpr uint32_t idesc_acc = umma_idesc_bf16(128, D, 0, 1);
      const uint64_t dk0 = umma_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = umma_desc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dq0 = umma_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t ddo0 = umma_desc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dqmn0 = umma_desc_sw128(smem_u32(sQ), kBT * 128, 1024);    // Q as an MN-major B operand
      const uint64_t ddomn0 = umma_desc_sw128(smem_u32(sDO), kBT * 128, 1024);  // dout likewise
      constexpr uint32_t kStep = C::kTileBytes >> 4;
      QWalk w;
      w.init(&a, b, hk, n);
      bool ok = total > 0 && mbar_wait(&bars.fixed_full, 0, abort, a.status, a.wait_cycles);
      int m, g;
      bool f;
      for (int u = 0; ok && w.next(m, f, g); ++u) {
        const int s = u % NS;
        if (!mbar_wait(&bars.full[s], (u / NS) & 1, abort, a.status, a.wait_cycles)) break;
        tc_fence_after();
        bars.info[u & 1] = m | (f ? kInfoFullB : 0);
        bars.info_h[u & 1] = g;
        // S^T and dP^T in two halves of 64 queries each (columns 64 hf ..), so
        // the rows' math on the first half overlaps the products of the
        // second, and dV / dK over the first half the math on the second
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * (kBT * 128) + (kk & 3) * 32) >> 4;
            const uint32_t qoff = s * kStep + off + ((hf * 64 * 128) >> 4);  // query rows 64 hf ..
            umma_ss(tbase + 64 * hf, dk0 + off, dq0 + qoff, idesc_s, kk > 0 ? 1u : 0u);         // S^T = K Q^T
            umma_ss(tbase + 128 + 64 * hf, dv0 + off, ddo0 + qoff, idesc_s, kk > 0 ? 1u : 0u);  // dP^T = V dout^T
          }
          mbar_arrive(&bars.s_full[hf]);
          umma_commit(&bars.s_full[hf]);
        }
        bool half_ok = true;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if (!(half_ok = mbar_wait(&bars.p_full[hf], u & 1, abort, a.status, a.wait_cycles))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 4 * hf; kk < 4 * hf + 4; ++kk) {
            const uint32_t acc = (u > 0 || kk > 0) ? 1u : 0u;
            const uint32_t boff = s * kStep + ((kk * 16 * 128) >> 4);
            umma_ts(tbase + 256, tbase + pair_col(kk), ddomn0 + boff, idesc_acc, acc);          // dV += P^T dout
            umma_ts(tbase + 256 + D, tbase + 128 + pair_col(kk), dqmn0 + boff, idesc_acc, acc); // dK += dS^T Q
          }
        }
        if (!half_ok) break;
        umma_commit(&bars.empty[s]);
      }
      umma_commit(&bars.o_final);
      volatile int never = 0;
      mbar_wait(&bars.o_final, 0, &never, nullptr);
    }
  } else {
    // ------------------------------------------------------------ key rows
    const int quad = warp & 3;
    const int jg = (warp - 2) >> 2;  // math group: chunk jg of each 64-column half
    const int r = quad * 32 + lane;
    const int kv = n * kBT + r;
    const bool key_ok = kv < S_b;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int Hs = a.score.slope_heads > 0 ? a.score.slope_heads : a.Hq;
    constexpr bool kCapped = SCORE == FA_SCORE_SOFTCAP || SCORE == FA_SCORE_CAP_THEN_BIAS;
    const float c_in = kCapped ? a.scale / a.score.cap : 0.0f;
    const float c_out = kCapped ? a.score.cap * kLog2eB : a.scale * kLog2eB;
    const bool has_pos = SCORE == FA_SCORE_CAP_THEN_BIAS && a.score.pos != nullptr;
    const float pk_raw = has_pos ? static_cast<float>(pos_at(a.score, b, kv, a.S)) : 0.0f;
    const bool is_prog = a.mask.kind == FA_MASK_PROGRAM;
    const bool is_doc = a.mask.kind == FA_MASK_DOCUMENT || (is_prog && a.mask.reads_doc);
    const int* doc_row = is_doc ? a.mask.doc_id + static_cast<int64_t>(a.mask.doc_batch > 1 ? b : 0) * a.S : nullptr;
    const int my_doc = (is_doc && kv < a.S) ? __ldg(doc_row + kv) : 0;
    const int qshift = S_b - a.L;  // logical position of query row i: i + qshift
    bool alive = true;
    int cnt = 0;
    for (; cnt < total; ++cnt) {
      bool ok = alive && __all_sync(0xffffffffu, mbar_wait(&bars.s_full[0], cnt & 1, abort, a.status, a.wait_cycles));
      const int info = ok ? bars.info[cnt & 1] : 0;
      const int mq = info & (kInfoFullB - 1);
      const bool full = (info & kInfoFullB) != 0;
      const int g = ok ? bars.info_h[cnt & 1] : 0;
      const int h = hk * a.G + g;
      // the tile's query-side values (lse, D, positions, documents) into smem,
      // double-buffered by cnt & 1 (math group 0 writes them); the barrier
      // also tells every warp whether all eight got their S, so a timeout is
      // left together
      if (ok && jg == 0) {
        const int i = mq * kBT + r;
        const int64_t rid = (static_cast<int64_t>(b) * a.Hq + h) * a.L + i;
        const float l = i < a.L ? a.lse[rid] : -INFINITY;
        s_lse[cnt & 1][r] = l == -INFINITY ? INFINITY : l * kLog2eB;
        s_dsum[cnt & 1][r] = i < a.L ? a.dsum[rid] : 0.0f;
        const int q = i + qshift;
        if (has_pos) s_pq[cnt & 1][r] = static_cast<float>(pos_at(a.score, b, q, a.S));
        if (is_doc) s_doc[cnt & 1][r] = (q >= 0 && q < a.S && i < a.L) ? __ldg(doc_row + q) : 0;
      }
      ok = named_bar_and(1, kMathThreads, ok);
      if (!ok) {
        alive = false;
        break;
      }
      tc_fence_after();
      const float slope2 = distance_slope(h, Hs) * kLog2eB;
      const int i0 = mq * kBT;
      const bool edge = i0 + kBT > a.L || n * kBT + kBT > S_b;
      const bool need_mask = !full || edge || !key_ok;
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {
        if (hf == 1) {
          // the second half's products land on their own barrier
          if (!__all_sync(0xffffffffu, mbar_wait(&bars.s_full[1], cnt & 1, abort, a.status, a.wait_cycles))) {
            alive = false;
            break;
          }
          tc_fence_after();
        }
        const int j = 2 * hf + jg;  // this warp's 32-column chunk of the half
        uint32_t sr[32], dp[32];
        tmem_ld16(tbase + lane_base + 32 * j, *reinterpret_cast<uint32_t(*)[16]>(sr));
        tmem_ld16(tbase + lane_base + 32 * j + 16, *reinterpret_cast<uint32_t(*)[16]>(sr + 16));
        tmem_ld16(tbase + lane_base + 128 + 32 * j, *reinterpret_cast<uint32_t(*)[16]>(dp));
        tmem_ld16(tbase + lane_base + 128 + 32 * j + 16, *reinterpret_cast<uint32_t(*)[16]>(dp + 16));
        tmem_wait_ld();
        const int ib = i0 + 32 * j;     // first query row of this word
        const int qbase = ib + qshift;  // its logical position
        uint32_t bits = 0xFFFFFFFFu;
        if (need_mask) {
          uint32_t same = 0xFFFFFFFFu;
          if (is_doc) {
            same = 0u;
#pragma unroll
            for (int c = 0; c < 32; ++c) same |= (s_doc[cnt & 1][32 * j + c] == my_doc ? 1u : 0u) << c;
            same &= span_bits(-qbase, 31);  // queries at q >= 0 only
          }
          bits = is_prog ? program_bits_q(a.mask, h, kv, qbase, same) : (fixed_bits_q(a.mask, kv, qbase) & same);
          bits &= span_bits(-1, a.L - 1 - ib);  // query rows past L
          if (!key_ok) bits = 0u;
        }
        const float* lq = s_lse[cnt & 1] + 32 * j;
        const float* dq = s_dsum[cnt & 1] + 32 * j;
        const float* pqv = s_pq[cnt & 1] + 32 * j;
        const float bias0 = slope2 * static_cast<float>(kv - qbase);  // slope2 (kv - q) at c = 0
        float th[32];
        if constexpr (kCapped) tanh32(sr, c_in, th);
        // four columns per step: their query-side values in one 16-byte load
        // each, the arithmetic in f32x2 pairs
        uint32_t ppk[16], dpk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lq + i);
          const float4 d4 = *reinterpret_cast<const float4*>(dq + i);
          float4 q4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          if constexpr (SCORE == FA_SCORE_CAP_THEN_BIAS)
            if (has_pos) q4 = *reinterpret_cast<const float4*>(pqv + i);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int c = i + 2 * hh;
            const float2 lq2 = hh ? make_float2(l4.z, l4.w) : make_float2(l4.x, l4.y);
            const float2 dq2 = hh ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
            const float2 col = make_float2(static_cast<float>(c), static_cast<float>(c + 1));
            float2 bias = splat2(0.0f);
            if constexpr (SCORE == FA_SCORE_ALIBI) bias = fma2(splat2(-slope2), col, splat2(bias0));
            if constexpr (SCORE == FA_SCORE_CAP_THEN_BIAS) {
              const float2 pq2 = hh ? make_float2(q4.z, q4.w) : make_float2(q4.x, q4.y);
              bias = has_pos ? mul2(splat2(slope2), add2(splat2(pk_raw), make_float2(-pq2.x, -pq2.y)))
                             : fma2(splat2(-slope2), col, splat2(bias0));
            }
            float2 t, gp = splat2(1.0f);
            if constexpr (kCapped) {
              const float2 th2 = make_float2(th[c], th[c + 1]);
              t = fma2(th2, splat2(c_out), bias);
              gp = fma2(make_float2(-th2.x, -th2.y), th2, splat2(1.0f));
            } else {
              t = fma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), splat2(c_out), bias);
            }
            const float2 e = add2(t, make_float2(-lq2.x, -lq2.y));
            const float2 p = make_float2(((bits >> c) & 1u) ? ex2_approx(e.x) : 0.0f,
                                         ((bits >> (c + 1)) & 1u) ? ex2_approx(e.y) : 0.0f);
            float2 d = mul2(p, add2(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])),
                                    make_float2(-dq2.x, -dq2.y)));
            if constexpr (kCapped) d = mul2(d, gp);
            ppk[c >> 1] = pack_bf16x2(p.x, p.y);
            dpk[c >> 1] = pack_bf16x2(d.x, d.y);
          }
        }
        // P^T and dS^T of these 32 queries as bf16 pairs over columns already read
        tmem_st16(tbase + lane_base + 32 * j, ppk);
        tmem_st16(tbase + lane_base + 128 + 32 * j, dpk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[hf]);
      }
    }
    // epilogue: dv = dV, dk = scale dK (zero for a key tile no query lists)
    if (alive && cnt > 0) {
      alive = mbar_wait(&bars.o_final, 0, abort, a.status, a.wait_cycles);
      tc_fence_after();
    }
    if (__all_sync(0xffffffffu, alive)) {
      const bool row_ok = kv < a.S;
      const int kvr = row_ok ? kv : 0;
      {
        const int which = jg;  // math group 0 writes dV, group 1 dK
        void* base = which ? a.dk : a.dv;
        const int64_t* st = which ? a.dk_stride : a.dv_stride;
        const bool f32 = which ? a.dk_f32 : a.dv_f32;
        const float mul = which ? a.scale : 1.0f;
        const int64_t off = b * st[0] + hk * st[1] + static_cast<int64_t>(kvr) * st[2];
        // 64 columns per wait (four loads in flight)
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
          uint32_t rr[4][16];
          if (total > 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) tmem_ld16(tbase + lane_base + 256 + which * D + (4 * cb + i) * 16, rr[i]);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 4; ++i) hold16(rr[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int e = 0; e < 16; ++e) rr[i][e] = 0u;
          }
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 4; ++i) store16(base, off + (4 * cb + i) * 16, f32, rr[i], mul);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}

// D = rowsum(dout * out) in fp32.  Each thread reads 8 elements of a row
// with one 16-byte load from each tensor, E / 8 neighbouring lanes share a
// row (8 or 16), and a shuffle tree over those lanes sums it: 256 / (E / 8)
// rows of one (batch, head) per CTA, grid (row blocks, Hq, B).
__global__ void __launch_bounds__(256) bwd_dsum_kernel(const BwdArgs a) {
  const int lg = a.E == 64 ? 3 : 4;  // log2 of the threads per row
  const int tpr = 1 << lg;
  const int i = blockIdx.x * (256 >> lg) + (threadIdx.x >> lg);
  const int part = threadIdx.x & (tpr - 1);
  const int h = blockIdx.y, b = blockIdx.z;
  float acc = 0.0f;
  if (i < a.L) {
    const __nv_bfloat16* o =
        static_cast<const __nv_bfloat16*>(a.out) + b * a.o_stride[0] + h * a.o_stride[1] + i * a.o_stride[2];
    const __nv_bfloat16* d =
        static_cast<const __nv_bfloat16*>(a.dout) + b * a.do_stride[0] + h * a.do_stride[1] + i * a.do_stride[2];
    const uint4 ov = __ldg(reinterpret_cast<const uint4*>(o) + part);
    const uint4 dv = __ldg(reinterpret_cast<const uint4*>(d) + part);
    const __nv_bfloat162* op = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* dp = reinterpret_cast<const __nv_bfloat162*>(&dv);
    float2 s2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < 4; ++j) s2 = fma2(__bfloat1622float2(op[j]), __bfloat1622float2(dp[j]), s2);
    acc = s2.x + s2.y;
  }
  for (int off = tpr >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (i < a.L && part == 0) a.dsum[(static_cast<int64_t>(b) * a.Hq + h) * a.L + i] = acc;
}

// Query-side lists: one thread per key tile n of row set (b, h).
__global__ void __launch_bounds__(128) transpose_kernel(const TransposeArgs a) {
  // one warp per key tile n: lane l tests rows m = l, l + 32, ... (a binary
  // search of each ascending list), and ballots keep the rows in order
  const int b = blockIdx.y, h = blockIdx.z;
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (n >= a.Nb) return;
  const int64_t kv_row0 = (static_cast<int64_t>(b) * a.H + h) * a.Mb;
  const int64_t qr = (static_cast<int64_t>(b) * a.H + h) * a.Nb + n;
  auto listed = [&](const int* idx, int cnt) {
    int lo = 0, hi = cnt - 1;
    while (lo <= hi) {
      const int mid = (lo + hi) >> 1;
      const int x = idx[mid];
      if (x == n) return true;
      if (x < n) lo = mid + 1;
      else hi = mid - 1;
    }
    return false;
  };
  int np = 0, nf = 0;
  const unsigned below = (1u << lane) - 1u;
  for (int m0 = 0; m0 < a.Mb; m0 += 32) {
    const int m = m0 + lane;
    bool in_p = false, in_f = false;
    if (m < a.Mb) {
      const int64_t kr = kv_row0 + m;
      in_f = listed(a.full_kv_indices + kr * a.Nb, a.full_kv_num_blocks[kr]);
      in_p = !in_f && listed(a.kv_indices + kr * a.Nb, a.kv_num_blocks[kr]);
    }
    const unsigned bp = __ballot_sync(0xffffffffu, in_p), bf = __ballot_sync(0xffffffffu, in_f);
    if (in_p) a.q_indices[qr * a.Mb + np + __popc(bp & below)] = m;
    if (in_f) a.full_q_indices[qr * a.Mb + nf + __popc(bf & below)] = m;
    np += __popc(bp);
    nf += __popc(bf);
  }
  if (lane == 0) {
    a.q_num_blocks[qr] = np;
    a.full_q_num_blocks[qr] = nf;
  }
  for (int m = np + lane; m < a.Mb; m += 32) a.q_indices[qr * a.Mb + m] = 0;
  for (int m = nf + lane; m < a.Mb; m += 32) a.full_q_indices[qr * a.Mb + m] = 0;
}

template <int D, int SCORE>
cudaError_t launch_bwd_one(const BwdArgs& a, const BwdMaps& maps, cudaStream_t stream) {
  auto kdq = bwd_dq_kernel<D, SCORE>;
  auto kkv = bwd_dkdv_kernel<D, SCORE>;
  cudaError_t e = cudaFuncSetAttribute(kdq, cudaFuncAttributeMaxDynamicSharedMemorySize, BCfg<D>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, BCfg<D>::kSmemBytes);
  if (e != cudaSuccess) return e;
  kdq<<<dim3(a.Hq, a.B, a.bm.Mb), kBwdThreads, BCfg<D>::kSmemBytes, stream>>>(a, maps.q, maps.k, maps.v, maps.dout);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kkv<<<dim3(a.Hkv, a.B, a.bm.Nb), kBwdThreads, BCfg<D>::kSmemBytes, stream>>>(a, maps.q, maps.k, maps.v, maps.dout);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_d(const BwdArgs& a, const BwdMaps& maps, cudaStream_t stream) {
  switch (a.score.kind) {
    case FA_SCORE_NONE: return launch_bwd_one<D, FA_SCORE_NONE>(a, maps, stream);
    case FA_SCORE_SOFTCAP: return launch_bwd_one<D, FA_SCORE_SOFTCAP>(a, maps, stream);
    case FA_SCORE_ALIBI: return launch_bwd_one<D, FA_SCORE_ALIBI>(a, maps, stream);
    default: return launch_bwd_one<D, FA_SCORE_CAP_THEN_BIAS>(a, maps, stream);
  }
}

}  // namespace

cudaError_t launch_bwd(const BwdArgs& a, const BwdMaps& maps, cudaStream_t stream) {
  const int rows_per_cta = 256 / (a.E >> 3);
  bwd_dsum_kernel<<<dim3((a.L + rows_per_cta - 1) / rows_per_cta, a.Hq, a.B), 256, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return a.E == 64 ? launch_bwd_d<64>(a, maps, stream) : launch_bwd_d<128>(a, maps, stream);
}

cudaError_t launch_transpose(const TransposeArgs& a, cudaStream_t stream) {
  dim3 grid((a.Nb + 3) / 4, a.B, a.H);  // four warps (key tiles) per CTA
  transpose_kernel<<<grid, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fa
