// General forward kernel on the CUDA cores: any element type, any tile sizes up
// to 128 x 128, head dimensions up to 128.  It serves the fp32 path (where the
// tensor cores' tf32 rounding would miss a 1e-5 tolerance) and tile shapes the
// tensor-core kernel does not take (tiny teaching tiles, odd lengths).
//
// Per CTA: one query tile (b, h, m) with one thread per query row.  The CTA
// walks the row's full tiles, then its partial tiles, as listed in the
// BlockMask, 32 keys at a time staged in shared memory as fp32.  For each
// chunk a thread computes the 32 scaled scores of its row, applies the score
// rule, then (partial tiles, and keys past the valid length) the element
// mask, and folds the chunk into its running max / sum / output with an
// online softmax.  Definition: "flexattention-score-mod-block-mask"
// (charlestar.github.io), "What one connection goes through" and "mask_mod
// defines legal connections, BlockMask defines block work" (full tiles skip
// the element mask, partial tiles apply it after the score rule).
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "mods.cuh"

namespace fa {

namespace {

constexpr int kSimtThreads = 128;
constexpr int kChunk = 32;
constexpr int kSimtRows = 8;  // query rows per CTA: a query tile spreads over BM / 8 CTAs

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ void store_out(T* p, float x);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename T>
__global__ void __launch_bounds__(kSimtThreads, 1) fwd_simt_kernel(FwdArgs a) {
  extern __shared__ float smem[];
  const int h = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x;
  const int BM = a.bm.BM, BN = a.bm.BN;
  const int E = a.E, Ev = a.Ev;
  // A CTA takes RB = min(BM, 8) rows of query tile mt; R = 128 / RB threads
  // per row: thread t takes row t % RB and the keys j = sub (mod R) of every
  // chunk, sub = t / RB; the R partial (max, sum, O) of a row are merged at
  // the end.
  const int RB = BM < kSimtRows ? BM : kSimtRows;
  const int nsplit = (BM + RB - 1) / RB;
  const int mt = blockIdx.x / nsplit, part = blockIdx.x % nsplit;
  const int R = kSimtThreads / RB;
  const int qst = E | 1, ost = Ev | 1;  // odd row strides: no bank conflicts across rows
  float* sq = smem;
  float* so = sq + RB * qst;             // [R][RB] partial O rows
  float* sk = so + R * RB * ost;
  float* sv = sk + kChunk * E;
  float* sml = sv + kChunk * Ev;          // [R][RB] partial max, then [R][RB] partial sum
  float* ss = sml + 2 * R * RB;           // [128][kChunk + 1] each thread's chunk scores

  const int hk = h / a.G;
  const int S = a.S, L = a.L;
  const int S_b = seq_len_b(a.mask, b, S);
  const int r0 = mt * BM + part * RB;                     // first row of this CTA
  const int r_end = min(mt * BM + BM, L);                 // end of the tile's rows
  const T* qb = static_cast<const T*>(a.q) + b * a.q_stride[0] + h * a.q_stride[1];
  const T* kb = static_cast<const T*>(a.k) + b * a.k_stride[0] + hk * a.k_stride[1];
  const T* vb = static_cast<const T*>(a.v) + b * a.v_stride[0] + hk * a.v_stride[1];

  for (int i = t; i < RB * E; i += blockDim.x) {
    const int r = i / E, e = i % E;
    sq[r * qst + e] = (r0 + r < r_end) ? to_f(qb[(r0 + r) * a.q_stride[2] + e]) : 0.0f;
  }
  for (int i = t; i < R * RB * Ev; i += blockDim.x) so[(i / Ev) * ost + i % Ev] = 0.0f;

  const int rr = t % RB, sub = t / RB;
  const int row = r0 + rr;
  const bool active = sub < R && row < r_end;
  float* orow = so + (sub * RB + rr) * ost;
  const float* qrow = sq + rr * qst;
  const int qpos = query_pos(row, L, S_b);
  const int Hs = a.score.slope_heads > 0 ? a.score.slope_heads : a.Hq;
  const float slope = distance_slope(h, Hs);
  // running maximum from a finite floor below any real score: hidden keys
  // give exp(-inf) = 0 with no test of the maximum
  constexpr float kNoKeyMaxS = -1.0e30f;
  float m_run = kNoKeyMaxS, l_run = 0.0f;

  const int bmb = a.bm.B > 1 ? b : 0, bmh = a.bm.H > 1 ? h : 0;
  const int64_t brow = (static_cast<int64_t>(bmb) * a.bm.H + bmh) * a.bm.Mb + mt;
  const int nfull = a.bm.full_kv_num_blocks[brow];
  const int npart = a.bm.kv_num_blocks[brow];

  for (int it = 0; it < nfull + npart; ++it) {
    const bool is_full = it < nfull;
    const int n = is_full ? a.bm.full_kv_indices[brow * a.bm.Nb + it] : a.bm.kv_indices[brow * a.bm.Nb + it - nfull];
    const int cb = n * BN;
    const int ce = min(S, cb + BN);
    for (int cc = cb; cc < ce; cc += kChunk) {
      const int nk = min(kChunk, ce - cc);
      __syncthreads();
      if (a.page_table) {
        // paged pools: key j is slot j % page_size of its page
        const T* kp = static_cast<const T*>(a.k) + hk * a.k_stride[1];
        const T* vp = static_cast<const T*>(a.v) + hk * a.v_stride[1];
        for (int i = t; i < nk * E; i += blockDim.x) {
          const int j = cc + i / E;
          const int pg = cache_page(a.page_table, a.pages_per_seq, a.page_size, a.num_pages, a.status, b, j);
          sk[i] = to_f(kp[pg * a.k_stride[0] + (j % a.page_size) * a.k_stride[2] + i % E]);
        }
        for (int i = t; i < nk * Ev; i += blockDim.x) {
          const int j = cc + i / Ev;
          const int pg = cache_page(a.page_table, a.pages_per_seq, a.page_size, a.num_pages, a.status, b, j);
          sv[i] = to_f(vp[pg * a.v_stride[0] + (j % a.page_size) * a.v_stride[2] + i % Ev]);
        }
      } else {
        for (int i = t; i < nk * E; i += blockDim.x) sk[i] = to_f(kb[(cc + i / E) * a.k_stride[2] + i % E]);
        for (int i = t; i < nk * Ev; i += blockDim.x) sv[i] = to_f(vb[(cc + i / Ev) * a.v_stride[2] + i % Ev]);
      }
      __syncthreads();
      if (!active) continue;
      // this thread's keys of the chunk: j = sub, sub + R, ...
      const int mine = nk > sub ? (nk - sub + R - 1) / R : 0;
      // the scores live in shared memory, so the loops stay rolled (this
      // kernel is bound by latency, and unrolled it overflows the
      // instruction cache)
      float* s = ss + t * (kChunk + 1);
      float cmax = -INFINITY;
#pragma unroll 1
      for (int u = 0; u < mine; ++u) {
        const int j = sub + u * R;
        const float* krow = sk + j * E;
        float d0 = 0.0f, d1 = 0.0f, d2 = 0.0f, d3 = 0.0f;  // four chains
        int e = 0;
#pragma unroll 1
        for (; e + 4 <= E; e += 4) {
          d0 = fmaf(qrow[e], krow[e], d0);
          d1 = fmaf(qrow[e + 1], krow[e + 1], d1);
          d2 = fmaf(qrow[e + 2], krow[e + 2], d2);
          d3 = fmaf(qrow[e + 3], krow[e + 3], d3);
        }
        for (; e < E; ++e) d0 = fmaf(qrow[e], krow[e], d0);
        const float dot = (d0 + d1) + (d2 + d3);
        const int kv = cc + j;
        const float g = score_apply<true>(a.score, dot * a.scale, b, qpos, kv, S, slope);
        const bool vis = is_full ? (kv < S_b) : mask_visible(a.mask, b, h, qpos, kv, S_b, S);
        s[u] = vis ? g : -INFINITY;
        cmax = fmaxf(cmax, s[u]);
      }
      const float m_new = fmaxf(m_run, cmax);
      const float alpha = expf(m_run - m_new);
      float psum = 0.0f;
#pragma unroll 1
      for (int u = 0; u < mine; ++u) {
        s[u] = expf(s[u] - m_new);
        psum += s[u];
      }
      l_run = l_run * alpha + psum;
      for (int d = 0; d < Ev; ++d) {
        float acc0 = orow[d] * alpha, acc1 = 0.0f;
        int u = 0;
#pragma unroll 1
        for (; u + 2 <= mine; u += 2) {
          acc0 = fmaf(s[u], sv[(sub + u * R) * Ev + d], acc0);
          acc1 = fmaf(s[u + 1], sv[(sub + (u + 1) * R) * Ev + d], acc1);
        }
        if (u < mine) acc0 = fmaf(s[u], sv[(sub + u * R) * Ev + d], acc0);
        orow[d] = acc0 + acc1;
      }
      m_run = m_new;
    }
  }
  // merge the R partials of each row: thread sub 0 of the row writes it
  __syncthreads();
  if (sub < R) {
    sml[sub * RB + rr] = m_run;
    sml[(R + sub) * RB + rr] = l_run;
  }
  __syncthreads();
  if (!active || sub != 0) return;
  float m = sml[rr];
  for (int r = 1; r < R; ++r) m = fmaxf(m, sml[r * RB + rr]);
  float l = 0.0f;
  for (int r = 0; r < R; ++r) l += sml[(R + r) * RB + rr] * expf(sml[r * RB + rr] - m);
  const int64_t ooff = b * a.o_stride[0] + h * a.o_stride[1] + row * a.o_stride[2];
  // a row without a visible key has l = 0: out 0 and lse -inf, unless the
  // caller promised there is none (rows_safe), which drops this guard
  const bool live = a.rows_safe || l > 0.0f;
  const float inv = live ? 1.0f / l : 0.0f;
  for (int d = 0; d < Ev; ++d) {
    float o = 0.0f;
    for (int r = 0; r < R; ++r) o += so[(r * RB + rr) * ost + d] * expf(sml[r * RB + rr] - m);
    const float val = live ? o * inv : 0.0f;
    if (a.out_f32)
      static_cast<float*>(a.out)[ooff + d] = val;
    else
      store_out<T>(static_cast<T*>(a.out) + ooff + d, val);
  }
  const int64_t rid = (static_cast<int64_t>(b) * a.Hq + h) * L + row;
  if (a.lse) a.lse[rid] = live ? m + logf(l) : -INFINITY;
  if (a.max_scores) a.max_scores[rid] = m > kNoKeyMaxS ? m : -INFINITY;  // the exact running maximum
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t stream) {
  const int BM = a.bm.BM;
  const int RB = BM < kSimtRows ? BM : kSimtRows;
  const int R = kSimtThreads / RB;
  const size_t smem = sizeof(float) * (static_cast<size_t>(RB) * ((a.E | 1) + R * (a.Ev | 1)) +
                                       static_cast<size_t>(kChunk) * (a.E + a.Ev) + 2 * R * RB +
                                       static_cast<size_t>(kSimtThreads) * (kChunk + 1));
  dim3 grid(a.bm.Mb * ((BM + RB - 1) / RB), a.Hq, a.B);
  cudaError_t e;
  if (a.dtype == FA_DTYPE_F32) {
    e = cudaFuncSetAttribute(fwd_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    fwd_simt_kernel<float><<<grid, kSimtThreads, smem, stream>>>(a);
  } else {
    e = cudaFuncSetAttribute(fwd_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    fwd_simt_kernel<__nv_bfloat16><<<grid, kSimtThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace fa
