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
__global__ void __launch_bounds__(kSimtThreads) fwd_simt_kernel(FwdArgs a) {
  extern __shared__ float smem[];
  const int mt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x;
  const int BM = a.bm.BM, BN = a.bm.BN;
  const int E = a.E, Ev = a.Ev;
  const int qst = E | 1, ost = Ev | 1;  // odd row strides: no bank conflicts across rows
  float* sq = smem;
  float* so = sq + BM * qst;
  float* sk = so + BM * ost;
  float* sv = sk + kChunk * E;

  const int hk = h / a.G;
  const int S = a.S, L = a.L;
  const int S_b = seq_len_b(a.mask, b, S);
  const int r0 = mt * BM;
  const T* qb = static_cast<const T*>(a.q) + b * a.q_stride[0] + h * a.q_stride[1];
  const T* kb = static_cast<const T*>(a.k) + b * a.k_stride[0] + hk * a.k_stride[1];
  const T* vb = static_cast<const T*>(a.v) + b * a.v_stride[0] + hk * a.v_stride[1];

  for (int i = t; i < BM * E; i += blockDim.x) {
    const int r = i / E, e = i % E;
    sq[r * qst + e] = (r0 + r < L) ? to_f(qb[(r0 + r) * a.q_stride[2] + e]) : 0.0f;
  }
  for (int i = t; i < BM * Ev; i += blockDim.x) so[(i / Ev) * ost + i % Ev] = 0.0f;

  const int row = r0 + t;
  const bool active = t < BM && row < L;
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
      float s[kChunk];
      float cmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        float val = -INFINITY;
        if (j < nk) {
          float dot = 0.0f;
          for (int e = 0; e < E; ++e) dot = fmaf(sq[t * qst + e], sk[j * E + e], dot);
          const int kv = cc + j;
          const float g = score_apply<true>(a.score, dot * a.scale, b, qpos, kv, S, slope);
          const bool vis = is_full ? (kv < S_b) : mask_visible(a.mask, b, h, qpos, kv, S_b, S);
          val = vis ? g : -INFINITY;
        }
        s[j] = val;
        cmax = fmaxf(cmax, val);
      }
      const float m_new = fmaxf(m_run, cmax);
      const float alpha = expf(m_run - m_new);
      float psum = 0.0f;
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        s[j] = expf(s[j] - m_new);
        psum += s[j];
      }
      l_run = l_run * alpha + psum;
      for (int d = 0; d < Ev; ++d) {
        float acc = so[t * ost + d] * alpha;
#pragma unroll
        for (int j = 0; j < kChunk; ++j) acc = fmaf(s[j], (j < nk) ? sv[j * Ev + d] : 0.0f, acc);
        so[t * ost + d] = acc;
      }
      m_run = m_new;
    }
  }
  if (!active) return;
  const int64_t ooff = b * a.o_stride[0] + h * a.o_stride[1] + row * a.o_stride[2];
  // a row without a visible key has l_run = 0: out 0 and lse -inf, unless the
  // caller promised there is none (rows_safe), which drops this guard
  const bool live = a.rows_safe || l_run > 0.0f;
  const float inv = live ? 1.0f / l_run : 0.0f;
  if (a.out_f32) {
    float* ob = static_cast<float*>(a.out) + ooff;
    for (int d = 0; d < Ev; ++d) ob[d] = live ? so[t * ost + d] * inv : 0.0f;
  } else {
    T* ob = static_cast<T*>(a.out) + ooff;
    for (int d = 0; d < Ev; ++d) store_out<T>(ob + d, live ? so[t * ost + d] * inv : 0.0f);
  }
  const int64_t rid = (static_cast<int64_t>(b) * a.Hq + h) * L + row;
  if (a.lse) a.lse[rid] = live ? m_run + logf(l_run) : -INFINITY;
  if (a.max_scores) a.max_scores[rid] = m_run > kNoKeyMaxS ? m_run : -INFINITY;  // the exact running maximum
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t stream) {
  const int BM = a.bm.BM;
  const size_t smem = sizeof(float) * (static_cast<size_t>(BM) * ((a.E | 1) + (a.Ev | 1)) +
                                       static_cast<size_t>(kChunk) * (a.E + a.Ev));
  dim3 grid(a.bm.Mb, a.Hq, a.B);
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
