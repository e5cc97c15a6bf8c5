// Host-side launch interfaces between the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mods.cuh"

namespace fa {

struct ClassifyArgs {
  int* status;  // device status word
  MaskParams mask;
  int B, H, L, S, BM, BN, Mb, Nb;
  int* kv_num_blocks;
  int* kv_indices;
  int* full_kv_num_blocks;
  int* full_kv_indices;
};
cudaError_t launch_classify(const ClassifyArgs& a, cudaStream_t stream);

// Read-only view of a BlockMask; B and H may be 1 (broadcast).
struct BlockMaskView {
  int B, H, Mb, Nb, BM, BN;
  const int* kv_num_blocks;
  const int* kv_indices;
  const int* full_kv_num_blocks;
  const int* full_kv_indices;
};

struct FwdArgs {
  int* status;  // device status word
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;                 // [B, Hq, L] or null
  float* max_scores;          // [B, Hq, L] or null
  long long wait_cycles;      // budget of each main-path device wait
  int out_f32;                // out is fp32 (else the input dtype)
  int rows_safe;              // every row has a visible key: no empty-row guard
  // paged KV cache (page_table == null: k, v are (B, Hkv, S, D)): logical key
  // j of sequence b is slot j % page_size of page page_table[b * pages_per_seq
  // + j / page_size] of the pools k, v (num_pages, Hkv, page_size, D)
  const int* page_table;
  int page_size, pages_per_seq, num_pages;
  int64_t q_stride[4], k_stride[4], v_stride[4], o_stride[4];
  int B, Hq, Hkv, L, S, E, Ev, G;
  int dtype;                  // FA_DTYPE_*
  float scale;
  MaskParams mask;
  ScoreParams score;
  BlockMaskView bm;
};

// General kernel: any dtype, tiles up to 128 x 128, head dims up to 128.
cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t stream);

// Tensor-core prefill kernel (bf16, BM = BN = 128, E = Ev in {64, 128}).
struct Sm100Maps {
  CUtensorMap q, k, v;
};
// One CTA per pair of query tiles, persistent through cluster launch control.
cudaError_t launch_fwd_sm100(const FwdArgs& a, const Sm100Maps& maps, cudaStream_t stream);

// Split-KV decode for short queries (bf16, E = Ev in {64, 128}, L <= 16) and
// the log-sum-exp combination of its partial results.
struct DecodePlan {
  int rows_per_cta;     // query rows one CTA handles (heads of a group x L), <= 16
  int heads_per_cta;    // query heads per CTA
  int splits;           // KV splits per (b, head group)
  int tiles_per_split;  // listed tiles per split
  size_t workspace_bytes;
};
constexpr int kDecodeMaxRows = 16;
int plan_decode(const FwdArgs& a, int split_kv, int num_sms, DecodePlan* plan);
cudaError_t launch_decode(const FwdArgs& a, const DecodePlan& plan, const Sm100Maps& maps, void* workspace,
                          cudaStream_t stream);

// Backward pass (bf16, E = Ev in {64, 128}, 128 x 128 tiles).
struct BwdArgs {
  int* status;  // device status word
  long long wait_cycles;
  const void *q, *k, *v, *out, *dout;
  const float* lse;  // [B, Hq, L] from the forward pass
  float* dsum;       // workspace: D = rowsum(dout * out), [B, Hq, L]
  void *dq, *dk, *dv;
  int64_t q_stride[4], k_stride[4], v_stride[4], o_stride[4], do_stride[4];
  int64_t dq_stride[4], dk_stride[4], dv_stride[4];
  int dq_f32, dk_f32, dv_f32;  // gradient storage: fp32, else bf16
  int B, Hq, Hkv, L, S, E, G;
  float scale;
  MaskParams mask;
  ScoreParams score;
  BlockMaskView bm;  // key-side lists (the forward's)
  // query-side lists: for key tile n of row (b, h), the query tiles listing it
  int qB, qH;
  const int *q_num_blocks, *q_indices, *full_q_num_blocks, *full_q_indices;
};
struct BwdMaps {
  CUtensorMap q, k, v, dout;
};
cudaError_t launch_bwd(const BwdArgs& a, const BwdMaps& maps, cudaStream_t stream);

// Query-side lists from the key-side lists of a BlockMask.
struct TransposeArgs {
  int B, H, Mb, Nb;
  const int *kv_num_blocks, *kv_indices, *full_kv_num_blocks, *full_kv_indices;
  int *q_num_blocks, *q_indices, *full_q_num_blocks, *full_q_indices;
};
cudaError_t launch_transpose(const TransposeArgs& a, cudaStream_t stream);

}  // namespace fa
