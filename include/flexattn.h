/*
 * flexattn.h -- C ABI of the B200 (sm_100a) FlexAttention forward library.
 *
 * The library computes the forward pass of programmable block-sparse attention
 * and the BlockMask that drives it.  Definitions follow these pages (cited by
 * title and section):
 *
 *   [charlestar]  "flexattention-score-mod-block-mask" (charlestar.github.io)
 *   [guide]       "PyTorch Flex Attention complete guide: from score_mod to
 *                 BlockMask" (2kiu.com)
 *   [expressions] "Attention expressions" (docs.tensorcad.dev)
 *   [causal]      "Causal Mask" (quant67.com, Transformer series no. 17)
 *
 * Conventions shared by every entry point:
 *   - Every pointer to tensor data is DEVICE memory owned by the caller.  The
 *     library keeps no pointer after a call returns and allocates no device
 *     memory during a call: scratch comes from the caller's workspace, except
 *     in flexattn_forward_decode_noalloc, which uses a fixed array the library
 *     holds for that purpose.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Host-side argument checks happen
 *     before anything is enqueued; on an error nothing is enqueued.
 *   - Every call returns an int status: FA_OK (0) or one of FA_ERR_*.  No call
 *     throws or aborts.  flexattn_last_error() gives a message for the last
 *     failing call on the calling thread.
 *   - flexattn_build_block_mask, flexattn_forward and
 *     flexattn_forward_decode_noalloc only enqueue kernels, so a stream
 *     capture of them (CUDA graphs, relaxed capture mode) replays the same
 *     work; flexattn_poll_device_status synchronises and must stay outside a
 *     capture.
 *   - Integers on the device are int32; the host-side struct sizes are int32.
 */
#ifndef FLEXATTN_H_
#define FLEXATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ----------------------------------------------------------------------- */
/* Status codes                                                             */
/* ----------------------------------------------------------------------- */
enum {
  FA_OK = 0,
  FA_ERR_NULL = 1,         /* a required pointer is NULL                                   */
  FA_ERR_SHAPE = 2,        /* a size is non-positive, above 65535 for batch or heads, or sizes disagree */
  FA_ERR_HEADS = 3,        /* Hq != Hkv without enable_gqa, or Hq % Hkv != 0 ([guide] 1.3, 6.1) */
  FA_ERR_BATCH = 4,        /* batch sizes disagree, or a broadcast extent is neither 1 nor B    */
  FA_ERR_MASK_SHAPE = 5,   /* block mask built for other lengths/blocks: "too small / too large" ([guide] 1.3) */
  FA_ERR_DTYPE = 6,        /* unsupported or mismatched element type                        */
  FA_ERR_HEADDIM = 7,      /* head dimension outside what the kernels support              */
  FA_ERR_ALIGN = 8,        /* base pointer or stride not 16-byte aligned, or last stride != 1 */
  FA_ERR_PARAM = 9,        /* an invalid mod parameter (cap <= 0, window < 1, NULL doc_id, ...) */
  FA_ERR_WORKSPACE = 10,   /* workspace NULL or smaller than flexattn_forward_workspace_size() */
  FA_ERR_UNSUPPORTED = 11, /* a valid combination that no kernel implements                 */
  FA_ERR_CUDA = 12,        /* a CUDA runtime call failed (message in flexattn_last_error)  */
  FA_ERR_TIMEOUT = 13      /* a bounded device-side wait ran out (see flexattn_poll_device_status) */
};

/* ----------------------------------------------------------------------- */
/* Element types                                                            */
/* ----------------------------------------------------------------------- */
enum {
  FA_DTYPE_BF16 = 0, /* bfloat16 storage, fp32 arithmetic and accumulation  */
  FA_DTYPE_F32 = 1   /* fp32 storage and arithmetic                         */
};

/* ----------------------------------------------------------------------- */
/* mask_mod menu: M(b, h, q, kv) -> visible?                                */
/*                                                                          */
/* q is the LOGICAL query position q = i + (S_b - L) for query row i, where */
/* S_b is the valid KV length of sequence b (kv_len[b], or S when kv_len is */
/* NULL): causal alignment is bottom-right when L < S ([causal] section 4;  */
/* [charlestar] "At decode, q_idx = 0 is not position 0").  kv = j is the   */
/* key position.  Keys j >= S_b are invisible under every kind.             */
/* ----------------------------------------------------------------------- */
enum {
  FA_MASK_NONE = 0,           /* every key < S_b ([guide] 4.4, noop_mask)                          */
  FA_MASK_CAUSAL = 1,         /* kv <= q                                                           */
  FA_MASK_SLIDING_WINDOW = 2, /* kv <= q && (q - kv < window || kv < n_sink)  ([charlestar] "A call
                                 example pinned to one version": 0 <= p_i - p_j < W, self included;
                                 [expressions] "Examples": a window that keeps sink tokens)      */
  FA_MASK_DOCUMENT = 3,       /* kv <= q && doc_id[b][q] == doc_id[b][kv]  ([charlestar] "Packing") */
  FA_MASK_PREFIX_LM = 4,      /* kv <= q || kv < prefix   (causal off; [expressions] "Examples")   */
  FA_MASK_CHUNKED = 5,        /* kv <= q && q / chunk == kv / chunk  ([expressions] "Examples")    */
  FA_MASK_PROGRAM = 6         /* a composed rule: fa_mask_mod.program (below)                      */
};

/* Instructions of a composed rule ([guide] 4.3: and_masks / or_masks combine
 * any number of rules by intersection or union; [expressions] "Examples":
 * every fourth key, half the heads global and half local), in postfix order:
 * a predicate pushes its verdict for the pair (q, kv) of query head h,
 * FA_PROG_AND / FA_PROG_OR pop two verdicts and push one, FA_PROG_NOT
 * negates the top; one verdict must remain.  No predicate carries a causal
 * bound of its own (add FA_PROG_CAUSAL), and keys kv >= S_b stay invisible
 * whatever the program says.  The library rewrites the program as an AND of
 * at most 8 clauses, each an OR of at most 4 predicates or their negations;
 * a program that needs more returns FA_ERR_UNSUPPORTED. */
enum {
  FA_PROG_TRUE = 0,           /* every pair                                                    */
  FA_PROG_CAUSAL = 1,         /* kv <= q                                                       */
  FA_PROG_DISTANCE_BELOW = 2, /* q - kv < arg                                                  */
  FA_PROG_KEY_BELOW = 3,      /* kv < arg                                                      */
  FA_PROG_SAME_CHUNK = 4,     /* floor(q / arg) == floor(kv / arg), arg >= 1                   */
  FA_PROG_SAME_DOCUMENT = 5,  /* 0 <= q < S and doc_id[b][q] == doc_id[b][kv] (doc_id needed)  */
  FA_PROG_STRIDE = 6,         /* q - kv is a multiple of arg, arg >= 1                         */
  FA_PROG_HEAD_BELOW = 7,     /* h < arg (h is the query head): a head-dependent rule          */
  FA_PROG_AND = 16,
  FA_PROG_OR = 17,
  FA_PROG_NOT = 18
};

#define FA_MASK_PROGRAM_MAX 16

typedef struct fa_mask_instr {
  int32_t op;            /* FA_PROG_*                                                      */
  int32_t arg;           /* the predicate's parameter (unused by the others)               */
} fa_mask_instr;

typedef struct fa_mask_mod {
  int32_t kind;          /* FA_MASK_*                                                       */
  int32_t window;        /* SLIDING_WINDOW: W >= 1 keys, the query included                 */
  int32_t n_sink;        /* SLIDING_WINDOW: keys kv < n_sink stay visible (>= 0)            */
  int32_t prefix;        /* PREFIX_LM: P >= 0                                               */
  int32_t chunk;         /* CHUNKED: C >= 1                                                 */
  int32_t doc_batch;     /* DOCUMENT: rows of doc_id, 1 (broadcast) or B                     */
  const int32_t* doc_id; /* DOCUMENT: device int32 [doc_batch, S], document id per position  */
  const int32_t* kv_len; /* optional device int32 [B]: valid KV length per sequence, values in
                            [0, S] (clamped to that range); NULL means S for every sequence  */
  int32_t n_instr;       /* PROGRAM: number of instructions, 1..FA_MASK_PROGRAM_MAX         */
  int32_t reserved;      /* must be 0                                                       */
  fa_mask_instr program[FA_MASK_PROGRAM_MAX];  /* PROGRAM: postfix instructions (host memory,
                            read during the call)                                          */
} fa_mask_mod;

/* ----------------------------------------------------------------------- */
/* score_mod menu: g(s, b, h, q, kv), applied to the scaled score s BEFORE  */
/* the mask on every visited tile ([charlestar] "score_mod changes the      */
/* score, and the order changes the result"; [guide] 1.2).  h is the QUERY  */
/* head.  slope_h = 2^(-8 (h + 1) / H) with H = slope_heads (0 means Hq).   */
/* ----------------------------------------------------------------------- */
enum {
  FA_SCORE_NONE = 0,          /* g = s                                                       */
  FA_SCORE_SOFTCAP = 1,       /* g = cap * tanh(s / cap)          ([expressions] Gemma 2 cap) */
  FA_SCORE_ALIBI = 2,         /* g = s - slope_h * (q - kv)       ([expressions] ALiBi)       */
  FA_SCORE_CAP_THEN_BIAS = 3  /* g = cap * tanh(s / cap) + slope_h * (p[kv] - p[q]): the cap first,
                                 then the distance bias ([charlestar] "score_mod changes the
                                 score").  p = pos[b][.] when pos != NULL (positions outside
                                 [0, S) read the nearest end), else the position itself.       */
};

typedef struct fa_score_mod {
  int32_t kind;          /* FA_SCORE_*                                                     */
  float cap;             /* SOFTCAP, CAP_THEN_BIAS: c > 0                                   */
  int32_t slope_heads;   /* ALIBI, CAP_THEN_BIAS: H in slope_h (0 = Hq)                     */
  int32_t pos_batch;     /* CAP_THEN_BIAS with pos: rows of pos, 1 or B                      */
  const int32_t* pos;    /* CAP_THEN_BIAS: optional device int32 [pos_batch, S] positions    */
} fa_score_mod;

/* ----------------------------------------------------------------------- */
/* BlockMask ([guide] 3.1, 3.2, 4.1; [charlestar] "mask_mod defines legal   */
/* connections, BlockMask defines block work").  Tile (m, n) covers query   */
/* rows [m*BM, (m+1)*BM) and keys [n*BN, (n+1)*BN), clipped to L and S.     */
/* A tile is EMPTY when none of its in-range cells is visible (skipped),    */
/* FULL when all are (computed without the element mask; the score rule     */
/* still runs) and PARTIAL otherwise (score rule, then the element mask).   */
/* For every (b, h, m) the partial tile indices n are listed ascending in   */
/* kv_indices and counted in kv_num_blocks; full tiles likewise in          */
/* full_kv_indices / full_kv_num_blocks.  Unused slots hold 0.              */
/* All four arrays are caller-allocated device int32, row-major.            */
/* ----------------------------------------------------------------------- */
typedef struct fa_block_mask {
  int32_t B;                    /* 1 (broadcast over the batch) or the batch size          */
  int32_t H;                    /* 1 (broadcast over heads) or Hq; the fixed rules do not
                                   depend on the head, so their head rows are identical; a
                                   program with FA_PROG_HEAD_BELOW needs H == Hq           */
  int32_t L, S;                 /* query and key lengths the mask describes                */
  int32_t BM, BN;               /* query and key tile sizes, 1..128                        */
  int32_t Mb, Nb;               /* ceil(L / BM), ceil(S / BN)                              */
  int32_t* kv_num_blocks;       /* [B, H, Mb]                                              */
  int32_t* kv_indices;          /* [B, H, Mb, Nb]                                          */
  int32_t* full_kv_num_blocks;  /* [B, H, Mb]                                              */
  int32_t* full_kv_indices;     /* [B, H, Mb, Nb]                                          */
} fa_block_mask;

/* ----------------------------------------------------------------------- */
/* Dense 4-D tensor view (B, H, N, D) with element strides.                 */
/* ----------------------------------------------------------------------- */
typedef struct fa_tensor {
  void* data;          /* device pointer to element (0, 0, 0, 0)                            */
  int32_t dtype;       /* FA_DTYPE_*                                                         */
  int32_t reserved;    /* must be 0                                                          */
  int64_t size[4];     /* (B, H, N, D)                                                       */
  int64_t stride[4];   /* in elements; stride[3] must be 1                                   */
} fa_tensor;

/* ----------------------------------------------------------------------- */
/* Per-call options of flexattn_forward (pass NULL for the defaults).       */
/* ----------------------------------------------------------------------- */
enum {
  /* The caller promises that every query row has at least one visible key
   * whose transformed score is finite ("PyTorch Flex Attention complete
   * guide" section 5, ROWS_GUARANTEED_SAFE, default off; "flexattention-
   * score-mod-block-mask", "Correctness checks come before performance": a
   * property the caller has proven, not a speed switch).  The kernels then
   * drop their guard for rows without a visible key (the -inf tests of the
   * running maximum and the zero / -inf substitution at the end); a row that
   * breaks the promise gets unspecified out, lse and max_scores values,
   * possibly NaN. */
  FA_FLAG_ROWS_GUARANTEED_SAFE = 1
};

typedef struct fa_forward_options {
  float* max_scores;    /* optional device fp32 [B, Hq, L], contiguous (NULL: not written):
                           per row, the largest transformed score g_ij among the visible
                           keys, in the units of lse (natural log scale); -inf for a row
                           without a visible key ("PyTorch Flex Attention complete guide"
                           section 2, AuxRequest / AuxOutput max_scores)                   */
  int64_t wait_cycles;  /* budget of each device-side wait on the main path, in GPU clock
                           cycles; 0 = the default (about 2 s).  A small budget makes the
                           first wait that is not already satisfied give up, so that the
                           timeout path (FA_ERR_TIMEOUT in the device status word, outputs
                           unspecified) can be exercised; the waits that drain a CTA's own
                           copies and MMAs before it exits keep the default budget       */
  int32_t flags;        /* FA_FLAG_*                                                        */
  int32_t reserved;     /* must be 0                                                        */
  /* Paged KV cache ([charlestar] "At decode, q_idx = 0 is not position 0": a
   * paged or circular layout maps storage positions back to logical ones).
   * When page_table != NULL, k and v are page pools of shape
   * (num_pages, Hkv, page_size, E / Ev) -- any strides, so a pool stored as
   * (num_pages, page_size, Hkv, E) is passed with its strides -- and logical
   * key j of sequence b is slot j % page_size of page
   * page_table[b * pages_per_seq + j / page_size].  The logical length
   * S = pages_per_seq * page_size is what the block mask, kv_len and every
   * rule see.  A circular cache is a page table whose entries wrap around a
   * ring of pages; the caller's mask must hide the stale logical pages.
   * A page id outside [0, num_pages) is clamped into the pool (nothing
   * outside it is read), FA_ERR_PARAM is recorded in the device status word
   * and the outputs are unspecified.                                       */
  const int32_t* page_table;  /* device int32 [B, pages_per_seq], row-major, or NULL        */
  int32_t page_size;    /* keys per page: a multiple of 64 on the bf16 tensor-core and split-KV
                           kernels, any size >= 1 on the general kernel                   */
  int32_t pages_per_seq;/* columns of page_table                                            */
} fa_forward_options;

/* ----------------------------------------------------------------------- */
/* Entry points                                                             */
/* ----------------------------------------------------------------------- */

/* Library version (major * 10000 + minor * 100 + patch). */
int flexattn_version(void);

/* Message describing the last failing call on this thread ("" if none). */
const char* flexattn_last_error(void);

/* Tile-grid extents of a BlockMask: *Mb = ceil(L / BM), *Nb = ceil(S / BN).
 * Errors: FA_ERR_NULL, FA_ERR_SHAPE (L, S < 1 or BM, BN outside 1..128). */
int flexattn_block_mask_dims(int32_t L, int32_t S, int32_t BM, int32_t BN, int32_t* Mb, int32_t* Nb);

/* Classify every (b, m, n) tile of `mask_mod` and write the four arrays of
 * `block_mask` (dims B, H, L, S, BM, BN, Mb, Nb set by the caller, arrays
 * caller-allocated).  Definition: [guide] 4.1 (dense mask, per-block
 * reduction, full blocks kept apart) and 3.1 (a block is sparse only when
 * all its elements are masked); evaluated here tile by tile on the GPU
 * without a dense temporary.  Tiles are classified over in-range cells.
 * `mask_mod->kv_len`, when given, must hold block_mask->B entries.
 * Errors: FA_ERR_NULL, FA_ERR_SHAPE, FA_ERR_MASK_SHAPE (Mb/Nb inconsistent),
 * FA_ERR_PARAM, FA_ERR_CUDA. */
int flexattn_build_block_mask(const fa_mask_mod* mask_mod, const fa_block_mask* block_mask, void* stream);

/* Bytes of device workspace flexattn_forward needs for these arguments
 * (0 when the chosen kernel needs none).  Same argument checks as
 * flexattn_forward; options (NULL or those of the forward call) matter for a
 * paged cache. */
int flexattn_forward_workspace_size(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v,
                                    const fa_block_mask* block_mask, int32_t split_kv,
                                    const fa_forward_options* options, size_t* bytes);

/* Forward pass ([charlestar] "What one connection goes through"):
 *   s_ij  = scale * q_i . k_j                        (scale <= 0 or NaN: 1/sqrt(E), [guide] 6.2)
 *   g_ij  = score_mod(s_ij, b, h, q_pos(i), j)       on every cell of a visited tile
 *   s~_ij = g_ij if mask_mod(b, h, q_pos(i), j) else -inf   (element mask on partial tiles
 *                                                      and on ragged edges; none on full tiles)
 *   out_i = sum_j softmax_j(s~_ij) v_j ;  lse_i = ln sum_j exp(s~_ij)
 * Only tiles listed in block_mask are visited; EMPTY tiles contribute nothing.
 * A row without any visible key (or whose visible scores are all -inf) gets
 * out_i = 0 and lse_i = -inf, never NaN.
 *
 *   q   (B, Hq, L, E), k (B, Hkv, S, E), v (B, Hkv, S, Ev); out (B, Hq, L, Ev)
 *       with out->dtype == q->dtype or FA_DTYPE_F32 (fp32 output from bf16
 *       inputs: the fp32 result is stored without rounding to bf16); k, v,
 *       q share one dtype.
 *   lse optional device fp32 [B, Hq, L], contiguous (NULL: not written).
 *   enable_gqa: query head h reads KV head h / (Hq / Hkv) ([guide] 6.1).
 *   block_mask: built for (L, S) with B in {1, B}, H in {1, Hq}; its BM, BN
 *       are the kernel's tiles.  The bf16 tensor-core kernel needs
 *       BM == BN == 128 and E == Ev in {64, 128}; other shapes run on the
 *       general kernel.
 *   mask_mod: the same parameters the block mask was built from ([charlestar]
 *       "Construction cache and compile cache": rebuild the block mask when
 *       the visibility structure changes; the library keeps no cache).
 *   split_kv: 0 = automatic (short queries, L <= 16, use split-KV decode),
 *       1 = never split, n > 1 = split each row of tiles into n parts.
 *   options: NULL, or max_scores, the rows-guaranteed-safe flag and the wait
 *       budget (fa_forward_options above).
 *   workspace: device scratch of at least flexattn_forward_workspace_size()
 *       bytes (may be NULL when that size is 0); it must not be used by any
 *       other work in flight on the GPU during the call.
 * Errors: FA_ERR_NULL, FA_ERR_SHAPE, FA_ERR_HEADS, FA_ERR_BATCH,
 * FA_ERR_MASK_SHAPE, FA_ERR_DTYPE, FA_ERR_HEADDIM, FA_ERR_ALIGN, FA_ERR_PARAM,
 * FA_ERR_WORKSPACE, FA_ERR_UNSUPPORTED, FA_ERR_CUDA. */
int flexattn_forward(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* out,
                     float* lse, float scale, int32_t enable_gqa, const fa_score_mod* score_mod,
                     const fa_mask_mod* mask_mod, const fa_block_mask* block_mask, int32_t split_kv,
                     const fa_forward_options* options, void* workspace, size_t workspace_bytes,
                     void* stream);

/* The split-KV decode of flexattn_forward, for callers that must not allocate
 * device memory.  The pages have no counterpart of this entry point: it exists
 * for code that runs where cudaMalloc is off limits -- inside a serving loop
 * whose memory is fixed at start-up, between the steps of a captured CUDA
 * graph, or in a host runtime with no allocator of its own -- and so cannot
 * provide the workspace flexattn_forward asks for.
 *
 * Arguments and results are those of flexattn_forward, without the workspace:
 * the partial results of the KV splits go to a scratch array inside the
 * library, 16 MiB, which every GPU that loads the library holds until the
 * process exits.  This call allocates nothing and calls no allocating
 * routine.  The first call on a device looks up that array's device address
 * (with that device current) and caches it; make that first call before any
 * stream capture.
 *
 * All calls share the one array and it keeps whatever the last call wrote;
 * nothing in it has to start at zero, because every split writes its slot
 * before the combine step reads it.  Calls whose kernels overlap on the GPU
 * (other streams, other threads) race on the array: serialise them.
 *
 * Only the decode path runs here (bf16, E == Ev in {64, 128}, L <= 16, one
 * query tile, BN in {64, 128}, split_kv != 1); anything else returns
 * FA_ERR_UNSUPPORTED.  With split_kv == 0 the split count is the one
 * flexattn_forward would choose, lowered to what the scratch holds, and one
 * split (which needs no scratch) when not even two fit.  A call needing
 * more than 16 MiB of scratch (B * Hq * L * splits * (Ev + 2) * 4 bytes for
 * splits > 1) returns FA_ERR_WORKSPACE.
 * Other errors: those of flexattn_forward. */
int flexattn_forward_decode_noalloc(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* out,
                                    float* lse, float scale, int32_t enable_gqa, const fa_score_mod* score_mod,
                                    const fa_mask_mod* mask_mod, const fa_block_mask* block_mask, int32_t split_kv,
                                    void* stream);

/* ----------------------------------------------------------------------- */
/* Backward pass                                                            */
/* ----------------------------------------------------------------------- */

/* Query-side lists of a BlockMask ([guide] 3.3: from_kv_blocks derives them
 * for the backward pass): for key tile n of row (b, h), the query tiles m
 * whose row lists n as partial (q_indices, counted in q_num_blocks) or as
 * full (full_q_indices, full_q_num_blocks), ascending, unused slots 0.
 * B, H, Mb, Nb are those of the BlockMask it is built from; all four arrays
 * are caller-allocated device int32, row-major. */
typedef struct fa_block_mask_q {
  int32_t B, H, Mb, Nb;
  int32_t* q_num_blocks;        /* [B, H, Nb]     */
  int32_t* q_indices;           /* [B, H, Nb, Mb] */
  int32_t* full_q_num_blocks;   /* [B, H, Nb]     */
  int32_t* full_q_indices;      /* [B, H, Nb, Mb] */
} fa_block_mask_q;

/* Fill the query-side lists of `block_mask` on the GPU.
 * Errors: FA_ERR_NULL, FA_ERR_SHAPE, FA_ERR_MASK_SHAPE (dims disagree), FA_ERR_CUDA. */
int flexattn_transpose_block_mask(const fa_block_mask* block_mask, const fa_block_mask_q* q_side, void* stream);

/* Bytes of device workspace flexattn_backward needs (fp32 D = rowsum(dout * out),
 * [B, Hq, L]). */
int flexattn_backward_workspace_size(const fa_tensor* q, size_t* bytes);

/* Backward pass: the gradients of sum(out * dout) with respect to q, k and v
 * for the forward pass of flexattn_forward with the same arguments
 * ([charlestar] calls backward on the loss through flex_attention).  With P
 * the softmax weights recomputed from lse (0 on hidden keys),
 *   dv = P^T dout,  dP = dout v^T,  D = rowsum(dout * out),
 *   dS = P (dP - D) dg/ds  (dg/ds = 1 - tanh(s / cap)^2 under a soft-cap, else 1),
 *   dq = scale dS k,  dk = scale dS^T q;
 * dk and dv sum over the query heads that share a KV head (GQA).  The dk / dv
 * kernel walks each key tile's query-side list and the dq kernel each query
 * tile's key-side list, so every gradient is written once, in a fixed order
 * (deterministic; [guide] 5, WRITE_DQ).
 *   q, k, v, out (forward output), dout (B, Hq, L, Ev): bf16, E == Ev in
 *       {64, 128}; lse: the forward's fp32 [B, Hq, L].
 *   dq (B, Hq, L, E), dk (B, Hkv, S, E), dv (B, Hkv, S, Ev): bf16 or fp32,
 *       written in full.
 *   block_mask / block_mask_q: 128 x 128 tiles, with the query-side lists
 *       from flexattn_transpose_block_mask.
 *   workspace: flexattn_backward_workspace_size() bytes.
 * Every tensor's base and strides are 16-byte aligned (else FA_ERR_ALIGN).
 * No paged cache.  Errors: those of flexattn_forward, and FA_ERR_UNSUPPORTED
 * for other dtypes, head dims or tile sizes. */
int flexattn_backward(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* out,
                      const fa_tensor* dout, const float* lse, const fa_tensor* dq, const fa_tensor* dk,
                      const fa_tensor* dv, float scale, int32_t enable_gqa, const fa_score_mod* score_mod,
                      const fa_mask_mod* mask_mod, const fa_block_mask* block_mask,
                      const fa_block_mask_q* block_mask_q, void* workspace, size_t workspace_bytes, void* stream);

/* Wait for `stream`, then read and clear the device status word that the
 * kernels set when a bounded wait runs out (FA_ERR_TIMEOUT) or an index check
 * fails.  *status receives FA_OK or the first error recorded since the last
 * poll.  Returns FA_OK, or FA_ERR_CUDA if synchronising failed. */
int flexattn_poll_device_status(void* stream, int32_t* status);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* FLEXATTN_H_ */
