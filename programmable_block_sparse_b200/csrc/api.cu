// C ABI layer: argument checks, TMA descriptor encoding and kernel choice.
// Declarations and the contract of every entry point are in include/flexattn.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "launch.h"

namespace fa {

// First error a kernel recorded since the last flexattn_poll_device_status.
__device__ int g_device_status = 0;

namespace {

// Device address of g_device_status for the current device (looked up once
// per device; the CUDA runtime loads this module's globals per context).
int* status_word(int* err) {
  static int* cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  *err = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *err = 1;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
      *err = 1;
      return nullptr;
    }
    cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

// Scratch of flexattn_forward_decode_noalloc: a fixed device array that the
// library owns, so that entry point never allocates.  It occupies this many
// bytes on every GPU that loads the library, until the process exits.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.  Host code may
// not use the array's name as a device pointer (it is a host-side stand-in),
// so the address is asked of the runtime once per device, with that device
// current, and cached.
void* noalloc_scratch(int* err) {
  static void* cache[64] = {};
  static std::mutex mu;
  int dev = 0;
  *err = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *err = 1;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      *err = 1;
      return nullptr;
    }
    cache[dev] = p;
  }
  return cache[dev];
}

thread_local std::string t_last_error;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ----------------------------------------------------------------------------
// Composed rules: a postfix program of predicates and AND / OR / NOT,
// rewritten as an AND of clauses, each an OR of (possibly negated)
// predicates, which the kernels evaluate with fixed, unrolled loops.
// ----------------------------------------------------------------------------
struct ProgNode {
  int op, arg, a, b;  // a, b: operand nodes (-1 when absent)
};
struct ProgLit {
  int op, arg;
  bool neg;
  bool operator==(const ProgLit& o) const { return op == o.op && arg == o.arg && neg == o.neg; }
};
using ProgClause = std::vector<ProgLit>;
using ProgCnf = std::vector<ProgClause>;
constexpr size_t kCnfWork = 256;  // bound on intermediate clause counts

bool prog_is_pred(int op) { return op >= FA_PROG_TRUE && op <= FA_PROG_HEAD_BELOW; }

// Postfix -> tree; false when the stack discipline is broken.
bool prog_tree(const fa_mask_mod* m, std::vector<ProgNode>* t, int* root) {
  std::vector<int> st;
  for (int i = 0; i < m->n_instr; ++i) {
    const fa_mask_instr& in = m->program[i];
    if (prog_is_pred(in.op)) {
      t->push_back({in.op, in.arg, -1, -1});
    } else if (in.op == FA_PROG_NOT) {
      if (st.empty()) return false;
      t->push_back({in.op, 0, st.back(), -1});
      st.pop_back();
    } else {  // AND / OR (checked by the caller)
      if (st.size() < 2) return false;
      const int b = st.back();
      st.pop_back();
      const int a = st.back();
      st.pop_back();
      t->push_back({in.op, 0, a, b});
    }
    st.push_back(static_cast<int>(t->size()) - 1);
  }
  if (st.size() != 1) return false;
  *root = st[0];
  return true;
}

// Negations pushed to the predicates (De Morgan), then AND distributed over
// OR; false when the clause count would exceed kCnfWork.
bool prog_cnf(const std::vector<ProgNode>& t, int i, bool neg, ProgCnf* out) {
  const ProgNode& n = t[i];
  if (prog_is_pred(n.op)) {
    *out = ProgCnf{ProgClause{ProgLit{n.op, n.arg, neg}}};
    return true;
  }
  if (n.op == FA_PROG_NOT) return prog_cnf(t, n.a, !neg, out);
  ProgCnf x, y;
  if (!prog_cnf(t, n.a, neg, &x) || !prog_cnf(t, n.b, neg, &y)) return false;
  if ((n.op == FA_PROG_AND) != neg) {  // a conjunction
    x.insert(x.end(), y.begin(), y.end());
    *out = std::move(x);
  } else {  // a disjunction: every clause of x OR every clause of y
    ProgCnf r;
    for (const ProgClause& cx : x)
      for (const ProgClause& cy : y) {
        ProgClause c = cx;
        c.insert(c.end(), cy.begin(), cy.end());
        r.push_back(std::move(c));
        if (r.size() > kCnfWork) return false;
      }
    *out = std::move(r);
  }
  return out->size() <= kCnfWork;
}

// The composed rule of *m as device clauses; FA_ERR_UNSUPPORTED when it needs
// more than kMaxClauses clauses or kMaxLits predicates in a clause.
int prog_compile(const fa_mask_mod* m, MaskParams* p) {
  std::vector<ProgNode> tree;
  int root = -1;
  if (!prog_tree(m, &tree, &root)) return FA_ERR_PARAM;
  ProgCnf cnf;
  if (!prog_cnf(tree, root, false, &cnf))
    return fail(FA_ERR_UNSUPPORTED, "the composed mask rule expands to too many clauses");
  ProgCnf kept;
  bool never = false;
  for (const ProgClause& c : cnf) {
    ProgClause d;
    bool always = false;
    for (const ProgLit& l : c) {
      if (l.op == FA_PROG_TRUE) {
        if (!l.neg) always = true;  // the clause holds everywhere
        continue;                   // a false literal adds nothing to an OR
      }
      bool dup = false;
      for (const ProgLit& e : d) dup = dup || e == l;
      if (!dup) d.push_back(l);
    }
    if (always) continue;
    if (d.empty()) never = true;  // a clause that holds nowhere: the rule holds nowhere
    kept.push_back(d);
  }
  if (never) kept = ProgCnf{ProgClause{ProgLit{FA_PROG_TRUE, 0, true}}};
  if (kept.size() > static_cast<size_t>(kMaxClauses))
    return fail(FA_ERR_UNSUPPORTED, "the composed mask rule needs %zu clauses (at most %d)", kept.size(), kMaxClauses);
  p->n_clauses = static_cast<int>(kept.size());
  for (size_t c = 0; c < kept.size(); ++c) {
    if (kept[c].size() > static_cast<size_t>(kMaxLits))
      return fail(FA_ERR_UNSUPPORTED, "a clause of the composed mask rule has %zu predicates (at most %d)",
                  kept[c].size(), kMaxLits);
    p->clause_len[c] = static_cast<int>(kept[c].size());
    for (size_t l = 0; l < kept[c].size(); ++l) {
      const ProgLit& x = kept[c][l];
      MaskLit& lt = p->lit[c][l];
      lt.op = x.op | (x.neg ? kLitNeg : 0);
      lt.arg = x.arg;
      lt.pat = 0u;
      if (x.op == FA_PROG_STRIDE && x.arg < 32)
        for (int k = 0; k < 32; k += x.arg) lt.pat |= 1u << k;
      p->reads_head |= x.op == FA_PROG_HEAD_BELOW;
      p->reads_doc |= x.op == FA_PROG_SAME_DOCUMENT;
    }
  }
  return FA_OK;
}

// ----------------------------------------------------------------------------
// Parameter checks shared by the build and forward calls.
// ----------------------------------------------------------------------------
int check_program(const fa_mask_mod* m, int batch) {
  if (m->n_instr < 1 || m->n_instr > FA_MASK_PROGRAM_MAX)
    return fail(FA_ERR_PARAM, "a composed mask rule needs 1..%d instructions (got %d)", FA_MASK_PROGRAM_MAX,
                m->n_instr);
  if (m->reserved != 0) return fail(FA_ERR_PARAM, "mask_mod: reserved field must be 0");
  bool doc = false;
  for (int i = 0; i < m->n_instr; ++i) {
    const fa_mask_instr& in = m->program[i];
    const bool known = prog_is_pred(in.op) || in.op == FA_PROG_AND || in.op == FA_PROG_OR || in.op == FA_PROG_NOT;
    if (!known) return fail(FA_ERR_PARAM, "composed mask rule: unknown instruction %d at %d", in.op, i);
    if (in.arg < -(1 << 30) || in.arg > (1 << 30))
      return fail(FA_ERR_PARAM, "composed mask rule: argument %d at %d is outside [-2^30, 2^30]", in.arg, i);
    if ((in.op == FA_PROG_SAME_CHUNK || in.op == FA_PROG_STRIDE) && in.arg < 1)
      return fail(FA_ERR_PARAM, "composed mask rule: chunk and stride need an argument >= 1 (got %d at %d)", in.arg, i);
    doc = doc || in.op == FA_PROG_SAME_DOCUMENT;
  }
  std::vector<ProgNode> tree;
  int root = -1;
  if (!prog_tree(m, &tree, &root))
    return fail(FA_ERR_PARAM, "composed mask rule: the postfix program does not leave exactly one verdict");
  if (doc) {
    if (m->doc_id == nullptr) return fail(FA_ERR_PARAM, "a same-document predicate needs doc_id");
    if (m->doc_batch != 1 && m->doc_batch != batch)
      return fail(FA_ERR_BATCH, "doc_batch must be 1 or %d (got %d)", batch, m->doc_batch);
  }
  return FA_OK;
}

int check_mask_params(const fa_mask_mod* m, int batch) {
  switch (m->kind) {
    case FA_MASK_NONE:
    case FA_MASK_CAUSAL:
      break;
    case FA_MASK_SLIDING_WINDOW:
      if (m->window < 1) return fail(FA_ERR_PARAM, "sliding window needs window >= 1 (got %d)", m->window);
      if (m->n_sink < 0) return fail(FA_ERR_PARAM, "sliding window needs n_sink >= 0 (got %d)", m->n_sink);
      break;
    case FA_MASK_DOCUMENT:
      if (m->doc_id == nullptr) return fail(FA_ERR_PARAM, "document mask needs doc_id");
      if (m->doc_batch != 1 && m->doc_batch != batch)
        return fail(FA_ERR_BATCH, "doc_batch must be 1 or %d (got %d)", batch, m->doc_batch);
      break;
    case FA_MASK_PREFIX_LM:
      if (m->prefix < 0) return fail(FA_ERR_PARAM, "prefix-LM needs prefix >= 0 (got %d)", m->prefix);
      break;
    case FA_MASK_CHUNKED:
      if (m->chunk < 1) return fail(FA_ERR_PARAM, "chunked mask needs chunk >= 1 (got %d)", m->chunk);
      break;
    case FA_MASK_PROGRAM:
      return check_program(m, batch);
    default:
      return fail(FA_ERR_PARAM, "unknown mask kind %d", m->kind);
  }
  return FA_OK;
}

int check_score_params(const fa_score_mod* s, int batch) {
  switch (s->kind) {
    case FA_SCORE_NONE:
      break;
    case FA_SCORE_SOFTCAP:
    case FA_SCORE_CAP_THEN_BIAS:
      if (!(s->cap > 0.0f) || isinf(s->cap)) return fail(FA_ERR_PARAM, "cap must be finite and > 0 (got %g)", s->cap);
      // fallthrough
    case FA_SCORE_ALIBI:
      if (s->slope_heads < 0) return fail(FA_ERR_PARAM, "slope_heads must be >= 0 (got %d)", s->slope_heads);
      if (s->kind == FA_SCORE_CAP_THEN_BIAS && s->pos != nullptr && s->pos_batch != 1 && s->pos_batch != batch)
        return fail(FA_ERR_BATCH, "pos_batch must be 1 or %d (got %d)", batch, s->pos_batch);
      break;
    default:
      return fail(FA_ERR_PARAM, "unknown score kind %d", s->kind);
  }
  return FA_OK;
}

int check_block_mask_dims(const fa_block_mask* bm) {
  if (bm->L < 1 || bm->S < 1) return fail(FA_ERR_SHAPE, "block mask lengths must be >= 1 (L=%d, S=%d)", bm->L, bm->S);
  if (bm->BM < 1 || bm->BM > 128 || bm->BN < 1 || bm->BN > 128)
    return fail(FA_ERR_SHAPE, "block sizes must be in 1..128 (BM=%d, BN=%d)", bm->BM, bm->BN);
  if (bm->B < 1 || bm->H < 1) return fail(FA_ERR_SHAPE, "block mask B and H must be >= 1");
  if (bm->Mb != ceil_div(bm->L, bm->BM) || bm->Nb != ceil_div(bm->S, bm->BN))
    return fail(FA_ERR_MASK_SHAPE, "block mask grid %dx%d does not match ceil(L/BM) x ceil(S/BN) = %dx%d", bm->Mb,
                bm->Nb, ceil_div(bm->L, bm->BM), ceil_div(bm->S, bm->BN));
  if (!bm->kv_num_blocks || !bm->kv_indices || !bm->full_kv_num_blocks || !bm->full_kv_indices)
    return fail(FA_ERR_NULL, "block mask arrays must not be NULL");
  return FA_OK;
}

// The mask parameters as the kernels read them (after check_mask_params).
int mask_to_device(const fa_mask_mod* m, MaskParams* out) {
  MaskParams p{};
  p.kind = m->kind;
  p.window = m->window;
  p.n_sink = m->n_sink;
  p.prefix = m->prefix;
  p.chunk = m->chunk;
  p.doc_batch = m->doc_batch;
  p.doc_id = m->doc_id;
  p.kv_len = m->kv_len;
  if (m->kind == FA_MASK_PROGRAM) {
    const int rc = prog_compile(m, &p);
    if (rc) return rc;
  }
  *out = p;
  return FA_OK;
}

ScoreParams to_device(const fa_score_mod* s) {
  ScoreParams p;
  p.kind = s->kind;
  p.cap = s->cap;
  p.slope_heads = s->slope_heads;
  p.pos_batch = s->pos_batch;
  p.pos = s->kind == FA_SCORE_CAP_THEN_BIAS ? s->pos : nullptr;
  return p;
}

// ----------------------------------------------------------------------------
// TMA descriptors
// ----------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// (B, H, N, D) bf16 tensor -> 4-D map with a 64 x box_rows box, 128 B swizzle.
int encode_bf16_map(CUtensorMap* map, const fa_tensor* t, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(t->size[3]), static_cast<cuuint64_t>(t->size[2]),
                        static_cast<cuuint64_t>(t->size[1]), static_cast<cuuint64_t>(t->size[0])};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(t->stride[2]) * 2, static_cast<cuuint64_t>(t->stride[1]) * 2,
                           static_cast<cuuint64_t>(t->stride[0]) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, t->data, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_ALIGN, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FA_OK;
}

// ----------------------------------------------------------------------------
// Forward argument checks -> FwdArgs
// ----------------------------------------------------------------------------
enum class Path { kSimt, kSm100, kDecode };

int sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

int check_tensor(const fa_tensor* t, const char* name) {
  if (t == nullptr || t->data == nullptr) return fail(FA_ERR_NULL, "%s is NULL", name);
  if (t->dtype != FA_DTYPE_BF16 && t->dtype != FA_DTYPE_F32) return fail(FA_ERR_DTYPE, "%s: unknown dtype %d", name, t->dtype);
  if (t->reserved != 0) return fail(FA_ERR_PARAM, "%s: reserved field must be 0", name);
  for (int i = 0; i < 4; ++i)
    if (t->size[i] < 1 || t->size[i] > INT32_MAX) return fail(FA_ERR_SHAPE, "%s: size[%d] = %lld out of range", name, i, (long long)t->size[i]);
  if (t->stride[3] != 1) return fail(FA_ERR_ALIGN, "%s: the last dimension must be contiguous (stride %lld)", name, (long long)t->stride[3]);
  for (int i = 0; i < 3; ++i)
    if (t->stride[i] < 0) return fail(FA_ERR_ALIGN, "%s: negative stride", name);
  return FA_OK;
}

bool aligned16(const fa_tensor* t) {
  const int es = t->dtype == FA_DTYPE_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(t->data) % 16) return false;
  for (int i = 0; i < 3; ++i)
    if ((t->stride[i] * es) % 16) return false;
  return true;
}

int apply_options(const fa_forward_options* o, FwdArgs* a) {
  a->max_scores = nullptr;
  a->rows_safe = 0;
  a->wait_cycles = kWaitCycles;
  if (o == nullptr) return FA_OK;
  if (o->reserved != 0) return fail(FA_ERR_PARAM, "options: reserved field must be 0");
  if (o->flags & ~FA_FLAG_ROWS_GUARANTEED_SAFE) return fail(FA_ERR_PARAM, "options: unknown flags 0x%x", o->flags);
  if (o->wait_cycles < 0) return fail(FA_ERR_PARAM, "options: wait_cycles must be >= 0");
  a->max_scores = o->max_scores;
  a->rows_safe = (o->flags & FA_FLAG_ROWS_GUARANTEED_SAFE) ? 1 : 0;
  if (o->wait_cycles > 0) a->wait_cycles = o->wait_cycles;
  return FA_OK;
}

int prepare(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* out, float scale,
            int32_t enable_gqa, const fa_score_mod* score, const fa_mask_mod* mask, const fa_block_mask* bm,
            int32_t split_kv, const fa_forward_options* opt, FwdArgs* a, Path* path) {
  int rc;
  if ((rc = check_tensor(q, "q")) || (rc = check_tensor(k, "k")) || (rc = check_tensor(v, "v"))) return rc;
  if (out != nullptr && (rc = check_tensor(out, "out"))) return rc;
  if (!score || !mask || !bm) return fail(FA_ERR_NULL, "score_mod, mask_mod and block_mask must not be NULL");
  if (k->dtype != q->dtype || v->dtype != q->dtype) return fail(FA_ERR_DTYPE, "q, k and v must share one dtype");
  if (out && out->dtype != q->dtype && out->dtype != FA_DTYPE_F32)
    return fail(FA_ERR_DTYPE, "out must have the dtype of q, or be fp32");
  const int B = (int)q->size[0], Hq = (int)q->size[1], L = (int)q->size[2], E = (int)q->size[3];
  const int Hkv = (int)k->size[1], Ev = (int)v->size[3];
  const bool paged = opt != nullptr && opt->page_table != nullptr;
  int S = (int)k->size[2];
  if (paged) {
    // k and v are page pools (num_pages, Hkv, page_size, E); S is the logical length
    if (opt->page_size < 1 || opt->pages_per_seq < 1)
      return fail(FA_ERR_PARAM, "paged cache: page_size and pages_per_seq must be >= 1 (got %d, %d)", opt->page_size,
                  opt->pages_per_seq);
    if (static_cast<int64_t>(opt->page_size) * opt->pages_per_seq > INT32_MAX / 2)
      return fail(FA_ERR_SHAPE, "paged cache: logical length page_size * pages_per_seq is too large");
    if (k->size[2] != opt->page_size || v->size[2] != opt->page_size || v->size[0] != k->size[0])
      return fail(FA_ERR_SHAPE, "paged cache: k and v must be pools of (num_pages, Hkv, page_size, dim)");
    S = opt->page_size * opt->pages_per_seq;
  } else if (k->size[0] != B || v->size[0] != B) {
    return fail(FA_ERR_BATCH, "q, k and v must have the same batch size");
  }
  // launch grids carry the batch and the head count in their y / z extents
  if (B > 65535 || Hq > 65535) return fail(FA_ERR_SHAPE, "batch and head counts above 65535 are not supported");
  if (k->size[3] != E) return fail(FA_ERR_SHAPE, "k head dim %lld != q head dim %d", (long long)k->size[3], E);
  if (v->size[1] != Hkv || v->size[2] != k->size[2]) return fail(FA_ERR_SHAPE, "v must be (B, Hkv, S, Ev) like k");
  if (out && (out->size[0] != B || out->size[1] != Hq || out->size[2] != L || out->size[3] != Ev))
    return fail(FA_ERR_SHAPE, "out must be (B, Hq, L, Ev)");
  if (Hq != Hkv) {
    if (!enable_gqa) return fail(FA_ERR_HEADS, "Hq (%d) != Hkv (%d): set enable_gqa", Hq, Hkv);
    if (Hq % Hkv) return fail(FA_ERR_HEADS, "GQA needs Hq %% Hkv == 0 (Hq=%d, Hkv=%d)", Hq, Hkv);
  }
  if (E > 128 || Ev > 128) return fail(FA_ERR_HEADDIM, "head dims above 128 are not supported (E=%d, Ev=%d)", E, Ev);
  if ((rc = check_block_mask_dims(bm))) return rc;
  if (bm->L != L || bm->S != S)
    return fail(FA_ERR_MASK_SHAPE, "block mask is for L=%d, S=%d but the call has L=%d, S=%d (%s)", bm->L, bm->S, L, S,
                (bm->L < L || bm->S < S) ? "too small" : "too large");
  if (bm->B != 1 && bm->B != B) return fail(FA_ERR_BATCH, "block mask batch %d is neither 1 nor %d", bm->B, B);
  if (bm->H != 1 && bm->H != Hq) return fail(FA_ERR_MASK_SHAPE, "block mask heads %d is neither 1 nor %d", bm->H, Hq);
  if (mask->kv_len && bm->B != B)
    return fail(FA_ERR_BATCH, "with per-sequence kv_len the block mask needs batch %d (has %d)", B, bm->B);
  if ((rc = check_mask_params(mask, B)) || (rc = check_score_params(score, B))) return rc;

  *a = FwdArgs{};
  a->q = q->data;
  a->k = k->data;
  a->v = v->data;
  a->out = out ? out->data : nullptr;
  for (int i = 0; i < 4; ++i) {
    a->q_stride[i] = q->stride[i];
    a->k_stride[i] = k->stride[i];
    a->v_stride[i] = v->stride[i];
    a->o_stride[i] = out ? out->stride[i] : 0;
  }
  a->B = B;
  a->Hq = Hq;
  a->Hkv = Hkv;
  a->L = L;
  a->S = S;
  a->E = E;
  a->Ev = Ev;
  a->G = Hq / Hkv;
  a->dtype = q->dtype;
  a->out_f32 = out != nullptr && out->dtype == FA_DTYPE_F32;
  a->wait_cycles = kWaitCycles;
  a->scale = (scale > 0.0f && !isinf(scale)) ? scale : 1.0f / sqrtf(static_cast<float>(E));
  if (paged) {
    a->page_table = opt->page_table;
    a->page_size = opt->page_size;
    a->pages_per_seq = opt->pages_per_seq;
    a->num_pages = static_cast<int>(k->size[0]);
  }
  if ((rc = mask_to_device(mask, &a->mask))) return rc;
  if (a->mask.reads_head && bm->H != Hq && Hq > 1)
    return fail(FA_ERR_MASK_SHAPE, "a rule that reads the query head needs a per-head block mask (H = %d, got %d)", Hq,
                bm->H);
  a->score = to_device(score);
  a->bm = BlockMaskView{bm->B, bm->H, bm->Mb, bm->Nb, bm->BM, bm->BN, bm->kv_num_blocks, bm->kv_indices,
                        bm->full_kv_num_blocks, bm->full_kv_indices};

  // the tensor-core kernels read a paged pool in 64-key boxes
  const bool tc_shape = q->dtype == FA_DTYPE_BF16 && E == Ev && (E == 64 || E == 128) &&
                        (!paged || opt->page_size % 64 == 0);
  const bool tma_ok = aligned16(q) && aligned16(k) && aligned16(v);
  if (split_kv < 0) return fail(FA_ERR_PARAM, "split_kv must be >= 0");
  if (split_kv > 1 && !(tc_shape && L <= kDecodeMaxRows && bm->Mb == 1 && bm->BN % 64 == 0))
    return fail(FA_ERR_UNSUPPORTED,
                "split_kv > 1 needs bf16, E == Ev in {64,128}, L <= 16, one query tile, BN in {64, 128} and, for "
                "a paged cache, pages of a multiple of 64 keys");
  if (split_kv > 1 && !tma_ok) return fail(FA_ERR_ALIGN, "split_kv > 1 needs 16-byte aligned q, k, v and strides");
  const bool out_ok = out == nullptr || aligned16(out);
  const bool decode_ok = tc_shape && tma_ok && L <= kDecodeMaxRows && bm->Mb == 1 && bm->BN % 64 == 0;
  if (split_kv != 1 && decode_ok) {
    *path = Path::kDecode;
  } else if (tc_shape && tma_ok && out_ok && bm->BM == 128 && bm->BN == 128 && (bm->Mb + 1) / 2 <= 65535) {
    *path = Path::kSm100;
  } else {
    *path = Path::kSimt;
  }
  return FA_OK;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

int flexattn_version(void) { return 100; }

const char* flexattn_last_error(void) { return t_last_error.c_str(); }

int flexattn_block_mask_dims(int32_t L, int32_t S, int32_t BM, int32_t BN, int32_t* Mb, int32_t* Nb) {
  if (!Mb || !Nb) return fail(FA_ERR_NULL, "Mb and Nb must not be NULL");
  if (L < 1 || S < 1) return fail(FA_ERR_SHAPE, "L and S must be >= 1");
  if (BM < 1 || BM > 128 || BN < 1 || BN > 128) return fail(FA_ERR_SHAPE, "BM and BN must be in 1..128");
  *Mb = ceil_div(L, BM);
  *Nb = ceil_div(S, BN);
  return FA_OK;
}

int flexattn_build_block_mask(const fa_mask_mod* mask_mod, const fa_block_mask* bm, void* stream) {
  if (!mask_mod || !bm) return fail(FA_ERR_NULL, "mask_mod and block_mask must not be NULL");
  int rc;
  if ((rc = check_block_mask_dims(bm))) return rc;
  if ((rc = check_mask_params(mask_mod, bm->B))) return rc;
  ClassifyArgs a;
  int serr = 0;
  a.status = status_word(&serr);
  if (serr) return fail(FA_ERR_CUDA, "cannot locate the device status word");
  if ((rc = mask_to_device(mask_mod, &a.mask))) return rc;
  a.B = bm->B;
  a.H = bm->H;
  a.L = bm->L;
  a.S = bm->S;
  a.BM = bm->BM;
  a.BN = bm->BN;
  a.Mb = bm->Mb;
  a.Nb = bm->Nb;
  a.kv_num_blocks = bm->kv_num_blocks;
  a.kv_indices = bm->kv_indices;
  a.full_kv_num_blocks = bm->full_kv_num_blocks;
  a.full_kv_indices = bm->full_kv_indices;
  cudaError_t e = launch_classify(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "block-mask classifier launch");
  return FA_OK;
}

int flexattn_forward_workspace_size(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v,
                                    const fa_block_mask* block_mask, int32_t split_kv,
                                    const fa_forward_options* options, size_t* bytes) {
  if (!bytes) return fail(FA_ERR_NULL, "bytes must not be NULL");
  fa_score_mod none_score{FA_SCORE_NONE, 0.0f, 0, 0, nullptr};
  fa_mask_mod none_mask{};
  none_mask.kind = FA_MASK_NONE;
  FwdArgs a;
  Path path;
  int rc = prepare(q, k, v, nullptr, 0.0f, 1, &none_score, &none_mask, block_mask, split_kv, options, &a, &path);
  if (rc) return rc;
  *bytes = 0;
  if (path == Path::kDecode) {
    DecodePlan plan;
    plan_decode(a, split_kv, sm_count(), &plan);
    *bytes = plan.workspace_bytes;
  }
  return FA_OK;
}

int flexattn_forward(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* out, float* lse,
                     float scale, int32_t enable_gqa, const fa_score_mod* score_mod, const fa_mask_mod* mask_mod,
                     const fa_block_mask* block_mask, int32_t split_kv, const fa_forward_options* options,
                     void* workspace, size_t workspace_bytes, void* stream) {
  if (!out) return fail(FA_ERR_NULL, "out is NULL");
  FwdArgs a;
  Path path;
  int rc = prepare(q, k, v, out, scale, enable_gqa, score_mod, mask_mod, block_mask, split_kv, options, &a, &path);
  if (rc) return rc;
  if ((rc = apply_options(options, &a))) return rc;
  int serr = 0;
  a.status = status_word(&serr);
  if (serr) return fail(FA_ERR_CUDA, "cannot locate the device status word");
  a.lse = lse;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (path == Path::kSm100) {
    Sm100Maps maps;
    const int kv_box = a.page_table ? 64 : 128;  // a paged pool is read in 64-key boxes
    if ((rc = encode_bf16_map(&maps.q, q, 128)) || (rc = encode_bf16_map(&maps.k, k, kv_box)) ||
        (rc = encode_bf16_map(&maps.v, v, kv_box)))
      return rc;
    e = launch_fwd_sm100(a, maps, st);
  } else if (path == Path::kDecode) {
    DecodePlan plan;
    plan_decode(a, split_kv, sm_count(), &plan);
    if (plan.workspace_bytes > 0 && (workspace == nullptr || workspace_bytes < plan.workspace_bytes))
      return fail(FA_ERR_WORKSPACE, "split-KV decode needs %zu bytes of workspace (got %zu)", plan.workspace_bytes,
                  workspace ? workspace_bytes : static_cast<size_t>(0));
    if (plan.workspace_bytes > 0 && reinterpret_cast<uintptr_t>(workspace) % 16)
      return fail(FA_ERR_ALIGN, "workspace must be 16-byte aligned");
    Sm100Maps maps;
    if ((rc = encode_bf16_map(&maps.k, k, 64)) || (rc = encode_bf16_map(&maps.v, v, 64))) return rc;
    e = launch_decode(a, plan, maps, workspace, st);
  } else {
    e = launch_fwd_simt(a, st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "forward launch");
  return FA_OK;
}

int flexattn_forward_decode_noalloc(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* out,
                                    float* lse, float scale, int32_t enable_gqa, const fa_score_mod* score_mod,
                                    const fa_mask_mod* mask_mod, const fa_block_mask* block_mask, int32_t split_kv,
                                    void* stream) {
  if (!out) return fail(FA_ERR_NULL, "out is NULL");
  FwdArgs a;
  Path path;
  int rc = prepare(q, k, v, out, scale, enable_gqa, score_mod, mask_mod, block_mask, split_kv, nullptr, &a, &path);
  if (rc) return rc;
  if ((rc = apply_options(nullptr, &a))) return rc;
  if (path != Path::kDecode)
    return fail(FA_ERR_UNSUPPORTED,
                "the no-allocation entry point runs only the split-KV decode path (bf16, E == Ev in {64, 128}, "
                "L <= 16, one query tile, BN in {64, 128}, split_kv != 1)");
  DecodePlan plan;
  plan_decode(a, split_kv, sm_count(), &plan);
  if (split_kv == 0 && plan.workspace_bytes > kNoAllocScratchBytes) {
    // automatic split count: the most splits the built-in scratch holds, or a
    // single split (results straight to out / lse, no scratch) when not even
    // two fit
    const size_t per_split = static_cast<size_t>(a.B) * a.Hq * a.L * (a.Ev + 2) * sizeof(float);
    const size_t fit = kNoAllocScratchBytes / per_split;
    if (fit >= 2) {
      plan_decode(a, static_cast<int32_t>(fit < 65536 ? fit : 65536), sm_count(), &plan);
    } else {
      plan.splits = 1;
      plan.tiles_per_split = a.bm.Nb;
      plan.workspace_bytes = 0;
    }
  }
  if (plan.workspace_bytes > kNoAllocScratchBytes)
    return fail(FA_ERR_WORKSPACE,
                "this call needs %zu bytes of scratch but the built-in scratch holds %zu: pass fewer splits, or "
                "use flexattn_forward with a caller-owned workspace",
                plan.workspace_bytes, kNoAllocScratchBytes);
  int err = 0;
  void* scratch = noalloc_scratch(&err);
  if (err) return fail(FA_ERR_CUDA, "cannot locate the built-in decode scratch on the current device");
  a.status = status_word(&err);
  if (err) return fail(FA_ERR_CUDA, "cannot locate the device status word");
  a.lse = lse;
  Sm100Maps maps;
  if ((rc = encode_bf16_map(&maps.k, k, 64)) || (rc = encode_bf16_map(&maps.v, v, 64))) return rc;
  cudaError_t e = launch_decode(a, plan, maps, scratch, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return FA_OK;
}

int flexattn_transpose_block_mask(const fa_block_mask* bm, const fa_block_mask_q* qs, void* stream) {
  if (!bm || !qs) return fail(FA_ERR_NULL, "block_mask and q_side must not be NULL");
  int rc;
  if ((rc = check_block_mask_dims(bm))) return rc;
  if (qs->B != bm->B || qs->H != bm->H || qs->Mb != bm->Mb || qs->Nb != bm->Nb)
    return fail(FA_ERR_MASK_SHAPE, "query-side lists must have the block mask's B, H, Mb, Nb");
  if (!qs->q_num_blocks || !qs->q_indices || !qs->full_q_num_blocks || !qs->full_q_indices)
    return fail(FA_ERR_NULL, "query-side arrays must not be NULL");
  TransposeArgs t{bm->B, bm->H, bm->Mb, bm->Nb, bm->kv_num_blocks, bm->kv_indices, bm->full_kv_num_blocks,
                  bm->full_kv_indices, qs->q_num_blocks, qs->q_indices, qs->full_q_num_blocks, qs->full_q_indices};
  cudaError_t e = launch_transpose(t, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "block-mask transpose launch");
  return FA_OK;
}

int flexattn_backward_workspace_size(const fa_tensor* q, size_t* bytes) {
  if (!bytes) return fail(FA_ERR_NULL, "bytes must not be NULL");
  int rc;
  if ((rc = check_tensor(q, "q"))) return rc;
  *bytes = static_cast<size_t>(q->size[0]) * q->size[1] * q->size[2] * sizeof(float);
  return FA_OK;
}

int flexattn_backward(const fa_tensor* q, const fa_tensor* k, const fa_tensor* v, const fa_tensor* out,
                      const fa_tensor* dout, const float* lse, const fa_tensor* dq, const fa_tensor* dk,
                      const fa_tensor* dv, float scale, int32_t enable_gqa, const fa_score_mod* score_mod,
                      const fa_mask_mod* mask_mod, const fa_block_mask* block_mask, const fa_block_mask_q* qs,
                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!out || !dout || !dq || !dk || !dv || !lse || !qs) return fail(FA_ERR_NULL, "backward arguments must not be NULL");
  FwdArgs f;
  Path path;
  int rc = prepare(q, k, v, out, scale, enable_gqa, score_mod, mask_mod, block_mask, 1, nullptr, &f, &path);
  if (rc) return rc;
  if ((rc = check_tensor(dout, "dout")) || (rc = check_tensor(dq, "dq")) || (rc = check_tensor(dk, "dk")) ||
      (rc = check_tensor(dv, "dv")))
    return rc;
  const int B = f.B, Hq = f.Hq, Hkv = f.Hkv, L = f.L, S = f.S, E = f.E;
  if (q->dtype != FA_DTYPE_BF16 || out->dtype != FA_DTYPE_BF16 || dout->dtype != FA_DTYPE_BF16)
    return fail(FA_ERR_UNSUPPORTED, "the backward pass takes bf16 q, k, v, out and dout");
  if (f.E != f.Ev || (E != 64 && E != 128))
    return fail(FA_ERR_UNSUPPORTED, "the backward pass needs E == Ev in {64, 128}");
  if (block_mask->BM != 128 || block_mask->BN != 128)
    return fail(FA_ERR_UNSUPPORTED, "the backward pass needs 128 x 128 tiles");
  for (int i = 0; i < 4; ++i)
    if (dout->size[i] != out->size[i]) return fail(FA_ERR_SHAPE, "dout must have the shape of out");
  const int64_t want_q[4] = {B, Hq, L, E}, want_k[4] = {B, Hkv, S, E};
  for (int i = 0; i < 4; ++i) {
    if (dq->size[i] != want_q[i]) return fail(FA_ERR_SHAPE, "dq must be (B, Hq, L, E)");
    if (dk->size[i] != want_k[i] || dv->size[i] != want_k[i]) return fail(FA_ERR_SHAPE, "dk and dv must be (B, Hkv, S, E)");
  }
  for (const fa_tensor* g : {dq, dk, dv})
    if (g->dtype != FA_DTYPE_BF16 && g->dtype != FA_DTYPE_F32) return fail(FA_ERR_DTYPE, "gradients are bf16 or fp32");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return fail(FA_ERR_ALIGN, "the backward pass needs 16-byte aligned tensors and strides");
  if (qs->B != block_mask->B || qs->H != block_mask->H || qs->Mb != block_mask->Mb || qs->Nb != block_mask->Nb)
    return fail(FA_ERR_MASK_SHAPE, "query-side lists must have the block mask's B, H, Mb, Nb");
  if (!qs->q_num_blocks || !qs->q_indices || !qs->full_q_num_blocks || !qs->full_q_indices)
    return fail(FA_ERR_NULL, "query-side arrays must not be NULL");
  const size_t need = static_cast<size_t>(B) * Hq * L * sizeof(float);
  if (workspace == nullptr || workspace_bytes < need)
    return fail(FA_ERR_WORKSPACE, "the backward pass needs %zu bytes of workspace (got %zu)", need,
                workspace ? workspace_bytes : static_cast<size_t>(0));
  if (reinterpret_cast<uintptr_t>(workspace) % 16) return fail(FA_ERR_ALIGN, "workspace must be 16-byte aligned");
  if (B > 65535 || Hq > 65535 || block_mask->Nb > 65535) return fail(FA_ERR_SHAPE, "grid extents above 65535");

  BwdArgs a{};
  int serr = 0;
  a.status = status_word(&serr);
  if (serr) return fail(FA_ERR_CUDA, "cannot locate the device status word");
  a.wait_cycles = kWaitCycles;
  a.q = q->data;
  a.k = k->data;
  a.v = v->data;
  a.out = out->data;
  a.dout = dout->data;
  a.lse = lse;
  a.dsum = static_cast<float*>(workspace);
  a.dq = dq->data;
  a.dk = dk->data;
  a.dv = dv->data;
  for (int i = 0; i < 4; ++i) {
    a.q_stride[i] = q->stride[i];
    a.k_stride[i] = k->stride[i];
    a.v_stride[i] = v->stride[i];
    a.o_stride[i] = out->stride[i];
    a.do_stride[i] = dout->stride[i];
    a.dq_stride[i] = dq->stride[i];
    a.dk_stride[i] = dk->stride[i];
    a.dv_stride[i] = dv->stride[i];
  }
  a.dq_f32 = dq->dtype == FA_DTYPE_F32;
  a.dk_f32 = dk->dtype == FA_DTYPE_F32;
  a.dv_f32 = dv->dtype == FA_DTYPE_F32;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.L = L;
  a.S = S;
  a.E = E;
  a.G = f.G;
  a.scale = f.scale;
  a.mask = f.mask;
  a.score = f.score;
  a.bm = f.bm;
  a.qB = qs->B;
  a.qH = qs->H;
  a.q_num_blocks = qs->q_num_blocks;
  a.q_indices = qs->q_indices;
  a.full_q_num_blocks = qs->full_q_num_blocks;
  a.full_q_indices = qs->full_q_indices;
  BwdMaps maps;
  if ((rc = encode_bf16_map(&maps.q, q, 128)) || (rc = encode_bf16_map(&maps.k, k, 128)) ||
      (rc = encode_bf16_map(&maps.v, v, 128)) || (rc = encode_bf16_map(&maps.dout, dout, 128)))
    return rc;
  cudaError_t e = launch_bwd(a, maps, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "backward launch");
  return FA_OK;
}

int flexattn_poll_device_status(void* stream, int32_t* status) {
  if (!status) return fail(FA_ERR_NULL, "status must not be NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e == cudaSuccess && v != 0) e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  *status = v;
  return FA_OK;
}

}  // extern "C"
