"""B200 (sm_100a) FlexAttention forward: Python binding of ``libflexattn_b200.so``.

The functions here carry the C entry points' names and only marshal
arguments: torch tensors become device pointers, sizes and strides; mask and
score specifications (plain dicts) become the C structs.  Every step of the
computation runs in the CUDA library; there is no CPU fallback -- importing
works without the library, but any call raises if it is not built.

Specification dicts (the menu of include/flexattn.h):

* mask_mod: ``{"kind": "none" | "causal" | "sliding_window" | "document" |
  "prefix_lm" | "chunked", "window": W, "n_sink": n, "prefix": P,
  "chunk": C, "doc_id": int32 tensor (B or 1, S), "kv_len": int32 tensor (B,)}``,
  or a composed rule: ``{"kind": "and" | "or", "masks": [rule, ...]}``,
  ``{"kind": "not", "mask": rule}`` over the rules above and the predicates
  ``{"kind": "distance_below" | "key_below" | "same_chunk" | "stride" |
  "head_below", "value": v}`` and ``{"kind": "same_document", "doc_id": ...}``
  (see :func:`and_masks`, :func:`or_masks`, :func:`not_mask`); ``kv_len``
  goes on the outermost rule.
* score_mod: ``{"kind": "none" | "softcap" | "alibi" | "cap_then_bias",
  "cap": c, "slope_heads": H, "pos": int32 tensor (B or 1, S) or None}``
"""

from __future__ import annotations

import ctypes as C
import math
import os
from dataclasses import dataclass

from . import _abi

__all__ = [
    "BlockMask", "FlexAttnError", "library_path", "load_library", "and_masks", "or_masks", "not_mask",
    "flexattn_version", "flexattn_last_error", "flexattn_block_mask_dims", "flexattn_build_block_mask",
    "flexattn_forward_workspace_size", "flexattn_forward", "flexattn_forward_decode_noalloc",
    "flexattn_poll_device_status", "BlockMaskQ", "flexattn_transpose_block_mask", "flexattn_backward",
]

_LIB = None
_PKG = os.path.dirname(os.path.abspath(__file__))


class FlexAttnError(RuntimeError):
    """A non-zero status from the library; ``.status`` holds the code."""

    def __init__(self, status, message):
        self.status = status
        super().__init__(f"{_abi.STATUS_NAMES.get(status, status)}: {message}")


def library_path():
    return os.path.join(_PKG, "libflexattn_b200.so")


def load_library():
    """Load the CUDA library (built in-tree by ``build.py``); raise if it is missing."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is not built: run `python -m programmable_block_sparse_b200.build` "
                "(the CUDA library is required; there is no fallback)")
        _LIB = _abi.bind(C.CDLL(path))
    return _LIB


def _check(status):
    if status != _abi.FA_OK:
        raise FlexAttnError(status, load_library().flexattn_last_error().decode())


def _stream_handle(stream):
    import torch
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return C.c_void_p(stream)
    return C.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _tensor_struct(t):
    import torch
    if t.dim() != 4:
        raise FlexAttnError(2, f"expected a 4-D tensor (B, H, N, D), got shape {tuple(t.shape)}")
    if t.dtype == torch.bfloat16:
        dt = _abi.FA_DTYPE_BF16
    elif t.dtype == torch.float32:
        dt = _abi.FA_DTYPE_F32
    else:
        raise FlexAttnError(6, f"unsupported dtype {t.dtype}")
    s = _abi.fa_tensor()
    s.data = t.data_ptr()
    s.dtype = dt
    s.reserved = 0
    for i in range(4):
        s.size[i] = t.shape[i]
        s.stride[i] = t.stride(i)
    return s


def and_masks(*rules, **extra):
    """A rule that allows a pair when every rule does (the guide's and_masks)."""
    return {"kind": "and", "masks": list(rules), **extra}


def or_masks(*rules, **extra):
    """A rule that allows a pair when any rule does (the guide's or_masks)."""
    return {"kind": "or", "masks": list(rules), **extra}


def not_mask(rule, **extra):
    """A rule that allows exactly the pairs ``rule`` hides."""
    return {"kind": "not", "mask": rule, **extra}


def _flatten(spec, out, docs):
    """Postfix instructions of a rule spec (the fixed rules spelled out)."""
    P = _abi.PROG_PRED
    k = spec["kind"]
    if k in ("and", "or"):
        subs = spec["masks"]
        op = _abi.PROG_AND if k == "and" else _abi.PROG_OR
        if not subs:  # the empty AND holds everywhere, the empty OR nowhere
            out.append((P["true"], 0))
            if k == "or":
                out.append((_abi.PROG_NOT, 0))
            return
        _flatten(subs[0], out, docs)
        for sub in subs[1:]:
            _flatten(sub, out, docs)
            out.append((op, 0))
    elif k == "not":
        _flatten(spec["mask"], out, docs)
        out.append((_abi.PROG_NOT, 0))
    elif k == "none":
        out.append((P["true"], 0))
    elif k == "causal":
        out.append((P["causal"], 0))
    elif k == "sliding_window":
        out += [(P["causal"], 0), (P["distance_below"], int(spec["window"])),
                (P["key_below"], int(spec.get("n_sink", 0))), (_abi.PROG_OR, 0), (_abi.PROG_AND, 0)]
    elif k == "prefix_lm":
        out += [(P["causal"], 0), (P["key_below"], int(spec["prefix"])), (_abi.PROG_OR, 0)]
    elif k == "chunked":
        out += [(P["causal"], 0), (P["same_chunk"], int(spec["chunk"])), (_abi.PROG_AND, 0)]
    elif k in ("document", "same_document"):
        docs.append(spec["doc_id"])
        if k == "document":
            out += [(P["causal"], 0), (P["same_document"], 0), (_abi.PROG_AND, 0)]
        else:
            out.append((P["same_document"], 0))
    elif k in P:
        out.append((P[k], int(spec.get("value", 0))))
    else:
        raise FlexAttnError(9, f"unknown mask rule {k!r}")


def _mask_struct(spec):
    spec = spec or {"kind": "none"}
    m = _abi.fa_mask_mod()
    if spec["kind"] not in _abi.MASK_KIND or spec["kind"] == "program":
        prog, docs = [], []
        _flatten(spec, prog, docs)
        if len(prog) > _abi.MASK_PROGRAM_MAX:
            raise FlexAttnError(11, f"the composed rule needs {len(prog)} instructions "
                                    f"(at most {_abi.MASK_PROGRAM_MAX})")
        m.kind = _abi.MASK_KIND["program"]
        m.n_instr = len(prog)
        for i, (op, arg) in enumerate(prog):
            m.program[i].op = op
            m.program[i].arg = arg
        if docs:
            if any(d.data_ptr() != docs[0].data_ptr() for d in docs):
                raise FlexAttnError(9, "a composed rule reads one doc_id tensor")
            m.doc_id = docs[0].data_ptr()
            m.doc_batch = docs[0].shape[0] if docs[0].dim() == 2 else 1
        kv_len = spec.get("kv_len")
        if kv_len is not None:
            m.kv_len = kv_len.data_ptr()
        return m
    m.kind = _abi.MASK_KIND[spec["kind"]]
    m.window = int(spec.get("window", 0))
    m.n_sink = int(spec.get("n_sink", 0))
    m.prefix = int(spec.get("prefix", 0))
    m.chunk = int(spec.get("chunk", 0))
    doc = spec.get("doc_id")
    if doc is not None:
        m.doc_id = doc.data_ptr()
        m.doc_batch = doc.shape[0] if doc.dim() == 2 else 1
    kv_len = spec.get("kv_len")
    if kv_len is not None:
        m.kv_len = kv_len.data_ptr()
    return m


def _score_struct(spec):
    spec = spec or {"kind": "none"}
    s = _abi.fa_score_mod()
    s.kind = _abi.SCORE_KIND[spec["kind"]]
    s.cap = float(spec.get("cap", 0.0))
    s.slope_heads = int(spec.get("slope_heads", 0) or 0)
    pos = spec.get("pos")
    if pos is not None and not isinstance(pos, str):
        s.pos = pos.data_ptr()
        s.pos_batch = pos.shape[0] if pos.dim() == 2 else 1
    return s


@dataclass
class BlockMask:
    """Device-resident BlockMask: the four int32 arrays and their extents."""

    B: int
    H: int
    L: int
    S: int
    BM: int
    BN: int
    Mb: int
    Nb: int
    kv_num_blocks: object
    kv_indices: object
    full_kv_num_blocks: object
    full_kv_indices: object

    def as_struct(self):
        s = _abi.fa_block_mask()
        s.B, s.H, s.L, s.S, s.BM, s.BN, s.Mb, s.Nb = (self.B, self.H, self.L, self.S, self.BM, self.BN,
                                                      self.Mb, self.Nb)
        s.kv_num_blocks = self.kv_num_blocks.data_ptr()
        s.kv_indices = self.kv_indices.data_ptr()
        s.full_kv_num_blocks = self.full_kv_num_blocks.data_ptr()
        s.full_kv_indices = self.full_kv_indices.data_ptr()
        return s


def flexattn_version():
    return load_library().flexattn_version()


def flexattn_last_error():
    return load_library().flexattn_last_error().decode()


def flexattn_block_mask_dims(L, S, BM, BN):
    mb, nb = C.c_int32(), C.c_int32()
    _check(load_library().flexattn_block_mask_dims(L, S, BM, BN, C.byref(mb), C.byref(nb)))
    return mb.value, nb.value


def flexattn_build_block_mask(mask_mod, B, H, L, S, BM=128, BN=128, device="cuda", stream=None, out=None):
    """Allocate the BlockMask arrays on ``device`` and classify every tile on the GPU."""
    import torch
    Mb, Nb = flexattn_block_mask_dims(L, S, BM, BN)
    if out is None:
        z = dict(dtype=torch.int32, device=device)
        out = BlockMask(B, H, L, S, BM, BN, Mb, Nb, torch.empty((B, H, Mb), **z), torch.empty((B, H, Mb, Nb), **z),
                        torch.empty((B, H, Mb), **z), torch.empty((B, H, Mb, Nb), **z))
    m = _mask_struct(mask_mod)
    bm = out.as_struct()
    _check(load_library().flexattn_build_block_mask(C.byref(m), C.byref(bm), _stream_handle(stream)))
    return out


def flexattn_forward_workspace_size(q, k, v, block_mask, split_kv=0, paged=None):
    n = C.c_size_t()
    qs, ks, vs, bm = _tensor_struct(q), _tensor_struct(k), _tensor_struct(v), block_mask.as_struct()
    opts = _options_struct(None, False, 0, paged)
    _check(load_library().flexattn_forward_workspace_size(C.byref(qs), C.byref(ks), C.byref(vs), C.byref(bm),
                                                          int(split_kv), None if opts is None else C.byref(opts),
                                                          C.byref(n)))
    return n.value


def _options_struct(max_scores, rows_guaranteed_safe, wait_cycles, paged=None):
    if max_scores is None and not rows_guaranteed_safe and not wait_cycles and paged is None:
        return None
    o = _abi.fa_forward_options()
    o.max_scores = None if max_scores is None else max_scores.data_ptr()
    o.wait_cycles = int(wait_cycles or 0)
    o.flags = _abi.FA_FLAG_ROWS_GUARANTEED_SAFE if rows_guaranteed_safe else 0
    o.reserved = 0
    if paged is not None:
        table = paged["page_table"]
        o.page_table = table.data_ptr()
        o.page_size = int(paged["page_size"])
        o.pages_per_seq = int(table.shape[-1])
    return o


def flexattn_forward(q, k, v, block_mask, score_mod=None, mask_mod=None, scale=None, enable_gqa=False,
                     out=None, lse=True, split_kv=0, workspace=None, stream=None, out_dtype=None,
                     max_scores=None, rows_guaranteed_safe=False, wait_cycles=0, paged=None):
    """Run the forward pass; returns ``(out, lse)`` (lse None when ``lse=False``),
    or ``(out, lse, max_scores)`` when ``max_scores`` is requested.

    ``out`` / ``lse`` may be preallocated tensors; ``out_dtype`` (torch.float32
    or the input dtype) picks the output type when ``out`` is None;
    ``workspace`` a uint8 device tensor of at least
    :func:`flexattn_forward_workspace_size` bytes (allocated here when None and
    needed).  ``max_scores``: True (allocate) or an fp32 (B, Hq, L) tensor for
    the per-row maximum score.  ``rows_guaranteed_safe`` sets
    FA_FLAG_ROWS_GUARANTEED_SAFE; ``wait_cycles`` the device wait budget.
    ``paged``: ``{"page_table": int32 (B, pages_per_seq), "page_size": P}``
    when k and v are page pools (num_pages, Hkv, P, D).
    """
    import torch
    B, Hq, L, _ = q.shape
    Ev = v.shape[3]
    if out is None:
        out = torch.empty((B, Hq, L, Ev), dtype=out_dtype or q.dtype, device=q.device)
    if lse is True:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    elif lse is False:
        lse = None
    want_max = max_scores is not None and max_scores is not False
    if max_scores is True:
        max_scores = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    elif max_scores is False:
        max_scores = None
    opts = _options_struct(max_scores, rows_guaranteed_safe, wait_cycles, paged)
    ws_bytes = flexattn_forward_workspace_size(q, k, v, block_mask, split_kv, paged)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    qs, ks, vs, os_ = _tensor_struct(q), _tensor_struct(k), _tensor_struct(v), _tensor_struct(out)
    bm = block_mask.as_struct()
    sm, mm = _score_struct(score_mod), _mask_struct(mask_mod)
    sc = 0.0 if scale is None else float(scale)
    if math.isnan(sc):
        sc = 0.0
    _check(load_library().flexattn_forward(
        C.byref(qs), C.byref(ks), C.byref(vs), C.byref(os_), _ptr(lse), C.c_float(sc), int(bool(enable_gqa)),
        C.byref(sm), C.byref(mm), C.byref(bm), int(split_kv), None if opts is None else C.byref(opts),
        _ptr(workspace), C.c_size_t(workspace.numel() if workspace is not None else 0), _stream_handle(stream)))
    if want_max:
        return out, lse, max_scores
    return out, lse


def flexattn_forward_decode_noalloc(q, k, v, block_mask, score_mod=None, mask_mod=None, scale=None,
                                    enable_gqa=False, out=None, lse=True, split_kv=0, stream=None):
    """Split-KV decode without a workspace: for callers that cannot allocate
    device memory at call time.  The library's built-in 16 MiB scratch holds
    the per-split partial results; calls that overlap on the GPU share it and
    must be serialised.  Returns ``(out, lse)``; ``out``/``lse`` may be
    preallocated so that the call allocates nothing at all."""
    import torch
    B, Hq, L, _ = q.shape
    if out is None:
        out = torch.empty((B, Hq, L, v.shape[3]), dtype=q.dtype, device=q.device)
    if lse is True:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    elif lse is False:
        lse = None
    qs, ks, vs, os_ = _tensor_struct(q), _tensor_struct(k), _tensor_struct(v), _tensor_struct(out)
    bm = block_mask.as_struct()
    sm, mm = _score_struct(score_mod), _mask_struct(mask_mod)
    sc = 0.0 if scale is None or math.isnan(float(scale)) else float(scale)
    _check(load_library().flexattn_forward_decode_noalloc(
        C.byref(qs), C.byref(ks), C.byref(vs), C.byref(os_), _ptr(lse), C.c_float(sc), int(bool(enable_gqa)),
        C.byref(sm), C.byref(mm), C.byref(bm), int(split_kv), _stream_handle(stream)))
    return out, lse


def flexattn_poll_device_status(stream=None):
    """Synchronise ``stream`` and return (and clear) the kernels' device status code."""
    st = C.c_int32()
    _check(load_library().flexattn_poll_device_status(_stream_handle(stream), C.byref(st)))
    return st.value


@dataclass
class BlockMaskQ:
    """Device-resident query-side lists of a BlockMask (for the backward pass)."""

    B: int
    H: int
    Mb: int
    Nb: int
    q_num_blocks: object
    q_indices: object
    full_q_num_blocks: object
    full_q_indices: object

    def as_struct(self):
        s = _abi.fa_block_mask_q()
        s.B, s.H, s.Mb, s.Nb = self.B, self.H, self.Mb, self.Nb
        s.q_num_blocks = self.q_num_blocks.data_ptr()
        s.q_indices = self.q_indices.data_ptr()
        s.full_q_num_blocks = self.full_q_num_blocks.data_ptr()
        s.full_q_indices = self.full_q_indices.data_ptr()
        return s


def flexattn_transpose_block_mask(block_mask, stream=None, out=None):
    """Query-side lists of ``block_mask`` (allocated here unless ``out`` is given)."""
    import torch
    bm = block_mask
    if out is None:
        z = dict(dtype=torch.int32, device=bm.kv_num_blocks.device)
        out = BlockMaskQ(bm.B, bm.H, bm.Mb, bm.Nb, torch.empty((bm.B, bm.H, bm.Nb), **z),
                         torch.empty((bm.B, bm.H, bm.Nb, bm.Mb), **z), torch.empty((bm.B, bm.H, bm.Nb), **z),
                         torch.empty((bm.B, bm.H, bm.Nb, bm.Mb), **z))
    s, q = bm.as_struct(), out.as_struct()
    _check(load_library().flexattn_transpose_block_mask(C.byref(s), C.byref(q), _stream_handle(stream)))
    return out


def flexattn_backward(q, k, v, out, dout, lse, block_mask, q_side=None, score_mod=None, mask_mod=None, scale=None,
                      enable_gqa=False, dq=None, dk=None, dv=None, grad_dtype=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv) of sum(out * dout) for the forward pass with the
    same arguments; ``lse`` is the forward's.  ``q_side`` defaults to the
    transposed lists of ``block_mask``; gradients are allocated in
    ``grad_dtype`` (default: the input dtype) unless given."""
    import torch
    gd = grad_dtype or q.dtype
    dq = torch.empty(q.shape, dtype=gd, device=q.device) if dq is None else dq
    dk = torch.empty(k.shape, dtype=gd, device=q.device) if dk is None else dk
    dv = torch.empty(v.shape, dtype=gd, device=q.device) if dv is None else dv
    if q_side is None:
        q_side = flexattn_transpose_block_mask(block_mask, stream=stream)
    n = C.c_size_t()
    qs = _tensor_struct(q)
    _check(load_library().flexattn_backward_workspace_size(C.byref(qs), C.byref(n)))
    if workspace is None:
        workspace = torch.empty(max(1, n.value), dtype=torch.uint8, device=q.device)
    ks, vs, os_, ds = _tensor_struct(k), _tensor_struct(v), _tensor_struct(out), _tensor_struct(dout)
    gq, gk, gv = _tensor_struct(dq), _tensor_struct(dk), _tensor_struct(dv)
    bm, qsd = block_mask.as_struct(), q_side.as_struct()
    sm, mm = _score_struct(score_mod), _mask_struct(mask_mod)
    sc = 0.0 if scale is None or math.isnan(float(scale)) else float(scale)
    _check(load_library().flexattn_backward(
        C.byref(qs), C.byref(ks), C.byref(vs), C.byref(os_), C.byref(ds), _ptr(lse), C.byref(gq), C.byref(gk),
        C.byref(gv), C.c_float(sc), int(bool(enable_gqa)), C.byref(sm), C.byref(mm), C.byref(bm), C.byref(qsd),
        _ptr(workspace), C.c_size_t(workspace.numel()), _stream_handle(stream)))
    return dq, dk, dv
