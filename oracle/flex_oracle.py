"""Plain fp64 CPU oracle for the FlexAttention forward pass and BlockMask.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import or run this module.
The CUDA library never calls it, and it shares no code, constants or tables
with the CUDA library: mask and score kinds here are strings, interpreted
below from the pages' formulas.

Sources ("page" = the web page, cited by its title and section):

* "flexattention-score-mod-block-mask" (charlestar.github.io), sections
  "What one connection goes through" (the semantic definition of s_ij,
  s~_ij and o_i), "score_mod changes the score, and the order changes the
  result" (cap-then-bias combination, masking after the score transform),
  "mask_mod defines legal connections, BlockMask defines block work"
  (empty / full / partial tiles), "A call example pinned to one version"
  (window 0 <= p_i - p_j < W), "Packing" (same document), "At decode,
  q_idx = 0 is not position 0" (logical query position), "Correctness
  checks come before performance" (fully masked rows).
* "PyTorch Flex Attention complete guide" (2kiu.com), sections 1.2
  (score_mod receives the *query* head), 2 (lse output), 3.1 (a block is
  sparse only if all its elements are masked), 3.2 (dense reconstruction of
  the ordered block lists), 4.1 (create_block_mask pipeline: dense mask,
  pad, per-block reduction, separate full blocks), 6.1 (GQA broadcast),
  6.2 (default scale 1/sqrt(E)).
* "Attention expressions" (docs.tensorcad.dev), section "Examples" (prefix-LM,
  sinks, chunked attention, ALiBi slope, Gemma-2 soft-cap).
* "Causal Mask" (quant67.com, Transformer series no. 17), section 4
  "query shorter than key: bottom-right alignment" and section 7 "-inf,
  finfo.min and fully masked rows".

Readings taken where the pages leave a step open (each is listed in the
design notes too):

* Query positions are logical: q_pos = i + (S_b - L), S_b the valid KV
  length of sequence b (S when none is given).  All mask and score rules see
  q_pos; key positions are kv = j.  Keys j >= S_b are never visible.
* A fully masked row (no visible key, or every visible score mapped to -inf
  by the score rule) gives output 0 and lse = -inf, never NaN.
* lse is the natural-log log-sum-exp of the transformed, scaled scores over
  the visible keys.
* GQA maps query head h to KV head h // (Hq // Hkv); the score rule sees the
  query head.
* ALiBi / distance slope for head h is 2^(-8 (h + 1) / H), h from 0.
* Tiles at a ragged edge are classified over their in-range cells only.
  Index lists are ascending; unused slots hold 0.
* max_scores (the guide's per-row maximum, section 2) is the largest
  transformed score among the visible keys, in lse's units; -inf for a row
  with no visible key.
* Composed rules (guide section 4.3, and_masks / or_masks; "Attention
  expressions", Examples): the predicates carry no causal bound of their own;
  same-chunk divides by floor; stride means q = kv (mod a); head-below reads
  the query head; NOT complements over in-range keys.
* A paged cache holds logical key j of sequence b in slot j % page_size of
  page page_table[b][j // page_size]; every rule sees logical positions.
* The backward is the chain rule of the forward definition; D is formed from
  the output the backward receives (the stored output when one is given).

Rows are computed in groups of whole rows purely to bound memory; every row
is evaluated in full, exactly as the definition states.
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf

MASK_KINDS = ("none", "causal", "sliding_window", "document", "prefix_lm", "chunked", "dense",
              # predicates and combinators for composed masks
              "distance_below", "key_below", "same_chunk", "same_document", "stride", "head_below",
              "and", "or", "not")
SCORE_KINDS = ("none", "softcap", "alibi", "cap_then_bias")


# ---------------------------------------------------------------------------
# Positions
# ---------------------------------------------------------------------------

def query_positions(L, S_b):
    """Logical query positions q_pos = i + (S_b - L) (bottom-right alignment).

    "Causal Mask" (quant67.com) section 4: with L < S the r-th query sees the
    first S - L + r + 1 keys; "flexattention-score-mod-block-mask" section
    "At decode, q_idx = 0 is not position 0": q_position = q_idx + q_offset.
    """
    return np.arange(L, dtype=np.int64) + (int(S_b) - int(L))


def _row_for_batch(arr, b):
    """Row b of a (B, S) array, or its only row when it broadcasts (1, S) / (S,)."""
    arr = np.asarray(arr)
    if arr.ndim == 1:
        return arr
    return arr[b] if arr.shape[0] > 1 else arr[0]


def doc_positions_from_ids(doc_row):
    """Position of each token inside its own document (restarting at 0).

    "flexattention-score-mod-block-mask" section "Packing": the in-segment
    position column of the packing table restarts at 0 for every sample.
    """
    doc_row = np.asarray(doc_row)
    pos = np.zeros(len(doc_row), dtype=np.int64)
    for t in range(1, len(doc_row)):
        pos[t] = pos[t - 1] + 1 if doc_row[t] == doc_row[t - 1] else 0
    return pos


# ---------------------------------------------------------------------------
# mask_mod: visibility M(b, h, q_pos, kv)
# ---------------------------------------------------------------------------

def visible(mask, b, h, qp, kv, S_b):
    """Boolean visibility for query positions ``qp`` (column) x keys ``kv`` (row).

    ``mask`` is a dict with ``kind`` in MASK_KINDS:

    * none -- every in-range key (the noop mask; guide section 4.4).
    * causal -- kv <= q.
    * sliding_window -- kv <= q and (q - kv < W or kv < n_sink): window of W
      keys including the query itself ("flexattention-score-mod-block-mask",
      "A call example pinned to one version": 0 <= p_i - p_j < W), plus sink
      tokens ("Attention expressions", Examples: q - kv < W or kv < 4 with
      causal on).
    * document -- kv <= q and doc[q] == doc[kv] ("flexattention-score-mod-
      block-mask", "Packing"; "Causal Mask" section 3, intra-document causal).
    * prefix_lm -- kv <= q or kv < P, causal off ("Attention expressions",
      Examples; "Causal Mask" section 3, Prefix LM).
    * chunked -- kv <= q and floor(q / C) == floor(kv / C)
      ("Attention expressions", Examples, causal on).
    * dense -- an explicit (L, S) boolean matrix (oracle-only, for the pages'
      key-padding example).

    Composed masks ("PyTorch Flex Attention complete guide" section 4.3:
    and_masks / or_masks combine any number of mask rules into one, by
    intersection or union; "Attention expressions", Examples: every fourth
    key, half the heads global and half local):

    * and / or -- every / any rule of ``masks`` allows the pair; not -- the
      rule ``mask`` does not.
    * distance_below -- q - kv < value (no causal bound of its own).
    * key_below -- kv < value.
    * same_chunk -- floor(q / value) == floor(kv / value).
    * same_document -- doc[q] == doc[kv] (no causal bound of its own).
    * stride -- q - kv is a multiple of value (q = kv modulo value).
    * head_below -- h < value (the query head).

    Keys at or beyond the valid length S_b are invisible under every kind.
    """
    qp1 = np.asarray(qp, dtype=np.int64)
    kv1 = np.asarray(kv, dtype=np.int64)
    qp = qp1[:, None]
    kv = kv1[None, :]
    kind = mask["kind"]
    in_range = kv < S_b
    causal = kv <= qp
    if kind == "none":
        m = np.ones(np.broadcast(qp, kv).shape, dtype=bool)
    elif kind == "causal":
        m = causal
    elif kind == "sliding_window":
        W, n_sink = int(mask["window"]), int(mask.get("n_sink", 0))
        m = causal & (((qp - kv) < W) | (kv < n_sink))
    elif kind == "document":
        doc_b = _row_for_batch(mask["doc_id"], b)
        qi = np.clip(qp, 0, len(doc_b) - 1)
        ki = np.clip(kv, 0, len(doc_b) - 1)
        m = causal & (qp >= 0) & (doc_b[qi] == doc_b[ki])
    elif kind == "prefix_lm":
        P = int(mask["prefix"])
        m = causal | (kv < P)
    elif kind == "chunked":
        C = int(mask["chunk"])
        m = causal & (np.floor_divide(qp, C) == np.floor_divide(kv, C))
    elif kind == "dense":
        m = np.asarray(mask["matrix"], dtype=bool)
        rows = mask.get("rows")
        m = m if rows is None else m[np.asarray(rows)]
    elif kind == "and":
        m = np.ones(np.broadcast(qp, kv).shape, dtype=bool)
        for sub in mask["masks"]:
            m = m & visible(sub, b, h, qp1, kv1, S_b)
    elif kind == "or":
        m = np.zeros(np.broadcast(qp, kv).shape, dtype=bool)
        for sub in mask["masks"]:
            m = m | visible(sub, b, h, qp1, kv1, S_b)
    elif kind == "not":
        m = ~visible(mask["mask"], b, h, qp1, kv1, S_b)
    elif kind == "distance_below":
        m = (qp - kv) < int(mask["value"])
    elif kind == "key_below":
        m = kv < int(mask["value"])
    elif kind == "same_chunk":
        C = int(mask["value"])
        m = np.floor_divide(qp, C) == np.floor_divide(kv, C)
    elif kind == "same_document":
        doc_b = _row_for_batch(mask["doc_id"], b)
        qi = np.clip(qp, 0, len(doc_b) - 1)
        ki = np.clip(kv, 0, len(doc_b) - 1)
        m = (qp >= 0) & (qp < len(doc_b)) & (doc_b[qi] == doc_b[ki])
    elif kind == "stride":
        m = np.mod(qp - kv, int(mask["value"])) == 0
    elif kind == "head_below":
        m = np.full(np.broadcast(qp, kv).shape, h < int(mask["value"]))
    else:
        raise ValueError(f"unknown mask kind {kind!r}")
    return np.broadcast_to(m, np.broadcast(qp, kv).shape) & in_range


# ---------------------------------------------------------------------------
# score_mod: g(s, b, h, q_pos, kv)
# ---------------------------------------------------------------------------

def distance_slope(h, H):
    """2^(-8 (h+1) / H) ("Attention expressions", Examples: ALiBi)."""
    return 2.0 ** (-8.0 * (h + 1) / H)


def score_mod(score, s, b, h, qp, kv, Hq):
    """Apply the score transform g to the scaled scores ``s`` (rows qp, cols kv).

    * none -- g = s.
    * softcap -- g = c tanh(s / c) ("flexattention-score-mod-block-mask",
      "score_mod changes the score"; "Attention expressions", Gemma 2's cap).
    * alibi -- g = s - slope_h (q - kv) ("Attention expressions", Examples).
    * cap_then_bias -- g = c tanh(s / c) + slope_h (p_kv - p_q): cap first,
      then the distance bias ("flexattention-score-mod-block-mask", "score_mod
      changes the score": the bias-then-cap form is a different rule).  p is
      the in-document position when ``pos == 'in_doc'`` (computed here from
      the document ids), else the global position.
    """
    kind = score["kind"]
    if kind == "none":
        return s
    if kind == "softcap":
        c = float(score["cap"])
        return c * np.tanh(s / c)
    H = int(score.get("slope_heads") or Hq)
    slope = distance_slope(h, H)
    qp = np.asarray(qp, dtype=np.int64)[:, None]
    kv = np.asarray(kv, dtype=np.int64)[None, :]
    if kind == "alibi":
        return s - slope * (qp - kv).astype(np.float64)
    if kind == "cap_then_bias":
        c = float(score["cap"])
        if score.get("pos", "global") == "in_doc":
            doc_b = _row_for_batch(score["doc_id"], b)
            p = doc_positions_from_ids(doc_b)
            pq = p[np.clip(qp, 0, len(p) - 1)]
            pk = p[np.clip(kv, 0, len(p) - 1)]
        else:
            pq, pk = qp, kv
        return c * np.tanh(s / c) + slope * (pk - pq).astype(np.float64)
    raise ValueError(f"unknown score kind {kind!r}")


# ---------------------------------------------------------------------------
# Forward
# ---------------------------------------------------------------------------

def _as_f64(x):
    if hasattr(x, "detach"):  # a torch tensor: upcast exactly
        import torch
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def attention_rows(q_rows, k, v, scale, mask, score, b, h, qp, S_b, Hq, with_max=False):
    """Output rows and lse for one (b, h) and a set of query positions.

    The definition in "flexattention-score-mod-block-mask", "What one
    connection goes through": s_ij = scale q_i . k_j; s~_ij = g(s_ij, ...) where
    M_ij, -inf elsewhere; o_i = sum_j softmax_j(s~_ij) v_j.  The score rule is
    applied first and the mask second (section "score_mod changes the score").

    With ``with_max`` the row maximum of s~ is returned third: the per-row
    maximum score that "PyTorch Flex Attention complete guide" section 2
    (AuxRequest / AuxOutput) offers beside lse, read here as the largest
    transformed score among the visible keys (natural units, the quantity
    whose log-sum-exp is lse) and -inf for a row with no visible key.
    """
    S = k.shape[0]
    kv = np.arange(S, dtype=np.int64)
    s = scale * (q_rows @ k.T)                      # full score rows
    g = score_mod(score, s, b, h, qp, kv, Hq)       # transform everywhere
    vis = visible(mask, b, h, qp, kv, S_b)
    bad = vis & (np.isnan(g) | (g == np.inf))
    assert not bad.any(), "score rule produced NaN or +inf on a visible cell"
    st = np.where(vis, g, NEG_INF)                  # mask after the transform
    m = st.max(axis=1)
    out = np.zeros((q_rows.shape[0], v.shape[1]), dtype=np.float64)
    lse = np.full(q_rows.shape[0], NEG_INF)
    live = m > NEG_INF
    if live.any():
        p = np.exp(st[live] - m[live, None])
        l = p.sum(axis=1)
        out[live] = (p @ v) / l[:, None]
        lse[live] = m[live] + np.log(l)
    if with_max:
        return out, lse, st.max(axis=1)
    return out, lse


def forward(q, k, v, scale=None, mask=None, score=None, kv_len=None, enable_gqa=False, row_group=512, aux=False):
    """fp64 FlexAttention forward: returns (out (B,Hq,L,Ev), lse (B,Hq,L)).

    q (B,Hq,L,E), k (B,Hkv,S,E), v (B,Hkv,S,Ev); numpy arrays or torch
    tensors (upcast exactly).  ``scale`` defaults to 1/sqrt(E) (guide section
    6.2).  GQA broadcasts KV head h // (Hq // Hkv) (guide section 6.1).
    With ``aux`` a third array, max_scores (B,Hq,L), is returned (see
    :func:`attention_rows`).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, Hq, L, E = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    if Hq != Hkv:
        assert enable_gqa and Hq % Hkv == 0, "Hq != Hkv needs enable_gqa and Hq % Hkv == 0"
    G = Hq // Hkv
    mask = mask or {"kind": "none"}
    score = score or {"kind": "none"}
    scale = 1.0 / math.sqrt(E) if scale is None else float(scale)
    out = np.zeros((B, Hq, L, v.shape[3]))
    lse = np.full((B, Hq, L), NEG_INF)
    mxs = np.full((B, Hq, L), NEG_INF)
    for b in range(B):
        S_b = S if kv_len is None else int(np.asarray(kv_len)[b])
        for h in range(Hq):
            hk = h // G
            out[b, h], lse[b, h], mxs[b, h] = forward_unit(q[b, h], k[b, hk], v[b, hk], b, h, Hq, S_b, scale,
                                                           mask, score, row_group)
    return (out, lse, mxs) if aux else (out, lse)


def forward_unit(q_bh, k_bh, v_bh, b, h, Hq, S_b, scale, mask, score, row_group=512):
    """Every query row of one (batch b, query head h) unit: (out (L,Ev), lse (L,), max_scores (L,)).

    q_bh (L,E) are the unit's queries; k_bh (S,E), v_bh (S,Ev) its KV head's
    keys and values; S_b the valid KV length of sequence b; Hq the number of
    query heads (the slope of the distance rules reads h and Hq).  This is
    the body of :func:`forward` for one (b, h), exposed so that large
    workloads can be checked unit by unit.  Rows are evaluated in groups of
    ``row_group`` only to bound memory.
    """
    q_bh, k_bh, v_bh = _as_f64(q_bh), _as_f64(k_bh), _as_f64(v_bh)
    L = q_bh.shape[0]
    qp_all = query_positions(L, S_b)
    out = np.zeros((L, v_bh.shape[1]))
    lse = np.full(L, NEG_INF)
    mxs = np.full(L, NEG_INF)
    for r0 in range(0, L, row_group):
        r1 = min(L, r0 + row_group)
        mk = dict(mask)
        if mask["kind"] == "dense":
            mk["rows"] = np.arange(r0, r1)
        out[r0:r1], lse[r0:r1], mxs[r0:r1] = attention_rows(q_bh[r0:r1], k_bh, v_bh, scale, mk, score, b, h,
                                                            qp_all[r0:r1], S_b, Hq, with_max=True)
    return out, lse, mxs


def forward_sampled(q, k, v, samples, scale=None, mask=None, score=None, kv_len=None, enable_gqa=False, aux=False):
    """Output and lse for sampled (b, h, row) triples; returns (out[n,Ev], lse[n]).

    Used on workloads too large for :func:`forward`: each sampled row is
    computed in full by :func:`attention_rows`.  With ``aux`` the rows'
    max_scores come third.
    """
    Bq, Hq, L, E = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    G = Hq // Hkv
    mask = mask or {"kind": "none"}
    score = score or {"kind": "none"}
    scale = 1.0 / math.sqrt(E) if scale is None else float(scale)
    outs, lses, mxs = [], [], []
    for (b, h, r) in samples:
        S_b = S if kv_len is None else int(np.asarray(kv_len)[b])
        qp = query_positions(L, S_b)[r:r + 1]
        qrow = _as_f64(q[b, h, r:r + 1])
        kk = _as_f64(k[b, h // G])
        vv = _as_f64(v[b, h // G])
        o, ls, mx = attention_rows(qrow, kk, vv, scale, mask, score, b, h, qp, S_b, Hq, with_max=True)
        outs.append(o[0])
        lses.append(ls[0])
        mxs.append(mx[0])
    if aux:
        return np.stack(outs), np.array(lses), np.array(mxs)
    return np.stack(outs), np.array(lses)


# ---------------------------------------------------------------------------
# Backward pass
# ---------------------------------------------------------------------------

def score_mod_slope(score, s):
    """dg/ds of the score rule at the scaled scores ``s``.

    The distance biases do not depend on s (slope 1); the soft-cap
    g = c tanh(s / c) has dg/ds = 1 - tanh(s / c)^2.
    """
    kind = score["kind"]
    if kind in ("softcap", "cap_then_bias"):
        c = float(score["cap"])
        return 1.0 - np.tanh(s / c) ** 2
    if kind in ("none", "alibi"):
        return np.ones_like(s)
    raise ValueError(f"unknown score kind {kind!r}")


def backward_unit(q_bh, k_bh, v_bh, do_bh, b, h, Hq, S_b, scale, mask, score, out_bh=None):
    """Gradients of one (batch b, query head h) unit: (dq (L,E), dk (S,E), dv (S,Ev)).

    "flexattention-score-mod-block-mask" shows the loss's backward call
    through flex_attention; the gradients are those of the forward
    definition ("What one connection goes through"), by the chain rule:
    with P the softmax weights (0 on hidden keys) and O = P V,
        dV = P^T dO,  dP = dO V^T,  D_i = sum_e dO_ie O_ie,
        dS~ = P * (dP - D),  ds = dS~ * dg/ds,
        dQ = scale ds K,  dK = scale ds^T Q.
    A row without a visible key has P = 0 and contributes nothing.  k and v
    gradients are those of this unit alone; GQA sums them over the query
    heads that share a KV head (:func:`backward`).

    ``out_bh`` is the forward output as the caller stored it (for bf16
    outputs, O rounded to bf16).  A backward call receives the stored output
    and forms D from it, so D carries that rounding; by default D uses the
    exact O.
    """
    q_bh, k_bh, v_bh, do_bh = _as_f64(q_bh), _as_f64(k_bh), _as_f64(v_bh), _as_f64(do_bh)
    L, S = q_bh.shape[0], k_bh.shape[0]
    qp = query_positions(L, S_b)
    kv = np.arange(S, dtype=np.int64)
    s = scale * (q_bh @ k_bh.T)
    g = score_mod(score, s, b, h, qp, kv, Hq)
    vis = visible(mask, b, h, qp, kv, S_b)
    masked = np.where(vis, g, NEG_INF)
    m = masked.max(axis=1)
    p = np.zeros_like(s)
    live = m > NEG_INF
    if live.any():
        e = np.exp(masked[live] - m[live, None])
        p[live] = e / e.sum(axis=1, keepdims=True)
    o = p @ v_bh if out_bh is None else _as_f64(out_bh)
    dv = p.T @ do_bh
    dp = do_bh @ v_bh.T
    D = (do_bh * o).sum(axis=1)
    dst = p * (dp - D[:, None])
    ds = dst * score_mod_slope(score, s)
    dq = scale * (ds @ k_bh)
    dk = scale * (ds.T @ q_bh)
    return dq, dk, dv


def backward_rows(q_rows, k, v, do_rows, scale, mask, score, b, h, qp, S_b, Hq, out_rows=None):
    """The part of one unit's gradients that a set of its query rows gives:
    (dq of those rows, their contribution to dk (S,E), to dv (S,Ev)).

    The same chain rule as :func:`backward_unit`, restricted to the rows at
    logical positions ``qp``: every row's dq depends on that row alone, and
    dk, dv are sums over rows, so a unit's gradients are the row blocks' dq
    stacked and their dk, dv parts added.  ``out_rows`` is the stored output
    of those rows (D is formed from it), by default the exact one.
    """
    q_rows, k, v, do_rows = _as_f64(q_rows), _as_f64(k), _as_f64(v), _as_f64(do_rows)
    kv = np.arange(k.shape[0], dtype=np.int64)
    s = (q_rows @ k.T) * scale
    g = score_mod(score, s, b, h, qp, kv, Hq)
    vis = visible(mask, b, h, qp, kv, S_b)
    masked = np.where(vis, g, NEG_INF)
    m = masked.max(axis=1)
    p = np.zeros_like(s)
    live = m > NEG_INF
    if live.any():
        e = np.exp(masked[live] - m[live, None])
        p[live] = e / e.sum(axis=1, keepdims=True)
    o = p @ v if out_rows is None else _as_f64(out_rows)
    D = (do_rows * o).sum(axis=1)
    ds = p * (do_rows @ v.T - D[:, None]) * score_mod_slope(score, s)
    return scale * (ds @ k), scale * (ds.T @ q_rows), p.T @ do_rows


def backward(q, k, v, do, scale=None, mask=None, score=None, kv_len=None, enable_gqa=False, out=None):
    """fp64 gradients (dq (B,Hq,L,E), dk (B,Hkv,S,E), dv (B,Hkv,S,Ev)) of
    sum(out * do) for the forward of :func:`forward`; GQA sums dk and dv over
    the query heads of each KV head ("PyTorch Flex Attention complete guide"
    section 6.1: the KV heads are broadcast to the query heads).  ``out``
    (B,Hq,L,Ev), optional: the stored forward output that D is formed from
    (see :func:`backward_unit`)."""
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, Hq, L, E = q.shape
    Hkv, S = k.shape[1], k.shape[2]
    if Hq != Hkv:
        assert enable_gqa and Hq % Hkv == 0, "Hq != Hkv needs enable_gqa and Hq % Hkv == 0"
    G = Hq // Hkv
    mask = mask or {"kind": "none"}
    score = score or {"kind": "none"}
    scale = 1.0 / math.sqrt(E) if scale is None else float(scale)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        S_b = S if kv_len is None else int(np.asarray(kv_len)[b])
        for h in range(Hq):
            kvh = h // G
            uq, uk, uv = backward_unit(q[b, h], k[b, kvh], v[b, kvh], do[b, h], b, h, Hq, S_b, scale, mask, score,
                                       None if out is None else out[b, h])
            dq[b, h] = uq
            dk[b, kvh] += uk
            dv[b, kvh] += uv
    return dq, dk, dv


def transpose_block_mask(bm):
    """Query-side lists of a BlockMask: for every key tile n, the query tiles
    m whose row lists n as full or as partial, ascending, unused slots 0.

    "PyTorch Flex Attention complete guide" section 3.3: from_kv_blocks
    derives the query-side block information (_transpose_ordered) that the
    backward pass walks.  Returns q_num_blocks (B,H,Nb), q_indices (B,H,Nb,Mb),
    full_q_num_blocks, full_q_indices.
    """
    B, H, Mb = bm["kv_num_blocks"].shape
    Nb = bm["Nb"]
    out = {"q_num_blocks": np.zeros((B, H, Nb), np.int32), "q_indices": np.zeros((B, H, Nb, Mb), np.int32),
           "full_q_num_blocks": np.zeros((B, H, Nb), np.int32),
           "full_q_indices": np.zeros((B, H, Nb, Mb), np.int32)}
    for b in range(B):
        for h in range(H):
            for kind, cnt, idx in (("", "kv_num_blocks", "kv_indices"),
                                   ("full_", "full_kv_num_blocks", "full_kv_indices")):
                lists = [[] for _ in range(Nb)]
                for m in range(Mb):
                    for i in range(int(bm[cnt][b, h, m])):
                        lists[int(bm[idx][b, h, m, i])].append(m)
                for n in range(Nb):
                    out[kind + "q_num_blocks"][b, h, n] = len(lists[n])
                    out[kind + "q_indices"][b, h, n, :len(lists[n])] = sorted(lists[n])
    return out


# ---------------------------------------------------------------------------
# Paged KV cache
# ---------------------------------------------------------------------------

def gather_pages(pool, page_table, page_size, pages_per_seq):
    """The logical cache (B, H, pages_per_seq * page_size, D) of a paged pool.

    "flexattention-score-mod-block-mask", "At decode, q_idx = 0 is not
    position 0": in a paged or circular cache layout the storage position
    has to be mapped back to the logical position.  Reading taken: the pool
    is (num_pages, H, page_size, D); logical key j of sequence b lives in
    physical page page_table[b][j // page_size], slot j % page_size.  Every
    rule (mask, score, valid length) sees logical positions only.
    """
    pool = _as_f64(pool)
    table = np.asarray(page_table, dtype=np.int64)
    B = table.shape[0]
    H, D = pool.shape[1], pool.shape[3]
    out = np.zeros((B, H, pages_per_seq * page_size, D))
    for b in range(B):
        for i in range(pages_per_seq):
            out[b, :, i * page_size:(i + 1) * page_size] = pool[table[b, i]]
    return out


def forward_paged(q, k_pages, v_pages, page_table, page_size, pages_per_seq, scale=None, mask=None, score=None,
                  kv_len=None, enable_gqa=False, aux=False):
    """Forward pass against a paged KV cache: :func:`forward` on the logical
    cache that :func:`gather_pages` reads out of the page pools."""
    k = gather_pages(k_pages, page_table, page_size, pages_per_seq)
    v = gather_pages(v_pages, page_table, page_size, pages_per_seq)
    return forward(q, k, v, scale, mask, score, kv_len=kv_len, enable_gqa=enable_gqa, aux=aux)


# ---------------------------------------------------------------------------
# BlockMask
# ---------------------------------------------------------------------------

def block_mask(mask, B, H, L, S, BM, BN, kv_len=None):
    """Brute-force BlockMask: classify every (m, n) tile as empty / full / partial.

    "flexattention-score-mod-block-mask", "mask_mod defines legal
    connections": an all-invisible tile is skipped, an all-visible tile is
    full (no element mask, score_mod still runs), anything else is partial.
    Guide section 3.1: a block is sparse only when *all* its elements are
    masked.  Guide section 4.1: the dense mask is evaluated, reduced per
    block, and full blocks are stored separately from partial ones.

    Returns int32 arrays kv_num_blocks (B,H,Mb), kv_indices (B,H,Mb,Nb) of the
    partial tiles, full_kv_num_blocks (B,H,Mb), full_kv_indices (B,H,Mb,Nb),
    indices ascending, unused slots 0.  Tiles at a ragged edge are classified
    over their in-range cells only.  Row h of the arrays is classified for
    query head h, so a head-dependent rule (head_below) gets per-head lists
    when H = Hq.
    """
    Mb, Nb = -(-L // BM), -(-S // BN)
    kv_num = np.zeros((B, H, Mb), np.int32)
    kv_idx = np.zeros((B, H, Mb, Nb), np.int32)
    full_num = np.zeros((B, H, Mb), np.int32)
    full_idx = np.zeros((B, H, Mb, Nb), np.int32)
    kv = np.arange(S, dtype=np.int64)
    for b in range(B):
        S_b = S if kv_len is None else int(np.asarray(kv_len)[b])
        qp_all = query_positions(L, S_b)
        for h in range(H):
            for mt in range(Mb):
                r0, r1 = mt * BM, min(L, (mt + 1) * BM)
                mk = dict(mask)
                if mask["kind"] == "dense":
                    mk["rows"] = np.arange(r0, r1)
                vis = visible(mk, b, h, qp_all[r0:r1], kv, S_b)
                nf = npart = 0
                for nt in range(Nb):
                    c0, c1 = nt * BN, min(S, (nt + 1) * BN)
                    cell = vis[:, c0:c1]
                    if cell.all():
                        full_idx[b, h, mt, nf] = nt
                        nf += 1
                    elif cell.any():
                        kv_idx[b, h, mt, npart] = nt
                        npart += 1
                kv_num[b, h, mt] = npart
                full_num[b, h, mt] = nf
    return dict(kv_num_blocks=kv_num, kv_indices=kv_idx,
                full_kv_num_blocks=full_num, full_kv_indices=full_idx, Mb=Mb, Nb=Nb)


def block_map(bm, b=0, h=0):
    """Dense tile map from the ordered lists: 'F' full, 'P' partial, '0' empty.

    Guide section 3.2: the dense form is rebuilt by walking each row's first
    num_blocks indices.
    """
    Mb, Nb = bm["Mb"], bm["Nb"]
    grid = [["0"] * Nb for _ in range(Mb)]
    for mt in range(Mb):
        for i in range(int(bm["kv_num_blocks"][b, h, mt])):
            grid[mt][int(bm["kv_indices"][b, h, mt, i])] = "P"
        for i in range(int(bm["full_kv_num_blocks"][b, h, mt])):
            grid[mt][int(bm["full_kv_indices"][b, h, mt, i])] = "F"
    return grid


def sparsity(bm, b=0, h=0):
    """Percentage of tiles that are skipped (guide section 3.3, sparsity())."""
    grid = block_map(bm, b, h)
    cells = [c for row in grid for c in row]
    return 100.0 * sum(c == "0" for c in cells) / len(cells)


# ---------------------------------------------------------------------------
# Split-KV partials and their combination
# ---------------------------------------------------------------------------

def split_partials(q_rows, k, v, scale, mask, score, b, h, qp, S_b, Hq, bounds):
    """Per-split (o_s, lse_s) over key ranges [bounds[i], bounds[i+1]).

    Each split is the same definition restricted to its key range: keys
    outside it are treated as invisible.
    """
    parts = []
    S = k.shape[0]
    kv = np.arange(S, dtype=np.int64)
    base = visible(mask, b, h, qp, kv, S_b)
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        sub = dict(kind="dense", matrix=base & ((kv >= lo) & (kv < hi))[None, :])
        o, ls = attention_rows(q_rows, k, v, scale, sub, score, b, h, qp, S_b, Hq)
        parts.append((o, ls))
    return parts


def combine(parts):
    """Merge split results: lse = ln sum_s e^{lse_s}; o = sum_s e^{lse_s - lse} o_s.

    Follows from the lse definition (guide section 2): the softmax over the
    union of disjoint key sets is the lse-weighted mixture of the per-set
    softmaxes.  All-empty rows stay (0, -inf).
    """
    lses = np.stack([p[1] for p in parts])          # (n_split, rows)
    outs = np.stack([p[0] for p in parts])          # (n_split, rows, Ev)
    m = lses.max(axis=0)
    out = np.zeros(outs.shape[1:])
    lse = np.full(lses.shape[1], NEG_INF)
    live = m > NEG_INF
    w = np.exp(lses[:, live] - m[live])
    tot = w.sum(axis=0)
    out[live] = np.einsum("sr,sre->re", w, outs[:, live]) / tot[:, None]
    lse[live] = m[live] + np.log(tot)
    return out, lse
