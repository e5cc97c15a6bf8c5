"""Pure-Python scalar restatement of the forward definition, for tiny shapes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  It checks the numpy
oracle against a second, independently written evaluation of the same
definition: triple loops over (query, key, feature) with ``math`` only, no
numpy, no vectorised masks.  Intended for shapes up to about 8 x 8 x 4.

Definition followed: "flexattention-score-mod-block-mask" (charlestar.github.io),
section "What one connection goes through" -- score, then the score rule g,
then the visibility rule (invisible -> -inf), then the softmax-weighted sum of
values; rules as in section "score_mod changes the score" (cap, then distance
bias) and "Attention expressions" (docs.tensorcad.dev), "Examples".
"""

from __future__ import annotations

import math


def _rule(params, b, h, q, kv):
    """A composed rule's verdict for one (query, key) pair, in-range keys only."""
    kind = params["kind"]
    if kind == "and":
        return all(_rule(m, b, h, q, kv) for m in params["masks"])
    if kind == "or":
        return any(_rule(m, b, h, q, kv) for m in params["masks"])
    if kind == "not":
        return not _rule(params["mask"], b, h, q, kv)
    if kind == "distance_below":
        return q - kv < params["value"]
    if kind == "key_below":
        return kv < params["value"]
    if kind == "same_chunk":
        return math.floor(q / params["value"]) == math.floor(kv / params["value"])
    if kind == "same_document":
        doc = params["doc_id"]
        row = doc[b] if isinstance(doc[0], (list, tuple)) else doc
        return 0 <= q < len(row) and row[q] == row[kv]
    if kind == "stride":
        return (q - kv) % params["value"] == 0
    if kind == "head_below":
        return h < params["value"]
    return _visible(kind, params, b, q, kv, 1 << 62)


def _visible(kind, params, b, q, kv, S_b, h=0):
    if kv >= S_b:
        return False
    if kind in ("and", "or", "not", "distance_below", "key_below", "same_chunk", "same_document", "stride",
                "head_below"):
        return _rule(params, b, h, q, kv)
    if kind == "none":
        return True
    if kind == "causal":
        return kv <= q
    if kind == "sliding_window":
        return kv <= q and (q - kv < params["window"] or kv < params.get("n_sink", 0))
    if kind == "document":
        doc = params["doc_id"]
        row = doc[b] if isinstance(doc[0], (list, tuple)) else doc
        return 0 <= q and kv <= q and row[q] == row[kv]
    if kind == "prefix_lm":
        return kv <= q or kv < params["prefix"]
    if kind == "chunked":
        C = params["chunk"]
        return kv <= q and math.floor(q / C) == math.floor(kv / C)
    raise ValueError(kind)


def _in_doc_position(row, t):
    start = t
    while start > 0 and row[start - 1] == row[t]:
        start -= 1
    return t - start


def _g(kind, params, s, b, h, q, kv, Hq):
    if kind == "none":
        return s
    if kind == "softcap":
        c = params["cap"]
        return c * math.tanh(s / c)
    H = params.get("slope_heads") or Hq
    slope = math.pow(2.0, -8.0 * (h + 1) / H)
    if kind == "alibi":
        return s - slope * (q - kv)
    if kind == "cap_then_bias":
        c = params["cap"]
        if params.get("pos", "global") == "in_doc":
            doc = params["doc_id"]
            row = doc[b] if isinstance(doc[0], (list, tuple)) else doc
            pq, pk = _in_doc_position(row, q), _in_doc_position(row, kv)
        else:
            pq, pk = q, kv
        return c * math.tanh(s / c) + slope * (pk - pq)
    raise ValueError(kind)


def forward_scalar(q, k, v, scale, mask, score, kv_len=None, with_max=False):
    """q[B][Hq][L][E], k[B][Hkv][S][E], v[B][Hkv][S][Ev] as nested lists of floats.

    Returns (out[B][Hq][L][Ev], lse[B][Hq][L]); a row with no visible key gives
    zeros and -inf.  With ``with_max`` a third nested list holds each row's
    largest visible transformed score (-inf for a row with none).
    """
    B, Hq, L = len(q), len(q[0]), len(q[0][0])
    Hkv, S = len(k[0]), len(k[0][0])
    G = Hq // Hkv
    out, lse, top = [], [], []
    for b in range(B):
        S_b = S if kv_len is None else int(kv_len[b])
        ob, lb, tb = [], [], []
        for h in range(Hq):
            hk = h // G
            oh, lh, th = [], [], []
            for i in range(L):
                qpos = i + (S_b - L)
                scores = []
                for j in range(S):
                    dot = 0.0
                    for e in range(len(q[b][h][i])):
                        dot += q[b][h][i][e] * k[b][hk][j][e]
                    g = _g(score["kind"], score, scale * dot, b, h, qpos, j, Hq)
                    scores.append(g if _visible(mask["kind"], mask, b, qpos, j, S_b, h) else -math.inf)
                m = -math.inf
                for x in scores:
                    if x > m:
                        m = x
                th.append(m)
                Ev = len(v[b][hk][0])
                if m == -math.inf:
                    oh.append([0.0] * Ev)
                    lh.append(-math.inf)
                    continue
                w = [math.exp(x - m) for x in scores]
                tot = sum(w)
                oh.append([sum(w[j] * v[b][hk][j][d] for j in range(S)) / tot for d in range(Ev)])
                lh.append(m + math.log(tot))
            ob.append(oh)
            lb.append(lh)
            tb.append(th)
        out.append(ob)
        lse.append(lb)
        top.append(tb)
    return (out, lse, top) if with_max else (out, lse)


def tile_classes_scalar(mask, L, S, BM, BN, b=0, kv_len=None, h=0):
    """Tile classes 'F' / 'P' / '0' by visiting every in-range cell of every tile."""
    S_b = S if kv_len is None else int(kv_len[b])
    grid = []
    for m0 in range(0, L, BM):
        row = []
        for n0 in range(0, S, BN):
            seen_vis = seen_hidden = False
            for i in range(m0, min(L, m0 + BM)):
                for j in range(n0, min(S, n0 + BN)):
                    if _visible(mask["kind"], mask, b, i + (S_b - L), j, S_b, h):
                        seen_vis = True
                    else:
                        seen_hidden = True
            row.append("F" if seen_vis and not seen_hidden else ("P" if seen_vis else "0"))
        grid.append(row)
    return grid
