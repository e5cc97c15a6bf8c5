"""Checks that pin the fp64 oracle to facts outside itself.

Each check takes the oracle module and raises AssertionError when the oracle
disagrees with: a worked example printed on the pages (fixtures under
tests/golden/, each citing its page and section), a closed form, an invariant
of the definition, a library routine (torch's SDPA on the CPU in fp64), or
brute force (the scalar restatement in oracle/scalar_reference.py).

The same checks are run against deliberately broken copies of the oracle in
test_oracle_mutations.py, to show that each plausible mistake is caught.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

from _golden import floats, ints, load

RNG = np.random.default_rng(12345)


def _scalar():
    import oracle.scalar_reference as sr
    return sr


# ---------------------------------------------------------------------------
# Worked examples printed on the pages
# ---------------------------------------------------------------------------

def check_m1_six_token_tiles(o):
    g = load("m1_causal_len6_tile2.txt")
    n, t = int(g["length"]), int(g["tile"])
    bm = o.block_mask({"kind": "causal"}, 1, 1, n, n, t, t)
    grid = ["".join(r) for r in o.block_map(bm)]
    assert grid == g["block_map"].split(), grid
    flat = "".join(grid)
    assert flat.count("F") == int(g["count_F"]) and flat.count("P") == int(g["count_P"])
    assert flat.count("0") == int(g["count_0"])
    vis = o.visible({"kind": "causal"}, 0, 0, o.query_positions(n, n), np.arange(n), n)
    assert vis.size == int(g["pairs"]) and int(vis.sum()) == int(g["visible_pairs"])
    visited = (flat.count("F") + flat.count("P")) * t * t
    assert visited == int(g["visited_cells"])
    hidden = 0
    for mt, row in enumerate(grid):
        for nt, c in enumerate(row):
            if c != "0":
                hidden += int((~vis[mt * t:(mt + 1) * t, nt * t:(nt + 1) * t]).sum())
    assert hidden == int(g["masked_cells_in_visited_tiles"])


def check_m6_packed_documents(o):
    g = load("m6_packed_docs_len16_block4.txt")
    n, blk = int(g["n"]), int(g["block"])
    lens = ints(g["doc_lengths"])
    doc = np.repeat(np.arange(len(lens)), lens)
    for kind, key in (({"kind": "causal"}, "causal"), ({"kind": "document", "doc_id": doc}, "doc_causal")):
        bm = o.block_mask(kind, 1, 1, n, n, blk, blk)
        dense = ["".join("0" if c == "0" else "1" for c in row) for row in o.block_map(bm)]
        assert dense == g[f"{key}_map"].split(), (key, dense)
        assert abs(o.sparsity(bm) - float(g[f"{key}_sparsity"])) < 5e-3
    # every visited tile of the document mask straddles a boundary or the diagonal
    bm = o.block_mask({"kind": "document", "doc_id": doc}, 1, 1, n, n, blk, blk)
    assert int(bm["full_kv_num_blocks"].sum()) == 0 and int(bm["kv_num_blocks"].sum()) == 7


def check_m2_softcap_after_mask(o):
    g = load("m2_softcap_trap.txt")
    cap = float(g["cap"])
    # two keys with raw score 0 (q = 0); the first query of a 2x2 causal
    # attention sees key 0 only, as in the page's allow = [True, False]
    q = np.zeros((1, 1, 2, 4))
    k = RNG.standard_normal((1, 1, 2, 4))
    v = np.eye(2).reshape(1, 1, 2, 2)
    out, _ = o.forward(q, k, v, 0.5, {"kind": "causal"}, {"kind": "softcap", "cap": cap})
    assert np.allclose(out[0, 0, 0], floats(g["correct"]), atol=0, rtol=0), out[0, 0, 0]
    # the wrong order, written out here, reproduces the page's printed numbers
    wrong = [cap * math.tanh(s / cap) for s in (0.0, -math.inf)]
    mx = max(wrong)
    w = [math.exp(x - mx) for x in wrong]
    w = [x / sum(w) for x in w]
    assert [round(x, 6) for x in w] == floats(g["incorrect_rounded6"])


def check_m3_decode_offset(o):
    g = load("m3_decode_offset.txt")
    cap, valid, W = int(g["capacity"]), int(g["valid_length"]), int(g["window"])
    qp = o.query_positions(1, valid)
    assert int(qp[0]) == int(g["q_idx"]) + int(g["q_offset"])
    vis = o.visible({"kind": "sliding_window", "window": W, "n_sink": 0}, 0, 0, qp, np.arange(cap), valid)
    assert np.flatnonzero(vis[0]).tolist() == ints(g["visible"])


def check_m4_bottom_right(o):
    g = load("m4_bottom_right.txt")
    L, S, E = int(g["L"]), int(g["S"]), int(g["E"])
    q = np.ones((1, 1, L, E))
    k = np.ones((1, 1, S, E))
    v = np.eye(S).reshape(1, 1, S, S)
    out, lse = o.forward(q, k, v, None, {"kind": "causal"}, None)
    assert np.allclose(out[0, 0, 0], floats(g["bottom_right"]), atol=1e-15)
    assert not np.allclose(out[0, 0, 0], floats(g["top_left"]))
    assert abs(lse[0, 0, 0] - (E / math.sqrt(E) + math.log(S))) < 1e-12


def check_m5_left_padding(o):
    g = load("m5_left_padding.txt")
    causal = np.tril(np.ones((3, 3), bool))
    pad = np.array([True, False, False])
    vis = causal & ~pad[None, :]
    q = np.zeros((1, 1, 3, 2))
    k = RNG.standard_normal((1, 1, 3, 2))
    v = np.eye(3).reshape(1, 1, 3, 3)
    out, lse = o.forward(q, k, v, 1.0, {"kind": "dense", "matrix": vis}, None)
    assert np.allclose(out[0, 0, 1], floats(g["row1"]), atol=1e-15)
    assert np.allclose(out[0, 0, 2], floats(g["row2"]), atol=1e-15)
    # the library's convention for the fully masked row 0: zeros and -inf
    assert np.all(out[0, 0, 0] == 0.0) and lse[0, 0, 0] == -np.inf
    assert not np.isnan(out).any()


# ---------------------------------------------------------------------------
# Closed forms
# ---------------------------------------------------------------------------

def check_causal_block_fraction(o):
    """(T+1)/2T of the tiles are computed ("Causal Mask" section 7)."""
    for T in (1, 2, 3, 4, 16, 33):
        bm = o.block_mask({"kind": "causal"}, 1, 1, 4 * T, 4 * T, 4, 4)
        full = int(bm["full_kv_num_blocks"].sum())
        part = int(bm["kv_num_blocks"].sum())
        assert Fraction(full + part, T * T) == Fraction(T + 1, 2 * T)
        assert part == T and full == T * (T - 1) // 2


def check_window_count(o):
    """Visible pairs of a causal window W: exact sum vs the page's W - W^2/2T.

    "Attention expressions" (docs.tensorcad.dev), "What the engine does with
    them": a causal window keeps W - W^2/2T keys per query on average once the
    sequence outgrows it.  The exact mean is W - W^2/2T + W/2T; the page's
    form is its continuum limit.
    """
    for T, W, n_sink in ((64, 16, 0), (257, 32, 0), (300, 40, 4), (129, 128, 3)):
        vis = o.visible({"kind": "sliding_window", "window": W, "n_sink": n_sink}, 0, 0,
                        o.query_positions(T, T), np.arange(T), T)
        total = int(vis.sum())
        exact = W * (W + 1) // 2 + (T - W) * W + sum(min(n_sink, q - W + 1) for q in range(W, T))
        assert total == exact, (T, W, n_sink, total, exact)
        if n_sink == 0:
            mean = Fraction(total, T)
            assert mean == Fraction(W) - Fraction(W * W, 2 * T) + Fraction(W, 2 * T)


def check_single_visible_key(o):
    """A row with one visible key returns that key's value; lse = its score."""
    B, H, L, E = 1, 3, 9, 5
    q = RNG.standard_normal((B, H, L, E))
    k = RNG.standard_normal((B, H, L, E))
    v = RNG.standard_normal((B, H, L, E))
    score = {"kind": "cap_then_bias", "cap": 7.0, "slope_heads": 3, "pos": "global"}
    out, lse = o.forward(q, k, v, 0.3, {"kind": "causal"}, score)
    for h in range(H):
        assert np.array_equal(out[0, h, 0], v[0, h, 0])
        s = 0.3 * float(q[0, h, 0] @ k[0, h, 0])
        assert abs(lse[0, h, 0] - 7.0 * math.tanh(s / 7.0)) < 1e-12
    # first token of every packed document sees only itself
    doc = np.array([0, 0, 1, 1, 1, 2, 2, 2, 2])
    out, lse = o.forward(q, k, v, 0.3, {"kind": "document", "doc_id": doc}, None)
    for start in (0, 2, 5):
        assert np.array_equal(out[0, 1, start], v[0, 1, start])


def check_equal_scores(o):
    """q = 0: every visible key weighs the same; o = mean, lse = ln(count)."""
    B, H, L, S, E = 2, 2, 7, 11, 3
    q = np.zeros((B, H, L, E))
    k = RNG.standard_normal((B, H, S, E))
    v = RNG.standard_normal((B, H, S, 4))
    kv_len = np.array([11, 8])
    for mask in ({"kind": "causal"}, {"kind": "prefix_lm", "prefix": 3},
                 {"kind": "sliding_window", "window": 3, "n_sink": 1}, {"kind": "chunked", "chunk": 4}):
        out, lse = o.forward(q, k, v, 1.0, mask, None, kv_len=kv_len)
        for b in range(B):
            S_b = int(kv_len[b])
            vis = o.visible(mask, b, 0, o.query_positions(L, S_b), np.arange(S), S_b)
            for i in range(L):
                n = int(vis[i].sum())
                if n == 0:
                    assert lse[b, 0, i] == -np.inf and np.all(out[b, 0, i] == 0)
                    continue
                assert np.allclose(out[b, 0, i], v[b, 0, vis[i]].mean(axis=0), atol=1e-13)
                assert abs(lse[b, 0, i] - math.log(n)) < 1e-13


def check_alibi_geometric(o):
    """Equal raw scores under ALiBi: causal weights form a geometric sequence.

    With g = -slope_h (q - kv), softmax over keys 0..i gives weights
    proportional to e^{-slope_h (i - j)}: consecutive keys differ by the
    factor e^{slope_h}, the nearest key weighs most ("flexattention-score-mod-
    block-mask": the distance term biases far history negatively).  For 8
    heads the slopes are 1/2, 1/4, ..., 1/256, the textbook ALiBi set.
    """
    H, L = 8, 6
    q = np.zeros((1, H, L, 2))
    k = RNG.standard_normal((1, H, L, 2))
    v = np.eye(L)[None, None].repeat(H, axis=1)
    out, _ = o.forward(q, k, v, 1.0, {"kind": "causal"}, {"kind": "alibi", "slope_heads": H})
    for h in range(H):
        w = out[0, h, L - 1]
        ratio = w[1:] / w[:-1]
        assert np.allclose(ratio, math.exp(2.0 ** -(h + 1)), rtol=1e-12), (h, ratio)


def check_softcap_limits(o):
    """c -> infinity: the soft-cap is the identity; a cap bounds scores in (-c, c)."""
    q = RNG.standard_normal((1, 2, 6, 4))
    k = RNG.standard_normal((1, 2, 6, 4))
    v = RNG.standard_normal((1, 2, 6, 4))
    a, la = o.forward(q, k, v, 2.0, {"kind": "causal"}, {"kind": "softcap", "cap": 1e9})
    b, lb = o.forward(q, k, v, 2.0, {"kind": "causal"}, None)
    assert np.allclose(a, b, atol=1e-12) and np.allclose(la, lb, atol=1e-12)
    _, lc = o.forward(q * 50, k, v, 2.0, {"kind": "none"}, {"kind": "softcap", "cap": 1.5})
    assert np.all(lc < 1.5 + math.log(6) + 1e-12)


def check_cap_then_bias_order(o):
    """cap-then-bias differs from bias-then-cap, and equals its two parts.

    "flexattention-score-mod-block-mask", "score_mod changes the score":
    c tanh(s/c) + a(p_j - p_i) is the rule; c tanh((s + a(p_j - p_i))/c) is
    another.  With c -> infinity both reduce to ALiBi, and with a single
    head of slope 2^-8 the bias part is tiny but nonzero.
    """
    q = RNG.standard_normal((1, 1, 5, 3)) * 3
    k = RNG.standard_normal((1, 1, 5, 3)) * 3
    v = RNG.standard_normal((1, 1, 5, 3))
    big = o.forward(q, k, v, 1.0, {"kind": "causal"}, {"kind": "cap_then_bias", "cap": 1e9, "slope_heads": 1})
    ali = o.forward(q, k, v, 1.0, {"kind": "causal"}, {"kind": "alibi", "slope_heads": 1})
    assert np.allclose(big[0], ali[0], atol=1e-9) and np.allclose(big[1], ali[1], atol=1e-9)
    # q = 0: g = slope (kv - q) exactly, whatever the cap
    z = np.zeros_like(q)
    _, l1 = o.forward(z, k, v, 1.0, {"kind": "none"}, {"kind": "cap_then_bias", "cap": 0.01, "slope_heads": 1})
    i = np.arange(5)[:, None]
    j = np.arange(5)[None, :]
    ref = np.log(np.exp(2.0 ** -8 * (j - i)).sum(axis=1))
    assert np.allclose(l1[0, 0], ref, atol=1e-13)


def check_convex_combination(o):
    """Each output is a convex combination of visible values; lse >= max score."""
    B, H, L, S, E = 1, 2, 13, 17, 4
    q = RNG.standard_normal((B, H, L, E))
    k = RNG.standard_normal((B, H, S, E))
    v = RNG.standard_normal((B, H, S, E))
    mask = {"kind": "sliding_window", "window": 5, "n_sink": 2}
    out, lse = o.forward(q, k, v, 0.5, mask, {"kind": "softcap", "cap": 2.0})
    vis = o.visible(mask, 0, 0, o.query_positions(L, S), np.arange(S), S)
    for h in range(H):
        s = 2.0 * np.tanh(0.5 * (q[0, h] @ k[0, h].T) / 2.0)
        for i in range(L):
            vv = v[0, h, vis[i]]
            assert np.all(out[0, h, i] >= vv.min(axis=0) - 1e-12)
            assert np.all(out[0, h, i] <= vv.max(axis=0) + 1e-12)
            assert lse[0, h, i] >= s[i, vis[i]].max() - 1e-12


# ---------------------------------------------------------------------------
# Library routine and brute force
# ---------------------------------------------------------------------------

def check_against_torch_sdpa(o):
    """No score rule + a boolean mask = torch's SDPA (CPU, fp64, explicit mask)."""
    import torch
    import torch.nn.functional as F
    B, H, L, S, E = 2, 3, 19, 23, 8
    q = RNG.standard_normal((B, H, L, E))
    k = RNG.standard_normal((B, H, S, E))
    v = RNG.standard_normal((B, H, S, 6))
    kv_len = np.array([23, 20])
    masks = ({"kind": "causal"}, {"kind": "sliding_window", "window": 6, "n_sink": 2},
             {"kind": "prefix_lm", "prefix": 5}, {"kind": "chunked", "chunk": 7},
             {"kind": "document", "doc_id": np.repeat(np.arange(4), [5, 9, 3, 6])}, {"kind": "none"})
    for mask in masks:
        out, lse = o.forward(q, k, v, 0.37, mask, None, kv_len=kv_len)
        for b in range(B):
            S_b = int(kv_len[b])
            vis = o.visible(mask, b, 0, o.query_positions(L, S_b), np.arange(S), S_b)
            live = vis.any(axis=1)
            ref = F.scaled_dot_product_attention(
                torch.from_numpy(q[b:b + 1, :, live]), torch.from_numpy(k[b:b + 1]),
                torch.from_numpy(v[b:b + 1]), attn_mask=torch.from_numpy(vis[live]), scale=0.37)
            assert np.allclose(out[b][:, live], ref[0].numpy(), atol=1e-12), mask["kind"]


def _tiny_case(seed, L, S, E, Ev, B=2, Hq=2, Hkv=1):
    r = np.random.default_rng(seed)
    return (r.standard_normal((B, Hq, L, E)), r.standard_normal((B, Hkv, S, E)),
            r.standard_normal((B, Hkv, S, Ev)))


TINY_MASKS = (
    {"kind": "none"}, {"kind": "causal"}, {"kind": "sliding_window", "window": 3, "n_sink": 1},
    {"kind": "sliding_window", "window": 2, "n_sink": 0}, {"kind": "prefix_lm", "prefix": 2},
    {"kind": "chunked", "chunk": 3}, {"kind": "document", "doc_id": [[0, 0, 0, 1, 1, 2, 2, 2], [0, 1, 1, 1, 1, 1, 2, 2]]},
)
TINY_SCORES = (
    {"kind": "none"}, {"kind": "softcap", "cap": 1.5}, {"kind": "alibi", "slope_heads": 2},
    {"kind": "cap_then_bias", "cap": 2.0, "slope_heads": 0, "pos": "global"},
    {"kind": "cap_then_bias", "cap": 2.5, "slope_heads": 4, "pos": "in_doc",
     "doc_id": [[0, 0, 0, 1, 1, 2, 2, 2], [0, 1, 1, 1, 1, 1, 2, 2]]},
)


def check_against_scalar_loops(o):
    """numpy oracle == pure-Python triple loops on tiny shapes, every mask and score kind."""
    sr = _scalar()
    seed = 0
    for mask in TINY_MASKS:
        for score in TINY_SCORES:
            for (L, S, kv_len) in ((8, 8, None), (3, 8, [8, 6]), (8, 8, [8, 5])):
                seed += 1
                q, k, v = _tiny_case(seed, L, S, 3, 2)
                out, lse = o.forward(q, k, v, 0.7, mask, score, kv_len=kv_len, enable_gqa=True)
                so, sl = sr.forward_scalar(q.tolist(), k.tolist(), v.tolist(), 0.7, mask, score, kv_len)
                so, sl = np.array(so), np.array(sl)
                assert np.allclose(out, so, atol=1e-12, rtol=0), (mask, score, L, S)
                fin = np.isfinite(sl)
                assert np.array_equal(fin, np.isfinite(lse)) and np.allclose(lse[fin], sl[fin], atol=1e-12)


def check_block_mask_against_scalar(o):
    """Oracle tile classes == a cell-by-cell scalar visit, ragged shapes included."""
    sr = _scalar()
    doc = [0] * 7 + [1] * 3 + [2] * 11 + [3] * 2
    cases = [({"kind": "causal"}, 23, 23, 4, 4, None), ({"kind": "causal"}, 9, 23, 4, 8, [23]),
             ({"kind": "sliding_window", "window": 5, "n_sink": 2}, 23, 23, 4, 3, None),
             ({"kind": "prefix_lm", "prefix": 6}, 23, 23, 8, 4, None),
             ({"kind": "chunked", "chunk": 6}, 23, 23, 4, 4, None),
             ({"kind": "document", "doc_id": doc}, 23, 23, 4, 4, None),
             ({"kind": "none"}, 5, 23, 2, 8, [17]), ({"kind": "causal"}, 23, 19, 8, 8, [11])]
    for mask, L, S, BM, BN, kv_len in cases:
        bm = o.block_mask(mask, 1, 1, L, S, BM, BN, kv_len=kv_len)
        ref = sr.tile_classes_scalar(mask, L, S, BM, BN, 0, kv_len)
        assert o.block_map(bm) == ref, (mask, L, S, BM, BN)
        # ordering and padding convention
        for mt in range(bm["Mb"]):
            for name, cnt in (("kv_indices", "kv_num_blocks"), ("full_kv_indices", "full_kv_num_blocks")):
                n = int(bm[cnt][0, 0, mt])
                idx = bm[name][0, 0, mt]
                assert list(idx[:n]) == sorted(idx[:n]) and np.all(idx[n:] == 0)


def check_split_combine(o):
    """Split-KV partials merged by lse weights equal the unsplit result."""
    L, S, E = 6, 40, 5
    q, k, v = _tiny_case(7, L, S, E, 3, B=1, Hq=1, Hkv=1)
    mask = {"kind": "causal"}
    score = {"kind": "softcap", "cap": 3.0}
    qp = o.query_positions(L, S)
    full_o, full_l = o.attention_rows(q[0, 0], k[0, 0], v[0, 0], 0.4, mask, score, 0, 0, qp, S, 1)
    for bounds in ([0, 40], [0, 13, 40], [0, 1, 2, 17, 36, 40], [0, 10, 20, 30, 40]):
        parts = o.split_partials(q[0, 0], k[0, 0], v[0, 0], 0.4, mask, score, 0, 0, qp, S, 1, bounds)
        co, cl = o.combine(parts)
        assert np.allclose(co, full_o, atol=1e-12) and np.allclose(cl, full_l, atol=1e-12)


def check_gqa_is_broadcast(o):
    """GQA equals explicitly repeating each KV head for its group of query heads."""
    q, k, v = _tiny_case(3, 5, 7, 4, 3, B=1, Hq=6, Hkv=2)
    a = o.forward(q, k, v, 0.5, {"kind": "causal"}, {"kind": "alibi"}, enable_gqa=True)
    b = o.forward(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), 0.5, {"kind": "causal"}, {"kind": "alibi"})
    assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-14)


def check_workload_tile_counts(o):
    """Tile counts of the causal 2048/128 and window+sink 16384/128 workloads.

    Causal with T tiles per side: T(T+1)/2 visited, T(T-1)/2 full, T partial.
    Window W=1024 with 4 sinks, tiles of 128: counted here tile by tile from
    the interval of keys each query row sees (not cell by cell).
    """
    bm = o.block_mask({"kind": "causal"}, 1, 1, 2048, 2048, 128, 128)
    assert int(bm["full_kv_num_blocks"].sum()) == 120 and int(bm["kv_num_blocks"].sum()) == 16
    T, W, ns, t = 16384, 1024, 4, 128
    nb = T // t
    full = part = 0
    for m in range(nb):
        rows = np.arange(m * t, (m + 1) * t)
        lo = np.maximum(rows - W + 1, 0)
        for n in range(nb):
            c0, c1 = n * t, (n + 1) * t - 1
            win = np.clip(np.minimum(rows, c1) - np.maximum(lo, c0) + 1, 0, None)
            sink_hi = np.minimum(ns - 1, np.minimum(rows, c1))
            sink = np.clip(np.minimum(sink_hi, lo - 1) - c0 + 1, 0, None)
            cnt = win + sink
            if np.all(cnt == t):
                full += 1
            elif np.any(cnt > 0):
                part += 1
    assert (full, part) == (868, 367), (full, part)
    bm = o.block_mask({"kind": "sliding_window", "window": W, "n_sink": ns}, 1, 1, T, T, t, t)
    assert int(bm["full_kv_num_blocks"].sum()) == full and int(bm["kv_num_blocks"].sum()) == part


def check_sampled_rows_match_forward(o):
    """Rows from forward_sampled equal the same rows of forward.

    forward_sampled is the checker of every full-size comparison, so it is held
    to forward on a case where a slip in its own bookkeeping would show: GQA
    with three query heads per KV head, a different valid KV length per
    sequence (so the logical query positions differ per batch), a document
    mask, the cap-then-in-document-bias score rule (which reads the query
    head), and sampled rows at every tile edge of a 4-row tiling plus rows
    that see no key.
    """
    B, Hq, Hkv, L, S, E = 3, 6, 2, 12, 16, 4
    r = np.random.default_rng(77)
    q = r.standard_normal((B, Hq, L, E))
    k = r.standard_normal((B, Hkv, S, E))
    v = r.standard_normal((B, Hkv, S, 3))
    kv_len = np.array([16, 13, 9])
    doc = np.array([[0] * 5 + [1] * 4 + [2] * 7, [0] * 3 + [1] * 8 + [2] * 5, [0] * 9 + [1] * 7])
    mask = {"kind": "document", "doc_id": doc}
    score = {"kind": "cap_then_bias", "cap": 3.0, "slope_heads": 0, "pos": "in_doc", "doc_id": doc}
    out, lse = o.forward(q, k, v, 0.45, mask, score, kv_len=kv_len, enable_gqa=True)
    rows = sorted({0, 1, 3, 4, 7, 8, 11} | set(range(0, L, 5)))
    samples = [(b, h, i) for b in range(B) for h in range(Hq) for i in rows]
    so, sl = o.forward_sampled(q, k, v, samples, 0.45, mask, score, kv_len=kv_len, enable_gqa=True)
    ref_o = np.stack([out[b, h, i] for b, h, i in samples])
    ref_l = np.array([lse[b, h, i] for b, h, i in samples])
    assert np.array_equal(np.isfinite(sl), np.isfinite(ref_l)) and (~np.isfinite(ref_l)).any()
    fin = np.isfinite(ref_l)
    assert np.allclose(so, ref_o, atol=1e-13, rtol=0) and np.allclose(sl[fin], ref_l[fin], atol=1e-13, rtol=0)


def check_max_scores(o):
    """max_scores: the largest visible transformed score of each row.

    Pinned by closed forms (a row with one visible key: max = lse = that
    key's g; q = 0 under ALiBi: max = 0, reached at the query's own key; a
    row with no visible key: -inf), by the bound max <= lse <= max + ln n
    with n the row's visible-key count, by a case whose largest raw score
    sits on a hidden key, and by the pure-Python loops on tiny shapes.
    """
    sr = _scalar()
    B, H, L, E = 1, 3, 9, 5
    r = np.random.default_rng(31)
    q = r.standard_normal((B, H, L, E))
    k = r.standard_normal((B, H, L, E))
    v = r.standard_normal((B, H, L, E))
    score = {"kind": "cap_then_bias", "cap": 7.0, "slope_heads": 3, "pos": "global"}
    out, lse, mx = o.forward(q, k, v, 0.3, {"kind": "causal"}, score, aux=True)
    for h in range(H):
        s = 0.3 * float(q[0, h, 0] @ k[0, h, 0])
        assert abs(mx[0, h, 0] - 7.0 * math.tanh(s / 7.0)) < 1e-12 and mx[0, h, 0] == lse[0, h, 0]
    # q = 0 under ALiBi: g = -slope (q - kv) <= 0, equal to 0 at kv = q
    z = np.zeros_like(q)
    _, _, mz = o.forward(z, k, v, 1.0, {"kind": "causal"}, {"kind": "alibi"}, aux=True)
    assert np.all(mz == 0.0)
    # the largest raw score on a hidden key must not leak into the max
    k2 = k.copy()
    k2[0, :, L - 1] = 50.0 * q[0, :, 0]            # key L-1 scores highest for query 0
    _, _, m2 = o.forward(q, k2, v, 1.0, {"kind": "causal"}, None, aux=True)
    assert np.allclose(m2[0, :, 0], np.einsum("he,he->h", q[0, :, 0], k2[0, :, 0]), atol=1e-12)
    # no visible key: -inf; otherwise max <= lse <= max + ln n
    kv_len = np.array([4])
    o2, l2, m3 = o.forward(q, k, v, 0.5, {"kind": "causal"}, {"kind": "softcap", "cap": 2.0}, kv_len=kv_len,
                           aux=True)
    vis = o.visible({"kind": "causal"}, 0, 0, o.query_positions(L, 4), np.arange(L), 4)
    n = vis.sum(axis=1)
    assert np.all(m3[0, :, n == 0] == -np.inf) and np.all(l2[0, :, n == 0] == -np.inf)
    live = n > 0
    assert np.all(m3[0][:, live] <= l2[0][:, live] + 1e-12)
    assert np.all(l2[0][:, live] <= m3[0][:, live] + np.log(n[live]) + 1e-12)
    # brute force on tiny shapes, every mask and score kind
    seed = 500
    for mask in TINY_MASKS:
        for sc in TINY_SCORES:
            seed += 1
            q, k, v = _tiny_case(seed, 3, 8, 3, 2)
            _, _, m = o.forward(q, k, v, 0.7, mask, sc, kv_len=[8, 5], enable_gqa=True, aux=True)
            _, _, sm = sr.forward_scalar(q.tolist(), k.tolist(), v.tolist(), 0.7, mask, sc, [8, 5], with_max=True)
            sm = np.array(sm)
            fin = np.isfinite(sm)
            assert np.array_equal(fin, np.isfinite(m)) and np.allclose(m[fin], sm[fin], atol=1e-12, rtol=0)
    # the sampled-row checker returns the same maxima
    samples = [(0, 1, 0), (1, 0, 2)]
    _, _, ms = o.forward_sampled(q, k, v, samples, 0.7, TINY_MASKS[1], TINY_SCORES[1], kv_len=[8, 5],
                                 enable_gqa=True, aux=True)
    _, _, mf = o.forward(q, k, v, 0.7, TINY_MASKS[1], TINY_SCORES[1], kv_len=[8, 5], enable_gqa=True, aux=True)
    assert np.array_equal(ms, np.array([mf[b, h, i] for b, h, i in samples]))


def check_forward_unit_matches_forward(o):
    """forward_unit on one (b, h) slice gives forward's rows of that unit.

    The full-size checks call forward_unit with slices regenerated per unit,
    so its arguments (batch b for the document row, query head h and Hq for
    the slope, the valid length S_b for positions) are held to forward on GQA
    with per-sequence valid lengths, a per-batch document mask and the
    in-document cap-then-bias rule.
    """
    B, Hq, Hkv, L, S, E = 2, 4, 2, 10, 14, 3
    r = np.random.default_rng(91)
    q = r.standard_normal((B, Hq, L, E))
    k = r.standard_normal((B, Hkv, S, E))
    v = r.standard_normal((B, Hkv, S, 2))
    kv_len = np.array([14, 11])
    doc = np.array([[0] * 6 + [1] * 8, [0] * 2 + [1] * 9 + [2] * 3])
    mask = {"kind": "document", "doc_id": doc}
    score = {"kind": "cap_then_bias", "cap": 2.5, "slope_heads": 0, "pos": "in_doc", "doc_id": doc}
    out, lse, mx = o.forward(q, k, v, 0.6, mask, score, kv_len=kv_len, enable_gqa=True, aux=True)
    for b in range(B):
        for h in range(Hq):
            uo, ul, um = o.forward_unit(q[b, h], k[b, h // 2], v[b, h // 2], b, h, Hq, int(kv_len[b]), 0.6, mask,
                                        score, row_group=3)
            assert np.allclose(uo, out[b, h], atol=1e-14, rtol=0)
            assert np.array_equal(np.isfinite(ul), np.isfinite(lse[b, h]))
            fin = np.isfinite(ul)
            assert np.allclose(ul[fin], lse[b, h][fin], atol=1e-14)
            assert np.array_equal(np.isfinite(um), fin) and np.allclose(um[fin], mx[b, h][fin], atol=1e-14)


def check_composed_masks(o):
    """and / or / not over predicates ("PyTorch Flex Attention complete guide"
    section 4.3; "Attention expressions", Examples).

    Pinned by identities with the fixed rules -- causal AND (distance < W OR
    key < n) is the sliding window with sinks, causal OR key < P is prefix-LM,
    causal AND same chunk is chunked attention, causal AND same document is
    the document rule (the guide's and_masks(causal_mask, sliding_window_mask)
    example) -- by De Morgan, by closed-form counts of the pages' every-fourth-
    key and half-heads-global examples, by the block-granularity remark (a
    sliver of every block leaves no full block), and by the scalar loops.
    """
    sr = _scalar()
    T, W, ns, P, C = 70, 9, 3, 11, 16
    qp, kv = o.query_positions(T, T), np.arange(T)
    causal = {"kind": "causal"}
    doc = np.repeat(np.arange(5), [13, 20, 7, 22, 8])
    ident = [
        ({"kind": "and", "masks": [causal, {"kind": "or", "masks": [{"kind": "distance_below", "value": W},
                                                                    {"kind": "key_below", "value": ns}]}]},
         {"kind": "sliding_window", "window": W, "n_sink": ns}),
        ({"kind": "or", "masks": [causal, {"kind": "key_below", "value": P}]}, {"kind": "prefix_lm", "prefix": P}),
        ({"kind": "and", "masks": [causal, {"kind": "same_chunk", "value": C}]}, {"kind": "chunked", "chunk": C}),
        ({"kind": "and", "masks": [causal, {"kind": "same_document", "doc_id": doc}]},
         {"kind": "document", "doc_id": doc}),
    ]
    for comp, fixed in ident:
        for S_b in (T, 51):
            q2 = o.query_positions(T, S_b)
            assert np.array_equal(o.visible(comp, 0, 0, q2, kv, S_b), o.visible(fixed, 0, 0, q2, kv, S_b)), fixed
    # chunks are floor-divided: a row at a negative logical position (more
    # queries than valid keys) shares no chunk with any key, causal bound or not
    qneg = o.query_positions(T, 40)
    same = o.visible({"kind": "same_chunk", "value": C}, 0, 0, qneg, kv, 40)
    assert not same[qneg < 0].any() and same[qneg >= 0].any(axis=1).all()
    # De Morgan over in-range keys
    a, bb = {"kind": "stride", "value": 3}, {"kind": "distance_below", "value": 5}
    lhs = o.visible({"kind": "not", "mask": {"kind": "and", "masks": [a, bb]}}, 0, 0, qp, kv, 60)
    rhs = o.visible({"kind": "or", "masks": [{"kind": "not", "mask": a}, {"kind": "not", "mask": bb}]}, 0, 0, qp, kv,
                    60)
    assert np.array_equal(lhs, rhs) and not lhs[:, 60:].any()
    # every fourth key, causal: query q sees floor(q / 4) + 1 keys
    sliver = {"kind": "and", "masks": [causal, {"kind": "stride", "value": 4}]}
    vis = o.visible(sliver, 0, 0, qp, kv, T)
    assert vis.sum(axis=1).tolist() == [q // 4 + 1 for q in range(T)]
    assert vis[T - 1].nonzero()[0].tolist() == list(range((T - 1) % 4, T, 4))
    # half the heads global, half local (window W), causal on, H = 6
    H = 6
    half = {"kind": "and", "masks": [causal, {"kind": "or", "masks": [{"kind": "head_below", "value": H // 2},
                                                                      {"kind": "distance_below", "value": W}]}]}
    for h in range(H):
        n = int(o.visible(half, 0, h, qp, kv, T).sum())
        assert n == (T * (T + 1) // 2 if h < H // 2 else W * (W + 1) // 2 + (T - W) * W), (h, n)
    # block granularity: a sliver of every block leaves no full block
    t = 8
    bm = o.block_mask(sliver, 1, 1, 8 * t, 8 * t, t, t)
    assert int(bm["full_kv_num_blocks"].sum()) == 0 and int(bm["kv_num_blocks"].sum()) == 8 * 9 // 2
    bmh = o.block_mask(half, 1, H, 8 * t, 8 * t, t, t)
    assert int(bmh["full_kv_num_blocks"][0, 0].sum()) == 8 * 7 // 2  # global heads: causal tiles
    assert int(bmh["full_kv_num_blocks"][0, 0].sum() + bmh["kv_num_blocks"][0, 0].sum()) == 36
    assert int(bmh["full_kv_num_blocks"][0, H - 1].sum() + bmh["kv_num_blocks"][0, H - 1].sum()) == 8 + 7
    # brute force: oracle forward and tile classes against the scalar loops
    rules = [sliver, half, ident[0][0],
             {"kind": "not", "mask": {"kind": "or", "masks": [{"kind": "key_below", "value": 2},
                                                              {"kind": "stride", "value": 3}]}},
             {"kind": "and", "masks": [{"kind": "same_document", "doc_id": [[0, 0, 1, 1, 1, 2, 2, 2],
                                                                            [0, 1, 1, 1, 2, 2, 2, 2]]},
                                       {"kind": "same_chunk", "value": 3}]}]
    seed = 900
    for mask in rules:
        for (L, S, kv_len) in ((8, 8, None), (3, 8, [8, 6])):
            seed += 1
            q, k, v = _tiny_case(seed, L, S, 3, 2, Hq=4, Hkv=2)
            out, lse = o.forward(q, k, v, 0.7, mask, TINY_SCORES[3], kv_len=kv_len, enable_gqa=True)
            so, sl = sr.forward_scalar(q.tolist(), k.tolist(), v.tolist(), 0.7, mask, TINY_SCORES[3], kv_len)
            so, sl = np.array(so), np.array(sl)
            assert np.allclose(out, so, atol=1e-12, rtol=0), mask
            fin = np.isfinite(sl)
            assert np.array_equal(fin, np.isfinite(lse)) and np.allclose(lse[fin], sl[fin], atol=1e-12)
    doc23 = [0] * 5 + [1] * 9 + [2] * 9
    tile_rules = rules[:4] + [{"kind": "and", "masks": [{"kind": "same_document", "doc_id": doc23},
                                                        {"kind": "same_chunk", "value": 3}]}]
    for mask in tile_rules:
        bm = o.block_mask(mask, 1, 4, 23, 23, 4, 3)
        for h in range(4):
            assert o.block_map(bm, 0, h) == sr.tile_classes_scalar(mask, 23, 23, 4, 3, 0, None, h), (mask, h)


def check_paged_cache(o):
    """A paged cache gives the dense cache's result; storage order is invisible.

    Pinned by: the page's decode example (capacity 8, valid length 6, window
    3, the query at position 5 sees keys 3, 4, 5) stored in shuffled pages of
    2; an identity page table over a contiguous pool, and a shuffled pool
    with its page table, equal the dense forward; a distance bias reads
    logical, not storage, positions; a circular layout (a ring of pages under
    a sliding window) whose stale pages hold garbage equals the dense window.
    """
    g = load("m3_decode_offset.txt")
    cap, valid, W = int(g["capacity"]), int(g["valid_length"]), int(g["window"])
    P = 2
    perm = np.array([2, 0, 3, 1])                    # logical page i -> physical page perm[i]
    pos = np.arange(cap, dtype=np.float64)
    kd = np.zeros((1, 1, cap, 1))                    # q = 0: every score equal
    vd = pos.reshape(1, 1, cap, 1)                   # each value its logical position
    kp = np.zeros((4, 1, P, 1))
    vp = np.zeros((4, 1, P, 1))
    for i in range(4):
        vp[perm[i], 0] = vd[0, 0, i * P:(i + 1) * P]
    mask = {"kind": "sliding_window", "window": W, "n_sink": 0}
    out, _ = o.forward_paged(np.zeros((1, 1, 1, 1)), kp, vp, perm[None, :], P, 4, 1.0, mask, None, kv_len=[valid])
    assert abs(out[0, 0, 0, 0] - np.mean(ints(g["visible"]))) < 1e-13  # the mean of keys 3, 4, 5
    # dense vs paged, identity and shuffled tables, GQA, per-sequence lengths, ALiBi
    r = np.random.default_rng(33)
    B, Hq, Hkv, L, P, npg, E = 3, 4, 2, 4, 4, 6, 5
    q = r.standard_normal((B, Hq, L, E))
    kd = r.standard_normal((B, Hkv, P * npg, E))
    vd = r.standard_normal((B, Hkv, P * npg, 3))
    kv_len = np.array([24, 17, 5])
    score = {"kind": "cap_then_bias", "cap": 4.0, "slope_heads": 0, "pos": "global"}
    ref_o, ref_l = o.forward(q, kd, vd, 0.5, {"kind": "causal"}, score, kv_len=kv_len, enable_gqa=True)
    for shuffle in (False, True):
        n_pool = B * npg + 3
        order = r.permutation(n_pool)[:B * npg] if shuffle else np.arange(B * npg)
        table = order.reshape(B, npg)
        kp = r.standard_normal((n_pool, Hkv, P, E)) * 50.0   # unused pages hold large values
        vp = r.standard_normal((n_pool, Hkv, P, 3)) * 50.0
        for b in range(B):
            for i in range(npg):
                kp[table[b, i]] = kd[b, :, i * P:(i + 1) * P]
                vp[table[b, i]] = vd[b, :, i * P:(i + 1) * P]
        po, pl = o.forward_paged(q, kp, vp, table, P, npg, 0.5, {"kind": "causal"}, score, kv_len=kv_len,
                                 enable_gqa=True)
        assert np.allclose(po, ref_o, atol=1e-13) and np.allclose(pl, ref_l, atol=1e-13)
        assert np.allclose(o.gather_pages(kp, table, P, npg), kd, atol=0)
    # circular layout: a window of W = 8 keys over a ring of 3 pages of 4; the
    # pages the window has left are reused, so a 20-key logical cache needs
    # logical page i at physical page i mod 3; stale logical pages map to
    # whatever the ring holds now and must stay hidden by the window
    P, ring, n_log, Wn = 4, 3, 5, 8
    kd = r.standard_normal((1, 1, P * n_log, E))
    vd = r.standard_normal((1, 1, P * n_log, 3))
    qd = r.standard_normal((1, 1, 1, E))
    kp = np.zeros((ring, 1, P, E))
    vp = np.zeros((ring, 1, P, 3))
    for i in range(n_log):                            # writes in order: the ring keeps the last 3 pages
        kp[i % ring] = kd[0, :, i * P:(i + 1) * P]
        vp[i % ring] = vd[0, :, i * P:(i + 1) * P]
    table = (np.arange(n_log) % ring)[None, :]
    win = {"kind": "sliding_window", "window": Wn, "n_sink": 0}
    po, pl = o.forward_paged(qd, kp, vp, table, P, n_log, 0.4, win, None, kv_len=[P * n_log])
    ro, rl = o.forward(qd, kd, vd, 0.4, win, None, kv_len=[P * n_log])
    assert np.allclose(po, ro, atol=1e-13) and np.allclose(pl, rl, atol=1e-13)


def check_backward(o):
    """Gradients of sum(out * W) for a random W.

    Pinned by central finite differences of the oracle's forward (step 1e-5,
    fp64) on tiny shapes for every score kind and several masks; by torch
    autograd (CPU, fp64) through a plain torch statement of the forward
    (scores, score rule, mask, softmax, values); by closed forms (a row with
    one visible key passes dO straight to that key's value and gives q and k
    nothing; a row with no visible key gives nothing at all); by GQA
    (dk, dv of a KV head = the sum over its query heads); and, for D formed
    from a stored output, by the closed-form shift that a changed D gives dq.
    """
    import torch
    r = np.random.default_rng(61)
    B, Hq, Hkv, L, S, E, Ev = 1, 4, 2, 5, 7, 3, 2
    masks = [{"kind": "causal"}, {"kind": "sliding_window", "window": 3, "n_sink": 1},
             {"kind": "and", "masks": [{"kind": "causal"}, {"kind": "stride", "value": 2}]}]
    scores = [{"kind": "none"}, {"kind": "softcap", "cap": 1.5}, {"kind": "alibi"},
              {"kind": "cap_then_bias", "cap": 2.0, "slope_heads": 0, "pos": "global"}]
    for mask in masks:
        for score in scores:
            q = r.standard_normal((B, Hq, L, E))
            k = r.standard_normal((B, Hkv, S, E))
            v = r.standard_normal((B, Hkv, S, Ev))
            W = r.standard_normal((B, Hq, L, Ev))
            kv_len = [6]
            dq, dk, dv = o.backward(q, k, v, W, 0.8, mask, score, kv_len=kv_len, enable_gqa=True)

            def loss(q_, k_, v_):
                out, _ = o.forward(q_, k_, v_, 0.8, mask, score, kv_len=kv_len, enable_gqa=True)
                return float((out * W).sum())
            eps = 1e-5
            for x, gx in ((q, dq), (k, dk), (v, dv)):
                num = np.zeros_like(x)
                for idx in np.ndindex(x.shape):
                    xp = x.copy()
                    xp[idx] += eps
                    args_p = [xp if y is x else y for y in (q, k, v)]
                    xm = x.copy()
                    xm[idx] -= eps
                    args_m = [xm if y is x else y for y in (q, k, v)]
                    num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
                assert np.allclose(num, gx, atol=1e-7, rtol=1e-6), (mask["kind"], score["kind"])
            # torch autograd through a plain statement of the forward
            tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
            G = Hq // Hkv
            kk = tk.repeat_interleave(G, dim=1)
            vv = tv.repeat_interleave(G, dim=1)
            sc = 0.8 * tq @ kk.transpose(-1, -2)
            qpos = torch.arange(L) + (kv_len[0] - L)
            kpos = torch.arange(S)
            if score["kind"] in ("softcap", "cap_then_bias"):
                g = score["cap"] * torch.tanh(sc / score["cap"])
            else:
                g = sc
            if score["kind"] in ("alibi", "cap_then_bias"):
                slope = torch.tensor([2.0 ** (-8.0 * (hh + 1) / Hq) for hh in range(Hq)], dtype=torch.float64)
                dist = (qpos[:, None] - kpos[None, :]).to(torch.float64)
                g = g - slope[None, :, None, None] * dist if score["kind"] == "alibi" else \
                    g + slope[None, :, None, None] * (-dist)
            vis = torch.from_numpy(o.visible(mask, 0, 0, qpos.numpy(), kpos.numpy(), kv_len[0]))
            out = torch.softmax(g.masked_fill(~vis, float("-inf")), dim=-1) @ vv
            (out * torch.from_numpy(W)).sum().backward()
            for t, gx in ((tq, dq), (tk, dk), (tv, dv)):
                assert np.allclose(t.grad.numpy(), gx, atol=1e-12), (mask["kind"], score["kind"])
    # one visible key (row 0, causal): dv gets dO, q gets nothing from that row
    q = r.standard_normal((1, 1, 4, 3))
    k = r.standard_normal((1, 1, 4, 3))
    v = r.standard_normal((1, 1, 4, 2))
    W = np.zeros((1, 1, 4, 2))
    W[0, 0, 0] = [1.5, -2.0]
    dq, dk, dv = o.backward(q, k, v, W, 1.0, {"kind": "causal"}, {"kind": "softcap", "cap": 3.0})
    assert np.allclose(dv[0, 0, 0], [1.5, -2.0], atol=0) and np.all(dv[0, 0, 1:] == 0)
    assert np.all(dq == 0) and np.all(dk == 0)
    # rows without a visible key (bottom-right, 3 keys for 5 queries) give nothing
    q = r.standard_normal((1, 1, 5, 3))
    k = r.standard_normal((1, 1, 3, 3))
    v = r.standard_normal((1, 1, 3, 2))
    W = np.zeros((1, 1, 5, 2))
    W[0, 0, :2] = 1.0
    dq, dk, dv = o.backward(q, k, v, W, 1.0, {"kind": "causal"}, None)
    assert np.all(dq == 0) and np.all(dk == 0) and np.all(dv == 0)
    # GQA: dk, dv of a KV head are the sums over its query heads
    q, k, v = _tiny_case(8, 5, 6, 3, 2, B=1, Hq=6, Hkv=2)
    W = r.standard_normal((1, 6, 5, 2))
    a = o.backward(q, k, v, W, 0.5, {"kind": "causal"}, {"kind": "alibi"}, enable_gqa=True)
    bq, bk, bv = o.backward(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), W, 0.5, {"kind": "causal"},
                            {"kind": "alibi"})
    assert np.allclose(a[0], bq, atol=1e-14)
    assert np.allclose(a[1], bk.reshape(1, 2, 3, 6, 3).sum(axis=2), atol=1e-13)
    assert np.allclose(a[2], bv.reshape(1, 2, 3, 6, 2).sum(axis=2), atol=1e-13)
    # the stored output: D is formed from the out the caller passes.  With
    # out = O + c_i dO_i / |dO_i|^2 (so D grows by c_i), dv is unchanged and,
    # with no score rule, dq_i moves by -scale c_i sum_j P_ij k_j, which is the
    # forward's output for v = k.
    q, k, v = _tiny_case(9, 6, 8, 3, 2, B=1, Hq=2, Hkv=2)
    W = r.standard_normal((1, 2, 6, 2))
    c = r.standard_normal((1, 2, 6))
    out, _ = o.forward(q, k, v, 0.7, {"kind": "causal"}, None)
    stored = out + c[..., None] * W / (W * W).sum(axis=-1, keepdims=True)
    ex = o.backward(q, k, v, W, 0.7, {"kind": "causal"}, None)
    st = o.backward(q, k, v, W, 0.7, {"kind": "causal"}, None, out=stored)
    same = o.backward(q, k, v, W, 0.7, {"kind": "causal"}, None, out=out)
    pk, _ = o.forward(q, k, k, 0.7, {"kind": "causal"}, None)
    assert np.allclose(st[2], ex[2], atol=1e-14)
    assert np.allclose(st[0] - ex[0], -0.7 * c[..., None] * pk, atol=1e-12)
    assert all(np.allclose(a_, b_, atol=1e-14) for a_, b_ in zip(same, ex))
    # row blocks: a unit's dq rows stacked and dk, dv parts summed give the unit
    q, k, v = _tiny_case(12, 9, 11, 3, 2, B=1, Hq=1, Hkv=1)
    W = r.standard_normal((1, 1, 9, 2))
    qp_all = o.query_positions(9, 10)
    score = {"kind": "cap_then_bias", "cap": 2.0, "slope_heads": 2, "pos": "global"}
    ref = o.backward_unit(q[0, 0], k[0, 0], v[0, 0], W[0, 0], 0, 1, 2, 10, 0.6, {"kind": "causal"}, score)
    parts = [o.backward_rows(q[0, 0, r0:r1], k[0, 0], v[0, 0], W[0, 0, r0:r1], 0.6, {"kind": "causal"}, score, 0, 1,
                             qp_all[r0:r1], 10, 2) for r0, r1 in ((0, 4), (4, 5), (5, 9))]
    assert np.allclose(np.concatenate([pt[0] for pt in parts]), ref[0], atol=1e-13)
    assert np.allclose(sum(pt[1] for pt in parts), ref[1], atol=1e-13)
    assert np.allclose(sum(pt[2] for pt in parts), ref[2], atol=1e-13)
    # query-side lists: the transpose of the tile map, ascending
    doc = np.repeat(np.arange(4), [9, 14, 5, 12])
    for mask in ({"kind": "causal"}, {"kind": "document", "doc_id": doc},
                 {"kind": "sliding_window", "window": 9, "n_sink": 2}):
        bm = o.block_mask(mask, 1, 1, 40, 40, 4, 8)
        tq = o.transpose_block_mask(bm)
        grid = o.block_map(bm)
        for n in range(bm["Nb"]):
            part = [m for m in range(bm["Mb"]) if grid[m][n] == "P"]
            full = [m for m in range(bm["Mb"]) if grid[m][n] == "F"]
            assert tq["q_indices"][0, 0, n, :len(part)].tolist() == part and tq["q_num_blocks"][0, 0, n] == len(part)
            assert tq["full_q_indices"][0, 0, n, :len(full)].tolist() == full
            assert tq["full_q_num_blocks"][0, 0, n] == len(full)
            assert np.all(tq["q_indices"][0, 0, n, len(part):] == 0)


ALL_CHECKS = [
    check_m1_six_token_tiles, check_m6_packed_documents, check_m2_softcap_after_mask,
    check_m3_decode_offset, check_m4_bottom_right, check_m5_left_padding,
    check_causal_block_fraction, check_window_count, check_single_visible_key, check_equal_scores,
    check_alibi_geometric, check_softcap_limits, check_cap_then_bias_order, check_convex_combination,
    check_against_torch_sdpa, check_against_scalar_loops, check_block_mask_against_scalar,
    check_split_combine, check_gqa_is_broadcast, check_sampled_rows_match_forward,
    check_max_scores, check_forward_unit_matches_forward, check_composed_masks,
    check_paged_cache,
]
SLOW_CHECKS = [check_workload_tile_counts, check_backward]
