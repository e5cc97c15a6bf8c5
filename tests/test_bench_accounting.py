"""bench.py's exact work counts agree with the oracle's visibility on small shapes."""
import numpy as np

import bench
import oracle.flex_oracle as o
import workloads as wl


def _oracle_pairs(c, kv_len=None, doc_ids=None):
    mask = dict(c["mask"])
    if doc_ids is not None:
        mask["doc_id"] = doc_ids
    tot = 0
    for b in range(c["B"]):
        S_b = c["S"] if kv_len is None else int(kv_len[b])
        vis = o.visible(mask, b, 0, o.query_positions(c["L"], S_b), np.arange(c["S"]), S_b)
        tot += int(vis.sum())
    return tot


def test_visible_pair_counts():
    c = wl.config("causal_softcap_alibi", B=2, L=300, S=300)
    assert bench.visible_pairs_per_head(c) == _oracle_pairs(c)
    c = wl.config("gqa_sliding_window", B=1, L=700, S=700, mask=dict(kind="sliding_window", window=100, n_sink=4))
    assert bench.visible_pairs_per_head(c) == _oracle_pairs(c)
    lens = wl.doc_lengths(500, 20, 90, 3)
    c = wl.config("packed_docs", L=500, S=500)
    assert bench.visible_pairs_per_head(c, doc_lengths=lens) == _oracle_pairs(c, doc_ids=wl.doc_ids_from_lengths(lens))
    c = wl.config("decode_kv_cache", B=5, S=900)
    kv = np.array([900, 13, 400, 4, 77])
    assert bench.visible_pairs_per_head(c, kv_len=kv) == _oracle_pairs(c, kv_len=kv)


def test_full_size_counts_match_closed_forms():
    c = wl.config("causal_softcap_alibi")
    assert bench.visible_pairs_per_head(c) == 4 * 2048 * 2049 // 2
    c = wl.config("gqa_sliding_window")
    assert bench.visible_pairs_per_head(c) == 2 * 16314874


def test_kernel_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    """Recorded ncu counters stay valid across comment edits, not code edits."""
    import bench
    csrc = tmp_path / "programmable_block_sparse_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES["prefill"]:
        (csrc / name).write_text("int f(int x) {\n  return x + 1;  // add one\n}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash("prefill")
    (csrc / "fwd_sm100.cu").write_text("/* a new\n   block comment */\nint f(int x) {\n\n  return x + 1;\n}\n")
    assert bench.kernel_source_hash("prefill") == h0
    (csrc / "fwd_sm100.cu").write_text("int f(int x) {\n  return x + 2;\n}\n")
    assert bench.kernel_source_hash("prefill") != h0


def test_backward_items_and_their_oracle_sample():
    """Backward bench items reuse a workload's config (their mode key is not a
    config key) and the cpu sample times the oracle's backward of a row
    block, counting (6E + 4Ev) FLOPs per visible pair (S, dP, dV, dK, dQ)."""
    back = [it for it in bench.BENCH_ITEMS if it[2].get("backward")]
    assert back
    for label, name, over in back:
        assert bench.config_over(over) == {}
        wl.config(name, **bench.config_over(over))
    s = bench.OracleSampler("causal_softcap_alibi", backward=True, L=256, S=256, B=1, Hq=2, Hkv=2)
    work, el = s.block(0)
    c = s.c
    b, h = divmod(0, c["Hq"])
    assert work == float(s.visible(b, h)[:s.rows].sum()) * (6 * c["E"] + 4 * c["Ev"])
    assert el > 0


def test_composed_rule_counts():
    """The bench's closed forms for its composed-rule items (a sliver of every
    fourth key; half the heads global, half a 256-key window) against the
    oracle's visibility, head by head."""
    for label in ("sliver_every_fourth_key", "half_heads_global"):
        _, name, over = bench.item(label)
        c = wl.config(name, **bench.config_over(over), B=2, L=700, S=700, Hq=16, Hkv=16)
        want = 0
        for b in range(c["B"]):
            for h in range(c["Hq"]):
                vis = o.visible(c["mask"], b, h, o.query_positions(c["L"], c["S"]), np.arange(c["S"]), c["S"])
                got = bench.visible_counts_rows(c, b, h=h)
                assert np.array_equal(got, vis.sum(axis=1)), (label, b, h)
                want += int(vis.sum())
        assert bench.visible_pairs_all_heads(c) == want
