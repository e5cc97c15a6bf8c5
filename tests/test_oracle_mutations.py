"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each.

Every mutation below is a one-line edit of the oracle's source (a dropped term,
a wrong sign or index, an off-by-one bound, a transposed operand, the wrong
order of the score rule and the mask).  The edited source is loaded as a fresh
module on the CPU; the real oracle is untouched.  Each edited oracle must fail
at least one check of tests/oracle_pins.py.
"""

import importlib.util
import os

import pytest

import oracle_pins as pins

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "flex_oracle.py")

MUTATIONS = {
    "top_left_alignment": ("+ (int(S_b) - int(L))", "+ 0"),
    "strict_causal": ("causal = kv <= qp", "causal = kv < qp"),
    "window_includes_W_plus_1": ("(qp - kv) < W", "(qp - kv) <= W"),
    "sink_off_by_one": ("(kv < n_sink)", "(kv <= n_sink)"),
    "prefix_off_by_one": ("m = causal | (kv < P)", "m = causal | (kv <= P)"),
    "chunk_ignored": ("m = causal & (np.floor_divide(qp, C) == np.floor_divide(kv, C))",
                      "m = causal & (np.floor_divide(qp, C) >= np.floor_divide(kv, C))"),
    "document_ignored": ("m = causal & (qp >= 0) & (doc_b[qi] == doc_b[ki])",
                         "m = causal & (qp >= 0) & (doc_b[qi] >= doc_b[ki])"),
    "kv_len_ignored": ("in_range = kv < S_b", "in_range = kv >= 0"),
    "alibi_sign": ("return s - slope * (qp - kv)", "return s + slope * (qp - kv)"),
    "slope_index": ("2.0 ** (-8.0 * (h + 1) / H)", "2.0 ** (-8.0 * h / H)"),
    "bias_then_cap": ("return c * np.tanh(s / c) + slope * (pk - pq).astype(np.float64)",
                      "return c * np.tanh((s + slope * (pk - pq).astype(np.float64)) / c)"),
    "bias_sign": ("slope * (pk - pq)", "slope * (pq - pk)"),
    "softcap_scale_dropped": ("return c * np.tanh(s / c)\n", "return np.tanh(s / c)\n"),
    "mask_before_score_rule": ("st = np.where(vis, g, NEG_INF)", "st = score_mod(score, np.where(vis, s, NEG_INF), b, h, qp, kv, Hq)"),
    "scale_twice": ("s = scale * (q_rows @ k.T)", "s = scale * scale * (q_rows @ k.T)"),
    "scale_dropped": ("s = scale * (q_rows @ k.T)", "s = (q_rows @ k.T)"),
    "lse_base2": ("lse[live] = m[live] + np.log(l)", "lse[live] = m[live] + np.log2(l)"),
    "not_normalised": ("out[live] = (p @ v) / l[:, None]", "out[live] = (p @ v)"),
    "k_for_v": ("out[live] = (p @ v) / l[:, None]", "out[live] = (p @ k) / l[:, None]"),
    "gqa_head_map": ("hk = h // G\n", "hk = h % Hkv\n"),
    "nan_on_empty_rows": ("m = st.max(axis=1)", "m = np.where(np.isneginf(st.max(axis=1)), 0.0, st.max(axis=1))"),
    "partial_as_full": ("if cell.all():", "if cell.any():"),
    "ragged_cells_counted_hidden": ("cell = vis[:, c0:c1]", "cell = np.pad(vis[:, c0:c1], ((0, 0), (0, BN - (c1 - c0))))"),
    "indices_descending": ("full_idx[b, h, mt, nf] = nt", "full_idx[b, h, mt, Nb - 1 - nf] = nt"),
    "sampled_head_map": ("kk = _as_f64(k[b, h // G])", "kk = _as_f64(k[b, h % Hkv])"),
    "sampled_positions_ignore_kv_len": ("qp = query_positions(L, S_b)[r:r + 1]", "qp = query_positions(L, S)[r:r + 1]"),
    "sampled_row_shifted": ("qrow = _as_f64(q[b, h, r:r + 1])", "qrow = _as_f64(q[b, h, max(r - 1, 0):max(r - 1, 0) + 1])"),
    "max_scores_unmasked": ("return out, lse, st.max(axis=1)", "return out, lse, g.max(axis=1)"),
    "max_scores_log2_units": ("return out, lse, st.max(axis=1)", "return out, lse, st.max(axis=1) * 1.4426950408889634"),
    "max_scores_raw_score": ("return out, lse, st.max(axis=1)", "return out, lse, np.where(vis, s, NEG_INF).max(axis=1)"),
    "or_as_and": ("            m = m | visible(sub, b, h, qp1, kv1, S_b)", "            m = m & visible(sub, b, h, qp1, kv1, S_b)"),
    "not_ignored": ('m = ~visible(mask["mask"], b, h, qp1, kv1, S_b)', 'm = visible(mask["mask"], b, h, qp1, kv1, S_b)'),
    "distance_below_inclusive": ('m = (qp - kv) < int(mask["value"])', 'm = (qp - kv) <= int(mask["value"])'),
    "stride_on_key_only": ('m = np.mod(qp - kv, int(mask["value"])) == 0', 'm = np.mod(kv, int(mask["value"])) == 0'),
    "head_below_inclusive": ('np.full(np.broadcast(qp, kv).shape, h < int(mask["value"]))',
                             'np.full(np.broadcast(qp, kv).shape, h <= int(mask["value"]))'),
    "same_chunk_truncated": ('m = np.floor_divide(qp, C) == np.floor_divide(kv, C)\n    elif kind == "same_document"',
                             'm = np.trunc(qp / C) == np.trunc(kv / C)\n    elif kind == "same_document"'),
    "page_slot_order": ("out[b, :, i * page_size:(i + 1) * page_size] = pool[table[b, i]]",
                        "out[b, :, i * page_size:(i + 1) * page_size] = pool[table[b, i]][:, ::-1]"),
    "page_table_ignored": ("out[b, :, i * page_size:(i + 1) * page_size] = pool[table[b, i]]",
                           "out[b, :, i * page_size:(i + 1) * page_size] = pool[b * pages_per_seq + i]"),
    "backward_slope_dropped": ("ds = dst * score_mod_slope(score, s)", "ds = dst"),
    "backward_rowsum_dropped": ("dst = p * (dp - D[:, None])", "dst = p * dp"),
    "backward_dk_unscaled": ("dk = scale * (ds.T @ q_bh)", "dk = ds.T @ q_bh"),
    "backward_gqa_overwrite": ("dk[b, kvh] += uk", "dk[b, kvh] = uk"),
    "backward_stored_out_ignored": ("o = p @ v_bh if out_bh is None else _as_f64(out_bh)", "o = p @ v_bh"),
    "backward_rows_rowsum_dropped": ("ds = p * (do_rows @ v.T - D[:, None])", "ds = p * (do_rows @ v.T)"),
    "backward_cap_slope": ("return 1.0 - np.tanh(s / c) ** 2", "return 1.0 - np.tanh(s / c)"),
    "transpose_unsorted": ("= sorted(lists[n])", "= lists[n][::-1]"),
    "combine_unweighted": ('out[live] = np.einsum("sr,sre->re", w, outs[:, live]) / tot[:, None]',
                           "out[live] = outs[:, live].mean(axis=0)"),
}

# cheapest checks first; the first one that fails ends the search
ORDER = sorted(pins.ALL_CHECKS + pins.SLOW_CHECKS,
               key=lambda f: (f is pins.check_against_torch_sdpa, f in pins.SLOW_CHECKS))


def _mutant(name, old, new):
    src = open(ORACLE_SRC).read()
    assert src.count(old) == 1, f"mutation {name}: pattern must occur exactly once"
    spec = importlib.util.spec_from_loader(f"oracle_mutant_{name}", loader=None)
    mod = importlib.util.module_from_spec(spec)
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name):
    old, new = MUTATIONS[name]
    mod = _mutant(name, old, new)
    for check in ORDER:
        try:
            check(mod)
        except Exception:  # noqa: BLE001 - any failure counts as a detection
            return
    pytest.fail(f"no pin detects the mutation {name!r}")
