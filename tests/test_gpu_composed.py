"""Composed mask rules on the GPU: block masks bit for bit against the oracle,
forward passes element by element, on the tensor-core, decode and general
kernels, with per-head block masks for head-dependent rules.

Rules ("PyTorch Flex Attention complete guide" section 4.3, and_masks /
or_masks; "Attention expressions", Examples): every fourth key; half the
heads global and half local; the fixed rules written as compositions; a
negated union; documents crossed with chunks; a window with sinks spelled
another way.
"""

import numpy as np
import pytest
import torch

import oracle.flex_oracle as o
import programmable_block_sparse_b200 as fa
import workloads as wl
from gpu_cases import Case, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


def _status_ok():
    assert fa.flexattn_poll_device_status() == 0


def _rules(H, doc):
    """name -> (rule spec, reads the head); ``doc`` fills same-document predicates."""
    causal = {"kind": "causal"}
    return {
        "every_fourth_key": (fa.and_masks(causal, {"kind": "stride", "value": 4}), False),
        "half_heads_global": (fa.and_masks(causal, fa.or_masks({"kind": "head_below", "value": H // 2},
                                                               {"kind": "distance_below", "value": 150})), True),
        "not_prefix_or_stride": (fa.not_mask(fa.or_masks({"kind": "key_below", "value": 40},
                                                         {"kind": "stride", "value": 3})), False),
        "documents_by_chunks": (fa.and_masks({"kind": "same_document", "doc_id": doc},
                                             {"kind": "same_chunk", "value": 96}), False),
        "window_sinks_other_spelling": (fa.or_masks(fa.and_masks(causal, {"kind": "distance_below", "value": 100}),
                                                    fa.and_masks(causal, {"kind": "key_below", "value": 4})), False),
        "chunked_as_composition": (fa.and_masks(causal, {"kind": "chunked", "chunk": 64}), False),
    }


def _case(name, B, Hq, Hkv, L, S, E, dtype, kv_len=None, seed=0, score=None):
    score = score or {"kind": "softcap", "cap": 20.0}
    case = Case(B, Hq, Hkv, L, S, E, E, dtype, {"kind": "causal"}, score, seed=seed, kv_len=kv_len,
                sentinel_tail=kv_len is not None)
    doc_np = wl.doc_ids_from_lengths(wl.doc_lengths(S, max(1, S // 12), max(2, S // 3), seed + 5))
    doc_dev = torch.from_numpy(doc_np).cuda().reshape(1, S)
    spec_o, reads_head = _rules(Hq, doc_np)[name]
    spec_d, _ = _rules(Hq, doc_dev)[name]
    case.oracle_mask = dict(spec_o)
    case.dev_mask = dict(spec_d)
    if kv_len is not None:
        case.dev_mask["kv_len"] = torch.from_numpy(np.asarray(kv_len, np.int32)).cuda()
    return case, reads_head


RULES = sorted(_rules(4, np.zeros(8, np.int32)))


@pytest.mark.parametrize("name", RULES)
@pytest.mark.parametrize("L,S,BM,BN,kv_len", [(300, 300, 128, 128, None), (1100, 1100, 128, 128, [1100, 1037]),
                                              (200, 333, 32, 64, [333, 17]), (4, 1000, 128, 128, [1000, 611])])
def test_block_mask_bit_exact(name, L, S, BM, BN, kv_len):
    B, H = 2, 4
    case, reads_head = _case(name, B, H, H, L, S, 64, "bf16", kv_len=kv_len, seed=L + S)
    Hm = H if reads_head else 1
    bm = case.block_mask(BM, BN, B_mask=B, H_mask=Hm)
    torch.cuda.synchronize()
    ref = o.block_mask(case.oracle_mask, B, Hm, L, S, BM, BN, kv_len=case.kv_len)
    for key in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        got = getattr(bm, key).cpu().numpy()
        assert np.array_equal(got, ref[key]), (name, key)
    _status_ok()


@pytest.mark.parametrize("name", RULES)
@pytest.mark.parametrize("path", ["tcgen05_e64", "tcgen05_e128", "general_fp32", "decode"])
def test_forward_matches_oracle(name, path):
    B, Hq, Hkv = 2, 4, 2
    if path == "decode":
        L, S, E, dtype, BM, kv_len, split = 4, 1000, 128, "bf16", 128, [1000, 611], 3
    elif path == "general_fp32":
        L, S, E, dtype, BM, kv_len, split = 300, 300, 64, "fp32", 64, [300, 257], 1
    else:
        E = 64 if path == "tcgen05_e64" else 128
        L, S, dtype, BM, kv_len, split = 1100, 1100, "bf16", 128, [1100, 1037], 1
    case, reads_head = _case(name, B, Hq, Hkv, L, S, E, dtype, kv_len=kv_len, seed=7)
    bm = case.block_mask(BM, BM, B_mask=B, H_mask=Hq if reads_head else 1)
    out, lse, mx = case.run(BM, BM, bm=bm, split_kv=split, max_scores=True)
    ro, rl, rm = case.oracle(aux=True)
    assert_close(case, out, lse, ro, rl, mx, rm)
    _status_ok()


@pytest.mark.parametrize("fixed", [{"kind": "causal"}, {"kind": "sliding_window", "window": 100, "n_sink": 4},
                                   {"kind": "prefix_lm", "prefix": 70}, {"kind": "chunked", "chunk": 96}],
                         ids=lambda m: m["kind"])
def test_fixed_rules_as_programs_give_identical_results(fixed):
    """A fixed rule and the same rule written as a composition give the same
    block mask and bit-identical outputs on the tensor-core kernel."""
    case = Case(2, 4, 2, 700, 700, 128, 128, "bf16", fixed, {"kind": "softcap", "cap": 30.0}, seed=3)
    bm_fixed = case.block_mask(128, 128)
    a = case.run(128, 128, bm=bm_fixed, split_kv=1)
    comp = fa.and_masks(fixed)  # a composition of one rule: the program form
    bm_prog = fa.flexattn_build_block_mask(comp, 1, 1, 700, 700, 128, 128)
    for key in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        assert torch.equal(getattr(bm_fixed, key), getattr(bm_prog, key)), key
    b = fa.flexattn_forward(case.q, case.k, case.v, bm_prog, score_mod=case.dev_score, mask_mod=comp,
                            scale=case.scale32, enable_gqa=True, split_kv=1)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    _status_ok()


def test_head_dependent_rule_needs_per_head_block_mask():
    case, _ = _case("half_heads_global", 1, 4, 4, 256, 256, 64, "bf16")
    bm = case.block_mask(128, 128, B_mask=1, H_mask=1)
    with pytest.raises(fa.FlexAttnError) as e:
        case.run(128, 128, bm=bm)
    assert e.value.status == 5


@pytest.mark.parametrize("name", ["half_heads_global", "every_fourth_key"])
def test_persistent_kernel_with_composed_rules(name):
    """256 pairs of query tiles, more than the SMs, so running CTAs take over
    the launches of the rest; the head-dependent rule with a block mask per
    head, whose items alternate long and short along the head index."""
    B, H, L = 2, 16, 2048
    case, reads_head = _case(name, B, H, H, L, L, 128, "bf16", seed=31)
    bm = case.block_mask(128, 128, B_mask=1, H_mask=H if reads_head else 1)
    out, lse, mx = case.run(128, 128, bm=bm, split_kv=1, max_scores=True)
    ro, rl, rm = case.oracle(aux=True)
    assert_close(case, out, lse, ro, rl, mx, rm)
    _status_ok()
