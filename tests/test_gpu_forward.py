"""GPU forward pass vs the fp64 oracle, element by element, through the C ABI."""

import math

import numpy as np
import pytest
import torch

from gpu_cases import Case, assert_close, assert_max_scores

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


def _status_ok():
    import programmable_block_sparse_b200 as fa
    assert fa.flexattn_poll_device_status() == 0


# ---------------------------------------------------------------------------
# The pages' worked examples through the GPU
# ---------------------------------------------------------------------------

def test_softcap_after_mask_trap_through_tensor_cores():
    """The same trap in bf16 with 128 x 128 tiles and head dim 64: split_kv=1
    runs the tcgen05 prefill kernel, split_kv=0 the split-KV decode kernel."""
    import programmable_block_sparse_b200 as fa
    q = torch.zeros(1, 1, 2, 64, device="cuda", dtype=torch.bfloat16)
    k = torch.randn(1, 1, 2, 64, device="cuda").to(torch.bfloat16)
    v = torch.zeros(1, 1, 2, 64, device="cuda", dtype=torch.bfloat16)
    v[0, 0, 0, 0] = 1.0
    v[0, 0, 1, 1] = 1.0
    mask = {"kind": "causal"}
    bm = fa.flexattn_build_block_mask(mask, 1, 1, 2, 2, 128, 128)
    for split in (1, 0):
        out, lse = fa.flexattn_forward(q, k, v, bm, score_mod={"kind": "softcap", "cap": 5.0}, mask_mod=mask,
                                       scale=1.0, split_kv=split)
        assert out[0, 0, 0, :2].float().tolist() == [1.0, 0.0], (split, out[0, 0, 0, :2])
        assert abs(lse[0, 0, 0].item()) < 1e-6
    _status_ok()


def test_softcap_after_mask_trap_on_gpu():
    """Cap 5, equal raw scores, key 1 hidden: the GPU must give [1, 0], not [0.993307, 0.006693]."""
    import programmable_block_sparse_b200 as fa
    q = torch.zeros(1, 1, 2, 8, device="cuda")
    k = torch.randn(1, 1, 2, 8, device="cuda")
    v = torch.eye(2, device="cuda").reshape(1, 1, 2, 2)
    mask = {"kind": "causal"}
    for BM in (2, 128):
        bm = fa.flexattn_build_block_mask(mask, 1, 1, 2, 2, BM, BM)
        out, lse = fa.flexattn_forward(q, k, v, bm, score_mod={"kind": "softcap", "cap": 5.0}, mask_mod=mask, scale=1.0)
        assert out[0, 0, 0].tolist() == [1.0, 0.0]
        assert abs(lse[0, 0, 0].item()) < 1e-7
    _status_ok()


def test_bottom_right_decode_example_on_gpu():
    """One query against 5 keys, equal scores: bottom-right alignment gives 0.2 each."""
    import programmable_block_sparse_b200 as fa
    q = torch.ones(1, 1, 1, 4, device="cuda")
    k = torch.ones(1, 1, 5, 4, device="cuda")
    v = torch.eye(5, device="cuda").reshape(1, 1, 5, 5)
    bm = fa.flexattn_build_block_mask({"kind": "causal"}, 1, 1, 1, 5, 1, 5)
    out, lse = fa.flexattn_forward(q, k, v, bm, mask_mod={"kind": "causal"})
    assert np.allclose(out[0, 0, 0].cpu().numpy(), [0.2] * 5, atol=1e-6)
    assert abs(lse.item() - (2.0 + math.log(5))) < 1e-5
    _status_ok()


def test_six_token_two_by_two_tiles_forward():
    case = Case(1, 2, 2, 6, 6, 4, 4, "fp32", {"kind": "causal"}, {"kind": "softcap", "cap": 5.0}, seed=3)
    out, lse = case.run(2, 2)
    assert_close(case, out, lse, *case.oracle())
    _status_ok()


# ---------------------------------------------------------------------------
# Small cases: every mask x score kind, ragged tiles, GQA, fp32 and bf16
# ---------------------------------------------------------------------------

MASKS = [{"kind": "none"}, {"kind": "causal"}, {"kind": "sliding_window", "window": 70, "n_sink": 4},
         {"kind": "document"}, {"kind": "prefix_lm", "prefix": 50}, {"kind": "chunked", "chunk": 96}]
SCORES = [{"kind": "none"}, {"kind": "softcap", "cap": 5.0}, {"kind": "alibi", "slope_heads": 0},
          {"kind": "cap_then_bias", "cap": 30.0, "slope_heads": 4, "pos": "global"},
          {"kind": "cap_then_bias", "cap": 20.0, "slope_heads": 0, "pos": "in_doc"}]


def _score_id(s):
    return s["kind"] + ("_doc" if s.get("pos") == "in_doc" else "")


@pytest.mark.parametrize("dtype,E", [("fp32", 64), ("bf16", 64), ("bf16", 128)])
@pytest.mark.parametrize("score", SCORES, ids=_score_id)
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: m["kind"])
def test_mask_score_matrix(mask, score, dtype, E):
    """Every mask x score kind at L = S = 300 (3 tile rows), GQA 4 / 2, with
    max_scores: bf16 on the tensor-core kernel at head dims 64 and 128, fp32
    on the general kernel."""
    case = Case(2, 4, 2, 300, 300, E, E, dtype, mask, score, seed=11)
    BM = 128 if dtype == "bf16" else 64
    out, lse, mx = case.run(BM, BM, max_scores=True)
    ro, rl, rm = case.oracle(aux=True)
    assert_close(case, out, lse, ro, rl, mx, rm)
    _status_ok()


@pytest.mark.parametrize("E", [64, 128])
@pytest.mark.parametrize("score", SCORES, ids=_score_id)
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: m["kind"])
def test_nine_tile_rows_every_rule(mask, score, E):
    """L = S = 1100: nine query tiles (the last pair has no second tile, the
    last tile is ragged) and rows of up to nine key tiles, so both K/V rings
    (4 stages at head dim 64, 2 at 128) wrap several times.  Per-sequence
    valid lengths (1100, 1037) with a block mask of explicit batch and heads;
    bf16 and fp32 outputs (the fp32 output held to a strict 1e-2)."""
    case = Case(2, 4, 2, 1100, 1100, E, E, "bf16", mask, score, seed=13, kv_len=[1100, 1037])
    ro, rl, rm = case.oracle(aux=True)
    bm = case.block_mask(128, 128, B_mask=2, H_mask=4)
    out, lse, mx = case.run(128, 128, bm=bm, max_scores=True)
    assert_close(case, out, lse, ro, rl, mx, rm)
    out32, lse32 = case.run(128, 128, bm=bm, out_dtype=torch.float32)
    assert out32.dtype == torch.float32
    assert_close(case, out32, lse32, ro, rl)
    _status_ok()


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("E", [64, 128])
@pytest.mark.parametrize("LS", [(129, 129), (1, 700), (77, 700), (700, 77), (256, 512)])
def test_ragged_lengths_and_head_dims(LS, E, dtype):
    L, S = LS
    case = Case(1, 2, 1, L, S, E, E, dtype, {"kind": "causal"}, {"kind": "softcap", "cap": 30.0}, seed=L + S)
    out, lse = case.run(128, 128, split_kv=1)
    assert_close(case, out, lse, *case.oracle())
    _status_ok()


def test_fully_masked_rows_give_zero_and_neg_inf():
    """L=8 queries against S=4 keys, bottom-right causal: rows 0-3 see no key."""
    for dtype in ("fp32", "bf16"):
        case = Case(1, 1, 1, 8, 4, 64, 64, dtype, {"kind": "causal"}, {"kind": "none"}, seed=5)
        out, lse = case.run(128, 128, split_kv=1)
        assert torch.all(out[0, 0, :4] == 0) and torch.all(lse[0, 0, :4] == -math.inf)
        assert torch.isfinite(lse[0, 0, 4:]).all()
        assert_close(case, out, lse, *case.oracle())
    _status_ok()


@pytest.mark.parametrize("E", [64, 128])
def test_persistent_prefill_with_empty_items(E):
    """More pairs of query tiles than SMs (384), so running CTAs take over
    the launches of the rest, and some pairs without a single key tile: a
    sequence with no valid key, and, under bottom-right causal with L > S,
    the query tiles before the first visible key."""
    case = Case(4, 16, 8, 1300, 1000, E, E, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 30.0}, seed=21,
                kv_len=[1000, 0, 513, 777], sentinel_tail=True)
    out, lse = case.run(128, 128, split_kv=1)
    assert torch.all(out[1] == 0) and torch.all(lse[1] == -math.inf)
    assert_close(case, out, lse, *case.oracle())
    _status_ok()


def test_kv_len_tails_never_leak():
    """Cache positions past the valid length hold +-1e4; they must not reach the output."""
    for dtype in ("fp32", "bf16"):
        case = Case(3, 4, 2, 4, 1000, 64, 64, dtype, {"kind": "causal"}, {"kind": "softcap", "cap": 50.0}, seed=9,
                    kv_len=[1000, 613, 129], sentinel_tail=True)
        out, lse = case.run(128, 128, split_kv=1)
        assert_close(case, out, lse, *case.oracle())
        assert out.abs().max().item() < 10.0
    _status_ok()


def test_fp32_causal_small_workload():
    """B=1, H=2, L=S=128, E=64, fp32, causal, BM=BN=32: every output within 1e-5."""
    case = Case.from_config("fp32_causal_small")
    out, lse = case.run(case.BM, case.BN)
    err = assert_close(case, out, lse, *case.oracle())
    assert err <= 1e-5
    _status_ok()


def test_block_mask_broadcast_vs_per_head():
    """A block mask with B=H=1 and one with B, H explicit give identical results."""
    import programmable_block_sparse_b200 as fa
    case = Case(2, 4, 4, 200, 200, 64, 64, "bf16", {"kind": "causal"}, {"kind": "alibi"}, seed=2)
    a = fa.flexattn_forward(case.q, case.k, case.v, case.block_mask(128, 128, 1, 1), score_mod=case.dev_score,
                            mask_mod=case.dev_mask)
    b = fa.flexattn_forward(case.q, case.k, case.v, case.block_mask(128, 128, 2, 4), score_mod=case.dev_score,
                            mask_mod=case.dev_mask)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    _status_ok()


# ---------------------------------------------------------------------------
# Auxiliary output and the rows-guaranteed-safe flag
# ---------------------------------------------------------------------------

ROWS_SAFE_CASES = {
    # (dtype, E, L, S, mask, BM, split_kv)
    "tcgen05_e64": ("bf16", 64, 600, 600, {"kind": "chunked", "chunk": 96}, 128, 1),
    "tcgen05_e128": ("bf16", 128, 600, 600, {"kind": "sliding_window", "window": 100, "n_sink": 2}, 128, 1),
    "decode": ("bf16", 128, 4, 900, {"kind": "causal"}, 128, 3),
    "general_fp32": ("fp32", 64, 200, 200, {"kind": "chunked", "chunk": 48}, 64, 1),
}


@pytest.mark.parametrize("name", sorted(ROWS_SAFE_CASES))
def test_rows_guaranteed_safe_changes_nothing_when_it_holds(name):
    """Every row sees a key (a chunk or window always holds the query), though
    for many rows the first tile visited holds none: with the flag set the
    results are bit for bit those without it, and match the oracle."""
    dtype, E, L, S, mask, BM, split = ROWS_SAFE_CASES[name]
    case = Case(2, 4, 2, L, S, E, E, dtype, mask, {"kind": "softcap", "cap": 20.0}, seed=17)
    bm = case.block_mask(BM, BM)
    a = case.run(BM, BM, bm=bm, split_kv=split, max_scores=True)
    b = case.run(BM, BM, bm=bm, split_kv=split, max_scores=True, rows_guaranteed_safe=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    ro, rl, rm = case.oracle(aux=True)
    assert_close(case, b[0], b[1], ro, rl, b[2], rm)
    _status_ok()


def test_max_scores_of_rows_without_keys():
    """Rows that see no key: max_scores -inf beside out 0 and lse -inf, on the
    tensor-core, decode and general kernels."""
    for dtype, split in (("bf16", 1), ("bf16", 2), ("fp32", 1)):
        case = Case(2, 2, 2, 8, 200, 64, 64, dtype, {"kind": "causal"}, {"kind": "none"}, seed=5, kv_len=[200, 5],
                    sentinel_tail=True)
        out, lse, mx = case.run(128, 128, split_kv=split, max_scores=True)
        assert torch.all(mx[1, :, :3] == -math.inf) and torch.all(lse[1, :, :3] == -math.inf)
        ro, rl, rm = case.oracle(aux=True)
        assert_close(case, out, lse, ro, rl, mx, rm)
    _status_ok()
