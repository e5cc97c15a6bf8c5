"""GPU forward pass vs the fp64 oracle, element by element, through the C ABI."""

import math

import numpy as np
import pytest
import torch

from gpu_cases import Case, assert_close

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


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("score", SCORES, ids=lambda s: s["kind"] + ("_doc" if s.get("pos") == "in_doc" else ""))
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: m["kind"])
def test_mask_score_matrix(mask, score, dtype):
    case = Case(2, 4, 2, 300, 300, 64, 64, dtype, mask, score, seed=11)
    BM = 128 if dtype == "bf16" else 64
    out, lse = case.run(BM, BM)
    assert_close(case, out, lse, *case.oracle())
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
