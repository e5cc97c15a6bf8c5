"""Split-KV decode (short queries, long KV caches) vs the fp64 oracle."""

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


@pytest.mark.parametrize("split_kv", [0, 3, 1])
@pytest.mark.parametrize("L,Hq,Hkv", [(1, 8, 2), (4, 8, 2), (16, 4, 4), (2, 32, 4), (3, 6, 2)])
@pytest.mark.parametrize("E", [64, 128])
def test_decode_against_oracle(L, Hq, Hkv, E, split_kv):
    kv_len = [1500, 700, 129, 64]
    case = Case(4, Hq, Hkv, L, 1500, E, E, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 50.0}, seed=L + E,
                kv_len=kv_len, sentinel_tail=True)
    ro, rl, rm = case.oracle(aux=True)
    out, lse, mx = case.run(128, 128, split_kv=split_kv, max_scores=True)
    assert_close(case, out, lse, ro, rl, mx, rm)
    assert out.abs().max().item() < 10.0  # the +-1e4 cache tail never leaks
    # an fp32 output (from the split path's combine, or straight from one split) within a strict 1e-2
    out32, lse32 = case.run(128, 128, split_kv=split_kv, out_dtype=torch.float32)
    assert_close(case, out32, lse32, ro, rl)
    _status_ok()


DECODE_MASKS = [{"kind": "none"}, {"kind": "sliding_window", "window": 200, "n_sink": 4},
                {"kind": "chunked", "chunk": 300}, {"kind": "prefix_lm", "prefix": 100}, {"kind": "document"}]
DECODE_SCORES = [{"kind": "none"}, {"kind": "alibi"}, {"kind": "cap_then_bias", "cap": 30.0, "pos": "global"},
                 {"kind": "cap_then_bias", "cap": 20.0, "pos": "in_doc"}]


@pytest.mark.parametrize("E", [64, 128])
@pytest.mark.parametrize("mask", DECODE_MASKS, ids=lambda m: m["kind"])
@pytest.mark.parametrize("score", DECODE_SCORES, ids=lambda s: s["kind"] + ("_doc" if s.get("pos") == "in_doc" else ""))
def test_decode_mask_and_score_kinds(mask, score, E):
    """The tensor-core decode kernel (tiles of 128 keys) on every mask and
    score kind, with max_scores."""
    case = Case(3, 8, 2, 4, 1000, E, E, "bf16", mask, score, seed=4, kv_len=[1000, 555, 77], sentinel_tail=True)
    out, lse, mx = case.run(128, 128, split_kv=4, max_scores=True)
    ro, rl, rm = case.oracle(aux=True)
    assert_close(case, out, lse, ro, rl, mx, rm)
    _status_ok()


@pytest.mark.parametrize("E", [64, 128])
@pytest.mark.parametrize("L,Hq,Hkv,split_kv", [(1, 4, 1, 0), (4, 8, 2, 3), (16, 4, 4, 0), (3, 6, 2, 2)])
@pytest.mark.parametrize("score", [{"kind": "softcap", "cap": 30.0}, {"kind": "alibi"}], ids=lambda s: s["kind"])
def test_decode_tiles_of_64_keys(L, Hq, Hkv, split_kv, score, E):
    """Block masks of 64-key tiles take the mma.sync decode kernel."""
    case = Case(2, Hq, Hkv, L, 640, E, E, "bf16", {"kind": "causal"}, score, seed=8 + L, kv_len=[640, 100],
                sentinel_tail=True)
    out, lse, mx = case.run(64, 64, split_kv=split_kv, max_scores=True)
    ro, rl, rm = case.oracle(aux=True)
    assert_close(case, out, lse, ro, rl, mx, rm)
    _status_ok()


def test_decode_rows_without_keys():
    """kv_len smaller than L: the first rows see no key and give (0, -inf)."""
    case = Case(2, 4, 2, 8, 256, 64, 64, "bf16", {"kind": "causal"}, {"kind": "none"}, seed=6, kv_len=[256, 5],
                sentinel_tail=True)
    out, lse = case.run(128, 128, split_kv=2)
    assert torch.all(lse[1, :, :3] == -np.inf) and torch.all(out[1, :, :3] == 0)
    assert_close(case, out, lse, *case.oracle())
    _status_ok()


@pytest.mark.parametrize("kv_len", [[64, 700, 1500, 129, 700], [300] * 3 + [1200] + [5] * 2,
                                    [(37 * i) % 900 + 40 for i in range(40)]],
                         ids=["ascending_and_ties", "equal_runs", "forty_sequences"])
@pytest.mark.parametrize("split_kv", [0, 3])
def test_decode_sequence_order(kv_len, split_kv):
    """The tensor-core decode takes sequences longest list first and cuts
    each into equal chunks: lengths out of order, ties, and more than 32
    sequences (then taken in batch order)."""
    case = Case(len(kv_len), 8, 2, 4, 1500, 128, 128, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 50.0},
                seed=len(kv_len), kv_len=kv_len, sentinel_tail=True)
    ro, rl, rm = case.oracle(aux=True)
    out, lse, mx = case.run(128, 128, split_kv=split_kv, max_scores=True)
    assert_close(case, out, lse, ro, rl, mx, rm)
    _status_ok()


def test_split_counts_agree():
    import programmable_block_sparse_b200 as fa
    case = Case(2, 8, 2, 4, 4096, 128, 128, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 50.0}, seed=1,
                kv_len=[4096, 3000], sentinel_tail=True)
    ref = None
    for split in (1, 0, 2, 7, 32):
        out, lse = case.run(128, 128, split_kv=split)
        if ref is None:
            ref = (out.float(), lse)
            continue
        assert (out.float() - ref[0]).abs().max().item() < 2e-2
        assert (lse - ref[1]).abs().max().item() < 1e-4
    bm = case.block_mask(128, 128)
    need = fa.flexattn_forward_workspace_size(case.q, case.k, case.v, bm, split_kv=7)
    assert need > 0
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(fa.FlexAttnError) as e:
        fa.flexattn_forward(case.q, case.k, case.v, bm, score_mod=case.dev_score, mask_mod=case.dev_mask,
                            enable_gqa=True, split_kv=7, workspace=small)
    assert e.value.status == 10
    _status_ok()
