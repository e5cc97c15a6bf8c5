"""The no-allocation decode entry point gives what the workspace entry point gives.

Some callers cannot allocate device memory when they call the library -- a
serving loop whose memory is fixed at start-up, a captured CUDA graph, a host
runtime without an allocator -- so they cannot hand flexattn_forward the
workspace its split-KV decode needs.  flexattn_forward_decode_noalloc keeps
those partial results in a scratch array inside the library instead.  This
file checks, through the C ABI, that two calls in a row (different inputs,
the same shared scratch) match flexattn_forward within the tests' usual
bf16 tolerance, and that a call needing more scratch than the array holds is
refused on the host.  It is collected last and passes alone or after the
other tests.
"""

import numpy as np
import pytest
import torch

from gpu_cases import Case, bf16_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


def _compare(case, split_kv):
    import programmable_block_sparse_b200 as fa
    bm = case.block_mask(128, 128)
    need = fa.flexattn_forward_workspace_size(case.q, case.k, case.v, bm, split_kv=split_kv)
    assert need > 0, "the case must use split-KV scratch"
    ref_out, ref_lse = fa.flexattn_forward(case.q, case.k, case.v, bm, score_mod=case.dev_score,
                                           mask_mod=case.dev_mask, scale=case.scale32, enable_gqa=True,
                                           split_kv=split_kv)
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    fa.flexattn_forward_decode_noalloc(case.q, case.k, case.v, bm, score_mod=case.dev_score, mask_mod=case.dev_mask,
                                       scale=case.scale32, enable_gqa=True, out=out, lse=lse, split_kv=split_kv)
    torch.cuda.synchronize()
    assert fa.flexattn_poll_device_status() == 0
    r = ref_out.float().cpu().numpy().astype(np.float64)
    g = out.float().cpu().numpy().astype(np.float64)
    assert not np.isnan(g).any()
    assert np.all(np.abs(g - r) <= bf16_tolerance(r)), np.abs(g - r).max()
    rl, gl = ref_lse.cpu().numpy(), lse.cpu().numpy()
    assert np.array_equal(np.isfinite(rl), np.isfinite(gl))
    fin = np.isfinite(rl)
    assert np.all(np.abs(gl[fin] - rl[fin]) <= 1e-3)


def test_noalloc_matches_workspace_entry_point_twice():
    first = Case(4, 16, 4, 4, 6000, 128, 128, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 50.0}, seed=21,
                 kv_len=[6000, 4100, 900, 129], sentinel_tail=True)
    _compare(first, split_kv=6)
    second = Case(3, 8, 2, 1, 3000, 64, 64, "bf16", {"kind": "sliding_window", "window": 700, "n_sink": 4},
                  {"kind": "alibi"}, seed=22, kv_len=[3000, 1234, 64], sentinel_tail=True)
    _compare(second, split_kv=4)


def test_noalloc_refuses_oversized_scratch():
    import programmable_block_sparse_b200 as fa
    # 8 x 32 heads x 16 rows x 32 splits x 66 floats = 34.6 MB: above the 16 MiB scratch
    case = Case(8, 32, 32, 16, 4096, 64, 64, "bf16", {"kind": "causal"}, {"kind": "none"}, seed=3)
    bm = case.block_mask(128, 128)
    with pytest.raises(fa.FlexAttnError) as e:
        fa.flexattn_forward_decode_noalloc(case.q, case.k, case.v, bm, mask_mod=case.dev_mask, split_kv=32)
    assert e.value.status == 10 and "scratch" in str(e.value)


def test_noalloc_automatic_split_count():
    """With split_kv = 0 the entry point takes the split count flexattn_forward
    would choose when its scratch fits the built-in array, and matches the
    workspace entry point on a decode-sized cache: 8 sequences of 4096-32768
    keys, 64 query heads over 8 KV heads, 16 query rows (three splits, 6.5 MB
    of scratch)."""
    rng = np.random.default_rng(5)
    kv_len = rng.integers(4096, 32769, 8).tolist()
    case = Case(8, 64, 8, 16, 32768, 64, 64, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 50.0}, seed=9,
                kv_len=kv_len, sentinel_tail=True)
    _compare(case, split_kv=0)


def test_noalloc_one_split_needs_no_scratch():
    """B=32, Hq=32, Hkv=8, 16 query rows, head dim 128: 1024 CTAs of work
    without splitting, so the automatic plan takes one split, which writes out
    and lse directly and needs no scratch; the entry point matches
    flexattn_forward.  (An automatic plan whose scratch exceeds the built-in
    array falls back to the most splits that fit, or to one split; on a
    148-SM B200 the automatic plans of the decode kernels stay below the
    array, so that branch is not reached here.)"""
    import programmable_block_sparse_b200 as fa
    rng = np.random.default_rng(6)
    kv_len = rng.integers(64, 700, 32).tolist()
    case = Case(32, 32, 8, 16, 700, 128, 128, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 50.0}, seed=10,
                kv_len=kv_len, sentinel_tail=True)
    bm = case.block_mask(128, 128)
    assert fa.flexattn_forward_workspace_size(case.q, case.k, case.v, bm, split_kv=0) == 0
    ref_out, ref_lse = fa.flexattn_forward(case.q, case.k, case.v, bm, score_mod=case.dev_score,
                                           mask_mod=case.dev_mask, scale=case.scale32, enable_gqa=True)
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    fa.flexattn_forward_decode_noalloc(case.q, case.k, case.v, bm, score_mod=case.dev_score, mask_mod=case.dev_mask,
                                       scale=case.scale32, enable_gqa=True, out=out, lse=lse, split_kv=0)
    torch.cuda.synchronize()
    assert fa.flexattn_poll_device_status() == 0
    r = ref_out.float().cpu().numpy().astype(np.float64)
    g = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - r) <= bf16_tolerance(r)), np.abs(g - r).max()
