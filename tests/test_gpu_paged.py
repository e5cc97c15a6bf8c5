"""Attention against a paged KV cache on the GPU, against the oracle.

"flexattention-score-mod-block-mask", "At decode, q_idx = 0 is not position
0": a paged or circular cache maps storage positions back to logical ones.
The pools hold the logical cache's pages in shuffled order among unused
pages of large finite values; every rule sees logical positions.  Covered:
the split-KV decode kernel (pages of 64 and 256 keys, forced splits), the
tensor-core prefill kernel reading a paged cache (pages of 64: a 128-key
tile spans two pages, and the logical length is not a multiple of 128), the
general kernel (pages of 48 keys), a pool stored (page, slot, head, dim)
and passed by its strides, a circular ring of pages under a sliding window,
and an out-of-range page id (clamped, FA_ERR_PARAM recorded).
"""

import math

import numpy as np
import pytest
import torch

import oracle.flex_oracle as o
import programmable_block_sparse_b200 as fa
import workloads as wl
from gpu_cases import out_tolerance

pytestmark = pytest.mark.gpu

FA_ERR_PARAM = 9


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


def _pool(k, v, P, seed, extra=5, table=None):
    """Pools (num_pages, Hkv, P, D) holding each sequence's logical pages in
    shuffled order among ``extra`` unused pages; returns pools and table."""
    B, Hkv, S, E = k.shape
    npg = S // P
    rng = np.random.default_rng(seed)
    n_pool = B * npg + extra
    if table is None:
        table = rng.permutation(n_pool)[:B * npg].reshape(B, npg).astype(np.int32)
    kp = (torch.randn((n_pool, Hkv, P, E), generator=torch.Generator().manual_seed(seed)) * 30).to(k.dtype)
    vp = (torch.randn((n_pool, Hkv, P, v.shape[3]), generator=torch.Generator().manual_seed(seed + 1)) * 30).to(k.dtype)
    for b in range(B):
        for i in range(npg):
            kp[table[b, i]] = k[b, :, i * P:(i + 1) * P]
            vp[table[b, i]] = v[b, :, i * P:(i + 1) * P]
    return kp, vp, table


def _check(out, lse, ro, rl, in_dtype):
    got = out.float().cpu().numpy().astype(np.float64)
    tol = out_tolerance(in_dtype, out.dtype == torch.float32, ro)
    err = np.abs(got - ro)
    assert np.all(err <= tol), f"max |out - ref| = {err.max():.3e}"
    gl = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.all(np.abs(gl[fin] - rl[fin]) <= 1e-3)


def _run(B, Hq, Hkv, L, P, npg, E, dtype, mask, score, kv_len, BM, split, seed=0, strided=False):
    S = P * npg
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q, k, v = wl.randn_qkv(B, Hq, Hkv, L, S, E, E, seed=seed, dtype=dt)
    kp, vp, table = _pool(k, v, P, seed + 100)
    scale = float(np.float32(1.0 / math.sqrt(E)))
    oracle_mask = dict(mask)
    dev_mask = dict(mask)
    if kv_len is not None:
        dev_mask["kv_len"] = torch.tensor(kv_len, dtype=torch.int32, device="cuda")
    ro, rl = o.forward_paged(q, kp, vp, table, P, npg, scale, oracle_mask, score, kv_len=kv_len,
                             enable_gqa=Hq != Hkv)
    if strided:  # the pool stored (page, slot, head, dim), passed as a strided view
        kd = kp.permute(0, 2, 1, 3).contiguous().cuda().permute(0, 2, 1, 3)
        vd = vp.permute(0, 2, 1, 3).contiguous().cuda().permute(0, 2, 1, 3)
    else:
        kd, vd = kp.cuda(), vp.cuda()
    tab = torch.from_numpy(table).cuda()
    bm = fa.flexattn_build_block_mask(dev_mask, B if kv_len is not None else 1, 1, L, S, BM, BM)
    out, lse = fa.flexattn_forward(q.cuda(), kd, vd, bm, score_mod=score, mask_mod=dev_mask, scale=scale,
                                   enable_gqa=Hq != Hkv, split_kv=split, paged={"page_table": tab, "page_size": P})
    torch.cuda.synchronize()
    assert fa.flexattn_poll_device_status() == 0
    _check(out, lse, ro, rl, dtype)
    return out, lse


@pytest.mark.parametrize("P,split", [(64, 0), (64, 3), (256, 1), (256, 0), (128, 5)])
@pytest.mark.parametrize("L", [1, 4])
def test_decode_paged(P, split, L):
    npg = 2048 // P
    _run(3, 8, 2, L, P, npg, 128, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 50.0}, [2048, 1300, 77],
         128, split, seed=P + L)


def test_decode_paged_strided_pool_and_window():
    _run(2, 4, 4, 4, 64, 20, 64, "bf16", {"kind": "sliding_window", "window": 300, "n_sink": 4},
         {"kind": "alibi"}, [1280, 900], 128, 0, seed=4, strided=True)


@pytest.mark.parametrize("E", [64, 128])
def test_prefill_paged_tensor_cores(E):
    # 11 pages of 64: logical length 704, not a multiple of the 128-key tile
    _run(2, 4, 2, 300, 64, 11, E, "bf16", {"kind": "causal"},
         {"kind": "cap_then_bias", "cap": 30.0, "slope_heads": 0, "pos": "global"}, [704, 650], 128, 1, seed=E)


def test_prefill_paged_persistent():
    # 256 pairs of query tiles over a pool of shuffled 64-key pages: the
    # persistent tensor-core kernel reads each key tile from two pages
    _run(2, 16, 4, 2048, 64, 32, 128, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 30.0}, [2048, 1500],
         128, 1, seed=41)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_paged_general_kernel(dtype):
    # pages of 48 keys: not a multiple of 64, so the general kernel reads them
    _run(2, 4, 2, 100, 48, 9, 64, dtype, {"kind": "chunked", "chunk": 100}, {"kind": "softcap", "cap": 20.0},
         [432, 300], 64, 1, seed=9)


def test_circular_ring_under_a_window():
    """A ring of 4 pages of 64 serves a window of 128: logical page i lives in
    ring page i mod 4, the pages the window left behind hold newer data; the
    result equals the dense cache's."""
    B, H, P, n_log, E, W = 1, 2, 64, 10, 64, 128
    S = P * n_log
    q, k, v = wl.randn_qkv(B, H, H, 4, S, E, E, seed=12, dtype=torch.bfloat16)
    kp = torch.zeros((4, H, P, E), dtype=torch.bfloat16)
    vp = torch.zeros((4, H, P, E), dtype=torch.bfloat16)
    for i in range(n_log):
        kp[i % 4] = k[0, :, i * P:(i + 1) * P]
        vp[i % 4] = v[0, :, i * P:(i + 1) * P]
    table = (np.arange(n_log) % 4).astype(np.int32)[None, :]
    mask = {"kind": "sliding_window", "window": W, "n_sink": 0}
    scale = 0.125
    ro, rl = o.forward(q, k, v, scale, mask, None)
    bm = fa.flexattn_build_block_mask(mask, 1, 1, 4, S, 128, 128)
    out, lse = fa.flexattn_forward(q.cuda(), kp.cuda(), vp.cuda(), bm, mask_mod=mask, scale=scale, split_kv=0,
                                   paged={"page_table": torch.from_numpy(table).cuda(), "page_size": P})
    torch.cuda.synchronize()
    assert fa.flexattn_poll_device_status() == 0
    _check(out, lse, ro, rl, "bf16")


def test_out_of_range_page_id_is_clamped_and_reported():
    B, H, P, npg, E = 1, 2, 64, 4, 64
    q, k, v = wl.randn_qkv(B, H, H, 4, P * npg, E, E, seed=13, dtype=torch.bfloat16)
    kp, vp, table = _pool(k, v, P, 5, extra=1)
    table = table.copy()
    table[0, 1] = 10_000
    bm = fa.flexattn_build_block_mask({"kind": "causal"}, 1, 1, 4, P * npg, 128, 128)
    for split in (0, 1):
        fa.flexattn_forward(q.cuda(), kp.cuda(), vp.cuda(), bm, mask_mod={"kind": "causal"}, split_kv=split,
                            paged={"page_table": torch.from_numpy(table).cuda(), "page_size": P})
        assert fa.flexattn_poll_device_status() == FA_ERR_PARAM
