"""GPU block-mask classifier vs the oracle: all four arrays bit-exact."""

import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


def _device_spec(mask):
    d = dict(mask)
    if "doc_id" in d:
        d["doc_id"] = torch.as_tensor(np.asarray(d["doc_id"], dtype=np.int32)).cuda().reshape(-1, np.shape(d["doc_id"])[-1])
    if d.get("kv_len") is not None:
        d["kv_len"] = torch.as_tensor(np.asarray(d["kv_len"], dtype=np.int32)).cuda()
    return d


def _compare(mask, B, H, L, S, BM, BN, kv_len=None):
    import oracle.flex_oracle as o
    import programmable_block_sparse_b200 as fa
    dev = _device_spec(dict(mask, kv_len=kv_len))
    bm = fa.flexattn_build_block_mask(dev, B, H, L, S, BM, BN)
    torch.cuda.synchronize()
    ref = o.block_mask(mask, B, H, L, S, BM, BN, kv_len=kv_len)
    for name in ("kv_num_blocks", "kv_indices", "full_kv_num_blocks", "full_kv_indices"):
        got = getattr(bm, name).cpu().numpy()
        assert got.dtype == np.int32
        assert np.array_equal(got, ref[name]), (name, mask["kind"], L, S, BM, BN)
    assert fa.flexattn_poll_device_status() == 0
    return bm


def _random_docs(S, seed, sorted_ids=True):
    lens = wl.doc_lengths(S, max(1, S // 12), max(2, S // 3), seed)
    ids = wl.doc_ids_from_lengths(lens)
    if not sorted_ids:  # document ids need not be increasing: relabel them
        perm = np.random.default_rng(seed).permutation(len(lens)).astype(np.int32)
        ids = perm[ids]
    return ids


MASKS = [
    {"kind": "none"},
    {"kind": "causal"},
    {"kind": "sliding_window", "window": 5, "n_sink": 0},
    {"kind": "sliding_window", "window": 37, "n_sink": 4},
    {"kind": "sliding_window", "window": 1, "n_sink": 2},
    {"kind": "prefix_lm", "prefix": 19},
    {"kind": "prefix_lm", "prefix": 0},
    {"kind": "chunked", "chunk": 24},
    {"kind": "chunked", "chunk": 1},
]
SHAPES = [(6, 6, 2, 2), (16, 16, 4, 4), (128, 128, 32, 32), (200, 333, 64, 32), (333, 200, 32, 64),
          (1, 300, 128, 128), (4, 1000, 128, 128), (257, 257, 128, 128), (100, 100, 7, 13), (64, 64, 1, 1)]


@pytest.mark.parametrize("mask", MASKS, ids=lambda m: "-".join(str(v) for v in m.values()))
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_interval_masks_bit_exact(mask, shape):
    L, S, BM, BN = shape
    _compare(mask, 1, 1, L, S, BM, BN)


@pytest.mark.parametrize("sorted_ids", [True, False])
@pytest.mark.parametrize("shape", [(16, 16, 4, 4), (200, 200, 16, 32), (257, 257, 128, 128), (500, 500, 64, 64)],
                         ids=lambda s: "x".join(map(str, s)) if isinstance(s, tuple) else str(s))
def test_document_mask_bit_exact(shape, sorted_ids):
    L, S, BM, BN = shape
    ids = _random_docs(S, seed=L + BN, sorted_ids=sorted_ids)
    _compare({"kind": "document", "doc_id": ids}, 1, 1, L, S, BM, BN)


@pytest.mark.parametrize("pattern", ["random3", "alternating", "single", "blocks_of_5"])
@pytest.mark.parametrize("shape", [(200, 200, 16, 32), (300, 300, 128, 128), (129, 257, 64, 128), (97, 97, 128, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_document_mask_interleaved_ids(shape, pattern):
    """Ids that repeat out of order: up to BN runs per tile, one id in many runs."""
    L, S, BM, BN = shape
    rng = np.random.default_rng(S + BN)
    if pattern == "random3":
        ids = rng.integers(0, 3, S)
    elif pattern == "alternating":
        ids = np.arange(S) % 2
    elif pattern == "single":
        ids = np.zeros(S)
    else:
        ids = (np.arange(S) // 5) % 3
    _compare({"kind": "document", "doc_id": ids.astype(np.int32)}, 1, 1, L, S, BM, BN)


@pytest.mark.parametrize("mask", MASKS[:6] + [{"kind": "document"}], ids=lambda m: m["kind"])
def test_per_sequence_kv_len_and_head_broadcast(mask):
    B, H, L, S = 3, 2, 7, 333
    kv_len = [333, 150, 1]
    if mask["kind"] == "document":
        mask = {"kind": "document", "doc_id": np.stack([_random_docs(S, s) for s in range(B)])}
    _compare(mask, B, H, L, S, 128, 32, kv_len=kv_len)
    _compare(mask, B, 1, 300, S, 64, 64, kv_len=[333, 300, 299])


def test_page_examples_on_gpu():
    """The 6-token 2x2 example and the 16-token packed example, classified on the GPU."""
    bm = _compare({"kind": "causal"}, 1, 1, 6, 6, 2, 2)
    assert bm.full_kv_num_blocks.sum().item() == 3 and bm.kv_num_blocks.sum().item() == 3
    doc = np.repeat(np.arange(3), [5, 4, 7]).astype(np.int32)
    bm = _compare({"kind": "document", "doc_id": doc}, 1, 1, 16, 16, 4, 4)
    assert bm.kv_num_blocks.sum().item() == 7 and bm.full_kv_num_blocks.sum().item() == 0


@pytest.mark.parametrize("name", ["fp32_causal_small", "causal_softcap_alibi", "packed_docs", "gqa_sliding_window",
                                  "decode_kv_cache"])
def test_workload_block_masks(name):
    c = wl.config(name)
    mask = dict(c["mask"])
    kv_len = None
    B = 1
    if name == "packed_docs":
        mask["doc_id"] = wl.doc_ids_from_lengths(wl.doc_lengths(c["doc_total"], c["doc_lo"], c["doc_hi"], c["seed"]))
    if name == "decode_kv_cache":
        kv_len = wl.decode_cache_lengths(c["B"], c["kv_lo"], c["kv_hi"], c["seed"]).tolist()
        B = c["B"]
    bm = _compare(mask, B, 1, c["L"], c["S"], c["BM"], c["BN"], kv_len=kv_len)
    visited = int(bm.kv_num_blocks.sum().item() + bm.full_kv_num_blocks.sum().item())
    expected = {"fp32_causal_small": 10, "causal_softcap_alibi": 136, "gqa_sliding_window": 1235}
    if name in expected:
        assert visited == expected[name]
