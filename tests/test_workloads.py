"""The seeded input recipes produce the documented shapes and draws."""
import numpy as np
import torch

import workloads as w


def test_packed_doc_lengths_seed0():
    lens = w.doc_lengths(8192, 128, 2048, seed=0)
    assert lens == [1762, 1351, 1109, 646, 719, 206, 272, 159, 464, 1504]
    assert sum(lens) == 8192
    ids = w.doc_ids_from_lengths(lens)
    pos = w.in_doc_positions(lens)
    assert ids.shape == (8192,) and pos.shape == (8192,)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    assert np.all(pos[starts] == 0) and np.all(np.diff(ids) >= 0)


def test_decode_cache_lengths_seed0():
    lens = w.decode_cache_lengths(32, 4096, 32768, seed=0)
    assert lens.dtype == np.int32 and lens.shape == (32,)
    assert int(lens.sum()) == 614602
    assert lens.min() >= 4096 and lens.max() <= 32768


def test_qkv_slices_regenerate_alone():
    q, k, v = w.randn_qkv(2, 3, 1, 5, 7, 4, 6, seed=0, dtype=torch.float32)
    for which, t in ((0, q), (1, k), (2, v)):
        B, H, N, D = t.shape
        for b in range(B):
            for h in range(H):
                g = torch.Generator("cpu").manual_seed(w.slice_seed(0, which, b, h))
                assert torch.equal(t[b, h], torch.randn((N, D), generator=g))
    qb, _, _ = w.randn_qkv(2, 3, 1, 5, 7, 4, 6, seed=0, dtype=torch.bfloat16)
    assert torch.equal(qb, q.to(torch.bfloat16))
    assert not torch.equal(q[0, 0], q[0, 1]) and not torch.equal(q[0, 0], q[1, 0])
    q1, _, _ = w.randn_qkv(2, 3, 1, 5, 7, 4, 6, seed=1, dtype=torch.float32)
    assert not torch.equal(q, q1)
    seeds = {w.slice_seed(s, t, b, h) for s in range(3) for t in range(3) for b in range(32) for h in range(64)}
    assert len(seeds) == 3 * 3 * 32 * 64 and max(seeds) < 2 ** 32


def test_cache_tail_sentinels():
    k = torch.zeros(2, 1, 8, 2)
    v = torch.zeros(2, 1, 8, 2)
    w.fill_cache_tail(k, v, np.array([8, 5]))
    assert torch.all(k[0] == 0) and torch.all(k[1, :, 5:] == 1e4) and torch.all(v[1, :, 5:] == -1e4)
    assert torch.all(k[1, :, :5] == 0)


def test_configs_are_complete():
    for name, c in w.CONFIGS.items():
        for key in ("B", "Hq", "Hkv", "L", "S", "E", "Ev", "dtype", "seed", "scale", "BM", "BN", "mask", "score"):
            assert key in c, (name, key)
        assert c["Hq"] % c["Hkv"] == 0


def test_oracle_pool_units_equal_whole_tensor_oracle():
    """The pool's per-unit oracle (slices regenerated per unit in spawned
    workers) equals the oracle on whole tensors drawn by randn_qkv, for a
    shrunken copy of each workload kind (slope per head, documents, GQA,
    per-sequence cache lengths with sentinel tails)."""
    import numpy as np
    import torch

    import oracle.flex_oracle as o
    import workloads as wl
    from oracle_pool import oracle_units, workload_specs

    cases = [("causal_softcap_alibi", dict(B=2, Hq=3, Hkv=3, L=160, S=160)),
             ("packed_docs", dict(Hq=2, Hkv=2, L=300, S=300, doc_total=300, doc_lo=20, doc_hi=90)),
             ("gqa_sliding_window", dict(B=1, Hq=4, Hkv=2, L=200, S=200, mask=dict(kind="sliding_window",
                                                                                    window=37, n_sink=4))),
             ("decode_kv_cache", dict(B=3, Hq=4, Hkv=2, L=4, S=300, kv_lo=20, kv_hi=300))]
    for name, over in cases:
        c, mask, score, kv_len = workload_specs(name, **over)
        q, k, v = wl.randn_qkv(c["B"], c["Hq"], c["Hkv"], c["L"], c["S"], c["E"], c["Ev"], seed=c["seed"],
                               dtype=torch.bfloat16)
        if kv_len is not None:
            wl.fill_cache_tail(k, v, kv_len)
        scale = float(np.float32(c["scale"]))
        ref_o, ref_l, ref_m = o.forward(q, k, v, scale, mask, score, kv_len=kv_len, enable_gqa=True, aux=True)
        units = [(b, h) for b in range(c["B"]) for h in range(c["Hq"])]
        got = oracle_units(name, units, workers=2, **over)
        for (b, h), (uo, ul, um) in got.items():
            assert np.allclose(uo, ref_o[b, h], atol=1e-13, rtol=0), (name, b, h)
            fin = np.isfinite(ref_l[b, h])
            assert np.array_equal(np.isfinite(ul), fin)
            assert np.allclose(ul[fin], ref_l[b, h][fin], atol=1e-13) and np.allclose(um[fin], ref_m[b, h][fin])
