"""Seeded synthetic inputs for the FlexAttention hot path.

This module is shared by the CPU oracle side (tests that pin the oracle) and by
the CUDA side (GPU parity tests, ``bench.py``).  It holds random draws, shapes
and the parameters of the workloads only -- none of the attention arithmetic.
Mask and score specifications are plain dictionaries of strings and numbers;
the oracle and the C-ABI binding each interpret them with their own code.

Recipes (stated so that every number below can be regenerated):

* Q/K/V: every (b, h) slice of q (which = 0), k (1) and v (2) is drawn with
  ``torch.randn`` in fp32 from its own ``torch.Generator('cpu')`` seeded with
  ``slice_seed(seed, which, b, h)`` (a 32-bit mix of the four indices), then
  cast to the workload dtype.  iid N(0, 1); any slice can be regenerated alone.
* Packed documents: lengths drawn one at a time from
  ``numpy.random.default_rng(seed).integers(lo, hi + 1)`` until their sum
  reaches the total, the last one trimmed so the sum is exact.
* Decode cache lengths: ``numpy.random.default_rng(seed).integers(lo, hi + 1, B)``.
* Unused cache tail (positions >= the valid length): K holds +1e4 and V holds
  -1e4, finite sentinels that must never leak into an output.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

__all__ = [
    "slice_seed",
    "randn_slice",
    "randn_qkv",
    "randn_dout",
    "doc_lengths",
    "doc_ids_from_lengths",
    "in_doc_positions",
    "decode_cache_lengths",
    "fill_cache_tail",
    "CONFIGS",
    "config",
]


def slice_seed(seed, which, b, h):
    """32-bit seed of the (b, h) slice of tensor ``which`` (0 = q, 1 = k, 2 = v).

    torch's CPU generator keeps 32 bits of a seed, so the four indices are
    folded into 32 bits: a weighted sum, then an integer bit mixer.
    """
    m = 0xFFFFFFFF
    x = (int(seed) * 0x9E3779B1 + int(which) * 0x85EBCA77 + int(b) * 0xC2B2AE3D + int(h) * 0x27D4EB2F) & m
    x ^= x >> 16
    x = (x * 0x7FEB352D) & m
    x ^= x >> 15
    x = (x * 0x846CA68B) & m
    x ^= x >> 16
    return x


def randn_slice(seed, which, b, h, N, D, dtype=torch.bfloat16):
    """One (N, D) slice: torch.randn in fp32 from its own generator, then cast."""
    g = torch.Generator("cpu").manual_seed(slice_seed(seed, which, b, h))
    return torch.randn((N, D), generator=g, dtype=torch.float32).to(dtype)


def _fill(t, seed, which):
    B, H, N, D = t.shape
    jobs = [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        b, h = bh
        t[b, h].copy_(randn_slice(seed, which, b, h, N, D, t.dtype))

    if len(jobs) * N * D >= (1 << 22):
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4)) as ex:
            list(ex.map(one, jobs))
    else:
        for bh in jobs:
            one(bh)
    return t


def randn_qkv(B, Hq, Hkv, L, S, E, Ev, seed=0, dtype=torch.bfloat16):
    """iid N(0,1) q (B,Hq,L,E), k (B,Hkv,S,E), v (B,Hkv,S,Ev) on the CPU.

    Every (b, h) slice of every tensor has its own generator (see
    :func:`randn_slice`), so any slice can be regenerated on its own.
    """
    q = _fill(torch.empty((B, Hq, L, E), dtype=dtype), seed, 0)
    k = _fill(torch.empty((B, Hkv, S, E), dtype=dtype), seed, 1)
    v = _fill(torch.empty((B, Hkv, S, Ev), dtype=dtype), seed, 2)
    return q, k, v


def randn_dout(B, Hq, L, Ev, seed=0, dtype=torch.bfloat16):
    """iid N(0,1) output gradient (B,Hq,L,Ev), one generator per (b, h) slice
    (the fourth stream after q, k, v)."""
    return _fill(torch.empty((B, Hq, L, Ev), dtype=dtype), seed, 3)


def doc_lengths(total, lo, hi, seed=0):
    """Document lengths ~ U{lo..hi}, drawn until they cover ``total``; last trimmed."""
    rng = np.random.default_rng(int(seed))
    out, acc = [], 0
    while acc < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - acc)
        out.append(n)
        acc += n
    return out


def doc_ids_from_lengths(lengths):
    """Per-token document index (int32) for documents packed back to back."""
    return np.repeat(np.arange(len(lengths), dtype=np.int32), np.asarray(lengths, dtype=np.int64))


def in_doc_positions(lengths):
    """Per-token position inside its own document, restarting at 0 (int32)."""
    return np.concatenate([np.arange(n, dtype=np.int32) for n in lengths]) if lengths else np.zeros(0, np.int32)


def decode_cache_lengths(B, lo, hi, seed=0):
    """Valid KV-cache length per sequence ~ U{lo..hi} (int32)."""
    rng = np.random.default_rng(int(seed))
    return rng.integers(lo, hi + 1, B).astype(np.int32)


def fill_cache_tail(k, v, kv_len, k_value=1.0e4, v_value=-1.0e4):
    """Overwrite positions >= kv_len[b] of k and v in place with finite sentinels."""
    for b, n in enumerate(np.asarray(kv_len).tolist()):
        k[b, :, n:, :] = k_value
        v[b, :, n:, :] = v_value
    return k, v


# The five workloads.  ``mask`` and ``score`` are specifications, not code.
CONFIGS = {
    "fp32_causal_small": dict(
        B=1, Hq=2, Hkv=2, L=128, S=128, E=64, Ev=64, dtype="fp32", seed=0,
        scale=1.0 / math.sqrt(64), BM=32, BN=32,
        mask=dict(kind="causal"), score=dict(kind="none"),
    ),
    "causal_softcap_alibi": dict(
        B=4, Hq=16, Hkv=16, L=2048, S=2048, E=64, Ev=64, dtype="bf16", seed=0,
        scale=1.0 / math.sqrt(64), BM=128, BN=128,
        mask=dict(kind="causal"),
        score=dict(kind="cap_then_bias", cap=50.0, slope_heads=16, pos="global"),
    ),
    "packed_docs": dict(
        B=1, Hq=16, Hkv=16, L=8192, S=8192, E=128, Ev=128, dtype="bf16", seed=0,
        scale=1.0 / math.sqrt(128), BM=128, BN=128,
        doc_total=8192, doc_lo=128, doc_hi=2048,
        mask=dict(kind="document"),
        score=dict(kind="cap_then_bias", cap=30.0, slope_heads=16, pos="in_doc"),
    ),
    "gqa_sliding_window": dict(
        B=2, Hq=32, Hkv=8, L=16384, S=16384, E=128, Ev=128, dtype="bf16", seed=0,
        scale=1.0 / math.sqrt(128), BM=128, BN=128,
        mask=dict(kind="sliding_window", window=1024, n_sink=4), score=dict(kind="none"),
    ),
    "decode_kv_cache": dict(
        B=32, Hq=32, Hkv=8, L=4, S=32768, E=128, Ev=128, dtype="bf16", seed=0,
        scale=1.0 / math.sqrt(128), BM=128, BN=128,
        kv_lo=4096, kv_hi=32768,
        mask=dict(kind="causal"), score=dict(kind="softcap", cap=50.0),
    ),
}


def config(name, **overrides):
    """A copy of one workload's parameters with fields overridden."""
    c = dict(CONFIGS[name])
    c["mask"] = dict(c["mask"])
    c["score"] = dict(c["score"])
    c.update(overrides)
    return c
