"""Seeded synthetic inputs for the FlexAttention hot path.

This module is shared by the CPU oracle side (tests that pin the oracle) and by
the CUDA side (GPU parity tests, ``bench.py``).  It holds random draws, shapes
and the parameters of the workloads only -- none of the attention arithmetic.
Mask and score specifications are plain dictionaries of strings and numbers;
the oracle and the C-ABI binding each interpret them with their own code.

Recipes (stated so that every number below can be regenerated):

* Q/K/V: ``torch.Generator('cpu').manual_seed(seed)``, then ``torch.randn`` in
  fp32 in the order q, k, v, each of its full (B, H, N, D) shape, then a cast to
  the workload dtype.  iid N(0, 1).
* Packed documents: lengths drawn one at a time from
  ``numpy.random.default_rng(seed).integers(lo, hi + 1)`` until their sum
  reaches the total, the last one trimmed so the sum is exact.
* Decode cache lengths: ``numpy.random.default_rng(seed).integers(lo, hi + 1, B)``.
* Unused cache tail (positions >= the valid length): K holds +1e4 and V holds
  -1e4, finite sentinels that must never leak into an output.
"""

from __future__ import annotations

import math

import numpy as np
import torch

__all__ = [
    "randn_qkv",
    "doc_lengths",
    "doc_ids_from_lengths",
    "in_doc_positions",
    "decode_cache_lengths",
    "fill_cache_tail",
    "CONFIGS",
    "config",
]


def randn_qkv(B, Hq, Hkv, L, S, E, Ev, seed=0, dtype=torch.bfloat16):
    """iid N(0,1) q (B,Hq,L,E), k (B,Hkv,S,E), v (B,Hkv,S,Ev) on the CPU."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    q = torch.randn((B, Hq, L, E), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, S, E), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, S, Ev), generator=g, dtype=torch.float32)
    return q.to(dtype), k.to(dtype), v.to(dtype)


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
