"""Whole (batch, query head) units of the workloads, evaluated by the fp64 oracle
in a pool of spawned worker processes.

Each worker regenerates the unit's own q slice and its KV head's k / v slices
from the workload's seed (``workloads.randn_slice``: every slice has its own
generator, so nothing large crosses the process boundary) and runs
``oracle.forward_unit`` on them with the unit's true batch and head indices.
The pool uses the ``spawn`` start method, so it is safe to create after the
process has touched the GPU; each worker limits its BLAS to one thread.
"""

from __future__ import annotations

import multiprocessing as mp
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np


def _init_worker(root):
    import sys
    if root not in sys.path:
        sys.path.insert(0, root)
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # noqa: BLE001 - the limit only speeds things up
        pass
    import torch
    torch.set_num_threads(1)


def workload_specs(name, **over):
    """(config, oracle mask spec, oracle score spec, kv_len or None)."""
    import workloads as wl
    c = wl.config(name, **over)
    mask, score = dict(c["mask"]), dict(c["score"])
    kv_len = None
    if name == "decode_kv_cache":
        kv_len = wl.decode_cache_lengths(c["B"], c["kv_lo"], c["kv_hi"], c["seed"])
    if name == "packed_docs":
        ids = wl.doc_ids_from_lengths(wl.doc_lengths(c["doc_total"], c["doc_lo"], c["doc_hi"], c["seed"]))
        mask["doc_id"] = ids
        score["doc_id"] = ids
    return c, mask, score, kv_len


def _unit(job):
    name, over, b, h = job
    import torch

    import oracle.flex_oracle as o
    import workloads as wl
    c, mask, score, kv_len = workload_specs(name, **over)
    dt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
    G = c["Hq"] // c["Hkv"]
    q = wl.randn_slice(c["seed"], 0, b, h, c["L"], c["E"], dt)
    k = wl.randn_slice(c["seed"], 1, b, h // G, c["S"], c["E"], dt)
    v = wl.randn_slice(c["seed"], 2, b, h // G, c["S"], c["Ev"], dt)
    S_b = c["S"] if kv_len is None else int(kv_len[b])
    if kv_len is not None:
        kk, vv = k[None, None], v[None, None]
        wl.fill_cache_tail(kk, vv, [S_b])
    scale = float(np.float32(c["scale"]))  # the kernel receives an fp32 scale
    out, lse, mx = o.forward_unit(q, k, v, b, h, c["Hq"], S_b, scale, mask, score)
    return (b, h), out, lse, mx


def oracle_units(name, units, workers=None, **over):
    """{(b, h): (out (L, Ev), lse (L,), max_scores (L,))} for the listed units."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    n = workers or max(1, min(len(units), len(os.sched_getaffinity(0))))
    jobs = [(name, over, int(b), int(h)) for b, h in units]
    res = {}
    with ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"), initializer=_init_worker,
                             initargs=(root,)) as ex:
        for key, out, lse, mx in ex.map(_unit, jobs, chunksize=max(1, len(jobs) // (4 * n))):
            res[key] = (out, lse, mx)
    return res
