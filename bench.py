"""Throughput of the FlexAttention hot path on B200: one JSON line on stdout.

A step is one pass of the whole path over one batch of synthetic input: the
BlockMask build (tile classifier) and the forward pass over the listed tiles.
By default every workload runs in turn, each with its own warm-up and timed
steps; the JSON line's headline fields belong to the largest single-GPU
prefill workload (GQA sliding window: B=2, Hq=32, Hkv=8, L=S=16384, E=128,
bf16), and every workload's own numbers are under ``detail.per_config``:

    gqa_sliding_window     headline; tensor roofline
    causal_softcap_alibi   B=4, H=16, L=S=2048, E=64; tensor roofline
    packed_docs            H=16, L=S=8192, E=128; tensor roofline
    decode_kv_cache        B=32, Hq=32, Hkv=8, q_len 4, caches of 4096-32768; HBM roofline
    decode_kv_cache_q1     the same with q_len 1
    fp32_causal_small      fp32, L=S=128, 32 x 32 tiles (a correctness workload, no roofline target)

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload LABEL|all] [--impl reference]

With N > 1 it runs under torchrun, one process per GPU; every rank processes
the same per-GPU workloads (weak scaling: the (batch, head) units shard with
no data-path exchange), times on the device, and rank 0 reports the max over
ranks.  ``--impl reference`` times the fp64 CPU oracle on bounded samples of
the headline workload instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "visible-score TFLOP/s & % BF16 tensor peak (prefill); KV GB/s % HBM (decode)"
METRIC_PREFILL = METRIC
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20

# (label, workload, overrides): the bench items, headline first.
BENCH_ITEMS = [
    ("gqa_sliding_window", "gqa_sliding_window", {}),
    ("causal_softcap_alibi", "causal_softcap_alibi", {}),
    ("packed_docs", "packed_docs", {}),
    ("decode_kv_cache", "decode_kv_cache", {}),
    ("decode_kv_cache_q1", "decode_kv_cache", {"L": 1}),
    ("fp32_causal_small", "fp32_causal_small", {}),
    # the backward pass (dq, dk, dv of sum(out * dout)) of two workloads
    ("backward_causal_softcap_alibi", "causal_softcap_alibi", {"backward": True}),
    ("backward_packed_docs", "packed_docs", {"backward": True}),
    # composed rules at the causal workload's shape: a sliver (every fourth
    # key: every causal tile is partial, the worst case for block sparsity)
    # and a head-dependent rule (half the heads global, half a 256-key window)
    ("sliver_every_fourth_key", "causal_softcap_alibi", {"rule": "every_fourth_key"}),
    ("half_heads_global", "causal_softcap_alibi", {"rule": "half_heads_global"}),
    # the decode workload against a paged cache: 64-key pages in shuffled order
    ("decode_kv_cache_paged", "decode_kv_cache", {"paged": 64}),
]

# Composed rules of the bench items: (rule spec, reads the query head).
RULES = {
    "every_fourth_key": ({"kind": "and", "masks": [{"kind": "causal"}, {"kind": "stride", "value": 4}]}, False),
    "half_heads_global": ({"kind": "and", "masks": [
        {"kind": "causal"},
        {"kind": "or", "masks": [{"kind": "head_below", "value": 8}, {"kind": "distance_below", "value": 256}]}]},
        True),
}
HEADLINE = BENCH_ITEMS[0][0]

# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant
# kernel, from the ncu captures summarised under profiles/, keyed by bench
# label; valid only while that kernel's sources hash to the recorded value
# (the hash ignores comments).  The scaling of each capture to the full
# workload is stated in the profile it comes from.
NCU_TRAFFIC = {
    # fwd_sm100_kernel<128, 0>, captured at batch 1 (profiles/fwd_sm100_gqa_sliding_window.md): x 2 sequences
    "gqa_sliding_window": {"bytes": 2 * (201789696 + 94654464), "source_hash": "e563253dfa69d1e2"},
    # fwd_sm100_kernel<64, 3> / <128, 3>, full size (profiles/fwd_sm100_causal_packed_sliver.md)
    "causal_softcap_alibi": {"bytes": 50418944 + 882688, "source_hash": "e563253dfa69d1e2"},
    "packed_docs": {"bytes": 100893440 + 10517248, "source_hash": "e563253dfa69d1e2"},
    "sliver_every_fourth_key": {"bytes": 50424320 + 783360, "source_hash": "e563253dfa69d1e2"},
    "half_heads_global": {"bytes": 50460928 + 648448, "source_hash": "e563253dfa69d1e2"},
    # decode_tc_kernel<128, 1>, captured at batch 16 (profiles/decode_tc_kernel_decode_kv_cache.md):
    # x 614602 / 296926 cached tokens
    "decode_kv_cache": {"bytes": round((1220940800 + 7898368) * 614602 / 296926), "source_hash": "ffab78b4d4eb3af3"},
    "decode_kv_cache_q1": {"bytes": round((1220451328 + 4600320) * 614602 / 296926),
                           "source_hash": "ffab78b4d4eb3af3"},
    # the same kernel over the shuffled 64-key page pool, at batch 16
    "decode_kv_cache_paged": {"bytes": round((1220960512 + 7605248) * 614602 / 296926),
                              "source_hash": "ffab78b4d4eb3af3"},
    # bwd_dkdv_kernel (the larger of the two backward kernels), full size
    # (profiles/bwd_dkdv_dq_backward.md)
    "backward_causal_softcap_alibi": {"bytes": 68308736 + 7811072, "source_hash": "6a65fba814bf1a59"},
    "backward_packed_docs": {"bytes": 135514112 + 36383488, "source_hash": "6a65fba814bf1a59"},
}

KERNEL_SOURCES = {
    "prefill": ("fwd_sm100.cu", "mods.cuh", "common.cuh", "fastmath.cuh"),
    "decode": ("decode.cu", "mods.cuh", "common.cuh", "fastmath.cuh"),
    "general": ("fwd_simt.cu", "mods.cuh", "common.cuh"),
    "backward": ("bwd_sm100.cu", "mods.cuh", "common.cuh", "fastmath.cuh"),
}


def config_over(over):
    """A bench item's overrides of the workload config (its mode keys removed)."""
    c = {k: v for k, v in over.items() if k not in ("backward", "rule", "paged")}
    if "rule" in over:
        c["mask"] = dict(RULES[over["rule"]][0])
    return c


def kernel_source_hash(kind="prefill"):
    """Hash of the kernel's sources with comments and blank space removed, so
    that only a change to the code itself invalidates recorded counters."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "programmable_block_sparse_b200", "csrc", name)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def item(label):
    for it in BENCH_ITEMS:
        if it[0] == label:
            return it
    raise KeyError(label)


# ---------------------------------------------------------------------------
# Work accounting (exact counts from the workload parameters)
# ---------------------------------------------------------------------------

def visible_counts_rows(c, b, kv_len=None, doc_lengths=None, h=0):
    """Visible keys of every query row of batch b, query head h (int64 array
    of length L)."""
    L, S = c["L"], c["S"]
    kind = c["mask"]["kind"]
    S_b = S if kv_len is None else int(kv_len[b])
    q = np.arange(L, dtype=np.int64) + (S_b - L)
    if kind == "causal":
        n = np.clip(np.minimum(q + 1, S_b), 0, None)
    elif kind == "sliding_window":
        W, ns = c["mask"]["window"], c["mask"].get("n_sink", 0)
        lo = np.maximum(q - W + 1, 0)
        win = np.clip(np.minimum(q, S_b - 1) - lo + 1, 0, None)
        sink = np.clip(np.minimum(np.minimum(ns - 1, q), lo - 1) + 1, 0, None)
        n = win + sink
    elif kind == "document":
        starts = np.repeat(np.concatenate([[0], np.cumsum(doc_lengths)[:-1]]), doc_lengths)
        n = q - starts[q] + 1
    elif c["mask"] == RULES["every_fourth_key"][0]:
        # keys kv <= q with kv = q (mod 4): q // 4 + 1 of them (S_b = S here)
        n = np.where(q >= 0, q // 4 + 1, 0)
    elif c["mask"] == RULES["half_heads_global"][0]:
        # heads below 8 see every earlier key, the others the last 256
        n = np.clip(np.minimum(q + 1, S_b), 0, None)
        if h >= 8:
            n = np.minimum(n, 256)
    else:
        raise ValueError(kind)
    return n


def visible_pairs_all_heads(c, kv_len=None, doc_lengths=None):
    """Visible pairs over every (b, h); a head-dependent rule counts per head."""
    if c["mask"] == RULES["half_heads_global"][0]:
        return sum(int(visible_counts_rows(c, b, kv_len, doc_lengths, h).sum())
                   for b in range(c["B"]) for h in range(c["Hq"]))
    return visible_pairs_per_head(c, kv_len, doc_lengths) * c["Hq"]


def visible_pairs_per_head(c, kv_len=None, doc_lengths=None):
    """Visible (query, key) pairs for one (b, h), summed over the batch."""
    return int(sum(int(visible_counts_rows(c, b, kv_len, doc_lengths).sum()) for b in range(c["B"])))


def visited_cells(bm):
    """Cells of all listed tiles (clipped to L x S), summed over B x H of the mask."""
    kvn = bm.kv_num_blocks.cpu().numpy()
    fn = bm.full_kv_num_blocks.cpu().numpy()
    kvi = bm.kv_indices.cpu().numpy()
    fi = bm.full_kv_indices.cpu().numpy()
    rows = np.minimum(bm.BM, bm.L - np.arange(bm.Mb) * bm.BM)
    cols = np.minimum(bm.BN, bm.S - np.arange(bm.Nb) * bm.BN)
    tot = 0
    for b in range(bm.B):
        for h in range(bm.H):
            for m in range(bm.Mb):
                c = cols[kvi[b, h, m, :kvn[b, h, m]]].sum() + cols[fi[b, h, m, :fn[b, h, m]]].sum()
                tot += int(rows[m] * c)
    return tot


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# Workload set-up
# ---------------------------------------------------------------------------

def describe(name, c):
    keys = ["B", "Hq", "Hkv", "L", "S", "E", "Ev", "dtype", "BM", "BN"]
    d = {k: c[k] for k in keys}
    d["mask"] = {k: v for k, v in c["mask"].items()}
    d["score"] = {k: v for k, v in c["score"].items()}
    return f"{name}", d


def make_inputs(name, device, seed_offset=0, batch=None, **over):
    import torch
    c = wl.config(name, **over)
    if batch:
        c["B"] = int(batch)
    kv_len = doc_lengths = None
    if name == "decode_kv_cache":
        kv_len = wl.decode_cache_lengths(c["B"], c["kv_lo"], c["kv_hi"], c["seed"])
    if name == "packed_docs":
        doc_lengths = wl.doc_lengths(c["doc_total"], c["doc_lo"], c["doc_hi"], c["seed"])
    dt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
    q, k, v = wl.randn_qkv(c["B"], c["Hq"], c["Hkv"], c["L"], c["S"], c["E"], c["Ev"], seed=c["seed"] + seed_offset,
                           dtype=dt)
    if kv_len is not None:
        wl.fill_cache_tail(k, v, kv_len)
    mask = dict(c["mask"])
    score = {k_: v_ for k_, v_ in c["score"].items() if k_ != "pos"}
    if doc_lengths is not None:
        ids = wl.doc_ids_from_lengths(doc_lengths)
        mask["doc_id"] = torch.from_numpy(ids).to(device).reshape(1, -1)
        if c["score"].get("pos") == "in_doc":
            score["pos"] = torch.from_numpy(wl.in_doc_positions(doc_lengths)).to(device).reshape(1, -1)
    if kv_len is not None:
        mask["kv_len"] = torch.from_numpy(kv_len).to(device)
    return c, (q, k, v), mask, score, kv_len, doc_lengths


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

class OracleSampler:
    """Bounded samples of a workload evaluated by the fp64 oracle.

    A sample is a block of query rows of one (batch, query head) unit -- all
    L rows for decode, else about 2^21 / S rows -- computed in full by the
    oracle's row function from slices regenerated for that unit (outside the
    timing).  Work per block: visible-pair FLOPs (2E + 2Ev per pair) for
    prefill, or the unit's share of its KV head's valid cache bytes for decode.
    """

    def __init__(self, name, backward=False, **over):
        import torch
        self.name = name
        self.backward = backward
        self.c = c = wl.config(name, **over)
        self.kv_len = self.doc_lengths = None
        if name == "decode_kv_cache":
            self.kv_len = wl.decode_cache_lengths(c["B"], c["kv_lo"], c["kv_hi"], c["seed"])
        if name == "packed_docs":
            self.doc_lengths = wl.doc_lengths(c["doc_total"], c["doc_lo"], c["doc_hi"], c["seed"])
        self.mask, self.score = dict(c["mask"]), dict(c["score"])
        if self.doc_lengths is not None:
            ids = wl.doc_ids_from_lengths(self.doc_lengths)
            self.mask["doc_id"] = ids
            self.score["doc_id"] = ids
        self.dt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
        self.decode = name == "decode_kv_cache"
        self.rows = c["L"] if self.decode else max(1, min(c["L"], (1 << 21) // c["S"]))
        self.blocks_per_unit = -(-c["L"] // self.rows)
        self.units = c["B"] * c["Hq"]
        self.counts = {}
        self.unit_desc = ("one (batch, query head) unit, all its query rows" if self.decode else
                          f"a block of {self.rows} query rows of one (batch, query head) unit, every row in full")
        if backward:
            self.unit_desc += " (the backward: dq of the rows and their parts of dk, dv)"

    def block(self, i):
        """(work, seconds) of the i-th sample; samples are spread over units and rows."""
        import torch

        import oracle.flex_oracle as o
        c = self.c
        total = self.units * self.blocks_per_unit
        j = (i * 7919) % total
        unit, blk = divmod(j, self.blocks_per_unit)
        b, h = divmod(unit, c["Hq"])
        G = c["Hq"] // c["Hkv"]
        q = wl.randn_slice(c["seed"], 0, b, h, c["L"], c["E"], self.dt)
        k = wl.randn_slice(c["seed"], 1, b, h // G, c["S"], c["E"], self.dt)
        v = wl.randn_slice(c["seed"], 2, b, h // G, c["S"], c["Ev"], self.dt)
        S_b = c["S"] if self.kv_len is None else int(self.kv_len[b])
        if self.kv_len is not None:
            wl.fill_cache_tail(k[None, None], v[None, None], [S_b])
        r0, r1 = blk * self.rows, min(c["L"], (blk + 1) * self.rows)
        qn = q[r0:r1].to(torch.float64).numpy()
        kn = k.to(torch.float64).numpy()
        vn = v.to(torch.float64).numpy()
        qp = o.query_positions(c["L"], S_b)[r0:r1]
        if self.backward:
            don = wl.randn_slice(c["seed"], 3, b, h, c["L"], c["Ev"], self.dt)[r0:r1].to(torch.float64).numpy()
            t0 = time.perf_counter()
            o.backward_rows(qn, kn, vn, don, c["scale"], self.mask, self.score, b, h, qp, S_b, c["Hq"])
            el = time.perf_counter() - t0
            return float(self.visible(b, h)[r0:r1].sum()) * (6 * c["E"] + 4 * c["Ev"]), el
        t0 = time.perf_counter()
        o.attention_rows(qn, kn, vn, c["scale"], self.mask, self.score, b, h, qp, S_b, c["Hq"])
        el = time.perf_counter() - t0
        if self.decode:
            work = S_b * (c["E"] + c["Ev"]) * 2 / G
        else:
            work = float(self.visible(b, h)[r0:r1].sum()) * (2 * c["E"] + 2 * c["Ev"])
        return work, el

    def visible(self, b, h):
        """Visible keys per query row of unit (b, h) (cached)."""
        key = (b, h if self.c["mask"] == RULES["half_heads_global"][0] else 0)
        if key not in self.counts:
            self.counts[key] = visible_counts_rows(self.c, b, self.kv_len, self.doc_lengths, key[1])
        return self.counts[key]

    def rate(self, target_s):
        """(rate, seconds, samples) running samples until ~target_s of oracle time."""
        work = el = 0.0
        n = 0
        while el < target_s or n == 0:
            w, t = self.block(n)
            work += w
            el += t
            n += 1
        scale = 1e9 if self.decode else 1e12
        return work / el / scale, el, n

    @property
    def unit(self):
        return "GB/s" if self.decode else "TFLOP/s"


def cpu_baseline(label, target_s):
    _, name, over = item(label)
    s = OracleSampler(name, backward=over.get("backward", False), **config_over(over))
    rate, el, n = s.rate(target_s)
    return {"value": rate, "unit": s.unit, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"{n} samples of {s.unit_desc}, spread over the workload's units and rows", "seconds": el}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    label = HEADLINE if args.workload == "all" else args.workload
    _, name, over = item(label)
    c = wl.config(name, **config_over(over))
    s = OracleSampler(name, backward=over.get("backward", False), **config_over(over))
    for i in range(args.warmup):
        s.block(i)
    times, works = [], []
    for i in range(args.steps):
        w, t = s.block(args.warmup + i)
        works.append(w)
        times.append(t)
    scale = 1e9 if s.decode else 1e12
    value = sum(works) / sum(times) / scale
    cores = len(os.sched_getaffinity(0))
    sample = f"each step: {s.unit_desc}, spread over the workload's units and rows"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": s.unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": label, **describe(name, c)[1], "sample": sample},
        "cpu_baseline": {"value": value, "unit": s.unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": s.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# Multi-rank plumbing (one process per GPU; no collective on the data path)
# ---------------------------------------------------------------------------

def dist_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value, device, world):
    """The largest of every rank's ``value`` (a device time in ms): the job's time."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(work_per_rank, world, ms_per_step, scale):
    """Weak scaling: every rank does ``work_per_rank`` per step; the job's rate
    is all ranks' work over the slowest rank's step time, in units of ``scale``."""
    return world * work_per_rank / (ms_per_step * 1e-3) / scale


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class Workload:
    """One bench item on the device: inputs, block mask, outputs, work counts."""

    def __init__(self, label, dev, rank, batch=None):
        import torch
        import programmable_block_sparse_b200 as fa
        self.fa = fa
        self.label = label
        _, self.name, over = item(label)
        self.backward = over.get("backward", False)
        (self.c, (self.q_h, self.k_h, self.v_h), self.mask, self.score, self.kv_len,
         self.doc_lengths) = make_inputs(self.name, dev, seed_offset=rank, batch=batch, **config_over(over))
        c = self.c
        self.B_mask = c["B"] if self.kv_len is not None else 1
        # a rule that reads the query head needs a block mask per head
        self.H_mask = c["Hq"] if over.get("rule") and RULES[over["rule"]][1] else 1
        self.gqa = c["Hq"] != c["Hkv"]
        self.q, self.k, self.v = self.q_h.to(dev), self.k_h.to(dev), self.v_h.to(dev)
        self.paged = None
        if over.get("paged"):
            # the cache as a pool of pages in a seeded shuffled order, and its page table
            P = int(over["paged"])
            B, Hkv, S = c["B"], c["Hkv"], c["S"]
            npg = S // P
            perm = torch.randperm(B * npg, generator=torch.Generator().manual_seed(c["seed"] + 7)).to(dev)

            def pool(t):
                pages = t.view(B, Hkv, npg, P, t.shape[-1]).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, P,
                                                                                           t.shape[-1])
                out = torch.empty_like(pages)
                out[perm] = pages
                return out
            self.k, self.v = pool(self.k), pool(self.v)
            self.k_h, self.v_h = self.k.cpu(), self.v.cpu()  # the host copies the end-to-end leg sends
            self.paged = {"page_table": perm.view(B, npg).to(torch.int32), "page_size": P}
        self.out = torch.empty((c["B"], c["Hq"], c["L"], c["Ev"]), dtype=self.q.dtype, device=dev)
        self.lse = torch.empty((c["B"], c["Hq"], c["L"]), dtype=torch.float32, device=dev)
        self.bm = fa.flexattn_build_block_mask(self.mask, self.B_mask, self.H_mask, c["L"], c["S"], c["BM"], c["BN"],
                                               device=dev)
        ws = fa.flexattn_forward_workspace_size(self.q, self.k, self.v, self.bm, paged=self.paged)
        self.ws_bytes = ws
        self.ws = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev)
        self.decode = self.name == "decode_kv_cache"
        self.general = c["dtype"] != "bf16" or c["BM"] != 128
        # classifier + forward kernel, + the log-sum-exp combine when decode splits the keys
        self.launches_per_step = 2 + (1 if self.decode and ws > 0 else 0)
        fp = 2 * c["E"] + 2 * c["Ev"]
        self.vis_flops = visible_pairs_all_heads(c, self.kv_len, self.doc_lengths) * fp
        cells = visited_cells(self.bm) * (c["Hq"] if self.bm.H == 1 else 1) * (c["B"] if self.bm.B == 1 else 1)
        self.visited_cells = cells
        self.visited_flops = cells * fp
        self.kv_bytes = (int(np.sum(self.kv_len)) * c["Hkv"] * (c["E"] + c["Ev"]) * self.q.element_size()
                         if self.decode else None)
        if self.backward:
            # the forward's out and lse once, then the backward is the timed call:
            # the query-side lists (as the block-mask step) and the gradients
            self.forward_call()
            self.dout = wl.randn_dout(c["B"], c["Hq"], c["L"], c["Ev"], seed=c["seed"] + rank).to(dev)
            self.q_side = fa.flexattn_transpose_block_mask(self.bm)
            self.grads = tuple(torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (self.q, self.k, self.v))
            self.bwd_ws = torch.empty(c["B"] * c["Hq"] * c["L"] * 4, dtype=torch.uint8, device=dev)
            self.launches_per_step = 4  # query-side lists, D = rowsum(dout * out), dk / dv, dq
            bf = 6 * c["E"] + 4 * c["Ev"]  # five products per cell: S, dP, dV, dK, dQ
            self.vis_flops = self.vis_flops // fp * bf
            self.visited_flops = cells * bf

    def build(self):
        c = self.c
        if self.backward:
            self.fa.flexattn_transpose_block_mask(self.bm, out=self.q_side)
            return
        self.fa.flexattn_build_block_mask(self.mask, self.B_mask, self.H_mask, c["L"], c["S"], c["BM"], c["BN"],
                                          out=self.bm)

    def forward_call(self):
        self.fa.flexattn_forward(self.q, self.k, self.v, self.bm, score_mod=self.score, mask_mod=self.mask,
                                 scale=self.c["scale"], enable_gqa=self.gqa, out=self.out, lse=self.lse,
                                 workspace=self.ws, paged=self.paged)

    def forward(self):
        """The timed call: the forward, or for a backward item the backward."""
        if not self.backward:
            return self.forward_call()
        dq, dk, dv = self.grads
        self.fa.flexattn_backward(self.q, self.k, self.v, self.out, self.dout, self.lse, self.bm, q_side=self.q_side,
                                  score_mod=self.score, mask_mod=self.mask, scale=self.c["scale"],
                                  enable_gqa=self.gqa, dq=dq, dk=dk, dv=dv, workspace=self.bwd_ws)

    def step(self):
        self.build()
        self.forward()

    def capture_graphs(self):
        """CUDA graphs of the two calls, used only after a replay into cleared
        outputs and a sentinel-filled block mask reproduces the eager result
        (block mask bit for bit, out within 1e-2, lse within 1e-3)."""
        import torch
        fa = self.fa
        if self.backward:
            return self._capture_backward()
        try:
            out_ref, lse_ref = self.out.float().clone(), self.lse.clone()
            bm_ref = [t.clone() for t in (self.bm.kv_num_blocks, self.bm.kv_indices, self.bm.full_kv_num_blocks,
                                          self.bm.full_kv_indices)]
            g_mask, g_fwd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_mask, capture_error_mode="relaxed"):
                self.build()
            with torch.cuda.graph(g_fwd, capture_error_mode="relaxed"):
                self.forward()
            for t in (self.bm.kv_num_blocks, self.bm.kv_indices, self.bm.full_kv_num_blocks,
                      self.bm.full_kv_indices):
                t.fill_(-1)
            self.out.zero_()
            self.lse.zero_()
            g_mask.replay()
            g_fwd.replay()
            torch.cuda.synchronize()
            same_mask = all(torch.equal(a, b) for a, b in zip(bm_ref, (self.bm.kv_num_blocks, self.bm.kv_indices,
                                                                       self.bm.full_kv_num_blocks,
                                                                       self.bm.full_kv_indices)))
            fin = torch.isfinite(lse_ref)
            same = (same_mask and torch.equal(fin, torch.isfinite(self.lse))
                    and (self.out.float() - out_ref).abs().max().item() <= 1e-2
                    and (self.lse[fin] - lse_ref[fin]).abs().max().item() <= 1e-3)
            if same and fa.flexattn_poll_device_status() == 0:
                return (g_mask, g_fwd), "CUDA graph replay, one graph per call"
            return None, "eager (graph replay did not reproduce the eager result)"
        except Exception as exc:  # capture unsupported here: keep the eager launches
            torch.cuda.synchronize()
            return None, f"eager (graph capture failed: {type(exc).__name__})"


def _capture_backward(self):
    """Graphs of the two backward calls, used only when a replay into cleared
    query-side lists and gradients reproduces the eager result bit for bit
    (the backward kernels write every gradient once, in a fixed order)."""
    import torch
    fa = self.fa
    try:
        qs = self.q_side
        lists = (qs.q_num_blocks, qs.q_indices, qs.full_q_num_blocks, qs.full_q_indices)
        ref = [t.clone() for t in lists + self.grads]
        g_lists, g_bwd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_lists, capture_error_mode="relaxed"):
            self.build()
        with torch.cuda.graph(g_bwd, capture_error_mode="relaxed"):
            self.forward()
        for t in lists:
            t.fill_(-1)
        for t in self.grads:
            t.zero_()
        g_lists.replay()
        g_bwd.replay()
        torch.cuda.synchronize()
        same = all(torch.equal(a, b) for a, b in zip(ref, lists + self.grads))
        if same and fa.flexattn_poll_device_status() == 0:
            return (g_lists, g_bwd), "CUDA graph replay, one graph per call"
        return None, "eager (graph replay did not reproduce the eager result)"
    except Exception as exc:
        torch.cuda.synchronize()
        return None, f"eager (graph capture failed: {type(exc).__name__})"


Workload._capture_backward = _capture_backward


def measure(wk, args, dev, world, flush, peaks, peak_src):
    """Warm-up, then K device-timed steps; numbers of one workload."""
    import torch
    import torch.distributed as dist
    fa = wk.fa
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        wk.step()
        flush.zero_()
    torch.cuda.synchronize()
    if fa.flexattn_poll_device_status() != 0:
        raise RuntimeError(f"{wk.label}: device status word set during warm-up")
    graphs, launch = (None, "eager") if args.eager else wk.capture_graphs()
    # the step (block-mask build + timed call) as one graph: its replay times
    # the step; the two per-call graphs time each part
    g_step = None
    if graphs:
        try:
            outs = wk.grads if wk.backward else (wk.out, wk.lse)
            ref = [t.clone() for t in outs]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="relaxed"):
                wk.build()
                wk.forward()
            for t in outs:
                t.zero_()
            g.replay()
            torch.cuda.synchronize()
            if all(torch.equal(a, b) for a, b in zip(ref, outs)) and fa.flexattn_poll_device_status() == 0:
                g_step = g
                launch = "CUDA graph replay: one graph per step (one per call for the split timings)"
        except Exception:  # keep the per-call graphs for the step as well
            torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        time.sleep(0.25)  # let the sampler start
        for i in range(args.steps):
            e0, e1, e2 = ev[i]
            e0.record(stream)
            if graphs:
                graphs[0].replay()
            else:
                wk.build()
            e1.record(stream)
            if graphs:
                graphs[1].replay()
            else:
                wk.forward()
            e2.record(stream)
            flush.zero_()
        step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)] if g_step else []
        for s0, s1 in step_ev:
            s0.record(stream)
            g_step.replay()
            s1.record(stream)
            flush.zero_()
        torch.cuda.synchronize()
        time.sleep(0.15)
    if world > 1:
        dist.barrier()
    mask_ms = [a.elapsed_time(b) for a, b, _ in ev]
    fwd_ms = [b.elapsed_time(c_) for _, b, c_ in ev]
    step_ms = ([a.elapsed_time(b) for a, b in step_ev] if step_ev else
               [a.elapsed_time(c_) for a, _, c_ in ev])
    total_ms = max_over_ranks(sum(step_ms), dev, world)
    if fa.flexattn_poll_device_status() != 0:
        raise RuntimeError(f"{wk.label}: device status word set during the timed region")
    del graphs, g_step

    ms_per_step = total_ms / args.steps
    fwd_mean = statistics.mean(fwd_ms)
    c = wk.c
    r = {"workload": wk.label, "config": describe(wk.name, c)[1], "launch": launch,
         "ms_per_step": ms_per_step, "forward_ms": fwd_mean, "forward_ms_median": statistics.median(fwd_ms),
         "block_mask_ms": statistics.mean(mask_ms), "gpu_launches": wk.launches_per_step * args.steps,
         "clocks": clocks.summary()}
    if wk.backward:
        r["step"] = "query-side lists + backward (dq, dk, dv in bf16)"
        r["backward_ms"] = r.pop("forward_ms")
        r["backward_ms_median"] = r.pop("forward_ms_median")
        r["transpose_ms"] = r.pop("block_mask_ms")
        r["value"] = whole_job_rate(wk.vis_flops, world, ms_per_step, 1e12)
        r["unit"] = "TFLOP/s"
        achieved = wk.visited_flops / (fwd_mean * 1e-3) / 1e12
        r["roofline"] = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "peak_source": f"bf16_tflops (burst) of {peak_src}",
                         "flops_counted_over": "visited-tile cells, (6E + 4Ev) per cell: S, dP, dV, dK, dQ"}
        r["visible_pairs_flops"] = wk.vis_flops
        r["visited_cells"] = wk.visited_cells
        kind = "backward"
    elif wk.decode:
        r["value"] = whole_job_rate(wk.kv_bytes, world, ms_per_step, 1e9)
        r["unit"] = "GB/s"
        achieved = wk.kv_bytes / (fwd_mean * 1e-3) / 1e9
        r["roofline"] = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "peak_source": f"hbm_gbs of {peak_src}",
                         "frac_of_8000_gbs": achieved / 8000.0,
                         "bytes_counted": "valid KV cache, sum_b len_b * Hkv * (E + Ev) * 2 B"}
        r["kv_bytes"] = wk.kv_bytes
        kind = "decode"
    else:
        r["value"] = whole_job_rate(wk.vis_flops, world, ms_per_step, 1e12)
        r["unit"] = "TFLOP/s"
        achieved = wk.visited_flops / (fwd_mean * 1e-3) / 1e12
        if wk.general:
            r["roofline"] = None
            kind = "general"
        else:
            r["roofline"] = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                             "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                             "peak_source": f"bf16_tflops (burst) of {peak_src}",
                             "flops_counted_over": "visited-tile cells, (2E + 2Ev) per cell"}
            kind = "prefill"
        r["visible_pairs_flops"] = wk.vis_flops
        r["visited_cells"] = wk.visited_cells
        r["visible_tflops_forward_only"] = wk.vis_flops / (fwd_mean * 1e-3) / 1e12
        r["visited_tflops_forward_only"] = achieved
    src_hash = kernel_source_hash(kind)
    r["kernel_source"] = src_hash
    if r["roofline"] is not None:
        tr = NCU_TRAFFIC.get(wk.label)
        r["roofline"]["traffic"] = tr["bytes"] if tr and tr["source_hash"] == src_hash and not args.batch else None
    return r


def measure_e2e(wk, args, dev, world, flush):
    """The same metric through the public Python API, with pinned-host inputs
    copied in and out / lse read back inside the timed region of every step.
    Steps alternate between two streams, each with its own device buffers, so
    that one step's device-to-host copy (one copy engine) runs while the next
    step's host-to-device copy (the other) does; the timed region runs from
    before the first step's input copy to after the last step's read-back.
    The inputs are larger than L2, so no flush runs between steps."""
    import copy
    import torch
    fa = wk.fa
    twin = copy.copy(wk)  # second device buffers; the rule tensors are read-only and shared
    twin.q, twin.k, twin.v = torch.empty_like(wk.q), torch.empty_like(wk.k), torch.empty_like(wk.v)
    twin.out, twin.lse = torch.empty_like(wk.out), torch.empty_like(wk.lse)
    c = wk.c
    twin.bm = fa.flexattn_build_block_mask(wk.mask, wk.B_mask, wk.H_mask, c["L"], c["S"], c["BM"], c["BN"], device=dev)
    twin.ws = torch.empty_like(wk.ws)
    sets = (wk, twin)
    streams = (torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev))
    q_p, k_p, v_p = wk.q_h.pin_memory(), wk.k_h.pin_memory(), wk.v_h.pin_memory()
    outs = [(torch.empty(wk.out.shape, dtype=wk.out.dtype).pin_memory(),
             torch.empty(wk.lse.shape, dtype=wk.lse.dtype).pin_memory()) for _ in sets]
    n = max(4, min(args.steps, 20))

    def step(i):
        w, st = sets[i % 2], streams[i % 2]
        with torch.cuda.stream(st):
            w.q.copy_(q_p, non_blocking=True)
            w.k.copy_(k_p, non_blocking=True)
            w.v.copy_(v_p, non_blocking=True)
            w.step()
            outs[i % 2][0].copy_(w.out, non_blocking=True)
            outs[i % 2][1].copy_(w.lse, non_blocking=True)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    main = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for st in streams:
        st.wait_event(e0)
    for i in range(n):
        step(i)
    for st in streams:
        done = torch.cuda.Event()
        done.record(st)
        main.wait_event(done)
    e1.record(main)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n, dev, world)
    # the read-back must be the result of the call
    if not (torch.equal(outs[(n - 1) % 2][0], wk.out.cpu()) and torch.equal(outs[(n - 1) % 2][1], wk.lse.cpu())):
        raise RuntimeError("end-to-end leg: read-back differs from the device result")
    h2d = sum(t.numel() * t.element_size() for t in (wk.q, wk.k, wk.v))
    d2h = wk.out.numel() * wk.out.element_size() + wk.lse.numel() * wk.lse.element_size()
    work, scale, unit = ((wk.kv_bytes, 1e9, "GB/s") if wk.decode else (wk.vis_flops, 1e12, "TFLOP/s"))
    return {"value": whole_job_rate(work, world, e2e_ms, scale), "unit": unit, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "overlap": "two streams alternate steps: a step's read-back overlaps the next step's input copy"}


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import programmable_block_sparse_b200 as fa

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    fa.load_library()
    peaks, peak_src = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    labels = [it[0] for it in BENCH_ITEMS] if args.workload == "all" else [args.workload]
    head = labels[0]
    per, e2e = {}, None
    for label in labels:
        wk = Workload(label, dev, rank, batch=args.batch)
        per[label] = measure(wk, args, dev, world, flush, peaks, peak_src)
        if label == head:
            e2e = measure_e2e(wk, args, dev, world, flush)
        del wk
        torch.cuda.empty_cache()

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    if not args.no_cpu_baseline and world == 1:
        for label in labels:
            per[label]["cpu_baseline"] = cpu_baseline(label, args.cpu_seconds if label == head else
                                                      args.cpu_seconds_other)
    h = per[head]
    _, hname, hover = item(head)
    hc = wl.config(hname, **config_over(hover))
    line = {
        "metric": METRIC, "value": h["value"], "unit": h["unit"], "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": h["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if hc["dtype"] == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": head, **describe(hname, hc)[1],
                   "l2": "flushed: 256 MiB written between timed steps, outside the events",
                   "step": "block-mask build + forward", "launch": h["launch"],
                   "parallelism": f"weak scaling over {world} GPU(s): each rank runs the full per-GPU workloads",
                   "workloads_run": labels},
        "roofline": h["roofline"],
        "detail": {"headline": head, "per_config": per},
        "e2e": e2e,
        "gpu_launches": h["gpu_launches"],
        "clocks": h["clocks"],
    }
    if "cpu_baseline" in h:
        line["cpu_baseline"] = h["cpu_baseline"]
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="all", choices=["all"] + [it[0] for it in BENCH_ITEMS],
                    help="one bench item (it becomes the headline), or all of them (default)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle seconds for the headline's cpu_baseline")
    ap.add_argument("--cpu-seconds-other", type=float, default=3.0,
                    help="oracle seconds for each other workload's cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed calls directly instead of replaying CUDA graphs of them")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workloads' batch size (smaller captures for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
