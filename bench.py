"""Throughput of the FlexAttention hot path on B200: one JSON line on stdout.

A step is one pass of the whole path over one batch of synthetic input: the
BlockMask build (tile classifier) and the forward pass over the listed tiles.
The default workload is the causal + soft-cap(50) + ALiBi prefill
(B=4, H=16, L=S=2048, E=64, bf16, 128 x 128 tiles).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

With N > 1 it runs under torchrun, one process per GPU; every rank processes
the same per-GPU workload (weak scaling: the (batch, head) units shard with no
data-path exchange), times on the device, and rank 0 reports the max over ranks.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import re
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC_PREFILL = "visible-score TFLOP/s & % BF16 tensor peak (prefill); KV GB/s % HBM (decode)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20

# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant
# kernel, from the ncu captures summarised under profiles/, keyed by workload;
# valid only while that kernel's sources hash to the recorded value.
#  - causal_softcap_alibi: fwd_sm100_kernel, full workload, one launch
#    (50.414848 MB read + 0.630272 MB written).
#  - gqa_sliding_window: fwd_sm100_kernel captured at batch 1 (201.801472 MB
#    read + 100.076544 MB written), doubled for the batch of 2: both
#    sequences carry the same work.
#  - decode_kv_cache: decode_kernel captured at batch 16 (1220.765 MB read +
#    12.79872 MB written over 296926 cached tokens), scaled to the full batch
#    of 32 by cached tokens (614602): traffic grows with the tokens streamed.
NCU_TRAFFIC = {
    "causal_softcap_alibi": {"bytes": 51045120, "source_hash": "3a07580eec5ff9d8"},
    "gqa_sliding_window": {"bytes": 603756032, "source_hash": "3a07580eec5ff9d8"},
    "decode_kv_cache": {"bytes": 2553332243, "source_hash": "da0da3a8d76e9df9"},
}

KERNEL_SOURCES = {
    "prefill": ("fwd_sm100.cu", "mods.cuh", "common.cuh"),
    "decode": ("decode.cu", "mods.cuh", "common.cuh"),
}


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


# ---------------------------------------------------------------------------
# Work accounting (exact counts from the workload parameters)
# ---------------------------------------------------------------------------

def visible_pairs_per_head(c, kv_len=None, doc_lengths=None):
    """Visible (query, key) pairs for one (b, h), summed over the batch."""
    L, S = c["L"], c["S"]
    kind = c["mask"]["kind"]
    total = 0
    for b in range(c["B"]):
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
        else:
            raise ValueError(kind)
        total += int(n.sum())
    return total


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


def make_inputs(name, device, seed_offset=0, batch=None):
    import torch
    c = wl.config(name)
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

def oracle_sample_rate(name, target_s=12.0, max_heads=None):
    """Run the fp64 oracle on whole (b, h) units until ~target_s of oracle time.

    Inputs are the workload's own seeded slices (regenerated per unit, outside
    the timing).  Returns (rate, seconds, cores, sample description, units
    done, unit): visible-pair FLOP/s (prefill) or KV bytes/s (decode: each
    query head's share of its KV head's valid cache).
    """
    import torch

    import oracle.flex_oracle as o
    c = wl.config(name)
    kv_len = doc_lengths = None
    if name == "decode_kv_cache":
        kv_len = wl.decode_cache_lengths(c["B"], c["kv_lo"], c["kv_hi"], c["seed"])
    if name == "packed_docs":
        doc_lengths = wl.doc_lengths(c["doc_total"], c["doc_lo"], c["doc_hi"], c["seed"])
    mask = dict(c["mask"])
    score = dict(c["score"])
    if doc_lengths is not None:
        ids = wl.doc_ids_from_lengths(doc_lengths)
        mask["doc_id"] = ids
        score["doc_id"] = ids
    dt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
    G = c["Hq"] // c["Hkv"]
    flop_pair = 2 * c["E"] + 2 * c["Ev"]
    per_head_pairs = visible_pairs_per_head(c, kv_len, doc_lengths) / c["B"]
    decode = name == "decode_kv_cache"
    el = 0.0
    heads = 0
    work = 0.0
    b = h = 0
    while True:
        qs = wl.randn_slice(c["seed"], 0, b, h, c["L"], c["E"], dt)[None, None]
        ks = wl.randn_slice(c["seed"], 1, b, h // G, c["S"], c["E"], dt)[None, None]
        vs = wl.randn_slice(c["seed"], 2, b, h // G, c["S"], c["Ev"], dt)[None, None]
        sub_kv = None
        if kv_len is not None:
            sub_kv = kv_len[b:b + 1]
            wl.fill_cache_tail(ks, vs, sub_kv)
        t0 = time.perf_counter()
        o.forward(qs, ks, vs, c["scale"], mask, score, kv_len=sub_kv)
        el += time.perf_counter() - t0
        heads += 1
        if decode:
            work += int(kv_len[b]) * (c["E"] + c["Ev"]) * 2 / G
        else:
            work += per_head_pairs * flop_pair
        h = (h + 1) % c["Hq"]
        b = (b + (h == 0)) % c["B"]
        if el >= target_s or (max_heads and heads >= max_heads):
            break
    cores = len(os.sched_getaffinity(0))
    units = c["B"] * c["Hq"]
    if heads <= units:
        sample = f"{heads} of the {units} (batch, query head) units, every query row in full"
    else:
        sample = (f"{heads} (batch, query head) unit evaluations, cycling over all {units} units "
                  f"({heads / units:.2f} passes), every query row in full")
    if decode:
        return work / el / 1e9, el, cores, sample, heads, "GB/s"
    return work / el / 1e12, el, cores, sample, heads, "TFLOP/s"


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    name = args.workload
    c = wl.config(name)
    for _ in range(args.warmup):
        oracle_sample_rate(name, target_s=0.0, max_heads=1)
    times, rates = [], []
    unit, cores = "TFLOP/s", len(os.sched_getaffinity(0))
    for _ in range(args.steps):
        rate, el, cores, _, _, unit = oracle_sample_rate(name, target_s=0.0, max_heads=1)
        times.append(el)
        rates.append(rate)
    value = statistics.mean(rates)
    sample = "one (batch, query head) unit of the workload per step, every query row in full"
    line = {
        "impl": "reference", "metric": METRIC_PREFILL, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": name, **describe(name, c)[1], "sample": sample},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
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

    name = args.workload
    c, (q_h, k_h, v_h), mask, score, kv_len, doc_lengths = make_inputs(name, dev, seed_offset=rank, batch=args.batch)
    B, Hq, L, E, Ev = c["B"], c["Hq"], c["L"], c["E"], c["Ev"]
    BM, BN = c["BM"], c["BN"]
    B_mask = B if kv_len is not None else 1
    gqa = c["Hq"] != c["Hkv"]
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty((B, Hq, L, Ev), dtype=q.dtype, device=dev)
    lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
    bm = fa.flexattn_build_block_mask(mask, B_mask, 1, L, c["S"], BM, BN, device=dev)
    ws_bytes = fa.flexattn_forward_workspace_size(q, k, v, bm)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    decode = name == "decode_kv_cache"
    # classifier + forward kernel, + the log-sum-exp combine when decode splits the keys
    launches_per_step = 2 + (1 if decode and ws_bytes > 0 else 0)
    flop_pair = 2 * E + 2 * Ev
    vis_pairs = visible_pairs_per_head(c, kv_len, doc_lengths) * Hq
    vis_flops = vis_pairs * flop_pair
    cells = visited_cells(bm) * (Hq if bm.H == 1 else 1) * (B if bm.B == 1 else 1)
    visited_flops = cells * flop_pair
    kv_bytes = None
    if decode:
        kv_bytes = int(np.sum(kv_len)) * c["Hkv"] * (E + Ev) * q.element_size()

    def step():
        fa.flexattn_build_block_mask(mask, B_mask, 1, L, c["S"], BM, BN, out=bm)
        fa.flexattn_forward(q, k, v, bm, score_mod=score, mask_mod=mask, scale=c["scale"], enable_gqa=gqa,
                            out=out, lse=lse, workspace=ws)

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step()
        flush.zero_()
    torch.cuda.synchronize()
    if fa.flexattn_poll_device_status() != 0:
        raise RuntimeError("device status word set during warm-up")

    # The step's two calls are captured into CUDA graphs (one per call, so
    # the events can split them) and replayed, as a serving loop would: the
    # launches then carry no host overhead.  A graph is used only after its
    # replay reproduces the eager result; otherwise the calls run eagerly.
    launch = "eager"
    graphs = None
    if not args.eager:
        try:
            out_ref, lse_ref = out.float().clone(), lse.clone()
            g_mask, g_fwd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_mask, capture_error_mode="relaxed"):
                fa.flexattn_build_block_mask(mask, B_mask, 1, L, c["S"], BM, BN, out=bm)
            with torch.cuda.graph(g_fwd, capture_error_mode="relaxed"):
                fa.flexattn_forward(q, k, v, bm, score_mod=score, mask_mod=mask, scale=c["scale"], enable_gqa=gqa,
                                    out=out, lse=lse, workspace=ws)
            out.zero_()
            lse.zero_()
            g_mask.replay()
            g_fwd.replay()
            torch.cuda.synchronize()
            fin = torch.isfinite(lse_ref)
            same = (torch.equal(fin, torch.isfinite(lse)) and (out.float() - out_ref).abs().max().item() <= 1e-2
                    and (lse[fin] - lse_ref[fin]).abs().max().item() <= 1e-3)
            if same and fa.flexattn_poll_device_status() == 0:
                graphs = (g_mask, g_fwd)
                launch = "CUDA graph replay, one graph per call"
            else:
                launch = "eager (graph replay did not reproduce the eager result)"
        except Exception as exc:  # capture unsupported here: keep the eager launches
            launch = f"eager (graph capture failed: {type(exc).__name__})"
            torch.cuda.synchronize()

    # ---- device-timed region: K steps, L2 flushed between steps (outside the events)
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
                fa.flexattn_build_block_mask(mask, B_mask, 1, L, c["S"], BM, BN, out=bm)
            e1.record(stream)
            if graphs:
                graphs[1].replay()
            else:
                fa.flexattn_forward(q, k, v, bm, score_mod=score, mask_mod=mask, scale=c["scale"], enable_gqa=gqa,
                                    out=out, lse=lse, workspace=ws)
            e2.record(stream)
            flush.zero_()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    mask_ms = [a.elapsed_time(b) for a, b, _ in ev]
    fwd_ms = [b.elapsed_time(c_) for _, b, c_ in ev]
    step_ms = [a.elapsed_time(c_) for a, _, c_ in ev]
    total_ms = max_over_ranks(sum(step_ms), dev, world)
    if fa.flexattn_poll_device_status() != 0:
        raise RuntimeError("device status word set during the timed region")

    # ---- end to end through the public API from pinned host buffers
    q_p, k_p, v_p = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    out_p = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_p = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))
    for _ in range(2):
        q.copy_(q_p, non_blocking=True)
        step()
    torch.cuda.synchronize()
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    for i in range(e2e_steps):
        ee[i][0].record(stream)
        q.copy_(q_p, non_blocking=True)
        k.copy_(k_p, non_blocking=True)
        v.copy_(v_p, non_blocking=True)
        step()
        out_p.copy_(out, non_blocking=True)
        lse_p.copy_(lse, non_blocking=True)
        ee[i][1].record(stream)
        flush.zero_()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ee), dev, world)
    h2d = (q.numel() * q.element_size() + k.numel() * k.element_size() + v.numel() * v.element_size())
    d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    ms_per_step = total_ms / args.steps
    fwd_mean = statistics.mean(fwd_ms)
    if decode:
        value = whole_job_rate(kv_bytes, world, ms_per_step, 1e9)
        unit = "GB/s"
        achieved = kv_bytes / (fwd_mean * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"], "peak_source": f"hbm_gbs of {peak_src}"}
        e2e_val = whole_job_rate(kv_bytes, world, e2e_ms, 1e9)
    else:
        value = whole_job_rate(vis_flops, world, ms_per_step, 1e12)
        unit = "TFLOP/s"
        achieved = visited_flops / (fwd_mean * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": achieved / peaks["bf16_tflops"], "peak_source": f"bf16_tflops (burst) of {peak_src}",
                    "flops_counted_over": "visited-tile cells, (2E + 2Ev) per cell"}
        e2e_val = whole_job_rate(vis_flops, world, e2e_ms, 1e12)
    src_hash = kernel_source_hash("decode" if decode else "prefill")
    tr = NCU_TRAFFIC.get(name)
    roofline["traffic"] = tr["bytes"] if tr and tr["source_hash"] == src_hash and not args.batch else None

    line = {
        "metric": METRIC_PREFILL, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if c["dtype"] == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": name, **describe(name, c)[1],
                   "l2": "flushed: 256 MiB written between timed steps, outside the events",
                   "step": "block-mask build + forward",
                   "launch": launch,
                   "parallelism": f"weak scaling over {world} GPU(s): each rank runs the full per-GPU workload"},
        "roofline": roofline,
        "detail": {"forward_ms": fwd_mean, "block_mask_ms": statistics.mean(mask_ms),
                   "visible_pairs": vis_pairs, "visited_cells": cells,
                   "visible_tflops_forward_only": vis_flops / (fwd_mean * 1e-3) / 1e12,
                   "visited_tflops_forward_only": visited_flops / (fwd_mean * 1e-3) / 1e12,
                   "kernel_source": src_hash},
        "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    if not args.no_cpu_baseline and world == 1:
        rate, el, cores, sample, _, rate_unit = oracle_sample_rate(name, target_s=args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": rate_unit, "cores": cores, "kind": "oracle",
                                "sample": sample, "seconds": el}
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="causal_softcap_alibi", choices=sorted(wl.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch the timed calls directly instead of replaying CUDA graphs of them")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (smaller captures for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
