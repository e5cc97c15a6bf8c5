"""Helpers shared by the GPU parity tests: build one seeded case for both sides.

The oracle receives numpy arrays (bf16 values upcast exactly to fp64); the CUDA
library receives device tensors of the same values.  Mask and score specs are
translated separately for each side.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import workloads as wl


def bf16_tolerance(ref):
    """Allowed |out - ref| for bf16 outputs: 1e-2 plus half a bf16 ulp of ref.

    A bf16 store of |o| in [4, 8) alone moves it by up to 2^-6 > 1e-2, so the
    1e-2 bound on the arithmetic is applied on top of the output rounding.
    """
    a = np.maximum(np.abs(ref), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(a)) - 7)
    return 1e-2 + 0.5 * ulp


TOL = {"fp32": dict(out=1e-5, lse=1e-3), "bf16": dict(out=None, lse=1e-3)}


def torch_dtype(name):
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


class Case:
    """Seeded inputs on the CPU and the GPU, plus mask/score specs for each side."""

    def __init__(self, B, Hq, Hkv, L, S, E, Ev, dtype, mask, score, seed=0, kv_len=None, doc_lengths=None,
                 scale=None, sentinel_tail=False):
        self.B, self.Hq, self.Hkv, self.L, self.S, self.E, self.Ev = B, Hq, Hkv, L, S, E, Ev
        self.dtype = dtype
        self.scale = (1.0 / math.sqrt(E)) if scale is None else scale
        # the kernel receives an fp32 scale; the oracle uses that same value
        self.scale32 = float(np.float32(self.scale))
        q, k, v = wl.randn_qkv(B, Hq, Hkv, L, S, E, Ev, seed=seed, dtype=torch_dtype(dtype))
        self.kv_len = None if kv_len is None else np.asarray(kv_len, dtype=np.int32)
        if sentinel_tail and self.kv_len is not None:
            wl.fill_cache_tail(k, v, self.kv_len)
        self.q_cpu, self.k_cpu, self.v_cpu = q, k, v
        self.q, self.k, self.v = q.cuda(), k.cuda(), v.cuda()
        self.oracle_mask = dict(mask)
        self.dev_mask = dict(mask)
        self.oracle_score = dict(score)
        self.dev_score = dict(score)
        if mask["kind"] == "document" or score.get("pos") == "in_doc":
            lens = doc_lengths if doc_lengths is not None else wl.doc_lengths(S, max(1, S // 16), max(2, S // 4), seed)
            ids = wl.doc_ids_from_lengths(lens)
            self.doc_ids = ids
            if mask["kind"] == "document":
                self.oracle_mask["doc_id"] = ids
                self.dev_mask["doc_id"] = torch.from_numpy(ids).cuda().reshape(1, S)
            if score.get("pos") == "in_doc":
                self.oracle_score["doc_id"] = ids
                self.dev_score["pos"] = torch.from_numpy(wl.in_doc_positions(lens)).cuda().reshape(1, S)
        if score.get("pos") in ("global", "in_doc") and "pos" in self.dev_score and isinstance(self.dev_score["pos"], str):
            self.dev_score["pos"] = None
        if self.kv_len is not None:
            self.dev_mask["kv_len"] = torch.from_numpy(self.kv_len).cuda()

    @classmethod
    def from_config(cls, name, **over):
        c = wl.config(name, **over)
        kv_len = None
        doc_lengths = None
        if name == "decode_kv_cache":
            kv_len = wl.decode_cache_lengths(c["B"], c["kv_lo"], c["kv_hi"], c["seed"])
        if name == "packed_docs":
            doc_lengths = wl.doc_lengths(c["doc_total"], c["doc_lo"], c["doc_hi"], c["seed"])
        case = cls(c["B"], c["Hq"], c["Hkv"], c["L"], c["S"], c["E"], c["Ev"], c["dtype"], c["mask"], c["score"],
                   seed=c["seed"], kv_len=kv_len, doc_lengths=doc_lengths, scale=c["scale"],
                   sentinel_tail=kv_len is not None)
        case.BM, case.BN = c["BM"], c["BN"]
        return case

    def block_mask(self, BM, BN, B_mask=None, H_mask=1):
        import programmable_block_sparse_b200 as fa
        B_mask = B_mask or (self.B if (self.kv_len is not None) else 1)
        return fa.flexattn_build_block_mask(self.dev_mask, B_mask, H_mask, self.L, self.S, BM, BN)

    def run(self, BM, BN, split_kv=0, bm=None, **kw):
        """(out, lse), or (out, lse, max_scores) with max_scores=True."""
        import programmable_block_sparse_b200 as fa
        bm = bm or self.block_mask(BM, BN)
        res = fa.flexattn_forward(self.q, self.k, self.v, bm, score_mod=self.dev_score, mask_mod=self.dev_mask,
                                  scale=self.scale32, enable_gqa=self.Hq != self.Hkv, split_kv=split_kv, **kw)
        torch.cuda.synchronize()
        return res

    def oracle(self, aux=False):
        import oracle.flex_oracle as o
        return o.forward(self.q_cpu, self.k_cpu, self.v_cpu, self.scale32, self.oracle_mask, self.oracle_score,
                         kv_len=self.kv_len, enable_gqa=self.Hq != self.Hkv, aux=aux)

    def oracle_rows(self, samples):
        import oracle.flex_oracle as o
        return o.forward_sampled(self.q_cpu, self.k_cpu, self.v_cpu, samples, self.scale32, self.oracle_mask,
                                 self.oracle_score, kv_len=self.kv_len, enable_gqa=self.Hq != self.Hkv)


def out_tolerance(in_dtype, out_is_fp32, ref):
    """fp32 I/O: 1e-5.  bf16 inputs with an fp32 output: a strict 1e-2 (the
    arithmetic alone).  bf16 output: 1e-2 plus half a bf16 ulp of ref."""
    if in_dtype == "fp32":
        return TOL["fp32"]["out"]
    return 1e-2 if out_is_fp32 else bf16_tolerance(ref)


def assert_close(case, out, lse, ref_out, ref_lse, max_scores=None, ref_max=None):
    """Element-wise comparison with the workload dtype's tolerance."""
    out_f32 = out.dtype == torch.float32
    out = out.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    assert not np.isnan(out).any(), "NaN in the output"
    assert not np.isnan(lse).any(), "NaN in the lse"
    tol = out_tolerance(case.dtype, out_f32, ref_out)
    err = np.abs(out - ref_out)
    bad = err > tol
    assert not bad.any(), f"max |out - ref| = {err.max():.3e} at {np.argwhere(bad)[0].tolist()} ({bad.sum()} elems)"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin), "lse finiteness differs (fully masked rows must give -inf)"
    assert np.all(lse[~fin] == -np.inf)
    if fin.any():
        lerr = np.abs(lse[fin] - ref_lse[fin])
        assert lerr.max() <= TOL[case.dtype]["lse"], f"max |lse - ref| = {lerr.max():.3e}"
    if max_scores is not None:
        assert_max_scores(max_scores, ref_max)
    return float(err.max())


def assert_max_scores(got, ref, tol=1e-3):
    """max_scores within the lse tolerance; rows without a visible key -inf."""
    got = got.cpu().numpy().astype(np.float64) if hasattr(got, "cpu") else np.asarray(got, np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), "max_scores finiteness differs"
    assert np.all(got[~fin] == -np.inf)
    if fin.any():
        err = np.abs(got[fin] - ref[fin])
        assert err.max() <= tol, f"max |max_scores - ref| = {err.max():.3e}"
