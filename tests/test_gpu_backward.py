"""The backward pass on the GPU against the fp64 oracle's gradients.

"flexattention-score-mod-block-mask" runs the loss's backward through
flex_attention; the oracle's gradients (oracle.backward) are pinned by finite
differences and autograd.  The GPU recomputes P from the lse it is given and
writes every gradient once: dk / dv per key tile over the query-side lists,
dq per query tile over the key-side lists.

Inputs.  A backward call receives the forward's output and lse; D =
rowsum(dout * out) is formed from that output.  The GPU backward is given
the oracle's forward results as the forward stores them (out rounded to
bf16, lse in fp32), and the oracle forms D from the same stored output, so
the comparison covers the backward kernels alone (the forward kernels have
their own parity tests).

Tolerance.  The kernels round P and dS to bf16 (relative error at most
2^-9) before the tensor-core products dv = P^T dout, dk = scale dS^T q,
dq = scale dS k.  Over n terms those roundings add up like a random walk:
their standard deviation is below 2^-9 / sqrt(3) times the root of the
sum of the squared terms, rms = sqrt(sum_i (P_ij dout_ie)^2) for dv and
likewise for dk and dq.  The bound is |g - ref| <= 2e-2 + 2e-2 |ref| +
8 * 2^-9 rms (about 14 standard deviations); bf16 gradients add their own
storage rounding, half a bf16 ulp of ref.
"""

import math

import numpy as np
import pytest
import torch

import oracle.flex_oracle as o
import programmable_block_sparse_b200 as fa
import workloads as wl
from gpu_cases import Case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


def grad_tolerance(ref, bf16, rms=0.0):
    tol = 2e-2 + 2e-2 * np.abs(ref) + 8 * 2.0 ** -9 * rms
    if bf16:
        a = np.maximum(np.abs(ref), 2.0 ** -126)
        tol = tol + 0.5 * 2.0 ** (np.floor(np.log2(a)) - 7)
    return tol


def _check_grads(got, ref, bf16, what, rms=(0.0, 0.0, 0.0)):
    worst = 0.0
    for name, g, r, w in zip(("dq", "dk", "dv"), got, ref, rms):
        g = g.float().cpu().numpy().astype(np.float64)
        assert not np.isnan(g).any(), f"{what}: NaN in {name}"
        err = np.abs(g - r)
        bad = err > grad_tolerance(r, bf16, w)
        assert not bad.any(), f"{what}: {name} max |g - ref| = {err.max():.3e} at {np.argwhere(bad)[0].tolist()}"
        worst = max(worst, float(err.max()))
    return worst


def _stored(x):
    """The oracle's output as the forward stores it (bf16)."""
    return torch.from_numpy(np.asarray(x)).to(torch.bfloat16).double().numpy()


def rounding_rms(q, k, v, dout, scale, mask, score, kv_len, G, units=None):
    """Root sums of squared terms of the three products whose bf16 operands
    (P, dS) the kernels round: (dq, dk, dv) shaped like the gradients, over
    all (batch, query head) units or the listed ones.  P and dS come from the
    oracle's building blocks, as in its backward."""
    q, k, v, do = (torch.as_tensor(x).double().numpy() for x in (q, k, v, dout))
    B, Hq, L, _ = q.shape
    S = k.shape[2]
    rq, rk, rv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b, h in units or [(b, h) for b in range(B) for h in range(Hq)]:
        S_b = S if kv_len is None else int(kv_len[b])
        qp, kv = o.query_positions(L, S_b), np.arange(S)
        kh = h // G
        s = scale * (q[b, h] @ k[b, kh].T)
        g = np.where(o.visible(mask, b, h, qp, kv, S_b), o.score_mod(score, s, b, h, qp, kv, Hq), -np.inf)
        m = g.max(axis=1, keepdims=True)
        p = np.zeros_like(g)
        live = np.isfinite(m[:, 0])
        p[live] = np.exp(g[live] - m[live])
        p[live] /= p[live].sum(axis=1, keepdims=True)
        out = p @ v[b, kh]
        ds = p * (do[b, h] @ v[b, kh].T - (do[b, h] * out).sum(axis=1, keepdims=True)) * o.score_mod_slope(score, s)
        rv[b, kh] += (p ** 2).T @ do[b, h] ** 2
        rk[b, kh] += scale ** 2 * (ds ** 2).T @ q[b, h] ** 2
        rq[b, h] = scale ** 2 * (ds ** 2) @ k[b, kh] ** 2
    return np.sqrt(rq), np.sqrt(rk), np.sqrt(rv)


def _run_case(case, grad_dtype=torch.float32, seed=0, bm=None, mask_mod=None):
    """Backward on the GPU from the oracle's stored forward results; returns
    (GPU grads, oracle grads, rounding rms)."""
    bm = bm or case.block_mask(128, 128, B_mask=case.B if case.kv_len is not None else 1,
                               H_mask=case.Hq if case.dev_mask.get("_per_head") else 1)
    ro, rl = case.oracle()
    stored = _stored(ro)
    dout = torch.randn(ro.shape, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    out_in = torch.from_numpy(stored).to(torch.bfloat16).cuda()
    lse_in = torch.from_numpy(np.asarray(rl, np.float32)).cuda()
    grads = fa.flexattn_backward(case.q, case.k, case.v, out_in, dout.cuda(), lse_in, bm, score_mod=case.dev_score,
                                 mask_mod=mask_mod or case.dev_mask, scale=case.scale32,
                                 enable_gqa=case.Hq != case.Hkv, grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    assert fa.flexattn_poll_device_status() == 0
    ref = o.backward(case.q_cpu, case.k_cpu, case.v_cpu, dout, case.scale32, case.oracle_mask, case.oracle_score,
                     kv_len=case.kv_len, enable_gqa=case.Hq != case.Hkv, out=stored)
    rms = rounding_rms(case.q_cpu, case.k_cpu, case.v_cpu, dout, case.scale32, case.oracle_mask, case.oracle_score,
                       case.kv_len, case.Hq // case.Hkv)
    return grads, ref, rms


MASKS = [{"kind": "none"}, {"kind": "causal"}, {"kind": "sliding_window", "window": 70, "n_sink": 4},
         {"kind": "document"}, {"kind": "prefix_lm", "prefix": 50}, {"kind": "chunked", "chunk": 96}]
SCORES = [{"kind": "none"}, {"kind": "softcap", "cap": 5.0}, {"kind": "alibi", "slope_heads": 0},
          {"kind": "cap_then_bias", "cap": 30.0, "slope_heads": 4, "pos": "global"},
          {"kind": "cap_then_bias", "cap": 20.0, "slope_heads": 0, "pos": "in_doc"}]


@pytest.mark.parametrize("E", [64, 128])
@pytest.mark.parametrize("score", SCORES, ids=lambda s: s["kind"] + ("_doc" if s.get("pos") == "in_doc" else ""))
@pytest.mark.parametrize("mask", MASKS, ids=lambda m: m["kind"])
def test_backward_mask_score_matrix(mask, score, E):
    """Every mask x score kind, L = S = 300 (3 tiles, ragged), GQA 4 / 2,
    per-sequence valid lengths (300, 263)."""
    case = Case(2, 4, 2, 300, 300, E, E, "bf16", mask, score, seed=21, kv_len=[300, 263])
    grads, ref, rms = _run_case(case, seed=E)
    _check_grads(grads, ref, False, f"{mask['kind']}/{score['kind']}", rms)


@pytest.mark.parametrize("E", [64, 128])
def test_backward_bf16_gradients_and_long_walks(E):
    """L = S = 1100 (9 tiles each way, both rings wrap), causal soft-cap, GQA
    8 / 2 (each key tile's walk covers four query heads), bf16 gradients."""
    case = Case(1, 8, 2, 1100, 1100, E, E, "bf16", {"kind": "causal"}, {"kind": "softcap", "cap": 30.0}, seed=5)
    grads, ref, rms = _run_case(case, grad_dtype=torch.bfloat16, seed=1)
    worst = _check_grads(grads, ref, True, "long walks", rms)
    print(f"E={E}: max |g - ref| = {worst:.3e}")


def test_backward_bottom_right_rows_without_keys():
    """L = 200 queries against 150 keys, bottom-right causal: the first 50
    rows see no key, their dq is 0 and they add nothing to dk, dv."""
    case = Case(1, 2, 2, 200, 150, 64, 64, "bf16", {"kind": "causal"}, {"kind": "none"}, seed=8)
    grads, ref, rms = _run_case(case, seed=3)
    assert torch.all(grads[0][0, :, :50] == 0)
    _check_grads(grads, ref, False, "rows without keys", rms)


def test_backward_composed_head_dependent_rule():
    """Half the heads global, half a window of 96 keys (a per-head block mask
    and per-head query-side lists)."""
    rule = fa.and_masks({"kind": "causal"}, fa.or_masks({"kind": "head_below", "value": 2},
                                                        {"kind": "distance_below", "value": 96}))
    case = Case(1, 4, 4, 500, 500, 64, 64, "bf16", {"kind": "causal"}, {"kind": "alibi"}, seed=9)
    case.oracle_mask = rule
    case.dev_mask = dict(rule, _per_head=True)
    bm = fa.flexattn_build_block_mask(rule, 1, 4, 500, 500, 128, 128)
    grads, ref, rms = _run_case(case, seed=4, bm=bm, mask_mod=rule)
    _check_grads(grads, ref, False, "head-dependent rule", rms)


@pytest.mark.parametrize("mask", [{"kind": "causal"}, {"kind": "sliding_window", "window": 300, "n_sink": 4},
                                  {"kind": "document"}], ids=lambda m: m["kind"])
def test_query_side_lists_bit_exact(mask):
    case = Case(2, 2, 2, 1000, 1000, 64, 64, "bf16", mask, {"kind": "none"}, seed=2, kv_len=[1000, 777])
    for BM, BN in ((128, 128), (64, 32)):
        bm = case.block_mask(BM, BN, B_mask=2)
        q_side = fa.flexattn_transpose_block_mask(bm)
        torch.cuda.synchronize()
        ref = o.transpose_block_mask(o.block_mask(case.oracle_mask, 2, 1, 1000, 1000, BM, BN, kv_len=case.kv_len))
        for key in ("q_num_blocks", "q_indices", "full_q_num_blocks", "full_q_indices"):
            assert np.array_equal(getattr(q_side, key).cpu().numpy(), ref[key]), (key, BM, BN)


def test_backward_causal_softcap_alibi_full_size_units():
    """The causal soft-cap ALiBi workload at full size (B=4, H=16, L=S=2048,
    E=64), chained: the GPU forward's out and lse feed the GPU backward, so D
    carries the forward's own rounding (small at E = 64).  Gradients of four
    whole (batch, head) units, among them the last, against the oracle's."""
    case = Case.from_config("causal_softcap_alibi")
    out, lse = case.run(128, 128, split_kv=1)
    dout = torch.randn(out.shape, generator=torch.Generator().manual_seed(11)).to(torch.bfloat16)
    grads = fa.flexattn_backward(case.q, case.k, case.v, out, dout.cuda(), lse, case.block_mask(128, 128),
                                 score_mod=case.dev_score, mask_mod=case.dev_mask, scale=case.scale32,
                                 grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert fa.flexattn_poll_device_status() == 0
    units = [(0, 0), (1, 7), (2, 15), (3, 15)]
    rms = rounding_rms(case.q_cpu, case.k_cpu, case.v_cpu, dout, case.scale32, case.oracle_mask, case.oracle_score,
                       None, 1, units=units)
    for b, h in units:
        args = (case.q_cpu[b, h], case.k_cpu[b, h], case.v_cpu[b, h])
        ro, _, _ = o.forward_unit(*args, b, h, case.Hq, case.S, case.scale32, case.oracle_mask, case.oracle_score)
        ref = o.backward_unit(*args, dout[b, h], b, h, case.Hq, case.S, case.scale32, case.oracle_mask,
                              case.oracle_score, out_bh=_stored(ro))
        _check_grads([g[b, h] for g in grads], ref, False, f"unit ({b}, {h})", [r[b, h] for r in rms])
