"""The five workloads at full size, in the launch configuration bench.py times,
compared element by element with the fp64 oracle.

The oracle evaluates whole (batch, query head) units in spawned worker
processes (tests/oracle_pool.py), each from slices regenerated from the
workload's seed.  Compared in full:

* causal + soft-cap + ALiBi, B=4, H=16, L=S=2048, E=64: all 64 units;
* packed documents, H=16, L=S=8192, E=128: all 16 heads;
* decode against a KV cache, B=32, Hq=32, Hkv=8, q_len 4 and 1: all rows;
* GQA sliding window, B=2, Hq=32, Hkv=8, L=S=16384, E=128: six whole units,
  among them the first and the last (batch, head) and every head of KV head 7
  of the last batch (a 16384-row unit costs the oracle about 70 GFLOP).

Each is run with a bf16 output (tolerance 1e-2 plus half a bf16 ulp) and
with an fp32 output (a strict 1e-2); lse within 1e-3 and max_scores within
1e-3 in both.  Over the whole output: no NaN, and a finite lse wherever the
mask leaves a key.
"""

import numpy as np
import pytest
import torch

from gpu_cases import Case, assert_max_scores, out_tolerance
from oracle_pool import oracle_units

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


def _run_both(case):
    """bf16-output and fp32-output runs of the workload, with max_scores."""
    import programmable_block_sparse_b200 as fa
    bm = case.block_mask(case.BM, case.BN)
    res = {}
    for name, dt in (("bf16", None), ("fp32", torch.float32)):
        out, lse, mx = case.run(case.BM, case.BN, bm=bm, out_dtype=dt, max_scores=True)
        assert fa.flexattn_poll_device_status() == 0
        assert not torch.isnan(out).any() and not torch.isnan(lse).any()
        res[name] = (out, lse, mx)
    return res


def _compare_units(case, res, ref):
    """Every element of every listed unit; returns the strict max-abs of each output type."""
    worst = {}
    for name, (out, lse, mx) in res.items():
        err_max = 0.0
        for (b, h), (ro, rl, rm) in ref.items():
            got = out[b, h].float().cpu().numpy().astype(np.float64)
            tol = out_tolerance(case.dtype, name == "fp32", ro)
            err = np.abs(got - ro)
            bad = err > tol
            assert not bad.any(), (f"{name} output, unit ({b}, {h}): max |out - ref| = {err.max():.3e}, "
                                   f"{int(bad.sum())} elements, first at row {np.argwhere(bad)[0][0]}")
            err_max = max(err_max, float(err.max()))
            gl = lse[b, h].cpu().numpy().astype(np.float64)
            fin = np.isfinite(rl)
            assert np.array_equal(np.isfinite(gl), fin), f"unit ({b}, {h}): lse finiteness differs"
            if fin.any():
                assert np.abs(gl[fin] - rl[fin]).max() <= 1e-3, (b, h, np.abs(gl[fin] - rl[fin]).max())
            assert_max_scores(mx[b, h], rm)
        worst[name] = err_max
    return worst


def test_causal_softcap_alibi_every_element():
    case = Case.from_config("causal_softcap_alibi")
    res = _run_both(case)
    assert torch.isfinite(res["bf16"][1]).all()  # causal: every row sees at least itself
    units = [(b, h) for b in range(case.B) for h in range(case.Hq)]
    worst = _compare_units(case, res, oracle_units("causal_softcap_alibi", units))
    print(f"causal_softcap_alibi: strict max-abs bf16 out {worst['bf16']:.3e}, fp32 out {worst['fp32']:.3e}")


def test_packed_docs_every_element():
    case = Case.from_config("packed_docs")
    res = _run_both(case)
    assert torch.isfinite(res["bf16"][1]).all()
    units = [(0, h) for h in range(case.Hq)]
    worst = _compare_units(case, res, oracle_units("packed_docs", units))
    print(f"packed_docs: strict max-abs bf16 out {worst['bf16']:.3e}, fp32 out {worst['fp32']:.3e}")


def test_gqa_sliding_window_whole_units():
    case = Case.from_config("gqa_sliding_window")
    res = _run_both(case)
    assert torch.isfinite(res["bf16"][1]).all()
    units = [(0, 0), (0, 13), (1, 28), (1, 29), (1, 30), (1, 31)]
    worst = _compare_units(case, res, oracle_units("gqa_sliding_window", units))
    print(f"gqa_sliding_window: strict max-abs bf16 out {worst['bf16']:.3e}, fp32 out {worst['fp32']:.3e}")


@pytest.mark.parametrize("L", [4, 1])
def test_decode_kv_cache_every_element(L):
    case = Case.from_config("decode_kv_cache", L=L)
    res = _run_both(case)
    out = res["bf16"][0]
    assert torch.isfinite(res["bf16"][1]).all()
    assert out.abs().max().item() < 10.0  # the +-1e4 cache tail never leaks
    units = [(b, h) for b in range(case.B) for h in range(case.Hq)]
    worst = _compare_units(case, res, oracle_units("decode_kv_cache", units, L=L))
    print(f"decode_kv_cache L={L}: strict max-abs bf16 out {worst['bf16']:.3e}, fp32 out {worst['fp32']:.3e}")
