"""The five workloads at full size, in the launch configuration bench.py times.

Outputs are compared with the fp64 oracle on sampled rows (each row computed
in full by the oracle) -- first rows, tile and window edges, document starts,
random rows -- and checked over the whole output for properties that hold at
any size: no NaN, a finite lse for every row that sees a key.
"""

import numpy as np
import pytest
import torch

import workloads as wl
from gpu_cases import Case, bf16_tolerance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


def _samples(case, rows, n_random=24, seed=0):
    rng = np.random.default_rng(seed)
    out = set()
    for r in rows:
        if 0 <= r < case.L:
            out.add((int(rng.integers(case.B)), int(rng.integers(case.Hq)), int(r)))
            out.add((case.B - 1, case.Hq - 1, int(r)))
    for _ in range(n_random):
        out.add((int(rng.integers(case.B)), int(rng.integers(case.Hq)), int(rng.integers(case.L))))
    return sorted(out)


def _check(case, out, lse, samples):
    assert not torch.isnan(out).any(), "NaN in output"
    assert not torch.isnan(lse).any(), "NaN in lse"
    ref_o, ref_l = case.oracle_rows(samples)
    got_o = np.stack([out[b, h, r].float().cpu().numpy() for b, h, r in samples]).astype(np.float64)
    got_l = np.array([lse[b, h, r].item() for b, h, r in samples])
    tol = bf16_tolerance(ref_o) if case.dtype == "bf16" else 1e-5
    err = np.abs(got_o - ref_o)
    assert np.all(err <= tol), f"max |out-ref| = {err.max():.3e}"
    fin = np.isfinite(ref_l)
    assert np.array_equal(fin, np.isfinite(got_l))
    assert np.all(np.abs(got_l[fin] - ref_l[fin]) <= 1e-3), np.abs(got_l[fin] - ref_l[fin]).max()
    return float(err.max())


def test_causal_softcap_alibi_full_size():
    case = Case.from_config("causal_softcap_alibi")
    out, lse = case.run(case.BM, case.BN)
    assert torch.isfinite(lse).all()  # causal: every row sees at least itself
    _check(case, out, lse, _samples(case, [0, 1, 2, 127, 128, 129, 1000, 2046, 2047]))


def test_packed_docs_full_size():
    case = Case.from_config("packed_docs")
    lens = wl.doc_lengths(8192, 128, 2048, 0)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).tolist()
    out, lse = case.run(case.BM, case.BN)
    assert torch.isfinite(lse).all()
    rows = starts + [s + 1 for s in starts] + [s - 1 for s in starts[1:]] + [8191]
    _check(case, out, lse, _samples(case, rows, n_random=16))


def test_gqa_sliding_window_full_size():
    case = Case.from_config("gqa_sliding_window")
    out, lse = case.run(case.BM, case.BN)
    assert torch.isfinite(lse).all()
    _check(case, out, lse, _samples(case, [0, 3, 4, 1023, 1024, 1025, 1026, 1027, 1028, 4095, 16383], n_random=16))
