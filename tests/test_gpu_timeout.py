"""A bounded device wait that runs out reports FA_ERR_TIMEOUT, and the GPU stays usable.

The forward call accepts a per-call budget for its main-path device waits
(fa_forward_options.wait_cycles).  With a budget of a few dozen cycles the
first wait that is not already satisfied gives up: the kernel records
FA_ERR_TIMEOUT in the device status word, its warps leave together, the
producer drains its own copies and the MMA issuer its own MMAs (with the
default budget), TMEM is freed and the kernel ends.  The outputs of that call
are unspecified.  The next call, with the default budget, must be correct and
leave the status word clear.  Nothing here faults or traps the GPU: the
timeout is an ordinary return path of the kernels.
"""

import pytest
import torch

from gpu_cases import Case, assert_close

pytestmark = pytest.mark.gpu

FA_ERR_TIMEOUT = 13

CASES = {
    # (B, Hq, Hkv, L, S, E, mask, score, kv_len, split_kv)
    "tcgen05_e64": (2, 4, 2, 700, 700, 64, {"kind": "causal"}, {"kind": "softcap", "cap": 30.0}, None, 1),
    "tcgen05_e128": (2, 4, 2, 700, 700, 128, {"kind": "sliding_window", "window": 200, "n_sink": 4},
                     {"kind": "none"}, None, 1),
    # document ids and in-document positions: the four warps of a softmax
    # group stage key-side values for one another behind a group barrier
    "tcgen05_documents": (1, 4, 4, 900, 900, 128, {"kind": "document"},
                          {"kind": "cap_then_bias", "cap": 30.0, "slope_heads": 0, "pos": "in_doc"}, None, 1),
    # head dim 128: the tensor-core decode kernel; head dim 64: the mma.sync one
    "decode": (4, 8, 2, 4, 3000, 128, {"kind": "causal"}, {"kind": "softcap", "cap": 50.0}, [3000, 2000, 900, 129],
               4),
    "decode_e64": (4, 8, 2, 4, 3000, 64, {"kind": "causal"}, {"kind": "softcap", "cap": 50.0},
                   [3000, 2000, 900, 129], 4),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from programmable_block_sparse_b200 import build
    build.build()


@pytest.mark.parametrize("name", sorted(CASES))
def test_short_wait_budget_times_out_then_recovers(name):
    import programmable_block_sparse_b200 as fa
    B, Hq, Hkv, L, S, E, mask, score, kv_len, split = CASES[name]
    case = Case(B, Hq, Hkv, L, S, E, E, "bf16", mask, score, seed=41, kv_len=kv_len, sentinel_tail=kv_len is not None)
    bm = case.block_mask(128, 128)
    assert fa.flexattn_poll_device_status() == 0
    case.run(128, 128, bm=bm, split_kv=split, wait_cycles=32)
    assert fa.flexattn_poll_device_status() == FA_ERR_TIMEOUT
    assert fa.flexattn_poll_device_status() == 0  # the poll cleared it
    out, lse = case.run(128, 128, bm=bm, split_kv=split)
    assert fa.flexattn_poll_device_status() == 0
    assert_close(case, out, lse, *case.oracle())
    torch.cuda.synchronize()
