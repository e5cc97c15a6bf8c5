"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host (no GPU needed: these calls return before any CUDA work)."""

import ctypes as C
import os
import re

import pytest

import programmable_block_sparse_b200 as fa
from programmable_block_sparse_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flexattn.h")
FAKE = 0x7F0000001000  # a 16-byte-aligned address never dereferenced by the host checks


@pytest.fixture(scope="module")
def lib():
    from programmable_block_sparse_b200 import build
    build.build()
    return fa.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(flexattn_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("flexattn_build_block_mask", "flexattn_forward", "flexattn_forward_workspace_size",
              "flexattn_block_mask_dims", "flexattn_last_error", "flexattn_poll_device_status", "flexattn_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == {p[0] for p in _abi.PROTOTYPES}


def test_struct_layouts_match_header_sizes():
    assert C.sizeof(_abi.fa_mask_mod) == 6 * 4 + 2 * 8 + 2 * 4 + 16 * 8
    assert C.sizeof(_abi.fa_score_mod) == 4 * 4 + 8
    assert C.sizeof(_abi.fa_block_mask) == 8 * 4 + 4 * 8
    assert C.sizeof(_abi.fa_tensor) == 8 + 4 + 4 + 8 * 8
    assert C.sizeof(_abi.fa_forward_options) == 8 + 8 + 4 + 4 + 8 + 4 + 4


def test_version(lib):
    assert fa.flexattn_version() >= 100


def test_block_mask_dims(lib):
    assert fa.flexattn_block_mask_dims(6, 6, 2, 2) == (3, 3)
    assert fa.flexattn_block_mask_dims(2048, 2048, 128, 128) == (16, 16)
    assert fa.flexattn_block_mask_dims(4, 32768, 128, 128) == (1, 256)
    assert fa.flexattn_block_mask_dims(129, 1, 128, 1) == (2, 1)
    with pytest.raises(fa.FlexAttnError) as e:
        fa.flexattn_block_mask_dims(8, 8, 0, 4)
    assert e.value.status == 2
    with pytest.raises(fa.FlexAttnError):
        fa.flexattn_block_mask_dims(8, 8, 4, 129)


def _t(B, H, N, D, dtype=_abi.FA_DTYPE_BF16, addr=FAKE, stride=None):
    t = _abi.fa_tensor()
    t.data = addr
    t.dtype = dtype
    for i, s in enumerate((B, H, N, D)):
        t.size[i] = s
    st = stride or (H * N * D, N * D, D, 1)
    for i, s in enumerate(st):
        t.stride[i] = s
    return t


def _bm(B, H, L, S, BM, BN):
    s = _abi.fa_block_mask()
    s.B, s.H, s.L, s.S, s.BM, s.BN = B, H, L, S, BM, BN
    s.Mb, s.Nb = -(-L // BM), -(-S // BN)
    s.kv_num_blocks = s.kv_indices = s.full_kv_num_blocks = s.full_kv_indices = FAKE
    return s


def _call(lib, q, k, v, out, bm, score=None, mask=None, gqa=0, split=0, opts=None):
    score = score or _abi.fa_score_mod(kind=0)
    mask = mask or _abi.fa_mask_mod(kind=1)
    return lib.flexattn_forward(C.byref(q), C.byref(k), C.byref(v), C.byref(out) if out is not None else None,
                                None, 0.0, gqa, C.byref(score), C.byref(mask), C.byref(bm), split,
                                C.byref(opts) if opts is not None else None, None, 0, None)


def test_forward_rejects_bad_arguments(lib):
    q, k, v, o = _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64)
    bm = _bm(1, 1, 256, 256, 128, 128)
    # heads: Hq != Hkv without GQA, and a non-divisible group
    assert _call(lib, q, _t(2, 2, 256, 64), _t(2, 2, 256, 64), o, bm) == 3
    assert "enable_gqa" in fa.flexattn_last_error()
    assert _call(lib, _t(2, 6, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 6, 256, 64), bm, gqa=1) == 3
    # batch
    assert _call(lib, q, _t(3, 4, 256, 64), _t(3, 4, 256, 64), o, bm) == 4
    assert _call(lib, q, k, v, o, _bm(3, 1, 256, 256, 128, 128)) == 4
    # block mask built for other lengths: too small / too large
    assert _call(lib, q, k, v, o, _bm(1, 1, 128, 256, 128, 128)) == 5
    assert "too small" in fa.flexattn_last_error()
    assert _call(lib, q, k, v, o, _bm(1, 1, 512, 256, 128, 128)) == 5
    assert "too large" in fa.flexattn_last_error()
    bad = _bm(1, 1, 256, 256, 128, 128)
    bad.Nb = 3
    assert _call(lib, q, k, v, o, bad) == 5
    # dtype
    assert _call(lib, q, _t(2, 4, 256, 64, dtype=_abi.FA_DTYPE_F32), v, o, bm) == 6
    # fp32 output from bf16 inputs is allowed; bf16 output from fp32 inputs is not
    f32 = _abi.FA_DTYPE_F32
    assert _call(lib, _t(2, 4, 256, 64, dtype=f32), _t(2, 4, 256, 64, dtype=f32), _t(2, 4, 256, 64, dtype=f32),
                 _t(2, 4, 256, 64), bm) == 6
    # head dim
    assert _call(lib, _t(2, 4, 256, 256), _t(2, 4, 256, 256), _t(2, 4, 256, 256), _t(2, 4, 256, 256), bm) == 7
    # strides
    assert _call(lib, _t(2, 4, 256, 64, stride=(4 * 256 * 64, 256 * 64, 64, 2)), k, v, o, bm) == 8
    # NULLs
    assert _call(lib, _t(2, 4, 256, 64, addr=0), k, v, o, bm) == 1
    assert _call(lib, q, k, v, None, bm) == 1
    nulls = _bm(1, 1, 256, 256, 128, 128)
    nulls.kv_indices = None
    assert _call(lib, q, k, v, o, nulls) == 1
    # out shape
    assert _call(lib, q, k, v, _t(2, 4, 255, 64), bm) == 2


def test_forward_rejects_bad_mod_parameters(lib):
    q, k, v, o = _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64)
    bm = _bm(1, 1, 256, 256, 128, 128)
    assert _call(lib, q, k, v, o, bm, mask=_abi.fa_mask_mod(kind=2, window=0)) == 9
    assert _call(lib, q, k, v, o, bm, mask=_abi.fa_mask_mod(kind=2, window=4, n_sink=-1)) == 9
    assert _call(lib, q, k, v, o, bm, mask=_abi.fa_mask_mod(kind=3)) == 9
    assert _call(lib, q, k, v, o, bm, mask=_abi.fa_mask_mod(kind=3, doc_id=FAKE, doc_batch=3)) == 4
    assert _call(lib, q, k, v, o, bm, mask=_abi.fa_mask_mod(kind=4, prefix=-1)) == 9
    assert _call(lib, q, k, v, o, bm, mask=_abi.fa_mask_mod(kind=5, chunk=0)) == 9
    assert _call(lib, q, k, v, o, bm, mask=_abi.fa_mask_mod(kind=9)) == 9
    assert _call(lib, q, k, v, o, bm, mask=_abi.fa_mask_mod(kind=1, kv_len=FAKE)) == 4  # needs a per-batch mask
    assert _call(lib, q, k, v, o, bm, score=_abi.fa_score_mod(kind=1, cap=0.0)) == 9
    assert _call(lib, q, k, v, o, bm, score=_abi.fa_score_mod(kind=3, cap=-1.0)) == 9
    assert _call(lib, q, k, v, o, bm, score=_abi.fa_score_mod(kind=1, cap=float("inf"))) == 9
    assert _call(lib, q, k, v, o, bm, score=_abi.fa_score_mod(kind=2, slope_heads=-2)) == 9
    assert _call(lib, q, k, v, o, bm, score=_abi.fa_score_mod(kind=3, cap=5.0, pos=FAKE, pos_batch=5)) == 4
    assert _call(lib, q, k, v, o, bm, score=_abi.fa_score_mod(kind=7)) == 9


def test_split_kv_rules(lib):
    # forced splits need a short query; a long one is rejected on the host
    q, k, v, o = _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64)
    assert _call(lib, q, k, v, o, _bm(1, 1, 256, 256, 128, 128), split=4) == 11
    assert _call(lib, q, k, v, o, _bm(1, 1, 256, 256, 128, 128), split=-1) == 9


def test_build_block_mask_rejects_bad_arguments(lib):
    bm = _bm(1, 1, 64, 64, 16, 16)
    m = _abi.fa_mask_mod(kind=2, window=0)
    assert lib.flexattn_build_block_mask(C.byref(m), C.byref(bm), None) == 9
    bm.Mb = 5
    assert lib.flexattn_build_block_mask(C.byref(_abi.fa_mask_mod(kind=1)), C.byref(bm), None) == 5
    assert lib.flexattn_build_block_mask(None, C.byref(bm), None) == 1
    big = _bm(1, 1, 64, 64, 256, 16)
    assert lib.flexattn_build_block_mask(C.byref(_abi.fa_mask_mod(kind=1)), C.byref(big), None) == 2


def test_python_binding_rejects_non_4d_tensors(lib):
    import torch
    with pytest.raises(fa.FlexAttnError):
        fa._tensor_struct(torch.zeros(2, 3, 4))


def test_forward_rejects_bad_options(lib):
    q, k, v, o = _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64)
    bm = _bm(1, 1, 256, 256, 128, 128)
    assert _call(lib, q, k, v, o, bm, opts=_abi.fa_forward_options(flags=2)) == 9
    assert "flags" in fa.flexattn_last_error()
    assert _call(lib, q, k, v, o, bm, opts=_abi.fa_forward_options(reserved=1)) == 9
    assert _call(lib, q, k, v, o, bm, opts=_abi.fa_forward_options(wait_cycles=-5)) == 9


def _prog(*instrs, doc=None):
    m = _abi.fa_mask_mod(kind=6)
    m.n_instr = len(instrs)
    for i, (op, arg) in enumerate(instrs):
        m.program[i].op, m.program[i].arg = op, arg
    if doc is not None:
        m.doc_id, m.doc_batch = doc, 1
    return m


def test_composed_rules_checked_on_the_host(lib):
    q, k, v, o = _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64)
    bm = _bm(1, 1, 256, 256, 128, 128)
    AND, OR, NOT = 16, 17, 18
    # broken postfix: two verdicts left, an operator without operands, no instruction
    assert _call(lib, q, k, v, o, bm, mask=_prog((1, 0), (6, 4))) == 9
    assert _call(lib, q, k, v, o, bm, mask=_prog((1, 0), (AND, 0))) == 9
    assert _call(lib, q, k, v, o, bm, mask=_prog()) == 9
    # bad arguments and unknown instructions; same-document without ids
    assert _call(lib, q, k, v, o, bm, mask=_prog((6, 0))) == 9
    assert _call(lib, q, k, v, o, bm, mask=_prog((4, -3))) == 9
    assert _call(lib, q, k, v, o, bm, mask=_prog((2, (1 << 30) + 1))) == 9
    assert _call(lib, q, k, v, o, bm, mask=_prog((12, 0))) == 9
    assert _call(lib, q, k, v, o, bm, mask=_prog((5, 0))) == 9
    # a head-dependent rule needs a per-head block mask
    assert _call(lib, q, k, v, o, bm, mask=_prog((1, 0), (7, 2), (AND, 0))) == 5
    assert "per-head" in fa.flexattn_last_error()
    # an OR of four ANDs of two predicates needs 2^4 = 16 clauses in AND-of-OR form
    big = []
    for i in range(4):
        big += [(2, 10 + i), (3, 20 + i), (AND, 0)]
        if i:
            big.append((OR, 0))
    assert _call(lib, q, k, v, o, bm, mask=_prog(*big)) == 11
    assert "clauses" in fa.flexattn_last_error()
    # a valid rule passes the host checks and reaches the launch-free build check
    bm2 = _bm(1, 1, 64, 64, 16, 16)
    bm2.Mb = 5
    assert lib.flexattn_build_block_mask(C.byref(_prog((1, 0), (6, 4), (AND, 0))), C.byref(bm2), None) == 5


def test_paged_cache_checked_on_the_host(lib):
    q, o = _t(2, 4, 4, 64), _t(2, 4, 4, 64)
    kp, vp = _t(10, 2, 64, 64), _t(10, 2, 64, 64)   # pools of 10 pages of 64 keys
    bm = _bm(2, 1, 4, 256, 128, 128)                  # logical length 4 pages x 64
    opts = _abi.fa_forward_options(page_table=FAKE, page_size=64, pages_per_seq=4)
    # pools whose slot extent is not the page size, or k and v of different pool sizes
    assert _call(lib, q, _t(10, 2, 32, 64), _t(10, 2, 32, 64), o, bm, gqa=1, opts=opts) == 2
    assert _call(lib, q, kp, _t(9, 2, 64, 64), o, bm, gqa=1, opts=opts) == 2
    # page size or table width below 1
    assert _call(lib, q, kp, vp, o, bm, gqa=1,
                 opts=_abi.fa_forward_options(page_table=FAKE, page_size=0, pages_per_seq=4)) == 9
    # the block mask must describe the logical length
    assert _call(lib, q, kp, vp, o, _bm(2, 1, 4, 640, 128, 128), gqa=1, opts=opts) == 5
    # forced splits need pages of a multiple of 64 keys
    odd = _abi.fa_forward_options(page_table=FAKE, page_size=48, pages_per_seq=4)
    assert _call(lib, q, _t(10, 2, 48, 64), _t(10, 2, 48, 64), o, _bm(2, 1, 4, 192, 128, 128), gqa=1, split=3,
                 opts=odd) == 11
    n = C.c_size_t()
    assert lib.flexattn_forward_workspace_size(C.byref(q), C.byref(_t(10, 2, 32, 64)), C.byref(vp), C.byref(bm), 0,
                                               C.byref(opts), C.byref(n)) == 2


def _bq(B, H, Mb, Nb):
    s = _abi.fa_block_mask_q()
    s.B, s.H, s.Mb, s.Nb = B, H, Mb, Nb
    s.q_num_blocks = s.q_indices = s.full_q_num_blocks = s.full_q_indices = FAKE
    return s


def test_backward_checked_on_the_host(lib):
    q, k, v, o, do = (_t(2, 4, 256, 64) for _ in range(5))
    dq, dk, dv = _t(2, 4, 256, 64), _t(2, 4, 256, 64), _t(2, 4, 256, 64)
    bm, bq = _bm(1, 1, 256, 256, 128, 128), _bq(1, 1, 2, 2)
    sc, mk = _abi.fa_score_mod(kind=0), _abi.fa_mask_mod(kind=1)

    def call(q=q, k=k, v=v, o=o, do=do, dq=dq, dk=dk, dv=dv, bm=bm, bq=bq, ws=FAKE, ws_bytes=1 << 20, lse=FAKE):
        return lib.flexattn_backward(C.byref(q), C.byref(k), C.byref(v), C.byref(o), C.byref(do), lse, C.byref(dq),
                                     C.byref(dk), C.byref(dv), 0.0, 0, C.byref(sc), C.byref(mk), C.byref(bm),
                                     C.byref(bq), ws, ws_bytes, None)
    f32 = _abi.FA_DTYPE_F32
    assert call(q=_t(2, 4, 256, 64, dtype=f32), k=_t(2, 4, 256, 64, dtype=f32), v=_t(2, 4, 256, 64, dtype=f32),
                o=_t(2, 4, 256, 64, dtype=f32)) == 11                       # fp32 inputs
    assert call(q=_t(2, 4, 256, 96), k=_t(2, 4, 256, 96), v=_t(2, 4, 256, 96), o=_t(2, 4, 256, 96),
                do=_t(2, 4, 256, 96), dq=_t(2, 4, 256, 96), dk=_t(2, 4, 256, 96), dv=_t(2, 4, 256, 96)) == 11
    assert call(bm=_bm(1, 1, 256, 256, 64, 64), bq=_bq(1, 1, 4, 4)) == 11  # other tiles
    assert call(dq=_t(2, 4, 255, 64)) == 2                                  # gradient shapes
    assert call(do=_t(2, 4, 128, 64)) == 2
    assert call(bq=_bq(1, 1, 2, 3)) == 5                                    # lists of another mask
    assert call(ws_bytes=16) == 10                                          # workspace
    assert call(lse=None) == 1
    assert call(dk=_t(2, 4, 256, 64, stride=(4 * 256 * 64, 256 * 64, 64, 2))) == 8
    assert call(o=_t(2, 4, 256, 64, addr=FAKE + 2)) == 8                    # out read with 16-byte loads
    assert call(o=_t(2, 4, 256, 64, stride=(4 * 256 * 68, 256 * 68, 68 + 1, 1))) == 8
    n = C.c_size_t()
    assert lib.flexattn_backward_workspace_size(C.byref(q), C.byref(n)) == 0 and n.value == 2 * 4 * 256 * 4


def test_transpose_checked_on_the_host(lib):
    bm = _bm(1, 1, 256, 256, 128, 128)
    assert lib.flexattn_transpose_block_mask(C.byref(bm), C.byref(_bq(1, 1, 2, 3)), None) == 5
    assert lib.flexattn_transpose_block_mask(None, C.byref(_bq(1, 1, 2, 2)), None) == 1
    nul = _bq(1, 1, 2, 2)
    nul.q_indices = None
    assert lib.flexattn_transpose_block_mask(C.byref(bm), C.byref(nul), None) == 1
