"""ctypes mirror of include/flexattn.h (structs, enums and prototypes)."""

from __future__ import annotations

import ctypes as C

FA_OK = 0
STATUS_NAMES = {
    0: "FA_OK", 1: "FA_ERR_NULL", 2: "FA_ERR_SHAPE", 3: "FA_ERR_HEADS", 4: "FA_ERR_BATCH",
    5: "FA_ERR_MASK_SHAPE", 6: "FA_ERR_DTYPE", 7: "FA_ERR_HEADDIM", 8: "FA_ERR_ALIGN", 9: "FA_ERR_PARAM",
    10: "FA_ERR_WORKSPACE", 11: "FA_ERR_UNSUPPORTED", 12: "FA_ERR_CUDA", 13: "FA_ERR_TIMEOUT",
}
FA_ERR_TIMEOUT = 13

FA_DTYPE_BF16 = 0
FA_DTYPE_F32 = 1

FA_FLAG_ROWS_GUARANTEED_SAFE = 1

MASK_KIND = {"none": 0, "causal": 1, "sliding_window": 2, "document": 3, "prefix_lm": 4, "chunked": 5,
             "program": 6}

# instructions of a composed rule (FA_PROG_*)
PROG_PRED = {"true": 0, "causal": 1, "distance_below": 2, "key_below": 3, "same_chunk": 4, "same_document": 5,
             "stride": 6, "head_below": 7}
PROG_AND, PROG_OR, PROG_NOT = 16, 17, 18
MASK_PROGRAM_MAX = 16
SCORE_KIND = {"none": 0, "softcap": 1, "alibi": 2, "cap_then_bias": 3}


class fa_mask_instr(C.Structure):
    _fields_ = [("op", C.c_int32), ("arg", C.c_int32)]


class fa_mask_mod(C.Structure):
    _fields_ = [
        ("kind", C.c_int32), ("window", C.c_int32), ("n_sink", C.c_int32), ("prefix", C.c_int32),
        ("chunk", C.c_int32), ("doc_batch", C.c_int32), ("doc_id", C.c_void_p), ("kv_len", C.c_void_p),
        ("n_instr", C.c_int32), ("reserved", C.c_int32), ("program", fa_mask_instr * MASK_PROGRAM_MAX),
    ]


class fa_score_mod(C.Structure):
    _fields_ = [
        ("kind", C.c_int32), ("cap", C.c_float), ("slope_heads", C.c_int32), ("pos_batch", C.c_int32),
        ("pos", C.c_void_p),
    ]


class fa_block_mask(C.Structure):
    _fields_ = [
        ("B", C.c_int32), ("H", C.c_int32), ("L", C.c_int32), ("S", C.c_int32), ("BM", C.c_int32),
        ("BN", C.c_int32), ("Mb", C.c_int32), ("Nb", C.c_int32),
        ("kv_num_blocks", C.c_void_p), ("kv_indices", C.c_void_p),
        ("full_kv_num_blocks", C.c_void_p), ("full_kv_indices", C.c_void_p),
    ]


class fa_tensor(C.Structure):
    _fields_ = [
        ("data", C.c_void_p), ("dtype", C.c_int32), ("reserved", C.c_int32),
        ("size", C.c_int64 * 4), ("stride", C.c_int64 * 4),
    ]


class fa_forward_options(C.Structure):
    _fields_ = [
        ("max_scores", C.c_void_p), ("wait_cycles", C.c_int64), ("flags", C.c_int32), ("reserved", C.c_int32),
        ("page_table", C.c_void_p), ("page_size", C.c_int32), ("pages_per_seq", C.c_int32),
    ]


class fa_block_mask_q(C.Structure):
    _fields_ = [
        ("B", C.c_int32), ("H", C.c_int32), ("Mb", C.c_int32), ("Nb", C.c_int32),
        ("q_num_blocks", C.c_void_p), ("q_indices", C.c_void_p),
        ("full_q_num_blocks", C.c_void_p), ("full_q_indices", C.c_void_p),
    ]


# (name, restype, argtypes) for every exported entry point.
PROTOTYPES = [
    ("flexattn_version", C.c_int, []),
    ("flexattn_last_error", C.c_char_p, []),
    ("flexattn_block_mask_dims", C.c_int,
     [C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.POINTER(C.c_int32), C.POINTER(C.c_int32)]),
    ("flexattn_build_block_mask", C.c_int, [C.POINTER(fa_mask_mod), C.POINTER(fa_block_mask), C.c_void_p]),
    ("flexattn_forward_workspace_size", C.c_int,
     [C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_block_mask), C.c_int32,
      C.POINTER(fa_forward_options), C.POINTER(C.c_size_t)]),
    ("flexattn_forward", C.c_int,
     [C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.c_void_p,
      C.c_float, C.c_int32, C.POINTER(fa_score_mod), C.POINTER(fa_mask_mod), C.POINTER(fa_block_mask),
      C.c_int32, C.POINTER(fa_forward_options), C.c_void_p, C.c_size_t, C.c_void_p]),
    ("flexattn_forward_decode_noalloc", C.c_int,
     [C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.c_void_p,
      C.c_float, C.c_int32, C.POINTER(fa_score_mod), C.POINTER(fa_mask_mod), C.POINTER(fa_block_mask),
      C.c_int32, C.c_void_p]),
    ("flexattn_transpose_block_mask", C.c_int, [C.POINTER(fa_block_mask), C.POINTER(fa_block_mask_q), C.c_void_p]),
    ("flexattn_backward_workspace_size", C.c_int, [C.POINTER(fa_tensor), C.POINTER(C.c_size_t)]),
    ("flexattn_backward", C.c_int,
     [C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor),
      C.c_void_p, C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.POINTER(fa_tensor), C.c_float, C.c_int32,
      C.POINTER(fa_score_mod), C.POINTER(fa_mask_mod), C.POINTER(fa_block_mask), C.POINTER(fa_block_mask_q),
      C.c_void_p, C.c_size_t, C.c_void_p]),
    ("flexattn_poll_device_status", C.c_int, [C.c_void_p, C.POINTER(C.c_int32)]),
]


def bind(lib):
    for name, res, args in PROTOTYPES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
