"""ctypes view of the C ABI in include/mla_decode.h (argument marshalling only).

Loads the in-tree ``libmla_decode_b200.so``; importing fails loudly when it is
missing (build it with ``python -m mla_decode_attention_get_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmla_decode_b200.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE = 3
MLA_ERR_CUDA = 4

MLA_DEVERR_BLOCK_TABLE = 1
MLA_DEVERR_INDEX = 2
MLA_DEVERR_TIMEOUT = 4
MLA_DEVERR_SEQLEN = 8
MLA_DEVERR_INTERNAL = 16

MD_WORDS = 8
PAGE_SIZE = 64
D_QK = 576
D_V = 512
FP8_ROW_BYTES = 656

# Every symbol include/mla_decode.h declares.
EXPORTS = ("mla_metadata_shape", "mla_get_metadata", "mla_workspace_bytes", "mla_decode",
           "mla_decode_attention", "mla_decode_combine", "mla_decode_noalloc", "mla_fp8_cache_write",
           "mla_set_pipeline_wait_limit", "mla_status_string")

# Size of the scratch array built into the library for mla_decode_noalloc.
NOALLOC_SCRATCH_BYTES = 64 << 20


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class DecodeArgs(ctypes.Structure):
    """Mirror of ``mla_decode_args``."""
    _fields_ = [
        ("q", ctypes.c_void_p),
        ("q_batch_stride", ctypes.c_int64),
        ("k_cache", ctypes.c_void_p),
        ("k_block_stride", ctypes.c_int64),
        ("num_blocks", ctypes.c_int32),
        ("block_table", ctypes.c_void_p),
        ("block_table_stride", ctypes.c_int32),
        ("block_table_width", ctypes.c_int32),
        ("cache_seqlens", ctypes.c_void_p),
        ("indices", ctypes.c_void_p),
        ("topk", ctypes.c_int32),
        ("tile_md", ctypes.c_void_p),
        ("num_splits", ctypes.c_void_p),
        ("num_parts", ctypes.c_int32),
        ("out", ctypes.c_void_p),
        ("lse", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("err_word", ctypes.c_void_p),
        ("batch", ctypes.c_int32),
        ("s_q", ctypes.c_int32),
        ("h_q", ctypes.c_int32),
        ("h_kv", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("causal", ctypes.c_int32),
        ("is_fp8", ctypes.c_int32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m mla_decode_attention_get_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i, p, v = ctypes.c_int, ctypes.POINTER, ctypes.c_void_p
        L.mla_metadata_shape.argtypes = [i, i, i, i, i, i, p(i), p(i)]
        L.mla_get_metadata.argtypes = [v, i, i, i, i, i, i, v, v, v]
        L.mla_workspace_bytes.argtypes = [i, i, i, i, i, p(ctypes.c_size_t)]
        for name in ("mla_decode", "mla_decode_attention", "mla_decode_combine", "mla_decode_noalloc"):
            getattr(L, name).argtypes = [p(DecodeArgs), v]
        L.mla_fp8_cache_write.argtypes = [v, ctypes.c_int64, i, v, v, ctypes.c_int64, i, v, v]
        L.mla_set_pipeline_wait_limit.argtypes = [ctypes.c_uint64]
        L.mla_status_string.argtypes = [i]
        L.mla_status_string.restype = ctypes.c_char_p
        for name in EXPORTS[:-1]:
            getattr(L, name).restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().mla_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MlaError(status, where)


def metadata_shape(batch, s_q, h_q, h_kv, topk, num_sm_parts):
    parts, nlen = ctypes.c_int(), ctypes.c_int()
    check(lib().mla_metadata_shape(batch, s_q, h_q, h_kv, topk, num_sm_parts,
                                   ctypes.byref(parts), ctypes.byref(nlen)), "mla_metadata_shape")
    return parts.value, nlen.value


def set_pipeline_wait_limit(ns: int) -> None:
    """Give-up limit of the kernels' pipeline waits for the calls that follow
    (0 = the default); see mla_set_pipeline_wait_limit."""
    check(lib().mla_set_pipeline_wait_limit(int(ns)), "mla_set_pipeline_wait_limit")


def workspace_bytes(batch, s_q, h_q, topk, num_parts) -> int:
    n = ctypes.c_size_t()
    check(lib().mla_workspace_bytes(batch, s_q, h_q, topk, num_parts, ctypes.byref(n)), "mla_workspace_bytes")
    return n.value
