"""ctypes mirror of ``include/sa.h``: structs, enums and entry-point prototypes.

Loading fails loudly when ``libsa.so`` has not been built; there is no other
implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsa.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_CUDA, \
    SA_ERR_DEVICE_FAULT, SA_ERR_TIMEOUT = range(7)
SA_F32, SA_BF16, SA_E4M3, SA_MXFP8 = 0, 1, 2, 3
SA_WS_INDEXER, SA_WS_TOPK, SA_WS_ATTN, SA_WS_DECODE, SA_WS_APPEND = 1, 2, 4, 8, 16
SA_DETAIL_NONE, SA_DETAIL_BAD_PAGE, SA_DETAIL_BAD_POSITION, SA_DETAIL_BAD_INDEX, \
    SA_DETAIL_WAIT_TIMEOUT = range(5)

DTYPES = {"f32": SA_F32, "bf16": SA_BF16, "e4m3": SA_E4M3, "mxfp8": SA_MXFP8}

# every symbol include/sa.h declares
EXPORTS = ("sa_workspace_size", "sa_indexer_score", "sa_topk", "sa_sparse_mla_attn",
           "sa_decode", "sa_decode_traced", "sa_decode_noalloc", "sa_noalloc_status",
           "sa_local_candidates", "sa_merge_candidates", "sa_combine_partials",
           "sa_quantize_index_query",
           "sa_append_tokens", "sa_device_status",
           "sa_kernel_launches", "sa_status_string", "sa_version")
NOALLOC_SCRATCH_BYTES = 32 << 20
DECODE_PHASES = ("indexer", "topk", "attention")

_P, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


class SaCache(ctypes.Structure):
    _fields_ = [("page_table", _P), ("seq_len", _P), ("batch", _I32), ("max_pages", _I32),
                ("num_pages", _I32), ("page_size", _I32),
                ("index_dtype", ctypes.c_int), ("k_index", _P), ("k_index_scale", _P),
                ("d_index", _I32),
                ("kv_dtype", ctypes.c_int), ("kv", _P), ("kv_rope", _P), ("kv_scale", _P),
                ("d_latent", _I32), ("d_rope", _I32),
                ("kv_scale_tokens", _I32), ("kv_scale_dims", _I32)]


class SaQuery(ctypes.Structure):
    _fields_ = [("n_q", _I32), ("q_seq", _P), ("q_pos", _P), ("max_visible", _I32),
                ("q_index", _P), ("q_index_scale", _P), ("w", _P), ("h_index", _I32),
                ("q_dtype", ctypes.c_int), ("q", _P), ("heads", _I32),
                ("sm_scale", ctypes.c_float), ("q_group", _I32)]


class SaNewTokens(ctypes.Structure):
    _fields_ = [("n_new", _I32), ("seq", _P), ("pos", _P), ("in_dtype", ctypes.c_int),
                ("k_index", _P), ("kv", _P)]


class SaError(RuntimeError):
    def __init__(self, status: int, where: str, detail: int | None = None):
        self.status = status
        self.detail = detail
        msg = f"{where}: {status_string(status)} (status {status}"
        msg += f", detail {detail})" if detail is not None else ")"
        super().__init__(msg)


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m indexed_sparse_attention_lightning_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        CP, QP = ctypes.POINTER(SaCache), ctypes.POINTER(SaQuery)
        L.sa_workspace_size.argtypes = [CP, QP, _I32, _I32]
        L.sa_workspace_size.restype = _SZ
        L.sa_indexer_score.argtypes = [CP, QP, _P, _I64, _P, _SZ, _P]
        L.sa_indexer_score.restype = ctypes.c_int
        L.sa_topk.argtypes = [_P, _I64, _P, _I32, _I32, _I32, _P, _P, _SZ, _P]
        L.sa_topk.restype = ctypes.c_int
        L.sa_sparse_mla_attn.argtypes = [CP, QP, _P, _I32, _P, ctypes.c_int, _P, _P, _SZ, _P]
        L.sa_sparse_mla_attn.restype = ctypes.c_int
        L.sa_decode.argtypes = [CP, QP, _I32, _P, _P, ctypes.c_int, _P, _P, _SZ, _P]
        L.sa_decode.restype = ctypes.c_int
        L.sa_decode_traced.argtypes = [CP, QP, _I32, _P, _P, ctypes.c_int, _P, _P, _SZ, _P, _P]
        L.sa_decode_traced.restype = ctypes.c_int
        L.sa_decode_noalloc.argtypes = [CP, QP, _I32, _P, _P, ctypes.c_int, _P, _P]
        L.sa_decode_noalloc.restype = ctypes.c_int
        L.sa_noalloc_status.argtypes = [_P, ctypes.POINTER(_I32)]
        L.sa_noalloc_status.restype = ctypes.c_int
        L.sa_local_candidates.argtypes = [CP, QP, _I32, _P, _P, _P, _P, _SZ, _P]
        L.sa_local_candidates.restype = ctypes.c_int
        L.sa_merge_candidates.argtypes = [_P, _P, _I32, _I32, _I32, _P, _P, _P, _P, _P]
        L.sa_merge_candidates.restype = ctypes.c_int
        L.sa_combine_partials.argtypes = [_P, _P, _I32, _I32, _I32, _I32, _P, ctypes.c_int, _P,
                                          _P]
        L.sa_combine_partials.restype = ctypes.c_int
        L.sa_quantize_index_query.argtypes = [_P, ctypes.c_int, _I32, _I32, _I32, _P, _P, _P]
        L.sa_quantize_index_query.restype = ctypes.c_int
        L.sa_append_tokens.argtypes = [CP, ctypes.POINTER(SaNewTokens), _P, _SZ, _P]
        L.sa_append_tokens.restype = ctypes.c_int
        L.sa_device_status.argtypes = [_P, _SZ, _P, ctypes.POINTER(_I32)]
        L.sa_device_status.restype = ctypes.c_int
        L.sa_status_string.argtypes = [ctypes.c_int]
        L.sa_status_string.restype = ctypes.c_char_p
        L.sa_kernel_launches.argtypes = []
        L.sa_kernel_launches.restype = ctypes.c_uint64
        L.sa_version.argtypes = []
        L.sa_version.restype = _I32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().sa_status_string(status).decode()


def check(status: int, where: str) -> None:
    if status != SA_OK:
        raise SaError(status, where)
