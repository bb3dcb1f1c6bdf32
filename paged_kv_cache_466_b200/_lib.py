"""ctypes declarations for ``libpagedattn.so`` (the C ABI of include/pagedattn.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation of any entry point.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpagedattn.so")

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_WORKSPACE = 3
PA_ERR_CUDA = 4
PA_ERR_BAD_TABLE = 5
PA_ERR_TIMEOUT = 6

PA_DERR_BAD_PAGE = 1
PA_DERR_BAD_CTX = 2
PA_DERR_BAD_SEQ = 4
PA_DERR_BAD_POS = 8
PA_DERR_TIMEOUT = 32

PA_KV_BF16 = 0
PA_KV_U8_PER_TOKEN = 1
PA_KV_FP8_PER_TOKEN = 2
PA_KV_U4_PER_TOKEN = 3

PA_NOALLOC_SCRATCH_BYTES = 16 << 20
PA_STEP_NEWEST_PER_SEQ = -1


class pa_kv_pool_t(ctypes.Structure):
    _fields_ = [
        ("num_pages", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("k_pool", ctypes.c_void_p),
        ("v_pool", ctypes.c_void_p),
        ("k_sz", ctypes.c_void_p),
        ("v_sz", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_POOL = ctypes.POINTER(pa_kv_pool_t)

SIGNATURES = {
    "pa_kv_append": (_I, [_POOL, _P, _P, _P, _P, _I, _P, _I, _I, _P, _P]),
    "pa_derr_status": (_I, [_I]),
    "pa_selftest_wait_timeout": (_I, [_I, _P, _P]),
    "pa_decode_auto_splits": (_I, [_I, _I, _I, _I]),
    "pa_decode_append": (_I, [_POOL, _P, _P, _P, _I, _I, _P, _I, _P, ctypes.c_float, _P, _P,
                              ctypes.c_size_t, _I, _P, _P]),
    "pa_decode_append_lens": (_I, [_POOL, _P, _P, _P, _I, _I, _P, _I, _P, _P, ctypes.c_float, _P, _P,
                              ctypes.c_size_t, _I, _P, _P]),
    "pa_decode_plan_splits": (_I, [ctypes.c_int64, _I, _I, _I, _I, _I]),
    "pa_prefix_plan_splits": (_I, [ctypes.c_int64, _I, _I, _I, ctypes.c_double]),
    "pa_decode_plan_lens": (_I, [_P, _I, _I, _I, _I, _I, _I, _P]),
    "pa_decode_num_splits_lens": (_I, [_POOL, _I, _I, _P, _I]),
    "pa_decode_num_splits": (_I, [_POOL, _I, _I, _I]),
    "pa_decode_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "pa_decode": (_I, [_POOL, _P, _I, _I, _P, _I, _P, ctypes.c_float, _P, _P, ctypes.c_size_t,
                       _I, _P, _P]),
    "pa_decode_shared_prefix_workspace_bytes": (ctypes.c_size_t, [_POOL, _I, _I, _I, _I, _I]),
    "pa_decode_shared_prefix": (_I, [_POOL, _P, _I, _I, _P, _I, _P, _I, _P, ctypes.c_float, _P,
                                     _P, ctypes.c_size_t, _I, _P, _P]),
    "pa_decode_window_workspace_bytes": (ctypes.c_size_t, [_POOL, _I, _I, _I, _I, _I, _I]),
    "pa_decode_window": (_I, [_POOL, _P, _I, _I, _P, _I, _P, _I, _I, ctypes.c_float, _P, _P,
                              ctypes.c_size_t, _I, _P, _P]),
    "pa_decode_noalloc": (_I, [_POOL, _P, _I, _I, _P, _I, _P, ctypes.c_float, _P, _I, _P, _P]),
    "pa_decode_range_workspace_bytes": (ctypes.c_size_t, [_POOL, _I, _I, _I, _I, _I, _I]),
    "pa_decode_range": (_I, [_POOL, _P, _I, _I, _P, _I, _P, _I, _I, ctypes.c_float, _P, _P, _P,
                             ctypes.c_size_t, _I, _P, _P]),
    "pa_step_packet_layout": (ctypes.c_size_t, [_POOL, _I, _I, _I, _I, _P]),
    "pa_decode_step_host": (_I, [_POOL, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, ctypes.c_float,
                                 _P, _P, _P, ctypes.c_size_t, _I, _P, _P, _I]),
    "pa_step_graph_create": (_I, [_POOL, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, ctypes.c_float,
                                  _P, _P, _P, ctypes.c_size_t, _I, _P, _P]),
    "pa_step_graph_launch": (_I, [_P, _P, _I]),
    "pa_step_graph_destroy": (None, [_P]),
    "pa_merge_partials": (_I, [_P, _P, _I, _I, _I, ctypes.c_int64, ctypes.c_int64, _P, _P,
                                _P]),
    "pa_splitkv_reduce": (_I, [_P, _P, _I, _I, _I, _I, _P, _P]),
    "pa_validate_tables": (_I, [_P, _I, _I, _P, _I, _I, _P, _P]),
    "pa_status_str": (ctypes.c_char_p, [_I]),
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_abi_version": (_I, []),
}

_LIB = None


def load() -> ctypes.CDLL:
    """The loaded library; raises if it is missing (build it with build())."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build the CUDA library first "
                "(python -m paged_kv_cache_466_b200.build); there is no fallback")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        self.status = status
        msg = lib.pa_last_error().decode() or lib.pa_status_str(status).decode()
        super().__init__(f"{where}: {lib.pa_status_str(status).decode()} ({msg})")


def check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PagedAttnError(status, where)
