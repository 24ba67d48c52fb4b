"""ctypes declarations of the C ABI in include/pagedkv.h (raw pointers and sizes).

Loading fails loudly if libpagedkv.so has not been built: there is no other
implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

from ._build import LIB

PA_OK = 0
PA_ERR_INVALID = -1
PA_ERR_DTYPE = -2
PA_ERR_OVERFLOW = -3
PA_ERR_CUDA = -4
PA_ERR_WORKSPACE = -5

PA_DEV_BAD_SLOT = 1
PA_DEV_BAD_BLOCK = 2
PA_DEV_CTX_OVER_TABLE = 4
PA_DEV_CTX_OVER_BOUND = 8
PA_DEV_BAD_PAIR = 16
PA_DEV_WAIT_TIMEOUT = 32
PA_DEV_PREFIX = 64
PA_DEV_BAD_CHUNK = 128

PA_F16 = 0
PA_E4M3 = 1


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_size", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


class DecodeConfig(ctypes.Structure):
    _fields_ = [("partition_size", ctypes.c_int32), ("heads_per_cta", ctypes.c_int32),
                ("warps_per_head", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("units_per_cta", ctypes.c_int32)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float

SIGNATURES = {
    "pa_version": (_I, []),
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_check_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "pa_test_stall_next_decode": (_I, [_I, _I, _I, ctypes.c_uint64]),
    "pa_slot_mapping": (_I, [_P, _P, _I, _P, _I, CacheDesc, _P]),
    "pa_kv_cache_write": (_I, [_P, _P, _I64, _I64, _P, _P, CacheDesc, _P, _I, _F, _F, _P]),
    "pa_copy_blocks": (_I, [_P, _P, CacheDesc, _P, _I, _P]),
    "pa_swap_blocks": (_I, [_P, _P, _I, _P, _P, _I, CacheDesc, _P, _I, _P]),
    "pa_paged_attention_decode": (_I, [_P, _P, _P, _P, CacheDesc, _P, _I, _P, _I, _I, _F, _F, _F, _P]),
    "pa_decode_choose_config": (_I, [CacheDesc, _I, _I, ctypes.POINTER(DecodeConfig)]),
    "pa_decode_workspace_size": (ctypes.c_size_t, [CacheDesc, _I, _I, ctypes.POINTER(DecodeConfig)]),
    "pa_paged_attention_decode_ws": (_I, [_P, _P, _P, _P, CacheDesc, _P, _I, _P, _I, _I, _F, _F, _F,
                                          ctypes.POINTER(DecodeConfig), _P, ctypes.c_size_t, _P]),
    "pa_paged_attention_decode_append": (_I, [_P, _P, _P, _P, _I64, _I64, _P, _P, CacheDesc, _P, _I, _P,
                                              _I, _I, _F, _F, _F, _P, ctypes.POINTER(DecodeConfig),
                                              _P, ctypes.c_size_t, _P]),
    "pa_paged_attention_decode_shared_prefix": (_I, [_P, _P, _P, _P, _I64, _I64, _P, _P, CacheDesc, _P, _I,
                                                     _P, _I, _I, _I, _F, _F, _F, _P,
                                                     ctypes.POINTER(DecodeConfig), _P, ctypes.c_size_t, _P]),
    "pa_shared_prefix_workspace_size": (ctypes.c_size_t, [CacheDesc, _I, _I, _I, ctypes.POINTER(DecodeConfig)]),
    "pa_paged_attention_decode_noalloc": (_I, [_P, _P, _P, _P, CacheDesc, _P, _I, _P, _I, _I, _F, _F,
                                               _F, _P]),
    "pa_prefill_slot_mapping": (_I, [_P, _P, _P, _I, _P, _I, _I, _I, CacheDesc, _P]),
    "pa_paged_prefill": (_I, [_P, _P, _P, _P, _P, CacheDesc, _P, _I, _P, _I, _I, _I, _F, _P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libpagedkv.so with argument types declared."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise ImportError(f"{LIB} is missing: build it with "
                              "`python -m pagedattention_paged_kv_decode_b200._build`")
        handle = ctypes.CDLL(LIB)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


class PagedKVError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"[{code}] {message}")
        self.code = code


def check(rc: int) -> None:
    if rc != PA_OK:
        raise PagedKVError(rc, lib().pa_last_error().decode(errors="replace"))
