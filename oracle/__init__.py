"""CPU oracle for the paged-KV decode path and the paged prefill (test
infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It wraps ``pagedkv_oracle.c`` -- plain
scalar C in double precision -- through ctypes, and shares no code with the
CUDA library. The functions take and return numpy arrays; fp16 data are
passed as ``np.float16`` arrays (their bits are what the C code reads) and
E4M3 caches as ``np.uint8`` arrays of codes.

What each function computes, and the passages it follows, is stated in the
C source. Parity pins for every function live in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pagedkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F16 = 0
E4M3 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction; OpenMP
    only spreads independent (sequence, head) pairs over threads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
             "-Wall", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _declare(lib):
    """Declare the C signatures on a loaded oracle library."""
    P = ctypes.c_void_p
    I = ctypes.c_int
    I64 = ctypes.c_int64
    F = ctypes.c_float
    lib.oracle_f16_to_double.restype = ctypes.c_double
    lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_e4m3_to_double.restype = ctypes.c_double
    lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_from_float.restype = ctypes.c_uint8
    lib.oracle_e4m3_from_float.argtypes = [F]
    lib.oracle_slot_mapping.restype = I
    lib.oracle_slot_mapping.argtypes = [P, P, I, P, I, I]
    lib.oracle_kv_cache_write.restype = I
    lib.oracle_kv_cache_write.argtypes = [P, P, I64, I64, P, P, I, I, I, I, I, P, I, F, F]
    lib.oracle_kv_cache_write_threads.restype = I
    lib.oracle_kv_cache_write_threads.argtypes = [P, P, I64, I64, P, P, I, I, I, I, I, P, I, F, F, I]
    lib.oracle_copy_blocks.restype = I
    lib.oracle_copy_blocks.argtypes = [P, P, I64, I, P, I]
    lib.oracle_swap_blocks.restype = I
    lib.oracle_swap_blocks.argtypes = [P, P, I, P, P, I, I64, P, I]
    lib.oracle_paged_attention.restype = I
    lib.oracle_paged_attention.argtypes = [P, P, P, P, I, I, I, I, I, P, I, P, I, F, F, F, P, I]
    lib.oracle_paged_attention_threads.restype = I
    lib.oracle_paged_attention_threads.argtypes = [P, P, P, P, I, I, I, I, I, P, I, P, I, F, F, F, P, I, I]
    lib.oracle_max_threads.restype = I
    lib.oracle_max_threads.argtypes = []
    lib.oracle_attention_partials.restype = I
    lib.oracle_attention_partials.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P, I, F, F, F, I, I]
    lib.oracle_prefill_slot_mapping.restype = I
    lib.oracle_prefill_slot_mapping.argtypes = [P, P, P, I, P, I, I]
    lib.oracle_paged_prefill.restype = I
    lib.oracle_paged_prefill.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P, I, F, F, F, P, I]
    lib.oracle_lse_combine.restype = None
    lib.oracle_lse_combine.argtypes = [P, P, P, I, I]
    lib.oracle_f16_array_to_double.restype = None
    lib.oracle_f16_array_to_double.argtypes = [P, P, I64]
    lib.oracle_e4m3_array_to_double.restype = None
    lib.oracle_e4m3_array_to_double.argtypes = [P, P, I64]
    lib.oracle_e4m3_array_from_float.restype = None
    lib.oracle_e4m3_array_from_float.argtypes = [P, P, I64]
    return lib


class using_library:
    """Context manager: route this module's calls through another build of the
    oracle's C source (the mutation tests plant mistakes in such builds)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = _declare(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _dtype_code(cache: np.ndarray) -> int:
    if cache.dtype == np.float16:
        return F16
    if cache.dtype == np.uint8:
        return E4M3
    raise TypeError(f"cache dtype {cache.dtype} is neither float16 nor uint8 (E4M3 codes)")


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its input (rc={rc})")


# ----------------------------------------------------------------- numbers

def f16_to_double(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float16)
    out = np.empty(x.shape, np.float64)
    _load().oracle_f16_array_to_double(_ptr(out), _ptr(x.view(np.uint16)), x.size)
    return out


def e4m3_to_double(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, np.float64)
    _load().oracle_e4m3_array_to_double(_ptr(out), _ptr(codes), codes.size)
    return out


def e4m3_from_float(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e4m3_array_from_float(_ptr(out), _ptr(x), x.size)
    return out


# ------------------------------------------------------------ path steps

def slot_mapping(block_tables: np.ndarray, context_lens: np.ndarray, block_size: int) -> np.ndarray:
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.empty(ctx.shape[0], np.int32)
    _check(_load().oracle_slot_mapping(_ptr(out), _ptr(bt), bt.shape[1], _ptr(ctx),
                                       ctx.shape[0], block_size), "slot_mapping")
    return out


def prefill_slot_mapping(query_start: np.ndarray, block_tables: np.ndarray,
                         context_lens: np.ndarray, block_size: int) -> np.ndarray:
    """One slot per new token of a prefill chunk ([total_q] int32)."""
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.full(int(qs[-1]), -1, np.int32)
    _check(_load().oracle_prefill_slot_mapping(_ptr(out), _ptr(qs), _ptr(bt), bt.shape[1], _ptr(ctx),
                                               ctx.shape[0], block_size), "prefill_slot_mapping")
    return out


def kv_cache_write(key: np.ndarray, value: np.ndarray, key_cache: np.ndarray,
                   value_cache: np.ndarray, slot_mapping: np.ndarray,
                   k_scale: float = 1.0, v_scale: float = 1.0, threads: int | None = None) -> None:
    """In place on key_cache/value_cache ([NB, B, H, D], float16 or uint8 codes).
    threads=None runs on the calling thread; threads=n (0: the host's
    default) spreads each token's row over n OpenMP threads, tokens still in
    order, with the same result bit for bit."""
    assert key.dtype == np.float16 and value.dtype == np.float16
    nb, bs, nh, hd = key_cache.shape
    n = slot_mapping.shape[0]
    k2 = key.reshape(n, -1)
    v2 = value.reshape(n, -1)
    assert k2.shape[1] == nh * hd and k2.strides[1] == 2 and v2.strides[1] == 2
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int32)
    lib = _load()
    args = (k2.ctypes.data, v2.ctypes.data, k2.strides[0] // 2, v2.strides[0] // 2,
            _ptr(key_cache), _ptr(value_cache), _dtype_code(key_cache), nb, bs, nh, hd,
            _ptr(slots), n, float(np.float32(k_scale)), float(np.float32(v_scale)))
    if threads is None:
        rc = lib.oracle_kv_cache_write(*args)
    else:
        rc = lib.oracle_kv_cache_write_threads(*args, int(threads))
    _check(rc, "kv_cache_write")


def copy_blocks(key_cache: np.ndarray, value_cache: np.ndarray, src_dst_pairs: np.ndarray) -> None:
    pairs = np.ascontiguousarray(src_dst_pairs, dtype=np.int32).reshape(-1, 2)
    nb = key_cache.shape[0]
    block_bytes = key_cache[0].nbytes
    _check(_load().oracle_copy_blocks(_ptr(key_cache), _ptr(value_cache), block_bytes, nb,
                                      _ptr(pairs), pairs.shape[0]), "copy_blocks")


def swap_blocks(dst_key: np.ndarray, dst_value: np.ndarray, src_key: np.ndarray,
                src_value: np.ndarray, src_dst_pairs: np.ndarray) -> None:
    """In place on dst_key/dst_value ([NB', B, H, D]); blocks copied from the source pools."""
    assert dst_key.shape[1:] == src_key.shape[1:] and dst_key.dtype == src_key.dtype
    pairs = np.ascontiguousarray(src_dst_pairs, dtype=np.int32).reshape(-1, 2)
    _check(_load().oracle_swap_blocks(_ptr(dst_key), _ptr(dst_value), dst_key.shape[0],
                                      _ptr(src_key), _ptr(src_value), src_key.shape[0],
                                      src_key[0].nbytes, _ptr(pairs), pairs.shape[0]), "swap_blocks")


def max_threads() -> int:
    """Threads the oracle's threaded calls use by default on this host."""
    return int(_load().oracle_max_threads())


def paged_attention(query: np.ndarray, key_cache: np.ndarray, value_cache: np.ndarray,
                    block_tables: np.ndarray, context_lens: np.ndarray, scale: float,
                    k_scale: float = 1.0, v_scale: float = 1.0,
                    seq_head: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    """Returns float64 [S, H, D], or [n, D] for an explicit (s, h) list.
    threads=None runs on the calling thread; threads=n (0: the host's
    default) spreads the (s, h) pairs over n OpenMP threads, each pair
    computed by the same code, so the result is the same bit for bit."""
    assert query.dtype == np.float16
    q = np.ascontiguousarray(query)
    nb, bs, nh, hd = key_cache.shape
    S = q.shape[0]
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    pairs = None if seq_head is None else np.ascontiguousarray(seq_head, dtype=np.int32).reshape(-1, 2)
    n = S * nh if pairs is None else pairs.shape[0]
    out = np.empty((n, hd), np.float64)
    args = (_ptr(out), _ptr(q.view(np.uint16)), _ptr(key_cache), _ptr(value_cache),
            _dtype_code(key_cache), nb, bs, nh, hd, _ptr(bt), bt.shape[1], _ptr(ctx), S,
            float(np.float32(scale)), float(np.float32(k_scale)), float(np.float32(v_scale)),
            _ptr(pairs), 0 if pairs is None else pairs.shape[0])
    if threads is None:
        rc = _load().oracle_paged_attention(*args)
    else:
        rc = _load().oracle_paged_attention_threads(*args, int(threads))
    _check(rc, "paged_attention")
    return out.reshape(S, nh, hd) if pairs is None else out


def paged_prefill(query: np.ndarray, query_start: np.ndarray, key_cache: np.ndarray,
                  value_cache: np.ndarray, block_tables: np.ndarray, context_lens: np.ndarray,
                  scale: float, k_scale: float = 1.0, v_scale: float = 1.0,
                  row_head: np.ndarray | None = None) -> np.ndarray:
    """Causal attention of packed query rows: float64 [total_q, H, D], or [n, D]
    for an explicit (row, head) list."""
    assert query.dtype == np.float16
    q = np.ascontiguousarray(query)
    nb, bs, nh, hd = key_cache.shape
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    S = qs.shape[0] - 1
    assert q.shape[0] == int(qs[-1])
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    pairs = None if row_head is None else np.ascontiguousarray(row_head, dtype=np.int32).reshape(-1, 2)
    n = q.shape[0] * nh if pairs is None else pairs.shape[0]
    out = np.empty((n, hd), np.float64)
    rc = _load().oracle_paged_prefill(
        _ptr(out), _ptr(q.view(np.uint16)), _ptr(qs), _ptr(key_cache), _ptr(value_cache),
        _dtype_code(key_cache), nb, bs, nh, hd, _ptr(bt), bt.shape[1], _ptr(ctx), S,
        float(np.float32(scale)), float(np.float32(k_scale)), float(np.float32(v_scale)),
        _ptr(pairs), 0 if pairs is None else pairs.shape[0])
    _check(rc, "paged_prefill")
    return out.reshape(q.shape[0], nh, hd) if pairs is None else out


def attention_partials(query, key_cache, value_cache, block_tables, context_lens, scale,
                       partition_size: int, k_scale: float = 1.0, v_scale: float = 1.0):
    """Per-partition (o_p, lse_p) of every (s, h): o [S,H,P,D], lse [S,H,P] (natural log)."""
    q = np.ascontiguousarray(query)
    nb, bs, nh, hd = key_cache.shape
    S = q.shape[0]
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    ctx = np.ascontiguousarray(context_lens, dtype=np.int32)
    max_parts = max(1, int(-(-int(ctx.max(initial=0)) // partition_size)))
    o = np.empty((S, nh, max_parts, hd), np.float64)
    lse = np.empty((S, nh, max_parts), np.float64)
    rc = _load().oracle_attention_partials(
        _ptr(o), _ptr(lse), _ptr(q.view(np.uint16)), _ptr(key_cache), _ptr(value_cache),
        _dtype_code(key_cache), nb, bs, nh, hd, _ptr(bt), bt.shape[1], _ptr(ctx), S,
        float(np.float32(scale)), float(np.float32(k_scale)), float(np.float32(v_scale)),
        partition_size, max_parts)
    _check(rc, "attention_partials")
    return o, lse


def lse_combine(o_parts: np.ndarray, lse_parts: np.ndarray) -> np.ndarray:
    """Combine n partials of one (s, h): o_parts [n, D], lse_parts [n] -> [D]."""
    o = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse = np.ascontiguousarray(lse_parts, dtype=np.float64)
    out = np.empty(o.shape[1], np.float64)
    _load().oracle_lse_combine(_ptr(out), _ptr(o), _ptr(lse), o.shape[0], o.shape[1])
    return out
