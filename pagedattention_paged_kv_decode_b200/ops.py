"""Torch-tensor binding of the C ABI: the same calls, argument marshalling only.

Every function validates dtype/device/shape of the tensors it is given, then
passes raw device pointers, sizes and the current CUDA stream to the
library; all work runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import capi
from .capi import CacheDesc, DecodeConfig, check, lib

_E4M3_DTYPES = (torch.uint8, torch.float8_e4m3fn)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def cache_desc(key_cache: torch.Tensor) -> CacheDesc:
    if key_cache.dim() != 4:
        raise ValueError("caches are [num_blocks, block_size, num_heads, head_size]")
    if key_cache.dtype == torch.float16:
        dt = capi.PA_F16
    elif key_cache.dtype in _E4M3_DTYPES:
        dt = capi.PA_E4M3
    else:
        raise TypeError(f"cache dtype {key_cache.dtype}: use float16, or uint8/float8_e4m3fn for E4M3")
    nb, bs, nh, hd = key_cache.shape
    return CacheDesc(nb, bs, nh, hd, dt)


def _check_pair(key_cache, value_cache):
    if key_cache.shape != value_cache.shape or key_cache.dtype != value_cache.dtype:
        raise ValueError("key_cache and value_cache differ in shape or dtype")
    for t in (key_cache, value_cache):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("caches must be contiguous CUDA tensors")


def _i32(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
    return t


def _on_current_device(*tensors) -> None:
    """The library launches on the current CUDA device; a device tensor on
    another GPU would be a foreign pointer there."""
    dev = None
    for t in tensors:
        if t is None or not t.is_cuda:
            continue
        if dev is None:
            dev = torch.cuda.current_device()
        if t.device.index != dev:
            raise ValueError(f"a tensor is on {t.device}, but the current CUDA device is cuda:{dev}")


def _table(block_tables: torch.Tensor, S: int) -> None:
    _i32(block_tables, "block_tables")
    if block_tables.dim() != 2 or block_tables.shape[0] < S:
        raise ValueError("block_tables must be int32 [num_seqs, max_blocks_per_seq]")


def _f16_rows(t: torch.Tensor, name: str, shape) -> None:
    """fp16 CUDA [n, H, D] of the given shape, each token's row contiguous
    (the token stride is free)."""
    if t.dtype != torch.float16 or not t.is_cuda or t.dim() != 3:
        raise ValueError(f"{name} must be a float16 CUDA tensor [n, H, D]")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.stride(2) != 1 or t.stride(1) != t.shape[2]:
        raise ValueError(f"{name} rows must be contiguous within a token")


def _slots_out(slot_mapping: torch.Tensor | None, S: int) -> None:
    if slot_mapping is not None:
        _i32(slot_mapping, "slot_mapping")
        if slot_mapping.dim() != 1 or slot_mapping.shape[0] < S:
            raise ValueError("slot_mapping must be int32 [num_seqs]")


def _workspace(workspace: torch.Tensor | None):
    if workspace is None:
        return None, 0
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return workspace.data_ptr(), workspace.numel() * workspace.element_size()


def _pairs(src_dst_pairs: torch.Tensor) -> None:
    _i32(src_dst_pairs, "src_dst_pairs")
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be int32 [n_pairs, 2]")


def slot_mapping(block_tables: torch.Tensor, context_lens: torch.Tensor, key_cache: torch.Tensor,
                 out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Slot of each sequence's appended token (position context_len - 1)."""
    _i32(context_lens, "context_lens")
    S = context_lens.shape[0]
    _table(block_tables, S)
    if out is None:
        out = torch.empty(S, dtype=torch.int32, device=context_lens.device)
    _slots_out(out, S)
    _on_current_device(block_tables, context_lens, out)
    check(lib().pa_slot_mapping(out.data_ptr(), block_tables.data_ptr(), block_tables.shape[1],
                                context_lens.data_ptr(), S, cache_desc(key_cache), _stream(stream)))
    return out


def kv_cache_write(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                   value_cache: torch.Tensor, slot_mapping: torch.Tensor,
                   k_scale: float = 1.0, v_scale: float = 1.0, stream=None) -> None:
    """Scatter new K/V rows ([n, H, D] fp16, row stride free) into their slots."""
    _check_pair(key_cache, value_cache)
    _i32(slot_mapping, "slot_mapping")
    n = slot_mapping.shape[0]
    _, _, H, D = key_cache.shape
    _f16_rows(key, "key", (n, H, D))
    _f16_rows(value, "value", (n, H, D))
    _on_current_device(key, value, key_cache, value_cache, slot_mapping)
    check(lib().pa_kv_cache_write(key.data_ptr(), value.data_ptr(), key.stride(0), value.stride(0),
                                  key_cache.data_ptr(), value_cache.data_ptr(), cache_desc(key_cache),
                                  slot_mapping.data_ptr(), n, float(k_scale), float(v_scale),
                                  _stream(stream)))


def copy_blocks(key_cache: torch.Tensor, value_cache: torch.Tensor, src_dst_pairs: torch.Tensor,
                stream=None) -> None:
    """Copy whole physical blocks (both caches) for each (src, dst) pair."""
    _check_pair(key_cache, value_cache)
    _pairs(src_dst_pairs)
    n = src_dst_pairs.shape[0]
    _on_current_device(key_cache, value_cache, src_dst_pairs)
    check(lib().pa_copy_blocks(key_cache.data_ptr(), value_cache.data_ptr(), cache_desc(key_cache),
                               src_dst_pairs.data_ptr(), n, _stream(stream)))


def swap_blocks(dst_key_cache: torch.Tensor, dst_value_cache: torch.Tensor,
                src_key_cache: torch.Tensor, src_value_cache: torch.Tensor,
                src_dst_pairs: torch.Tensor, stream=None) -> None:
    """Copy whole blocks from the source pools into the destination pools.

    One side may be a pinned CPU tensor (``pin_memory()``), which the kernel
    reads or writes over the host link; ``src_dst_pairs`` is int32 [n, 2] on
    the device."""
    for a, b in ((dst_key_cache, dst_value_cache), (src_key_cache, src_value_cache)):
        if a.shape != b.shape or a.dtype != b.dtype or not a.is_contiguous() or not b.is_contiguous():
            raise ValueError("key/value pools of one side differ or are not contiguous")
        if not a.is_cuda and not a.is_pinned():
            raise ValueError("a CPU pool must be pinned (pin_memory())")
    if dst_key_cache.shape[1:] != src_key_cache.shape[1:] or dst_key_cache.dtype != src_key_cache.dtype:
        raise ValueError("source and destination block shapes differ")
    _pairs(src_dst_pairs)
    n = src_dst_pairs.shape[0]
    _on_current_device(dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, src_dst_pairs)
    check(lib().pa_swap_blocks(dst_key_cache.data_ptr(), dst_value_cache.data_ptr(),
                               dst_key_cache.shape[0], src_key_cache.data_ptr(),
                               src_value_cache.data_ptr(), src_key_cache.shape[0],
                               cache_desc(src_key_cache), src_dst_pairs.data_ptr(), n,
                               _stream(stream)))


def _config(config) -> DecodeConfig | None:
    if config is None:
        return None
    if isinstance(config, DecodeConfig):
        return config
    return DecodeConfig(**{k: int(config.get(k, 0)) for k, _ in DecodeConfig._fields_})


def choose_config(key_cache: torch.Tensor, num_seqs: int, max_context_len: int, config=None) -> dict:
    cfg = _config(config) or DecodeConfig(0, 0, 0, 0, 0)
    check(lib().pa_decode_choose_config(cache_desc(key_cache), num_seqs, max_context_len,
                                        ctypes.byref(cfg)))
    return cfg.as_dict()


def decode_choose_config(key_cache: torch.Tensor, num_seqs: int, max_context_len: int, config=None) -> dict:
    """The launch shape the decode would use (``choose_config`` under the C
    entry point's name)."""
    return choose_config(key_cache, num_seqs, max_context_len, config)


def decode_workspace_size(key_cache: torch.Tensor, num_seqs: int, max_context_len: int,
                          config=None) -> int:
    cfg = _config(config)
    return int(lib().pa_decode_workspace_size(cache_desc(key_cache), num_seqs, max_context_len,
                                              ctypes.byref(cfg) if cfg is not None else None))


def _decode_args(out, query, key_cache, value_cache, block_tables, context_lens, scale, k_scale, v_scale,
                 max_context_len, workspace=None) -> tuple:
    """Checks of a plain decode call; returns its C arguments up to the
    launch options (the stream, and for the _ws call config and workspace)."""
    _check_pair(key_cache, value_cache)
    _i32(block_tables, "block_tables")
    _i32(context_lens, "context_lens")
    for t in (out, query):
        if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("out and query must be contiguous float16 CUDA tensors")
    S, H, D = query.shape
    if out.shape != query.shape or context_lens.shape[0] != S or block_tables.shape[0] != S:
        raise ValueError("shape mismatch between out, query, block_tables and context_lens")
    _table(block_tables, S)
    desc = cache_desc(key_cache)
    if desc.num_heads != H or desc.head_size != D:
        raise ValueError("query heads/head_size differ from the cache's")
    if max_context_len is None:
        max_context_len = block_tables.shape[1] * desc.block_size
    _on_current_device(out, query, key_cache, value_cache, block_tables, context_lens, workspace)
    return (out.data_ptr(), query.data_ptr(), key_cache.data_ptr(), value_cache.data_ptr(), desc,
            block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(), S,
            int(max_context_len), float(scale), float(k_scale), float(v_scale))


def paged_attention_decode(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                           value_cache: torch.Tensor, block_tables: torch.Tensor,
                           context_lens: torch.Tensor, scale: float, k_scale: float = 1.0,
                           v_scale: float = 1.0, max_context_len: int | None = None,
                           config=None, workspace: torch.Tensor | None = None, stream=None) -> None:
    """Decode attention into ``out`` ([S, H, D] fp16).

    ``max_context_len`` is a host-side bound on every context length; by
    default the table capacity ``block_tables.shape[1] * block_size`` (no
    device sync). With ``config`` or ``workspace`` given, the caller-workspace
    entry point is used (``workspace`` a uint8 CUDA tensor of at least
    ``decode_workspace_size`` bytes).
    """
    if config is not None or workspace is not None:
        paged_attention_decode_ws(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                                  k_scale, v_scale, max_context_len, config, workspace, stream)
        return
    args = _decode_args(out, query, key_cache, value_cache, block_tables, context_lens, scale, k_scale,
                        v_scale, max_context_len)
    check(lib().pa_paged_attention_decode(*args, _stream(stream)))


def paged_attention_decode_ws(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                              value_cache: torch.Tensor, block_tables: torch.Tensor,
                              context_lens: torch.Tensor, scale: float, k_scale: float = 1.0,
                              v_scale: float = 1.0, max_context_len: int | None = None,
                              config=None, workspace: torch.Tensor | None = None, stream=None) -> None:
    """Decode with an explicit launch shape (``config``: a dict or DecodeConfig,
    zero fields = library choice) and/or a caller workspace (a contiguous
    CUDA tensor of at least ``decode_workspace_size`` bytes, 256-byte
    aligned); either may be None."""
    args = _decode_args(out, query, key_cache, value_cache, block_tables, context_lens, scale, k_scale,
                        v_scale, max_context_len, workspace)
    cfg = _config(config)
    ws_ptr, ws_bytes = _workspace(workspace)
    check(lib().pa_paged_attention_decode_ws(*args, ctypes.byref(cfg) if cfg is not None else None,
                                             ws_ptr, ws_bytes, _stream(stream)))


def paged_attention_decode_noalloc(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                                   value_cache: torch.Tensor, block_tables: torch.Tensor,
                                   context_lens: torch.Tensor, scale: float, k_scale: float = 1.0,
                                   v_scale: float = 1.0, max_context_len: int | None = None,
                                   stream=None) -> None:
    """``paged_attention_decode`` that allocates nothing (library-chosen launch
    shape). The split partials go to a 16 MiB static array inside the
    library, one per device: a larger decode is rejected before any launch,
    calls whose kernels may overlap (other streams or threads) must be
    serialised, and the first call on a device must precede any stream
    capture (it looks up the array's address)."""
    args = _decode_args(out, query, key_cache, value_cache, block_tables, context_lens, scale, k_scale,
                        v_scale, max_context_len)
    check(lib().pa_paged_attention_decode_noalloc(*args, _stream(stream)))


def paged_attention_decode_append(out: torch.Tensor, query: torch.Tensor, new_key: torch.Tensor,
                                  new_value: torch.Tensor, key_cache: torch.Tensor,
                                  value_cache: torch.Tensor, block_tables: torch.Tensor,
                                  context_lens: torch.Tensor, scale: float, k_scale: float = 1.0,
                                  v_scale: float = 1.0, max_context_len: int | None = None,
                                  slot_mapping: torch.Tensor | None = None, config=None,
                                  workspace: torch.Tensor | None = None, stream=None) -> None:
    """Fused step: slot of each appended token, its K/V store, and the decode.

    ``slot_mapping`` (int32 [S], optional) receives the slots."""
    _check_pair(key_cache, value_cache)
    _i32(block_tables, "block_tables")
    _i32(context_lens, "context_lens")
    for t in (out, query):
        if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("out and query must be contiguous float16 CUDA tensors")
    S, H, D = query.shape
    for t in (new_key, new_value):
        if t.dtype != torch.float16 or not t.is_cuda or tuple(t.shape) != (S, H, D):
            raise ValueError("new_key/new_value must be float16 CUDA tensors [S, H, D]")
        if t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError("new_key/new_value rows must be contiguous within a token")
    if out.shape != query.shape or context_lens.shape[0] != S or block_tables.shape[0] != S:
        raise ValueError("shape mismatch between out, query, block_tables and context_lens")
    _table(block_tables, S)
    desc = cache_desc(key_cache)
    if desc.num_heads != H or desc.head_size != D:
        raise ValueError("query heads/head_size differ from the cache's")
    if max_context_len is None:
        max_context_len = block_tables.shape[1] * desc.block_size
    _slots_out(slot_mapping, S)
    cfg = _config(config)
    ws_ptr, ws_bytes = _workspace(workspace)
    _on_current_device(out, query, new_key, new_value, key_cache, value_cache, block_tables, context_lens,
                       slot_mapping, workspace)
    check(lib().pa_paged_attention_decode_append(
        out.data_ptr(), query.data_ptr(), new_key.data_ptr(), new_value.data_ptr(),
        new_key.stride(0), new_value.stride(0), key_cache.data_ptr(), value_cache.data_ptr(), desc,
        block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(), S,
        int(max_context_len), float(scale), float(k_scale), float(v_scale),
        slot_mapping.data_ptr() if slot_mapping is not None else None,
        ctypes.byref(cfg) if cfg is not None else None, ws_ptr, ws_bytes, _stream(stream)))


def shared_prefix_workspace_size(key_cache: torch.Tensor, num_seqs: int, max_context_len: int,
                                 shared_prefix_blocks: int, config=None) -> int:
    """Workspace bytes of a ``paged_attention_decode_shared_prefix`` call (0 on
    invalid arguments)."""
    cfg = _config(config)
    return int(lib().pa_shared_prefix_workspace_size(cache_desc(key_cache), int(num_seqs), int(max_context_len),
                                                     int(shared_prefix_blocks),
                                                     ctypes.byref(cfg) if cfg is not None else None))


def paged_attention_decode_shared_prefix(out: torch.Tensor, query: torch.Tensor,
                                         key_cache: torch.Tensor, value_cache: torch.Tensor,
                                         block_tables: torch.Tensor, context_lens: torch.Tensor,
                                         shared_prefix_blocks: int, scale: float,
                                         k_scale: float = 1.0, v_scale: float = 1.0,
                                         new_key: torch.Tensor | None = None,
                                         new_value: torch.Tensor | None = None,
                                         max_context_len: int | None = None,
                                         slot_mapping: torch.Tensor | None = None, config=None,
                                         workspace: torch.Tensor | None = None, stream=None) -> None:
    """Decode (with the fused append when new_key/new_value are given) for a
    batch whose tables all start with the same ``shared_prefix_blocks`` blocks."""
    _check_pair(key_cache, value_cache)
    _i32(block_tables, "block_tables")
    _i32(context_lens, "context_lens")
    for t in (out, query):
        if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("out and query must be contiguous float16 CUDA tensors")
    S, H, D = query.shape
    if (new_key is None) != (new_value is None):
        raise ValueError("give both new_key and new_value, or neither")
    for t in (new_key, new_value):
        if t is not None and (t.dtype != torch.float16 or not t.is_cuda or tuple(t.shape) != (S, H, D)
                              or t.stride(2) != 1 or t.stride(1) != D):
            raise ValueError("new_key/new_value must be float16 CUDA tensors [S, H, D] with contiguous rows")
    if out.shape != query.shape or context_lens.shape[0] != S or block_tables.shape[0] != S:
        raise ValueError("shape mismatch between out, query, block_tables and context_lens")
    _table(block_tables, S)
    desc = cache_desc(key_cache)
    if desc.num_heads != H or desc.head_size != D:
        raise ValueError("query heads/head_size differ from the cache's")
    if max_context_len is None:
        max_context_len = block_tables.shape[1] * desc.block_size
    _slots_out(slot_mapping, S)
    cfg = _config(config)
    ws_ptr, ws_bytes = _workspace(workspace)
    _on_current_device(out, query, new_key, new_value, key_cache, value_cache, block_tables, context_lens,
                       slot_mapping, workspace)
    check(lib().pa_paged_attention_decode_shared_prefix(
        out.data_ptr(), query.data_ptr(),
        new_key.data_ptr() if new_key is not None else None,
        new_value.data_ptr() if new_value is not None else None,
        new_key.stride(0) if new_key is not None else H * D,
        new_value.stride(0) if new_value is not None else H * D,
        key_cache.data_ptr(), value_cache.data_ptr(), desc, block_tables.data_ptr(),
        block_tables.shape[1], context_lens.data_ptr(), S, int(max_context_len),
        int(shared_prefix_blocks), float(scale), float(k_scale), float(v_scale),
        slot_mapping.data_ptr() if slot_mapping is not None else None,
        ctypes.byref(cfg) if cfg is not None else None, ws_ptr, ws_bytes, _stream(stream)))


def check_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device error bits (PA_DEV_*)."""
    code = ctypes.c_uint32(0)
    check(lib().pa_check_status(_stream(stream), ctypes.byref(code)))
    return int(code.value)


def version() -> int:
    return int(lib().pa_version())


def test_stall_next_decode(seq: int, head: int = 0, partition: int = 0, wait_limit_ns: int = 1_000_000) -> None:
    """Test hook of the bounded waits: the next decode launched on this
    thread issues no tile loads for the work unit holding (seq, head,
    partition) and limits each wait to wait_limit_ns; that unit then reports
    PA_DEV_WAIT_TIMEOUT and its output rows are undefined. seq < 0 clears a
    pending request."""
    if int(seq) >= 0:
        if int(head) < 0 or int(partition) < 0:
            raise ValueError(f"head {head} and partition {partition} must be >= 0")
        if not 1000 <= int(wait_limit_ns) <= 2_000_000_000:
            raise ValueError(f"wait_limit_ns {wait_limit_ns} outside [1000, 2e9]")
    check(lib().pa_test_stall_next_decode(int(seq), int(head), int(partition), int(wait_limit_ns)))


def last_error() -> str:
    """Message of the last nonzero status on this thread ("" if none); the
    binding also raises it as PagedKVError."""
    return lib().pa_last_error().decode(errors="replace")


def load_cache(key_cache: torch.Tensor, value_cache: torch.Tensor, key_src: torch.Tensor,
               value_src: torch.Tensor, k_scale: float = 1.0, v_scale: float = 1.0,
               stream=None) -> None:
    """Write whole fp16 pools [NB, B, H, D] into the caches, slot by slot.

    This is ``kv_cache_write`` with the identity slot list, in slices of at
    most 65535 tokens (the slot list stays small); for E4M3 caches it
    quantises with the given scales.
    """
    _check_pair(key_cache, value_cache)
    nb, bs, nh, hd = key_cache.shape
    if key_src.shape != key_cache.shape or value_src.shape != key_cache.shape:
        raise ValueError("source pools must have the cache's shape")
    n = nb * bs
    ks = key_src.reshape(n, nh, hd)
    vs = value_src.reshape(n, nh, hd)
    chunk = 65535
    slots = torch.arange(min(n, chunk), dtype=torch.int32, device=key_cache.device)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        kv_cache_write(ks[i:i + m], vs[i:i + m], key_cache, value_cache, slots[:m] + i,
                       k_scale, v_scale, stream)


def decode_step(out: torch.Tensor, query: torch.Tensor, new_key: torch.Tensor,
                new_value: torch.Tensor, key_cache: torch.Tensor, value_cache: torch.Tensor,
                block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                k_scale: float = 1.0, v_scale: float = 1.0, cow_pairs: torch.Tensor | None = None,
                slots: torch.Tensor | None = None, max_context_len: int | None = None,
                config=None, workspace: torch.Tensor | None = None, stream=None,
                fused: bool = True, shared_prefix_blocks: int = 0) -> torch.Tensor:
    """One decode step of the whole path, all on the device, in order:
    copy-on-write block copies (if any pairs), slot of each appended token,
    scatter of the new K/V rows into those slots, decode attention.
    ``block_tables`` are the tables after any copy-on-write repoint. With
    ``fused`` the last three run as one launch (paged_attention_decode_append);
    otherwise as three separate calls. With ``shared_prefix_blocks`` > 0 the
    decode reads the shared prefix once per head (paged_attention_decode_shared_prefix).
    Returns the slot tensor."""
    if cow_pairs is not None and cow_pairs.numel():
        copy_blocks(key_cache, value_cache, cow_pairs, stream)
    if shared_prefix_blocks:
        if slots is None:
            slots = torch.empty(query.shape[0], dtype=torch.int32, device=query.device)
        paged_attention_decode_shared_prefix(out, query, key_cache, value_cache, block_tables,
                                             context_lens, shared_prefix_blocks, scale, k_scale,
                                             v_scale, new_key, new_value, max_context_len, slots,
                                             config, workspace, stream)
        return slots
    if fused:
        if slots is None:
            slots = torch.empty(query.shape[0], dtype=torch.int32, device=query.device)
        paged_attention_decode_append(out, query, new_key, new_value, key_cache, value_cache,
                                      block_tables, context_lens, scale, k_scale, v_scale,
                                      max_context_len, slots, config, workspace, stream)
        return slots
    slots = slot_mapping(block_tables, context_lens, key_cache, out=slots, stream=stream)
    kv_cache_write(new_key, new_value, key_cache, value_cache, slots, k_scale, v_scale, stream)
    paged_attention_decode(out, query, key_cache, value_cache, block_tables, context_lens, scale,
                           k_scale, v_scale, max_context_len, config, workspace, stream)
    return slots


# ------------------------------------------------------------ paged prefill

def prefill_slot_mapping(query_start: torch.Tensor, block_tables: torch.Tensor,
                         context_lens: torch.Tensor, key_cache: torch.Tensor,
                         max_query_len: int, out: torch.Tensor | None = None,
                         total_q: int | None = None, stream=None) -> torch.Tensor:
    """Slot of every new token of a prefill chunk ([total_q] int32).

    ``total_q`` (= query_start[-1]) must be given when ``out`` is not, since
    reading it from the device would synchronise."""
    _i32(query_start, "query_start")
    _i32(context_lens, "context_lens")
    S = context_lens.shape[0]
    _table(block_tables, S)
    if query_start.dim() != 1 or query_start.shape[0] != S + 1 or block_tables.shape[0] != S:
        raise ValueError("query_start must hold num_seqs + 1 entries and block_tables num_seqs rows")
    if out is None:
        if total_q is None:
            raise ValueError("give out or total_q")
        out = torch.empty(int(total_q), dtype=torch.int32, device=context_lens.device)
    _i32(out, "out")
    if out.dim() != 1 or (total_q is not None and out.shape[0] != int(total_q)):
        raise ValueError("out must be a 1-D int32 tensor of total_q entries")
    _on_current_device(query_start, block_tables, context_lens, out)
    check(lib().pa_prefill_slot_mapping(out.data_ptr(), query_start.data_ptr(), block_tables.data_ptr(),
                                        block_tables.shape[1], context_lens.data_ptr(), S, out.shape[0],
                                        int(max_query_len), cache_desc(key_cache), _stream(stream)))
    return out


def paged_prefill(out: torch.Tensor, query: torch.Tensor, query_start: torch.Tensor,
                  key_cache: torch.Tensor, value_cache: torch.Tensor, block_tables: torch.Tensor,
                  context_lens: torch.Tensor, max_query_len: int, scale: float, stream=None) -> None:
    """Causal attention of packed query rows ([total_q, H, D] fp16) over the
    paged fp16 cache, which must already hold each sequence's chunk."""
    _check_pair(key_cache, value_cache)
    _i32(query_start, "query_start")
    _i32(context_lens, "context_lens")
    for t in (out, query):
        if t.dtype != torch.float16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3:
            raise ValueError("out and query must be contiguous float16 CUDA tensors [total_q, H, D]")
    S = context_lens.shape[0]
    _table(block_tables, S)
    if (out.shape != query.shape or query_start.dim() != 1 or query_start.shape[0] != S + 1
            or block_tables.shape[0] != S):
        raise ValueError("shape mismatch between out, query, query_start, block_tables and context_lens")
    desc = cache_desc(key_cache)
    if desc.num_heads != query.shape[1] or desc.head_size != query.shape[2]:
        raise ValueError("query heads/head_size differ from the cache's")
    _on_current_device(out, query, query_start, key_cache, value_cache, block_tables, context_lens)
    check(lib().pa_paged_prefill(out.data_ptr(), query.data_ptr(), query_start.data_ptr(),
                                 key_cache.data_ptr(), value_cache.data_ptr(), desc, block_tables.data_ptr(),
                                 block_tables.shape[1], context_lens.data_ptr(), S, query.shape[0],
                                 int(max_query_len), float(scale), _stream(stream)))


def prefill_step(out: torch.Tensor, query: torch.Tensor, new_key: torch.Tensor, new_value: torch.Tensor,
                 query_start: torch.Tensor, key_cache: torch.Tensor, value_cache: torch.Tensor,
                 block_tables: torch.Tensor, context_lens: torch.Tensor, max_query_len: int,
                 scale: float, slots: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One prefill step on the device, in order: slots of the chunk's tokens,
    scatter of their K/V rows into the cache, causal attention. Returns the
    slot tensor."""
    T = query.shape[0]
    slots = prefill_slot_mapping(query_start, block_tables, context_lens, key_cache, max_query_len,
                                 out=slots, total_q=T, stream=stream)
    kv_cache_write(new_key, new_value, key_cache, value_cache, slots, stream=stream)
    paged_prefill(out, query, query_start, key_cache, value_cache, block_tables, context_lens,
                  max_query_len, scale, stream)
    return slots
