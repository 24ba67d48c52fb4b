"""Paged-KV decode attention for NVIDIA B200 (sm_100a), with the cache
write, slot derivation, block copy and swap around it and a paged prefill.

The calls below marshal torch tensors into the C ABI of ``libpagedkv.so``
(``include/pagedkv.h``); every step runs in that library's CUDA kernels.
Importing this package does not touch the GPU; the first call loads the
library and fails loudly if it has not been built.
"""
from .capi import PagedKVError  # noqa: F401
from .ops import (  # noqa: F401
    cache_desc,
    check_status,
    choose_config,
    decode_choose_config,
    copy_blocks,
    decode_step,
    decode_workspace_size,
    kv_cache_write,
    last_error,
    load_cache,
    paged_attention_decode,
    paged_attention_decode_append,
    paged_attention_decode_noalloc,
    paged_attention_decode_shared_prefix,
    paged_attention_decode_ws,
    paged_prefill,
    prefill_slot_mapping,
    prefill_step,
    shared_prefix_workspace_size,
    slot_mapping,
    swap_blocks,
    test_stall_next_decode,
    version,
)
