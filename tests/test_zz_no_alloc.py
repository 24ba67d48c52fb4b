"""The decode entry point that allocates nothing (pa_paged_attention_decode_noalloc).

It serves callers that may not allocate device memory on the decode path --
engine plugins whose framework owns every buffer, code under CUDA stream
capture, fixed-memory-plan loops. Its split partials live in a static array
inside the library. This file is collected last on purpose, and every test
here must pass both alone in a fresh process and after the rest of the suite.

The check: through the C ABI, two calls in a row with different batches that
both need the split path, each compared with the CPU oracle and with the
allocating entry point pa_paged_attention_decode on the same inputs
(max-abs 2e-3, the fp16-KV tolerance of the parity tests), the clear
rejection of a batch whose partials exceed the static scratch, and the torch
binding giving the C call's result bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
import pagedattention_paged_kv_decode_b200 as pk
from pagedattention_paged_kv_decode_b200 import capi
import workloads as W

pytestmark = pytest.mark.gpu


def _batch(dev, seed, ctx):
    B, H, D = 16, 8, 128
    need = sum(-(-int(L) // B) for L in ctx)
    w = W.build(f"noalloc{seed}", H, D, B, "f16", ctx, need + 4, -(-max(ctx) // B), seed,
                q_std=0.5, kv_std=0.5)
    dw = W.to_device(w, dev)
    pk.slot_mapping(dw.block_tables, dw.context_lens, dw.key_cache, out=dw.slots)
    pk.kv_cache_write(dw.new_key, dw.new_value, dw.key_cache, dw.value_cache, dw.slots)
    return w, dw


def _args(w, dw, out):
    return (out.data_ptr(), dw.query.data_ptr(), dw.key_cache.data_ptr(), dw.value_cache.data_ptr(),
            pk.cache_desc(dw.key_cache), dw.block_tables.data_ptr(), w.max_blocks_per_seq,
            dw.context_lens.data_ptr(), w.num_seqs, w.max_blocks_per_seq * w.block_size,
            w.scale, 1.0, 1.0)


def test_noalloc_matches_allocating_entry_point_two_calls(cuda_device):
    L = capi.lib()
    stream = torch.cuda.current_stream().cuda_stream
    batches = [_batch(cuda_device, 21, [1500, 33, 700, 2047, 512, 513]),
               _batch(cuda_device, 22, [900, 1800, 16, 1025])]
    for w, dw in batches:
        cfg = pk.choose_config(dw.key_cache, w.num_seqs, w.max_blocks_per_seq * w.block_size)
        assert -(-w.max_context_len // cfg["partition_size"]) > 1     # the split path (scratch) is used
        ref = torch.full_like(dw.out, float("nan"))
        got = torch.full_like(dw.out, float("nan"))
        assert L.pa_paged_attention_decode(*_args(w, dw, ref), stream) == 0, L.pa_last_error()
        rc = L.pa_paged_attention_decode_noalloc(*_args(w, dw, got), stream)
        assert rc == 0, L.pa_last_error()
        assert pk.check_status() == 0
        a = got.cpu().numpy().astype(np.float64)
        b = ref.cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all()
        assert np.abs(a - b).max() <= 2e-3
        assert np.abs(a - _oracle_out(w)).max() <= 2e-3


def _oracle_out(w):
    """The oracle's own slots, cache write and attention on the batch's inputs."""
    kc, vc = w.pool_host()
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, w.block_size)
    oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots)
    return oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, threads=0)


def test_noalloc_rejects_partials_beyond_the_static_scratch(cuda_device):
    L = capi.lib()
    desc = capi.CacheDesc(100000, 16, 32, 128, capi.PA_F16)
    need = L.pa_decode_workspace_size(desc, 1024, 32768, None)
    assert need > (16 << 20)
    p = 0x10000
    rc = L.pa_paged_attention_decode_noalloc(p, p, p, p, desc, p, 2048, p, 1024, 32768, 0.1, 1.0,
                                             1.0, None)
    assert rc == capi.PA_ERR_WORKSPACE
    assert b"static scratch" in L.pa_last_error()


def test_binding_gives_the_c_call_result(cuda_device):
    # the torch binding marshals the same arguments (its default bound is the
    # table capacity, as in _args): bit-identical outputs
    w, dw = _batch(cuda_device, 23, [600, 40, 1300])
    assert dw.block_tables.shape[1] == w.max_blocks_per_seq
    stream = torch.cuda.current_stream().cuda_stream
    a = torch.full_like(dw.out, float("nan"))
    b = torch.full_like(dw.out, float("nan"))
    assert capi.lib().pa_paged_attention_decode_noalloc(*_args(w, dw, a), stream) == 0
    pk.paged_attention_decode_noalloc(b, dw.query, dw.key_cache, dw.value_cache, dw.block_tables,
                                      dw.context_lens, w.scale)
    assert pk.check_status() == 0
    assert torch.equal(a, b)
