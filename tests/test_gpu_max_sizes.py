"""Decode at the documented maximum sizes of a call, against the oracle.

- num_seqs = 65535, the most one decode launch takes (its grid's units are
  sequences x head groups x partitions), with ragged short contexts;
- contexts that fill their table row exactly (L = max_blocks_per_seq *
  block_size), in a batch where the bound passed is that capacity;
- head_size 64 and 128, fp16 and E4M3 caches.
Whole outputs are compared; slots and the written rows bit-exact.
"""
import numpy as np
import pytest

import pagedattention_paged_kv_decode_b200 as pk
import workloads as W
from _oracle_step import oracle_step

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "e4m3": 1e-2}


def _check(w, dev):
    dw = W.to_device(w, dev, encode=pk.load_cache)
    bound = w.max_blocks_per_seq * w.block_size
    pk.paged_attention_decode_append(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache,
                                     dw.value_cache, dw.block_tables, dw.context_lens, w.scale,
                                     w.k_scale, w.v_scale, max_context_len=bound, slot_mapping=dw.slots)
    assert pk.check_status() == 0
    slots, kc, vc, out_ref, _ = oracle_step(w)
    assert np.array_equal(dw.slots.cpu().numpy(), slots)
    got = dw.out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.abs(got - out_ref).max() <= TOL[w.kv_dtype]


@pytest.mark.parametrize("kv", ["f16", "e4m3"])
def test_most_sequences_one_call_takes(cuda_device, kv):
    S, H, D, B = 65535, 2, 64, 16
    ctx = np.random.default_rng(5).integers(1, 41, S)
    need = int(sum(-(-int(L) // B) for L in ctx))
    w = W.build(f"max_seqs_{kv}", H, D, B, kv, ctx, need + 8, 3, 61, q_std=1.0, kv_std=1.0)
    _check(w, cuda_device)


@pytest.mark.parametrize("D,B,kv", [(128, 16, "f16"), (64, 32, "e4m3"), (128, 32, "f16")])
def test_contexts_that_fill_their_table_row(cuda_device, D, B, kv):
    width = 40
    ctx = [width * B, width * B, 1, width * B - 1, (width - 1) * B + 1, width * B // 2 + 3]
    need = sum(-(-L // B) for L in ctx)
    w = W.build(f"full_rows_{kv}_d{D}_b{B}", 4, D, B, kv, ctx, need + 5, width, 62, q_std=1.0, kv_std=1.0)
    _check(w, cuda_device)
