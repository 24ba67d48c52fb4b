"""Pins for the oracle's paged prefill: prefill slot mapping and causal
multi-query attention over the block table.

The pages name FlashAttention-style attention as part of the path and a
32-token block size for long prompts, but print no formula. The oracle's
reading: row i of an n-token chunk of a sequence whose context is L tokens
sits at position L - n + i and attends tokens 0 .. L - n + i. It is pinned by
the worked slot example (a full prompt maps exactly the page's token ->
block table), equality with the decode slots for one-token chunks, torch's
CPU scaled_dot_product_attention with its own causal mask on identity tables
(full prompts) and with an explicit position mask (chunks after a cached
context), the closed form "position 0 -> V_0", brute force with exact
summation, relabelling of physical blocks, and the decode kernel's oracle for
the last row of every chunk.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def written_case(ctx, n, H=3, D=16, B=8, seed=0, deal="permuted", poison=W.POISON_HUGE):
    """A prefill step whose chunk K/V have been stored by the oracle's own steps."""
    ctx = np.asarray(ctx)
    need = sum(-(-int(L) // B) for L in ctx)
    w = W.build_prefill("case", H, D, B, ctx, n, need + 5, max(1, -(-int(ctx.max()) // B)), seed,
                        q_std=1.0, kv_std=1.0, poison=poison, deal_order=deal)
    kc, vc = w.pool_host()
    slots = oracle.prefill_slot_mapping(w.query_start, w.block_tables, w.context_lens, B)
    oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots)
    return w, kc, vc


def run(w, kc, vc, **kw):
    return oracle.paged_prefill(w.query, w.query_start, kc, vc, w.block_tables, w.context_lens, w.scale, **kw)


def test_full_prompt_slots_reproduce_the_worked_example():
    # sequence A: 32-token prompt in blocks 5, 8; sequence B: 16 tokens in block 3
    tables = np.array([[5, 8], [3, -1]], np.int32)
    got = oracle.prefill_slot_mapping(np.array([0, 32, 48], np.int32), tables, np.array([32, 16], np.int32), 16)
    want = {(sq, int(t)): int(sl) for sq, t, _, _, sl in _rows("slot_mapping_worked_example.txt")}
    assert [int(x) for x in got[:32]] == [want[("A", t)] for t in range(32)]
    assert [int(x) for x in got[32:]] == [want[("B", t)] for t in range(16)]


def test_one_token_chunks_give_the_decode_slots():
    w = W.build("d", 2, 8, 4, "f16", np.array([1, 4, 5, 13, 16]), 40, 4, 3, 1.0, 1.0)
    qs = np.arange(w.num_seqs + 1, dtype=np.int32)
    got = oracle.prefill_slot_mapping(qs, w.block_tables, w.context_lens, 4)
    np.testing.assert_array_equal(got, oracle.slot_mapping(w.block_tables, w.context_lens, 4))


def test_chunks_partition_the_prompt_slots():
    w = W.build_prefill("p", 2, 8, 4, [23], [23], 8, 6, 4, 1.0, 1.0)
    full = oracle.prefill_slot_mapping(w.query_start, w.block_tables, w.context_lens, 4)
    parts = []
    for L, n in [(9, 9), (20, 11), (23, 3)]:
        parts.append(oracle.prefill_slot_mapping(np.array([0, n], np.int32), w.block_tables,
                                                 np.array([L], np.int32), 4))
    np.testing.assert_array_equal(np.concatenate(parts), full)


def test_prefill_slot_mapping_rejects_chunk_longer_than_context():
    with pytest.raises(ValueError):
        oracle.prefill_slot_mapping(np.array([0, 5], np.int32), np.array([[0, 1]], np.int32),
                                    np.array([4], np.int32), 4)


def _dense(w, cache, s):
    B = w.block_size
    base = int(w.block_tables[s, 0]) * B
    return cache.reshape(-1, w.num_heads, w.head_size)[base:base + int(w.context_lens[s])]


def test_full_prompts_equal_torch_causal_attention():
    w, kc, vc = written_case([1, 7, 8, 9, 30], [1, 7, 8, 9, 30], H=4, D=32, B=8, deal="identity", seed=1)
    got = run(w, kc, vc)
    for s in range(w.num_seqs):
        r0, r1 = int(w.query_start[s]), int(w.query_start[s + 1])
        K = torch.from_numpy(_dense(w, kc, s).astype(np.float64)).permute(1, 0, 2)
        V = torch.from_numpy(_dense(w, vc, s).astype(np.float64)).permute(1, 0, 2)
        q = torch.from_numpy(w.query[r0:r1].astype(np.float64)).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, is_causal=True, scale=w.scale)
        np.testing.assert_allclose(got[r0:r1], ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_chunks_after_cached_context_equal_masked_torch_attention():
    ctx, n = [12, 30, 17, 40], [5, 1, 17, 24]
    w, kc, vc = written_case(ctx, n, H=2, D=16, B=8, deal="identity", seed=2)
    got = run(w, kc, vc)
    for s in range(w.num_seqs):
        r0, r1 = int(w.query_start[s]), int(w.query_start[s + 1])
        L = ctx[s]
        pos = np.arange(L - n[s], L)
        mask = torch.from_numpy(np.arange(L)[None, :] <= pos[:, None])      # [n, L]: token t visible to row i
        K = torch.from_numpy(_dense(w, kc, s).astype(np.float64)).permute(1, 0, 2)
        V = torch.from_numpy(_dense(w, vc, s).astype(np.float64)).permute(1, 0, 2)
        q = torch.from_numpy(w.query[r0:r1].astype(np.float64)).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=w.scale)
        np.testing.assert_allclose(got[r0:r1], ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)


def test_first_prompt_token_returns_its_own_value():
    w, kc, vc = written_case([1, 6, 19], [1, 6, 19], seed=3)
    got = run(w, kc, vc)
    for s in range(w.num_seqs):
        r0 = int(w.query_start[s])
        np.testing.assert_array_equal(got[r0], w.new_value[r0].astype(np.float64))


def test_brute_force_tiny_inputs():
    rng = np.random.default_rng(5)
    H, D, B = 2, 3, 2
    kc = rng.standard_normal((8, B, H, D)).astype(np.float16)
    vc = rng.standard_normal((8, B, H, D)).astype(np.float16)
    bt = np.array([[6, 1, 4], [0, 7, -1]], np.int32)
    ctx = np.array([5, 3], np.int32)
    qs = np.array([0, 3, 5], np.int32)       # 3 rows at positions 2..4, 2 rows at 1..2
    q = rng.standard_normal((5, H, D)).astype(np.float16)
    sc = float(np.float32(0.7))
    got = oracle.paged_prefill(q, qs, kc, vc, bt, ctx, sc)
    for s in range(2):
        n = int(qs[s + 1] - qs[s])
        for i in range(n):
            row = int(qs[s]) + i
            p_end = int(ctx[s]) - n + i + 1
            for h in range(H):
                toks = [(int(bt[s][t // B]), t % B) for t in range(p_end)]
                z = [sc * math.fsum(float(q[row, h, d]) * float(kc[b, r, h, d]) for d in range(D)) for b, r in toks]
                e = [math.exp(x) for x in z]
                for d in range(D):
                    ref = math.fsum(e[j] * float(vc[b, r, h, d]) for j, (b, r) in enumerate(toks)) / math.fsum(e)
                    assert abs(got[row, h, d] - ref) <= 1e-12


def test_invariant_under_physical_block_relabelling():
    w, kc, vc = written_case([9, 25, 33], [9, 10, 2], seed=4)
    base = run(w, kc, vc)
    perm = np.random.default_rng(9).permutation(w.num_blocks).astype(np.int32)
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    bt2 = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    got = oracle.paged_prefill(w.query, w.query_start, kc2, vc2, bt2, w.context_lens, w.scale)
    np.testing.assert_array_equal(base, got)


def test_last_row_of_each_chunk_is_the_decode_of_that_query():
    w, kc, vc = written_case([14, 33, 8], [14, 6, 1], seed=6)
    got = run(w, kc, vc)
    last = w.query_start[1:] - 1
    dec = oracle.paged_attention(np.ascontiguousarray(w.query[last]), kc, vc, w.block_tables, w.context_lens, w.scale)
    np.testing.assert_array_equal(got[last], dec)


def test_later_tokens_are_never_read():
    # rows of a chunk do not change when the cache holds NaN beyond each row's position
    w, kc, vc = written_case([20, 35], [20, 35], seed=7, poison=W.POISON_NAN)
    base = run(w, kc, vc)
    assert np.isfinite(base).all()
    s, cut = 1, 20                                  # sequence 1, rows 0 .. cut-1 only
    r0 = int(w.query_start[s])
    kc2, vc2 = kc.copy(), vc.copy()
    for t in range(cut, 35):
        b, r = int(w.block_tables[s, t // 8]), t % 8
        kc2[b, r] = np.nan
        vc2[b, r] = np.nan
    rows = np.array([[r0 + i, h] for i in range(cut) for h in range(w.num_heads)], np.int32)
    got = oracle.paged_prefill(w.query, w.query_start, kc2, vc2, w.block_tables, w.context_lens, w.scale,
                               row_head=rows)
    np.testing.assert_array_equal(got, base[r0:r0 + cut].reshape(-1, w.head_size))


def test_row_head_subset_matches_full():
    w, kc, vc = written_case([11, 3], [4, 3], H=3, seed=8)
    full = run(w, kc, vc)
    pairs = np.array([[6, 2], [0, 0], [3, 1]], np.int32)
    got = run(w, kc, vc, row_head=pairs)
    for k, (r, h) in enumerate(pairs):
        np.testing.assert_array_equal(got[k], full[r, h])


def test_empty_chunks_and_rejected_inputs():
    w, kc, vc = written_case([5, 9, 4], [0, 3, 0], seed=9)
    assert run(w, kc, vc).shape == (3, w.num_heads, w.head_size)
    bad = w.context_lens.copy()
    bad[1] = 2                                   # chunk of 3 rows in a 2-token context
    with pytest.raises(ValueError):
        oracle.paged_prefill(w.query, w.query_start, kc, vc, w.block_tables, bad, w.scale)


@pytest.mark.parametrize("cfg", [1, 3])
def test_named_prefill_workload_laws(cfg):
    w = W.prefill_named(cfg)
    assert w.query_start[0] == 0 and (np.diff(w.query_start) >= 0).all()
    assert (w.chunk_lens <= w.context_lens).all()
    assert w.query.shape == (w.total_q, w.num_heads, w.head_size)
    if cfg == 3:
        assert (w.chunk_lens == 512).all() and w.block_size == 16 and w.num_heads == 32
    pos = w.positions()
    assert pos.min(initial=0) >= 0
    assert w.flops() == 4 * w.num_heads * w.head_size * int((pos + 1).sum())
