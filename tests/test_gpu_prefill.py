"""GPU parity of the paged prefill against the CPU oracle.

Bars: prefill slots and the chunk's cache write bit-exact; attention within
max-abs 2e-3 (fp16 cache, the decode's bar: fp16 operands with P rounded to
fp16, fp32 accumulation). head_size 64 and 128 with a positive scale run on the
tcgen05 kernel (128-row tiles), scales <= 0 on the mma.sync kernel (64-row
tiles).
Full sizes are checked on sampled (row, head) pairs that include every
sequence's first and last rows and the rows on both sides of each 64-row
tile edge.
"""
import numpy as np
import pytest
import torch

import oracle
import pagedattention_paged_kv_decode_b200 as pk
from pagedattention_paged_kv_decode_b200 import capi
import workloads as W

pytestmark = pytest.mark.gpu

TOL = 2e-3


def host(t):
    return t.cpu().numpy()


def run_prefill(w, dev, max_query_len=None):
    dp = W.prefill_to_device(w, dev)
    mql = int(w.chunk_lens.max(initial=0)) if max_query_len is None else max_query_len
    pk.prefill_step(dp.out, dp.query, dp.new_key, dp.new_value, dp.query_start, dp.key_cache,
                    dp.value_cache, dp.block_tables, dp.context_lens, mql, w.scale, slots=dp.slots)
    return dp


def oracle_cache(w):
    kc, vc = w.pool_host()
    slots = oracle.prefill_slot_mapping(w.query_start, w.block_tables, w.context_lens, w.block_size)
    oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots)
    return slots, kc, vc


def sample_pairs(w, n_random, seed):
    rng = np.random.default_rng(seed)
    rows = set()
    for s in range(w.num_seqs):
        r0, r1 = int(w.query_start[s]), int(w.query_start[s + 1])
        if r1 == r0:
            continue
        rows.update({r0, r1 - 1})
        for e in range(64, r1 - r0, 64):
            rows.update({r0 + e - 1, r0 + e})
    if w.total_q:
        rows.update(int(x) for x in rng.integers(0, w.total_q, n_random))
    rows = sorted(rows)
    heads = rng.integers(0, w.num_heads, len(rows))
    return np.array([[r, int(h)] for r, h in zip(rows, heads)], np.int32).reshape(-1, 2)


def check(w, dp, pairs=None, whole_cache=True):
    slots, kc, vc = oracle_cache(w)
    assert np.array_equal(host(dp.slots), slots)
    if whole_cache:
        assert np.array_equal(host(dp.key_cache).view(np.uint16), kc.view(np.uint16))
        assert np.array_equal(host(dp.value_cache).view(np.uint16), vc.view(np.uint16))
    else:
        blocks = np.unique(slots // w.block_size)
        idx = torch.from_numpy(blocks).to(dp.key_cache.device)
        assert np.array_equal(host(dp.key_cache[idx]).view(np.uint16), kc[blocks].view(np.uint16))
        assert np.array_equal(host(dp.value_cache[idx]).view(np.uint16), vc[blocks].view(np.uint16))
    got = host(dp.out).astype(np.float64)
    if pairs is None:
        ref = oracle.paged_prefill(w.query, w.query_start, kc, vc, w.block_tables, w.context_lens, w.scale)
        got_sel = got
    else:
        ref = oracle.paged_prefill(w.query, w.query_start, kc, vc, w.block_tables, w.context_lens, w.scale,
                                   row_head=pairs)
        got_sel = got[pairs[:, 0], pairs[:, 1]]
    assert np.isfinite(got_sel).all()
    err = np.abs(got_sel - ref).max(initial=0.0)
    assert err <= TOL, f"max-abs error {err}"
    return err


def test_tiny_prefill_workload(cuda_device):
    w = W.prefill_named(1)
    dp = run_prefill(w, cuda_device)
    assert pk.check_status() == 0
    check(w, dp)


@pytest.mark.parametrize("cfg", [2, 3])
def test_full_size_prefill_workloads_sampled(cuda_device, cfg):
    w = W.prefill_named(cfg)
    dp = run_prefill(w, cuda_device)
    assert pk.check_status() == 0
    check(w, dp, pairs=sample_pairs(w, 48, seed=cfg), whole_cache=False)


def ragged_prefill(D, B, seed, poison=W.POISON_HUGE, H=3):
    # full prompts, chunks after cached context, single tokens, empty chunks,
    # multi-tile chunks with ragged last tiles
    ctx = [1, 16, 17, 64, 65, 150, 300, 40, 9]
    n = [1, 16, 17, 64, 65, 130, 47, 1, 0]
    need = sum(-(-L // B) for L in ctx)
    return W.build_prefill(f"ragged_d{D}_b{B}", H, D, B, ctx, n, need + 7, -(-max(ctx) // B) + 2, seed,
                           1.0, 0.5, poison)


@pytest.mark.parametrize("D,B", [(64, 16), (64, 32), (128, 16), (128, 32)])
def test_all_prefill_variants(cuda_device, D, B):
    w = ragged_prefill(D, B, seed=10 + D + B)
    dp = run_prefill(w, cuda_device)
    assert pk.check_status() == 0
    check(w, dp)


def test_nan_in_unused_slots_is_never_used(cuda_device):
    # the tail of each sequence's last block holds NaN; masked tokens enter P.V as zeros
    w = ragged_prefill(128, 32, seed=3, poison=W.POISON_NAN)
    dp = run_prefill(w, cuda_device)
    assert pk.check_status() == 0
    check(w, dp)


def test_larger_max_query_len_bound(cuda_device):
    w = ragged_prefill(128, 16, seed=4)
    dp = run_prefill(w, cuda_device, max_query_len=1000)
    assert pk.check_status() == 0
    check(w, dp)


def test_one_token_chunks_equal_the_decode(cuda_device):
    # n_s = 1 for every sequence: the prefill of that token is the decode step
    w = W.named(2)
    dw = W.to_device(w, cuda_device)
    pk.decode_step(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache, dw.value_cache,
                   dw.block_tables, dw.context_lens, w.scale, slots=dw.slots)
    out = torch.empty_like(dw.out)
    qs = torch.arange(w.num_seqs + 1, dtype=torch.int32, device=cuda_device)
    pk.paged_prefill(out, dw.query, qs, dw.key_cache, dw.value_cache, dw.block_tables, dw.context_lens, 1,
                     w.scale)
    assert pk.check_status() == 0
    err = (out.float() - dw.out.float()).abs().max().item()
    assert err <= 2 * TOL


def test_bad_chunk_and_bad_block_are_flagged(cuda_device):
    w = ragged_prefill(128, 16, seed=5)
    dp = W.prefill_to_device(w, cuda_device)
    mql = int(w.chunk_lens.max())
    pk.prefill_step(dp.out, dp.query, dp.new_key, dp.new_value, dp.query_start, dp.key_cache, dp.value_cache,
                    dp.block_tables, dp.context_lens, mql, w.scale, slots=dp.slots)
    assert pk.check_status() == 0
    good = dp.out.clone()
    # sequence 6 claims a 2-token context for its 47-row chunk: skipped, flagged
    bad_ctx = dp.context_lens.clone()
    bad_ctx[6] = 2
    dp.out.fill_(7.0)
    pk.paged_prefill(dp.out, dp.query, dp.query_start, dp.key_cache, dp.value_cache, dp.block_tables, bad_ctx,
                     mql, w.scale)
    assert pk.check_status() & capi.PA_DEV_BAD_CHUNK
    r0, r1 = int(w.query_start[6]), int(w.query_start[7])
    assert bool((dp.out[r0:r1] == 7.0).all())
    mask = torch.ones(dp.out.shape[0], dtype=torch.bool, device=cuda_device)
    mask[r0:r1] = False
    assert torch.equal(dp.out[mask], good[mask])
    # a block id outside the pool reads as zeros and is flagged
    bt = dp.block_tables.clone()
    bt[5, 0] = w.num_blocks + 3
    pk.paged_prefill(dp.out, dp.query, dp.query_start, dp.key_cache, dp.value_cache, bt, dp.context_lens,
                     mql, w.scale)
    assert pk.check_status() & capi.PA_DEV_BAD_BLOCK
    slots = pk.prefill_slot_mapping(dp.query_start, dp.block_tables, bad_ctx, dp.key_cache, mql,
                                    total_q=w.total_q)
    assert pk.check_status() & capi.PA_DEV_BAD_CHUNK
    assert bool((slots[r0:r1] == -1).all())


def test_prefill_is_deterministic(cuda_device):
    w = W.prefill_named(3)
    dp = run_prefill(w, cuda_device)
    first = dp.out.clone()
    mql = int(w.chunk_lens.max())
    pk.paged_prefill(dp.out, dp.query, dp.query_start, dp.key_cache, dp.value_cache, dp.block_tables,
                     dp.context_lens, mql, w.scale)
    assert torch.equal(first, dp.out)


@pytest.mark.parametrize("D,B", [(64, 16), (64, 32), (128, 16), (128, 32)])
def test_non_positive_scale(cuda_device, D, B):
    # a scale <= 0 (a degenerate but valid input) is computed on the warp-MMA path
    w = ragged_prefill(D, B, seed=6 + D + B)
    for sc in (-w.scale, 0.0):
        w.scale = sc
        dp = run_prefill(w, cuda_device)
        assert pk.check_status() == 0
        check(w, dp)


def test_rows_outside_total_q_are_flagged_and_untouched(cuda_device):
    # query_start past the rows the caller holds, or negative: that sequence
    # is skipped and flagged; guard rows after the views stay as they were
    w = ragged_prefill(128, 16, seed=7)
    dp = run_prefill(w, cuda_device)
    assert pk.check_status() == 0
    good = dp.out.clone()
    T, H, D = dp.out.shape
    mql = int(w.chunk_lens.max())
    out_full = torch.full((T + 8, H, D), 7.0, dtype=torch.float16, device=cuda_device)
    q_full = torch.zeros((T + 8, H, D), dtype=torch.float16, device=cuda_device)
    q_full[:T] = dp.query
    slots_full = torch.full((T + 8,), 12345, dtype=torch.int32, device=cuda_device)

    # the last sequence (an empty chunk, context 9) claims 5 rows past total_q
    qs = dp.query_start.clone()
    qs[-1] = T + 5
    pk.paged_prefill(out_full[:T], q_full[:T], qs, dp.key_cache, dp.value_cache, dp.block_tables,
                     dp.context_lens, mql, w.scale)
    assert pk.check_status() & capi.PA_DEV_BAD_CHUNK
    assert torch.equal(out_full[:T], good)
    assert bool((out_full[T:] == 7.0).all())
    pk.prefill_slot_mapping(qs, dp.block_tables, dp.context_lens, dp.key_cache, mql, out=slots_full[:T])
    assert pk.check_status() & capi.PA_DEV_BAD_CHUNK
    assert torch.equal(slots_full[:T], dp.slots)
    assert bool((slots_full[T:] == 12345).all())

    # a negative start: sequence 0 (context raised to 4, so that its 4 rows
    # fit the context and only the row range is wrong) is skipped
    qs = dp.query_start.clone()
    qs[0] = -3
    ctx = dp.context_lens.clone()
    ctx[0] = 4
    out_full.fill_(7.0)
    pk.paged_prefill(out_full[:T], q_full[:T], qs, dp.key_cache, dp.value_cache, dp.block_tables,
                     ctx, mql, w.scale)
    assert pk.check_status() & capi.PA_DEV_BAD_CHUNK
    r1 = int(w.query_start[1])
    assert bool((out_full[:r1] == 7.0).all())
    assert torch.equal(out_full[r1:T], good[r1:])
    assert bool((out_full[T:] == 7.0).all())
