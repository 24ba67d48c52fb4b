"""The oracle's threaded decode attention (the multi-core CPU baseline)
against its single-thread form.

The threaded call spreads independent (sequence, head) pairs over OpenMP
threads; each pair runs the same scalar code, so the two results must be
equal bit for bit, whatever the thread count, on fp16 and E4M3 caches, on an
explicit (s, h) subset, and with a bad table entry reported the same way.
"""
import numpy as np
import pytest

import oracle
import workloads as W


def written_case(ctx, H=4, D=32, B=16, kv="f16", seed=3):
    ctx = np.asarray(ctx)
    need = sum(-(-int(L) // B) for L in ctx)
    w = W.build("threads", H, D, B, kv, ctx, need + 7, max(1, -(-int(ctx.max()) // B)), seed,
                q_std=1.0, kv_std=1.0)
    kc, vc = w.pool_host()
    if kv == "e4m3":
        ek = np.zeros(kc.shape, np.uint8)
        ev = np.zeros(vc.shape, np.uint8)
        ident = np.arange(w.num_blocks * B, dtype=np.int32)
        oracle.kv_cache_write(kc.reshape(-1, H, D), vc.reshape(-1, H, D), ek, ev, ident, w.k_scale, w.v_scale)
        kc, vc = ek, ev
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, B)
    oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots, w.k_scale, w.v_scale)
    return w, kc, vc


@pytest.mark.parametrize("kv", ["f16", "e4m3"])
@pytest.mark.parametrize("threads", [0, 1, 2, 3, 8])
def test_threaded_equals_single_thread_bit_for_bit(kv, threads):
    w, kc, vc = written_case([1, 15, 16, 17, 40, 100, 0, 77], kv=kv)
    ref = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale,
                                 w.k_scale, w.v_scale)
    got = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale,
                                 w.k_scale, w.v_scale, threads=threads)
    assert np.array_equal(got.view(np.uint64), ref.view(np.uint64))


def test_threaded_subset_equals_single_thread():
    w, kc, vc = written_case([33, 5, 64, 2])
    pairs = np.array([[3, 1], [0, 0], [2, 3], [2, 3], [1, 2]], np.int32)
    ref = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, seq_head=pairs)
    got = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, seq_head=pairs,
                                 threads=4)
    assert np.array_equal(got.view(np.uint64), ref.view(np.uint64))


def test_threaded_reports_a_bad_table_entry():
    w, kc, vc = written_case([20, 40, 9])
    bt = w.block_tables.copy()
    bt[1, 1] = w.num_blocks  # outside the pool
    with pytest.raises(ValueError):
        oracle.paged_attention(w.query, kc, vc, bt, w.context_lens, w.scale)
    with pytest.raises(ValueError):
        oracle.paged_attention(w.query, kc, vc, bt, w.context_lens, w.scale, threads=3)


def test_max_threads_is_positive():
    assert oracle.max_threads() >= 1


@pytest.mark.parametrize("kv", ["f16", "e4m3"])
def test_threaded_cache_write_equals_single_thread(kv):
    """Duplicate slots (the later token wins), padding slots and a strided
    source row, on both cache types."""
    rng = np.random.default_rng(11)
    NB, B, H, D = 9, 16, 3, 32
    n = 40
    src = (rng.standard_normal((n, H, D + 8)) * 3).astype(np.float16)[:, :, :D]  # strided rows
    key = np.ascontiguousarray(src)
    val = (rng.standard_normal((n, H, D)) * 200).astype(np.float16)
    slots = rng.integers(-2, NB * B, n).astype(np.int32)
    slots[5] = slots[17] = slots[30]          # duplicates
    dt = np.float16 if kv == "f16" else np.uint8
    a = [np.zeros((NB, B, H, D), dt) for _ in range(2)]
    b = [np.zeros((NB, B, H, D), dt) for _ in range(2)]
    oracle.kv_cache_write(key, val, a[0], a[1], slots, 0.05, 0.7)
    oracle.kv_cache_write(key, val, b[0], b[1], slots, 0.05, 0.7, threads=4)
    for x, y in zip(a, b):
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8))


def test_threaded_cache_write_stops_at_the_same_bad_slot():
    NB, B, H, D = 4, 16, 2, 16
    key = np.ones((6, H, D), np.float16)
    slots = np.array([0, 5, NB * B, 7, 8, 9], np.int32)   # the third is beyond the pool
    a = [np.zeros((NB, B, H, D), np.float16) for _ in range(2)]
    b = [np.zeros((NB, B, H, D), np.float16) for _ in range(2)]
    with pytest.raises(ValueError):
        oracle.kv_cache_write(key, key, a[0], a[1], slots)
    with pytest.raises(ValueError):
        oracle.kv_cache_write(key, key, b[0], b[1], slots, threads=3)
    assert np.array_equal(a[0].view(np.uint16), b[0].view(np.uint16))
    assert np.array_equal(a[0].reshape(-1, H, D)[[0, 5]], key[:2])
    assert not a[0].reshape(-1, H, D)[[7, 8, 9]].any()
