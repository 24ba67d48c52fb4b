"""Pins for the oracle's slot mapping, cache write and block copy.

Slot mapping is pinned to the worked example printed on the l189.com/news/180929
article (section 2.2) and to the growth example of the "在A10G上榨干LLaMA-7B" page
(section 2.1); both are stored under tests/golden/. Cache write and block copy are
pinned by reading back through plain numpy indexing of the [block, row, head, dim]
layout, and by checking that nothing outside the target rows changes. The block
copy moves exactly the per-block bytes that the article's section 2.1 prints,
restated for 2- and 1-byte elements (tests/golden/block_bytes_example.txt).
"""
import os

import numpy as np
import pytest

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_slot_mapping_worked_example():
    rows = _rows("slot_mapping_worked_example.txt")
    tables = {"A": [5, 8], "B": [3, -1]}
    for seq, tok, blk, off, slot in rows:
        tok, blk, off, slot = int(tok), int(blk), int(off), int(slot)
        bt = np.array([tables[seq]], np.int32)
        got = oracle.slot_mapping(bt, np.array([tok + 1], np.int32), 16)
        assert got[0] == slot, (seq, tok)
        assert got[0] // 16 == blk and got[0] % 16 == off


def test_slot_mapping_growth_example():
    bt = np.array([[7, 2, 3, -1]], np.int32)
    for tok, ctx, logical, phys, off, slot in _rows("block_growth_example.txt"):
        got = oracle.slot_mapping(bt, np.array([int(ctx)], np.int32), 4)[0]
        assert got == int(slot), tok
        assert bt[0, int(logical)] == int(phys) and got % 4 == int(off)


def test_slot_mapping_empty_sequence_and_table_overrun():
    bt = np.array([[4, 9], [1, 2]], np.int32)
    assert list(oracle.slot_mapping(bt, np.array([0, 3], np.int32), 16)) == [-1, 18]
    with pytest.raises(ValueError):
        oracle.slot_mapping(bt, np.array([33, 1], np.int32), 16)


def _small_pool(nb=6, bs=4, nh=3, hd=8, seed=0, poison=np.float16(7.0)):
    rng = np.random.default_rng(seed)
    kc = np.full((nb, bs, nh, hd), poison, np.float16)
    vc = np.full((nb, bs, nh, hd), -poison, np.float16)
    key = rng.standard_normal((5, nh, hd)).astype(np.float16)
    val = rng.standard_normal((5, nh, hd)).astype(np.float16)
    return kc, vc, key, val


def test_cache_write_f16_places_rows_and_touches_nothing_else():
    kc, vc, key, val = _small_pool()
    slots = np.array([0, 23, -1, 9, 14], np.int32)
    k0, v0 = kc.copy(), vc.copy()
    oracle.kv_cache_write(key, val, kc, vc, slots)
    touched = np.zeros(kc.shape[:2], bool)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        b, r = divmod(int(s), 4)
        touched[b, r] = True
        assert np.array_equal(kc[b, r].view(np.uint16), key[i].view(np.uint16))
        assert np.array_equal(vc[b, r].view(np.uint16), val[i].view(np.uint16))
    assert np.array_equal(kc[~touched], k0[~touched]) and np.array_equal(vc[~touched], v0[~touched])


def test_cache_write_strided_rows():
    kc, vc, key, val = _small_pool()
    qkv = np.random.default_rng(3).standard_normal((5, 3, 3, 8)).astype(np.float16)  # [n, 3, H, D]
    slots = np.array([1, 2, 3, 4, 5], np.int32)
    oracle.kv_cache_write(qkv[:, 1], qkv[:, 2], kc, vc, slots)
    for i in range(5):
        assert np.array_equal(kc[0 if i < 3 else 1, (i + 1) % 4], qkv[i, 1])
        assert np.array_equal(vc[0 if i < 3 else 1, (i + 1) % 4], qkv[i, 2])


def test_cache_write_rejects_slot_beyond_pool():
    kc, vc, key, val = _small_pool()
    with pytest.raises(ValueError):
        oracle.kv_cache_write(key, val, kc, vc, np.array([0, 24, 1, 2, 3], np.int32))


def test_cache_write_e4m3_encodes_each_element():
    nb, bs, nh, hd = 4, 4, 2, 8
    kc = np.full((nb, bs, nh, hd), 0x55, np.uint8)
    vc = np.full((nb, bs, nh, hd), 0x66, np.uint8)
    rng = np.random.default_rng(1)
    key = (rng.standard_normal((3, nh, hd)) * 3).astype(np.float16)
    val = (rng.standard_normal((3, nh, hd)) * 3).astype(np.float16)
    ks, vs = np.float32(0.0123), np.float32(2.5)
    oracle.kv_cache_write(key, val, kc, vc, np.array([5, -1, 15], np.int32), ks, vs)
    for i, s in ((0, 5), (2, 15)):
        b, r = divmod(s, bs)
        assert np.array_equal(kc[b, r], oracle.e4m3_from_float(key[i].astype(np.float32) / ks))
        assert np.array_equal(vc[b, r], oracle.e4m3_from_float(val[i].astype(np.float32) / vs))
    assert (kc[0, 0] == 0x55).all() and (kc[0, 2] == 0x55).all()


def test_copy_blocks_in_order_and_bounds():
    kc, vc, _, _ = _small_pool()
    rng = np.random.default_rng(5)
    kc[:] = rng.standard_normal(kc.shape).astype(np.float16)
    vc[:] = rng.standard_normal(vc.shape).astype(np.float16)
    k0, v0 = kc.copy(), vc.copy()
    oracle.copy_blocks(kc, vc, np.array([[1, 4], [4, 2]], np.int32))   # 4 <- 1, then 2 <- 4 (= old 1)
    assert np.array_equal(kc[4], k0[1]) and np.array_equal(kc[2], k0[1])
    assert np.array_equal(vc[4], v0[1]) and np.array_equal(vc[2], v0[1])
    for b in (0, 1, 3, 5):
        assert np.array_equal(kc[b], k0[b]) and np.array_equal(vc[b], v0[b])
    with pytest.raises(ValueError):
        oracle.copy_blocks(kc, vc, np.array([[0, 6]], np.int32))


def test_generator_layout_equals_writes_through_slot_mapping():
    """The generator's placement of context tokens agrees with the oracle's own
    slot mapping + cache write, token by token (so neither can hide a layout slip)."""
    w = W.build("t", 3, 16, 8, "f16", [1, 9, 20, 8], 16, 4, seed=11, q_std=1, kv_std=1)
    pk, pv = w.pool_host()
    kc = np.zeros_like(pk)
    vc = np.zeros_like(pv)
    i = 0
    order = []
    for s, L in enumerate(w.context_lens):
        for t in range(int(L) - 1):
            order.append((s, t))
    assert len(order) == len(w.live_blocks)
    for j, (s, t) in enumerate(order):
        slot = oracle.slot_mapping(w.block_tables[s:s + 1], np.array([t + 1], np.int32), 8)
        oracle.kv_cache_write(w.live_key[j:j + 1], w.live_value[j:j + 1], kc, vc, slot)
        b, r = divmod(int(slot[0]), 8)
        assert np.array_equal(pk[b, r], w.live_key[j]) and np.array_equal(pv[b, r], w.live_value[j])
        i += 1
    assert i == len(order)


@pytest.mark.parametrize("cfg", [1, 2])
def test_named_workload_laws(cfg):
    w = W.named(cfg)
    S, B = w.num_seqs, w.block_size
    if cfg == 1:
        assert (S, w.num_heads, w.head_size, B, w.num_blocks) == (4, 4, 64, 16, 32)
        assert w.context_lens.min() >= 1 and w.context_lens.max() <= 64
    else:
        assert (S, w.num_heads, w.head_size, B, w.num_blocks) == (16, 32, 128, 16, 2048)
        assert w.context_lens.min() >= 50 and w.context_lens.max() <= 178
    used = w.block_tables[w.block_tables >= 0]
    assert len(np.unique(used)) == len(used) and used.max() < w.num_blocks
    for s in range(S):
        n = -(-int(w.context_lens[s]) // B)
        assert (w.block_tables[s, :n] >= 0).all() and (w.block_tables[s, n:] == -1).all()
    pk, _ = w.pool_host()
    live = np.zeros(pk.shape[:2], bool)
    live[w.live_blocks, w.live_offsets] = True
    assert (np.abs(pk[~live].astype(np.float32)) == 60000).all()


def test_swap_blocks_between_pools():
    rng = np.random.default_rng(8)
    gk = rng.standard_normal((6, 4, 2, 8)).astype(np.float16)
    gv = rng.standard_normal((6, 4, 2, 8)).astype(np.float16)
    ck = np.zeros((3, 4, 2, 8), np.float16)
    cv = np.zeros((3, 4, 2, 8), np.float16)
    oracle.swap_blocks(ck, cv, gk, gv, np.array([[5, 0], [2, 2]], np.int32))   # out: device -> host pool
    assert np.array_equal(ck[0], gk[5]) and np.array_equal(cv[2], gv[2]) and not ck[1].any()
    g0 = gk.copy()
    oracle.swap_blocks(gk, gv, ck, cv, np.array([[0, 1]], np.int32))           # in: host -> device pool
    assert np.array_equal(gk[1], g0[5])
    for b in (0, 2, 3, 4, 5):
        assert np.array_equal(gk[b], g0[b])
    with pytest.raises(ValueError):
        oracle.swap_blocks(ck, cv, gk, gv, np.array([[6, 0]], np.int32))
    with pytest.raises(ValueError):
        oracle.swap_blocks(ck, cv, gk, gv, np.array([[0, 3]], np.int32))


def test_block_bytes_follow_the_printed_block_size():
    # [P3] §2.1 sizes a 16-token x 32-head x 128-dim K+V block at about 512 KB
    # with 4-byte elements; the oracle's block copy moves exactly one block
    # of B*H*D*elem bytes per cache, i.e. the fixture's K+V figure for fp16
    # and E4M3
    rows = {}
    with open(os.path.join(GOLDEN, "block_bytes_example.txt")) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                B, H, D, caches, elem, nbytes = map(int, ln.split())
                assert B * H * D * caches * elem == nbytes
                rows[elem] = (B, H, D, nbytes)
    assert rows[4][3] == 512 * 1024
    rng = np.random.default_rng(17)
    for elem, dtype in ((2, np.float16), (1, np.uint8)):
        B, H, D, nbytes = rows[elem]
        src = rng.integers(1, 256, (3, B, H, D * elem), dtype=np.uint8).view(dtype)
        kc, vc = src.copy(), src.copy()
        kc[2] = 0
        vc[2] = 0
        k0, v0 = kc.copy(), vc.copy()
        oracle.copy_blocks(kc, vc, np.array([[0, 2]], np.int32))
        changed = int((kc.view(np.uint8) != k0.view(np.uint8)).sum() + (vc.view(np.uint8) != v0.view(np.uint8)).sum())
        assert changed == nbytes
