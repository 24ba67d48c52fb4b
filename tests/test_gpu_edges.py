"""GPU edge cases: device-side bounds checks (error word, no fault), copy-on-write
semantics, strided new-token rows, empty batches."""
import numpy as np
import pytest
import torch

import oracle
import pagedattention_paged_kv_decode_b200 as pk
from pagedattention_paged_kv_decode_b200 import capi
import workloads as W

pytestmark = pytest.mark.gpu


def small(dev, kv="f16", ctx=(5, 40, 17), B=16, H=2, D=128, seed=1):
    w = W.build("edge", H, D, B, kv, list(ctx), 20, 4, seed, q_std=1.0, kv_std=1.0)
    return w, W.to_device(w, dev, encode=pk.load_cache)


def test_slot_beyond_pool_is_skipped_and_flagged(cuda_device):
    w, dw = small(cuda_device)
    before = dw.key_cache.clone()
    slots = torch.tensor([3, 20 * 16, 7], dtype=torch.int32, device=cuda_device)
    pk.kv_cache_write(dw.new_key, dw.new_value, dw.key_cache, dw.value_cache, slots)
    assert pk.check_status() == capi.PA_DEV_BAD_SLOT
    assert pk.check_status() == 0                       # read clears
    after = dw.key_cache
    assert torch.equal(after[0, 3], dw.new_key[0]) and torch.equal(after[0, 7], dw.new_key[2])
    mask = torch.ones(20, 16, dtype=torch.bool)
    mask[0, 3] = mask[0, 7] = False
    assert torch.equal(after.cpu()[mask], before.cpu()[mask])


def test_bad_block_ids_read_as_zero_rows_and_flag(cuda_device):
    w, dw = small(cuda_device)
    bt = dw.block_tables.clone()
    bt[1, 1] = 20 + 5            # seq 1 (L=40) reads logical blocks 0..2
    bt[2, 1] = -3                # seq 2 (L=17) reads logical blocks 0..1 and appends into block 1
    pk.paged_attention_decode(dw.out, dw.query, dw.key_cache, dw.value_cache, bt, dw.context_lens,
                              w.scale, max_context_len=64)
    assert pk.check_status() == capi.PA_DEV_BAD_BLOCK
    assert torch.isfinite(dw.out.float()).all()
    assert pk.check_status() == 0
    pk.slot_mapping(bt, dw.context_lens, dw.key_cache, out=dw.slots)
    assert pk.check_status() == capi.PA_DEV_BAD_BLOCK   # seq 2 appends into logical block 1 (-3)
    assert dw.slots.cpu().tolist()[2] == -1


def test_context_beyond_table_and_bound_are_clamped_and_flagged(cuda_device):
    w, dw = small(cuda_device)
    ctx = dw.context_lens.clone()
    ctx[0] = 4 * 16 + 9                                  # table holds 4 blocks
    pk.paged_attention_decode(dw.out, dw.query, dw.key_cache, dw.value_cache, dw.block_tables, ctx,
                              w.scale)
    assert pk.check_status() & capi.PA_DEV_CTX_OVER_TABLE
    pk.slot_mapping(dw.block_tables, ctx, dw.key_cache, out=dw.slots)
    assert pk.check_status() == capi.PA_DEV_CTX_OVER_TABLE
    pk.paged_attention_decode(dw.out, dw.query, dw.key_cache, dw.value_cache, dw.block_tables,
                              dw.context_lens, w.scale, max_context_len=20)
    assert pk.check_status() == capi.PA_DEV_CTX_OVER_BOUND


def test_bad_copy_pair_is_skipped_and_flagged(cuda_device):
    w, dw = small(cuda_device)
    before = dw.key_cache.clone()
    pairs = torch.tensor([[2, 19], [1, 99]], dtype=torch.int32, device=cuda_device)
    pk.copy_blocks(dw.key_cache, dw.value_cache, pairs)
    assert pk.check_status() == capi.PA_DEV_BAD_PAIR
    assert torch.equal(dw.key_cache[19], before[2])
    before[19] = before[2]
    assert torch.equal(dw.key_cache, before)


def test_copy_on_write_keeps_sharers_independent(cuda_device):
    """Two sequences share a prefix block; the first one appends into it after
    a copy ("在A10G上榨干LLaMA-7B" §2.2): the sharer's output and the shared
    block must not change, and the writer must see its new token. The
    expected pools and outputs come from the oracle's own steps on the host."""
    B, H, D = 16, 2, 64
    w = W.build("cow", H, D, B, "f16", [12, 12], 8, 2, 3, q_std=1.0, kv_std=1.0,
                deal_order="identity")
    dw = W.to_device(w, cuda_device)
    kc, vc = w.pool_host()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(cuda_device)
    # both sequences read block 0 (tokens 0..10 present); seq 1's own block 1 is unused
    bt = np.array([[0, -1], [0, -1]], np.int32)
    ctx = np.array([11, 11], np.int32)
    out0 = torch.empty_like(dw.query)
    pk.paged_attention_decode(out0, dw.query, dw.key_cache, dw.value_cache, dev(bt), dev(ctx), w.scale)
    # seq 0 appends token 11: copy block 0 -> 5, repoint its table, write into block 5
    pairs = np.array([[0, 5]], np.int32)
    bt2 = np.array([[5, -1], [0, -1]], np.int32)
    ctx2 = np.array([12, 11], np.int32)
    pk.copy_blocks(dw.key_cache, dw.value_cache, dev(pairs))
    slots = pk.slot_mapping(dev(bt2), dev(ctx2), dw.key_cache)
    pk.kv_cache_write(dw.new_key[:1], dw.new_value[:1], dw.key_cache, dw.value_cache, slots[:1])
    out1 = torch.empty_like(dw.query)
    pk.paged_attention_decode(out1, dw.query, dw.key_cache, dw.value_cache, dev(bt2), dev(ctx2), w.scale)
    assert pk.check_status() == 0
    ref_slots = oracle.slot_mapping(bt2, ctx2, B)
    assert slots.cpu().tolist() == ref_slots.tolist() == [5 * 16 + 11, 0 * 16 + 10]
    shared = kc[0].copy()
    oracle.copy_blocks(kc, vc, pairs)
    oracle.kv_cache_write(w.new_key[:1], w.new_value[:1], kc, vc, ref_slots[:1])
    assert np.array_equal(kc[0], shared)
    assert np.array_equal(dw.key_cache.cpu().numpy().view(np.uint16), kc.view(np.uint16))
    assert np.array_equal(dw.value_cache.cpu().numpy().view(np.uint16), vc.view(np.uint16))
    assert torch.equal(out1[1], out0[1])
    ref = oracle.paged_attention(w.query, kc, vc, bt2, ctx2, w.scale)
    assert np.abs(out1.cpu().numpy().astype(np.float64) - ref).max() <= 2e-3
    assert not torch.equal(out1[0], out0[0])


def test_strided_rows_from_a_fused_qkv_buffer(cuda_device):
    S, H, D, B = 5, 4, 64, 16
    h = np.random.default_rng(4).standard_normal((S, 3, H, D)).astype(np.float16)
    qkv = torch.from_numpy(h).to(cuda_device)
    kc = torch.zeros(4, B, H, D, dtype=torch.float16, device=cuda_device)
    vc = torch.zeros_like(kc)
    slots = torch.tensor([0, 17, -1, 33, 63], dtype=torch.int32, device=cuda_device)
    pk.kv_cache_write(qkv[:, 1], qkv[:, 2], kc, vc, slots)
    rk = np.zeros((4, B, H, D), np.float16)
    rv = np.zeros_like(rk)
    oracle.kv_cache_write(h[:, 1], h[:, 2], rk, rv, slots.cpu().numpy())
    assert np.array_equal(kc.cpu().numpy().view(np.uint16), rk.view(np.uint16))
    assert np.array_equal(vc.cpu().numpy().view(np.uint16), rv.view(np.uint16))


def test_empty_batch_is_a_no_op(cuda_device):
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.float16, device=cuda_device)
    e = torch.empty(0, 2, 64, dtype=torch.float16, device=cuda_device)
    pk.paged_attention_decode(e, e, kc, kc.clone(), torch.empty(0, 1, dtype=torch.int32, device=cuda_device),
                              torch.empty(0, dtype=torch.int32, device=cuda_device), 0.125)
    pk.kv_cache_write(e, e, kc, kc.clone(), torch.empty(0, dtype=torch.int32, device=cuda_device))
    assert pk.check_status() == 0


def test_fused_append_skips_bad_blocks_and_clamped_contexts(cuda_device):
    """The fused step derives the same slots as pa_slot_mapping: -1 (and no
    store) for an invalid block id or a context beyond the table."""
    w, dw = small(cuda_device)
    bt = dw.block_tables.clone()
    bt[2, 1] = -3                       # seq 2 (L=17) appends into logical block 1
    ctx = dw.context_lens.clone()
    ctx[0] = 4 * 16 + 9                 # beyond the 4-block table
    before = dw.key_cache.clone()
    pk.paged_attention_decode_append(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache,
                                     dw.value_cache, bt, ctx, w.scale, slot_mapping=dw.slots)
    code = pk.check_status()
    assert code == capi.PA_DEV_BAD_BLOCK | capi.PA_DEV_CTX_OVER_TABLE
    slots = dw.slots.cpu().tolist()
    assert slots[0] == -1 and slots[2] == -1
    ref = oracle.slot_mapping(w.block_tables, w.context_lens, 16)
    assert slots[1] == ref[1]
    changed = (dw.key_cache != before).reshape(20 * 16, -1).any(dim=1).nonzero().flatten().tolist()
    assert changed == [int(ref[1])]      # only seq 1's new row was stored
    assert torch.isfinite(dw.out.float()).all()


@pytest.mark.parametrize("kv", ["f16", "e4m3"])
def test_swap_blocks_device_and_pinned_host(cuda_device, kv):
    """Swap out to a pinned CPU pool and back in, against the oracle's copies."""
    dt = torch.float16 if kv == "f16" else torch.uint8
    rng = np.random.default_rng(9)
    shape = (12, 16, 4, 128)
    if kv == "f16":
        hk = rng.standard_normal(shape).astype(np.float16)
        hv = rng.standard_normal(shape).astype(np.float16)
    else:
        hk = rng.integers(0, 256, shape, dtype=np.uint8)
        hv = rng.integers(0, 256, shape, dtype=np.uint8)
    gk = torch.from_numpy(hk).to(cuda_device)
    gv = torch.from_numpy(hv).to(cuda_device)
    ck = torch.zeros((5,) + shape[1:], dtype=dt).pin_memory()
    cv = torch.zeros((5,) + shape[1:], dtype=dt).pin_memory()
    out_pairs = np.array([[3, 0], [11, 4], [7, 2]], np.int32)
    pk.swap_blocks(ck, cv, gk, gv, torch.from_numpy(out_pairs).to(cuda_device))
    assert pk.check_status() == 0
    rk = np.zeros((5,) + shape[1:], hk.dtype)
    rv = np.zeros_like(rk)
    oracle.swap_blocks(rk, rv, hk, hv, out_pairs)
    assert np.array_equal(ck.numpy().view(np.uint8), rk.view(np.uint8))
    assert np.array_equal(cv.numpy().view(np.uint8), rv.view(np.uint8))
    in_pairs = np.array([[0, 1], [4, 5], [2, 9]], np.int32)
    pk.swap_blocks(gk, gv, ck, cv, torch.from_numpy(in_pairs).to(cuda_device))
    bad = torch.tensor([[0, 12]], dtype=torch.int32, device=cuda_device)
    pk.swap_blocks(gk, gv, ck, cv, bad)
    assert pk.check_status() == capi.PA_DEV_BAD_PAIR
    oracle.swap_blocks(hk, hv, rk, rv, in_pairs)
    assert np.array_equal(gk.cpu().numpy().view(np.uint8), hk.view(np.uint8))
    assert np.array_equal(gv.cpu().numpy().view(np.uint8), hv.view(np.uint8))


def test_counts_above_one_grid_slice(cuda_device):
    # 70000 tokens written and 70000 block pairs copied in one call each: the
    # library launches slices of 65535; results bit-exact against the oracle
    rng = np.random.default_rng(11)
    n = 70000
    nb, B, H, D = 17500, 16, 1, 64
    key = rng.standard_normal((n, H, D)).astype(np.float16)
    val = rng.standard_normal((n, H, D)).astype(np.float16)
    slots = rng.permutation(nb * B)[:n].astype(np.int32)
    kc = np.zeros((nb, B, H, D), np.float16)
    vc = np.zeros_like(kc)
    gk, gv = torch.from_numpy(kc).to(cuda_device), torch.from_numpy(vc).to(cuda_device)
    pk.kv_cache_write(torch.from_numpy(key).to(cuda_device), torch.from_numpy(val).to(cuda_device), gk, gv,
                      torch.from_numpy(slots).to(cuda_device))
    assert pk.check_status() == 0
    oracle.kv_cache_write(key, val, kc, vc, slots)
    assert np.array_equal(gk.cpu().numpy().view(np.uint16), kc.view(np.uint16))
    assert np.array_equal(gv.cpu().numpy().view(np.uint16), vc.view(np.uint16))
    # block copy on an E4M3 pool of 2n one-KiB blocks: block i -> block n + i
    ek = rng.integers(0, 256, (2 * n, B, H, D), dtype=np.uint8)
    ev = rng.integers(0, 256, (2 * n, B, H, D), dtype=np.uint8)
    gek, gev = torch.from_numpy(ek).to(cuda_device), torch.from_numpy(ev).to(cuda_device)
    pairs = np.stack([np.arange(n), np.arange(n) + n], 1).astype(np.int32)
    pk.copy_blocks(gek, gev, torch.from_numpy(pairs).to(cuda_device))
    assert pk.check_status() == 0
    oracle.copy_blocks(ek, ev, pairs)
    assert np.array_equal(gek.cpu().numpy(), ek)
    assert np.array_equal(gev.cpu().numpy(), ev)


def test_binding_rejects_mismatched_tensors(cuda_device):
    # every rejection happens on the host, before any launch
    w, dw = small(cuda_device)
    S, H, D = dw.query.shape
    with pytest.raises(ValueError, match="key"):
        pk.kv_cache_write(dw.new_key[:, :H - 1], dw.new_value[:, :H - 1], dw.key_cache, dw.value_cache,
                          dw.slots)
    with pytest.raises(ValueError, match="slot_mapping"):
        pk.slot_mapping(dw.block_tables, dw.context_lens, dw.key_cache, out=dw.slots[:S - 1])
    with pytest.raises(ValueError, match="block_tables"):
        pk.slot_mapping(dw.block_tables[0], dw.context_lens, dw.key_cache)
    with pytest.raises(ValueError, match="src_dst_pairs"):
        pk.copy_blocks(dw.key_cache, dw.value_cache, torch.tensor([0, 1], dtype=torch.int32, device=cuda_device))
    with pytest.raises(ValueError, match="slot_mapping"):
        pk.paged_attention_decode_append(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache,
                                         dw.value_cache, dw.block_tables, dw.context_lens, w.scale,
                                         slot_mapping=dw.slots[:S - 1])
    with pytest.raises(ValueError, match="workspace"):
        pk.paged_attention_decode_append(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache,
                                         dw.value_cache, dw.block_tables, dw.context_lens, w.scale,
                                         workspace=torch.zeros(1 << 20, dtype=torch.uint8))
    with pytest.raises(ValueError, match="shape mismatch"):
        pk.paged_attention_decode_shared_prefix(dw.out[:S - 1], dw.query, dw.key_cache, dw.value_cache,
                                                dw.block_tables, dw.context_lens, 0, w.scale)
    assert pk.check_status() == 0
