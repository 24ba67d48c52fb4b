"""Every check of the torch binding refuses its input before any C call.

Each case starts from a valid call (which goes through to the recorded C
call) and breaks one input: a host tensor where a device one is needed,
another dtype, a non-contiguous layout, another shape. The binding must
raise ValueError and make no C call. The library is replaced by a
recorder, so nothing is called on any machine.
"""
import pytest
import torch

from _binding_fakes import Recorder, fake, pinned
from pagedattention_paged_kv_decode_b200 import ops

S, H, D, NB, B, W, T = 3, 2, 64, 10, 16, 4, 7
F16, I32 = torch.float16, torch.int32


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(ops, "lib", lambda: r)
    monkeypatch.setattr(ops, "_on_current_device", lambda *t: None)
    return r


def f16(*shape):
    return fake(torch.zeros(shape, dtype=F16))


def i32(*shape):
    return fake(torch.zeros(shape, dtype=I32))


def host(t):
    return torch.zeros(t.shape, dtype=t.dtype)            # a plain host tensor


def other_dtype(t):
    return fake(torch.zeros(t.shape, dtype=torch.float32 if t.dtype != torch.float32 else F16))


def strided(t):
    # same shape and dtype, not contiguous
    return fake(torch.zeros(tuple(reversed(t.shape)), dtype=t.dtype).permute(*reversed(range(t.dim()))))


def decode_inputs():
    return dict(out=f16(S, H, D), query=f16(S, H, D), key_cache=f16(NB, B, H, D), value_cache=f16(NB, B, H, D),
                block_tables=i32(S, W), context_lens=fake(torch.ones(S, dtype=I32)))


def expect(rec, name, fn, kw):
    rec.calls.clear()
    fn(**kw)
    assert [c[0] for c in rec.calls] == [name]


def refuse(rec, fn, kw, **change):
    rec.calls.clear()
    with pytest.raises(ValueError):
        fn(**dict(kw, **change))
    assert rec.calls == [], change


def test_slot_mapping(rec):
    d = decode_inputs()
    kw = dict(block_tables=d["block_tables"], context_lens=d["context_lens"], key_cache=d["key_cache"],
              out=i32(S), stream=0)
    expect(rec, "pa_slot_mapping", ops.slot_mapping, kw)
    for change in (dict(block_tables=host(d["block_tables"])), dict(block_tables=strided(d["block_tables"])),
                   dict(block_tables=i32(S * W)), dict(block_tables=i32(S - 1, W)),
                   dict(context_lens=fake(torch.ones(S, dtype=torch.int64))),
                   dict(out=i32(S - 1)), dict(out=i32(S, 1)), dict(out=host(i32(S)))):
        refuse(rec, ops.slot_mapping, kw, **change)


def test_kv_cache_write(rec):
    d = decode_inputs()
    kw = dict(key=f16(S, H, D), value=f16(S, H, D), key_cache=d["key_cache"], value_cache=d["value_cache"],
              slot_mapping=i32(S), stream=0)
    expect(rec, "pa_kv_cache_write", ops.kv_cache_write, kw)
    # rows of a wider buffer: a token stride larger than the row is fine
    expect(rec, "pa_kv_cache_write", ops.kv_cache_write, dict(kw, key=f16(S, 2 * H, D)[:, :H]))
    for name in ("key", "value"):
        for bad in (host(kw[name]), other_dtype(kw[name]), f16(S, H * D), f16(S, H, D + 8), f16(S + 1, H, D),
                    strided(kw[name]), f16(S, H, 2 * D)[:, :, :D]):
            refuse(rec, ops.kv_cache_write, kw, **{name: bad})
    for bad in (f16(NB, B, H, D + 64), fake(torch.zeros(NB, B, H, D, dtype=torch.uint8)),
                strided(d["value_cache"]), host(d["value_cache"])):
        refuse(rec, ops.kv_cache_write, kw, value_cache=bad)


def test_copy_and_swap(rec):
    d = decode_inputs()
    kw = dict(key_cache=d["key_cache"], value_cache=d["value_cache"], src_dst_pairs=i32(2, 2), stream=0)
    expect(rec, "pa_copy_blocks", ops.copy_blocks, kw)
    for change in (dict(src_dst_pairs=i32(4)), dict(src_dst_pairs=i32(2, 3)), dict(src_dst_pairs=host(i32(2, 2))),
                   dict(value_cache=strided(d["value_cache"]))):
        refuse(rec, ops.copy_blocks, kw, **change)
    hk = pinned(torch.zeros(4, B, H, D, dtype=F16))
    hv = pinned(torch.zeros(4, B, H, D, dtype=F16))
    sw = dict(dst_key_cache=hk, dst_value_cache=hv, src_key_cache=d["key_cache"], src_value_cache=d["value_cache"],
              src_dst_pairs=i32(2, 2), stream=0)
    expect(rec, "pa_swap_blocks", ops.swap_blocks, sw)         # a pinned host pool is allowed
    for change in (dict(dst_value_cache=pinned(torch.zeros(5, B, H, D, dtype=F16))),    # K/V pools differ
                   dict(dst_value_cache=pinned(torch.zeros(4, B, H, D, dtype=torch.float32))),
                   dict(dst_key_cache=torch.zeros(4, B, H, D, dtype=F16),
                        dst_value_cache=torch.zeros(4, B, H, D, dtype=F16)),              # not pinned
                   dict(src_value_cache=strided(d["value_cache"])),
                   dict(dst_key_cache=pinned(torch.zeros(4, B, H, D + 64, dtype=F16)),
                        dst_value_cache=pinned(torch.zeros(4, B, H, D + 64, dtype=F16))),  # block shapes differ
                   dict(src_dst_pairs=i32(2, 3))):
        refuse(rec, ops.swap_blocks, sw, **change)
    # a non-contiguous pool on one side only
    refuse(rec, ops.swap_blocks, sw, dst_key_cache=pinned(torch.zeros(B, 4, H, D, dtype=F16).transpose(0, 1)))


def _decode_refusals(d):
    for name in ("out", "query"):
        yield {name: host(d[name])}
        yield {name: other_dtype(d[name])}
        yield {name: strided(d[name])}
    yield dict(out=f16(S + 1, H, D))
    yield dict(context_lens=fake(torch.ones(S + 1, dtype=I32)))
    yield dict(block_tables=i32(S + 1, W))
    yield dict(block_tables=i32(S * W))
    yield dict(out=f16(S, H + 1, D), query=f16(S, H + 1, D))                  # heads differ from the cache's
    yield dict(out=f16(S, H, 128), query=f16(S, H, 128))                      # head_size differs


def test_decodes(rec):
    d = decode_inputs()
    kw = dict(d, scale=0.1, stream=0)
    expect(rec, "pa_paged_attention_decode", ops.paged_attention_decode, kw)
    expect(rec, "pa_paged_attention_decode_noalloc", ops.paged_attention_decode_noalloc, kw)
    ws = dict(kw, workspace=fake(torch.zeros(4096, dtype=torch.uint8)))
    expect(rec, "pa_paged_attention_decode_ws", ops.paged_attention_decode_ws, ws)
    for change in _decode_refusals(d):
        refuse(rec, ops.paged_attention_decode, kw, **change)
        refuse(rec, ops.paged_attention_decode_noalloc, kw, **change)
    for bad in (torch.zeros(4096, dtype=torch.uint8), strided(fake(torch.zeros(64, 64, dtype=torch.uint8)))):
        refuse(rec, ops.paged_attention_decode_ws, ws, workspace=bad)


def test_append_and_shared_prefix(rec):
    d = decode_inputs()
    ws = fake(torch.zeros(4096, dtype=torch.uint8))
    kw = dict(d, new_key=f16(S, H, D), new_value=f16(S, H, D), scale=0.1, slot_mapping=i32(S), workspace=ws,
              stream=0)
    expect(rec, "pa_paged_attention_decode_append", ops.paged_attention_decode_append, kw)
    pre = dict(kw, shared_prefix_blocks=2)
    expect(rec, "pa_paged_attention_decode_shared_prefix", ops.paged_attention_decode_shared_prefix, pre)
    expect(rec, "pa_paged_attention_decode_shared_prefix", ops.paged_attention_decode_shared_prefix,
           dict(pre, new_key=None, new_value=None))                        # a plain decode of the batch
    changes = list(_decode_refusals(d))
    for name in ("new_key", "new_value"):
        changes += [{name: host(kw[name])}, {name: other_dtype(kw[name])}, {name: f16(S + 1, H, D)},
                    {name: f16(S, H, 2 * D)[:, :, :D]}]
    for h, dd in ((H + 1, D), (H, 128)):          # every row tensor agrees, the cache does not
        changes.append(dict(out=f16(S, h, dd), query=f16(S, h, dd), new_key=f16(S, h, dd), new_value=f16(S, h, dd)))
    changes += [dict(slot_mapping=i32(S - 1)), dict(slot_mapping=i32(S, 1)), dict(workspace=host(ws)),
                dict(workspace=strided(fake(torch.zeros(64, 64, dtype=torch.uint8))))]
    for change in changes:
        refuse(rec, ops.paged_attention_decode_append, kw, **change)
        refuse(rec, ops.paged_attention_decode_shared_prefix, pre, **change)
    refuse(rec, ops.paged_attention_decode_shared_prefix, pre, new_value=None)
    refuse(rec, ops.paged_attention_decode_shared_prefix, pre, new_key=None)


def test_load_cache_and_decode_step(rec):
    d = decode_inputs()
    src = f16(NB, B, H, D)
    # (its valid path allocates the slot list on the cache's device, a host device here)
    for ks, vs in ((f16(NB, B, H, D + 64), src), (src, f16(NB + 1, B, H, D))):
        refuse(rec, ops.load_cache, dict(key_cache=d["key_cache"], value_cache=d["value_cache"], key_src=ks,
                                         value_src=vs, stream=0))
    step = dict(d, new_key=f16(S, H, D), new_value=f16(S, H, D), scale=0.1, slots=i32(S), stream=0)
    for pairs, calls in ((None, ["pa_paged_attention_decode_append"]),
                         (i32(0, 2), ["pa_paged_attention_decode_append"]),
                         (i32(2, 2), ["pa_copy_blocks", "pa_paged_attention_decode_append"])):
        rec.calls.clear()
        ops.decode_step(**step, cow_pairs=pairs)
        assert [c[0] for c in rec.calls] == calls
    rec.calls.clear()
    ops.decode_step(**step, fused=False)
    assert [c[0] for c in rec.calls] == ["pa_slot_mapping", "pa_kv_cache_write", "pa_paged_attention_decode"]


def test_prefill(rec):
    d = decode_inputs()
    qs = fake(torch.tensor([0, 3, 3, T], dtype=I32))
    sk = dict(query_start=qs, block_tables=d["block_tables"], context_lens=d["context_lens"],
              key_cache=d["key_cache"], max_query_len=4, out=i32(T), total_q=T, stream=0)
    expect(rec, "pa_prefill_slot_mapping", ops.prefill_slot_mapping, sk)
    for change in (dict(query_start=i32(1, S + 1)), dict(query_start=i32(S)), dict(block_tables=i32(S + 1, W)),
                   dict(out=i32(T, 1)), dict(out=i32(T - 1)), dict(out=None, total_q=None)):
        refuse(rec, ops.prefill_slot_mapping, sk, **change)
    pf = dict(out=f16(T, H, D), query=f16(T, H, D), query_start=qs, key_cache=d["key_cache"],
              value_cache=d["value_cache"], block_tables=d["block_tables"], context_lens=d["context_lens"],
              max_query_len=4, scale=0.1, stream=0)
    expect(rec, "pa_paged_prefill", ops.paged_prefill, pf)
    changes = []
    for name in ("out", "query"):
        changes += [{name: host(pf[name])}, {name: other_dtype(pf[name])}, {name: strided(pf[name])},
                    {name: f16(T, H * D)}]
    changes += [dict(out=f16(T + 1, H, D)), dict(query_start=i32(1, S + 1)), dict(query_start=i32(S)),
                dict(block_tables=i32(S + 1, W)), dict(block_tables=i32(S * W)),
                dict(out=f16(T, H + 1, D), query=f16(T, H + 1, D)), dict(out=f16(T, H, 128), query=f16(T, H, 128))]
    for change in changes:
        refuse(rec, ops.paged_prefill, pf, **change)
