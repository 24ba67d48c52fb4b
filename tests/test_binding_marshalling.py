"""Every torch-binding call reaches its C entry point with arguments of the
declared types.

The C library is replaced by a recorder: nothing is called, launched or
dereferenced, so these tests run the same with or without a GPU. The inputs
are CPU tensors that report themselves as CUDA tensors; the device check is
stubbed (it has its own test). Each binding function must make exactly the
expected C call, and every argument must convert to the ctypes type that
the library declares for that position (which a separate test ties to the
header's prototypes).
"""

import pytest
import torch

from _binding_fakes import Recorder as _Recorder, fake as _fake
from pagedattention_paged_kv_decode_b200 import capi, ops


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(ops, "lib", lambda: r)
    monkeypatch.setattr(ops, "_on_current_device", lambda *t: None)
    return r


def _check(rec, name):
    assert [c[0] for c in rec.calls] == [name], rec.calls
    args = rec.calls[0][1]
    argtypes = capi.SIGNATURES[name][1]
    assert len(args) == len(argtypes), (name, len(args), len(argtypes))
    for i, (a, ty) in enumerate(zip(args, argtypes)):
        try:
            ty.from_param(a)
        except Exception as e:  # noqa: BLE001
            raise AssertionError(f"{name} argument {i}: {a!r} does not convert to {ty}") from e
    rec.calls.clear()
    return args


S, H, D, NB, B, W = 3, 2, 64, 10, 16, 4
F16, I32 = torch.float16, torch.int32


def _decode_tensors():
    return dict(out=_fake(torch.zeros(S, H, D, dtype=F16)), query=_fake(torch.zeros(S, H, D, dtype=F16)),
                key_cache=_fake(torch.zeros(NB, B, H, D, dtype=F16)),
                value_cache=_fake(torch.zeros(NB, B, H, D, dtype=F16)),
                block_tables=_fake(torch.zeros(S, W, dtype=I32)), context_lens=_fake(torch.ones(S, dtype=I32)))


def test_cache_calls(rec):
    t = _decode_tensors()
    slots = _fake(torch.zeros(S, dtype=I32))
    ops.slot_mapping(t["block_tables"], t["context_lens"], t["key_cache"], out=slots, stream=0)
    args = _check(rec, "pa_slot_mapping")
    assert args[0] == slots.data_ptr() and args[4] == S
    new = _fake(torch.zeros(S, H, D, dtype=F16))
    ops.kv_cache_write(new, new, t["key_cache"], t["value_cache"], slots, stream=0)
    args = _check(rec, "pa_kv_cache_write")
    assert args[2] == H * D and args[8] == S
    pairs = _fake(torch.zeros(2, 2, dtype=I32))
    ops.copy_blocks(t["key_cache"], t["value_cache"], pairs, stream=0)
    assert _check(rec, "pa_copy_blocks")[4] == 2
    ops.swap_blocks(t["key_cache"], t["value_cache"], t["key_cache"], t["value_cache"], pairs, stream=0)
    args = _check(rec, "pa_swap_blocks")
    assert args[2] == NB and args[5] == NB and args[8] == 2


def test_decode_calls(rec):
    t = _decode_tensors()
    ops.paged_attention_decode(**t, scale=0.1, stream=0)
    args = _check(rec, "pa_paged_attention_decode")
    assert args[6] == W and args[8] == S and args[9] == W * B
    ops.paged_attention_decode(**t, scale=0.1, config={"partition_size": 32}, stream=0)
    _check(rec, "pa_paged_attention_decode_ws")
    ws = _fake(torch.zeros(1 << 16, dtype=torch.uint8))
    ops.paged_attention_decode_ws(**t, scale=0.1, workspace=ws, stream=0)
    args = _check(rec, "pa_paged_attention_decode_ws")
    assert args[13] is None and args[14] == ws.data_ptr() and args[15] == 1 << 16
    ops.paged_attention_decode_noalloc(**t, scale=0.1, stream=0)
    _check(rec, "pa_paged_attention_decode_noalloc")
    new = _fake(torch.zeros(S, H, D, dtype=F16))
    slots = _fake(torch.zeros(S, dtype=I32))
    ops.paged_attention_decode_append(t["out"], t["query"], new, new, t["key_cache"], t["value_cache"],
                                      t["block_tables"], t["context_lens"], 0.1, slot_mapping=slots, stream=0)
    args = _check(rec, "pa_paged_attention_decode_append")
    assert args[4] == H * D and args[17] == slots.data_ptr()
    ops.paged_attention_decode_shared_prefix(t["out"], t["query"], t["key_cache"], t["value_cache"],
                                             t["block_tables"], t["context_lens"], 2, 0.1, stream=0)
    args = _check(rec, "pa_paged_attention_decode_shared_prefix")
    assert args[2] is None and args[14] == 2


def test_prefill_calls(rec):
    T = 7
    q = _fake(torch.zeros(T, H, D, dtype=F16))
    qs = _fake(torch.tensor([0, 3, 3, 7], dtype=I32))
    t = _decode_tensors()
    slots = _fake(torch.zeros(T, dtype=I32))
    ops.prefill_slot_mapping(qs, t["block_tables"], t["context_lens"], t["key_cache"], 4, out=slots, stream=0)
    args = _check(rec, "pa_prefill_slot_mapping")
    assert args[0] == slots.data_ptr() and args[5] == S and args[6] == T and args[7] == 4
    ops.paged_prefill(_fake(torch.zeros(T, H, D, dtype=F16)), q, qs, t["key_cache"], t["value_cache"],
                      t["block_tables"], t["context_lens"], 4, 0.1, stream=0)
    args = _check(rec, "pa_paged_prefill")
    assert args[9] == S and args[10] == T and args[11] == 4


def test_size_and_status_calls(rec):
    kc = torch.zeros(NB, B, H, D, dtype=F16)
    assert ops.decode_workspace_size(kc, S, 64) == 4096
    _check(rec, "pa_decode_workspace_size")
    assert ops.shared_prefix_workspace_size(kc, S, 64, 2) == 4096
    _check(rec, "pa_shared_prefix_workspace_size")
    ops.decode_choose_config(kc, S, 64)
    _check(rec, "pa_decode_choose_config")
    assert ops.check_status(stream=0) == 0
    _check(rec, "pa_check_status")
    assert ops.version() == 202
    _check(rec, "pa_version")
    assert ops.last_error() == ""
    _check(rec, "pa_last_error")


def test_every_entry_point_has_a_binding_of_its_name():
    # the binding's name is the entry point's without the pa_ prefix
    import pagedattention_paged_kv_decode_b200 as pk
    for name in capi.SIGNATURES:
        assert callable(getattr(pk, name[3:], None)), name
