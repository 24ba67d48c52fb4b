"""Host-side checks of the torch binding that need no GPU."""
import ctypes

import pytest
import torch

from pagedattention_paged_kv_decode_b200 import capi, ops


class _OnGpu1:
    """Stands in for a CUDA tensor that lives on cuda:1."""
    is_cuda = True
    device = torch.device("cuda", 1)


def test_tensor_on_another_device_is_rejected(monkeypatch):
    # the library launches on the current device; a pointer into another
    # GPU's memory must not reach it
    monkeypatch.setattr(ops.torch.cuda, "current_device", lambda: 0)
    with pytest.raises(ValueError, match="current CUDA device"):
        ops._on_current_device(None, _OnGpu1())
    monkeypatch.setattr(ops.torch.cuda, "current_device", lambda: 1)
    ops._on_current_device(None, _OnGpu1())


def test_host_tensors_are_not_device_checked():
    # CPU tensors (the pinned pool of a swap) are left to the other checks
    ops._on_current_device(torch.zeros(2), None)


@pytest.mark.parametrize("bad", [torch.zeros(4, dtype=torch.int32), torch.zeros((2, 3), dtype=torch.int32)])
def test_cpu_tensors_are_rejected_before_shape_checks(bad):
    with pytest.raises(ValueError, match="CUDA"):
        ops._pairs(bad)
    with pytest.raises(ValueError, match="CUDA"):
        ops._table(bad, 1)


class _FakeCuda(torch.Tensor):
    """A CPU tensor that reports itself as a CUDA tensor, so that the
    binding's checks and marshalling run without a GPU (nothing launches)."""

    @property
    def is_cuda(self):
        return True


def _fake(t):
    return torch.Tensor._make_subclass(_FakeCuda, t)


def _decode_inputs(S=3, H=2, D=64, NB=10, B=16, W=4):
    f16 = torch.float16
    return (_fake(torch.zeros(S, H, D, dtype=f16)), _fake(torch.zeros(S, H, D, dtype=f16)),
            _fake(torch.zeros(NB, B, H, D, dtype=f16)), _fake(torch.zeros(NB, B, H, D, dtype=f16)),
            _fake(torch.zeros(S, W, dtype=torch.int32)), _fake(torch.ones(S, dtype=torch.int32)))


def test_decode_arguments_marshal_to_the_c_declarations(monkeypatch):
    monkeypatch.setattr(ops, "_on_current_device", lambda *t: None)
    out, q, kc, vc, bt, ctx = _decode_inputs()
    args = ops._decode_args(out, q, kc, vc, bt, ctx, 0.125, 1.0, 2.0, None)
    assert args[:4] == (out.data_ptr(), q.data_ptr(), kc.data_ptr(), vc.data_ptr())
    d = args[4]
    assert (d.num_blocks, d.block_size, d.num_heads, d.head_size, d.dtype) == (10, 16, 2, 64, capi.PA_F16)
    # table width, contexts, S, default bound = table capacity, scales
    assert args[5:] == (bt.data_ptr(), 4, ctx.data_ptr(), 3, 4 * 16, 0.125, 1.0, 2.0)
    assert ops._decode_args(out, q, kc, vc, bt, ctx, 0.125, 1.0, 2.0, 50)[9] == 50
    # the same arguments plus the stream fit both entry points' declared types
    for name in ("pa_paged_attention_decode", "pa_paged_attention_decode_noalloc"):
        argtypes = capi.SIGNATURES[name][1]
        assert len(argtypes) == len(args) + 1
        for a, ty in zip(args + (0,), argtypes):
            ty.from_param(a)


def test_decode_arguments_reject_mismatches(monkeypatch):
    monkeypatch.setattr(ops, "_on_current_device", lambda *t: None)
    out, q, kc, vc, bt, ctx = _decode_inputs()
    with pytest.raises(ValueError, match="shape mismatch"):
        ops._decode_args(out[:2], q, kc, vc, bt, ctx, 0.1, 1.0, 1.0, None)
    one_head = _fake(torch.zeros(10, 16, 1, 64, dtype=torch.float16))
    with pytest.raises(ValueError, match="heads"):
        ops._decode_args(out, q, one_head, one_head, bt, ctx, 0.1, 1.0, 1.0, None)
    with pytest.raises(ValueError, match="differ"):
        ops._decode_args(out, q, kc, vc[:5], bt, ctx, 0.1, 1.0, 1.0, None)


def test_shared_prefix_workspace_size_is_the_c_call():
    kc = torch.zeros(64, 32, 4, 128, dtype=torch.float16)   # only its shape and dtype are read
    want = capi.lib().pa_shared_prefix_workspace_size(ops.cache_desc(kc), 8, 4096, 20, None)
    assert want > 0
    assert ops.shared_prefix_workspace_size(kc, 8, 4096, 20) == want
    assert ops.shared_prefix_workspace_size(kc, 8, 4096, 20, {"partition_size": 512}) == \
        capi.lib().pa_shared_prefix_workspace_size(ops.cache_desc(kc), 8, 4096, 20,
                                                   ctypes.byref(capi.DecodeConfig(512, 0, 0, 0, 0)))
