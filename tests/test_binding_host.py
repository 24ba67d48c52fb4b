"""Host-side checks of the torch binding that need no GPU."""
import pytest
import torch

from pagedattention_paged_kv_decode_b200 import ops


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
