"""Stand-ins for binding tests that run without a GPU and call nothing.

_fake(t) turns a CPU tensor into one that reports itself as a CUDA tensor,
so the binding's checks and marshalling run; Recorder replaces the loaded
library and records each pa_* call instead of making it.
"""
import ctypes

import torch

from pagedattention_paged_kv_decode_b200 import capi


class FakeCuda(torch.Tensor):
    @property
    def is_cuda(self):
        return True


class FakePinned(torch.Tensor):
    """A CPU tensor that reports itself as pinned host memory."""

    def is_pinned(self, *args, **kwargs):
        return True


def fake(t):
    return torch.Tensor._make_subclass(FakeCuda, t)


def pinned(t):
    return torch.Tensor._make_subclass(FakePinned, t)


class Recorder:
    """Stands in for the loaded library: records each pa_* call."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name not in capi.SIGNATURES:
            raise AttributeError(name)
        res = capi.SIGNATURES[name][0]

        def call(*args):
            self.calls.append((name, args))
            if res is ctypes.c_size_t:
                return 4096
            if res is ctypes.c_char_p:
                return b""
            return 202 if name == "pa_version" else 0
        return call
