"""A CUDA graph captured before the library's split workspace grows still
replays correctly: the library keeps an outgrown workspace instead of
freeing it (pagedkv.h, pa_paged_attention_decode)."""
import numpy as np
import pytest
import torch

import pagedattention_paged_kv_decode_b200 as pk
import workloads as W
from _oracle_step import oracle_step

pytestmark = pytest.mark.gpu


def _batch(seed, ctx):
    B, H, D = 16, 4, 128
    need = sum(-(-L // B) for L in ctx)
    return W.build(f"graph_ws{seed}", H, D, B, "f16", ctx, need + 4, -(-max(ctx) // B), seed,
                   q_std=1.0, kv_std=1.0)


def test_graph_replays_after_the_workspace_grew(cuda_device):
    small = _batch(71, [600, 40, 1100])            # a few partials
    large = _batch(72, [2000, 1900, 2047, 1500] * 40)  # over 1 MiB of partials: the workspace grows
    ds, dl = W.to_device(small, cuda_device), W.to_device(large, cuda_device)
    stream = torch.cuda.Stream(cuda_device)

    def step(w, dw):
        pk.paged_attention_decode_append(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache,
                                         dw.value_cache, dw.block_tables, dw.context_lens, w.scale,
                                         max_context_len=w.max_blocks_per_seq * w.block_size,
                                         slot_mapping=dw.slots)

    with torch.cuda.stream(stream):
        step(small, ds)                       # sizes the workspace for the small batch
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(small, ds)
        stream.synchronize()
        step(large, dl)                       # grows the workspace past the captured one
        stream.synchronize()
        ds.out.fill_(float("nan"))
        for _ in range(3):
            g.replay()
        stream.synchronize()
    assert pk.check_status() == 0
    _, _, _, out_ref, _ = oracle_step(small)
    got = ds.out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.abs(got - out_ref).max() <= 2e-3
    _, _, _, out_l, _ = oracle_step(large)
    assert np.abs(dl.out.cpu().numpy().astype(np.float64) - out_l).max() <= 2e-3
