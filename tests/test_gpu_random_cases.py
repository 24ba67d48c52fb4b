"""Seeded random decode steps against the oracle: 48 cases drawn over head
size (64, 128), block size (16, 32), cache type (fp16, E4M3), head count,
batch size, context lengths (empty, one token, block edges, past one
partition), launch shapes (the library's choice or a random valid shape)
and the fused or separate path. Slots, the written rows and the whole
output are checked on each case."""
import numpy as np
import pytest
import torch

import pagedattention_paged_kv_decode_b200 as pk
import workloads as W
from _oracle_step import oracle_step

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "e4m3": 1e-2}


def _case(i):
    rng = np.random.default_rng(9000 + i)
    D = int(rng.choice([64, 128]))
    B = int(rng.choice([16, 32]))
    kv = str(rng.choice(["f16", "e4m3"]))
    H = int(rng.choice([1, 2, 3, 4, 8, 12]))
    S = int(rng.integers(1, 24))
    edges = [0, 1, B - 1, B, B + 1, 2 * B, 511, 512, 513]
    ctx = [int(rng.choice(edges)) if rng.random() < 0.4 else int(rng.integers(1, 1400)) for _ in range(S)]
    if max(ctx) == 0:
        ctx[0] = 1
    width = max(1, max(-(-L // B) for L in ctx)) + int(rng.integers(0, 3))
    need = sum(-(-L // B) for L in ctx)
    w = W.build(f"random{i}_{kv}_d{D}_b{B}", H, D, B, kv, ctx, need + int(rng.integers(1, 9)), width,
                9100 + i, q_std=float(rng.choice([0.3, 1.0, 3.0])), kv_std=float(rng.choice([0.5, 1.0])))
    launch = None
    if rng.random() < 0.6:
        G = int(rng.choice([g for g in (1, 2, 4, 8) if H % g == 0]))
        Wp = int(rng.choice([1, 2, 4]))
        C = int(rng.choice([1, 1, 1, 2, 3]))
        while C * G * Wp > 16:
            Wp = max(1, Wp // 2) if Wp > 1 else Wp
            if C * G * Wp > 16:
                C = 1
        stages = Wp * int(rng.integers(1, 8 // Wp + 1)) if Wp <= 8 else Wp
        stages = max(2, stages) if stages % Wp == 0 else Wp * 2
        if stages % Wp or stages > 8:
            stages = Wp * 2 if Wp * 2 <= 8 else 8
        P = B * int(rng.choice([1, 2, 4, 8, 32, 64]))
        launch = dict(partition_size=P, heads_per_cta=G, warps_per_head=Wp, stages=stages, units_per_cta=C)
    fused = bool(rng.random() < 0.5)
    return w, launch, fused


@pytest.mark.parametrize("i", range(48))
def test_random_case(cuda_device, i):
    w, launch, fused = _case(i)
    dt = torch.float16 if w.kv_dtype == "f16" else torch.uint8
    if launch is not None:
        try:
            pk.choose_config(torch.empty((1, w.block_size, w.num_heads, w.head_size), dtype=dt),
                             w.num_seqs, w.max_blocks_per_seq * w.block_size, dict(launch))
        except pk.PagedKVError as e:
            assert "shared memory" in str(e), str(e)
            launch = None     # the shape does not fit: the library's own choice instead
    dw = W.to_device(w, cuda_device, encode=pk.load_cache)
    bound = w.max_blocks_per_seq * w.block_size
    ws = None
    if launch is not None and not fused:  # an explicit shape on the separate path takes a caller workspace
        nbytes = pk.decode_workspace_size(dw.key_cache, w.num_seqs, bound, launch)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=cuda_device)
    pk.decode_step(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache, dw.value_cache,
                   dw.block_tables, dw.context_lens, w.scale, w.k_scale, w.v_scale, slots=dw.slots,
                   max_context_len=bound, config=launch, workspace=ws, fused=fused)
    assert pk.check_status() == 0
    slots, kc, vc, out_ref, blocks = oracle_step(w)
    assert np.array_equal(dw.slots.cpu().numpy(), slots)
    got = dw.out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.abs(got - out_ref).max() <= TOL[w.kv_dtype], (launch, fused)
