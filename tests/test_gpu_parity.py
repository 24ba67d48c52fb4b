"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Bars: slot mapping, cache write and block copy bit-exact; decode attention
within max-abs 2e-3 for fp16 caches and 1e-2 for E4M3 caches (the oracle runs
on the same E4M3 codes, dequantised exactly, in fp64).
"""
import numpy as np
import pytest
import torch

import oracle
import pagedattention_paged_kv_decode_b200 as pk
from pagedattention_paged_kv_decode_b200 import capi
import workloads as W
from _oracle_step import oracle_step, sample_seqs

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "e4m3": 1e-2}


def run_step(w, dev, config=None, max_context_len=None, fused=True, shared=False):
    dw = W.to_device(w, dev, encode=pk.load_cache)
    ws = None
    if config is not None and not fused:
        nbytes = pk.decode_workspace_size(dw.key_cache, w.num_seqs,
                                          max_context_len or w.max_context_len, config)
        ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    pk.decode_step(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache, dw.value_cache,
                   dw.block_tables, dw.context_lens, w.scale, w.k_scale, w.v_scale,
                   cow_pairs=dw.cow_pairs, slots=dw.slots,
                   max_context_len=max_context_len or w.max_context_len, config=config, workspace=ws,
                   fused=fused, shared_prefix_blocks=w.shared_blocks if shared else 0)
    assert pk.check_status() == 0
    return dw


def host(t):
    return t.cpu().numpy()


def same_cache(a: np.ndarray, b: np.ndarray) -> bool:
    """Bitwise equality of two caches, with every NaN code of E4M3 counted
    as the same NaN (the encoders agree on values; NaN poison may differ in
    its sign)."""
    if a.dtype == np.uint8:
        nan_a = (a & 0x7F) == 0x7F
        nan_b = (b & 0x7F) == 0x7F
        return bool(np.array_equal(nan_a, nan_b) and np.array_equal(np.where(nan_a, 0, a), np.where(nan_b, 0, b)))
    return bool(np.array_equal(a.view(np.uint16), b.view(np.uint16)))


_ORACLE_STEPS = {}


def oracle_full_step(w):
    """Oracle step of a named workload over every sequence and the whole pool
    (cached: the fused and separate GPU runs check against the same result)."""
    if w.name not in _ORACLE_STEPS:
        _ORACLE_STEPS.clear()
        _ORACLE_STEPS[w.name] = oracle_step(w, whole_pool=True)
    return _ORACLE_STEPS[w.name]


def compare_step(w, dw, seqs, check_all_blocks, ref=None):
    slots, kc, vc, out_ref, blocks = ref if ref is not None else oracle_step(w, seqs)
    assert np.array_equal(host(dw.slots), slots)
    gk, gv = dw.key_cache, dw.value_cache
    if check_all_blocks and (w.kv_dtype == "f16" or ref is not None):
        assert same_cache(host(gk), kc)
        assert same_cache(host(gv), vc)
    else:
        idx = torch.from_numpy(blocks).to(gk.device)
        a, b = host(gk[idx]), kc[blocks]
        if w.kv_dtype == "f16":
            a, b = a.view(np.uint16), b.view(np.uint16)
        assert np.array_equal(a, b)
        a, b = host(gv[idx]), vc[blocks]
        if w.kv_dtype == "f16":
            a, b = a.view(np.uint16), b.view(np.uint16)
        assert np.array_equal(a, b)
    got = host(dw.out).astype(np.float64)[seqs]
    assert np.isfinite(got).all()
    err = np.abs(got - out_ref).max()
    assert err <= TOL[w.kv_dtype], f"max-abs error {err}"
    return err


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "separate"])
@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_named_workload_step(cuda_device, cfg, fused):
    """Every sequence and head of the workload, and the whole pool after the
    step (E4M3 pools encoded in full by the oracle)."""
    w = W.named(cfg)
    dw = run_step(w, cuda_device, fused=fused)
    compare_step(w, dw, list(range(w.num_seqs)), check_all_blocks=True, ref=oracle_full_step(w))


def ragged_case(D, B, kv, seed, ctx=None, poison=W.POISON_HUGE, H=4):
    ctx = ctx if ctx is not None else [0, 1, B - 1, B, B + 1, 3 * B + 5, 64, 130, 511, 512, 513, 1100]
    need = sum(-(-int(L) // B) for L in ctx)
    width = max(1, max(-(-int(L) // B) for L in ctx))
    return W.build(f"ragged_{kv}_d{D}_b{B}", H, D, B, kv, ctx, need + 7, width, seed,
                   q_std=1.0, kv_std=1.0, poison=poison)


SHAPES = [(D, B, kv) for kv in ("f16", "e4m3") for D in (64, 128) for B in (16, 32)]


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "separate"])
@pytest.mark.parametrize("D,B,kv", SHAPES)
def test_all_kernel_variants_default_config(cuda_device, D, B, kv, fused):
    w = ragged_case(D, B, kv, seed=D + B)
    dw = run_step(w, cuda_device, fused=fused)
    compare_step(w, dw, list(range(w.num_seqs)), check_all_blocks=True)


LAUNCH = [
    dict(partition_size=16, heads_per_cta=1, warps_per_head=1, stages=2),
    dict(partition_size=32, heads_per_cta=2, warps_per_head=2, stages=6),
    dict(partition_size=64, heads_per_cta=4, warps_per_head=4, stages=4),
    dict(partition_size=128, heads_per_cta=4, warps_per_head=1, stages=4),
    dict(partition_size=512, heads_per_cta=2, warps_per_head=4, stages=8),
    dict(partition_size=2048, heads_per_cta=1, warps_per_head=2, stages=2),
    dict(partition_size=128, heads_per_cta=1, warps_per_head=1, stages=3),
    dict(partition_size=64, heads_per_cta=1, warps_per_head=2, stages=4, units_per_cta=4),
    dict(partition_size=32, heads_per_cta=2, warps_per_head=1, stages=3, units_per_cta=3),
    dict(partition_size=512, heads_per_cta=1, warps_per_head=1, stages=2, units_per_cta=2),
    dict(partition_size=128, heads_per_cta=4, warps_per_head=2, stages=2, units_per_cta=2),
    # nine-warp CTAs whose ring leaves room for three per SM: the register-capped
    # instantiation of the decode kernel is the one launched
    dict(partition_size=512, heads_per_cta=4, warps_per_head=2, stages=2),
    dict(partition_size=256, heads_per_cta=4, warps_per_head=2, stages=4),
]


@pytest.mark.parametrize("launch", LAUNCH, ids=lambda d: "p{partition_size}_g{heads_per_cta}_w{warps_per_head}_s{stages}_c{}".format(d.get("units_per_cta", 1), **d))
@pytest.mark.parametrize("D,B,kv", [(128, 16, "f16"), (128, 32, "f16"), (128, 16, "e4m3"), (64, 32, "e4m3")])
def test_launch_shapes(cuda_device, launch, D, B, kv):
    if launch["partition_size"] % B:
        pytest.skip("partition size must be a multiple of the block size")
    w = ragged_case(D, B, kv, seed=7)
    try:
        pk.choose_config(torch.empty((1, B, 4, D), dtype=torch.float16 if kv == "f16" else torch.uint8),
                         w.num_seqs, w.max_context_len, dict(launch))
    except pk.PagedKVError as e:
        assert "shared memory" in str(e)
        pytest.skip("launch shape does not fit in shared memory (rejected by the library)")
    dw = run_step(w, cuda_device, config=dict(launch))
    compare_step(w, dw, list(range(w.num_seqs)), check_all_blocks=True)


@pytest.mark.parametrize("kv", ["f16", "e4m3"])
def test_nan_poison_is_never_touched(cuda_device, kv):
    w = ragged_case(128, 16, kv, seed=3, poison=W.POISON_NAN)
    for launch in (None, dict(partition_size=32, heads_per_cta=2, warps_per_head=2, stages=4),
                   dict(partition_size=64, heads_per_cta=1, warps_per_head=2, stages=2, units_per_cta=3)):
        for fused in (True, False):
            dw = run_step(w, cuda_device, config=launch, fused=fused)
            compare_step(w, dw, list(range(w.num_seqs)), check_all_blocks=False)


def test_split_partials_match_oracle_partitions(cuda_device):
    """Row by row check of the partition kernel's workspace (lse, o).

    Tolerances follow from the kernel's arithmetic: each softmax weight p_t
    is rounded to fp16 once (p'_t = p_t (1 + e_t), |e_t| <= 2^-12) and the
    same p'_t enters the numerator and the denominator. A normalised partial
    o = sum p'_t v_t / sum p'_t then differs from the exact one by at most
    2^-12 / (1 - 2^-12) * max_t |v_t[d] - o[d]| per element (the exact
    weights sum p_t (v_t - o) to zero), and its log-sum-exp by at most
    ln(1 + 2^-12) in natural-log units; 2e-5 covers the fp32 sums and the
    hardware exp2/log2."""
    w = ragged_case(128, 16, "f16", seed=5, ctx=[600, 1100, 40, 1024])
    cfg = dict(partition_size=256, heads_per_cta=2, warps_per_head=2, stages=4)
    dw = W.to_device(w, cuda_device)
    pk.decode_step(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache, dw.value_cache,
                   dw.block_tables, dw.context_lens, w.scale, slots=dw.slots,
                   max_context_len=w.max_context_len, config=cfg,
                   workspace=torch.zeros(pk.decode_workspace_size(dw.key_cache, w.num_seqs, w.max_context_len, cfg),
                                         dtype=torch.uint8, device=cuda_device))
    # rerun the decode alone into a workspace we keep
    nbytes = pk.decode_workspace_size(dw.key_cache, w.num_seqs, w.max_context_len, cfg)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=cuda_device)
    pk.paged_attention_decode(dw.out, dw.query, dw.key_cache, dw.value_cache, dw.block_tables,
                              dw.context_lens, w.scale, max_context_len=w.max_context_len,
                              config=cfg, workspace=ws)
    torch.cuda.synchronize()
    S, H, D = w.query.shape
    P = -(-w.max_context_len // 256)
    lse_bytes = -(-(S * H * P * 4) // 256) * 256
    raw = host(ws)
    lse2 = raw[:S * H * P * 4].view(np.float32).reshape(S, H, P)
    o = raw[lse_bytes:lse_bytes + S * H * P * D * 4].view(np.float32).reshape(S, H, P, D)
    _, kc, vc, _, _ = oracle_step(w)
    ro, rlse = oracle.attention_partials(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, 256)
    eps = 2.0 ** -12
    B = w.block_size
    for s, L in enumerate(w.context_lens):
        n = -(-int(L) // 256)
        if n <= 1:
            continue                              # single partitions write the output directly
        np.testing.assert_allclose(lse2[s, :, :n] * np.log(2.0), rlse[s, :, :n], rtol=0,
                                   atol=np.log1p(eps) + 2e-5)
        for p in range(n):
            t = np.arange(p * 256, min(int(L), (p + 1) * 256))
            rows = vc[w.block_tables[s, t // B], t % B].astype(np.float64)    # [tokens, H, D]
            spread = np.abs(rows - ro[s, :, p][None]).max(axis=0)           # [H, D]
            bound = eps / (1 - eps) * spread + 2e-5
            assert (np.abs(o[s, :, p] - ro[s, :, p]) <= bound).all(), \
                float((np.abs(o[s, :, p] - ro[s, :, p]) - bound).max())


def test_e4m3_encode_every_f16_value(cuda_device):
    """All 65536 fp16 bit patterns through the quantising cache write, several scales."""
    H, D, B = 4, 128, 16
    x = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16).reshape(128, H, D)
    for scale in (1.0, 0.0137, 3.5, 1e-3):
        kc = torch.zeros((8, B, H, D), dtype=torch.uint8, device=cuda_device)
        vc = torch.zeros_like(kc)
        slots = torch.arange(128, dtype=torch.int32, device=cuda_device)
        src = torch.from_numpy(x).to(cuda_device)
        pk.kv_cache_write(src, src, kc, vc, slots, k_scale=scale, v_scale=2 * scale)
        rk = np.zeros((8, B, H, D), np.uint8)
        rv = np.zeros_like(rk)
        oracle.kv_cache_write(x, x, rk, rv, np.arange(128, dtype=np.int32), scale, 2 * scale)
        for got, ref in ((host(kc), rk), (host(vc), rv)):
            nan_g = (got & 0x7F) == 0x7F
            nan_r = (ref & 0x7F) == 0x7F
            assert np.array_equal(nan_g, nan_r)
            assert np.array_equal(got[~nan_g], ref[~nan_r])


def test_determinism(cuda_device):
    w = W.named(2)
    a = host(run_step(w, cuda_device).out)
    b = host(run_step(w, cuda_device).out)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


# ------------------------------------------------------------ shared prefix

def test_shared_prefix_named_workload_4(cuda_device):
    w = W.named(4)
    assert w.shared_blocks == 95
    dw = run_step(w, cuda_device, shared=True)
    compare_step(w, dw, sample_seqs(w, 8, seed=4), check_all_blocks=False)


def prefix_case(D, B, kv, prefix_blocks, suffixes, seed, cow=False, H=4):
    prefix = prefix_blocks * B
    ctx = [prefix + x for x in suffixes]
    need = prefix_blocks + sum(-(-max(0, L - prefix) // B) for L in ctx) + (len(ctx) if cow else 0)
    width = max(-(-L // B) for L in ctx)
    return W.build(f"prefix_{kv}_d{D}_b{B}", H, D, B, kv, ctx, need + 5, width, seed,
                   q_std=1.0, kv_std=1.0, shared_prefix=prefix, cow=cow)


@pytest.mark.parametrize("cow", [False, True], ids=["shared", "cow"])
@pytest.mark.parametrize("D,B,kv", [(128, 16, "f16"), (128, 32, "f16"), (64, 16, "e4m3"), (128, 32, "e4m3")])
def test_shared_prefix_matches_oracle(cuda_device, D, B, kv, cow):
    suffixes = [1, B, B + 3, 700, 1300, 40, 2 * B - 1]
    w = prefix_case(D, B, kv, 40 if B == 16 else 20, suffixes, seed=D + B + cow, cow=cow)
    assert w.shared_blocks == (39 if B == 16 else 19) if cow else (40 if B == 16 else 20)
    dw = run_step(w, cuda_device, shared=True)
    compare_step(w, dw, list(range(w.num_seqs)), check_all_blocks=True)


def test_shared_prefix_plain_decode_with_short_contexts(cuda_device):
    """Without an append, contexts may end inside the shared prefix; the
    prefix kernel masks each sequence to its own length."""
    B, prefix_blocks = 16, 12
    w = prefix_case(128, B, "f16", prefix_blocks, [5, 300, 17, 1], seed=31)
    ctx = w.context_lens.copy()
    ctx[1] = 100       # ends inside the prefix
    ctx[3] = 1
    dw = W.to_device(w, cuda_device)
    pk.paged_attention_decode_shared_prefix(dw.out, dw.query, dw.key_cache, dw.value_cache,
                                            dw.block_tables, torch.from_numpy(ctx).to(cuda_device),
                                            prefix_blocks, w.scale)
    assert pk.check_status() == 0
    kc, vc = w.pool_host()
    ref = oracle.paged_attention(w.query, kc, vc, w.block_tables, ctx, w.scale)
    got = host(dw.out).astype(np.float64)
    assert np.abs(got - ref).max() <= 2e-3


def test_shared_prefix_contract_is_checked(cuda_device):
    B, prefix_blocks = 16, 8
    w = prefix_case(128, B, "f16", prefix_blocks, [5, 20, 33], seed=32)
    dw = W.to_device(w, cuda_device)
    bt = dw.block_tables.clone()
    bt[2, 3] = bt[1, prefix_blocks]      # row 2 no longer shares logical block 3
    pk.paged_attention_decode_shared_prefix(dw.out, dw.query, dw.key_cache, dw.value_cache, bt,
                                            dw.context_lens, prefix_blocks, w.scale)
    assert pk.check_status() == capi.PA_DEV_PREFIX
    ctx = dw.context_lens.clone()
    ctx[0] = prefix_blocks * B           # the appended token would land in a shared block
    pk.paged_attention_decode_shared_prefix(dw.out, dw.query, dw.key_cache, dw.value_cache,
                                            dw.block_tables, ctx, prefix_blocks, w.scale,
                                            new_key=dw.new_key, new_value=dw.new_value,
                                            slot_mapping=dw.slots)
    assert pk.check_status() == capi.PA_DEV_PREFIX
    assert dw.slots.cpu().tolist()[0] == -1


@pytest.mark.parametrize("q_std", [30.0, 300.0])
@pytest.mark.parametrize("kv", ["f16", "e4m3"])
def test_large_queries(cuda_device, kv, q_std):
    """Queries far above a trained model's scale (|q * scale| per element up
    to ~100): the logits' products are exact and summed in fp32, so neither
    cache type overflows and the result stays within the parity bar."""
    ctx = [1, 17, 300, 1100, 64]
    B, H, D = 16, 4, 128
    need = sum(-(-L // B) for L in ctx)
    w = W.build(f"large_q_{kv}", H, D, B, kv, ctx, need + 6, -(-max(ctx) // B), 41,
                q_std=q_std, kv_std=1.0)
    dw = run_step(w, cuda_device)
    compare_step(w, dw, list(range(w.num_seqs)), check_all_blocks=True)
