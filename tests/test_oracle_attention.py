"""Pins for the oracle's decode attention and its split-context pieces.

The pages give no attention formula; the oracle uses the plain definition of
single-query softmax attention over the tokens a block table addresses. It is
pinned here by: torch's CPU scaled_dot_product_attention on identity block
tables (paged = dense), invariance under any relabelling of physical blocks,
the closed forms L=1 -> V and equal keys / scale 0 -> mean of V, exact-sum
brute force on tiny inputs, convexity bounds, immunity to poisoned unused
slots, E4M3 caches against fp16 caches holding the same values, and the
log-sum-exp identity that joins split partitions.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W


def complete_case(ctx, H=3, D=16, B=8, nb=None, seed=0, deal="permuted", poison=W.POISON_HUGE, kv="f16"):
    """A workload whose appended token has been written (by the oracle's own steps)."""
    ctx = np.asarray(ctx)
    need = sum(-(-int(L) // B) for L in ctx)
    nb = nb or need + 5
    w = W.build("case", H, D, B, "f16", ctx, nb, max(1, -(-int(ctx.max()) // B)), seed,
                q_std=1.0, kv_std=1.0, poison=poison, deal_order=deal)
    kc, vc = w.pool_host()
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, B)
    oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots)
    return w, kc, vc


def dense_kv(w, kc, s, which_cache):
    """Rows of sequence s under identity dealing: a contiguous slice of the flattened pool."""
    B = w.block_size
    base = int(w.block_tables[s, 0]) * B
    flat = which_cache.reshape(-1, w.num_heads, w.head_size)
    return flat[base:base + int(w.context_lens[s])]


def test_identity_tables_equal_torch_dense_attention():
    w, kc, vc = complete_case([1, 7, 8, 9, 30, 64], H=4, D=32, B=8, deal="identity", seed=1)
    got = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
    for s in range(w.num_seqs):
        K = torch.from_numpy(dense_kv(w, kc, s, kc).astype(np.float64)).permute(1, 0, 2)  # [H, L, D]
        V = torch.from_numpy(dense_kv(w, kc, s, vc).astype(np.float64)).permute(1, 0, 2)
        q = torch.from_numpy(w.query[s].astype(np.float64))[:, None, :]                # [H, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, scale=w.scale)[:, 0, :]
        np.testing.assert_allclose(got[s], ref.numpy(), rtol=0, atol=1e-12)


def test_invariant_under_physical_block_relabelling():
    w, kc, vc = complete_case([5, 17, 33, 40], seed=2)
    base = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
    perm = np.random.default_rng(9).permutation(w.num_blocks).astype(np.int32)
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    bt2 = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    moved = oracle.paged_attention(w.query, kc2, vc2, bt2, w.context_lens, w.scale)
    assert np.array_equal(base, moved)


def test_context_one_returns_v_exactly():
    w, kc, vc = complete_case([1, 1, 1], seed=3)
    got = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
    assert np.array_equal(got, w.new_value.astype(np.float64))


@pytest.mark.parametrize("mode", ["equal_keys", "zero_scale"])
def test_uniform_logits_give_mean_of_v(mode):
    w, kc, vc = complete_case([3, 16, 29], seed=4, deal="identity")
    scale = w.scale
    if mode == "equal_keys":
        kc[:] = kc[w.block_tables[0, 0], 0]       # every row (all heads) equal to one key row
    else:
        scale = 0.0
    got = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, scale)
    for s in range(3):
        mean = dense_kv(w, kc, s, vc).astype(np.float64).mean(axis=0)
        np.testing.assert_allclose(got[s], mean, rtol=0, atol=1e-12)


def test_brute_force_tiny_inputs():
    rng = np.random.default_rng(5)
    for trial in range(20):
        H, D, B = int(rng.integers(1, 3)), int(rng.integers(1, 5)), int(rng.integers(1, 4))
        ctx = rng.integers(1, 6, int(rng.integers(1, 3)))
        nb = int(sum(-(-int(L) // B) for L in ctx)) + 2
        kc = rng.standard_normal((nb, B, H, D)).astype(np.float16)
        vc = rng.standard_normal((nb, B, H, D)).astype(np.float16)
        q = rng.standard_normal((len(ctx), H, D)).astype(np.float16)
        perm = rng.permutation(nb)
        width = max(-(-int(L) // B) for L in ctx)
        bt = np.full((len(ctx), width), -1, np.int32)
        c = 0
        for s, L in enumerate(ctx):
            n = -(-int(L) // B)
            bt[s, :n] = perm[c:c + n]
            c += n
        scale = float(np.float32(rng.uniform(0.1, 2.0)))
        got = oracle.paged_attention(q, kc, vc, bt, ctx, scale)
        for s, L in enumerate(ctx):
            for h in range(H):
                rows = [(int(bt[s][t // B]), t % B) for t in range(int(L))]
                z = [scale * math.fsum(float(q[s, h, d]) * float(kc[b, r, h, d]) for d in range(D))
                     for b, r in rows]
                p = [math.exp(x) for x in z]                       # no max subtraction
                for d in range(D):
                    ref = math.fsum(p[i] * float(vc[b, r, h, d]) for i, (b, r) in enumerate(rows)) / math.fsum(p)
                    assert abs(got[s, h, d] - ref) <= 1e-12 * max(1.0, abs(ref)), (trial, s, h, d)


def test_output_is_a_convex_combination_of_v():
    w, kc, vc = complete_case([2, 13, 50, 64], H=2, D=8, deal="identity", seed=6)
    got = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
    for s in range(w.num_seqs):
        V = dense_kv(w, kc, s, vc).astype(np.float64)
        assert (got[s] >= V.min(axis=0) - 1e-15).all() and (got[s] <= V.max(axis=0) + 1e-15).all()


def test_unused_slots_are_never_read():
    a = complete_case([3, 17, 31], seed=7, poison=W.POISON_HUGE)
    b = complete_case([3, 17, 31], seed=7, poison=W.POISON_NAN)
    oa = oracle.paged_attention(a[0].query, a[1], a[2], a[0].block_tables, a[0].context_lens, a[0].scale)
    ob = oracle.paged_attention(b[0].query, b[1], b[2], b[0].block_tables, b[0].context_lens, b[0].scale)
    assert np.array_equal(oa, ob) and np.isfinite(oa).all()


def test_zero_length_context_gives_zeros():
    w, kc, vc = complete_case([4, 9], seed=8)
    ctx = w.context_lens.copy()
    ctx[1] = 0
    got = oracle.paged_attention(w.query, kc, vc, w.block_tables, ctx, w.scale)
    assert (got[1] == 0).all()


def test_seq_head_subset_matches_full():
    w, kc, vc = complete_case([4, 9, 22], seed=12)
    full = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
    pairs = np.array([[2, 1], [0, 2], [1, 0]], np.int32)
    sub = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, seq_head=pairs)
    for i, (s, h) in enumerate(pairs):
        assert np.array_equal(sub[i], full[s, h])


@pytest.mark.parametrize("k_pow,v_pow", [(0, 0), (-3, 2), (2, -1)])
def test_e4m3_cache_equals_f16_cache_of_the_same_values(k_pow, v_pow):
    """Every E4M3 value times a power of two is exactly an fp16 value, so an E4M3
    cache and an fp16 cache holding its decoded values must give equal outputs.
    Distinct K and V scales pin which scale goes with which cache."""
    rng = np.random.default_rng(13)
    nb, B, H, D = 6, 4, 2, 8
    codes_k = rng.integers(0, 256, (nb, B, H, D), dtype=np.uint8)
    codes_v = rng.integers(0, 256, (nb, B, H, D), dtype=np.uint8)
    for c in (codes_k, codes_v):
        c[(c & 0x7F) == 0x7F] = 0x3C           # no NaN codes
        c[(c & 0x78) >= 0x60] &= 0x9F          # keep magnitudes small (exponent field < 12)
    sk, sv = float(2.0 ** k_pow), float(2.0 ** v_pow)
    f16_k = (oracle.e4m3_to_double(codes_k) * sk).astype(np.float16)
    f16_v = (oracle.e4m3_to_double(codes_v) * sv).astype(np.float16)
    assert np.array_equal(f16_k.astype(np.float64), oracle.e4m3_to_double(codes_k) * sk)
    assert np.array_equal(f16_v.astype(np.float64), oracle.e4m3_to_double(codes_v) * sv)
    q = rng.standard_normal((2, H, D)).astype(np.float16)
    bt = np.array([[3, 0, 5], [1, 4, -1]], np.int32)
    ctx = np.array([11, 6], np.int32)
    a = oracle.paged_attention(q, codes_k, codes_v, bt, ctx, 0.25, k_scale=sk, v_scale=sv)
    b = oracle.paged_attention(q, f16_k, f16_v, bt, ctx, 0.25)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("P", [1, 5, 16, 24, 64])
def test_partitions_recombine_to_the_unsplit_result(P):
    w, kc, vc = complete_case([1, 15, 16, 17, 48, 61], seed=14)
    full = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
    o, lse = oracle.attention_partials(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, P)
    for s, L in enumerate(w.context_lens):
        n = -(-int(L) // P)
        assert np.isnan(lse[s, :, n:]).all()
        for h in range(w.num_heads):
            comb = oracle.lse_combine(o[s, h, :n], lse[s, h, :n])
            np.testing.assert_allclose(comb, full[s, h], rtol=0, atol=1e-12)


def test_single_partition_is_the_full_result_and_lse_is_logsumexp():
    w, kc, vc = complete_case([7, 30], seed=15, deal="identity")
    full = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
    o, lse = oracle.attention_partials(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, 64)
    assert np.array_equal(o[:, :, 0], full)
    from scipy.special import logsumexp
    for s in range(2):
        K = dense_kv(w, kc, s, kc).astype(np.float64)
        for h in range(w.num_heads):
            z = w.scale * (K[:, h, :] @ w.query[s, h].astype(np.float64))
            assert abs(lse[s, h, 0] - logsumexp(z)) < 1e-12
