"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake in a copy of oracle/pagedkv_oracle.c (a
text substitution), builds it, routes the oracle through it and runs the
pin battery: the worked and growth slot examples, binary16 and E4M3 decoding
against numpy/torch, E4M3 encoding against torch, the saturation points,
signed zeros and every tie between neighbouring codes (to the even code),
dense attention on identity tables against torch's SDPA, the closed forms,
exact-sum brute force, physical-block relabelling, cache-write read-back,
block copy and swap semantics, E4M3 attention against fp16 caches holding
the decoded values at distinct K and V scales, an empty context (slot -1,
zero output), the log-sum-exp identity, and for the
prefill the worked example as a full prompt, one-token chunks against the
decode slots, and chunks after a cached context against torch's SDPA with a
position mask. Every mutant
must fail at least one pin; the unmodified source must pass all of them.
"""
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
import workloads as W

SRC = os.path.join(os.path.dirname(oracle.__file__), "pagedkv_oracle.c")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

MUTANTS = {
    "slot offset uses division": ("slot_mapping[s] = physical * block_size + pos % block_size;",
                                  "slot_mapping[s] = physical * block_size + pos / block_size;"),
    "prefill slot offset uses division": ("slot_mapping[query_start[s] + i] = physical * block_size + pos % block_size;",
                                          "slot_mapping[query_start[s] + i] = physical * block_size + pos / block_size;"),
    "slot of position L instead of L-1": ("int pos = L - 1;", "int pos = L;"),
    "f16 exponent bias": ("v = ldexp((double)(1024 + f), e - 25);", "v = ldexp((double)(1024 + f), e - 24);"),
    "e4m3 exponent bias": ("v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 9);"),
    "e4m3 encode truncates": ("double n = nearbyint(a / quantum);", "double n = floor(a / quantum);"),
    "e4m3 ties away from zero": ("double n = nearbyint(a / quantum);", "double n = round(a / quantum);"),
    "e4m3 negative zero loses its sign": ("    if (a == 0.0)\n        return sign;", "    if (a == 0.0)\n        return 0;"),
    "e4m3 saturates to NaN": ("        return sign | 0x7e;\n    if (a == 0.0)", "        return sign | 0x7f;\n    if (a == 0.0)"),
    "softmax scale dropped": ("z[t - t0] = scale * dot;", "z[t - t0] = dot;"),
    "row offset by block division": ("int64_t base = (((int64_t)blk * block_size + t % block_size) * num_heads + h) * head_size;",
                                     "int64_t base = (((int64_t)blk * block_size + t / block_size) * num_heads + h) * head_size;"),
    "logical block by modulo": ("int logical = t / block_size;", "int logical = t % block_size;"),
    "keys read from the value cache": ("dot += oracle_f16_to_double(q[d]) * cache_value(key_cache, kv_dtype, base + d, k_scale);",
                                       "dot += oracle_f16_to_double(q[d]) * cache_value(value_cache, kv_dtype, base + d, k_scale);"),
    "softmax weight sign": ("acc += exp(z[i] - m) * cache_value", "acc += exp(m - z[i]) * cache_value"),
    "normaliser omitted": ("o[d] = acc / l;", "o[d] = acc;"),
    "E4M3 V written with k_scale": ("float vq = vf / v_scale;", "float vq = vf / k_scale;"),
    "E4M3 K written with v_scale": ("float kq = kf / k_scale;", "float kq = kf / v_scale;"),
    "E4M3 K scale multiplied": ("float kq = kf / k_scale;", "float kq = kf * k_scale;"),
    "copy direction reversed": ("memmove((char *)key_cache + dst * block_bytes,\n                (char *)key_cache + src * block_bytes",
                                "memmove((char *)key_cache + src * block_bytes,\n                (char *)key_cache + dst * block_bytes"),
    "swap copies only K": ("memcpy((char *)dst_value + dst * block_bytes", "memcpy((char *)dst_key + dst * block_bytes"),
    "lse combine weight sign": ("acc += exp(lse[p] - M) * o", "acc += exp(M - lse[p]) * o"),
    "last partition dropped": ("int nparts = L > 0 ? (L + partition_size - 1) / partition_size : 0;",
                               "int nparts = L > 0 ? L / partition_size : 0;"),
    "partial lse without log": ("lse[slot] = m + log(l);", "lse[slot] = m + l;"),
    "prefill slot position from the chunk start": ("int pos = L - n + i;", "int pos = i;"),
    "prefill row misses its own token": ("s, h, 0, pos + 1, (double)scale,", "s, h, 0, pos, (double)scale,"),
    "prefill row sees one token ahead": ("s, h, 0, pos + 1, (double)scale,", "s, h, 0, pos + 2, (double)scale,"),
    "prefill position ignores the cached context": ("int pos = context_lens[s] - n + (row - query_start[s]);",
                                                    "int pos = row - query_start[s];"),
    "prefill query row taken by sequence": ("const uint16_t *q = query + ((int64_t)row * num_heads + h) * head_size;",
                                            "const uint16_t *q = query + ((int64_t)s * num_heads + h) * head_size;"),
    "keys dequantised with v_scale": ("cache_value(key_cache, kv_dtype, base + d, k_scale)",
                                      "cache_value(key_cache, kv_dtype, base + d, v_scale)"),
    "values dequantised with k_scale": ("cache_value(value_cache, kv_dtype, rowbase[i] + d, v_scale)",
                                        "cache_value(value_cache, kv_dtype, rowbase[i] + d, k_scale)"),
    "E4M3 cache scale dropped": ("return oracle_e4m3_to_double(((const uint8_t *)cache)[idx]) * scale;",
                                 "return oracle_e4m3_to_double(((const uint8_t *)cache)[idx]);"),
    "empty context gets a slot": ("if (L <= 0) {\n            slot_mapping[s] = -1;",
                                  "if (L < 0) {\n            slot_mapping[s] = -1;"),
    "empty context attends over nothing": ("if (L <= 0) {\n        for (int d = 0; d < head_size; ++d)\n            o[d] = 0.0;",
                                           "if (L < 0) {\n        for (int d = 0; d < head_size; ++d)\n            o[d] = 0.0;"),
    "head index ignored": ("const uint16_t *q = query + ((int64_t)s * num_heads + h) * head_size;",
                           "const uint16_t *q = query + ((int64_t)s * num_heads + 0) * head_size;"),
}


def _build(source: str, path: str):
    with open(path + ".c", "w") as f:
        f.write(source)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-shared",
                           "-fPIC", path + ".c", "-o", path, "-lm"])


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _complete(ctx, H=3, D=16, B=8, seed=0, deal="permuted"):
    ctx = np.asarray(ctx)
    need = sum(-(-int(L) // B) for L in ctx)
    w = W.build("m", H, D, B, "f16", ctx, need + 4, max(1, -(-int(ctx.max()) // B)), seed,
                q_std=1.0, kv_std=1.0, deal_order=deal)
    kc, vc = w.pool_host()
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, B)
    oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots)
    return w, kc, vc


def pin_battery():
    """Returns the names of the pins that fail (each pin is a small check)."""
    failed = []

    def pin(name, fn):
        try:
            ok = fn()
        except Exception:
            ok = False
        if not ok:
            failed.append(name)

    def worked_example():
        tables = {"A": [5, 8], "B": [3, -1]}
        return all(oracle.slot_mapping(np.array([tables[sq]], np.int32), np.array([int(t) + 1], np.int32), 16)[0] == int(sl)
                   for sq, t, _, _, sl in _rows("slot_mapping_worked_example.txt"))

    def growth_example():
        bt = np.array([[7, 2, 3, -1]], np.int32)
        return all(oracle.slot_mapping(bt, np.array([int(ctx)], np.int32), 4)[0] == int(sl)
                   for _, ctx, _, _, _, sl in _rows("block_growth_example.txt"))

    def f16_decode():
        bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
        ref = bits.view(np.float16).astype(np.float64)
        got = oracle.f16_to_double(bits.view(np.float16))
        fin = np.isfinite(ref)
        return np.array_equal(got[fin], ref[fin])

    def e4m3_decode():
        ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        got = oracle.e4m3_to_double(np.arange(256, dtype=np.uint8))
        fin = ~np.isnan(ref)
        return np.array_equal(got[fin], ref[fin])

    def e4m3_encode():
        x = np.random.default_rng(0).standard_normal(20000).astype(np.float32) * 40
        x = x[np.abs(x) <= 448]
        ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        sat = oracle.e4m3_from_float(np.float32([449, 1e9, -500, 0.0, -0.0]))
        # codes 0x00..0x7E ascend in magnitude, so the value halfway between
        # codes k and k+1 rounds (ties to even) to whichever of them is even
        codes = np.arange(0x7F, dtype=np.uint8)
        vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)   # exact: five significant bits at most
        even = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[1:]).astype(np.uint8)
        return (np.array_equal(oracle.e4m3_from_float(x), ref) and list(sat) == [0x7E, 0x7E, 0xFE, 0x00, 0x80]
                and np.array_equal(oracle.e4m3_from_float(mids), even)
                and np.array_equal(oracle.e4m3_from_float(-mids), even | 0x80)
                and np.array_equal(oracle.e4m3_from_float(vals.astype(np.float32)), codes)       # codes themselves
                and np.array_equal(oracle.e4m3_from_float(-vals.astype(np.float32)), codes | 0x80))

    def dense_equivalence():
        w, kc, vc = _complete([1, 9, 30], H=3, D=16, B=8, deal="identity", seed=1)
        got = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
        for s in range(3):
            base = int(w.block_tables[s, 0]) * 8
            L = int(w.context_lens[s])
            K = torch.from_numpy(kc.reshape(-1, 3, 16)[base:base + L].astype(np.float64)).permute(1, 0, 2)
            V = torch.from_numpy(vc.reshape(-1, 3, 16)[base:base + L].astype(np.float64)).permute(1, 0, 2)
            q = torch.from_numpy(w.query[s].astype(np.float64))[:, None, :]
            ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, scale=w.scale)[:, 0, :].numpy()
            if not np.abs(got[s] - ref).max() <= 1e-12:   # NaN fails too
                return False
        return True

    def context_one():
        w, kc, vc = _complete([1, 1], seed=3)
        got = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
        return np.array_equal(got, w.new_value.astype(np.float64))

    def brute_force():
        rng = np.random.default_rng(5)
        H, D, B, ctx = 2, 3, 2, np.array([5, 3])
        nb = 8
        kc = rng.standard_normal((nb, B, H, D)).astype(np.float16)
        vc = rng.standard_normal((nb, B, H, D)).astype(np.float16)
        q = rng.standard_normal((2, H, D)).astype(np.float16)
        bt = np.array([[6, 1, 4], [0, 7, -1]], np.int32)
        sc = float(np.float32(0.7))   # the scale crosses the boundary as fp32
        got = oracle.paged_attention(q, kc, vc, bt, ctx, sc)
        for s, L in enumerate(ctx):
            for h in range(H):
                rows = [(int(bt[s][t // B]), t % B) for t in range(int(L))]
                z = [sc * math.fsum(float(q[s, h, d]) * float(kc[b, r, h, d]) for d in range(D)) for b, r in rows]
                p = [math.exp(x) for x in z]
                for d in range(D):
                    ref = math.fsum(p[i] * float(vc[b, r, h, d]) for i, (b, r) in enumerate(rows)) / math.fsum(p)
                    if not abs(got[s, h, d] - ref) <= 1e-12:
                        return False
        return True

    def relabelling():
        w, kc, vc = _complete([5, 17, 33], seed=2)
        base = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
        perm = np.random.default_rng(9).permutation(w.num_blocks).astype(np.int32)
        kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
        kc2[perm], vc2[perm] = kc, vc
        bt2 = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
        return np.array_equal(base, oracle.paged_attention(w.query, kc2, vc2, bt2, w.context_lens, w.scale))

    def cache_write_readback():
        # slots 0 (the first), 6, 13 and 15 (the last) of a 4 x 4 pool; a
        # negative slot is padding; every other slot must stay zero
        slots = np.array([0, 6, -1, 13, 15], np.int32)
        key = np.random.default_rng(1).standard_normal((5, 2, 8)).astype(np.float16) + np.float16(0.25)
        kc = np.zeros((4, 4, 2, 8), np.float16)
        vc = np.zeros_like(kc)
        oracle.kv_cache_write(key, key + 1, kc, vc, slots)
        ek = np.zeros((4, 4, 2, 8), np.uint8)
        ev = np.zeros_like(ek)
        oracle.kv_cache_write(key, key, ek, ev, slots, 0.5, 2.0)
        want_k, want_v = np.zeros_like(kc), np.zeros_like(kc)
        want_ek, want_ev = np.zeros_like(ek), np.zeros_like(ek)
        for i, sl in enumerate(slots):
            if sl >= 0:
                b, r = divmod(int(sl), 4)
                want_k[b, r], want_v[b, r] = key[i], key[i] + 1
                want_ek[b, r] = oracle.e4m3_from_float(key[i].astype(np.float32) / np.float32(0.5))
                want_ev[b, r] = oracle.e4m3_from_float(key[i].astype(np.float32) / np.float32(2.0))
        return (np.array_equal(kc.view(np.uint16), want_k.view(np.uint16))
                and np.array_equal(vc.view(np.uint16), want_v.view(np.uint16))
                and np.array_equal(ek, want_ek) and np.array_equal(ev, want_ev) and want_ek.any())

    def copy_semantics():
        kc = np.random.default_rng(2).standard_normal((5, 2, 1, 8)).astype(np.float16)
        vc = kc + 1
        k0 = kc.copy()
        v0 = vc.copy()
        oracle.copy_blocks(kc, vc, np.array([[1, 3], [2, 0]], np.int32))   # block 0 as a destination
        oracle.copy_blocks(kc, vc, np.array([[0, 4]], np.int32))           # and then as a source
        wk, wv = k0.copy(), v0.copy()
        wk[3], wv[3], wk[0], wv[0], wk[4], wv[4] = k0[1], v0[1], k0[2], v0[2], k0[2], v0[2]
        return np.array_equal(kc, wk) and np.array_equal(vc, wv)

    def swap_semantics():
        src = np.random.default_rng(3).standard_normal((3, 2, 1, 8)).astype(np.float16)
        dk = np.zeros((4,) + src.shape[1:], np.float16)
        dv = np.zeros_like(dk)
        oracle.swap_blocks(dk, dv, src, src + 1, np.array([[2, 1], [0, 3], [1, 0]], np.int32))
        wk, wv = np.zeros_like(dk), np.zeros_like(dk)
        wk[1], wv[1], wk[3], wv[3], wk[0], wv[0] = src[2], src[2] + 1, src[0], src[0] + 1, src[1], src[1] + 1
        return np.array_equal(dk, wk) and np.array_equal(dv, wv)

    def empty_context():
        # a sequence with no context has no slot and a zero output row (the
        # last row, so that a write past it leaves the array)
        rng = np.random.default_rng(22)
        bt = np.array([[1, 3], [2, -1]], np.int32)
        ctx = np.array([5, 0], np.int32)
        slots = oracle.slot_mapping(bt, ctx, 4)
        kc = rng.standard_normal((4, 4, 1, 8)).astype(np.float16)
        vc = rng.standard_normal((4, 4, 1, 8)).astype(np.float16)
        q = rng.standard_normal((2, 1, 8)).astype(np.float16)
        out = oracle.paged_attention(q, kc, vc, bt, ctx, 0.5)
        return list(slots) == [12, -1] and np.array_equal(out[1], np.zeros((1, 8))) and np.isfinite(out).all()

    def subsets():
        # selected (sequence, head) / (row, head) pairs equal those rows of the full result
        w, kc, vc = _complete([5, 17, 33], seed=24)
        full = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
        pairs = np.array([[2, 1], [0, 2], [1, 0], [2, 2]], np.int32)
        sub = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, seq_head=pairs)
        if not all(np.array_equal(sub[i], full[s, h]) for i, (s, h) in enumerate(pairs)):
            return False
        ctx, n = [12, 9], [5, 9]
        pw = W.build_prefill("sub", 3, 16, 8, ctx, n, 6, 2, 25, 1.0, 1.0)
        pk_, pv_ = pw.pool_host()
        oracle.kv_cache_write(pw.new_key, pw.new_value, pk_, pv_,
                              oracle.prefill_slot_mapping(pw.query_start, pw.block_tables, pw.context_lens, 8))
        pfull = oracle.paged_prefill(pw.query, pw.query_start, pk_, pv_, pw.block_tables, pw.context_lens, pw.scale)
        rows = np.array([[13, 2], [0, 1], [6, 0], [4, 2]], np.int32)
        psub = oracle.paged_prefill(pw.query, pw.query_start, pk_, pv_, pw.block_tables, pw.context_lens, pw.scale,
                                    row_head=rows)
        return all(np.array_equal(psub[i], pfull[r, h]) for i, (r, h) in enumerate(rows))

    def input_validation():
        # each input one step past a bound is rejected; the last valid value
        # at that bound is accepted
        def rejects(fn):
            try:
                fn()
            except ValueError:
                return True
            return False

        rng = np.random.default_rng(26)
        pool = rng.standard_normal((4, 4, 1, 8)).astype(np.float16)
        q = rng.standard_normal((2, 1, 8)).astype(np.float16)
        bt = np.array([[1, 3], [0, 2]], np.int32)
        row = np.zeros((1, 1, 8), np.float16)
        ok = [
            oracle.slot_mapping(bt, np.array([8, 1], np.int32), 4)[0] == 3 * 4 + 3,            # last table slot
            rejects(lambda: oracle.slot_mapping(bt, np.array([9, 1], np.int32), 4)),           # one past the table
            list(oracle.prefill_slot_mapping(np.array([0, 0, 1], np.int32), bt, np.array([3, 1], np.int32), 4))
            == [0],                                                                             # empty chunk
            rejects(lambda: oracle.prefill_slot_mapping(np.array([0, 4, 5], np.int32), bt,
                                                        np.array([3, 1], np.int32), 4)),        # chunk > context
            rejects(lambda: oracle.prefill_slot_mapping(np.array([0, 9, 10], np.int32), bt,
                                                        np.array([9, 1], np.int32), 4)),        # past the table
            rejects(lambda: oracle.kv_cache_write(row, row, pool.copy(), pool.copy(), np.array([16], np.int32))),
            rejects(lambda: oracle.copy_blocks(pool.copy(), pool.copy(), np.array([[4, 0]], np.int32))),
            rejects(lambda: oracle.copy_blocks(pool.copy(), pool.copy(), np.array([[0, 4]], np.int32))),
            rejects(lambda: oracle.copy_blocks(pool.copy(), pool.copy(), np.array([[-1, 0]], np.int32))),
            rejects(lambda: oracle.swap_blocks(pool[:2].copy(), pool[:2].copy(), pool, pool,
                                               np.array([[3, 2]], np.int32))),                  # dst past its pool
            rejects(lambda: oracle.swap_blocks(pool[:2].copy(), pool[:2].copy(), pool, pool,
                                               np.array([[4, 1]], np.int32))),                  # src past its pool
            rejects(lambda: oracle.paged_attention(q, pool, pool, np.array([[1, 4], [0, 2]], np.int32),
                                                   np.array([8, 1], np.int32), 0.5)),           # block id = pool size
            rejects(lambda: oracle.paged_attention(q, pool, pool, np.array([[1, -1], [0, 2]], np.int32),
                                                   np.array([8, 1], np.int32), 0.5)),           # hole in the table
            rejects(lambda: oracle.paged_attention(q, pool, pool, bt, np.array([9, 1], np.int32), 0.5)),
            rejects(lambda: oracle.paged_attention(q, pool, pool, bt, np.array([8, 1], np.int32), 0.5,
                                                   seq_head=np.array([[2, 0]], np.int32))),
            rejects(lambda: oracle.paged_attention(q, pool, pool, bt, np.array([8, 1], np.int32), 0.5,
                                                   seq_head=np.array([[0, 1]], np.int32))),
            rejects(lambda: oracle.paged_prefill(q, np.array([0, 2, 2], np.int32), pool, pool, bt,
                                                 np.array([1, 1], np.int32), 0.5)),             # first chunk > context
            rejects(lambda: oracle.paged_prefill(q, np.array([0, 1, 2], np.int32), pool, pool, bt,
                                                 np.array([3, 1], np.int32), 0.5,
                                                 row_head=np.array([[2, 0]], np.int32))),
            rejects(lambda: oracle.paged_prefill(q, np.array([0, 1, 2], np.int32), pool, pool, bt,
                                                 np.array([3, 1], np.int32), 0.5,
                                                 row_head=np.array([[0, 1]], np.int32))),
        ]
        return all(ok)

    def e4m3_attention():
        # an E4M3 cache at scales (1/2, 4) against fp16 caches holding its
        # decoded values times those scales (exact: small powers of two)
        rng = np.random.default_rng(21)
        codes_k = rng.integers(0, 256, (5, 4, 2, 8), dtype=np.uint8)
        codes_v = rng.integers(0, 256, (5, 4, 2, 8), dtype=np.uint8)
        for c in (codes_k, codes_v):
            c[(c & 0x7F) == 0x7F] = 0x3C
            c[(c & 0x78) >= 0x60] &= 0x9F
        f16_k = (torch.from_numpy(codes_k).view(torch.float8_e4m3fn).to(torch.float64).numpy() * 0.5).astype(np.float16)
        f16_v = (torch.from_numpy(codes_v).view(torch.float8_e4m3fn).to(torch.float64).numpy() * 4.0).astype(np.float16)
        q = rng.standard_normal((2, 2, 8)).astype(np.float16)
        bt = np.array([[3, 0], [1, 4]], np.int32)
        ctx = np.array([7, 5], np.int32)
        a = oracle.paged_attention(q, codes_k, codes_v, bt, ctx, 0.3, k_scale=0.5, v_scale=4.0)
        return np.array_equal(a, oracle.paged_attention(q, f16_k, f16_v, bt, ctx, 0.3))

    def lse_identity():
        w, kc, vc = _complete([1, 15, 16, 17, 32, 40], seed=14)
        full = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
        o, lse = oracle.attention_partials(w.query, kc, vc, w.block_tables, w.context_lens, w.scale, 16)
        for s, L in enumerate(w.context_lens):
            n = -(-int(L) // 16)
            if not (np.isnan(lse[s, :, n:]).all() and np.isnan(o[s, :, n:]).all()):
                return False           # a partition past the context holds nothing
            for h in range(w.num_heads):
                if not np.abs(oracle.lse_combine(o[s, h, :n], lse[s, h, :n]) - full[s, h]).max() <= 1e-12:
                    return False
        # an empty context has no partition at all (the last sequence, so
        # that a write past its rows leaves the arrays)
        bt = np.array([[0, 2], [1, -1]], np.int32)
        pool = np.random.default_rng(23).standard_normal((3, 16, 1, 8)).astype(np.float16)
        q = np.ones((2, 1, 8), np.float16)
        o, lse = oracle.attention_partials(q, pool, pool, bt, np.array([20, 0], np.int32), 0.5, 16)
        return bool(np.isnan(o[1]).all() and np.isnan(lse[1]).all() and np.isfinite(lse[0]).all())

    def prefill_worked_example():
        got = oracle.prefill_slot_mapping(np.array([0, 32, 48], np.int32), np.array([[5, 8], [3, -1]], np.int32),
                                          np.array([32, 16], np.int32), 16)
        want = [int(sl) for sq, t, _, _, sl in _rows("slot_mapping_worked_example.txt")]
        return [int(x) for x in got] == want

    def prefill_one_token_chunks():
        w = W.build("d", 2, 8, 4, "f16", np.array([1, 4, 5, 13]), 30, 4, 3, 1.0, 1.0)
        got = oracle.prefill_slot_mapping(np.arange(5, dtype=np.int32), w.block_tables, w.context_lens, 4)
        return np.array_equal(got, oracle.slot_mapping(w.block_tables, w.context_lens, 4))

    def prefill_dense_causal():
        ctx, n = [12, 9, 17, 6], [5, 9, 1, 0]
        need = sum(-(-L // 8) for L in ctx)
        w = W.build_prefill("p", 2, 16, 8, ctx, n, need + 2, 3, 2, 1.0, 1.0, deal_order="identity")
        kc, vc = w.pool_host()
        oracle.kv_cache_write(w.new_key, w.new_value, kc, vc,
                              oracle.prefill_slot_mapping(w.query_start, w.block_tables, w.context_lens, 8))
        got = oracle.paged_prefill(w.query, w.query_start, kc, vc, w.block_tables, w.context_lens, w.scale)
        for s in range(3):
            r0, r1, L = int(w.query_start[s]), int(w.query_start[s + 1]), ctx[s]
            base = int(w.block_tables[s, 0]) * 8
            K = torch.from_numpy(kc.reshape(-1, 2, 16)[base:base + L].astype(np.float64)).permute(1, 0, 2)
            V = torch.from_numpy(vc.reshape(-1, 2, 16)[base:base + L].astype(np.float64)).permute(1, 0, 2)
            q = torch.from_numpy(w.query[r0:r1].astype(np.float64)).permute(1, 0, 2)
            mask = torch.from_numpy(np.arange(L)[None, :] <= np.arange(L - n[s], L)[:, None])
            ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=w.scale)
            if not np.abs(got[r0:r1] - ref.permute(1, 0, 2).numpy()).max() <= 1e-12:
                return False
        return True

    for name, fn in [("worked example", worked_example), ("growth example", growth_example),
                     ("f16 decode", f16_decode), ("e4m3 decode", e4m3_decode), ("e4m3 encode", e4m3_encode),
                     ("dense equivalence", dense_equivalence), ("context one", context_one),
                     ("brute force", brute_force), ("relabelling", relabelling),
                     ("cache write", cache_write_readback), ("copy", copy_semantics), ("swap", swap_semantics),
                     ("empty context", empty_context), ("e4m3 attention", e4m3_attention),
                     ("subsets", subsets), ("input validation", input_validation),
                     ("lse identity", lse_identity), ("prefill worked example", prefill_worked_example),
                     ("prefill one-token chunks", prefill_one_token_chunks),
                     ("prefill dense causal", prefill_dense_causal)]:
        pin(name, fn)
    return failed


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


def test_unmodified_source_passes_every_pin(source, tmp_path):
    path = str(tmp_path / "liborig.so")
    _build(source, path)
    with oracle.using_library(path):
        assert pin_battery() == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(source, tmp_path, name):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation anchor not unique: {name}"
    path = str(tmp_path / "libmutant.so")
    _build(source.replace(old, new), path)
    with oracle.using_library(path):
        failed = pin_battery()
    assert failed, f"no pin caught: {name}"
