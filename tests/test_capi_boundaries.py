"""Each host-side check of the C ABI rejects exactly what it should.

For every check: each pointer alone null or misaligned is refused, and a
bound one step past is refused, while the last valid value is accepted.
Acceptance is observed without running anything on a device: the call
also carries an argument that a later check refuses, so the message of
that later check proves the boundary value got through. No call here gets
past the checks to a CUDA call or a launch, on any machine (the pointers
are fake addresses).
"""
import ctypes

import pytest

from pagedattention_paged_kv_decode_b200 import capi

P = 0x10000                      # fake, 16-byte aligned address
F = capi.CacheDesc(64, 16, 8, 128, capi.PA_F16)
E = capi.CacheDesc(64, 16, 8, 128, capi.PA_E4M3)
ROW = 8 * 128
NAN = float("nan")
INV = capi.PA_ERR_INVALID


@pytest.fixture(scope="module")
def L():
    return capi.lib()


def said(L, rc, needle, code=INV):
    msg = L.pa_last_error().decode()
    return rc == code and needle in msg


def test_cache_descriptor_bounds(L):
    # one block and 65535 heads are valid (a write of zero tokens stops right after the checks)
    for d in (capi.CacheDesc(1, 16, 8, 128, 0), capi.CacheDesc(64, 16, 65535, 64, 0)):
        assert L.pa_kv_cache_write(P, P, ROW, ROW, P, P, d, P, 0, 1.0, 1.0, None) == capi.PA_OK, L.pa_last_error()


def test_slot_mapping_checks(L):
    for i in range(3):
        args = [P] * 3
        args[i] = None
        assert said(L, L.pa_slot_mapping(args[0], args[1], 4, args[2], 2, F, None), "null pointer")
    assert said(L, L.pa_slot_mapping(P, P, 0, P, 2, F, None), "max_blocks_per_seq")


def test_kv_cache_write_checks(L):
    w = lambda k, v, ks, vs, kc, vc, sl, desc=F, kscale=1.0: L.pa_kv_cache_write(  # noqa: E731
        k, v, ks, vs, kc, vc, desc, sl, 4, kscale, 1.0, None)
    for i in range(5):                                       # each pointer alone null
        args = [P] * 5
        args[i] = None
        assert said(L, w(args[0], args[1], ROW, ROW, args[2], args[3], args[4]), "null pointer")
    for i in range(4):                                       # each buffer alone misaligned
        args = [P] * 4
        args[i] = P + 8
        assert said(L, w(args[0], args[1], ROW, ROW, args[2], args[3], P), "aligned")
    # strides: the row length is the smallest valid one (E4M3 with a zero scale then fails later)
    assert said(L, w(P, P, ROW, ROW, P, P, P, E, 0.0), "k_scale")
    for ks, vs in ((ROW - 8, ROW), (ROW, ROW - 8), (ROW + 4, ROW), (ROW, ROW + 4)):
        assert said(L, w(P, P, ks, vs, P, P, P), "stride")


def test_copy_and_swap_checks(L):
    assert said(L, L.pa_copy_blocks(P, P + 8, F, P, 1, None), "aligned")
    assert said(L, L.pa_copy_blocks(P + 8, P, F, P, 1, None), "aligned")
    for i in range(3):
        args = [P] * 3
        args[i] = None
        assert said(L, L.pa_copy_blocks(args[0], args[1], F, args[2], 1, None), "null pointer")
    # one-block pools are valid: the null pair list then fails
    assert said(L, L.pa_swap_blocks(P, P, 1, P, P, 8, F, None, 1, None), "null pointer")
    assert said(L, L.pa_swap_blocks(P, P, 8, P, P, 1, F, None, 1, None), "null pointer")
    assert said(L, L.pa_swap_blocks(P, P, 8, P, P, 0, F, P, 1, None), "must be >= 1")
    for i in range(5):
        args = [P] * 5
        args[i] = None
        assert said(L, L.pa_swap_blocks(args[0], args[1], 8, args[2], args[3], 8, F, args[4], 1, None),
                    "null pointer")


def _decode(L, out=P, q=P, kc=P, vc=P, bt=P, width=4, ctx=P, S=2, max_ctx=64, scale=0.1, desc=F):
    return L.pa_paged_attention_decode(out, q, kc, vc, desc, bt, width, ctx, S, max_ctx, scale, 1.0, 1.0, None)


def test_decode_argument_checks(L):
    # shared by every decode entry point; a NaN scale is the later check that fails
    assert said(L, _decode(L, S=65535, scale=NAN), "scale")
    assert said(L, _decode(L, S=65536), "num_seqs")
    assert said(L, _decode(L, width=1, scale=NAN), "scale")
    assert said(L, _decode(L, width=0), "max_blocks_per_seq")
    assert said(L, _decode(L, width=(1 << 27) - 1, scale=NAN), "scale")        # 2^31 - 16 slots
    assert said(L, _decode(L, width=1 << 27), "overflows", capi.PA_ERR_OVERFLOW)
    assert said(L, _decode(L, max_ctx=0, scale=NAN), "scale")
    assert said(L, _decode(L, max_ctx=-1), "max_context_len")
    names = ("out", "q", "kc", "vc", "bt", "ctx")
    for n in names:
        assert said(L, _decode(L, **{n: None}), "null pointer"), n
    for n in ("out", "q", "kc", "vc"):
        assert said(L, _decode(L, **{n: P + 8}), "aligned"), n


def test_append_and_shared_prefix_checks(L):
    bad_cfg = ctypes.byref(capi.DecodeConfig(24, 0, 0, 0, 0))    # fails in the launch-shape check
    app = lambda S, nk, nv, ks, vs, cfg=bad_cfg: L.pa_paged_attention_decode_append(  # noqa: E731
        P, P, nk, nv, ks, vs, P, P, F, P, 4, P, S, 64, 0.1, 1.0, 1.0, None, cfg, None, 0, None)
    assert said(L, app(1, None, P, ROW, ROW), "null new_key")                 # one sequence is work to do
    assert said(L, app(2, P, P, ROW, ROW), "partition_size")                  # row-length strides are valid
    for nk, nv in ((P + 8, P), (P, P + 8)):
        assert said(L, app(2, nk, nv, ROW, ROW), "aligned")
    for ks, vs in ((ROW - 8, ROW), (ROW, ROW - 8), (ROW + 4, ROW), (ROW, ROW + 4)):
        assert said(L, app(2, P, P, ks, vs), "stride")
    pre = lambda nk, nv, ks, vs, blocks, cfg=bad_cfg: L.pa_paged_attention_decode_shared_prefix(  # noqa: E731
        P, P, nk, nv, ks, vs, P, P, F, P, 4, P, 2, 64, blocks, 0.1, 1.0, 1.0, None, cfg, None, 0, None)
    assert said(L, pre(None, None, ROW, ROW, 4), "partition_size")             # prefix = the whole table
    assert said(L, pre(None, None, ROW, ROW, 5), "shared_prefix_blocks")
    assert said(L, pre(None, None, ROW, ROW, 1), "partition_size")             # one block is valid
    assert said(L, pre(P, P, ROW, ROW, 2), "partition_size")                   # row-length strides are valid
    for nk, nv in ((P + 8, P), (P, P + 8)):
        assert said(L, pre(nk, nv, ROW, ROW, 2), "aligned")
    for ks, vs in ((ROW - 8, ROW), (ROW, ROW - 8), (ROW + 4, ROW), (ROW, ROW + 4)):
        assert said(L, pre(P, P, ks, vs, 2), "stride")
    assert L.pa_shared_prefix_workspace_size(F, 2, 64, 1, None) > 0
    assert L.pa_shared_prefix_workspace_size(F, 2, 64, 4, None) > 0           # prefix exactly at the bound
    assert L.pa_shared_prefix_workspace_size(F, 2, 63, 4, None) == 0


def _choose(L, desc, S, maxL, **kw):
    cfg = capi.DecodeConfig(kw.get("partition_size", 0), kw.get("heads_per_cta", 0), kw.get("warps_per_head", 0),
                            kw.get("stages", 0), kw.get("units_per_cta", 0))
    return L.pa_decode_choose_config(desc, S, maxL, ctypes.byref(cfg))


def test_launch_shape_checks(L):
    assert _choose(L, F, 0, 64) == capi.PA_OK and _choose(L, F, 16, 0) == capi.PA_OK
    assert said(L, _choose(L, F, -1, 64), "num_seqs") and said(L, _choose(L, F, 16, -1), "max_context_len")
    assert _choose(L, F, 16, 512, partition_size=16) == capi.PA_OK            # one block per partition
    assert _choose(L, F, 16, 512, heads_per_cta=8, stages=2) == capi.PA_OK
    H12 = capi.CacheDesc(64, 16, 12, 128, 0)
    assert said(L, _choose(L, H12, 16, 512, heads_per_cta=3), "heads_per_cta")  # divides 12, still not allowed
    assert _choose(L, F, 16, 512, units_per_cta=4, heads_per_cta=1, warps_per_head=1, stages=2) == capi.PA_OK
    assert said(L, _choose(L, F, 16, 512, warps_per_head=3, heads_per_cta=1, stages=3), "warps_per_head")


def test_prefill_checks(L):
    T = 100
    slots = lambda S, tq, mql, ptrs=(P, P, P, P): L.pa_prefill_slot_mapping(  # noqa: E731
        ptrs[0], ptrs[1], ptrs[2], 4, ptrs[3], S, tq, mql, F, None)
    assert said(L, slots(65535, -1, 64), "total_q")                           # 65535 sequences are valid
    assert said(L, slots(65536, T, 64), "num_seqs")
    assert said(L, slots(2, T, 0, (None, P, P, P)), "null pointer")           # max_query_len 0 is valid
    for i in range(4):
        ptrs = [P] * 4
        ptrs[i] = None
        assert said(L, slots(2, T, 64, ptrs), "null pointer")
    pf = lambda ptrs=(P,) * 7, width=4, scale=NAN: L.pa_paged_prefill(  # noqa: E731
        ptrs[0], ptrs[1], ptrs[2], ptrs[3], ptrs[4], F, ptrs[5], width, ptrs[6], 2, T, 64, scale, None)
    for i in range(7):
        ptrs = [P] * 7
        ptrs[i] = None
        assert said(L, pf(ptrs), "null pointer")
    for i in (0, 1, 3, 4):                                                    # out, query, caches
        ptrs = [P] * 7
        ptrs[i] = P + 8
        assert said(L, pf(ptrs), "aligned")
    assert said(L, pf(width=1), "scale")
    assert said(L, pf(width=(1 << 27) - 1), "scale")
    assert said(L, pf(width=1 << 27), "overflows", capi.PA_ERR_OVERFLOW)
