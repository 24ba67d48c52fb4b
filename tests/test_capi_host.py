"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol that include/pagedkv.h declares, and rejects bad arguments before any
CUDA call (so these run on a machine without a GPU)."""
import ctypes
import os
import re

import pytest

from pagedattention_paged_kv_decode_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")


def declared_functions():
    with open(HEADER, encoding="utf-8") as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path_calls():
    names = declared_functions()
    for n in ("pa_kv_cache_write", "pa_paged_attention_decode", "pa_copy_blocks", "pa_slot_mapping",
              "pa_paged_attention_decode_ws", "pa_check_status", "pa_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(capi.LIB)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(declared_functions()) == set(capi.SIGNATURES)


def test_version_and_empty_error():
    assert capi.lib().pa_version() == 202


F = capi.CacheDesc(64, 16, 8, 128, capi.PA_F16)
P = 0x10000  # fake, 16-byte aligned "device" address: validation fails before any use


def _last():
    return capi.lib().pa_last_error().decode()


@pytest.mark.parametrize("desc,code", [
    (capi.CacheDesc(64, 16, 8, 128, 7), capi.PA_ERR_DTYPE),
    (capi.CacheDesc(64, 8, 8, 128, 0), capi.PA_ERR_INVALID),
    (capi.CacheDesc(64, 16, 8, 96, 0), capi.PA_ERR_INVALID),
    (capi.CacheDesc(0, 16, 8, 128, 0), capi.PA_ERR_INVALID),
    (capi.CacheDesc(64, 16, 0, 128, 0), capi.PA_ERR_INVALID),
    (capi.CacheDesc(64, 16, 65536, 128, 0), capi.PA_ERR_INVALID),
    (capi.CacheDesc(1 << 27, 16, 8, 128, 0), capi.PA_ERR_OVERFLOW),
])
def test_bad_cache_descriptors(desc, code):
    L = capi.lib()
    assert L.pa_kv_cache_write(P, P, 1024, 1024, P, P, desc, P, 4, 1.0, 1.0, None) == code
    assert _last()
    assert L.pa_copy_blocks(P, P, desc, P, 4, None) == code
    assert L.pa_slot_mapping(P, P, 4, P, 4, desc, None) == code
    assert L.pa_paged_attention_decode(P, P, P, P, desc, P, 4, P, 4, 64, 0.1, 1.0, 1.0, None) == code


def test_null_and_misaligned_pointers():
    L = capi.lib()
    assert L.pa_kv_cache_write(None, P, 1024, 1024, P, P, F, P, 4, 1.0, 1.0, None) == capi.PA_ERR_INVALID
    assert L.pa_kv_cache_write(P + 2, P, 1024, 1024, P, P, F, P, 4, 1.0, 1.0, None) == capi.PA_ERR_INVALID
    assert "aligned" in _last()
    assert L.pa_kv_cache_write(P, P, 1020, 1024, P, P, F, P, 4, 1.0, 1.0, None) == capi.PA_ERR_INVALID
    assert L.pa_copy_blocks(P, None, F, P, 4, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_attention_decode(P, P + 8, P, P, F, P, 4, P, 4, 64, 0.1, 1.0, 1.0, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_attention_decode(P, P, P, P, F, None, 4, P, 4, 64, 0.1, 1.0, 1.0, None) == capi.PA_ERR_INVALID


def test_bad_scales_and_counts():
    L = capi.lib()
    E = capi.CacheDesc(64, 16, 8, 128, capi.PA_E4M3)
    assert L.pa_kv_cache_write(P, P, 1024, 1024, P, P, E, P, 4, 0.0, 1.0, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_attention_decode(P, P, P, P, E, P, 4, P, 4, 64, 0.1, 1.0, float("nan"), None) == capi.PA_ERR_INVALID
    assert L.pa_paged_attention_decode(P, P, P, P, F, P, 4, P, 4, 64, float("inf"), 1.0, 1.0, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_attention_decode(P, P, P, P, F, P, 0, P, 4, 64, 0.1, 1.0, 1.0, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_attention_decode(P, P, P, P, F, P, 4, P, -1, 64, 0.1, 1.0, 1.0, None) == capi.PA_ERR_INVALID
    assert L.pa_kv_cache_write(P, P, 1024, 1024, P, P, F, P, -3, 1.0, 1.0, None) == capi.PA_ERR_INVALID
    # zero-sized work is a no-op that launches nothing
    assert L.pa_kv_cache_write(P, P, 1024, 1024, P, P, F, P, 0, 1.0, 1.0, None) == capi.PA_OK
    assert L.pa_copy_blocks(P, P, F, P, 0, None) == capi.PA_OK
    assert L.pa_slot_mapping(P, P, 4, P, 0, F, None) == capi.PA_OK
    assert L.pa_paged_attention_decode(P, P, P, P, F, P, 4, P, 0, 64, 0.1, 1.0, 1.0, None) == capi.PA_OK


def _choose(desc, S, maxL, **kw):
    cfg = capi.DecodeConfig(kw.get("partition_size", 0), kw.get("heads_per_cta", 0),
                            kw.get("warps_per_head", 0), kw.get("stages", 0),
                            kw.get("units_per_cta", 0))
    rc = capi.lib().pa_decode_choose_config(desc, S, maxL, ctypes.byref(cfg))
    return rc, cfg


def test_config_choice_is_valid_and_fills_the_gpu():
    for desc, S, maxL in [(capi.CacheDesc(2048, 16, 32, 128, 0), 16, 192),
                          (capi.CacheDesc(16384, 16, 40, 128, 0), 64, 2048),
                          (capi.CacheDesc(700, 32, 32, 128, 0), 32, 4096),
                          (capi.CacheDesc(13600, 16, 32, 128, 1), 256, 4096),
                          (capi.CacheDesc(32, 16, 4, 64, 0), 4, 64)]:
        rc, cfg = _choose(desc, S, maxL)
        assert rc == capi.PA_OK, _last()
        assert cfg.partition_size % desc.block_size == 0
        assert desc.num_heads % cfg.heads_per_cta == 0
        units = S * (desc.num_heads // cfg.heads_per_cta) * -(-maxL // cfg.partition_size)
        assert units >= 3 * 148 or cfg.heads_per_cta == 1
        assert cfg.stages % cfg.warps_per_head == 0
        assert cfg.units_per_cta * cfg.heads_per_cta * cfg.warps_per_head <= 16
        ctas = max(-(-units // cfg.units_per_cta), min(units, 148))   # the library's grid
        assert ctas * cfg.units_per_cta >= units and ctas >= min(units, 148)


def test_config_validation_and_workspace_size():
    desc = capi.CacheDesc(2048, 16, 32, 128, 0)
    assert _choose(desc, 16, 512, partition_size=24)[0] == capi.PA_ERR_INVALID
    assert _choose(desc, 16, 512, heads_per_cta=3)[0] == capi.PA_ERR_INVALID
    assert _choose(desc, 16, 512, heads_per_cta=8, warps_per_head=4)[0] == capi.PA_ERR_INVALID  # 32 warps
    assert _choose(desc, 16, 512, stages=9)[0] == capi.PA_ERR_INVALID
    assert _choose(desc, 16, 512, units_per_cta=5)[0] == capi.PA_ERR_INVALID
    # a given warps_per_head bounds the default number of units per CTA
    small = capi.CacheDesc(100, 16, 4, 128, 0)
    rc, c = _choose(small, 12, 1100, partition_size=64, heads_per_cta=4, warps_per_head=4, stages=4)
    assert rc == 0 and c.units_per_cta * 4 * 4 <= 16
    assert _choose(desc, 16, 512, units_per_cta=4, heads_per_cta=2, warps_per_head=4)[0] == capi.PA_ERR_INVALID
    # a warp waits on a stage's barrier by phase parity: stages must be a multiple of warps
    assert _choose(desc, 16, 512, heads_per_cta=1, warps_per_head=4, stages=2)[0] == capi.PA_ERR_INVALID
    assert _choose(desc, 16, 512, heads_per_cta=2, warps_per_head=2, stages=3)[0] == capi.PA_ERR_INVALID
    rc, c = _choose(desc, 16, 512, stages=6)
    assert rc == 0 and c.stages % c.warps_per_head == 0
    rc, c = _choose(desc, 16, 512, heads_per_cta=1, warps_per_head=4)
    assert rc == 0 and c.stages % 4 == 0
    assert _choose(desc, 16, 512, heads_per_cta=8, stages=8)[0] == capi.PA_ERR_INVALID  # smem > 227 KB
    rc, cfg = _choose(desc, 16, 512, partition_size=128, heads_per_cta=2, warps_per_head=2, stages=4)
    assert rc == 0
    L = capi.lib()
    ws = L.pa_decode_workspace_size(desc, 16, 512, ctypes.byref(cfg))
    lse = -(-(16 * 32 * 4 * 4) // 256) * 256
    assert ws == lse + 16 * 32 * 4 * 128 * 4
    one = capi.DecodeConfig(512, 2, 2, 4, 1)
    assert L.pa_decode_workspace_size(desc, 16, 512, ctypes.byref(one)) == 0
    small = L.pa_paged_attention_decode_ws(P, P, P, P, desc, P, 32, P, 16, 512, 0.1, 1.0, 1.0,
                                           ctypes.byref(cfg), P, ws - 1, None)
    assert small == capi.PA_ERR_WORKSPACE
    unaligned = L.pa_paged_attention_decode_ws(P, P, P, P, desc, P, 32, P, 16, 512, 0.1, 1.0, 1.0,
                                               ctypes.byref(cfg), P + 16, ws, None)
    assert unaligned == capi.PA_ERR_WORKSPACE


def test_prefill_argument_checks():
    L = capi.lib()
    E = capi.CacheDesc(64, 16, 8, 128, capi.PA_E4M3)
    T = 100  # total_q
    # (out, query, query_start, kc, vc, desc, tables, width, ctx, S, total_q, max_query_len, scale, stream)
    assert L.pa_paged_prefill(P, P, P, P, P, E, P, 4, P, 2, T, 64, 0.1, None) == capi.PA_ERR_DTYPE
    assert "fp16" in _last()
    assert L.pa_paged_prefill(P, P, P, P, P, F, P, 4, P, -1, T, 64, 0.1, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_prefill(P, P, P, P, P, F, P, 4, P, 2, -5, 64, 0.1, None) == capi.PA_ERR_INVALID
    assert "total_q" in _last()
    assert L.pa_paged_prefill(P, P, P, P, P, F, P, 4, P, 2, T, -3, 0.1, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_prefill(P, P, None, P, P, F, P, 4, P, 2, T, 64, 0.1, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_prefill(P, P + 4, P, P, P, F, P, 4, P, 2, T, 64, 0.1, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_prefill(P, P, P, P, P, F, P, 0, P, 2, T, 64, 0.1, None) == capi.PA_ERR_INVALID
    assert L.pa_paged_prefill(P, P, P, P, P, F, P, 4, P, 2, T, 64, float("nan"), None) == capi.PA_ERR_INVALID
    assert L.pa_paged_prefill(P, P, P, P, P, capi.CacheDesc(64, 16, 8, 96, 0), P, 4, P, 2, T, 64, 0.1,
                              None) == capi.PA_ERR_INVALID
    # nothing to do: no launch, no CUDA call
    assert L.pa_paged_prefill(None, None, None, None, None, F, None, 4, None, 0, T, 64, 0.1, None) == capi.PA_OK
    assert L.pa_paged_prefill(None, None, None, None, None, F, None, 4, None, 3, T, 0, 0.1, None) == capi.PA_OK
    assert L.pa_paged_prefill(None, None, None, None, None, F, None, 4, None, 3, 0, 64, 0.1, None) == capi.PA_OK
    # (slots, query_start, tables, width, ctx, S, total_q, max_query_len, desc, stream)
    assert L.pa_prefill_slot_mapping(P, None, P, 4, P, 2, T, 64, F, None) == capi.PA_ERR_INVALID
    assert L.pa_prefill_slot_mapping(P, P, P, 0, P, 2, T, 64, F, None) == capi.PA_ERR_INVALID
    assert L.pa_prefill_slot_mapping(P, P, P, 4, P, 2, T, -1, F, None) == capi.PA_ERR_INVALID
    assert L.pa_prefill_slot_mapping(P, P, P, 4, P, 2, -1, 64, F, None) == capi.PA_ERR_INVALID
    assert L.pa_prefill_slot_mapping(P, P, P, 4, P, 70000, T, 64, F, None) == capi.PA_ERR_INVALID
    # a grid of more than 2^31 - 1 CTAs is refused before any CUDA call:
    # 65535 sequences x 8 heads x ceil(2^30 / 128) row tiles
    assert L.pa_paged_prefill(P, P, P, P, P, F, P, 4, P, 65535, T, 1 << 30, 0.1, None) == capi.PA_ERR_INVALID
    assert "too many prefill tiles" in _last()
    assert L.pa_prefill_slot_mapping(None, None, None, 4, None, 0, T, 64, F, None) == capi.PA_OK
    assert L.pa_prefill_slot_mapping(None, None, None, 4, None, 2, 0, 64, F, None) == capi.PA_OK


def test_default_config_is_valid_over_a_sweep_of_shapes():
    # every default choice must satisfy the kernel's constraints (the
    # library itself refuses a choice over the shared-memory limit)
    L = capi.lib()
    n = 0
    for D in (64, 128):
        for B in (16, 32):
            for dt in (capi.PA_F16, capi.PA_E4M3):
                for H in (1, 2, 3, 4, 8, 12, 32, 40, 64):
                    desc = capi.CacheDesc(4096, B, H, D, dt)
                    for S in (1, 2, 7, 16, 64, 256, 1024):
                        for maxL in (1, 15, 16, 17, 200, 512, 513, 4096, 32768):
                            rc, c = _choose(desc, S, maxL)
                            assert rc == capi.PA_OK, (D, B, dt, H, S, maxL, _last())
                            assert c.partition_size >= B and c.partition_size % B == 0
                            assert c.heads_per_cta in (1, 2, 4, 8) and H % c.heads_per_cta == 0
                            assert c.warps_per_head in (1, 2, 4)
                            assert 2 <= c.stages <= 8 and c.stages % c.warps_per_head == 0
                            assert 1 <= c.units_per_cta <= 4
                            assert c.units_per_cta * c.heads_per_cta * c.warps_per_head <= 16
                            parts = max(1, -(-maxL // c.partition_size))
                            ws = L.pa_decode_workspace_size(desc, S, maxL, ctypes.byref(c))
                            assert (ws == 0) == (parts == 1), (D, B, H, S, maxL, ws, parts)
                            n += 1
    assert n == 2 * 2 * 2 * 9 * 7 * 9


def test_swap_append_and_shared_prefix_argument_checks():
    L = capi.lib()
    D = capi.CacheDesc(64, 16, 8, 128, capi.PA_F16)
    # (dst_k, dst_v, dst_nb, src_k, src_v, src_nb, desc, pairs, n, stream)
    assert L.pa_swap_blocks(P, P, 0, P, P, 8, D, P, 1, None) == capi.PA_ERR_INVALID
    assert L.pa_swap_blocks(P, P, 8, P, P, 8, D, P, -1, None) == capi.PA_ERR_INVALID
    assert L.pa_swap_blocks(P, P, 8, P, P, 8, D, None, 1, None) == capi.PA_ERR_INVALID
    assert L.pa_swap_blocks(P, P + 8, 8, P, P, 8, D, P, 1, None) == capi.PA_ERR_INVALID
    assert L.pa_swap_blocks(P, P, 8, P, P, 1 << 27, D, P, 1, None) == capi.PA_ERR_OVERFLOW
    assert L.pa_swap_blocks(None, None, 8, None, None, 8, D, None, 0, None) == capi.PA_OK
    row = 8 * 128
    # (out, q, new_k, new_v, k_stride, v_stride, kc, vc, desc, bt, width, ctx, S, max_ctx,
    #  scale, k_scale, v_scale, slots, cfg, ws, ws_bytes, stream)
    app = lambda nk, ks, cfg=None: L.pa_paged_attention_decode_append(  # noqa: E731
        P, P, nk, P, ks, row, P, P, D, P, 4, P, 2, 64, 0.1, 1.0, 1.0, None, cfg, None, 0, None)
    assert app(None, row) == capi.PA_ERR_INVALID
    assert app(P + 4, row) == capi.PA_ERR_INVALID
    assert app(P, row - 8) == capi.PA_ERR_INVALID
    assert app(P, row + 4) == capi.PA_ERR_INVALID
    assert "stride" in _last()
    assert app(P, row, ctypes.byref(capi.DecodeConfig(24, 0, 0, 0, 0))) == capi.PA_ERR_INVALID
    # (..., S, max_ctx, prefix_blocks, scale, ...)
    pre = lambda nk, nv, blocks: L.pa_paged_attention_decode_shared_prefix(  # noqa: E731
        P, P, nk, nv, row, row, P, P, D, P, 4, P, 2, 64, blocks, 0.1, 1.0, 1.0, None, None, None, 0, None)
    assert pre(P, None, 1) == capi.PA_ERR_INVALID
    assert pre(None, None, 5) == capi.PA_ERR_INVALID      # more than the 4-entry table
    assert pre(None, None, 0) == capi.PA_ERR_INVALID
    assert pre(None, None, -2) == capi.PA_ERR_INVALID
    # the size query: a prefix past the context bound, however large, gives 0
    assert L.pa_shared_prefix_workspace_size(D, 2, 64, 5, None) == 0
    assert L.pa_shared_prefix_workspace_size(D, 2, 64, 1 << 28, None) == 0
    assert L.pa_shared_prefix_workspace_size(D, 2, 64, 2, None) > 0


def test_bounds_at_the_int32_limit():
    # ceiling divisions of caller-given bounds are done in 64-bit: a context
    # or query-length bound of 2^31 - 1 gives a valid plan, or a clean
    # refusal before any CUDA call
    L = capi.lib()
    big = 2**31 - 1
    desc = capi.CacheDesc(2048, 16, 32, 128, capi.PA_F16)
    rc, c = _choose(desc, 16, big)
    assert rc == capi.PA_OK, _last()
    assert c.partition_size % 16 == 0 and c.stages % c.warps_per_head == 0
    ws = L.pa_decode_workspace_size(desc, 16, big, None)
    parts = -(-big // c.partition_size)
    assert ws >= 16 * 32 * parts * 128 * 4
    T = 100
    assert L.pa_paged_prefill(P, P, P, P, P, F, P, 4, P, 65535, T, big, 0.1, None) == capi.PA_ERR_INVALID
    assert "too many prefill tiles" in _last()


def _prototypes():
    """name -> (return type, [parameter types]) of every pa_* prototype in the header."""
    with open(HEADER, encoding="utf-8") as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    out = {}
    for ret, name, params in re.findall(r"([A-Za-z_][\w \*]*?)\s*\b(pa_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", text):
        types = []
        for prm in (p.strip() for p in params.split(",")):
            if prm in ("", "void"):
                continue
            types.append(re.sub(r"\s*\b\w+$", "", prm).replace(" *", "*").strip())   # drop the name
        out[name] = (" ".join(ret.split()).replace(" *", "*"), types)
    return out


_CTYPE_OF = {
    "int": ctypes.c_int, "int64_t": ctypes.c_int64, "uint64_t": ctypes.c_uint64, "float": ctypes.c_float,
    "size_t": ctypes.c_size_t,
    "pa_cache_desc": capi.CacheDesc, "const char*": ctypes.c_char_p,
}


def _expected_ctype(ctype: str):
    if ctype in _CTYPE_OF:
        return _CTYPE_OF[ctype]
    if ctype in ("const pa_decode_config*", "pa_decode_config*"):
        return ctypes.POINTER(capi.DecodeConfig)
    if ctype == "uint32_t*":
        return ctypes.POINTER(ctypes.c_uint32)
    assert ctype.endswith("*"), ctype
    return ctypes.c_void_p            # every other pointer crosses as an address


def test_ctypes_signatures_match_the_header():
    protos = _prototypes()
    assert set(protos) == set(capi.SIGNATURES), set(protos) ^ set(capi.SIGNATURES)
    for name, (ret, params) in protos.items():
        res, args = capi.SIGNATURES[name]
        assert res is _expected_ctype(ret), (name, ret, res)
        assert len(args) == len(params), (name, params)
        for i, (ct, a) in enumerate(zip(params, args)):
            want = _expected_ctype(ct)
            assert a is want or (isinstance(a, type) and issubclass(want, ctypes._Pointer)
                                 and a._type_ is want._type_), (name, i, ct, a)


def test_python_constants_match_the_header():
    with open(HEADER, encoding="utf-8") as f:
        defines = dict(re.findall(r"^#define (PA_\w+)\s+\(?(-?\d+)u?\)?", f.read(), flags=re.M))
    assert len(defines) >= 15
    for name, value in defines.items():
        assert getattr(capi, name) == int(value), name


def test_ctypes_structs_match_the_header():
    with open(HEADER, encoding="utf-8") as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    structs = {name: re.findall(r"(\w+)\s+(\w+);", body)
               for body, name in re.findall(r"typedef struct \{(.*?)\} (pa_\w+);", text, flags=re.S)}
    for cname, cls in (("pa_cache_desc", capi.CacheDesc), ("pa_decode_config", capi.DecodeConfig)):
        fields = structs[cname]
        assert [n for _, n in fields] == [n for n, _ in cls._fields_], cname
        assert all(t == "int32_t" for t, _ in fields) and all(ty is ctypes.c_int32 for _, ty in cls._fields_)
        assert ctypes.sizeof(cls) == 4 * len(fields)


def _partials_bytes(S, H, D, parts):
    lse = (S * H * parts * 4 + 255) // 256 * 256
    return lse + S * H * parts * D * 4


def test_shared_prefix_suffix_shape_counts_the_prefix_kernel():
    # 32 sequences x 32 heads, head_size 128, 32-token blocks, a 96-block
    # (3072-token) shared prefix under a 4096-token bound: the prefix kernel
    # runs 32 heads x 12 partitions of 256 tokens = 384 CTAs beside the
    # decode of the private parts. Counting them, the private parts' grid
    # (2 heads per CTA: 512 units with 1024-token partitions) plus the prefix
    # grid reaches 4 CTAs per SM, so the suffix takes one 1024-token partition:
    # 12 + 1 partials per (sequence, head). Without the prefix kernel's CTAs the
    # rule would have split the suffix in two (12 + 2).
    L = capi.lib()
    desc = capi.CacheDesc(4096, 32, 32, 128, capi.PA_F16)
    got = L.pa_shared_prefix_workspace_size(desc, 32, 4096, 96, None)
    assert got == _partials_bytes(32, 32, 128, 12 + 1)
    # an explicit 512-token suffix partition gives the two-partition layout
    cfg = capi.DecodeConfig(512, 0, 0, 0, 0)
    assert L.pa_shared_prefix_workspace_size(desc, 32, 4096, 96, ctypes.byref(cfg)) == \
        _partials_bytes(32, 32, 128, 12 + 2)
    # a small batch (8 sequences) stays at two heads per CTA and 512-token partitions:
    # 8 x 16 x 2 = 256 units + 384 prefix CTAs are below 4 per SM at 1024 tokens
    assert L.pa_shared_prefix_workspace_size(desc, 8, 4096, 96, None) == _partials_bytes(8, 32, 128, 12 + 2)
