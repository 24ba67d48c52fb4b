"""A bounded on-chip wait that runs out, on the GPU, without a fault.

Every mbarrier wait of the decode kernel has a wall-time limit. Here the
test hook pa_test_stall_next_decode makes the next decode's producer issue
no tile loads for the work unit holding one (sequence, head, partition) and
shortens the limit to 1 ms: that unit's consumer warps must give up, set
PA_DEV_WAIT_TIMEOUT in the device error word and return. The call must end well inside a second (not the default
2 s limit, and never hang), and the very next decode on the same device
must match the oracle with a clean error word.
"""
import time

import numpy as np
import pytest

import pagedattention_paged_kv_decode_b200 as pk
from pagedattention_paged_kv_decode_b200 import capi
import workloads as W
from _oracle_step import oracle_step

pytestmark = pytest.mark.gpu

LAUNCHES = [None,
            dict(partition_size=64, heads_per_cta=2, warps_per_head=2, stages=4),
            dict(partition_size=32, heads_per_cta=1, warps_per_head=1, stages=2, units_per_cta=3)]


def _case(kv, seed):
    ctx = [200, 1, 17, 96, 0, 300]
    B, H, D = 16, 4, 128
    need = sum(-(-L // B) for L in ctx)
    return W.build(f"stall_{kv}", H, D, B, kv, ctx, need + 5, -(-max(ctx) // B), seed,
                   q_std=1.0, kv_std=1.0)


@pytest.mark.parametrize("launch", LAUNCHES, ids=["default", "p64_g2_w2", "p32_c3"])
@pytest.mark.parametrize("kv", ["f16", "e4m3"])
def test_stalled_unit_times_out_and_the_next_decode_is_clean(cuda_device, kv, launch):
    w = _case(kv, seed=31)
    dw = W.to_device(w, cuda_device, encode=pk.load_cache)
    bound = w.max_blocks_per_seq * w.block_size

    def step():
        pk.paged_attention_decode_append(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache,
                                         dw.value_cache, dw.block_tables, dw.context_lens, w.scale,
                                         w.k_scale, w.v_scale, max_context_len=bound,
                                         slot_mapping=dw.slots, config=launch)

    step()  # loads the kernels and sizes the workspace outside the timed calls
    assert pk.check_status() == 0
    # sequence 0 (200 tokens): its first partition, and a later one of another head
    for seq, head, part in ((0, 0, 0), (0, 1, 2)):
        pk.test_stall_next_decode(seq, head, part, 1_000_000)
        t0 = time.perf_counter()
        step()
        code = pk.check_status()
        elapsed = time.perf_counter() - t0
        assert code == capi.PA_DEV_WAIT_TIMEOUT, code
        assert elapsed < 1.0, elapsed
    # the request was consumed: the next step runs normally and matches the oracle
    step()
    assert pk.check_status() == 0
    slots, kc, vc, out_ref, _ = oracle_step(w)
    assert np.array_equal(dw.slots.cpu().numpy(), slots)
    got = dw.out.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    assert np.abs(got - out_ref).max() <= (2e-3 if kv == "f16" else 1e-2)


@pytest.mark.parametrize("request_", ["cleared", "empty unit", "outside the launch"])
def test_requests_that_stall_nothing(cuda_device, request_):
    w = _case("f16", seed=32)
    dw = W.to_device(w, cuda_device)
    if request_ == "cleared":
        pk.test_stall_next_decode(0, 0, 0, 1_000_000)
        pk.test_stall_next_decode(-1)
    elif request_ == "empty unit":
        pk.test_stall_next_decode(4, 0, 0, 1_000_000)      # sequence 4 has no tokens
    else:
        pk.test_stall_next_decode(0, 0, 1000, 1_000_000)   # no such partition
    pk.decode_step(dw.out, dw.query, dw.new_key, dw.new_value, dw.key_cache, dw.value_cache,
                   dw.block_tables, dw.context_lens, w.scale, slots=dw.slots,
                   max_context_len=w.max_context_len)
    assert pk.check_status() == 0
    _, _, _, out_ref, _ = oracle_step(w)
    assert np.abs(dw.out.cpu().numpy().astype(np.float64) - out_ref).max() <= 2e-3
