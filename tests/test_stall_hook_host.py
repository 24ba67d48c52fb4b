"""Host-side checks of the wait test hook (no GPU needed: nothing launches)."""
import pytest

import pagedattention_paged_kv_decode_b200 as pk
from pagedattention_paged_kv_decode_b200 import capi


@pytest.mark.parametrize("limit", [0, 999, 2_000_000_001])
def test_limits_outside_the_range_are_refused(limit):
    assert capi.lib().pa_test_stall_next_decode(0, 0, 0, limit) == capi.PA_ERR_INVALID
    assert b"wait_limit_ns" in capi.lib().pa_last_error()
    with pytest.raises(ValueError):
        pk.test_stall_next_decode(0, 0, 0, limit)


@pytest.mark.parametrize("head,part", [(-1, 0), (0, -1)])
def test_negative_head_or_partition_is_refused(head, part):
    assert capi.lib().pa_test_stall_next_decode(0, head, part, 1_000_000) == capi.PA_ERR_INVALID
    with pytest.raises(ValueError):
        pk.test_stall_next_decode(0, head, part, 1_000_000)


@pytest.mark.parametrize("limit", [1000, 2_000_000_000])
def test_limits_at_the_bounds_are_accepted_and_cleared(limit):
    assert capi.lib().pa_test_stall_next_decode(3, 1, 2, limit) == capi.PA_OK
    assert capi.lib().pa_test_stall_next_decode(-1, 0, 0, 0) == capi.PA_OK
