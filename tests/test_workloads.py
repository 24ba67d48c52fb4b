"""The seeded input generator follows its stated recipe.

Shapes, context laws, pool sizes and table widths of the workloads that
build in seconds (decode configs 1 and 2, prefill workloads 1 and 3) are
checked against the recipe, together with the structure every workload
must have: physical blocks dealt without repeats inside the pool, -1 in
the table beyond each sequence's blocks, and poison in every pool slot
that holds no context token yet (the appended token's slot included).
"""
import numpy as np
import pytest

import workloads as W

HUGE = np.float16(60000)


def _check_tables(w, ctx):
    dealt = []
    for s, L in enumerate(ctx):
        n = -(-int(L) // w.block_size)
        row = w.block_tables[s]
        assert (row[:n] >= 0).all() and (row[:n] < w.num_blocks).all()
        assert (row[n:] == -1).all()
        dealt += [int(b) for b in row[:n]]
    assert len(dealt) == len(set(dealt))          # no physical block serves two sequences


def _check_poison(w, present):
    """`present[s]`: context tokens of sequence s in the pool before the step."""
    kc, _ = w.pool_host()
    live = np.zeros(kc.shape[:2], bool)
    for s, n in enumerate(present):
        for t in range(int(n)):
            live[w.block_tables[s][t // w.block_size], t % w.block_size] = True
    dead = kc[~live]
    assert np.all(np.abs(dead) == HUGE)
    assert not np.any(np.abs(kc[live]) == HUGE)


@pytest.mark.parametrize("cid,S,H,D,B,lo,hi,pool,width", [
    (1, 4, 4, 64, 16, 1, 64, 32, 4),
    (2, 16, 32, 128, 16, 50, 178, 2048, 12),
])
def test_decode_workload_recipe(cid, S, H, D, B, lo, hi, pool, width):
    w = W.named(cid)
    assert w.name == W.NAMES[cid]
    assert (w.num_seqs, w.num_heads, w.head_size, w.block_size) == (S, H, D, B)
    assert w.query.shape == w.new_key.shape == w.new_value.shape == (S, H, D)
    assert w.num_blocks == pool and w.block_tables.shape == (S, width)
    assert lo <= w.context_lens.min() and w.context_lens.max() <= hi
    assert np.float32(w.scale) == np.float32(1.0 / np.sqrt(D))
    _check_tables(w, w.context_lens)
    _check_poison(w, w.context_lens - 1)          # position L-1 waits for the step's write
    # same seed, same workload; another seed, another batch of the same shape
    again = W.named(cid)
    assert np.array_equal(again.context_lens, w.context_lens)
    assert np.array_equal(again.query.view(np.uint16), w.query.view(np.uint16))
    other = W.named(cid, seed=W.rank_seed(1000 + cid, 1))
    assert other.query.shape == w.query.shape


def test_prefill_workload_recipes():
    w = W.prefill_named(1)
    assert list(w.context_lens) == [37, 300, 129, 1] and list(w.chunk_lens) == [37, 100, 1, 1]
    assert (w.num_heads, w.head_size, w.block_size) == (4, 128, 32)
    _check_tables(w, w.context_lens)
    _check_poison(w, w.context_lens - w.chunk_lens)  # the chunk's own positions wait for its write
    w = W.prefill_named(3)
    assert (w.num_seqs, w.num_heads, w.head_size, w.block_size) == (8, 32, 128, 16)
    assert (w.chunk_lens == 512).all()
    assert 512 <= w.context_lens.min() and w.context_lens.max() <= 512 + 2048
    assert w.total_q == 8 * 512 and w.query.shape == (w.total_q, 32, 128)
    assert list(w.query_start) == list(range(0, 8 * 512 + 1, 512))
    _check_tables(w, w.context_lens)


def test_default_seeds():
    assert np.array_equal(W.named(1).query.view(np.uint16), W.named(1, seed=1001).query.view(np.uint16))
    a, b = W.prefill_named(1), W.prefill_named(1, seed=2001)
    assert np.array_equal(a.query.view(np.uint16), b.query.view(np.uint16))


def test_shared_prefix_workload_with_copy_on_write():
    # 32 sequences share a 3072-token prompt (96 blocks of 32); the step
    # copies the last shared block into one spare block per sequence and the
    # decode tables point logical block 95 at that copy
    w = W.named(4)
    S, B = 32, 32
    assert (w.num_seqs, w.block_size, w.block_tables.shape) == (S, B, (S, 128))
    assert 3073 <= w.context_lens.min() and w.context_lens.max() <= 3072 + 1024
    private = sum(-(-(int(L) - 3072) // B) for L in w.context_lens)
    assert w.num_blocks == 96 + private + S
    shared = w.block_tables_shared
    assert (shared[:, :96] == shared[0, :96]).all()                  # one physical prefix for all
    assert (w.block_tables[:, :95] == shared[:, :95]).all()
    spare = w.block_tables[:, 95]
    assert len(set(spare.tolist())) == S and not set(spare.tolist()) & set(shared[0, :96].tolist())
    assert (w.cow_pairs[:, 0] == shared[0, 95]).all() and (w.cow_pairs[:, 1] == spare).all()
    assert w.shared_blocks == 95
    # every block of the pool is used once: the prefix, the spares and the private suffixes
    used = list(shared[0, :96]) + list(spare) + [int(b) for s in range(S) for b in w.block_tables[s, 96:] if b >= 0]
    assert sorted(used) == list(range(w.num_blocks))


def test_e4m3_scales_cover_every_value_the_cache_holds():
    w = W.build("e", 2, 64, 16, "e4m3", [5, 40, 17], 12, 3, 9, 1.0, 1.0)
    for scale, live, new in ((w.k_scale, w.live_key, w.new_key), (w.v_scale, w.live_value, w.new_value)):
        amax = max(np.abs(live.astype(np.float32)).max(), np.abs(new.astype(np.float32)).max())
        assert np.float32(scale) == np.float32(amax) / np.float32(448.0)
    f = W.build("f", 2, 64, 16, "f16", [5, 40, 17], 12, 3, 9, 1.0, 1.0)
    assert f.k_scale == f.v_scale == 1.0


def test_fused_step_bytes_count_the_tensors_of_the_step():
    for kv, elem in (("f16", 2), ("e4m3", 1)):
        w = W.build("b", 2, 64, 16, kv, [5, 40, 17], 12, 3, 9, 1.0, 1.0)
        extra = (w.new_key.nbytes + w.new_value.nbytes            # new rows read (fp16)
                 + w.new_key.size * elem + w.new_value.size * elem  # and stored in the cache format
                 + 4 * w.num_seqs)                                  # slots written
        assert W.fused_step_bytes(w) == w.decode_bytes() + extra


def test_shared_block_count_edges():
    # the shared-prefix path is offered only when two or more sequences all
    # reach past the shared blocks
    def shared(ctx, cow=False):
        return W.build("s", 1, 64, 16, "f16", ctx, 16, 4, 3, 1.0, 1.0, shared_prefix=32, cow=cow).shared_blocks
    assert shared([40]) == 0                         # one sequence: nothing to share
    assert shared([32, 40]) == 2                      # the shortest sequence ends exactly at the prefix
    assert shared([32, 40], cow=True) == 1            # the copied block is no longer shared
    assert shared([20, 40]) == 2
    assert shared([10, 40]) == 0                      # one sequence ends inside the prefix


def test_prefill_positions_flops_and_bytes():
    w = W.prefill_named(1)                            # contexts 37, 300, 129, 1; chunks 37, 100, 1, 1
    want = np.concatenate([np.arange(0, 37), np.arange(200, 300), [128], [0]])
    assert np.array_equal(w.positions(), want)
    # (row, token) pairs the causal mask admits, counted one by one
    pairs = sum(int(p) + 1 for p in want)
    assert w.flops() == 4 * w.num_heads * w.head_size * pairs
    # every context token's K and V once (those already in the pool and the chunk's own), Q and the output
    kv = w.live_key.nbytes + w.live_value.nbytes + w.new_key.nbytes + w.new_value.nbytes
    assert w.io_bytes() == kv + 2 * w.query.nbytes
