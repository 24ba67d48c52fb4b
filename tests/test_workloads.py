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
