"""Multi-rank host logic on CPU (gloo, world size 2).

The path shards by sequence: every rank decodes its own, independently
seeded batch and no data crosses ranks. These tests run the ranks' host
side -- their workloads, their oracle decode step, the max-over-ranks timing
reduction and the aggregate value -- as two gloo processes."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.named(1, seed=W.rank_seed(1001, rank))
        kc, vc = w.pool_host()
        slots = oracle.slot_mapping(w.block_tables, w.context_lens, w.block_size)
        oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots)
        out = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale)
        # each rank's own time; rank 1 is "slower"
        mine = [1.0 + rank, 0.5 + 2 * rank, 3.0 - rank]
        slow = bench.slowest_rank(mine, dist, torch.device("cpu"))
        q.put((rank, float(out.sum()), w.query.tobytes()[:64], slow, w.kv_bytes()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_independent_batches_and_slowest_rank_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, q0, slow0, kv0), (r1, s1, q1, slow1, kv1) = res
    assert q0 != q1 and s0 != s1                     # independent seeded batches
    assert slow0 == slow1 == [2.0, 2.5, 3.0]        # elementwise max over ranks, same on every rank
    v = bench.aggregate_gbs(2, kv0, 2.0)
    assert v == pytest.approx(2 * kv0 / 2e-3 / 1e9)


def test_rank_seeds_keep_the_shape_of_the_workload():
    a = W.named(2, seed=W.rank_seed(1002, 0))
    b = W.named(2, seed=W.rank_seed(1002, 1))
    assert a.query.shape == b.query.shape and a.num_blocks == b.num_blocks
    assert not np.array_equal(a.context_lens, b.context_lens)
