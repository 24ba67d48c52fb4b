"""Oracle-side expectations for one decode step of a workload (test helper).

Runs the oracle's own slot mapping, block copy, cache write and attention on
host copies of a workload's inputs. E4M3 pools are encoded by the oracle's
own cache write. The oracle's threaded calls (OpenMP over token rows and over
(sequence, head) pairs; identical results to its single-thread calls) keep
the full-size workloads to seconds."""
from __future__ import annotations

import numpy as np

import oracle
import workloads as W


def needed_blocks(w: W.Workload, seqs) -> np.ndarray:
    bt = w.block_tables[list(seqs)]
    blocks = [bt[bt >= 0].ravel()]
    if w.cow_pairs.size:
        blocks.append(w.cow_pairs.ravel())
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, w.block_size)
    blocks.append(slots[slots >= 0] // w.block_size)
    return np.unique(np.concatenate(blocks)).astype(np.int64)


def oracle_pools(w: W.Workload, blocks: np.ndarray | None):
    """Host caches before the step: fp16 pools, or E4M3 codes of `blocks`
    (every block of the pool when blocks is None)."""
    pk, pv = w.pool_host()
    if w.kv_dtype == "f16":
        return pk, pv
    kc = np.zeros(pk.shape, np.uint8)
    vc = np.zeros(pv.shape, np.uint8)
    B, H, D = w.block_size, w.num_heads, w.head_size
    if blocks is None:
        slots = np.arange(w.num_blocks * B, dtype=np.int32)
        oracle.kv_cache_write(pk.reshape(-1, H, D), pv.reshape(-1, H, D), kc, vc, slots,
                              w.k_scale, w.v_scale, threads=0)
        return kc, vc
    slots = (blocks[:, None] * B + np.arange(B)[None, :]).reshape(-1).astype(np.int32)
    oracle.kv_cache_write(pk[blocks].reshape(-1, H, D), pv[blocks].reshape(-1, H, D), kc, vc,
                          slots, w.k_scale, w.v_scale, threads=0)
    return kc, vc


def oracle_step(w: W.Workload, seqs=None, whole_pool: bool = False):
    """Returns (slots, key_cache, value_cache, out[len(seqs), H, D], blocks
    checked). With whole_pool, an E4M3 pool is encoded in full (so that the
    whole pool can be compared) and `blocks` lists every block."""
    seqs = list(range(w.num_seqs)) if seqs is None else list(seqs)
    blocks = np.arange(w.num_blocks) if whole_pool else needed_blocks(w, seqs)
    kc, vc = oracle_pools(w, None if whole_pool else (blocks if w.kv_dtype == "e4m3" else None))
    if w.cow_pairs.size:
        oracle.copy_blocks(kc, vc, w.cow_pairs)
    slots = oracle.slot_mapping(w.block_tables, w.context_lens, w.block_size)
    oracle.kv_cache_write(w.new_key, w.new_value, kc, vc, slots, w.k_scale, w.v_scale)
    pairs = np.array([(s, h) for s in seqs for h in range(w.num_heads)], np.int32)
    out = oracle.paged_attention(w.query, kc, vc, w.block_tables, w.context_lens, w.scale,
                                 w.k_scale, w.v_scale, seq_head=pairs, threads=0)
    return slots, kc, vc, out.reshape(len(seqs), w.num_heads, w.head_size), blocks


def sample_seqs(w: W.Workload, n: int, seed: int = 0):
    """Longest and shortest sequences plus a seeded random sample."""
    if w.num_seqs <= n:
        return list(range(w.num_seqs))
    order = np.argsort(w.context_lens, kind="stable")
    pick = {int(order[0]), int(order[-1])}
    rng = np.random.default_rng(seed)
    for s in rng.permutation(w.num_seqs):
        if len(pick) >= n:
            break
        pick.add(int(s))
    return sorted(pick)
