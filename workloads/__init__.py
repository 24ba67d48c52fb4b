"""Seeded synthetic inputs for the paged-KV decode path and the paged prefill.

This module is shared by the tests, the benchmark and the smoke check, and it
holds none of the method's arithmetic: it draws context lengths, deals
physical blocks to sequences from a seeded permutation, draws fp16 query and
K/V values, fills every pool slot that holds no context token with poison,
and (for fp8 caches) derives per-tensor scales from the drawn data. It never
computes a slot, an encoding, an attention output or a block copy.

Layout of the pools it returns: ``[num_blocks, block_size, num_heads,
head_size]`` fp16. For E4M3 workloads the fp16 pool is the *source* that each
side (the CUDA library and the CPU oracle) encodes with its own cache-write
step, with the identity slot list ``0 .. num_blocks*block_size - 1``.

Context tokens 0 .. L-2 of each sequence are present in the pool before the
step; position L-1 (the token the decode step appends) holds poison until the
step's cache write stores ``new_key``/``new_value`` there.

The five named decode workloads follow the shapes and value laws of the
pages' serving setups (LLaMA-7B: 32 heads x 128; Llama2-13B: 40 heads x 128;
16-token blocks, 32-token blocks for long shared prompts, FP8 KV cache). The
three named prefill workloads (``prefill_named``) bring a chunk of new tokens
per sequence: whole prompts, or chunks after tokens already in the pool,
whose own positions hold poison until the chunk's cache write. No public
dataset is involved; every input is drawn from ``numpy.random.PCG64``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

POISON_HUGE = "huge"   # +/-60000 in an alternating pattern (finite, dominates any softmax it leaks into)
POISON_NAN = "nan"     # fp16 NaN: any arithmetic use of an unused slot shows up as NaN


class _Pools:
    """Pool construction shared by the decode and prefill workloads (needs
    num_blocks, block_size, num_heads, head_size, poison, live_*)."""

    def pool_host(self) -> tuple[np.ndarray, np.ndarray]:
        """The fp16 pools [NB, B, H, D] before the step (E4M3: the source to encode)."""
        shape = (self.num_blocks, self.block_size, self.num_heads, self.head_size)
        pk = _poison_fill(shape, self.poison)
        pv = _poison_fill(shape, self.poison)
        pk[self.live_blocks, self.live_offsets] = self.live_key
        pv[self.live_blocks, self.live_offsets] = self.live_value
        return pk, pv

    def pool_device(self, device) -> tuple:
        """The same pools as torch fp16 tensors on ``device`` (filled there)."""
        import torch
        shape = (self.num_blocks, self.block_size, self.num_heads, self.head_size)
        out = []
        for live in (self.live_key, self.live_value):
            pool = torch.empty(shape, dtype=torch.float16, device=device)
            if self.poison == POISON_NAN:
                pool.fill_(float("nan"))
            else:
                pool.view(torch.int32).fill_(_HUGE_PAIR_I32)
            blk = torch.from_numpy(self.live_blocks.astype(np.int64)).to(device)
            off = torch.from_numpy(self.live_offsets.astype(np.int64)).to(device)
            pool[blk, off] = torch.from_numpy(live).to(device)
            out.append(pool)
        return out[0], out[1]


@dataclass
class Workload(_Pools):
    name: str
    num_seqs: int
    num_heads: int
    head_size: int
    block_size: int
    num_blocks: int
    kv_dtype: str                  # "f16" or "e4m3"
    scale: float                   # softmax scale (fp32 value)
    k_scale: float                 # per-tensor K scale (1.0 for fp16 caches)
    v_scale: float
    query: np.ndarray              # float16 [S, H, D]
    new_key: np.ndarray            # float16 [S, H, D], the token appended at position L-1
    new_value: np.ndarray
    block_tables: np.ndarray       # int32 [S, W], -1 beyond each sequence's blocks (post copy-on-write)
    context_lens: np.ndarray       # int32 [S], including the appended token
    live_blocks: np.ndarray        # int32 [n]: physical block of each context token present before the step
    live_offsets: np.ndarray       # int32 [n]: its row inside that block
    live_key: np.ndarray           # float16 [n, H, D]
    live_value: np.ndarray
    poison: str = POISON_HUGE
    cow_pairs: np.ndarray = field(default_factory=lambda: np.zeros((0, 2), np.int32))
    block_tables_shared: np.ndarray | None = None   # tables before the copy-on-write repoint
    shared_blocks: int = 0         # leading table entries identical in every row of block_tables
    seed: int = 0

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max(initial=0))

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def elem_bytes(self) -> int:
        return 2 if self.kv_dtype == "f16" else 1

    def kv_bytes(self) -> int:
        """Logical K+V bytes the decode reads: sum_s L_s * H * D * elem * 2."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_heads * self.head_size * self.elem_bytes * 2

    def unique_kv_bytes(self) -> int:
        """K+V bytes of distinct cache rows the decode reads: the leading
        shared_blocks blocks, which every table row points at, count once."""
        shared = self.shared_blocks * self.block_size
        L = self.context_lens.astype(np.int64)
        tokens = int(np.maximum(L - shared, 0).sum()) + (shared if (L > 0).any() else 0)
        return tokens * self.num_heads * self.head_size * self.elem_bytes * 2

    def decode_bytes(self) -> int:
        """Algorithmic bytes of one decode: K/V + query + output + block-table entries + lengths."""
        S, H, D, B = self.num_seqs, self.num_heads, self.head_size, self.block_size
        tables = 4 * int(sum(-(-int(L) // B) for L in self.context_lens))
        return self.kv_bytes() + 2 * S * H * D * 2 + tables + 4 * S


_HUGE_PAIR = np.array([60000.0, -60000.0], np.float16)
_HUGE_PAIR_I32 = int(_HUGE_PAIR.view(np.int32)[0])


def fused_step_bytes(w: "Workload") -> int:
    """Algorithmic bytes of one fused append+decode launch: the decode's bytes
    plus the new K/V rows read (fp16) and stored (cache dtype) and the slots."""
    S, H, D = w.num_seqs, w.num_heads, w.head_size
    return w.decode_bytes() + S * H * D * 2 * 2 + S * H * D * w.elem_bytes * 2 + 4 * S


def _poison_fill(shape, poison: str) -> np.ndarray:
    if poison == POISON_NAN:
        return np.full(shape, np.nan, np.float16)
    out = np.empty(shape, np.float16)
    out.view(np.int32).fill(_HUGE_PAIR_I32)     # head_size is even: pairs (+60000, -60000)
    return out


_QUANTILES: dict = {}


def _normal_table() -> np.ndarray:
    """Quantiles of N(0, 1) at the 65536 midpoints (i + 0.5) / 65536, as float32."""
    if "t" not in _QUANTILES:
        from scipy.special import ndtri
        _QUANTILES["t"] = ndtri((np.arange(65536, dtype=np.float64) + 0.5) / 65536.0).astype(np.float32)
    return _QUANTILES["t"]


def _draw_f16(rng: np.random.Generator, shape, std: float, chunk: int = 1 << 22) -> np.ndarray:
    """float16 samples of N(0, std^2) by inverse-CDF sampling at 16-bit resolution.

    Each value is the N(0,1) quantile at a uniformly drawn 16-bit level, times
    std, rounded to fp16 (tails are cut at |z| ~= 4.17). This is much faster
    than Gaussian sampling for the multi-GB pools of the larger workloads.
    """
    table = (_normal_table() * np.float32(std)).astype(np.float16).view(np.uint16)
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        levels = rng.integers(0, 65536, m, dtype=np.uint16).astype(np.intp)
        np.take(table, levels, out=out[i:i + m])
    return out.view(np.float16).reshape(shape)


def _amax_f16(*arrays: np.ndarray) -> float:
    """Largest |x| over fp16 arrays holding no NaN (sign bit cleared, compared as bits)."""
    best = 0
    for a in arrays:
        if a.size:
            best = max(best, int((a.view(np.uint16) & np.uint16(0x7FFF)).max()))
    return float(np.array([best], np.uint16).view(np.float16)[0])


def build(name: str, num_heads: int, head_size: int, block_size: int, kv_dtype: str,
          context_lens, num_blocks: int, table_width: int, seed: int,
          q_std: float, kv_std: float, poison: str = POISON_HUGE,
          shared_prefix: int = 0, cow: bool = False, rng: np.random.Generator | None = None,
          deal_order: str = "permuted") -> Workload:
    """Assemble a workload from explicit context lengths.

    Blocks are dealt to sequences from ``rng.permutation(num_blocks)``
    (``deal_order="identity"`` deals 0, 1, 2, ... instead, which makes every
    sequence's blocks contiguous and in order). With ``shared_prefix`` > 0 the
    first ``shared_prefix // block_size`` blocks of every table are the same
    physical blocks; with ``cow`` each sequence also gets a spare block, and
    the returned decode tables point the last shared logical block at that
    spare block, with ``cow_pairs`` = (shared block, spare block) per sequence.
    """
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    ctx = np.asarray(context_lens, dtype=np.int32)
    S, H, D, B = len(ctx), num_heads, head_size, block_size
    assert shared_prefix % B == 0
    n_shared = shared_prefix // B
    need = [-(-int(L) // B) for L in ctx]
    private = [max(0, n - n_shared) for n in need]
    total = n_shared + sum(private) + (S if cow else 0)
    assert total <= num_blocks, f"pool of {num_blocks} blocks is too small for {total}"
    assert max(need, default=0) <= table_width
    order = rng.permutation(num_blocks).astype(np.int32) if deal_order == "permuted" \
        else np.arange(num_blocks, dtype=np.int32)

    tables = np.full((S, table_width), -1, np.int32)
    shared_ids = order[:n_shared]
    cursor = n_shared
    for s in range(S):
        tables[s, :min(n_shared, need[s])] = shared_ids[:min(n_shared, need[s])]
        tables[s, n_shared:n_shared + private[s]] = order[cursor:cursor + private[s]]
        cursor += private[s]
    spare = order[cursor:cursor + S] if cow else None

    # Context tokens present before the step: shared prefix once, then each
    # sequence's private tokens (positions max(prefix, 0) .. L-2).
    blk_list, off_list = [], []
    if n_shared:
        pos = np.arange(shared_prefix)
        blk_list.append(shared_ids[pos // B])
        off_list.append(pos % B)
    for s in range(S):
        pos = np.arange(shared_prefix if n_shared else 0, int(ctx[s]) - 1)
        if pos.size:
            blk_list.append(tables[s, pos // B])
            off_list.append(pos % B)
    blk = np.concatenate(blk_list) if blk_list else np.zeros(0, np.int32)
    off = np.concatenate(off_list) if off_list else np.zeros(0, np.int32)

    query = _draw_f16(rng, (S, H, D), q_std)
    new_key = _draw_f16(rng, (S, H, D), kv_std)
    new_value = _draw_f16(rng, (S, H, D), kv_std)
    live_k = _draw_f16(rng, (blk.size, H, D), kv_std)
    live_v = _draw_f16(rng, (blk.size, H, D), kv_std)

    scale = float(np.float32(1.0) / np.sqrt(np.float32(D)))
    k_scale = v_scale = 1.0
    if kv_dtype == "e4m3":
        # per-tensor scales: amax over all K (V) values the cache will hold, / 448
        amax_k = _amax_f16(live_k, new_key)
        amax_v = _amax_f16(live_v, new_value)
        k_scale = float(np.float32(amax_k) / np.float32(448.0))
        v_scale = float(np.float32(amax_v) / np.float32(448.0))
    else:
        assert kv_dtype == "f16"

    cow_pairs = np.zeros((0, 2), np.int32)
    shared_tables = None
    if cow:
        last = n_shared - 1
        cow_pairs = np.stack([np.full(S, shared_ids[last], np.int32), spare.astype(np.int32)], axis=1)
        shared_tables = tables.copy()
        tables[:, last] = spare

    return Workload(name=name, num_seqs=S, num_heads=H, head_size=D, block_size=B,
                    num_blocks=num_blocks, kv_dtype=kv_dtype, scale=scale,
                    k_scale=k_scale, v_scale=v_scale, query=query, new_key=new_key,
                    new_value=new_value, block_tables=tables, context_lens=ctx,
                    live_blocks=blk.astype(np.int32), live_offsets=off.astype(np.int32),
                    live_key=live_k, live_value=live_v, poison=poison, cow_pairs=cow_pairs,
                    block_tables_shared=shared_tables,
                    shared_blocks=(n_shared - 1 if cow else n_shared) if (S > 1 and min(need, default=0) >= n_shared) else 0,
                    seed=seed)


# --------------------------------------------------------- named workloads

NAMES = {
    1: "tiny_s4_h4_d64_b16_f16",
    2: "llama7b_decode_s16_h32_d128_b16_f16",
    3: "llama13b_mixed_s64_h40_d128_b16_f16",
    4: "shared_prefix_cow_s32_h32_d128_b32_f16",
    5: "fp8_kv_s256_h32_d128_b16_e4m3",
}


def named(config_id: int, seed: int | None = None, poison: str = POISON_HUGE,
          num_seqs: int | None = None) -> Workload:
    """The five workloads (seed defaults to 1000 + config_id). num_seqs gives
    a smaller (or larger) batch drawn by the same recipe -- the same length
    law, head count, head size, block size and pool rule -- for profiler
    captures that must stay small; its name carries its own batch size."""
    seed = 1000 + config_id if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    name = NAMES[config_id]
    S0 = {1: 4, 2: 16, 3: 64, 4: 32, 5: 256}[config_id]
    S = S0 if num_seqs is None else int(num_seqs)
    if S != S0:
        if config_id == 3 and S % 2:
            raise ValueError("the mixed-length batch needs an even number of sequences")
        name = name.replace(f"_s{S0}_", f"_s{S}_")
    if config_id == 1:
        ctx = rng.integers(1, 65, S)
        return build(name, 4, 64, 16, "f16", ctx, 32 * S // 4, 4, seed, 1.0, 1.0, poison, rng=rng)
    if config_id == 2:
        ctx = 50 + rng.integers(0, 129, S)
        return build(name, 32, 128, 16, "f16", ctx, 2048 * S // 16, 12, seed, 0.5, 0.5, poison, rng=rng)
    if config_id == 3:
        ctx = np.concatenate([rng.integers(64, 129, S // 2), rng.integers(1024, 2049, S // 2)])
        ctx = ctx[rng.permutation(S)]
        return build(name, 40, 128, 16, "f16", ctx, 16384 * S // 64, 128, seed, 0.5, 0.5, poison, rng=rng)
    if config_id == 4:
        ctx = 3072 + rng.integers(1, 1025, S)
        private = sum(-(-(int(L) - 3072) // 32) for L in ctx)
        nb = 96 + private + S
        return build(name, 32, 128, 32, "f16", ctx, nb, 128, seed, 0.5, 0.5, poison,
                     shared_prefix=3072, cow=True, rng=rng)
    if config_id == 5:
        ctx = np.floor(np.exp(rng.uniform(math.log(16), math.log(4096), S))).astype(np.int64)
        nb = int(math.ceil(1.1 * sum(-(-int(L) // 16) for L in ctx)))
        return build(name, 32, 128, 16, "e4m3", ctx, nb, 256, seed, 1.0, 1.0, poison, rng=rng)
    raise KeyError(config_id)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s independent batch in a multi-GPU run."""
    return seed + 7919 * rank


@dataclass
class DeviceWorkload:
    """A workload's tensors on a CUDA device (torch), ready for one decode step."""
    w: Workload
    query: object
    new_key: object
    new_value: object
    block_tables: object
    context_lens: object
    cow_pairs: object
    key_cache: object
    value_cache: object
    out: object
    slots: object


def to_device(w: Workload, device, encode=None) -> DeviceWorkload:
    """Upload a workload. fp16 caches are the pools as drawn; E4M3 caches are
    produced by ``encode(key_cache, value_cache, key_src, value_src, k_scale,
    v_scale)``, which the caller supplies (the library's bulk cache write)."""
    import torch

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    pk, pv = w.pool_device(device)
    if w.kv_dtype == "e4m3":
        if encode is None:
            raise ValueError("E4M3 workloads need an encode callable")
        kc = torch.empty(pk.shape, dtype=torch.uint8, device=device)
        vc = torch.empty(pv.shape, dtype=torch.uint8, device=device)
        encode(kc, vc, pk, pv, w.k_scale, w.v_scale)
        del pk, pv
        torch.cuda.synchronize(device)
        torch.cuda.empty_cache()    # release the fp16 source pools
    else:
        kc, vc = pk, pv
    S, H, D = w.query.shape
    return DeviceWorkload(
        w=w, query=up(w.query), new_key=up(w.new_key), new_value=up(w.new_value),
        block_tables=up(w.block_tables), context_lens=up(w.context_lens),
        cow_pairs=up(w.cow_pairs.astype(np.int32)), key_cache=kc, value_cache=vc,
        out=torch.empty((S, H, D), dtype=torch.float16, device=device),
        slots=torch.empty(S, dtype=torch.int32, device=device))


# ------------------------------------------------------------ paged prefill

@dataclass
class PrefillWorkload(_Pools):
    """One prefill step: sequence s brings n_s new tokens (the last n_s
    positions of its L_s-token context); tokens 0 .. L_s - n_s - 1 are already
    in the pool, the chunk's own positions hold poison until its cache write."""
    name: str
    num_seqs: int
    num_heads: int
    head_size: int
    block_size: int
    num_blocks: int
    scale: float
    query: np.ndarray              # float16 [total_q, H, D], rows of sequence s at query_start[s] ..
    new_key: np.ndarray            # float16 [total_q, H, D], the chunk's K rows (same order)
    new_value: np.ndarray
    query_start: np.ndarray        # int32 [S + 1], query_start[0] = 0
    block_tables: np.ndarray       # int32 [S, W], -1 beyond each sequence's blocks
    context_lens: np.ndarray       # int32 [S], L_s including the chunk
    live_blocks: np.ndarray
    live_offsets: np.ndarray
    live_key: np.ndarray
    live_value: np.ndarray
    poison: str = POISON_HUGE
    seed: int = 0
    kv_dtype: str = "f16"
    k_scale: float = 1.0
    v_scale: float = 1.0

    @property
    def total_q(self) -> int:
        return int(self.query_start[-1])

    @property
    def chunk_lens(self) -> np.ndarray:
        return np.diff(self.query_start).astype(np.int64)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    def positions(self) -> np.ndarray:
        """Position of every query row in its sequence ([total_q] int64)."""
        n = self.chunk_lens
        start = self.context_lens.astype(np.int64) - n
        return np.concatenate([start[s] + np.arange(n[s]) for s in range(self.num_seqs)]) \
            if self.total_q else np.zeros(0, np.int64)

    def flops(self) -> int:
        """Algorithmic FLOPs of the attention: each (row, head) at position p
        does (p + 1) * D multiply-adds for Q.K and as many for P.V."""
        return 4 * self.num_heads * self.head_size * int((self.positions() + 1).sum())

    def io_bytes(self) -> int:
        """Bytes the attention must move at least once: every context token's K
        and V (all heads), the queries and the outputs."""
        H, D = self.num_heads, self.head_size
        return int(self.context_lens.astype(np.int64).sum()) * H * D * 2 * 2 + self.total_q * H * D * 2 * 2


def build_prefill(name: str, num_heads: int, head_size: int, block_size: int, context_lens,
                  chunk_lens, num_blocks: int, table_width: int, seed: int, q_std: float,
                  kv_std: float, poison: str = POISON_HUGE,
                  rng: np.random.Generator | None = None,
                  deal_order: str = "permuted") -> PrefillWorkload:
    """Assemble a prefill step from explicit context and chunk lengths
    (chunk_lens[s] <= context_lens[s]); blocks are dealt as in ``build``."""
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    ctx = np.asarray(context_lens, dtype=np.int32)
    n = np.asarray(chunk_lens, dtype=np.int32)
    assert ctx.shape == n.shape and (n >= 0).all() and (n <= ctx).all()
    S, H, D, B = len(ctx), num_heads, head_size, block_size
    need = [-(-int(L) // B) for L in ctx]
    assert sum(need) <= num_blocks, f"pool of {num_blocks} blocks is too small for {sum(need)}"
    assert max(need, default=0) <= table_width
    order = rng.permutation(num_blocks).astype(np.int32) if deal_order == "permuted" \
        else np.arange(num_blocks, dtype=np.int32)
    tables = np.full((S, table_width), -1, np.int32)
    cursor = 0
    for s in range(S):
        tables[s, :need[s]] = order[cursor:cursor + need[s]]
        cursor += need[s]
    blk_list, off_list = [], []
    for s in range(S):
        pos = np.arange(0, int(ctx[s]) - int(n[s]))
        if pos.size:
            blk_list.append(tables[s, pos // B])
            off_list.append(pos % B)
    blk = np.concatenate(blk_list) if blk_list else np.zeros(0, np.int32)
    off = np.concatenate(off_list) if off_list else np.zeros(0, np.int32)
    qs = np.zeros(S + 1, np.int32)
    qs[1:] = np.cumsum(n)
    T = int(qs[-1])
    query = _draw_f16(rng, (T, H, D), q_std)
    new_key = _draw_f16(rng, (T, H, D), kv_std)
    new_value = _draw_f16(rng, (T, H, D), kv_std)
    live_k = _draw_f16(rng, (blk.size, H, D), kv_std)
    live_v = _draw_f16(rng, (blk.size, H, D), kv_std)
    scale = float(np.float32(1.0) / np.sqrt(np.float32(D)))
    return PrefillWorkload(name=name, num_seqs=S, num_heads=H, head_size=D, block_size=B,
                           num_blocks=num_blocks, scale=scale, query=query, new_key=new_key,
                           new_value=new_value, query_start=qs, block_tables=tables,
                           context_lens=ctx, live_blocks=blk.astype(np.int32),
                           live_offsets=off.astype(np.int32), live_key=live_k, live_value=live_v,
                           poison=poison, seed=seed)


PREFILL_NAMES = {
    1: "prefill_tiny_s4_h4_d128_b32_f16",
    2: "llama13b_prefill_long_s4_h40_d128_b32_f16",
    3: "llama7b_chunked_prefill_s8_h32_d128_b16_f16",
}


def prefill_named(config_id: int, seed: int | None = None, poison: str = POISON_HUGE) -> PrefillWorkload:
    """The prefill workloads (seed defaults to 2000 + config_id):

    1. tiny, for the oracle: 4 sequences (a full 37-token prompt, a 100-token
       chunk after 200 cached tokens, a single token after 128, a full
       1-token prompt), 4 heads, head_size 128, 32-token blocks;
    2. long prompts, the long-text setting of the Llama2-13B comparison: 4
       full prompts of uniform[2048, 8192] tokens, 40 heads, head_size 128,
       32-token blocks (the size the pages advise above 4k tokens);
    3. chunked prefill, LLaMA-7B shapes: 8 sequences each bringing a
       512-token chunk after uniform[0, 2048] cached tokens, 32 heads,
       head_size 128, 16-token blocks.
    K/V are N(0, 0.5^2), queries N(0, 1), blocks dealt from a random permutation.
    """
    seed = 2000 + config_id if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    name = PREFILL_NAMES[config_id]
    if config_id == 1:
        ctx, n = [37, 300, 129, 1], [37, 100, 1, 1]
        return build_prefill(name, 4, 128, 32, ctx, n, 24, 12, seed, 1.0, 0.5, poison, rng=rng)
    if config_id == 2:
        ctx = rng.integers(2048, 8193, 4)
        need = sum(-(-int(L) // 32) for L in ctx)
        return build_prefill(name, 40, 128, 32, ctx, ctx, need + 64, 256, seed, 1.0, 0.5, poison, rng=rng)
    if config_id == 3:
        ctx = 512 + rng.integers(0, 2049, 8)
        need = sum(-(-int(L) // 16) for L in ctx)
        return build_prefill(name, 32, 128, 16, ctx, np.full(8, 512), need + 64, 160, seed, 1.0, 0.5,
                             poison, rng=rng)
    raise KeyError(config_id)


@dataclass
class DevicePrefill:
    """A prefill workload's tensors on a CUDA device (torch)."""
    w: PrefillWorkload
    query: object
    new_key: object
    new_value: object
    query_start: object
    block_tables: object
    context_lens: object
    key_cache: object
    value_cache: object
    out: object
    slots: object


def prefill_to_device(w: PrefillWorkload, device) -> DevicePrefill:
    import torch

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    kc, vc = w.pool_device(device)
    T, H, D = w.query.shape
    return DevicePrefill(w=w, query=up(w.query), new_key=up(w.new_key), new_value=up(w.new_value),
                         query_start=up(w.query_start), block_tables=up(w.block_tables),
                         context_lens=up(w.context_lens), key_cache=kc, value_cache=vc,
                         out=torch.empty((T, H, D), dtype=torch.float16, device=device),
                         slots=torch.empty(T, dtype=torch.int32, device=device))
