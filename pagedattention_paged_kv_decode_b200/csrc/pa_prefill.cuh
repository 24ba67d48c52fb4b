// pa_prefill.cuh -- paged prefill: causal multi-query attention of a prompt
// (or a chunk of one) over its sequence's block table, on tensor cores.
//
// "vLLM-v0.17.1技术解析" §3.2 names FlashAttention-style attention as part
// of the kernel work; the l189.com/news/180929 article §4 runs long texts
// (over 4k tokens) with 32-token blocks. Reading used: sequence s brings
// n = query_start[s+1] - query_start[s] query rows, the last n positions of
// its L-token context (the cache already holds all L tokens); row i sits at
// position L - n + i and attends tokens 0 .. L - n + i with the decode's
// softmax.
#pragma once

#include "pa_decode.cuh"

namespace pa {

constexpr int kPrefillRows = 64;  // query rows per CTA: 4 consumer warps x 16

struct PrefillParams {
    __half *out;                  // [total_q][H][D]
    const __half *query;          // [total_q][H][D]
    const int32_t *query_start;   // [S + 1]
    const int32_t *block_tables;  // [S][max_blocks_per_seq]
    const int32_t *context_lens;  // [S]
    int num_seqs;
    int total_q;                  // rows of query and out
    int num_heads;
    int num_blocks;
    int max_blocks_per_seq;
    int max_query_len;
    int row_tiles;                // ceil(max_query_len / rows per CTA): grid = row_tiles * S * H
    int stages;
    float qk_scale_log2;          // scale * log2(e)
};

// Rows [q_begin, q_begin + n) of sequence s. False when they do not lie
// inside the total_q rows the caller allocated (query_start negative,
// decreasing or past total_q): such a sequence is touched nowhere.
__device__ __forceinline__ bool chunk_rows(const int32_t *query_start, int s, int total_q, int &q_begin,
                                           int &n) {
    const int64_t a = __ldg(query_start + s), b = __ldg(query_start + s + 1);
    q_begin = (int)a;
    n = (int)(b - a);
    return a >= 0 && b >= a && b <= total_q;
}

// a1 for a prefill chunk: one thread per new token, grid (row chunks, S);
// rows beyond the grid are covered by the stride loop.
__global__ void prefill_slot_mapping_kernel(int32_t *__restrict__ slot_mapping, int total_q,
                                            const int32_t *__restrict__ query_start,
                                            const int32_t *__restrict__ block_tables,
                                            int max_blocks_per_seq,
                                            const int32_t *__restrict__ context_lens, int block_size,
                                            int num_blocks) {
    const int s = blockIdx.y;
    int q0, n;
    if (!chunk_rows(query_start, s, total_q, q0, n)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(PA_DEV_BAD_CHUNK);
        return;
    }
    const int L = context_lens[s];
    const bool bad_chunk = n > L;
    if (bad_chunk && blockIdx.x == 0 && threadIdx.x == 0) flag_error(PA_DEV_BAD_CHUNK);
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        int slot = -1;
        if (!bad_chunk) {
            const int pos = L - n + i;
            const int logical = pos / block_size;
            if (logical >= max_blocks_per_seq) {
                flag_error(PA_DEV_CTX_OVER_TABLE);
            } else {
                const int blk = block_tables[(size_t)s * max_blocks_per_seq + logical];
                if (blk < 0 || blk >= num_blocks)
                    flag_error(PA_DEV_BAD_BLOCK);
                else
                    slot = blk * block_size + pos % block_size;
            }
        }
        slot_mapping[q0 + i] = slot;
    }
}

// One CTA = one head x one tile of up to 64 consecutive query rows of one
// sequence. Consumer warp w takes rows 16w .. 16w+15 of the tile (MmaRows);
// the producer warp streams the K/V blocks 0 .. (last row's position) / B of
// the sequence through a ring of TMA half tiles. Tiles are numbered from the
// end of each sequence, so within a (sequence, head) the CTAs with the
// longest causal range launch first. A warp whose rows all end before a
// tile only passes the tile on.
template <int D, int B>
__global__ void __launch_bounds__(32 * 5, 1)
paged_prefill_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const PrefillParams p) {
    using Lay = PrefixMmaLayout<D, B>;
    constexpr int ON = D / 8;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int stages = p.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)stages * Lay::kStage);
    uint64_t *empty = full + stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // the row tiles of one (sequence, head) are neighbours in the grid, so
    // they run together and share its K/V blocks through L2
    const int t_rev = blockIdx.x % p.row_tiles;
    const int sh = blockIdx.x / p.row_tiles;
    const int h = sh % p.num_heads;
    const int s = sh / p.num_heads;
    int q_begin, n;
    if (!chunk_rows(p.query_start, s, p.total_q, q_begin, n)) {
        if (t_rev == 0 && h == 0 && threadIdx.x == 0) flag_error(PA_DEV_BAD_CHUNK);
        return;
    }
    const int L = __ldg(p.context_lens + s);
    if (n == 0) return;
    if (n > L || n > p.max_query_len) {  // the whole sequence is skipped
        if (t_rev == 0 && h == 0 && threadIdx.x == 0) flag_error(PA_DEV_BAD_CHUNK);
        return;
    }
    if (L > p.max_blocks_per_seq * B) {
        if (t_rev == 0 && h == 0 && threadIdx.x == 0) flag_error(PA_DEV_CTX_OVER_TABLE);
        return;
    }
    const int n_tiles = (n + kPrefillRows - 1) / kPrefillRows;
    if (t_rev >= n_tiles) return;
    const int r0 = (n_tiles - 1 - t_rev) * kPrefillRows;  // first row of the tile
    const int rows_here = min(kPrefillRows, n - r0);
    const int n_consumers = (rows_here + 15) / 16;
    const int base = L - n;                                 // position of row 0
    const int nblk = (base + r0 + rows_here + B - 1) / B;   // blocks up to the last row's position
    const int32_t *table = p.block_tables + (size_t)s * p.max_blocks_per_seq;

    if (warp == n_consumers) {
        // ---------------------------------------------------------- producer
        int pre = 0;
        if (lane < nblk) pre = __ldg(table + lane);
        if (lane == 0) {
            prefetch_tensor_map(&tmap_k);
            prefetch_tensor_map(&tmap_v);
            for (int i = 0; i < stages; ++i) {
                mbar_init(&full[i], 1);
                mbar_init(&empty[i], n_consumers);
            }
            fence_mbar_init();
        }
        __syncwarp();
        asm volatile("bar.arrive 1, %0;" ::"r"((n_consumers + 1) * 32) : "memory");
        const uint64_t policy = l2_policy_evict_normal();  // other row tiles of the sequence re-read these
        bool ok = true;
        for (int i = 0; i < nblk && ok; ++i) {
            if (i > 0 && (i & 31) == 0) {
                pre = 0;
                if (i + lane < nblk) pre = __ldg(table + i + lane);
            }
            int blk = __shfl_sync(0xffffffffu, pre, i & 31);
            const bool bad = blk < 0 || blk >= p.num_blocks;
            if (bad) blk = p.num_blocks;  // outside the tensor map: zero filled
            const int st = i % stages, use = i / stages;
            if (lane == 0) {
                if (bad) flag_error(PA_DEV_BAD_BLOCK);
                if (use > 0) ok = mbar_wait(&empty[st], (use - 1) & 1);
                if (ok) {
                    unsigned char *kdst = smem + (size_t)st * Lay::kStage;
                    mbar_arrive_expect_tx(&full[st], (uint32_t)Lay::kStage);
#pragma unroll
                    for (int hf = 0; hf < Lay::kHalves; ++hf) {
                        tma_load_4d(kdst + hf * Lay::kHalfTile, &tmap_k, &full[st], 64 * hf, h, 0, blk, policy);
                        tma_load_4d(kdst + Lay::kTile + hf * Lay::kHalfTile, &tmap_v, &full[st], 64 * hf, h, 0,
                                    blk, policy);
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        return;
    }
    if (warp > n_consumers) return;

    // -------------------------------------------------------------- consumers
    const int g = lane >> 2;
    const int c = (lane & 3) * 2;
    const int rl[2] = {r0 + warp * 16 + g, r0 + warp * 16 + g + 8};  // rows within the sequence
    int lim[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) lim[r] = rl[r] < n ? base + rl[r] + 1 : 0;
    const int warp_lim = base + min(n - 1, r0 + warp * 16 + 15) + 1;  // the warp's last row
    MmaRows<D, B> mr;
    mr.load_q(rl[0] < n ? p.query + ((size_t)(q_begin + rl[0]) * p.num_heads + h) * D : nullptr,
              rl[1] < n ? p.query + ((size_t)(q_begin + rl[1]) * p.num_heads + h) * D : nullptr,
              p.qk_scale_log2, lane);
    asm volatile("bar.sync 1, %0;" ::"r"((n_consumers + 1) * 32) : "memory");

    for (int i = 0; i < nblk; ++i) {
        const int st = i % stages, use = i / stages;
        if (!mbar_wait(&full[st], use & 1)) break;
        if (i * B < warp_lim) {
            const unsigned char *kt = smem + (size_t)st * Lay::kStage;
            mr.attend(kt, kt + Lay::kTile, i * B, lim, L, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }

    mr.reduce_l();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (rl[r] >= n) continue;
        const float inv = 1.0f / mr.l[r];  // token 0 is always visible: l >= 1
        __half *op = p.out + ((size_t)(q_begin + rl[r]) * p.num_heads + h) * D;
#pragma unroll
        for (int j = 0; j < ON; ++j)
            *reinterpret_cast<__half2 *>(op + j * 8 + c) =
                __floats2half2_rn(mr.o[j][2 * r] * inv, mr.o[j][2 * r + 1] * inv);
    }
}

}  // namespace pa

namespace pa {

// -------------------------------- prefill on tcgen05 (head_size 64 or 128)
//
// One CTA = one head x one tile of up to 128 consecutive query rows of one
// sequence; K/V are consumed 128 tokens at a time. Per K/V tile j:
//   S_j = Q . K_j^T   128 x 128, D / 16 tcgen05.mma (K = 16 each) into tensor
//                     memory (three S buffers: S_{j+2} is computed while the
//                     softmax works on j, so the softmax never waits for S)
//   softmax           reads S, masks tokens after each row's position, keeps
//                     a reference maximum that moves only when the row
//                     maximum exceeds it by more than 2^8 (then O is rescaled
//                     in tensor memory), and writes P = 2^(s - m) as fp16 back
//                     into the S buffer it came from (tcgen05.st)
//   O += P_j . V_j    eight tcgen05.mma (N = D) with A (P) read from tensor
//                     memory and V from shared memory, N-contiguous (MN-major)
// An S buffer takes the next S only once the P.V that reads its P is done.
// One thread issues the MMAs: S_0, S_1, then per tile j, S_{j+2} (as soon
// as its buffer is free) before P.V of j (once P_j is written).
// K and V have rings of their own (3 and 2 tiles): a K tile is released as
// soon as its S is computed, a V tile when its P.V is, so each is reloaded
// as early as possible. Warps: 0-3 softmax (and Q staging, epilogue): warp
// w takes rows 32 w .. + 31 (its tensor-memory lanes), each thread a whole
// row of S, P and O, so no row is shared and no warp waits for another
// within a tile; the sub-partition's MUFU serves the row's exponentials
// alone. 4 K producer; 5 MMA issuer (also allocates the 512 tensor-memory
// columns); 6 V producer. Each producer keeps the next 32 block-table
// entries in flight.
// Every wait is bounded; a wait that runs out sets PA_DEV_WAIT_TIMEOUT and
// an abort flag that ends the other roles' waits, and the CTA still drains
// its copies and MMAs and frees its tensor memory before it exits.
constexpr int kTcRows = 128;
constexpr int kTcKv = 128;
constexpr int kTcKStages = 3;
constexpr int kTcVStages = 2;
constexpr int kTcSoftmaxWarps = 4;  // one per tensor-memory lane quadrant, one thread per row
constexpr int kTcWarpK = 4, kTcWarpMma = 5, kTcWarpV = 6;
constexpr int kTcThreads = 32 * (kTcSoftmaxWarps + 3);
constexpr int kTcSBufs = 3;        // S buffers (P of a tile is written over its S)
constexpr int kTcTmemCols = 512;   // S0 [0,128), S1 [128,256), S2 [256,384), O [384,384+D)
constexpr int kTcColO = kTcSBufs * kTcKv;

template <int D>
struct TcLayout {                                       // byte offsets from the 1024-aligned base
    static constexpr uint32_t kHalf = 128 * 128;         // [128 rows][128 B]: one 64-wide half
    static constexpr uint32_t kTile = (D / 64) * kHalf;  // a 128 x D fp16 tile in 64-wide halves
    static constexpr uint32_t kQ = 0;                    // Q (dims 0-63, 64-127)
    static constexpr uint32_t kK = kQ + kTile;           // K ring
    static constexpr uint32_t kV = kK + kTcKStages * kTile;  // V ring
    static constexpr uint32_t kBars = kV + kTcVStages * kTile;
    static constexpr uint32_t kBytes = kBars + 512;      // barriers, tensor-memory address, abort flag
};

// mbarrier indices
enum : int {
    kBarQ = 0,                              // Q staged (every softmax warp)
    kBarFullK = 1,                          // + stage: K tile landed (TMA bytes)
    kBarEmptyK = kBarFullK + kTcKStages,    // + stage: S of the stage's tile done (commit)
    kBarFullV = kBarEmptyK + kTcKStages,    // + stage: V tile landed
    kBarEmptyV = kBarFullV + kTcVStages,    // + stage: P.V of the stage's tile done (commit)
    kBarSFull = kBarEmptyV + kTcVStages,    // + buffer: S ready (commit)
    kBarPFull = kBarSFull + kTcSBufs,       // + buffer: P written into tensor memory, O corrected (every
                                            // softmax warp)
    kBarOReady = kBarPFull + kTcSBufs,      // + buffer: P.V of the buffer's tile done (commit); one
                                            // per buffer, as a warp may reach tile j before P.V of
                                            // j-2 is done, and a wait must stay within two phases
    kBarDone = kBarOReady + kTcSBufs,       // every MMA of the CTA done (commit)
    kNumBars = kBarDone + 1
};
static_assert(8 * kNumBars + 8 <= TcLayout<128>::kBytes - TcLayout<128>::kBars, "barrier area too small");
static_assert(TcLayout<128>::kBytes + 1024 <= 227 * 1024, "shared memory of the tcgen05 prefill kernel");

// Bounded wait that also ends when another role has aborted. It spins on
// the non-blocking test (these waits are short and on the critical path,
// where a suspended thread would wake up late).
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_test_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            flag_error(PA_DEV_WAIT_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
}

// Lane 0 waits; the warp goes on (all lanes, ordered after the wait) if it
// saw the phase.
__device__ __forceinline__ bool tc_wait_lane0(uint64_t *bar, uint32_t parity, volatile int *abort, int lane) {
    bool ok = true;
    if (lane == 0) ok = tc_wait(bar, parity, abort);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok;
}

// 16 bytes at chunk c (0..15) of row r of a [halves][128 rows][128 B]
// swizzled tile.
__device__ __forceinline__ uint32_t tc_chunk(uint32_t base, int r, int c) {
    return base + (uint32_t)(c >> 3) * TcLayout<128>::kHalf + (uint32_t)r * 128u +
           ((uint32_t)(((c & 7) ^ (r & 7))) << 4);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// One producer warp: streams the K (or V) tiles 0 .. n_kv-1 of the CTA
// through its ring. Lane b < BPT loads cache block b of each tile; lane l
// holds block-table entry 32c + l of the current chunk c while the next
// chunk's entries are already being read (the first two chunks, cur and
// nxt, are read by the caller before the CTA's set-up).
template <int D, int B, int STAGES>
__device__ __forceinline__ void tc_produce(const CUtensorMap *tmap, unsigned char *ring, uint64_t *full,
                                           uint64_t *empty, const int32_t *table, int nblk, int n_kv, int h,
                                           int num_blocks, volatile int *abort, int lane, int cur, int nxt) {
    constexpr int BPT = kTcKv / B;
    const uint64_t policy = l2_policy_evict_normal();  // other row tiles re-read these blocks
    auto fetch = [&](int chunk) {
        const int lb = chunk * 32 + lane;
        return lb < nblk ? __ldg(table + lb) : -1;
    };
    int issued = 0;
    for (int j = 0; j < n_kv; ++j) {
        const int st = j % STAGES, use = j / STAGES;
        const int lb0 = j * BPT;  // first block of the tile; tiles never straddle a chunk (BPT divides 32)
        if (lb0 > 0 && (lb0 & 31) == 0) {
            cur = nxt;
            nxt = fetch((lb0 >> 5) + 1);
        }
        int blk = __shfl_sync(0xffffffffu, cur, (lb0 & 31) + (lane < BPT ? lane : 0));
        if (lane < BPT) {
            if (lb0 + lane >= nblk) {
                blk = num_blocks;  // past the sequence: zero filled
            } else if (blk < 0 || blk >= num_blocks) {
                flag_error(PA_DEV_BAD_BLOCK);
                blk = num_blocks;
            }
        }
        bool ok = true;
        if (lane == 0 && use > 0) ok = tc_wait(&empty[st], (use - 1) & 1, abort);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)TcLayout<D>::kTile);
        __syncwarp();
        if (lane < BPT) {
            unsigned char *dst = ring + st * TcLayout<D>::kTile + lane * B * 128;
            tma_load_4d(dst, tmap, &full[st], 0, h, 0, blk, policy);
            if (D == 128) tma_load_4d(dst + TcLayout<D>::kHalf, tmap, &full[st], 64, h, 0, blk, policy);
        }
        issued = j + 1;
    }
    // let the copies in flight land before the warp retires
    if (lane == 0)
        for (int j = max(0, issued - STAGES); j < issued; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
}

template <int D, int B>
__global__ void __launch_bounds__(kTcThreads, 1)
paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                        const PrefillParams p) {
    static_assert(D == 64 || D == 128, "head_size 64 or 128");
    using Lay = TcLayout<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + Lay::kBars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Lay::kBars + 8 * kNumBars);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + Lay::kBars + 8 * kNumBars + 4);
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- the CTA's rows (uniform; every early exit precedes any barrier).
    // The row tiles of one (sequence, head) are neighbours in the grid, so
    // they run together and share its K/V blocks through L2.
    const int t_rev = blockIdx.x % p.row_tiles;
    const int sh = blockIdx.x / p.row_tiles;
    const int h = sh % p.num_heads;
    const int s = sh / p.num_heads;
    int q_begin, n;
    if (!chunk_rows(p.query_start, s, p.total_q, q_begin, n)) {
        if (t_rev == 0 && h == 0 && threadIdx.x == 0) flag_error(PA_DEV_BAD_CHUNK);
        return;
    }
    const int L = __ldg(p.context_lens + s);
    if (n == 0) return;
    if (n > L || n > p.max_query_len) {
        if (t_rev == 0 && h == 0 && threadIdx.x == 0) flag_error(PA_DEV_BAD_CHUNK);
        return;
    }
    if (L > p.max_blocks_per_seq * B) {
        if (t_rev == 0 && h == 0 && threadIdx.x == 0) flag_error(PA_DEV_CTX_OVER_TABLE);
        return;
    }
    const int n_tiles = (n + kTcRows - 1) / kTcRows;
    if (t_rev >= n_tiles) return;
    const int r0 = (n_tiles - 1 - t_rev) * kTcRows;
    const int rows_here = min(kTcRows, n - r0);
    const int base = L - n;                                  // position of row 0 of the chunk
    const int kv_end = base + r0 + rows_here;                // tokens the last row sees
    const int nblk = (kv_end + B - 1) / B;
    const int n_kv = (kv_end + kTcKv - 1) / kTcKv;
    const int32_t *table = p.block_tables + (size_t)s * p.max_blocks_per_seq;

    // ---- reads that depend on nothing set up below go out first: the
    // producers' first 64 block-table entries and each softmax thread's Q row
    int tab0 = -1, tab1 = -1;
    if (warp == kTcWarpK || warp == kTcWarpV) {
        tab0 = lane < nblk ? __ldg(table + lane) : -1;
        tab1 = 32 + lane < nblk ? __ldg(table + 32 + lane) : -1;
    }
    const int t = warp * 32 + lane;  // softmax warps: row of the tile = tensor-memory lane
    const int rl = r0 + t;
    const bool valid = warp < kTcSoftmaxWarps && rl < n;
    uint4 q_row[D / 8];
    if (warp < kTcSoftmaxWarps) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.query + ((size_t)(q_begin + (valid ? rl : 0)) * p.num_heads + h) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) q_row[c] = valid ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }

    // ---- set-up: tensor memory, barriers
    if (warp == kTcWarpMma) {
        tmem_alloc(tmem_slot, kTcTmemCols);
        tmem_relinquish();
    }
    if (warp == kTcWarpK && lane == 0) {
        prefetch_tensor_map(&tmap_k);
        prefetch_tensor_map(&tmap_v);
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(&bar[i], (i == kBarQ || (i >= kBarPFull && i < kBarPFull + kTcSBufs))
                                   ? kTcSoftmaxWarps : 1);
        *abort = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kTcWarpK) {
        tc_produce<D, B, kTcKStages>(&tmap_k, smem + Lay::kK, &bar[kBarFullK], &bar[kBarEmptyK], table, nblk, n_kv, h,
                                  p.num_blocks, abort, lane, tab0, tab1);
        return;
    }
    if (warp == kTcWarpV) {
        tc_produce<D, B, kTcVStages>(&tmap_v, smem + Lay::kV, &bar[kBarFullV], &bar[kBarEmptyV], table, nblk, n_kv, h,
                                  p.num_blocks, abort, lane, tab0, tab1);
        return;
    }

    if (warp == kTcWarpMma) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t kIdescS = tc_idesc_f16(kTcRows, kTcKv, false);
        constexpr uint32_t kIdescPV = tc_idesc_f16(kTcRows, D, true);
        // K-major operands (Q, K, P): 8-row groups 1024 B apart; V: MN-major,
        // the two 64-dim halves kHalf apart, 8-token groups 1024 B apart. A
        // k-step moves the start address (descriptor bits 0-13, in 16 B).
        const uint64_t dq = sw128_desc(sbase + Lay::kQ, 16, 1024);
        const uint64_t dk = sw128_desc(sbase + Lay::kK, 16, 1024);
        const uint64_t dv = sw128_desc(sbase + Lay::kV, Lay::kHalf, 1024);
        auto kstep = [](int k) { return (uint64_t)(((k >> 2) * Lay::kHalf + (k & 3) * 32) >> 4); };
        // One thread issues every MMA and takes every wait of this role
        // (a waiting lane costs the softmax warps of its sub-partition issue
        // slots); the other lanes wait for it at the end.
        auto issue_s = [&](int j) -> bool {
            const int st = j % kTcKStages, b = j % kTcSBufs;
            if (!tc_wait(&bar[kBarFullK + st], (j / kTcKStages) & 1, abort)) return false;
            // buffer b holds S_{j-3}, then P_{j-3}, until the P.V of tile j-3
            // is done (the last P.V issued). That P.V follows every softmax
            // warp's P of the tile, and each warp writes its P only after its
            // loads of S have completed, so the one wait covers both.
            if (j >= kTcSBufs && !tc_wait(&bar[kBarOReady + b], (j / kTcSBufs - 1) & 1, abort)) return false;
            tc_fence_after();
            const uint64_t dks = dk + ((st * Lay::kTile) >> 4);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
                tc_mma_f16(tmem + b * kTcKv, dq + kstep(ks), dks + kstep(ks), kIdescS, ks > 0 ? 1u : 0u);
            tc_commit(&bar[kBarSFull + b]);
            tc_commit(&bar[kBarEmptyK + st]);
            return true;
        };
        auto issue_pv = [&](int i) -> bool {
            const int st = i % kTcVStages, b = i % kTcSBufs;
            if (!tc_wait(&bar[kBarPFull + b], (i / kTcSBufs) & 1, abort)) return false;
            if (!tc_wait(&bar[kBarFullV + st], (i / kTcVStages) & 1, abort)) return false;
            tc_fence_after();
            const uint64_t dvs = dv + ((st * Lay::kTile) >> 4);
#pragma unroll
            for (int kt = 0; kt < kTcKv / 16; ++kt)
                // P_i in tensor memory, in S buffer i % 3: tokens 64 h .. 64 h + 63
                // packed in columns 64 h .. 64 h + 31 (two fp16 per column)
                tc_mma_f16_ts(tmem + kTcColO, tmem + b * kTcKv + (kt >> 2) * 64 + (kt & 3) * 8,
                              dvs + ((kt * 16 * 128) >> 4), kIdescPV, (i > 0 || kt > 0) ? 1u : 0u);
            tc_commit(&bar[kBarEmptyV + st]);
            tc_commit(&bar[kBarOReady + b]);
            return true;
        };
        if (lane == 0) {
            bool ok = tc_wait(&bar[kBarQ], 0, abort);
            for (int j = 0; ok && j < min(kTcSBufs - 1, n_kv); ++j) ok = issue_s(j);
            for (int j = 0; ok && j < n_kv; ++j) {
                if (j + kTcSBufs - 1 < n_kv) ok = issue_s(j + kTcSBufs - 1);
                if (ok) ok = issue_pv(j);
            }
            // every MMA issued above completes before the tensor memory is freed
            tc_commit(&bar[kBarDone]);
            mbar_wait(&bar[kBarDone], 0);
        }
        __syncwarp();
        tc_fence_before();
        asm volatile("bar.sync 2, %0;" ::"r"(32 * (kTcSoftmaxWarps + 1)) : "memory");
        tc_fence_after();
        tmem_dealloc(tmem, kTcTmemCols);
        return;
    }

    // -------------------------------------------------------------- softmax
    const int lim = valid ? base + rl + 1 : 0;  // tokens 0 .. lim-1 are visible
    {
#pragma unroll
        for (int c = 0; c < D / 8; ++c) st_shared_v4(tc_chunk(sbase + Lay::kQ, t, c), q_row[c]);  // the row's 16-byte chunks
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[kBarQ]);
    }
    const float c2 = p.qk_scale_log2;  // > 0 on this path
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
        const int sb = j % kTcSBufs;  // S / P buffer of this tile
        if (!tc_wait_lane0(&bar[kBarSFull + sb], (j / kTcSBufs) & 1, abort, lane)) { ok = false; break; }
        tc_fence_after();
        float sv[kTcKv];
#pragma unroll
        for (int q = 0; q < kTcKv / 32; ++q) {
            float v32[32];
            tmem_ld32(tl + sb * kTcKv + q * 32, v32);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[q * 32 + i] = v32[i];
        }

        const int t0 = j * kTcKv;  // position of the tile's first column
        if (t0 + kTcKv > lim) {
#pragma unroll
            for (int k = 0; k < kTcKv; ++k)
                if (t0 + k >= lim) sv[k] = -INFINITY;
        }
        float mx;
        {  // tree reduction: short dependence chains
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = sv[i];
#pragma unroll
            for (int k = 8; k < kTcKv; ++k) m8[k & 7] = fmaxf(m8[k & 7], sv[k]);
            mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        }
        mx *= c2;
        float alpha = 1.f;
        bool resc = false;
        if (mx > m_ref + 8.f) {  // the reference maximum moves only by more than 2^8
            alpha = fast_exp2(m_ref - mx);
            m_ref = mx;
            resc = true;
        }
        const float mr = m_ref == -INFINITY ? 0.f : m_ref;
        // P = 2^(s - m) as fp16 pairs: tokens 64 h .. 64 h + 63 of the tile go
        // to columns 64 h .. 64 h + 31 of the buffer (all S columns are in
        // registers by now)
        float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float pf[32];
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float p0 = fast_exp2(fmaf(sv[64 * hh + 2 * k], c2, -mr));
                const float p1 = fast_exp2(fmaf(sv[64 * hh + 2 * k + 1], c2, -mr));
                rs4[k & 3] += p0 + p1;
                pf[k] = __uint_as_float(pack_half2(p0, p1));
            }
            tmem_st32(tl + sb * kTcKv + 64 * hh, pf);
        }
        l = l * alpha + ((rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));

        // O must be current before a rescale: wait for P.V of tile j-1
        if (j >= 1 && __any_sync(0xffffffffu, resc)) {
            if (!tc_wait_lane0(&bar[kBarOReady + (j - 1) % kTcSBufs], ((j - 1) / kTcSBufs) & 1, abort, lane)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < D / 32; ++q) {
                float ov[32];
                tmem_ld32(tl + kTcColO + q * 32, ov);
#pragma unroll
                for (int i = 0; i < 32; ++i) ov[i] *= alpha;
                tmem_st32(tl + kTcColO + q * 32, ov);
            }
        }
        // tokens at or after the sequence end are unused cache slots (any
        // bits, NaN included): their V rows enter P.V as zeros
        const int tt = j * kTcKv;
        if (tt + kTcKv > L) {
            const int vst = j % kTcVStages;
            // V_{j-2} shares the stage and may not have landed yet (this warp
            // can be two tiles ahead of P.V): wait for its P.V first, so that
            // the stage's wait below names its last phase or the one before
            if (j >= kTcVStages &&
                !tc_wait_lane0(&bar[kBarOReady + (j - kTcVStages) % kTcSBufs], ((j - kTcVStages) / kTcSBufs) & 1, abort,
                               lane)) {
                ok = false;
                break;
            }
            if (!tc_wait_lane0(&bar[kBarFullV + vst], (j / kTcVStages) & 1, abort, lane)) { ok = false; break; }
            if (tt + t >= L) {
                const uint32_t v_addr = sbase + Lay::kV + vst * Lay::kTile;
#pragma unroll
                for (int c = 0; c < D / 8; ++c) st_shared_v4(tc_chunk(v_addr, t, c), make_uint4(0, 0, 0, 0));
            }
            fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[kBarPFull + sb]);
    }
    if (ok && tc_wait_lane0(&bar[kBarOReady + (n_kv - 1) % kTcSBufs], ((n_kv - 1) / kTcSBufs) & 1, abort, lane)) {
        tc_fence_after();
        const float inv = valid ? 1.0f / l : 0.f;
        __half *op = p.out + ((size_t)(q_begin + (valid ? rl : 0)) * p.num_heads + h) * D;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
            float ov[32];
            tmem_ld32(tl + kTcColO + q * 32, ov);
            if (valid) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 v = make_uint4(pack_half2(ov[8 * c] * inv, ov[8 * c + 1] * inv),
                                               pack_half2(ov[8 * c + 2] * inv, ov[8 * c + 3] * inv),
                                               pack_half2(ov[8 * c + 4] * inv, ov[8 * c + 5] * inv),
                                               pack_half2(ov[8 * c + 6] * inv, ov[8 * c + 7] * inv));
                    *reinterpret_cast<uint4 *>(op + q * 32 + c * 8) = v;
                }
            }
        }
    }
    tc_fence_before();
    asm volatile("bar.sync 2, %0;" ::"r"(32 * (kTcSoftmaxWarps + 1)) : "memory");
}

}  // namespace pa
