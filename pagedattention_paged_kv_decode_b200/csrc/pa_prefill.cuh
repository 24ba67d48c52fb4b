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
    int num_heads;
    int num_blocks;
    int max_blocks_per_seq;
    int max_query_len;
    int stages;
    float qk_scale_log2;          // scale * log2(e)
};

// a1 for a prefill chunk: one thread per new token, grid (row chunks, S);
// rows beyond the grid are covered by the stride loop.
__global__ void prefill_slot_mapping_kernel(int32_t *__restrict__ slot_mapping,
                                            const int32_t *__restrict__ query_start,
                                            const int32_t *__restrict__ block_tables,
                                            int max_blocks_per_seq,
                                            const int32_t *__restrict__ context_lens, int block_size,
                                            int num_blocks) {
    const int s = blockIdx.y;
    const int q0 = query_start[s];
    const int n = query_start[s + 1] - q0;
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
// end of each sequence, so the CTAs with the longest causal range launch
// first. A warp whose rows all end before a tile only passes the tile on.
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

    const int h = blockIdx.x % p.num_heads;
    const int rest = blockIdx.x / p.num_heads;
    const int s = rest % p.num_seqs;
    const int t_rev = rest / p.num_seqs;
    const int q_begin = __ldg(p.query_start + s);
    const int n = __ldg(p.query_start + s + 1) - q_begin;
    const int L = __ldg(p.context_lens + s);
    if (n <= 0) return;
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
