// pa_decode.cuh -- paged decode attention kernels for sm_100a.
//
// What is computed (the plain definition of single-query softmax attention
// over the tokens a block table addresses; the pages fix the block table and
// the physical block pool -- "vLLM-v0.17.1技术解析" §2.2, "在A10G上榨干LLaMA-7B"
// §2.1 -- but print no kernel):
//   z_t = scale * k_scale * q . K_t,   out = v_scale * sum_t softmax(z)_t V_t
//
// Design (one work unit = one sequence x a group of G heads x one partition
// of the context; a CTA serves C units, each in its own slot):
//   * a producer warp reads the block-table entries of every slot's
//     partition and issues, per physical block, two TMA tiled loads -- the K
//     and V tiles [block_size][G][head_size] of the 4-D cache view
//     [NB][B][H][D] -- into the slot's ring of shared-memory stages guarded by
//     full/empty mbarriers, a ring-full per slot first, then in turn;
//   * G x W consumer warps: warp (g, w) owns head g and every W-th block of
//     the partition. Per block it forms the logits with 16-byte shared loads
//     (exact fp16 x fp16 products summed in fp32; E4M3 codes are first
//     decoded exactly to fp16 pairs), reduces them with a transposing
//     butterfly (one shuffle per token per lane), runs the online-softmax
//     update with a lazily moved maximum and accumulates P.V in fp32;
//   * units are numbered long partitions first (see unit_coord);
//   * the W warps of a head merge (m, l, acc) through shared memory; a
//     sequence that fits one partition writes fp16 output directly, longer
//     ones write (lse, normalised o) for the log-sum-exp reduce kernel, which
//     is launched as a programmatic dependent of this one.
// The plain decode is not a dense contraction (one query row per head), so
// it runs on the CUDA cores and is bound by HBM bandwidth. The shared-prefix
// kernels further down are where one K/V tile meets many query rows (every
// sequence of the batch); the fp16 one computes that on tensor cores.
#pragma once

#include <type_traits>

#include "pa_device.cuh"

namespace pa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxConsumerWarps = 16;  // units_per_cta * heads_per_cta * warps_per_head
constexpr int kMaxUnitsPerCta = 4;
constexpr int kMaxDecodeThreads = 32 * (kMaxConsumerWarps + 1);

struct DecodeParams {
    __half *out;                 // [S][H][D]
    const __half *query;         // [S][H][D]
    const int32_t *block_tables; // [S][max_blocks_per_seq]
    const int32_t *context_lens; // [S]
    float *ws_lse;               // [S][H][max_parts] (split only)
    float *ws_o;                 // [S][H][max_parts][D] (split only)
    int num_seqs;
    int num_heads;
    int num_blocks;
    int block_size;
    int max_blocks_per_seq;
    int max_context_len;
    int partition_size;          // tokens, multiple of block_size
    int max_parts;               // ceil(max_context_len / partition_size)
    int heads_per_cta;           // G
    int warps_per_head;          // W
    int stages;
    int units_per_cta;           // C work units (slots) per CTA
    int64_t num_units;           // num_seqs * (num_heads / G) * max_parts
    // Shared prefix (all 0 for a plain decode): the first prefix_tokens
    // tokens of every sequence live in the same physical blocks (those of
    // table row 0). The decode kernel then covers tokens prefix_tokens.. only
    // and always writes partials, at index prefix_parts + part of each
    // (sequence, head); the prefix kernel fills indices 0..prefix_parts-1.
    int prefix_tokens;
    int prefix_parts;
    int prefix_partition;        // tokens per prefix partition (multiple of block_size)
    int queries_per_cta;         // prefix kernel: sequences sharing one CTA's tiles
    int ws_parts;                // partial slots per (sequence, head) in the workspace
    float qk_scale_log2;         // scale * log2(e)
    float logit_k_scale;         // k_scale, applied to each E4M3 logit (1 for fp16 caches)
    float out_scale;             // v_scale (1 for fp16 caches)
    // Fused append (all null/0 for a plain decode): each sequence's new token
    // at position L-1 is stored into its slot before the block holding it is
    // loaded; slot_out[s] receives that slot (-1 if none).
    const __half *new_key;       // [S][H][D], row stride new_key_stride elements
    const __half *new_value;
    int64_t new_key_stride;
    int64_t new_value_stride;
    void *key_cache;             // same pools the tensor maps describe
    void *value_cache;
    int32_t *slot_out;
    float k_scale;               // E4M3 encode scales (1 for fp16 caches)
    float v_scale;
    // Bounded waits of the decode kernel: the wall-time limit of each
    // mbarrier wait (0, the default: kWaitLimitNs; a test may shorten it),
    // and a test hook: with stall_unit_plus1 = u + 1 the producer issues no
    // tile loads for work unit u, so that unit's consumers must give up at
    // the limit (0, the default: no unit is stalled).
    uint64_t wait_limit_ns;
    int64_t stall_unit_plus1;
};


// Lane geometry of a consumer warp. Each lane holds EPL consecutive elements
// of a K/V row (16 bytes), LPR lanes cover one row of head_size elements,
// and the warp's NGRP lane groups take different tokens of a block.
template <int D, int B, bool kFp8>
struct Geometry {
    static constexpr int kElemBytes = kFp8 ? 1 : 2;
    static constexpr int EPL = 16 / kElemBytes;
    static constexpr int LPR = D / EPL;
    static constexpr int NGRP = 32 / LPR;
    static constexpr int TPG = B / NGRP;          // tokens of a block per lane group
    static constexpr int DUP = LPR / TPG;         // lanes holding the same logit after the butterfly
    static constexpr int kRowBytes = D * kElemBytes;
    static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "head_size / lane mapping");
    static_assert(TPG >= 1 && TPG <= LPR && LPR % TPG == 0, "block_size / lane mapping");
};

// Transposing butterfly: on entry part[j] is this lane's partial dot product
// for token j of its group (over its EPL dims). After the log2(LPR) rounds,
// part[0] is the full dot product of token (sub / DUP), where sub is the
// lane's index inside its group. Each split round hands half of the values
// to the partner lane and keeps the other half, so a group of LPR lanes
// reduces TPG dot products with TPG-1 (+ log2 DUP) shuffles per lane.
template <int TPG, int LPR>
__device__ __forceinline__ float butterfly_reduce(float (&part)[TPG], int lane) {
    int n = TPG;
#pragma unroll
    for (int mask = LPR / 2; mask >= 1; mask >>= 1) {
        if (n > 1) {
            const int half = n / 2;
            const bool upper = (lane & mask) != 0;
#pragma unroll
            for (int k = 0; k < TPG / 2; ++k) {
                if (k < half) {
                    const float send = upper ? part[k] : part[k + half];
                    const float keep = upper ? part[k + half] : part[k];
                    part[k] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
                }
            }
            n = half;
        } else {
            part[0] += __shfl_xor_sync(0xffffffffu, part[0], mask);
        }
    }
    return part[0];
}

// 16 bytes of a K/V row -> EPL floats.
template <bool kFp8>
__device__ __forceinline__ void unpack16(const uint4 &raw, float *f);

template <>
__device__ __forceinline__ void unpack16<false>(const uint4 &raw, float *f) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __half22float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

template <>
__device__ __forceinline__ void unpack16<true>(const uint4 &raw, float *f) {
    const uint16_t *c = reinterpret_cast<const uint16_t *>(&raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 x = __half22float2(e4m3x2_to_half2(c[i]));
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

// Online-softmax attention state of one warp for one (query, head): the
// per-tile arithmetic shared by the decode and the shared-prefix kernels.
// Lane layout (Geometry): lane group `grp` takes TPG tokens of each tile,
// lane `sub` of the group holds EPL elements of the query, K/V rows and
// output accumulator.
//
// Arithmetic: every product is formed exactly (fp16 x fp16 into fp32, one
// FMA-pipe instruction per element, fma.rn.f32.f16) and summed in fp32:
//   logits  z_t = (scale * log2 e * k_scale) * sum_d q[d] k_t[d]   (q as given, k
//           as stored: fp16, or the E4M3 code decoded exactly to fp16);
//   weights p_t = 2^(z_t - m), rounded to fp16 once, and that same fp16
//           value enters both l = sum_t p_t and acc[d] = sum_t p_t v_t[d],
//           so acc / l is an exact convex combination of the rows.
// The reference maximum m moves lazily: only when a tile holds a logit more
// than kLazyMax above it (then m becomes the running maximum and l, acc are
// rescaled). Weights therefore stay at most 2^kLazyMax, and most tiles of a
// long context cost no warp-wide maximum and no rescale.
template <int D, int B, bool kFp8>
struct HeadAttn {
    using Geo = Geometry<D, B, kFp8>;
    static constexpr int EPL = Geo::EPL, LPR = Geo::LPR, TPG = Geo::TPG, DUP = Geo::DUP;
    static constexpr float kLazyMax = 8.0f;
    uint32_t q2[EPL / 2];  // this lane's query elements as fp16 pairs (bits as given)
    float m, l;
    float acc[EPL];

    __device__ __forceinline__ void init(const uint4 (&q_raw)[EPL / 8]) {
#pragma unroll
        for (int c = 0; c < EPL / 8; ++c) {
            q2[4 * c + 0] = q_raw[c].x;
            q2[4 * c + 1] = q_raw[c].y;
            q2[4 * c + 2] = q_raw[c].z;
            q2[4 * c + 3] = q_raw[c].w;
        }
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    }

    // sum over this lane's EPL dims of q * k (16 bytes of one K row)
    __device__ __forceinline__ float dot16(const uint4 &raw) const {
        float c0 = 0.f, c1 = 0.f;
        const uint32_t *w = reinterpret_cast<const uint32_t *>(&raw);
        if constexpr (kFp8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t k01, k23;
                e4m3x4_to_half2x2(w[i], k01, k23);
                fma2_f16_f32(q2[2 * i], k01, c0, c1);
                fma2_f16_f32(q2[2 * i + 1], k23, c0, c1);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) fma2_f16_f32(q2[i], w[i], c0, c1);
        }
        return c0 + c1;
    }

    // acc += p * v over this lane's EPL dims (p: fp16 in the low half of p1)
    __device__ __forceinline__ void axpy16(uint32_t p1, const uint4 &raw) {
        const uint32_t *w = reinterpret_cast<const uint32_t *>(&raw);
        if constexpr (kFp8) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t v01, v23;
                e4m3x4_to_half2x2(w[i], v01, v23);
                fma1x2_f16_f32(p1, v01, acc[4 * i], acc[4 * i + 1]);
                fma1x2_f16_f32(p1, v23, acc[4 * i + 2], acc[4 * i + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) fma1x2_f16_f32(p1, w[i], acc[2 * i], acc[2 * i + 1]);
        }
    }

    // One tile: rows t < valid of the tile (row t at `ktile + t*row_stride +
    // head_off`, V likewise) take part; rows at or past `valid` are never
    // multiplied into acc (they may hold anything, NaN included).
    template <bool kFull>
    __device__ __forceinline__ void tile(const unsigned char *ktile, const unsigned char *vtile,
                                         size_t row_stride, size_t head_off, int valid, float qk_mul,
                                         int lane) {
        const int grp = lane / LPR, sub = lane % LPR;
        // ---- logits of this lane group's TPG tokens
        float part_dot[TPG];
#pragma unroll
        for (int j = 0; j < TPG; ++j) {
            const int t = grp * TPG + j;
            part_dot[j] = dot16(*reinterpret_cast<const uint4 *>(ktile + t * row_stride + head_off));
        }
        const int my_t = grp * TPG + sub / DUP;
        float z = butterfly_reduce<TPG, LPR>(part_dot, lane) * qk_mul;
        if (!kFull) z = (my_t < valid) ? z : -INFINITY;

        // ---- online softmax (base 2) with a lazily moved reference maximum
        if (__any_sync(0xffffffffu, z > m + kLazyMax)) {
            const float m_new = fmaxf(m, warp_max(z));
            const float alpha = fast_exp2(m - m_new);  // m = -inf on the first tile: 0
            l *= alpha;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] *= alpha;
            m = m_new;
        }
        const uint32_t p1 = f32_to_f16_bits(fast_exp2(z - m));  // <= 2^kLazyMax
        l = add_f16_f32(p1, l);

        // ---- P.V for this lane group's tokens
#pragma unroll
        for (int j = 0; j < TPG; ++j) {
            const int t = grp * TPG + j;
            const uint32_t pj = __shfl_sync(0xffffffffu, p1, grp * LPR + j * DUP);
            if (kFull || t < valid)
                axpy16(pj, *reinterpret_cast<const uint4 *>(vtile + t * row_stride + head_off));
        }
    }

    // One tile whose V rows at or past `valid` hold zeros (the caller wrote
    // them): the logits are masked, the P.V loop runs over every row.
    __device__ __forceinline__ void consume_v_zeroed(const unsigned char *ktile, const unsigned char *vtile,
                                                     size_t row_stride, size_t head_off, int valid,
                                                     float qk_mul, int lane) {
        const int grp = lane / LPR, sub = lane % LPR;
        float part_dot[TPG];
#pragma unroll
        for (int j = 0; j < TPG; ++j) {
            const int t = grp * TPG + j;
            part_dot[j] = dot16(*reinterpret_cast<const uint4 *>(ktile + t * row_stride + head_off));
        }
        const int my_t = grp * TPG + sub / DUP;
        float z = butterfly_reduce<TPG, LPR>(part_dot, lane) * qk_mul;
        z = (my_t < valid) ? z : -INFINITY;
        if (__any_sync(0xffffffffu, z > m + kLazyMax)) {
            const float m_new = fmaxf(m, warp_max(z));
            const float alpha = fast_exp2(m - m_new);
            l *= alpha;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] *= alpha;
            m = m_new;
        }
        const uint32_t p1 = f32_to_f16_bits(fast_exp2(z - m));
        l = add_f16_f32(p1, l);
#pragma unroll
        for (int j = 0; j < TPG; ++j) {
            const int t = grp * TPG + j;
            const uint32_t pj = __shfl_sync(0xffffffffu, p1, grp * LPR + j * DUP);
            axpy16(pj, *reinterpret_cast<const uint4 *>(vtile + t * row_stride + head_off));
        }
    }

    __device__ __forceinline__ void consume(const unsigned char *ktile, const unsigned char *vtile,
                                            size_t row_stride, size_t head_off, int valid, float qk_mul,
                                            int lane) {
        if (valid >= B) tile<true>(ktile, vtile, row_stride, head_off, valid, qk_mul, lane);
        else tile<false>(ktile, vtile, row_stride, head_off, valid, qk_mul, lane);
    }

    // Sums l over all lanes and acc over the lane groups (group 0 then holds
    // the warp's whole accumulator).
    __device__ __forceinline__ void finish() {
        l = warp_sum(l) * (1.0f / DUP);
#pragma unroll
        for (int mask = LPR; mask < 32; mask <<= 1) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], mask);
        }
    }
};

// Shared-memory carve-up, identical on host and device. A CTA serves C work
// units ("slots"); slot j owns a ring of `stages` K/V stages and a merge
// area. The mbarriers of all slots follow the slots: full[C][stages],
// empty[C][stages].
struct SmemLayout {
    size_t tile_bytes;   // one K (or V) tile: B * G * D * elem
    size_t stage_bytes;  // K tile + V tile
    size_t merge_off;    // within a slot: W * G * (D + 2) floats
    size_t slot_bytes;   // multiple of 128 (TMA destinations stay 128-byte aligned)
    size_t bars_off;
    size_t total;
    __host__ __device__ SmemLayout(int B, int G, int D, int elem, int W, int stages, int C) {
        tile_bytes = (size_t)B * G * D * elem;
        stage_bytes = 2 * tile_bytes;
        merge_off = stage_bytes * stages;
        slot_bytes = (merge_off + sizeof(float) * (size_t)W * G * (D + 2) + 127) / 128 * 128;
        bars_off = slot_bytes * C;
        total = bars_off + 8 * (size_t)C * 2 * stages;
    }
};

// One work unit: sequence s, heads h0 .. h0+G-1, partition `part` of the
// context (tokens t0 .. t1-1 in physical blocks blk0 .. blk0+nblk-1 of the
// table row). CTA c serves units c, c + gridDim.x, ... (one per slot).
//
// Units are numbered with the partition slowest and the highest partition
// first, then the sequence, then the head group. The highest partitions
// exist only for the longest contexts, so the grid starts with their (full)
// partitions and ends with partition 0 of every sequence, the short
// contexts' only work: long work first, short work last, without knowing
// the lengths on the host. Units of a partition beyond a context's length
// exit at once. Neighbouring CTAs take the head groups of one sequence, so
// together they read whole token rows of its blocks.
struct UnitCoord {
    int s, hg, part;
};

__device__ __forceinline__ UnitCoord unit_coord(const DecodeParams &p, uint32_t id) {
    // unit ids fit 32 bits: the host keeps num_units below 2^31
    const uint32_t HG = (uint32_t)(p.num_heads / p.heads_per_cta);
    const uint32_t per_part = (uint32_t)p.num_seqs * HG;
    UnitCoord c;
    c.part = p.max_parts - 1 - (int)(id / per_part);
    const uint32_t r = id % per_part;
    c.s = (int)(r / HG);
    c.hg = (int)(r % HG);
    return c;
}
struct Unit {
    int s, h0, part;
    int L_in, L;       // context length as given and as clamped to the table and bound
    int n_parts;       // partitions of this context
    int t0, t1, blk0, nblk;
    bool live;         // part < n_parts
    bool append;       // fused append happens in this unit
};

__device__ __forceinline__ Unit unit_of(const DecodeParams &p, int B, int j) {
    Unit u;
    // unit ids fit 32 bits: the host keeps num_units below 2^31, and C * grid
    // stays below 2^32 for every C
    const uint32_t id = blockIdx.x + (uint32_t)j * gridDim.x;
    const bool exists = (int64_t)id < p.num_units;
    const UnitCoord c = unit_coord(p, exists ? id : 0u);
    u.part = c.part;
    u.h0 = c.hg * p.heads_per_cta;
    u.s = c.s;
    u.L_in = exists ? __ldg(p.context_lens + u.s) : 0;
    int L = min(u.L_in, p.max_blocks_per_seq * B);
    L = min(L, p.max_context_len);
    u.L = max(L, 0);
    const int rem = max(u.L - p.prefix_tokens, 0);  // tokens after the shared prefix
    u.n_parts = (rem + p.partition_size - 1) / p.partition_size;
    u.live = exists && u.part < u.n_parts;
    u.t0 = p.prefix_tokens + u.part * p.partition_size;
    u.t1 = min(u.L, u.t0 + p.partition_size);
    u.blk0 = u.t0 / B;
    u.nblk = u.live ? (u.t1 - u.t0 + B - 1) / B : 0;
    u.append = u.live && p.new_key != nullptr && u.part == u.n_parts - 1 && u.L == u.L_in &&
               u.L > p.prefix_tokens;
    return u;
}

// Launch bounds: the default instantiation takes any launch shape (up to
// kMaxDecodeThreads threads); the "narrow" one (at most kNarrowDecodeThreads
// threads, registers capped so that kNarrowDecodeCtas CTAs fit an SM) is
// used when the cap lets more CTAs share an SM (two warps per head).
constexpr int kNarrowDecodeThreads = 288;
constexpr int kNarrowDecodeCtas = 3;

template <int D, int B, bool kFp8, int kThreads = kMaxDecodeThreads, int kMinCtas = 1>
__global__ void __launch_bounds__(kThreads, kMinCtas)
paged_decode_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
    using Geo = Geometry<D, B, kFp8>;
    constexpr int EPL = Geo::EPL, LPR = Geo::LPR;
    constexpr int EB = Geo::kElemBytes;

    extern __shared__ __align__(1024) unsigned char smem[];
    const int G = p.heads_per_cta, W = p.warps_per_head, stages = p.stages, C = p.units_per_cta;
    const SmemLayout lay(B, G, D, EB, W, stages, C);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + lay.bars_off);
    uint64_t *full_all = bars;                           // [C][stages]
    uint64_t *empty_all = bars + (size_t)C * stages;     // [C][stages]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int per_slot = G * W;
    const int n_consumers = C * per_slot;
    const uint64_t wait_limit = p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs;
    // A dependent reduce may be scheduled once every CTA of this grid runs
    // (it waits for this grid's completion before touching its partials).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == n_consumers) {
        // ================================================================ producer
        // Loads whose addresses do not depend on context lengths go first:
        // the first 32 table entries of every slot's partition.
        int pre_blk[kMaxUnitsPerCta];
#pragma unroll
        for (int j = 0; j < kMaxUnitsPerCta; ++j) {
            pre_blk[j] = 0;
            if (j < C) {
                const uint32_t id = blockIdx.x + (uint32_t)j * gridDim.x;
                if ((int64_t)id < p.num_units) {
                    const UnitCoord c = unit_coord(p, id);
                    const int e = (p.prefix_tokens + c.part * p.partition_size) / B + lane;
                    if (e < p.max_blocks_per_seq)
                        pre_blk[j] = __ldg(p.block_tables + (size_t)c.s * p.max_blocks_per_seq + e);
                }
            }
        }
        if (lane == 0) {
            prefetch_tensor_map(&tmap_k);
            prefetch_tensor_map(&tmap_v);
            for (int i = 0; i < C * stages; ++i) {
                mbar_init(&full_all[i], 1);
                mbar_init(&empty_all[i], G);
            }
            fence_mbar_init();
        }
        __syncwarp();
        asm volatile("bar.arrive 1, %0;" ::"r"((n_consumers + 1) * 32) : "memory");  // barriers ready

        Unit u[kMaxUnitsPerCta];
        int issued[kMaxUnitsPerCta];
        int cur_blk[kMaxUnitsPerCta];  // 32 table entries of the chunk being issued
#pragma unroll
        for (int j = 0; j < kMaxUnitsPerCta; ++j) {  // independent loads: all in flight together
            if (j < C) u[j] = unit_of(p, B, j);
            else u[j].live = u[j].append = false, u[j].nblk = 0;
            if (j < C && (int64_t)blockIdx.x + (int64_t)j * gridDim.x + 1 == p.stall_unit_plus1) u[j].nblk = 0;
            issued[j] = 0;
            cur_blk[j] = pre_blk[j];
        }
#pragma unroll
        for (int j = 0; j < kMaxUnitsPerCta; ++j) {
            if (j < C && lane == 0 && u[j].part == 0 && u[j].h0 == 0 &&
                (int64_t)blockIdx.x + (int64_t)j * gridDim.x < p.num_units) {
                if (u[j].L_in > p.max_blocks_per_seq * B) flag_error(PA_DEV_CTX_OVER_TABLE);
                else if (u[j].L_in > p.max_context_len) flag_error(PA_DEV_CTX_OVER_BOUND);
                // sequences with nothing to append report slot -1
                if (p.slot_out && !(p.new_key != nullptr && u[j].L == u[j].L_in && u[j].L > p.prefix_tokens))
                    p.slot_out[u[j].s] = -1;
                // shared prefix: appending inside the shared blocks breaks copy-on-write
                if (p.prefix_tokens > 0 && p.new_key != nullptr && u[j].L > 0 && u[j].L <= p.prefix_tokens)
                    flag_error(PA_DEV_PREFIX);
            }
        }
        // shared prefix: this sequence's first table entries must be row 0's
        if (p.prefix_tokens > 0) {
#pragma unroll
            for (int j = 0; j < kMaxUnitsPerCta; ++j) {
                const int64_t id = (int64_t)blockIdx.x + (int64_t)j * gridDim.x;
                if (j < C && id < p.num_units && u[j].part == 0 && u[j].h0 == 0 && u[j].s > 0) {
                    bool same = true;
                    for (int e = lane; e < p.prefix_tokens / B; e += 32)
                        same &= __ldg(p.block_tables + (size_t)u[j].s * p.max_blocks_per_seq + e) ==
                                __ldg(p.block_tables + e);
                    if (!__all_sync(0xffffffffu, same) && lane == 0) flag_error(PA_DEV_PREFIX);
                }
            }
        }
        const uint64_t policy = l2_policy_evict_first();
        const uint32_t tx_bytes = (uint32_t)lay.stage_bytes;
        bool ok = true;

        // Issues the next block of slot j (waiting for its stage to drain).
        auto issue = [&](int j) {
            const Unit &x = u[j];
            const int i = issued[j];
            if ((i & 31) == 0 && i > 0) {
                cur_blk[j] = 0;
                if (i + lane < x.nblk)
                    cur_blk[j] = __ldg(p.block_tables + (size_t)x.s * p.max_blocks_per_seq + x.blk0 + i + lane);
            }
            int blk = __shfl_sync(0xffffffffu, cur_blk[j], i & 31);
            const bool bad = blk < 0 || blk >= p.num_blocks;
            if (bad) blk = p.num_blocks;  // out of range: the TMA zero-fills the tile
            const int st = i % stages, use = i / stages;
            if (lane == 0) {
                if (bad) flag_error(PA_DEV_BAD_BLOCK);
                if (use > 0) ok = mbar_wait(&empty_all[j * stages + st], (use - 1) & 1, wait_limit);
                if (ok) {
                    unsigned char *kdst = smem + (size_t)j * lay.slot_bytes + (size_t)st * lay.stage_bytes;
                    uint64_t *fb = &full_all[j * stages + st];
                    mbar_arrive_expect_tx(fb, tx_bytes);
                    tma_load_4d(kdst, &tmap_k, fb, 0, x.h0, 0, blk, policy);
                    tma_load_4d(kdst + lay.tile_bytes, &tmap_v, fb, 0, x.h0, 0, blk, policy);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            issued[j] = i + 1;
        };

        // 1) the first ring-full of every slot (no waits)
#pragma unroll
        for (int j = 0; j < kMaxUnitsPerCta; ++j)
            if (j < C)
                while (ok && issued[j] < min(u[j].nblk, stages)) issue(j);

        // 2) the rest, one block per slot in turn
        bool more = true;
        while (ok && more) {
            more = false;
#pragma unroll
            for (int j = 0; j < kMaxUnitsPerCta; ++j) {
                if (j < C && ok && issued[j] < u[j].nblk) {
                    issue(j);
                    more = true;
                }
            }
        }
        return;
    }

    // ================================================================ consumers
    const int slot = warp / per_slot;
    const int gw = warp % per_slot;
    const int g = gw % G;
    const int w = gw / G;
    const int grp = lane / LPR;
    const int sub = lane % LPR;

    // Query row: its address depends on the unit id only.
    uint4 q_raw[EPL / 8], nk_raw[EPL / 8], nv_raw[EPL / 8];
    {
        const uint32_t id = blockIdx.x + (uint32_t)slot * gridDim.x;
        const UnitCoord c = unit_coord(p, (int64_t)id < p.num_units ? id : 0u);
        const int hq = c.hg * G + g;
        const int sq = c.s;
        const uint4 *qp = reinterpret_cast<const uint4 *>(p.query + ((size_t)sq * p.num_heads + hq) * D);
#pragma unroll
        for (int c = 0; c < EPL / 8; ++c) q_raw[c] = __ldg(qp + sub * (EPL / 8) + c);
        // Fused append: this lane's dims of the head's new K/V row, fetched
        // with the query (used only if this unit turns out to hold the token).
        if (p.new_key != nullptr) {
            const uint4 *kp = reinterpret_cast<const uint4 *>(p.new_key + (size_t)sq * p.new_key_stride + (size_t)hq * D);
            const uint4 *vp = reinterpret_cast<const uint4 *>(p.new_value + (size_t)sq * p.new_value_stride + (size_t)hq * D);
#pragma unroll
            for (int c = 0; c < EPL / 8; ++c) {
                nk_raw[c] = __ldg(kp + sub * (EPL / 8) + c);
                nv_raw[c] = __ldg(vp + sub * (EPL / 8) + c);
            }
        }
    }
    const Unit x = unit_of(p, B, slot);
    const int h = x.h0 + g;
    unsigned char *slot_base = smem + (size_t)slot * lay.slot_bytes;
    uint64_t *full = full_all + slot * stages;
    uint64_t *empty = empty_all + slot * stages;
    float *merge = reinterpret_cast<float *>(slot_base + lay.merge_off);
    asm volatile("bar.sync 1, %0;" ::"r"((n_consumers + 1) * 32) : "memory");  // barriers ready

    if (!x.live) {
        // empty context: zeros (partition 0 of a context of length 0)
        const int64_t id = (int64_t)blockIdx.x + (int64_t)slot * gridDim.x;
        if (id < p.num_units && x.L == 0 && x.part == 0 && p.prefix_tokens == 0 && w == 0 && lane < D / 8)
            reinterpret_cast<uint4 *>(p.out + ((size_t)x.s * p.num_heads + h) * D)[lane] = make_uint4(0, 0, 0, 0);
        return;  // (all warps of this slot leave together: no merge barrier to meet)
    }

    HeadAttn<D, B, kFp8> st;
    st.init(q_raw);
    const float qk_mul = p.qk_scale_log2 * p.logit_k_scale;

    const size_t row_stride = (size_t)G * D * EB;  // bytes between tokens in a tile
    const size_t head_off = (size_t)g * D * EB + (size_t)sub * 16;
    // Fused append (a1 + a2): the unit holding position L-1 takes the new
    // token in cache format (E4M3 codes for an fp8 cache, so that it is used
    // exactly as a later step will read it back). The lanes of group 0 park
    // their part of the row in this warp's merge area (unused until the
    // merge) instead of keeping it in registers through the loop; once the
    // block holding the token has landed, the lanes that read that row copy
    // it over their head's part of the row in shared memory. The first warp
    // of each head stores the head's row into the token's slot in the cache.
    // The loaded row itself is never used, so no tile load waits for the store.
    int t_new_block = -1, t_new_row = -1;
    uint2 *stash = reinterpret_cast<uint2 *>(merge + (size_t)(w * G + g) * (D + 2)) + sub * 4;
    if (x.append) {
        const int pos = x.L - 1;
        t_new_block = (pos - x.t0) / B;
        t_new_row = pos % B;
        uint4 k_new, v_new;
        if constexpr (!kFp8) {
            k_new = nk_raw[0];
            v_new = nv_raw[0];
        } else {
            const uint2 k0 = encode8_e4m3(nk_raw[0], p.k_scale), k1 = encode8_e4m3(nk_raw[1], p.k_scale);
            const uint2 v0 = encode8_e4m3(nv_raw[0], p.v_scale), v1 = encode8_e4m3(nv_raw[1], p.v_scale);
            k_new = make_uint4(k0.x, k0.y, k1.x, k1.y);
            v_new = make_uint4(v0.x, v0.y, v1.x, v1.y);
        }
        if (grp == 0) {
            stash[0] = make_uint2(k_new.x, k_new.y);
            stash[1] = make_uint2(k_new.z, k_new.w);
            stash[2] = make_uint2(v_new.x, v_new.y);
            stash[3] = make_uint2(v_new.z, v_new.w);
        }
        if (w == 0 && grp == 0) {
            const int blk = __ldg(p.block_tables + (size_t)x.s * p.max_blocks_per_seq + pos / B);
            const bool bad = blk < 0 || blk >= p.num_blocks;  // flagged where its tile is loaded
            if (!bad) {
                const size_t dst = (((size_t)blk * B + pos % B) * p.num_heads + h) * D * EB + (size_t)sub * 16;
                *reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.key_cache) + dst) = k_new;
                *reinterpret_cast<uint4 *>(static_cast<unsigned char *>(p.value_cache) + dst) = v_new;
            }
            if (p.slot_out && h == 0 && sub == 0) p.slot_out[x.s] = bad ? -1 : blk * B + pos % B;
        }
        __syncwarp();
    }
    int stage = w % stages, use = w / stages;
    for (int i = w; i < x.nblk; i += W) {
        if (!mbar_wait(&full[stage], use & 1, wait_limit)) break;
        unsigned char *ktile = slot_base + (size_t)stage * lay.stage_bytes;
        unsigned char *vtile = ktile + lay.tile_bytes;
        const int valid = min(B, x.t1 - (x.t0 + i * B));  // tokens of this block inside the context
        if (i == t_new_block) {
            if (grp == t_new_row / Geo::TPG) {
                const uint2 k0 = stash[0], k1 = stash[1], v0 = stash[2], v1 = stash[3];
                *reinterpret_cast<uint4 *>(ktile + t_new_row * row_stride + head_off) = make_uint4(k0.x, k0.y, k1.x, k1.y);
                *reinterpret_cast<uint4 *>(vtile + t_new_row * row_stride + head_off) = make_uint4(v0.x, v0.y, v1.x, v1.y);
                fence_proxy_async_smem();  // before the stage is refilled by the next TMA
            }
            __syncwarp();
        }
        // The context ends inside this block: zero this head's V rows past it
        // (they may hold anything, NaN included), so that one P.V loop serves
        // every tile; the logits of those rows are masked.
        if (valid < B) {
#pragma unroll
            for (int j = 0; j < Geo::TPG; ++j) {
                const int t = grp * Geo::TPG + j;
                if (t >= valid) *reinterpret_cast<uint4 *>(vtile + t * row_stride + head_off) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            __syncwarp();
        }
        st.consume_v_zeroed(ktile, vtile, row_stride, head_off, valid, qk_mul, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        stage += W;
        if (stage >= stages) {  // W <= stages
            stage -= stages;
            ++use;
        }
    }

    // ---- reduce this warp's state: l over all lanes, acc over lane groups
    st.finish();
    float m = st.m, l = st.l;
    float (&acc)[EPL] = st.acc;

    // ---- merge the W warps of each head through the slot's shared memory
    if (W > 1) {
        float *mine = merge + (size_t)(w * G + g) * (D + 2);
        if (grp == 0) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) mine[sub * EPL + e] = acc[e];
        }
        if (lane == 0) {
            mine[D] = m;
            mine[D + 1] = l;
        }
        asm volatile("bar.sync %0, %1;" ::"r"(2 + slot), "r"(per_slot * 32) : "memory");
        if (w != 0) return;
        float M = -INFINITY;
        for (int k = 0; k < W; ++k) M = fmaxf(M, merge[(size_t)(k * G + g) * (D + 2) + D]);
        float Lsum = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        for (int k = 0; k < W; ++k) {
            const float *o = merge + (size_t)(k * G + g) * (D + 2);
            const float f = fast_exp2(o[D] - M);  // warps without tokens: m = -inf -> 0
            Lsum += o[D + 1] * f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] += o[sub * EPL + e] * f;
        }
        m = M;
        l = Lsum;
    }

    if (grp != 0) return;
    const float inv_l = 1.0f / l;
    if (x.n_parts == 1 && p.prefix_tokens == 0) {
        __half *op = p.out + ((size_t)x.s * p.num_heads + h) * D + sub * EPL;
#pragma unroll
        for (int c = 0; c < EPL / 8; ++c) {
            uint4 pk;
            __half2 *hp = reinterpret_cast<__half2 *>(&pk);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                hp[i] = __floats2half2_rn(acc[c * 8 + 2 * i] * inv_l * p.out_scale,
                                          acc[c * 8 + 2 * i + 1] * inv_l * p.out_scale);
            reinterpret_cast<uint4 *>(op)[c] = pk;
        }
    } else {
        const size_t idx = ((size_t)x.s * p.num_heads + h) * p.ws_parts + p.prefix_parts + x.part;
        float *op = p.ws_o + idx * D + sub * EPL;
#pragma unroll
        for (int c = 0; c < EPL / 4; ++c)
            reinterpret_cast<float4 *>(op)[c] =
                make_float4(acc[4 * c] * inv_l, acc[4 * c + 1] * inv_l, acc[4 * c + 2] * inv_l,
                            acc[4 * c + 3] * inv_l);
        if (sub == 0) p.ws_lse[idx] = m + fast_log2(l);
    }
}

// Log-sum-exp reduction of the partial results of each (sequence, head):
// the partitions of a context longer than one partition, and with a shared
// prefix, the prefix partitions followed by the suffix partitions. One warp
// per (sequence, head):
//   M = max_p lse_p,  w_p = 2^(lse_p - M),  out = v_scale * sum_p w_p o_p / sum_p w_p
// Partials without tokens carry lse = -inf and o = 0 (weight 0).
template <int D>
__global__ void __launch_bounds__(128)
lse_reduce_kernel(const DecodeParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x * 4 + warp;
    const int s = blockIdx.y;
    if (h >= p.num_heads) return;
    int L = __ldg(p.context_lens + s);
    L = min(L, p.max_blocks_per_seq * p.block_size);   // same clamps as the partition kernels
    L = min(L, p.max_context_len);
    L = max(L, 0);
    const int rem = max(L - p.prefix_tokens, 0);
    const int n_suffix = (rem + p.partition_size - 1) / p.partition_size;
    const int n_parts = p.prefix_parts + n_suffix;
    constexpr int DPL = D / 32;  // dims per lane
    __half *op = p.out + ((size_t)s * p.num_heads + h) * D + lane * DPL;
    if (p.prefix_tokens == 0 && n_parts <= 1) return;  // written by the partition kernel
    // Launched as a programmatic dependent of the partition kernel: wait for
    // it (and its memory) before reading partials or writing the output.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (L == 0) {
#pragma unroll
        for (int e = 0; e < DPL; e += 2) *reinterpret_cast<__half2 *>(op + e) = __floats2half2_rn(0.f, 0.f);
        return;
    }
    const size_t base = ((size_t)s * p.num_heads + h) * p.ws_parts;
    // The partials' loads go out together, in chunks of kChunk, the first
    // chunk with the log-sum-exps: lane i of the warp holds the weight of
    // partial c0 + i of each 32-wide group, the others take it by shuffle.
    using Vec = typename std::conditional<DPL == 4, float4, float2>::type;
    constexpr int kChunk = 16;
    Vec v[kChunk];
    auto load_chunk = [&](int c0) {
#pragma unroll
        for (int k = 0; k < kChunk; ++k) {
            const int i = c0 + k;
            if (i < n_parts) v[k] = *reinterpret_cast<const Vec *>(p.ws_o + (base + i) * D + lane * DPL);
            else v[k] = Vec{};
        }
    };
    load_chunk(0);
    const float lse0 = lane < n_parts ? p.ws_lse[base + lane] : -INFINITY;
    float M = lse0;
    for (int i = lane + 32; i < n_parts; i += 32) M = fmaxf(M, p.ws_lse[base + i]);
    M = warp_max(M);
    float wl = fast_exp2(lse0 - M);  // lanes past the partials: 0
    float wsum = wl;
    float acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
    for (int c0 = 0; c0 < n_parts; c0 += kChunk) {
        if (c0 > 0) {
            load_chunk(c0);
            if ((c0 & 31) == 0) {
                const int i = c0 + lane;
                wl = fast_exp2((i < n_parts ? p.ws_lse[base + i] : -INFINITY) - M);
                wsum += wl;
            }
        }
#pragma unroll
        for (int k = 0; k < kChunk; ++k) {
            const float wgt = __shfl_sync(0xffffffffu, wl, (c0 + k) & 31);  // 0 past the partials
            const float *x = reinterpret_cast<const float *>(&v[k]);
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[e] = fmaf(wgt, x[e], acc[e]);
        }
    }
    wsum = warp_sum(wsum);
    const float f = p.out_scale / wsum;
#pragma unroll
    for (int e = 0; e < DPL; e += 2)
        *reinterpret_cast<__half2 *>(op + e) = __floats2half2_rn(acc[e] * f, acc[e + 1] * f);
}

// Shared-prefix attention ("在A10G上榨干LLaMA-7B" §2.2: requests sharing a
// prompt map its logical blocks to the same physical blocks). The prefix
// blocks -- the first prefix_tokens tokens of table row 0, which every row
// shares -- are read once per CTA and applied to the queries of up to
// queries_per_cta sequences: one CTA = G heads x one prefix partition x a
// block of sequences; consumer warp (g, i) computes head g of sequence
// qb * queries_per_cta + i over every tile (masked to that sequence's own
// length) with the same per-tile arithmetic as the decode, and writes the
// partition's partial (lse, o) at index pp of the sequence's partials.
template <int D, int B, bool kFp8>
__global__ void __launch_bounds__(kMaxDecodeThreads, 1)
paged_prefix_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
    using Geo = Geometry<D, B, kFp8>;
    constexpr int EPL = Geo::EPL, LPR = Geo::LPR;
    constexpr int EB = Geo::kElemBytes;
    extern __shared__ __align__(1024) unsigned char smem[];
    const int G = p.heads_per_cta, QC = p.queries_per_cta, stages = p.stages;
    const SmemLayout lay(B, G, D, EB, 1, stages, 1);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.bars_off);
    uint64_t *empty = full + stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_consumers = G * QC;

    const int n_qb = (p.num_seqs + QC - 1) / QC;
    const int qb = blockIdx.x % n_qb;
    const int rest = blockIdx.x / n_qb;
    const int pp = rest % p.prefix_parts;
    const int h0 = (rest / p.prefix_parts) * G;
    const int t0 = pp * p.prefix_partition;
    const int t1 = min(p.prefix_tokens, t0 + p.prefix_partition);
    const int blk0 = t0 / B;
    const int nblk = (t1 - t0 + B - 1) / B;

    if (warp == n_consumers) {
        // ---------------------------------------------------------- producer
        int pre = 0;
        if (lane < nblk) pre = __ldg(p.block_tables + blk0 + lane);  // row 0 holds the shared blocks
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
        const uint64_t policy = l2_policy_evict_first();
        bool ok = true;
        for (int i = 0; i < nblk && ok; ++i) {
            if (i > 0 && (i & 31) == 0) {
                pre = 0;
                if (i + lane < nblk) pre = __ldg(p.block_tables + blk0 + i + lane);
            }
            int blk = __shfl_sync(0xffffffffu, pre, i & 31);
            const bool bad = blk < 0 || blk >= p.num_blocks;
            if (bad) blk = p.num_blocks;
            const int st = i % stages, use = i / stages;
            if (lane == 0) {
                if (bad) flag_error(PA_DEV_BAD_BLOCK);
                if (use > 0) ok = mbar_wait(&empty[st], (use - 1) & 1);
                if (ok) {
                    unsigned char *kdst = smem + (size_t)st * lay.stage_bytes;
                    mbar_arrive_expect_tx(&full[st], (uint32_t)lay.stage_bytes);
                    tma_load_4d(kdst, &tmap_k, &full[st], 0, h0, 0, blk, policy);
                    tma_load_4d(kdst + lay.tile_bytes, &tmap_v, &full[st], 0, h0, 0, blk, policy);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int g = warp % G;
    const int s = qb * QC + warp / G;
    const int h = h0 + g;
    const bool active = s < p.num_seqs;
    const int sub = lane % LPR, grp = lane / LPR;
    uint4 q_raw[EPL / 8];
    int L = 0;
    if (active) {
        const uint4 *qp = reinterpret_cast<const uint4 *>(p.query + ((size_t)s * p.num_heads + h) * D);
#pragma unroll
        for (int c = 0; c < EPL / 8; ++c) q_raw[c] = __ldg(qp + sub * (EPL / 8) + c);
        L = __ldg(p.context_lens + s);
        L = min(L, p.max_blocks_per_seq * B);
        L = max(min(L, p.max_context_len), 0);
    } else {
#pragma unroll
        for (int c = 0; c < EPL / 8; ++c) q_raw[c] = make_uint4(0, 0, 0, 0);
    }
    asm volatile("bar.sync 1, %0;" ::"r"((n_consumers + 1) * 32) : "memory");
    HeadAttn<D, B, kFp8> st;
    st.init(q_raw);
    const float qk_mul = p.qk_scale_log2 * p.logit_k_scale;
    const int end = min(t1, L);  // this sequence's tokens in the partition
    const size_t row_stride = (size_t)G * D * EB;
    const size_t head_off = (size_t)g * D * EB + (size_t)sub * 16;
    for (int i = 0; i < nblk; ++i) {
        const int stg = i % stages, use = i / stages;
        if (!mbar_wait(&full[stg], use & 1)) break;
        const int valid = min(B, end - (t0 + i * B));
        if (valid > 0) {
            const unsigned char *ktile = smem + (size_t)stg * lay.stage_bytes;
            st.consume(ktile, ktile + lay.tile_bytes, row_stride, head_off, valid, qk_mul, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stg]);
    }
    if (!active) return;
    st.finish();
    if (grp != 0) return;
    const size_t idx = ((size_t)s * p.num_heads + h) * p.ws_parts + pp;
    float *op = p.ws_o + idx * D + sub * EPL;
    const bool any = st.l > 0.f;
    const float inv_l = any ? 1.0f / st.l : 0.f;
#pragma unroll
    for (int c = 0; c < EPL / 4; ++c)
        reinterpret_cast<float4 *>(op)[c] = make_float4(st.acc[4 * c] * inv_l, st.acc[4 * c + 1] * inv_l,
                                                        st.acc[4 * c + 2] * inv_l, st.acc[4 * c + 3] * inv_l);
    if (sub == 0) p.ws_lse[idx] = any ? st.m + fast_log2(st.l) : -INFINITY;
}

// Tensor-core attention of 16 query rows per warp over K/V tiles of B
// tokens held in shared memory as 64-dim half tiles with 128-byte swizzle
// (what a TMA load with box {64, 1, B, 1} and CU_TENSOR_MAP_SWIZZLE_128B
// writes). Fragment layout of mma.m16n8k16: lane l holds rows g = l / 4 and
// g + 8 and the column pair c = 2 (l % 4), c + 1 of each 8-wide n-tile.
// Per tile:
//   S (16 x B)  = Q (16 x D) . K^T        K fragments by ldmatrix
//   online softmax per row on the S fragments, tokens >= the row's limit masked
//   O (16 x D) += P (16 x B) . V          P reused from the S registers as the
//                                         A operand, V fragments by ldmatrix.trans
// Q and P are f16 (P <= 1: relative rounding <= 2^-11); S and O accumulate
// in fp32. Scores are in log2 units: Q is pre-scaled by scale * log2(e).
template <int D, int B>
struct MmaRows {
    static constexpr int KS = D / 16;   // k-steps over dims
    static constexpr int NT = B / 8;    // score n-tiles (8 tokens each)
    static constexpr int ON = D / 8;    // output n-tiles (8 dims each)
    static constexpr int kHalfTile = B * 128;  // bytes of one 64-dim half tile

    uint32_t qa[KS][4];
    float o[ON][4];
    float m[2], l[2];

    // q0 / q1: the D query values of fragment rows g and g + 8 (null: zeros).
    __device__ __forceinline__ void load_q(const __half *q0, const __half *q1, float sc, int lane) {
        const int c = (lane & 3) * 2;
        const __half *qr[2] = {q0, q1};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    uint32_t v = 0;
                    if (qr[r] != nullptr) {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(qr[r] + ks * 16 + c + 8 * hi));
                        v = pack_half2(f.x * sc, f.y * sc);
                    }
                    qa[ks][r + 2 * hi] = v;  // a0 (row g), a1 (row g+8), a2/a3: +8 columns
                }
            }
        }
#pragma unroll
        for (int j = 0; j < ON; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
    }

    // One tile: kt / vt the K and V tiles, tb the position of its first
    // token, lim[r] the exclusive token limit of fragment row r, vlim the
    // end of the sequence: V rows at or after it are unused cache slots
    // whose contents may be anything (NaN included) and enter P.V as zeros.
    __device__ __forceinline__ void attend(const unsigned char *kt, const unsigned char *vt, int tb,
                                           const int (&lim)[2], int vlim, int lane) {
        const int c = (lane & 3) * 2;
        // ---- S = Q K^T
        float sacc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                // matrices: (tokens +0..7, dims +0..7), (+0..7, +8..15), (+8..15, +0..7), (+8..15, +8..15)
                const int mi = lane >> 3, r = lane & 7;
                const int tok = np * 16 + ((mi >> 1) << 3) + r;
                const int dim = ks * 16 + ((mi & 1) << 3);
                const unsigned char *addr = kt + (dim >> 6) * kHalfTile + swz128(tok, (dim & 63) * 2);
                uint32_t b[4];
                ldmatrix_x4(b, addr);
                mma_16816(sacc[2 * np], qa[ks], b[0], b[1]);
                mma_16816(sacc[2 * np + 1], qa[ks], b[2], b[3]);
            }
        }

        // ---- online softmax per row (rows g and g+8 of this warp's 16)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = e >> 1;
                const int tok = tb + n * 8 + c + (e & 1);
                if (tok >= lim[r]) sacc[n][e] = -INFINITY;
                mx[r] = fmaxf(mx[r], sacc[n][e]);
            }
        }
        float alpha[2], mref[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            const float mn = fmaxf(m[r], mx[r]);
            mref[r] = mn == -INFINITY ? 0.f : mn;  // rows without tokens so far stay at zero
            alpha[r] = fast_exp2(m[r] - mref[r]);
            m[r] = mn;
        }
        uint32_t pa[NT / 2][4];
        float rs[2] = {0.f, 0.f};
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const float p0 = fast_exp2(sacc[n][0] - mref[0]);
            const float p1 = fast_exp2(sacc[n][1] - mref[0]);
            const float p2 = fast_exp2(sacc[n][2] - mref[1]);
            const float p3 = fast_exp2(sacc[n][3] - mref[1]);
            rs[0] += p0 + p1;
            rs[1] += p2 + p3;
            // A operand of P.V for token k-step n/2: a0/a1 from n-tile 2k, a2/a3 from 2k+1
            pa[n >> 1][(n & 1) * 2 + 0] = pack_half2(p0, p1);
            pa[n >> 1][(n & 1) * 2 + 1] = pack_half2(p2, p3);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) l[r] = l[r] * alpha[r] + rs[r];
#pragma unroll
        for (int j = 0; j < ON; ++j) {
            o[j][0] *= alpha[0];
            o[j][1] *= alpha[0];
            o[j][2] *= alpha[1];
            o[j][3] *= alpha[1];
        }

        // ---- O += P V
        // b[0] and b[2] hold tokens kt2*16 + c, c + 1 (low, high half); b[1]
        // and b[3] the same + 8. In the sequence's last tile, halves of
        // tokens >= vlim are cleared.
        const bool tail = tb + B > vlim;
#pragma unroll
        for (int kt2 = 0; kt2 < NT / 2; ++kt2) {
            uint32_t keep[2] = {0xffffffffu, 0xffffffffu};
            if (tail) {
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int t = tb + kt2 * 16 + 8 * hi + c;
                    keep[hi] = (t < vlim ? 0x0000ffffu : 0u) | (t + 1 < vlim ? 0xffff0000u : 0u);
                }
            }
#pragma unroll
            for (int dp = 0; dp < ON / 2; ++dp) {
                // matrices (transposed): (tokens +0..7, dims +0..7), (+8..15, +0..7), (+0..7, +8..15), (+8..15, +8..15)
                const int mi = lane >> 3, r = lane & 7;
                const int tok = kt2 * 16 + ((mi & 1) << 3) + r;
                const int dim = dp * 16 + ((mi >> 1) << 3);
                const unsigned char *addr = vt + (dim >> 6) * kHalfTile + swz128(tok, (dim & 63) * 2);
                uint32_t b[4];
                ldmatrix_x4_trans(b, addr);
                mma_16816(o[2 * dp], pa[kt2], b[0] & keep[0], b[1] & keep[1]);
                mma_16816(o[2 * dp + 1], pa[kt2], b[2] & keep[0], b[3] & keep[1]);
            }
        }
    }

    // Row sums over the quad that shares each row (after the last tile).
    __device__ __forceinline__ void reduce_l() {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
            l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
        }
    }
};

// Shared-prefix attention on tensor cores (fp16 caches). One CTA = one head
// x one prefix partition x up to 64 sequences; consumer warp w takes the 16
// sequences 16w .. 16w+15 of the CTA's block (MmaRows above). The producer
// streams the shared blocks' K and V tiles (64-dim halves, 128-byte swizzle)
// through a ring; after the last tile the partition's partial (lse, o) of
// each sequence is written.
constexpr int kPrefixMmaQueries = 64;  // sequences per CTA (4 warps x 16)

template <int D, int B>
struct PrefixMmaLayout {
    static constexpr int kHalves = D / 64;              // 64-dim half tiles per row
    static constexpr int kHalfTile = B * 128;            // bytes of one half tile
    static constexpr int kTile = kHalves * kHalfTile;    // one K (or V) tile
    static constexpr int kStage = 2 * kTile;
};

template <int D, int B>
__global__ void __launch_bounds__(32 * 5, 1)
paged_prefix_mma_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
    using Lay = PrefixMmaLayout<D, B>;
    constexpr int ON = D / 8;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 128-byte-swizzled TMA destinations must be 1024-byte aligned: align the
    // ring explicitly (the launch adds 1 KiB of slack).
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int stages = p.stages;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)stages * Lay::kStage);
    uint64_t *empty = full + stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.num_seqs;
    const int n_qb = (S + kPrefixMmaQueries - 1) / kPrefixMmaQueries;
    const int qb = blockIdx.x % n_qb;
    const int rest = blockIdx.x / n_qb;
    const int pp = rest % p.prefix_parts;
    const int h = rest / p.prefix_parts;
    const int q_base = qb * kPrefixMmaQueries;
    const int n_consumers = min(4, (S - q_base + 15) / 16);
    const int t0 = pp * p.prefix_partition;
    const int t1 = min(p.prefix_tokens, t0 + p.prefix_partition);
    const int blk0 = t0 / B;
    const int nblk = (t1 - t0 + B - 1) / B;

    if (warp == n_consumers) {
        // ---------------------------------------------------------- producer
        int pre = 0;
        if (lane < nblk) pre = __ldg(p.block_tables + blk0 + lane);  // row 0 holds the shared blocks
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
        const uint64_t policy = l2_policy_evict_first();
        bool ok = true;
        for (int i = 0; i < nblk && ok; ++i) {
            if (i > 0 && (i & 31) == 0) {
                pre = 0;
                if (i + lane < nblk) pre = __ldg(p.block_tables + blk0 + i + lane);
            }
            int blk = __shfl_sync(0xffffffffu, pre, i & 31);
            const bool bad = blk < 0 || blk >= p.num_blocks;
            if (bad) blk = p.num_blocks;
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
    const int g = lane >> 2;          // fragment row (and row + 8)
    const int c = (lane & 3) * 2;     // fragment column pair
    const int q0 = q_base + warp * 16;
    const int rows[2] = {q0 + g, q0 + g + 8};
    int lim[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        int L = 0;
        if (rows[r] < S) {
            L = __ldg(p.context_lens + rows[r]);
            L = min(L, p.max_blocks_per_seq * B);
            L = max(min(L, p.max_context_len), 0);
        }
        lim[r] = min(L, t1);  // this row's tokens end here (within the partition)
    }
    MmaRows<D, B> mr;
    mr.load_q(rows[0] < S ? p.query + ((size_t)rows[0] * p.num_heads + h) * D : nullptr,
              rows[1] < S ? p.query + ((size_t)rows[1] * p.num_heads + h) * D : nullptr, p.qk_scale_log2,
              lane);
    asm volatile("bar.sync 1, %0;" ::"r"((n_consumers + 1) * 32) : "memory");

    for (int i = 0; i < nblk; ++i) {
        const int st = i % stages, use = i / stages;
        if (!mbar_wait(&full[st], use & 1)) break;
        const unsigned char *kt = smem + (size_t)st * Lay::kStage;
        mr.attend(kt, kt + Lay::kTile, t0 + i * B, lim, t1, lane);  // shared blocks are full
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }

    // ---- partials: (lse, o) per sequence
    mr.reduce_l();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (rows[r] >= S) continue;
        const size_t idx = ((size_t)rows[r] * p.num_heads + h) * p.ws_parts + pp;
        const bool any = mr.l[r] > 0.f;
        const float inv = any ? 1.0f / mr.l[r] : 0.f;
        float *op = p.ws_o + idx * D;
#pragma unroll
        for (int j = 0; j < ON; ++j)
            *reinterpret_cast<float2 *>(op + j * 8 + c) =
                make_float2(mr.o[j][2 * r] * inv, mr.o[j][2 * r + 1] * inv);
        if ((lane & 3) == 0) p.ws_lse[idx] = any ? mr.m[r] + fast_log2(mr.l[r]) : -INFINITY;
    }
}

}  // namespace pa
