// pa_cache_ops.cuh -- slot derivation, cache-write scatter and block copy.
//
// Slot mapping ("槽位映射机制", §2.2 of the l189.com/news/180929 article): each
// token has one int32 slot = physical_block * block_size + row. The token a
// decode step appends sits at position L-1 ("在A10G上榨干LLaMA-7B" §2.1: it goes
// into the last block while that block has room, else into a newly mapped
// one). Copy-on-write ("在A10G上榨干LLaMA-7B" §2.2) copies a whole physical block.
#pragma once

#include "pa_device.cuh"

namespace pa {

// a1: one thread per sequence.
__global__ void slot_mapping_kernel(int32_t *__restrict__ slot_mapping,
                                    const int32_t *__restrict__ block_tables,
                                    int max_blocks_per_seq, const int32_t *__restrict__ context_lens,
                                    int num_seqs, int block_size, int num_blocks) {
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= num_seqs) return;
    const int L = context_lens[s];
    int slot = -1;
    if (L > 0) {
        const int pos = L - 1;
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
    slot_mapping[s] = slot;
}

// a2: grid (chunks of the row, tokens). Each thread moves one 16-byte chunk
// (8 fp16 elements) of the token's K row and of its V row. fp16 caches store
// the chunk unchanged; E4M3 caches store 8 codes e4m3(fp32(x) / scale) with
// an IEEE-rounded fp32 divide (__fdiv_rn), round to nearest even and
// saturation to +/-448.
template <bool kFp8>
__global__ void __launch_bounds__(128)
kv_cache_write_kernel(const __half *__restrict__ key, const __half *__restrict__ value,
                      int64_t key_stride, int64_t value_stride, void *__restrict__ key_cache,
                      void *__restrict__ value_cache, const int32_t *__restrict__ slot_mapping,
                      int row_elems, int64_t pool_slots, float k_scale, float v_scale) {
    const int i = blockIdx.y;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;  // chunk of 8 elements
    if (c * 8 >= row_elems) return;
    const int32_t slot = slot_mapping[i];
    if (slot < 0) return;
    if ((int64_t)slot >= pool_slots) {
        if (c == 0) flag_error(PA_DEV_BAD_SLOT);
        return;
    }
    const uint4 kraw = __ldg(reinterpret_cast<const uint4 *>(key + (size_t)i * key_stride) + c);
    const uint4 vraw = __ldg(reinterpret_cast<const uint4 *>(value + (size_t)i * value_stride) + c);
    const size_t dst = (size_t)slot * row_elems + (size_t)c * 8;
    if constexpr (!kFp8) {
        reinterpret_cast<uint4 *>(static_cast<__half *>(key_cache) + dst)[0] = kraw;
        reinterpret_cast<uint4 *>(static_cast<__half *>(value_cache) + dst)[0] = vraw;
    } else {
        const uint2 kq = encode8_e4m3(kraw, k_scale);
        const uint2 vq = encode8_e4m3(vraw, v_scale);
        reinterpret_cast<uint2 *>(static_cast<uint8_t *>(key_cache) + dst)[0] = kq;
        reinterpret_cast<uint2 *>(static_cast<uint8_t *>(value_cache) + dst)[0] = vq;
    }
}

// a3: grid (chunks of a block, pairs, 2 caches). Each thread copies
// kCopyVecs 16-byte vectors, all loads issued before the stores.
constexpr int kCopyThreads = 256;
constexpr int kCopyVecs = 4;

__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_kernel(void *__restrict__ key_cache, void *__restrict__ value_cache,
                   const int32_t *__restrict__ pairs, int64_t block_vecs, int num_blocks) {
    const int pr = blockIdx.y;
    const int32_t src = pairs[2 * pr];
    const int32_t dst = pairs[2 * pr + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) flag_error(PA_DEV_BAD_PAIR);
        return;
    }
    uint4 *base = static_cast<uint4 *>(blockIdx.z == 0 ? key_cache : value_cache);
    const uint4 *from = base + (size_t)src * block_vecs;
    uint4 *to = base + (size_t)dst * block_vecs;
    const int64_t v0 = (int64_t)blockIdx.x * kCopyThreads * kCopyVecs + threadIdx.x;
    uint4 r[kCopyVecs];
#pragma unroll
    for (int k = 0; k < kCopyVecs; ++k) {
        const int64_t v = v0 + (int64_t)k * kCopyThreads;
        if (v < block_vecs) r[k] = from[v];
    }
#pragma unroll
    for (int k = 0; k < kCopyVecs; ++k) {
        const int64_t v = v0 + (int64_t)k * kCopyThreads;
        if (v < block_vecs) to[v] = r[k];
    }
}

// Swap (the pages' --swap-space: KV blocks spilled to and restored from CPU
// memory): grid (chunks of a block, pairs, 2 caches). Block dst of the
// destination pool becomes a copy of block src of the source pool; either
// pool may be device memory or pinned host memory mapped into the device's
// address space, which the loads or stores then reach over the host link.
__global__ void __launch_bounds__(kCopyThreads)
swap_blocks_kernel(void *__restrict__ dst_key, void *__restrict__ dst_value,
                   const void *__restrict__ src_key, const void *__restrict__ src_value,
                   const int32_t *__restrict__ pairs, int64_t block_vecs, int src_blocks,
                   int dst_blocks) {
    const int pr = blockIdx.y;
    const int32_t src = pairs[2 * pr];
    const int32_t dst = pairs[2 * pr + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (blockIdx.x == 0 && blockIdx.z == 0 && threadIdx.x == 0) flag_error(PA_DEV_BAD_PAIR);
        return;
    }
    const uint4 *from = static_cast<const uint4 *>(blockIdx.z == 0 ? src_key : src_value) +
                        (size_t)src * block_vecs;
    uint4 *to = static_cast<uint4 *>(blockIdx.z == 0 ? dst_key : dst_value) + (size_t)dst * block_vecs;
    const int64_t v0 = (int64_t)blockIdx.x * kCopyThreads * kCopyVecs + threadIdx.x;
    uint4 r[kCopyVecs];
#pragma unroll
    for (int k = 0; k < kCopyVecs; ++k) {
        const int64_t v = v0 + (int64_t)k * kCopyThreads;
        if (v < block_vecs) r[k] = from[v];
    }
#pragma unroll
    for (int k = 0; k < kCopyVecs; ++k) {
        const int64_t v = v0 + (int64_t)k * kCopyThreads;
        if (v < block_vecs) to[v] = r[k];
    }
}

}  // namespace pa
