/*
 * pagedkv.h -- C ABI of libpagedkv.so: paged-KV decode attention for NVIDIA
 * B200 (sm_100a), with the cache-write scatter, the slot derivation and the
 * block copy that surround it, block swap to pinned host memory, and the
 * paged prefill of a prompt or chunk.
 *
 * Sources (each page is cited by its title and section):
 *   [P1] "vLLM-v0.17.1技术解析：PagedAttention内存管理与显存优化技巧",
 *        §2.2 PagedAttention的创新设计 (block table, physical block pool),
 *        §3.2 高效CUDA内核优化 (fused kernels, coalesced access), §3.3 量化支持 (FP8).
 *   [P2] "在A10G上榨干LLaMA-7B：vLLM与PagedAttention实战",
 *        §2.1 从逻辑块到物理块 (logical/physical blocks, growth on append),
 *        §2.2 内存共享与写时复制 (prefix sharing, copy-on-write).
 *   [P3] KV-cache / PagedAttention article at l189.com/news/180929,
 *        §2.1 块状存储结构 (16-token blocks, per-block byte size),
 *        §2.2 槽位映射机制 (slot mapping: one int32 per token),
 *        §4 (FP8 KV cache, block size 32 for long texts).
 *
 * Conventions shared by every call
 *   - All data pointers are DEVICE pointers owned by the caller, on the
 *     current CUDA device. The library never frees or retains them.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call
 *     only enqueues work on that stream and returns; none synchronises,
 *     except pa_check_status.
 *   - Return value: PA_OK (0) or a negative PA_ERR_* code. On an error no
 *     kernel has been launched, and pa_last_error() returns a message
 *     (thread-local, valid until the next call on the same thread).
 *   - Index contents that only the device can see (slots, block ids,
 *     context lengths, copy pairs) are bounds-checked in the kernels: an
 *     offending item is skipped or clamped, never dereferenced, and a bit is
 *     set in a per-device error word that pa_check_status reads and clears.
 *   - KV cache layout (both K and V): contiguous
 *     [num_blocks][block_size][num_heads][head_size] of fp16 or of E4M3 codes
 *     ([P1] §2.2 physical block pool; [P3] §2.1 block of block_size tokens x
 *     num_heads x head_size). Logical token t of a sequence lives in physical
 *     block block_tables[s][t / block_size], row t % block_size.
 *   - Supported shapes: head_size 64 or 128; block_size 16 or 32;
 *     1 <= num_heads <= 65535; num_blocks * block_size < 2^31.
 *   - Query, output, new K/V rows and caches must be 16-byte aligned.
 *   - Counts: num_seqs <= 65535 per decode or prefill call; token and pair
 *     counts of the cache write, block copy and swap have no such limit (the
 *     library launches them in slices of 65535, in stream order).
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_OK 0
#define PA_ERR_INVALID (-1)   /* null pointer, bad size, shape or alignment */
#define PA_ERR_DTYPE (-2)     /* unsupported cache dtype */
#define PA_ERR_OVERFLOW (-3)  /* num_blocks * block_size >= 2^31 */
#define PA_ERR_CUDA (-4)      /* a CUDA runtime or driver call failed */
#define PA_ERR_WORKSPACE (-5) /* caller workspace missing, too small or misaligned */

/* Bits of the device error word (pa_check_status). */
#define PA_DEV_BAD_SLOT 1u        /* slot >= num_blocks*block_size: token skipped */
#define PA_DEV_BAD_BLOCK 2u       /* table entry outside [0, num_blocks): rows read as zeros */
#define PA_DEV_CTX_OVER_TABLE 4u  /* context_len > max_blocks_per_seq*block_size: clamped */
#define PA_DEV_CTX_OVER_BOUND 8u  /* context_len > max_context_len given to the call: clamped */
#define PA_DEV_BAD_PAIR 16u       /* copy pair index outside [0, num_blocks): pair skipped */
#define PA_DEV_WAIT_TIMEOUT 32u   /* an on-chip pipeline wait ran out (never expected) */
#define PA_DEV_PREFIX 64u         /* shared-prefix contract broken (see ..._shared_prefix) */
#define PA_DEV_BAD_CHUNK 128u     /* prefill chunk longer than its context (or than
                                     max_query_len given to pa_paged_prefill), or
                                     rows outside [0, total_q): skipped */

/* KV cache element type: fp16, or OCP FP8 E4M3 ("fn" variant: no infinities,
 * max 448) with one fp32 scale per cache tensor ([P1] §3.3, [P3] §4). */
#define PA_F16 0
#define PA_E4M3 1

typedef struct {
    int32_t num_blocks;   /* physical blocks in the pool */
    int32_t block_size;   /* tokens per block: 16 or 32 */
    int32_t num_heads;    /* KV heads (= query heads) */
    int32_t head_size;    /* 64 or 128 */
    int32_t dtype;        /* PA_F16 or PA_E4M3 */
} pa_cache_desc;

/* Launch shape of the decode. Any field 0 = library choice.
 *   partition_size: tokens per split-context partition, a multiple of
 *       block_size. Sequences longer than one partition are computed as
 *       partial results plus a log-sum-exp reduction.
 *   heads_per_cta:  1, 2, 4 or 8 and a divisor of num_heads.
 *   warps_per_head: 1, 2 or 4 warps sharing one head's tokens in a CTA.
 *   stages:         2..8 K/V tiles in flight per work unit, a multiple of
 *                   warps_per_head.
 *   units_per_cta:  1..4 work units (sequence x head group x partition) that
 *                   one CTA serves, each with its own ring of stages;
 *                   units_per_cta * heads_per_cta * warps_per_head <= 16. */
typedef struct {
    int32_t partition_size;
    int32_t heads_per_cta;
    int32_t warps_per_head;
    int32_t stages;
    int32_t units_per_cta;
} pa_decode_config;

/* Library version: 100 * minor + patch for 0.minor.patch (202 = 0.2.2: the
 * paged prefill calls take total_q since 0.2.1; the decode sums exact
 * fp16 products in fp32 for both cache types, and pa_test_stall_next_decode
 * exists, since 0.2.2). */
int pa_version(void);

/* Message for the last nonzero status returned on this thread ("" if none). */
const char *pa_last_error(void);

/* Synchronise `stream`, then read and clear the device error word of the
 * current device into *code (0 = no device-side error since the last read).
 * Returns PA_OK or PA_ERR_CUDA. */
int pa_check_status(void *stream, uint32_t *code);

/* Test hook for the bounded on-chip waits (the pages have no counterpart:
 * it exists so that a test can make one wait run out on purpose). The next
 * decode this thread launches (pa_paged_attention_decode, _ws, _append,
 * _shared_prefix or _noalloc) issues no tile loads for the work unit that
 * holds head `head` of sequence `seq` in context partition `partition`
 * (partition p covers the tokens from p * partition_size, counted after a
 * shared prefix; see pa_decode_choose_config), and gives each of its
 * pipeline waits wait_limit_ns of wall time instead of 2 s. If that unit
 * has tokens, its consumer warps give up at the limit, set
 * PA_DEV_WAIT_TIMEOUT and return; its output rows are then undefined,
 * everything else is computed as usual, and no copy or wait is left
 * pending. A unit without tokens, or a (seq, head, partition) outside the
 * launch, stalls nothing. The request is consumed by the next decode
 * launch; seq < 0 clears it. Returns PA_OK, or PA_ERR_INVALID for a
 * negative head or partition or wait_limit_ns outside [1000, 2000000000]. */
int pa_test_stall_next_decode(int seq, int head, int partition, uint64_t wait_limit_ns);

/* ---------------------------------------------------------------- a1
 * Slot of the token each sequence appends in a decode step ([P3] §2.2 slot
 * mapping; [P2] §2.1 growth on append). With L = context_lens[s] (which
 * includes the appended token) and pos = L-1:
 *     slot_mapping[s] = block_tables[s][pos / block_size] * block_size
 *                       + pos % block_size
 * and -1 when L <= 0. block_tables: int32 [num_seqs][max_blocks_per_seq].
 * Device checks: L beyond the table row sets PA_DEV_CTX_OVER_TABLE, a block
 * id outside the pool sets PA_DEV_BAD_BLOCK; both give slot -1. */
int pa_slot_mapping(int32_t *slot_mapping, const int32_t *block_tables,
                    int max_blocks_per_seq, const int32_t *context_lens,
                    int num_seqs, pa_cache_desc cache, void *stream);

/* ---------------------------------------------------------------- a2
 * Store each new token's K and V rows (all heads) into the cache slot that
 * slot_mapping gives ([P2] §2.1: the new token's KV goes into the mapped
 * block; [P3] §2.2 slot mapping). key/value: fp16 [n_tokens][num_heads]
 * [head_size], row i at key + i*key_stride elements (stride a multiple of 8).
 * slot s -> block s / block_size, row s % block_size. Negative slots are
 * padding and are skipped. fp16 caches receive the bits unchanged; E4M3
 * caches receive e4m3_rn_satfinite(fp32(x) / scale) with an IEEE fp32 divide
 * (k_scale for K, v_scale for V; both ignored for fp16). Slots beyond the
 * pool set PA_DEV_BAD_SLOT and are skipped. Two tokens with the same slot in
 * one call: undefined which one lands. */
int pa_kv_cache_write(const void *key, const void *value, int64_t key_stride,
                      int64_t value_stride, void *key_cache, void *value_cache,
                      pa_cache_desc cache, const int32_t *slot_mapping,
                      int n_tokens, float k_scale, float v_scale, void *stream);

/* ---------------------------------------------------------------- a3
 * Copy-on-write block copy ([P2] §2.2): for each pair (src, dst) of
 * src_dst_pairs (int32 [n_pairs][2]), physical block dst of both caches
 * becomes a copy of block src (block_size*num_heads*head_size elements).
 * Pairs run concurrently: a dst that is also some pair's src, or that
 * appears twice, is undefined. Indices outside the pool set PA_DEV_BAD_PAIR
 * and the pair is skipped. */
int pa_copy_blocks(void *key_cache, void *value_cache, pa_cache_desc cache,
                   const int32_t *src_dst_pairs, int n_pairs, void *stream);

/* ---------------------------------------------------------------- swap
 * Block swap between two pools of the same block shape ([P1] §4.1 and
 * [P2] §5.2: --swap-space, KV blocks spilled to CPU memory and brought
 * back): for each pair (src, dst) of src_dst_pairs (int32 [n_pairs][2],
 * device memory), block dst of the destination caches becomes a copy of
 * block src of the source caches (K and V). Either pool may be device memory
 * or pinned host memory accessible from the device (cudaHostAlloc / torch
 * pin_memory under unified addressing); the kernel reaches host memory over
 * the host link. cache gives the block shape and dtype (its num_blocks is
 * not used); src_num_blocks and dst_num_blocks bound the indices (outside:
 * PA_DEV_BAD_PAIR, pair skipped). Pairs run concurrently; repeated dst
 * blocks are undefined. */
int pa_swap_blocks(void *dst_key_cache, void *dst_value_cache, int dst_num_blocks,
                   const void *src_key_cache, const void *src_value_cache, int src_num_blocks,
                   pa_cache_desc cache, const int32_t *src_dst_pairs, int n_pairs, void *stream);

/* ---------------------------------------------------------------- a4..a9
 * Decode attention of one query token per sequence over its cached K/V,
 * read through its block table ([P1] §2.2; [P2] §2.1). For each sequence s
 * and head h, with L = context_lens[s] and token t in physical block
 * block_tables[s][t / block_size], row t % block_size:
 *     z_t = scale * k_scale * sum_d q[s,h,d] * K_t[h,d]
 *     out[s,h,:] = v_scale * sum_t softmax(z)_t * V_t[h,:]       (t < L)
 * (k_scale, v_scale only for E4M3 caches, which hold K/k_scale, V/v_scale).
 * L = 0 gives zeros. query, out: fp16 [num_seqs][num_heads][head_size].
 * Arithmetic: each product q*K and p*V is formed exactly (fp16 x fp16, the
 * query as given, K/V as stored: fp16, or E4M3 codes decoded exactly) and
 * summed in fp32; the scales are applied to the fp32 sums. Softmax weights
 * are rounded to fp16 (relative error <= 2^-12) and the same rounded
 * weights form both the numerator and the denominator, so each output row
 * is a convex combination of V rows. No input range limit beyond fp32's.
 * max_context_len: a host-known upper bound on every context length (e.g.
 * max_blocks_per_seq*block_size); it sizes the split-context grid. Contexts
 * above it or above the table row are clamped and flagged.
 * Sequences longer than the partition size are split: each partition writes
 * a normalised partial output and its log-sum-exp, and a second kernel
 * combines them. The workspace for those partials is owned by the library:
 * one buffer per (device, stream), grown with cudaMallocAsync on `stream`
 * and never shrunk; an outgrown buffer is kept (not freed), so a CUDA graph
 * captured before the growth still replays into valid memory. It is not allocated when no sequence can span more than
 * one partition. Issue a first call with the largest shapes before
 * capturing a CUDA graph so that capture does not need to grow it. */
int pa_paged_attention_decode(void *out, const void *query,
                              const void *key_cache, const void *value_cache,
                              pa_cache_desc cache, const int32_t *block_tables,
                              int max_blocks_per_seq, const int32_t *context_lens,
                              int num_seqs, int max_context_len, float scale,
                              float k_scale, float v_scale, void *stream);

/* Fill *cfg with the launch shape the library would use (fields given as
 * nonzero are kept and validated). Returns PA_OK or PA_ERR_INVALID. */
int pa_decode_choose_config(pa_cache_desc cache, int num_seqs, int max_context_len,
                            pa_decode_config *cfg);

/* Bytes of workspace a pa_paged_attention_decode_ws call with this shape
 * and config needs (0 when no split is possible). cfg may be NULL (library
 * choice). Layout, when nonzero: float lse[num_seqs][num_heads][P] (base-2
 * log-sum-exp of each partition's logits, in units of z*log2(e)), then at
 * the next 256-byte boundary float o[num_seqs][num_heads][P][head_size]
 * (each partition's softmax-normalised output, before v_scale), with
 * P = ceil(max_context_len / partition_size). Entries of partitions that a
 * sequence does not have are left untouched. */
size_t pa_decode_workspace_size(pa_cache_desc cache, int num_seqs, int max_context_len,
                                const pa_decode_config *cfg);

/* pa_paged_attention_decode with an explicit launch shape (cfg may be NULL)
 * and a caller-owned workspace of at least pa_decode_workspace_size bytes,
 * 256-byte aligned (may be NULL when that size is 0). Allocates nothing. */
int pa_paged_attention_decode_ws(void *out, const void *query,
                                 const void *key_cache, const void *value_cache,
                                 pa_cache_desc cache, const int32_t *block_tables,
                                 int max_blocks_per_seq, const int32_t *context_lens,
                                 int num_seqs, int max_context_len, float scale,
                                 float k_scale, float v_scale,
                                 const pa_decode_config *cfg, void *workspace,
                                 size_t workspace_bytes, void *stream);

/* Fused append + decode ([P1] §3.2 fused kernels): one launch (plus the
 * log-sum-exp reduce when a context is split) performs, for every sequence,
 * the slot derivation of pa_slot_mapping, the store of pa_kv_cache_write for
 * its new token (fp16 copy or E4M3 encode with k_scale/v_scale), and the
 * decode of pa_paged_attention_decode over all L tokens including the new
 * one. The CTA that owns a sequence's last partition stores the new rows of
 * its heads before it loads the block holding them.
 *   new_key/new_value: fp16 [num_seqs][num_heads][head_size], row stride
 *       key_stride/value_stride elements (multiples of 8), 16-byte aligned.
 *   slot_mapping_out: int32 [num_seqs] receiving each sequence's slot (-1
 *       when L <= 0, the context is clamped, or the block id is invalid), or
 *       NULL. Sequences with L <= 0 write nothing.
 *   cfg / workspace: as in pa_paged_attention_decode_ws; workspace NULL =
 *       the library-owned workspace of pa_paged_attention_decode.
 * Results equal pa_slot_mapping + pa_kv_cache_write + the decode, in order. */
int pa_paged_attention_decode_append(void *out, const void *query, const void *new_key,
                                     const void *new_value, int64_t key_stride,
                                     int64_t value_stride, void *key_cache, void *value_cache,
                                     pa_cache_desc cache, const int32_t *block_tables,
                                     int max_blocks_per_seq, const int32_t *context_lens,
                                     int num_seqs, int max_context_len, float scale,
                                     float k_scale, float v_scale, int32_t *slot_mapping_out,
                                     const pa_decode_config *cfg, void *workspace,
                                     size_t workspace_bytes, void *stream);

/* Decode (optionally with the fused append) for a batch whose sequences all
 * start with the same shared_prefix_blocks physical blocks ([P2] §2.2:
 * requests with the same prompt map its logical blocks to the same physical
 * blocks). Contract: for every row s, block_tables[s][0 .. n-1] equals
 * block_tables[0][0 .. n-1] (n = shared_prefix_blocks, whole blocks); a row
 * that differs sets PA_DEV_PREFIX. Each shared tile is read once per head
 * and applied to up to 16 sequences' queries; the private rest of every
 * context is decoded as in pa_paged_attention_decode; a log-sum-exp
 * reduction merges both (three launches). The prefix kernel runs on a
 * second stream of the library's (one per device and caller stream, made
 * on the first call: make that call before any stream capture), forked
 * from `stream` after everything already queued there and joined back
 * before the reduce, so it overlaps the private-part decode while the call
 * keeps its place in the order of `stream` (a graph captured on `stream`
 * holds both branches). Results equal
 * pa_paged_attention_decode (or _append when new_key is given) on the same
 * tables. With new_key/new_value (both or neither), each sequence's new
 * token must lie after the prefix (L > n * block_size), else it is not
 * stored, its slot is -1 and PA_DEV_PREFIX is set. cfg shapes the decode of
 * the private part (NULL = library choice); workspace NULL = the library's
 * own, else at least pa_shared_prefix_workspace_size bytes, 256-aligned. */
int pa_paged_attention_decode_shared_prefix(void *out, const void *query, const void *new_key,
                                            const void *new_value, int64_t key_stride,
                                            int64_t value_stride, void *key_cache,
                                            void *value_cache, pa_cache_desc cache,
                                            const int32_t *block_tables, int max_blocks_per_seq,
                                            const int32_t *context_lens, int num_seqs,
                                            int max_context_len, int shared_prefix_blocks,
                                            float scale, float k_scale, float v_scale,
                                            int32_t *slot_mapping_out, const pa_decode_config *cfg,
                                            void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes of a pa_paged_attention_decode_shared_prefix call (0 on
 * invalid arguments). */
size_t pa_shared_prefix_workspace_size(pa_cache_desc cache, int num_seqs, int max_context_len,
                                       int shared_prefix_blocks, const pa_decode_config *cfg);

/* pa_paged_attention_decode for callers that cannot allocate device memory.
 * The paper has no counterpart to this call: it exists for callers such as
 * engine plugins whose host framework owns all device memory, code running
 * under CUDA stream capture, or loops with a fixed memory plan, none of which
 * may call cudaMalloc or an allocating library on this path. Arguments,
 * results and errors are those of pa_paged_attention_decode (library-chosen
 * launch shape); the split partials go to a static device array of 16 MiB
 * inside the library instead of a workspace, and the call allocates nothing.
 *   - Limit: a decode whose partials exceed 16 MiB (pa_decode_workspace_size
 *     with cfg NULL) returns PA_ERR_WORKSPACE before launching anything.
 *   - The array is held by every GPU that loads the library until exit.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; nothing in it has to start at zero (each partial is written
 *     before it is read). Calls whose kernels may overlap on the GPU (other
 *     streams, other threads) race on it: serialise them. */
int pa_paged_attention_decode_noalloc(void *out, const void *query,
                                      const void *key_cache, const void *value_cache,
                                      pa_cache_desc cache, const int32_t *block_tables,
                                      int max_blocks_per_seq, const int32_t *context_lens,
                                      int num_seqs, int max_context_len, float scale,
                                      float k_scale, float v_scale, void *stream);

/* ------------------------------------------------------- paged prefill
 * Prompt (or chunked-prompt) attention over the block table. [P1] §3.2 puts
 * FlashAttention-style attention on the kernel path; [P3] §4 runs long
 * texts (over 4k tokens) with 32-token blocks. The pages print no formula;
 * the reading used is causal attention at each row's position:
 *   sequence s brings n_s = query_start[s+1] - query_start[s] new tokens,
 *   the last n_s positions of its context of L_s = context_lens[s] tokens
 *   (0 <= n_s <= L_s); token query_start[s] + i sits at position
 *   L_s - n_s + i.
 * query_start: int32 [num_seqs + 1], non-decreasing, query_start[0] = 0
 * (device). A full prompt has n_s = L_s; a chunk after cached context has
 * n_s < L_s; n_s = 1 is a decode step.
 * total_q: the rows the caller allocated for the chunk's tokens (query, out,
 * slot_mapping), normally query_start[num_seqs]. A sequence whose rows do
 * not lie inside [0, total_q) (query_start negative, decreasing or past
 * total_q) is touched nowhere and sets PA_DEV_BAD_CHUNK; total_q = 0 is a
 * no-op. */

/* Slot of every new token of the chunk ([P3] §2.2 slot mapping, at each
 * token's position):
 *     slot_mapping[query_start[s] + i] = block_tables[s][pos / block_size]
 *                                        * block_size + pos % block_size,
 *     pos = L_s - n_s + i
 * max_query_len is a sizing hint (any n_s is covered). Device checks: a
 * chunk with n_s > L_s sets PA_DEV_BAD_CHUNK and gets slots -1; a position
 * beyond the table row sets PA_DEV_CTX_OVER_TABLE, a block id outside the
 * pool PA_DEV_BAD_BLOCK; both give slot -1. With pa_kv_cache_write these
 * slots store the chunk's K/V before pa_paged_prefill reads them. */
int pa_prefill_slot_mapping(int32_t *slot_mapping, const int32_t *query_start,
                            const int32_t *block_tables, int max_blocks_per_seq,
                            const int32_t *context_lens, int num_seqs, int total_q,
                            int max_query_len, pa_cache_desc cache, void *stream);

/* Causal attention of packed query rows over the paged cache:
 *   out[r][h] = sum_{t <= pos(r)} softmax_t(scale * q[r][h] . K_t[h]) V_t[h]
 * for every row r = query_start[s] + i (pos(r) = L_s - n_s + i) and head h.
 * query, out: fp16 [total_q][num_heads][head_size], total_q =
 * query_start[num_seqs]; the cache must already hold all L_s tokens of each
 * sequence (the chunk's own K/V included). fp16 caches only (PA_ERR_DTYPE
 * for E4M3). max_query_len: a host-known bound on every n_s (the grid is
 * sized from it). Computed on tensor cores: Q.K^T and P.V in fp16 x fp16 ->
 * fp32, softmax in fp32 with P rounded to fp16; a positive scale runs
 * tcgen05.mma over 128-row tiles with S and O in tensor memory, a scale
 * <= 0 the warp-level mma.m16n8k16 over 64-row tiles.
 * Device checks: n_s > L_s or n_s > max_query_len sets PA_DEV_BAD_CHUNK,
 * L_s beyond the table row PA_DEV_CTX_OVER_TABLE; such a sequence's rows
 * are not written. Block ids outside the pool read as zeros and set
 * PA_DEV_BAD_BLOCK. One launch; no workspace. */
int pa_paged_prefill(void *out, const void *query, const int32_t *query_start,
                     const void *key_cache, const void *value_cache, pa_cache_desc cache,
                     const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *context_lens, int num_seqs, int total_q, int max_query_len,
                     float scale, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
