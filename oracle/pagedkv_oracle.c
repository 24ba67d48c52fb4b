/*
 * pagedkv_oracle.c -- plain, slow, scalar CPU oracle for the paged-KV decode path
 * and the paged prefill.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load this file's shared library. The CUDA
 * library never links, includes or calls it, and it includes nothing of the
 * CUDA library: the two share no code.
 *
 * Every floating-point result is computed in double precision with no
 * blocking, fusion or reordering beyond what the definitions below state.
 * The two parallel entries only hand independent work to OpenMP threads:
 * oracle_paged_attention_threads whole (sequence, head) pairs, and
 * oracle_kv_cache_write_threads the elements of one token row at a time
 * (tokens in order). Each item runs the same serial code, so their results
 * equal the single-thread calls' bit for bit.
 * Sources (each page is cited by its title and section):
 *   [P1] "vLLM-v0.17.1技术解析：PagedAttention内存管理与显存优化技巧"
 *        (cnnetsun.cn/a/1550967), §2.2 PagedAttention的创新设计: block table +
 *        physical block pool; §3.3 量化支持: FP8.
 *   [P2] "在A10G上榨干LLaMA-7B：vLLM与PagedAttention实战" (devpress.csdn.net),
 *        §2.1 从逻辑块到物理块 (logical block -> physical block, growth);
 *        §2.2 内存共享与写时复制 (prefix sharing, copy-on-write).
 *   [P3] KV-cache / PagedAttention article (l189.com/news/180929),
 *        §2.1 块状存储结构 (16-token blocks, [block, token, head, dim] sizes);
 *        §2.2 槽位映射机制 (slot mapping, int32 per token); §4 FP8 KV cache.
 * The pages state no attention formula. What the decode computes is taken
 * as the plain definition of single-query scaled-dot-product attention over
 * the tokens that the block table addresses (softmax over all positions
 * 0..L-1, no causal mask beyond L, no bias).
 *
 * Pins (checked by tests that do not use this code's own formulas): the
 * worked slot example of [P3] §2.2, dense-attention equality on identity
 * tables against torch's CPU scaled_dot_product_attention, physical-block
 * permutation invariance, L=1 => V, equal keys / scale 0 => mean of V,
 * brute force with exact summation on tiny inputs, convexity bounds, the
 * log-sum-exp identity for partitions, an independent table-driven E4M3
 * encoder plus torch's float8_e4m3fn cast, E4M3 ties to the even code, E4M3
 * caches against fp16 caches of their decoded values at distinct K and V
 * scales, the printed per-block byte size ([P3] §2.1), and for the prefill
 * the worked slot example as a full prompt, one-token chunks against the
 * decode slots, and torch's SDPA with a causal / position mask.
 */
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F16 0
#define ORACLE_E4M3 1

/* Threads an OpenMP region of this library uses by default (1 in a build
 * without OpenMP, where the threaded calls run on the calling thread). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- numbers */

/* IEEE 754 binary16 -> double, exact: 1 sign bit, 5 exponent bits (bias 15),
 * 10 fraction bits; exponent 0 is subnormal, exponent 31 is inf/NaN. */
double oracle_f16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);              /* f * 2^-10 * 2^(1-15) */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);  /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* OCP 8-bit floating point, E4M3 ("fn": finite + NaN only) -> double, exact:
 * 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0 is
 * subnormal (m * 2^-9); S.1111.111 is NaN; there are no infinities; the
 * largest finite magnitude is S.1111.110 = 448. */
double oracle_e4m3_to_double(uint8_t c)
{
    int sign = c >> 7;
    int e = (c >> 3) & 0xf;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);               /* m/8 * 2^(1-7) */
    else
        v = ldexp((double)(8 + m), e - 10);     /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* float -> E4M3 with round-to-nearest-even and saturation of finite (and
 * infinite) magnitudes to 448; NaN -> the NaN code with the input's sign.
 * Written from the format definition: find the quantum (spacing of codes)
 * for the magnitude's binade, round |x|/quantum to an integer with ties to
 * even, and re-encode (a carry into the next binade is handled). */
uint8_t oracle_e4m3_from_float(float xf)
{
    double x = (double)xf; /* exact */
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    if (isnan(x))
        return sign | 0x7f;
    double a = fabs(x);
    if (a >= 448.0)
        return sign | 0x7e;
    if (a == 0.0)
        return sign;
    int e2;
    frexp(a, &e2);          /* a = f * 2^e2 with f in [0.5, 1): 2^(e2-1) <= a < 2^e2 */
    int E = e2 - 1;         /* binade: 2^E <= a < 2^(E+1) */
    if (E < -6)
        E = -6;             /* below 2^-6 the spacing stays 2^-9 (subnormals) */
    double quantum = ldexp(1.0, E - 3);
    double n = nearbyint(a / quantum); /* exact quotient; default mode rounds half to even */
    if (n < 8.0)                       /* only reachable in the subnormal binade */
        return sign | (uint8_t)n;
    if (n >= 16.0) {                   /* rounded up into the next binade */
        n = 8.0;
        E += 1;
    }
    int field = E + 7;
    int man = (int)n - 8;
    if (field > 15 || (field == 15 && man == 7))
        return sign | 0x7e;            /* cannot happen for a < 448; kept as a guard */
    return sign | (uint8_t)((field << 3) | man);
}

/* ----------------------------------------------------- slot mapping (a1) */

/* [P3] §2.2 maps each token of a sequence to a slot of a physical block
 * (tokens 0-15 of sequence A -> block 5, tokens 16-31 -> block 8). Reading
 * used here: slot = physical_block * block_size + offset, where the physical
 * block is block_tables[s][pos / block_size] and offset = pos % block_size.
 * The token being appended in a decode step sits at position L-1, where L
 * is the context length including that token ([P2] §2.1: the new token goes
 * into the last logical block while it has room, else into a newly mapped
 * block). L <= 0 gives slot -1 (nothing to write). Returns 0, or -1 if a
 * table read would fall outside the table row. */
int oracle_slot_mapping(int32_t *slot_mapping, const int32_t *block_tables,
                        int max_blocks_per_seq, const int32_t *context_lens,
                        int num_seqs, int block_size)
{
    for (int s = 0; s < num_seqs; ++s) {
        int L = context_lens[s];
        if (L <= 0) {
            slot_mapping[s] = -1;
            continue;
        }
        int pos = L - 1;
        int logical = pos / block_size;
        if (logical >= max_blocks_per_seq)
            return -1;
        int physical = block_tables[(int64_t)s * max_blocks_per_seq + logical];
        slot_mapping[s] = physical * block_size + pos % block_size;
    }
    return 0;
}

/* Slots of a prefill chunk. Sequence s brings n_s = query_start[s+1] -
 * query_start[s] new tokens, the last n_s positions of its context of
 * L_s = context_lens[s] tokens: token query_start[s] + i sits at position
 * L_s - n_s + i and gets slot block_tables[s][pos / block_size] * block_size
 * + pos % block_size, the same rule as above. A full prompt (n_s = L_s)
 * maps positions 0 .. L_s - 1; a decode step (n_s = 1) maps position L_s - 1.
 * Returns 0, or -1 if n_s < 0, n_s > L_s, or a table read would fall
 * outside the table row. */
int oracle_prefill_slot_mapping(int32_t *slot_mapping, const int32_t *query_start,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *context_lens, int num_seqs,
                                int block_size)
{
    for (int s = 0; s < num_seqs; ++s) {
        int n = query_start[s + 1] - query_start[s];
        int L = context_lens[s];
        if (n < 0 || n > L)
            return -1;
        for (int i = 0; i < n; ++i) {
            int pos = L - n + i;
            int logical = pos / block_size;
            if (logical >= max_blocks_per_seq)
                return -1;
            int physical = block_tables[(int64_t)s * max_blocks_per_seq + logical];
            slot_mapping[query_start[s] + i] = physical * block_size + pos % block_size;
        }
    }
    return 0;
}

/* ----------------------------------------------------- cache write (a2) */

/* Store token i's key and value rows (all heads) into the cache slot given
 * by slot_mapping[i]: cache layout is [num_blocks][block_size][num_heads]
 * [head_size], slot -> (slot / block_size, slot % block_size). Negative
 * slots are padding and are skipped. fp16 caches take the bits unchanged;
 * E4M3 caches take e4m3(fp32(x) / scale), with an IEEE fp32 divide.
 * key/value are fp16 bits, row i at key + i*key_stride (elements).
 * Returns 0, or -1 if a slot is beyond the pool (nothing after it is written). */
/* Element j of token i's key and value rows into cache row `base`. */
static void write_element(const uint16_t *key, const uint16_t *value,
                          int64_t key_stride, int64_t value_stride,
                          void *key_cache, void *value_cache, int kv_dtype,
                          int i, int64_t base, int64_t j, float k_scale, float v_scale)
{
    uint16_t kb = key[(int64_t)i * key_stride + j];
    uint16_t vb = value[(int64_t)i * value_stride + j];
    if (kv_dtype == ORACLE_F16) {
        ((uint16_t *)key_cache)[base + j] = kb;
        ((uint16_t *)value_cache)[base + j] = vb;
    } else {
        float kf = (float)oracle_f16_to_double(kb);
        float vf = (float)oracle_f16_to_double(vb);
        float kq = kf / k_scale;
        float vq = vf / v_scale;
        ((uint8_t *)key_cache)[base + j] = oracle_e4m3_from_float(kq);
        ((uint8_t *)value_cache)[base + j] = oracle_e4m3_from_float(vq);
    }
}

int oracle_kv_cache_write(const uint16_t *key, const uint16_t *value,
                          int64_t key_stride, int64_t value_stride,
                          void *key_cache, void *value_cache, int kv_dtype,
                          int num_blocks, int block_size, int num_heads,
                          int head_size, const int32_t *slot_mapping,
                          int n_tokens, float k_scale, float v_scale)
{
    int64_t row = (int64_t)num_heads * head_size;
    for (int i = 0; i < n_tokens; ++i) {
        int32_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if ((int64_t)slot >= (int64_t)num_blocks * block_size)
            return -1;
        int64_t blk = slot / block_size;
        int64_t off = slot % block_size;
        int64_t base = (blk * block_size + off) * row;
        for (int64_t j = 0; j < row; ++j)
            write_element(key, value, key_stride, value_stride, key_cache, value_cache,
                          kv_dtype, i, base, j, k_scale, v_scale);
    }
    return 0;
}

/* The same cache write with each token's row spread over n_threads OpenMP
 * threads (n_threads <= 0: the OpenMP default). Tokens are still taken in
 * order, one after the other, so duplicate slots end as in the serial call
 * (the later token wins) and the pools are identical to its result, bit for
 * bit; a slot beyond the pool stops the write at the same token, with the
 * same status. */
int oracle_kv_cache_write_threads(const uint16_t *key, const uint16_t *value,
                                  int64_t key_stride, int64_t value_stride,
                                  void *key_cache, void *value_cache, int kv_dtype,
                                  int num_blocks, int block_size, int num_heads,
                                  int head_size, const int32_t *slot_mapping,
                                  int n_tokens, float k_scale, float v_scale, int n_threads)
{
    int64_t row = (int64_t)num_heads * head_size;
    int n_ok = n_tokens, status = 0;
    for (int i = 0; i < n_tokens; ++i)
        if (slot_mapping[i] >= 0 && (int64_t)slot_mapping[i] >= (int64_t)num_blocks * block_size) {
            n_ok = i;
            status = -1;
            break;
        }
    if (n_threads <= 0)
        n_threads = oracle_max_threads();
#pragma omp parallel num_threads(n_threads)
    for (int i = 0; i < n_ok; ++i) {
        int32_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        int64_t base = ((int64_t)(slot / block_size) * block_size + slot % block_size) * row;
#pragma omp for schedule(static)
        for (int64_t j = 0; j < row; ++j)
            write_element(key, value, key_stride, value_stride, key_cache, value_cache,
                          kv_dtype, i, base, j, k_scale, v_scale);
    }
    return status;
}

/* ----------------------------------------------------- block copy (a3) */

/* Copy-on-write ([P2] §2.2): for each (src, dst) pair in order, the whole
 * physical block dst of both caches becomes a copy of block src (all tokens,
 * all heads). block_bytes = block_size*num_heads*head_size*element bytes.
 * Returns 0, or -1 on a block index outside [0, num_blocks). */
int oracle_copy_blocks(void *key_cache, void *value_cache, int64_t block_bytes,
                       int num_blocks, const int32_t *src_dst_pairs, int n_pairs)
{
    for (int i = 0; i < n_pairs; ++i) {
        int32_t src = src_dst_pairs[2 * i];
        int32_t dst = src_dst_pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks)
            return -1;
        memmove((char *)key_cache + dst * block_bytes,
                (char *)key_cache + src * block_bytes, (size_t)block_bytes);
        memmove((char *)value_cache + dst * block_bytes,
                (char *)value_cache + src * block_bytes, (size_t)block_bytes);
    }
    return 0;
}

/* Swap ([P1] §4.1 and [P2] §5.2, --swap-space: KV blocks moved to CPU
 * memory and back): for each (src, dst) pair in order, block dst of the
 * destination pools becomes a copy of block src of the source pools.
 * Returns 0, or -1 on an index outside its pool (nothing after it is copied). */
int oracle_swap_blocks(void *dst_key, void *dst_value, int dst_num_blocks,
                       const void *src_key, const void *src_value, int src_num_blocks,
                       int64_t block_bytes, const int32_t *src_dst_pairs, int n_pairs)
{
    for (int i = 0; i < n_pairs; ++i) {
        int32_t src = src_dst_pairs[2 * i];
        int32_t dst = src_dst_pairs[2 * i + 1];
        if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks)
            return -1;
        memcpy((char *)dst_key + dst * block_bytes, (const char *)src_key + src * block_bytes,
               (size_t)block_bytes);
        memcpy((char *)dst_value + dst * block_bytes, (const char *)src_value + src * block_bytes,
               (size_t)block_bytes);
    }
    return 0;
}

/* ----------------------------------------------------- decode attention */

static double cache_value(const void *cache, int kv_dtype, int64_t idx, double scale)
{
    if (kv_dtype == ORACLE_F16)
        return oracle_f16_to_double(((const uint16_t *)cache)[idx]);
    return oracle_e4m3_to_double(((const uint8_t *)cache)[idx]) * scale;
}

/* Attention of the query row q (head_size fp16 values) over the tokens
 * [t0, t1) of sequence s, head h,
 * walked through the block table ([P1] §2.2, [P2] §2.1): token t lives in
 * physical block block_tables[s][t / block_size] at row t % block_size.
 *   z_t = scale * sum_d q[d] * K_t[d]
 *   m = max_t z_t,  w_t = exp(z_t - m),  l = sum_t w_t
 *   o[d] = sum_t w_t * V_t[d] / l
 * E4M3 caches are dequantised as code value * k_scale (K) or * v_scale (V).
 * Writes o (head_size doubles), *m_out, *l_out. Returns -1 on a table entry
 * outside [0, num_blocks) or a position beyond the table row. */
static int attend_range(double *o, double *m_out, double *l_out,
                        const uint16_t *q, const void *key_cache,
                        const void *value_cache, int kv_dtype, int num_blocks,
                        int block_size, int num_heads, int head_size,
                        const int32_t *block_tables, int max_blocks_per_seq,
                        int s, int h, int t0, int t1, double scale,
                        double k_scale, double v_scale)
{
    int n = t1 - t0;
    double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    int64_t *rowbase = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
    if (!z || !rowbase) {
        free(z);
        free(rowbase);
        return -2;
    }
    for (int t = t0; t < t1; ++t) {
        int logical = t / block_size;
        if (logical >= max_blocks_per_seq) {
            free(z);
            free(rowbase);
            return -1;
        }
        int32_t blk = block_tables[(int64_t)s * max_blocks_per_seq + logical];
        if (blk < 0 || blk >= num_blocks) {
            free(z);
            free(rowbase);
            return -1;
        }
        int64_t base = (((int64_t)blk * block_size + t % block_size) * num_heads + h) * head_size;
        rowbase[t - t0] = base;
        double dot = 0.0;
        for (int d = 0; d < head_size; ++d)
            dot += oracle_f16_to_double(q[d]) * cache_value(key_cache, kv_dtype, base + d, k_scale);
        z[t - t0] = scale * dot;
    }
    double m = -INFINITY;
    for (int i = 0; i < n; ++i)
        if (z[i] > m)
            m = z[i];
    double l = 0.0;
    for (int i = 0; i < n; ++i)
        l += exp(z[i] - m);
    for (int d = 0; d < head_size; ++d) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i)
            acc += exp(z[i] - m) * cache_value(value_cache, kv_dtype, rowbase[i] + d, v_scale);
        o[d] = acc / l;
    }
    *m_out = m;
    *l_out = l;
    free(z);
    free(rowbase);
    return 0;
}

/* Decode attention of pair i: (s, h) = seq_head[i] when seq_head is given,
 * else (i / num_heads, i % num_heads). Writes head_size doubles at
 * out + i*head_size. A sequence with context length 0 gives a zero row.
 * Returns 0, or -1 on a pair out of range or a bad table entry. */
static int attend_pair(int i, double *out, const uint16_t *query,
                       const void *key_cache, const void *value_cache,
                       int kv_dtype, int num_blocks, int block_size,
                       int num_heads, int head_size,
                       const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *context_lens, int num_seqs,
                       float scale, float k_scale, float v_scale,
                       const int32_t *seq_head)
{
    int s = seq_head ? seq_head[2 * i] : i / num_heads;
    int h = seq_head ? seq_head[2 * i + 1] : i % num_heads;
    double *o = out + (int64_t)i * head_size;
    if (s < 0 || s >= num_seqs || h < 0 || h >= num_heads)
        return -1;
    int L = context_lens[s];
    if (L <= 0) {
        for (int d = 0; d < head_size; ++d)
            o[d] = 0.0;
        return 0;
    }
    const uint16_t *q = query + ((int64_t)s * num_heads + h) * head_size;
    double m, l;
    return attend_range(o, &m, &l, q, key_cache, value_cache, kv_dtype,
                        num_blocks, block_size, num_heads, head_size,
                        block_tables, max_blocks_per_seq, s, h, 0, L,
                        (double)scale, (double)k_scale, (double)v_scale);
}

/* Decode attention for the (sequence, head) pairs listed in seq_head
 * ([n_pairs][2]), or for every pair in (s, h) order when seq_head is NULL.
 * out holds one head_size row of doubles per computed pair. Returns 0, or
 * -1 on a bad pair or table entry. */
int oracle_paged_attention(double *out, const uint16_t *query,
                           const void *key_cache, const void *value_cache,
                           int kv_dtype, int num_blocks, int block_size,
                           int num_heads, int head_size,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int num_seqs,
                           float scale, float k_scale, float v_scale,
                           const int32_t *seq_head, int n_pairs)
{
    int total = seq_head ? n_pairs : num_seqs * num_heads;
    for (int i = 0; i < total; ++i) {
        int rc = attend_pair(i, out, query, key_cache, value_cache, kv_dtype,
                             num_blocks, block_size, num_heads, head_size,
                             block_tables, max_blocks_per_seq, context_lens,
                             num_seqs, scale, k_scale, v_scale, seq_head);
        if (rc)
            return rc;
    }
    return 0;
}

/* The same computation with the (sequence, head) pairs spread over
 * n_threads OpenMP threads (n_threads <= 0: the OpenMP default). Pairs are
 * independent and each is computed by the same attend_pair as above, so the
 * result is identical, bit for bit, to oracle_paged_attention's. Returns 0,
 * or the first nonzero status of any pair (a bad pair or table entry). */
int oracle_paged_attention_threads(double *out, const uint16_t *query,
                                   const void *key_cache, const void *value_cache,
                                   int kv_dtype, int num_blocks, int block_size,
                                   int num_heads, int head_size,
                                   const int32_t *block_tables, int max_blocks_per_seq,
                                   const int32_t *context_lens, int num_seqs,
                                   float scale, float k_scale, float v_scale,
                                   const int32_t *seq_head, int n_pairs, int n_threads)
{
    int total = seq_head ? n_pairs : num_seqs * num_heads;
    int status = 0;
    if (n_threads <= 0)
        n_threads = oracle_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
    for (int i = 0; i < total; ++i) {
        int rc = attend_pair(i, out, query, key_cache, value_cache, kv_dtype,
                             num_blocks, block_size, num_heads, head_size,
                             block_tables, max_blocks_per_seq, context_lens,
                             num_seqs, scale, k_scale, v_scale, seq_head);
        if (rc) {
#pragma omp critical
            if (status == 0)
                status = rc;
        }
    }
    return status;
}

/* --------------------------------------------------------- paged prefill */

/* Causal multi-query attention over the block table: the prompt (or a chunk
 * of it) attends its own and all earlier tokens ([P1] §3.2 puts
 * FlashAttention-style attention on this path; [P3] §4 runs long texts with
 * block_size 32). Query rows are packed [total_q][num_heads][head_size], the
 * rows of sequence s being query_start[s] .. query_start[s+1] - 1. With
 * n_s rows and context length L_s (the cache already holds all L_s tokens),
 * row query_start[s] + i sits at position L_s - n_s + i and attends the
 * tokens 0 .. L_s - n_s + i of its sequence, with the same softmax as the
 * decode above. Computes the (row, head) pairs of row_head ([n_pairs][2]),
 * or every row x head in (row, head) order when row_head is NULL; out holds
 * one head_size row of doubles per pair. Returns 0, or -1 on n_s < 0,
 * n_s > L_s, a pair out of range or a bad table entry. */
int oracle_paged_prefill(double *out, const uint16_t *query, const int32_t *query_start,
                         const void *key_cache, const void *value_cache,
                         int kv_dtype, int num_blocks, int block_size,
                         int num_heads, int head_size,
                         const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *context_lens, int num_seqs,
                         float scale, float k_scale, float v_scale,
                         const int32_t *row_head, int n_pairs)
{
    int total_q = query_start[num_seqs];
    for (int s = 0; s < num_seqs; ++s) {
        int n = query_start[s + 1] - query_start[s];
        if (n < 0 || n > context_lens[s])
            return -1;
    }
    int total = row_head ? n_pairs : total_q * num_heads;
    for (int i = 0; i < total; ++i) {
        int row = row_head ? row_head[2 * i] : i / num_heads;
        int h = row_head ? row_head[2 * i + 1] : i % num_heads;
        if (row < 0 || row >= total_q || h < 0 || h >= num_heads)
            return -1;
        int s = 0;
        while (query_start[s + 1] <= row)
            ++s;
        int n = query_start[s + 1] - query_start[s];
        int pos = context_lens[s] - n + (row - query_start[s]);
        const uint16_t *q = query + ((int64_t)row * num_heads + h) * head_size;
        double m, l;
        int rc = attend_range(out + (int64_t)i * head_size, &m, &l, q, key_cache,
                              value_cache, kv_dtype, num_blocks, block_size,
                              num_heads, head_size, block_tables,
                              max_blocks_per_seq, s, h, 0, pos + 1, (double)scale,
                              (double)k_scale, (double)v_scale);
        if (rc)
            return rc;
    }
    return 0;
}

/* ------------------------------------- split-context partitions (a8, a9) */

/* Partition p of sequence s covers tokens [p*P, min(L, (p+1)*P)). For each
 * (s, h, p) with p < ceil(L/P) this writes the normalised partial output
 * o_p = sum w_t V_t / l_p over that range and its log-sum-exp
 * lse_p = m_p + ln(l_p) (natural log). Layouts: o [S][H][max_parts][D],
 * lse [S][H][max_parts]; unused partition slots are set to NaN. */
int oracle_attention_partials(double *o, double *lse, const uint16_t *query,
                              const void *key_cache, const void *value_cache,
                              int kv_dtype, int num_blocks, int block_size,
                              int num_heads, int head_size,
                              const int32_t *block_tables, int max_blocks_per_seq,
                              const int32_t *context_lens, int num_seqs,
                              float scale, float k_scale, float v_scale,
                              int partition_size, int max_parts)
{
    for (int s = 0; s < num_seqs; ++s) {
        int L = context_lens[s];
        int nparts = L > 0 ? (L + partition_size - 1) / partition_size : 0;
        if (nparts > max_parts)
            return -1;
        for (int h = 0; h < num_heads; ++h) {
            for (int p = 0; p < max_parts; ++p) {
                int64_t slot = ((int64_t)s * num_heads + h) * max_parts + p;
                double *op = o + slot * head_size;
                if (p >= nparts) {
                    for (int d = 0; d < head_size; ++d)
                        op[d] = NAN;
                    lse[slot] = NAN;
                    continue;
                }
                int t0 = p * partition_size;
                int t1 = t0 + partition_size < L ? t0 + partition_size : L;
                double m, l;
                int rc = attend_range(op, &m, &l,
                                      query + ((int64_t)s * num_heads + h) * head_size,
                                      key_cache, value_cache,
                                      kv_dtype, num_blocks, block_size, num_heads,
                                      head_size, block_tables, max_blocks_per_seq,
                                      s, h, t0, t1, (double)scale,
                                      (double)k_scale, (double)v_scale);
                if (rc)
                    return rc;
                lse[slot] = m + log(l);
            }
        }
    }
    return 0;
}

/* Log-sum-exp combination of n partial results for one (sequence, head):
 *   M = max_p lse_p,  w_p = exp(lse_p - M),  out = sum_p w_p o_p / sum_p w_p.
 * This equals attention over the union of the partitions' token ranges,
 * because w_p / sum w is each partition's share of the full softmax mass. */
void oracle_lse_combine(double *out, const double *o, const double *lse,
                        int n_parts, int head_size)
{
    double M = -INFINITY;
    for (int p = 0; p < n_parts; ++p)
        if (lse[p] > M)
            M = lse[p];
    double wsum = 0.0;
    for (int p = 0; p < n_parts; ++p)
        wsum += exp(lse[p] - M);
    for (int d = 0; d < head_size; ++d) {
        double acc = 0.0;
        for (int p = 0; p < n_parts; ++p)
            acc += exp(lse[p] - M) * o[(int64_t)p * head_size + d];
        out[d] = acc / wsum;
    }
}

/* Element-wise helpers for tests: decode whole arrays. */
void oracle_f16_array_to_double(double *dst, const uint16_t *src, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = oracle_f16_to_double(src[i]);
}

void oracle_e4m3_array_to_double(double *dst, const uint8_t *src, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = oracle_e4m3_to_double(src[i]);
}

void oracle_e4m3_array_from_float(uint8_t *dst, const float *src, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = oracle_e4m3_from_float(src[i]);
}
