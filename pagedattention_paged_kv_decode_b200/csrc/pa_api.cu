// pa_api.cu -- the C ABI of libpagedkv.so (declared in include/pagedkv.h):
// argument validation, launch-shape choice, TMA descriptors, the split
// workspace and kernel launches. Every compute step runs in the kernels of
// pa_decode.cuh, pa_prefill.cuh and pa_cache_ops.cuh; nothing here touches
// KV data.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "pa_cache_ops.cuh"
#include "pa_decode.cuh"
#include "pa_prefill.cuh"
#include "pagedkv.h"

namespace {

thread_local char g_msg[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return code;
}

int ok() {
    g_msg[0] = '\0';
    return PA_OK;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cache(const pa_cache_desc &c) {
    if (c.dtype != PA_F16 && c.dtype != PA_E4M3)
        return fail(PA_ERR_DTYPE, "cache dtype %d is neither PA_F16 nor PA_E4M3", c.dtype);
    if (c.num_blocks < 1 || c.num_heads < 1)
        return fail(PA_ERR_INVALID, "num_blocks (%d) and num_heads (%d) must be >= 1",
                    c.num_blocks, c.num_heads);
    if (c.num_heads > 65535)  // keeps num_heads * head_size and the per-head grids in int
        return fail(PA_ERR_INVALID, "num_heads %d > 65535", c.num_heads);
    if (c.block_size != 16 && c.block_size != 32)
        return fail(PA_ERR_INVALID, "block_size %d: supported are 16 and 32", c.block_size);
    if (c.head_size != 64 && c.head_size != 128)
        return fail(PA_ERR_INVALID, "head_size %d: supported are 64 and 128", c.head_size);
    if ((int64_t)c.num_blocks * c.block_size >= (int64_t(1) << 31))
        return fail(PA_ERR_OVERFLOW, "num_blocks * block_size = %lld does not fit int32 slots",
                    (long long)c.num_blocks * c.block_size);
    return PA_OK;
}

int elem_bytes(const pa_cache_desc &c) { return c.dtype == PA_F16 ? 2 : 1; }

// ------------------------------------------------------------ TMA maps

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

struct MapKey {
    const void *ptr;
    int nb, bs, nh, hd, dtype, g, swz;
    bool operator==(const MapKey &o) const {
        return ptr == o.ptr && nb == o.nb && bs == o.bs && nh == o.nh && hd == o.hd &&
               dtype == o.dtype && g == o.g && swz == o.swz;
    }
};

std::mutex g_map_mu;
std::vector<std::pair<MapKey, CUtensorMap>> g_maps;  // small FIFO cache

// 4-D view of a cache, innermost first: {head_size, num_heads, block_size,
// num_blocks}; box {head_size, G, block_size, 1} = one physical block's rows
// for G heads. Zero fill outside the pool.
// swz = 1: box {64, 1, block_size, 1} (a 64-dim half of one head's rows)
// with 128-byte swizzle, for the tensor-core kernels (shared prefix, both
// prefills), whose MMA operands take that layout.
int cache_tensor_map(const void *cache, const pa_cache_desc &c, int G, CUtensorMap *out, int swz = 0) {
    const MapKey key{cache, c.num_blocks, c.block_size, c.num_heads, c.head_size, c.dtype, G, swz};
    {
        std::lock_guard<std::mutex> lk(g_map_mu);
        for (auto &e : g_maps)
            if (e.first == key) {
                *out = e.second;
                return PA_OK;
            }
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t eb = (cuuint64_t)elem_bytes(c);
    const cuuint64_t dims[4] = {(cuuint64_t)c.head_size, (cuuint64_t)c.num_heads,
                                (cuuint64_t)c.block_size, (cuuint64_t)c.num_blocks};
    const cuuint64_t strides[3] = {(cuuint64_t)c.head_size * eb,
                                   (cuuint64_t)c.head_size * c.num_heads * eb,
                                   (cuuint64_t)c.head_size * c.num_heads * c.block_size * eb};
    const cuuint32_t box[4] = {swz ? 64u : (cuuint32_t)c.head_size, swz ? 1u : (cuuint32_t)G,
                               (cuuint32_t)c.block_size, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap m;
    const CUresult r = enc(&m,
                           c.dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                           4, const_cast<void *>(cache), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE,
                           swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    {
        std::lock_guard<std::mutex> lk(g_map_mu);
        if (g_maps.size() >= 64) g_maps.erase(g_maps.begin());
        g_maps.emplace_back(key, m);
    }
    *out = m;
    return PA_OK;
}

// ----------------------------------------------------- launch shape

constexpr int kNumSMs = 148;
constexpr int kMaxGridY = 65535;  // grid y extent: token and pair counts are launched in slices of this
constexpr size_t kMaxSmem = 227 * 1024;

// `beside`: CTAs of a kernel that runs next to this decode (the shared-prefix
// kernel on its second stream). They keep SMs busy too, so the decode needs
// fewer, longer units of its own.
int fill_config(const pa_cache_desc &c, int num_seqs, int max_ctx, pa_decode_config *cfg,
                int64_t beside = 0) {
    const int H = c.num_heads, B = c.block_size;
    pa_decode_config r = *cfg;
    auto stage_bytes = [&](int G) {
        return pa::SmemLayout(B, G, c.head_size, elem_bytes(c), 1, 1, 1).stage_bytes;
    };
    auto units = [&](int G, int P) {  // CTAs of the grid, from the host-side length bound
        return (int64_t)num_seqs * (H / G) * std::max<int64_t>(1, ((int64_t)max_ctx + P - 1) / P);
    };
    // Defaults, fitted by launch-shape sweeps on B200 (sequences x heads x
    // contexts of 16x32x<=178, 64x40x<=2048, 32x32x<=4096, 256x32x<=4096):
    // about four consumer warps per CTA, a ring of about 64 KiB so that three
    // or more CTAs share an SM, enough CTAs for every SM, and long partitions
    // only when the grid stays large with them. Beside the shared-prefix
    // kernel (sweeps of 8-128 sequences sharing a 3072-token prefix, 1-1024
    // private tokens each) partitions of 1024 tokens already paid off from
    // 4 CTAs per SM in both grids together.
    if (r.heads_per_cta == 0) {
        int G = 4;
        while (G > 1 && (H % G || stage_bytes(G) * 2 > 96 * 1024)) G >>= 1;
        const int P0 = r.partition_size ? r.partition_size : 512;
        while (G > 1 && units(G, P0) + beside < 3 * kNumSMs) G >>= 1;
        r.heads_per_cta = G;
    }
    const int G0 = r.heads_per_cta;
    if (r.partition_size == 0) {
        const bool long_parts = beside > 0 ? units(G0, 1024) + beside >= 4 * kNumSMs
                                           : units(G0, 1024) >= 12 * kNumSMs;
        int P = long_parts ? 1024 : 512;
        while (P > 4 * B && units(G0, P) + beside < 3 * kNumSMs) P >>= 1;
        r.partition_size = P;
    }
    // One unit per CTA by default: measured on B200, packing 2-4 units of a
    // small batch into one CTA (one producer thread issuing every slot's tile
    // loads) was slower than one CTA per unit with several CTAs per SM.
    if (r.units_per_cta == 0) r.units_per_cta = 1;
    const int C0 = r.units_per_cta;
    // stages must be a multiple of warps_per_head (see the check below).
    if (r.warps_per_head == 0) {
        // one head per CTA: 4 warps; 2 heads: 2 warps each; 4 or more: 1 each
        int W = C0 > 1 ? 2 : (G0 >= 4 ? 1 : (G0 == 2 ? 2 : 4));
        while (W > 1 && (r.stages != 0 && r.stages % W)) W >>= 1;
        while (W > 1 && C0 * G0 * W > pa::kMaxConsumerWarps) W >>= 1;
        r.warps_per_head = W;
    }
    if (r.stages == 0) {
        const int W = r.warps_per_head;
        size_t ring = C0 > 1 ? (200 * 1024) / C0 : 64 * 1024;
        const int64_t n = units(G0, r.partition_size);
        if (C0 == 1 && n < 4 * kNumSMs) {  // small grid: keep every CTA resident at once
            const int64_t per_sm = std::max<int64_t>(1, (n + kNumSMs - 1) / kNumSMs);
            ring = std::min<size_t>(ring, (200 * 1024) / per_sm);
        }
        int st = (int)std::min<size_t>(8, std::max<size_t>(2, ring / stage_bytes(G0)));
        st = std::max(W, st / W * W);
        r.stages = std::max(2, st);
    }
    if (r.partition_size < B || r.partition_size % B)
        return fail(PA_ERR_INVALID, "partition_size %d must be a positive multiple of block_size %d",
                    r.partition_size, B);
    const int G = r.heads_per_cta;
    if (!(G == 1 || G == 2 || G == 4 || G == 8) || H % G)
        return fail(PA_ERR_INVALID, "heads_per_cta %d must be 1, 2, 4 or 8 and divide num_heads %d",
                    G, H);
    const int W = r.warps_per_head;
    const int C = r.units_per_cta;
    if (C < 1 || C > pa::kMaxUnitsPerCta)
        return fail(PA_ERR_INVALID, "units_per_cta %d must be in [1, %d]", C, pa::kMaxUnitsPerCta);
    if (!(W == 1 || W == 2 || W == 4) || C * G * W > pa::kMaxConsumerWarps)
        return fail(PA_ERR_INVALID,
                    "warps_per_head %d must be 1, 2 or 4 with units*heads*warps <= %d", W,
                    pa::kMaxConsumerWarps);
    if (r.stages < 2 || r.stages > 8)
        return fail(PA_ERR_INVALID, "stages %d must be in [2, 8]", r.stages);
    // Warp w of a head consumes blocks w, w+W, ... from stage i % stages and
    // waits on that stage's full barrier by phase parity. A parity wait is
    // only meaningful for the current or the immediately preceding phase, so
    // the previous use of the stage must be one the same warp has already
    // consumed: with stages % W == 0 every stage belongs to exactly one warp.
    if (r.stages % W)
        return fail(PA_ERR_INVALID, "stages %d must be a multiple of warps_per_head %d", r.stages, W);
    const pa::SmemLayout lay(B, G, c.head_size, elem_bytes(c), W, r.stages, C);
    if (lay.total > kMaxSmem)
        return fail(PA_ERR_INVALID, "launch shape needs %zu bytes of shared memory (max %zu)",
                    lay.total, kMaxSmem);
    *cfg = r;
    return PA_OK;
}

int max_parts_of(int max_ctx, int P) { return (int)std::max<int64_t>(1, ((int64_t)max_ctx + P - 1) / P); }

size_t ws_lse_bytes(const pa_cache_desc &c, int S, int parts) {
    return ((size_t)S * c.num_heads * parts * sizeof(float) + 255) / 256 * 256;
}

size_t ws_bytes(const pa_cache_desc &c, int S, int max_ctx, const pa_decode_config &cfg) {
    const int parts = max_parts_of(max_ctx, cfg.partition_size);
    if (parts <= 1) return 0;
    return ws_lse_bytes(c, S, parts) + (size_t)S * c.num_heads * parts * c.head_size * sizeof(float);
}

// ----------------------------------------------------- kernel tables

using DecodeKernel = void (*)(const CUtensorMap, const CUtensorMap, const pa::DecodeParams);
using ReduceKernel = void (*)(const pa::DecodeParams);

DecodeKernel pick_decode(int D, int B, bool fp8, bool narrow = false) {
#define PA_PICK(d, b, f)                                                                      \
    if (D == d && B == b && fp8 == f)                                                         \
        return narrow ? pa::paged_decode_kernel<d, b, f, pa::kNarrowDecodeThreads, pa::kNarrowDecodeCtas> \
                      : pa::paged_decode_kernel<d, b, f>;
    PA_PICK(64, 16, false) PA_PICK(64, 32, false) PA_PICK(128, 16, false) PA_PICK(128, 32, false)
    PA_PICK(64, 16, true) PA_PICK(64, 32, true) PA_PICK(128, 16, true) PA_PICK(128, 32, true)
#undef PA_PICK
    return nullptr;
}

DecodeKernel pick_prefix(int D, int B, bool fp8) {
#define PA_PICK(d, b, f) \
    if (D == d && B == b && fp8 == f) return pa::paged_prefix_kernel<d, b, f>;
    PA_PICK(64, 16, false) PA_PICK(64, 32, false) PA_PICK(128, 16, false) PA_PICK(128, 32, false)
    PA_PICK(64, 16, true) PA_PICK(64, 32, true) PA_PICK(128, 16, true) PA_PICK(128, 32, true)
#undef PA_PICK
    return nullptr;
}

DecodeKernel pick_prefix_mma(int D, int B) {
    if (D == 64 && B == 16) return pa::paged_prefix_mma_kernel<64, 16>;
    if (D == 64 && B == 32) return pa::paged_prefix_mma_kernel<64, 32>;
    if (D == 128 && B == 16) return pa::paged_prefix_mma_kernel<128, 16>;
    if (D == 128 && B == 32) return pa::paged_prefix_mma_kernel<128, 32>;
    return nullptr;
}

ReduceKernel pick_reduce(int D) {
    return D == 64 ? pa::lse_reduce_kernel<64> : pa::lse_reduce_kernel<128>;
}

std::mutex g_attr_mu;
std::vector<std::pair<const void *, int>> g_attr_done;  // (kernel, device) with max smem set

int ensure_smem_attr(const void *fn, int device) {
    std::lock_guard<std::mutex> lk(g_attr_mu);
    for (auto &e : g_attr_done)
        if (e.first == fn && e.second == device) return PA_OK;
    const cudaError_t e =
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    g_attr_done.emplace_back(fn, device);
    return PA_OK;
}

// Resident CTAs per SM of a kernel at a block size and dynamic shared
// memory, cached per (kernel, block, smem) (the answer depends on no state).
struct OccEntry {
    const void *fn;
    int threads;
    size_t smem;
    int ctas;
};
std::mutex g_occ_mu;
std::vector<OccEntry> g_occ;

int ctas_per_sm(const void *fn, int threads, size_t smem, int *out) {
    std::lock_guard<std::mutex> lk(g_occ_mu);
    for (const auto &e : g_occ)
        if (e.fn == fn && e.threads == threads && e.smem == smem) {
            *out = e.ctas;
            return PA_OK;
        }
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    g_occ.push_back({fn, threads, smem, n});
    *out = n;
    return PA_OK;
}

// ---------------------------------------------- second stream (shared prefix)

// One non-blocking stream and two events per (device, caller stream), made
// on first use and kept for the life of the process.
struct SideStream {
    int device;
    cudaStream_t caller;
    cudaStream_t stream;
    cudaEvent_t fork, join;
};
std::mutex g_side_mu;
std::vector<SideStream> g_side;

int side_stream(cudaStream_t st, int device, SideStream *out) {
    std::lock_guard<std::mutex> lk(g_side_mu);
    for (const auto &e : g_side)
        if (e.device == device && e.caller == st) {
            *out = e;
            return PA_OK;
        }
    SideStream s{device, st, nullptr, nullptr, nullptr};
    cudaError_t e = cudaStreamCreateWithFlags(&s.stream, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "second stream for the shared prefix");
    g_side.push_back(s);
    *out = s;
    return PA_OK;
}

// ---------------------------------------------- internal split workspace

struct WsEntry {
    int device;
    cudaStream_t stream;
    void *ptr;
    size_t bytes;
};
std::mutex g_ws_mu;
std::vector<WsEntry> g_ws;
// Outgrown workspaces are kept, not freed: a CUDA graph captured before a
// workspace grew still holds the old address, and replaying it must not
// touch freed memory. Growth is by at least 1.25x, so the kept buffers add
// up to at most about four times the current one.
std::vector<void *> g_ws_retired;

int internal_workspace(size_t need, cudaStream_t st, int device, void **out) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    WsEntry *ent = nullptr;
    for (auto &e : g_ws)
        if (e.device == device && e.stream == st) ent = &e;
    if (ent && ent->bytes >= need) {
        *out = ent->ptr;
        return PA_OK;
    }
    const size_t bytes = std::max<size_t>(need + need / 4, 1 << 20);
    void *p = nullptr;
    cudaError_t e = cudaMallocAsync(&p, bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync (split workspace)");
    if (ent) {
        g_ws_retired.push_back(ent->ptr);
        ent->ptr = p;
        ent->bytes = bytes;
    } else {
        g_ws.push_back(WsEntry{device, st, p, bytes});
    }
    *out = p;
    return PA_OK;
}

int check_decode_args(void *out, const void *query, const void *kc, const void *vc,
                      const pa_cache_desc &c, const int32_t *bt, int maxblk, const int32_t *ctx,
                      int S, int max_ctx, float scale, float k_scale, float v_scale) {
    int rc = check_cache(c);
    if (rc) return rc;
    if (S < 0) return fail(PA_ERR_INVALID, "num_seqs %d < 0", S);
    if (S > 65535) return fail(PA_ERR_INVALID, "num_seqs %d > 65535", S);
    if (S == 0) return PA_OK;
    if (!out || !query || !kc || !vc || !bt || !ctx)
        return fail(PA_ERR_INVALID, "null pointer argument");
    if (!aligned16(out) || !aligned16(query) || !aligned16(kc) || !aligned16(vc))
        return fail(PA_ERR_INVALID, "out, query and caches must be 16-byte aligned");
    if (maxblk < 1) return fail(PA_ERR_INVALID, "max_blocks_per_seq %d < 1", maxblk);
    if ((int64_t)maxblk * c.block_size >= (int64_t(1) << 31))
        return fail(PA_ERR_OVERFLOW, "max_blocks_per_seq * block_size overflows int32");
    if (max_ctx < 0) return fail(PA_ERR_INVALID, "max_context_len %d < 0", max_ctx);
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID, "scale is not finite");
    if (c.dtype == PA_E4M3 &&
        !(std::isfinite(k_scale) && std::isfinite(v_scale) && k_scale > 0 && v_scale > 0))
        return fail(PA_ERR_INVALID, "k_scale and v_scale must be finite and > 0");
    return PA_OK;
}

struct AppendArgs {
    const void *new_key;
    const void *new_value;
    int64_t key_stride;
    int64_t value_stride;
    int32_t *slot_out;
};

// Launch shape of the shared-prefix kernel (see pa_paged_attention_decode_shared_prefix).
struct PrefixPlan {
    int prefix_tokens;  // shared tokens (whole blocks)
    int partition;      // tokens per prefix partition
    int parts;          // prefix partitions
    int heads;          // heads per CTA
    int queries;        // sequences per CTA
    int stages;
    bool mma;           // fp16 caches: the tensor-core kernel
};

// pa_test_stall_next_decode: consumed (and cleared) by the next decode
// launch of this thread.
struct StallRequest {
    int seq = -1, head = 0, partition = 0;
    uint64_t wait_limit_ns = 0;
};
thread_local StallRequest g_stall;

int launch_decode(void *out, const void *query, const void *kc, const void *vc,
                  const pa_cache_desc &c, const int32_t *bt, int maxblk, const int32_t *ctx, int S,
                  int max_ctx, float scale, float k_scale, float v_scale,
                  const pa_decode_config &cfg, void *ws, cudaStream_t st, int device,
                  const AppendArgs *app = nullptr, const PrefixPlan *pre = nullptr) {
    const int B = c.block_size, D = c.head_size;
    const bool fp8 = c.dtype == PA_E4M3;
    max_ctx = std::min<int64_t>(max_ctx, (int64_t)maxblk * B);
    const int prefix_tokens = pre ? pre->prefix_tokens : 0;
    // suffix partitions (all partitions without a shared prefix); at least one
    // unit per sequence so that every sequence's slot and flags are handled
    const int parts = max_parts_of(std::max(max_ctx - prefix_tokens, 0), cfg.partition_size);
    const int ws_parts = parts + (pre ? pre->parts : 0);
    const int G = cfg.heads_per_cta, W = cfg.warps_per_head;

    CUtensorMap mk, mv;
    int rc = cache_tensor_map(kc, c, G, &mk);
    if (rc) return rc;
    rc = cache_tensor_map(vc, c, G, &mv);
    if (rc) return rc;

    pa::DecodeParams p{};
    p.out = static_cast<__half *>(out);
    p.query = static_cast<const __half *>(query);
    p.block_tables = bt;
    p.context_lens = ctx;
    if (ws_parts > 1 || pre) {
        p.ws_lse = static_cast<float *>(ws);
        p.ws_o = reinterpret_cast<float *>(static_cast<char *>(ws) + ws_lse_bytes(c, S, ws_parts));
    }
    p.ws_parts = ws_parts;
    if (pre) {
        p.prefix_tokens = pre->prefix_tokens;
        p.prefix_parts = pre->parts;
        p.prefix_partition = pre->partition;
        p.queries_per_cta = pre->queries;
    }
    p.num_seqs = S;
    p.num_heads = c.num_heads;
    p.num_blocks = c.num_blocks;
    p.block_size = B;
    p.max_blocks_per_seq = maxblk;
    p.max_context_len = max_ctx;
    p.partition_size = cfg.partition_size;
    p.max_parts = parts;
    p.heads_per_cta = G;
    p.warps_per_head = W;
    p.stages = cfg.stages;
    p.units_per_cta = cfg.units_per_cta;
    p.num_units = (int64_t)S * (c.num_heads / G) * parts;
    p.qk_scale_log2 = scale * pa::kLog2e;
    p.logit_k_scale = fp8 ? k_scale : 1.0f;
    p.out_scale = fp8 ? v_scale : 1.0f;
    if (app) {
        p.new_key = static_cast<const __half *>(app->new_key);
        p.new_value = static_cast<const __half *>(app->new_value);
        p.new_key_stride = app->key_stride;
        p.new_value_stride = app->value_stride;
        p.key_cache = const_cast<void *>(kc);
        p.value_cache = const_cast<void *>(vc);
        p.slot_out = app->slot_out;
        p.k_scale = fp8 ? k_scale : 1.0f;
        p.v_scale = fp8 ? v_scale : 1.0f;
    }

    if (g_stall.seq >= 0) {
        // the unit holding (seq, head, partition), numbered as unit_coord does
        // in the kernel: partition slowest (highest first), then sequence,
        // then head group
        const StallRequest r = g_stall;
        g_stall = StallRequest{};
        if (r.seq < S && r.head < c.num_heads && r.partition < parts) {
            const int64_t hg_count = c.num_heads / G;
            const int64_t unit = ((int64_t)(parts - 1 - r.partition) * S + r.seq) * hg_count + r.head / G;
            p.stall_unit_plus1 = unit + 1;
            p.wait_limit_ns = r.wait_limit_ns;
        }
    }

    const int C = cfg.units_per_cta;
    const pa::SmemLayout lay(B, G, D, elem_bytes(c), W, cfg.stages, C);
    const int threads = 32 * (C * G * W + 1);
    DecodeKernel kern = pick_decode(D, B, fp8);
    if (!kern) return fail(PA_ERR_INVALID, "no kernel for head_size %d block_size %d", D, B);
    rc = ensure_smem_attr(reinterpret_cast<const void *>(kern), device);
    if (rc) return rc;
    if (threads <= pa::kNarrowDecodeThreads) {
        // the register-capped instantiation, where it fits more CTAs on an SM
        DecodeKernel narrow = pick_decode(D, B, fp8, true);
        rc = ensure_smem_attr(reinterpret_cast<const void *>(narrow), device);
        if (rc) return rc;
        int wide_ctas = 0, narrow_ctas = 0;
        rc = ctas_per_sm(reinterpret_cast<const void *>(kern), threads, lay.total, &wide_ctas);
        if (rc) return rc;
        rc = ctas_per_sm(reinterpret_cast<const void *>(narrow), threads, lay.total, &narrow_ctas);
        if (rc) return rc;
        if (narrow_ctas > wide_ctas) kern = narrow;
    }
    cudaError_t e;
    // Shared prefix: the prefix kernel runs on a second stream beside the
    // decode of the private parts (the two write disjoint partials; the
    // prefix kernel reads only the shared blocks). The second stream waits
    // for everything before this call on `st`, and `st` waits for it before
    // the reduce, so the call keeps its place in the caller's stream order
    // (and a CUDA graph captured on `st` takes both branches).
    DecodeKernel pkern = nullptr;
    CUtensorMap pk_, pv_;
    pa::DecodeParams pp = p;
    int64_t pn = 0;
    size_t psmem = 0;
    int pthreads = 0;
    SideStream side{};
    if (pre) {
        pkern = pre->mma ? pick_prefix_mma(D, B) : pick_prefix(D, B, fp8);
        rc = ensure_smem_attr(reinterpret_cast<const void *>(pkern), device);
        if (rc) return rc;
        rc = cache_tensor_map(kc, c, pre->heads, &pk_, pre->mma ? 1 : 0);
        if (rc) return rc;
        rc = cache_tensor_map(vc, c, pre->heads, &pv_, pre->mma ? 1 : 0);
        if (rc) return rc;
        pp.heads_per_cta = pre->heads;
        pp.stages = pre->stages;
        const int64_t n_qb = (S + pre->queries - 1) / pre->queries;
        pn = (int64_t)(c.num_heads / pre->heads) * pre->parts * n_qb;
        if (pre->mma) {
            // ring + barriers + 1 KiB to align the ring to 1024 bytes in the kernel
            psmem = (size_t)pre->stages * 4 * B * D + 16 * (size_t)pre->stages + 1024;
            pthreads = 32 * 5;
        } else {
            psmem = pa::SmemLayout(B, pre->heads, D, elem_bytes(c), 1, pre->stages, 1).total;
            pthreads = 32 * (pre->heads * pre->queries + 1);
        }
        rc = side_stream(st, device, &side);
        if (rc) return rc;
        e = cudaEventRecord(side.fork, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side.stream, side.fork, 0);
        if (e != cudaSuccess) return cuda_fail(e, "shared-prefix stream fork");
    }
    // Every unit u is served by CTA u % grid, slot u / grid: grid * C >= units.
    // Packed CTAs are spread over all SMs (some slots of the last ones idle).
    const int64_t n_ctas = std::max<int64_t>((p.num_units + C - 1) / C,
                                             std::min<int64_t>(p.num_units, kNumSMs));
    // unit ids are 32-bit in the kernels
    if (n_ctas > 0x7fffffff || p.num_units > 0x7fffffff)
        return fail(PA_ERR_INVALID, "too many work units (%lld)", (long long)p.num_units);
    const dim3 grid((unsigned)n_ctas);
    const dim3 block(threads);
    kern<<<grid, block, lay.total, st>>>(mk, mv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "paged_decode_kernel launch");
    if (pre) {
        pkern<<<dim3((unsigned)pn), dim3(pthreads), psmem, side.stream>>>(pk_, pv_, pp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "paged_prefix_kernel launch");
        e = cudaEventRecord(side.join, side.stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, side.join, 0);
        if (e != cudaSuccess) return cuda_fail(e, "shared-prefix stream join");
    }
    if (ws_parts > 1 || pre) {
        // programmatic dependent launch: the reduce is scheduled while the
        // partition kernel drains and waits for it on the device
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3((c.num_heads + 3) / 4, S);
        lc.blockDim = dim3(128);
        lc.dynamicSmemBytes = 0;
        lc.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = attr;
        lc.numAttrs = 1;
        e = cudaLaunchKernelEx(&lc, pick_reduce(D), p);
        if (e != cudaSuccess) return cuda_fail(e, "lse_reduce_kernel launch");
    }
    return ok();
}

int current_device(int *dev) {
    const cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    return PA_OK;
}

}  // namespace

extern "C" {

int pa_version(void) { return 202; }

const char *pa_last_error(void) { return g_msg; }

int pa_test_stall_next_decode(int seq, int head, int partition, uint64_t wait_limit_ns) {
    if (seq < 0) {
        g_stall = StallRequest{};
        return ok();
    }
    if (head < 0 || partition < 0)
        return fail(PA_ERR_INVALID, "head %d and partition %d must be >= 0", head, partition);
    if (wait_limit_ns < 1000 || wait_limit_ns > pa::kWaitLimitNs)
        return fail(PA_ERR_INVALID, "wait_limit_ns %llu outside [1000, %llu]",
                    (unsigned long long)wait_limit_ns, (unsigned long long)pa::kWaitLimitNs);
    g_stall.seq = seq;
    g_stall.head = head;
    g_stall.partition = partition;
    g_stall.wait_limit_ns = wait_limit_ns;
    return ok();
}

int pa_check_status(void *stream, uint32_t *code) {
    if (!code) return fail(PA_ERR_INVALID, "code is null");
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, pa::g_error_word, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    e = cudaMemcpyToSymbol(pa::g_error_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    *code = v;
    return ok();
}

int pa_slot_mapping(int32_t *slot_mapping, const int32_t *block_tables, int max_blocks_per_seq,
                    const int32_t *context_lens, int num_seqs, pa_cache_desc cache, void *stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (num_seqs < 0) return fail(PA_ERR_INVALID, "num_seqs %d < 0", num_seqs);
    if (num_seqs == 0) return ok();
    if (!slot_mapping || !block_tables || !context_lens)
        return fail(PA_ERR_INVALID, "null pointer argument");
    if (max_blocks_per_seq < 1) return fail(PA_ERR_INVALID, "max_blocks_per_seq < 1");
    const int threads = 128;
    pa::slot_mapping_kernel<<<(unsigned)(((int64_t)num_seqs + threads - 1) / threads), threads, 0,
                              static_cast<cudaStream_t>(stream)>>>(
        slot_mapping, block_tables, max_blocks_per_seq, context_lens, num_seqs, cache.block_size,
        cache.num_blocks);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "slot_mapping_kernel launch");
    return ok();
}

int pa_kv_cache_write(const void *key, const void *value, int64_t key_stride, int64_t value_stride,
                      void *key_cache, void *value_cache, pa_cache_desc cache,
                      const int32_t *slot_mapping, int n_tokens, float k_scale, float v_scale,
                      void *stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (n_tokens < 0) return fail(PA_ERR_INVALID, "n_tokens %d < 0", n_tokens);
    if (n_tokens == 0) return ok();
    if (!key || !value || !key_cache || !value_cache || !slot_mapping)
        return fail(PA_ERR_INVALID, "null pointer argument");
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return fail(PA_ERR_INVALID, "key, value and caches must be 16-byte aligned");
    const int row = cache.num_heads * cache.head_size;
    if (key_stride < row || value_stride < row || key_stride % 8 || value_stride % 8)
        return fail(PA_ERR_INVALID,
                    "key_stride/value_stride (%lld/%lld) must be >= %d and multiples of 8",
                    (long long)key_stride, (long long)value_stride, row);
    if (cache.dtype == PA_E4M3 &&
        !(std::isfinite(k_scale) && std::isfinite(v_scale) && k_scale > 0 && v_scale > 0))
        return fail(PA_ERR_INVALID, "k_scale and v_scale must be finite and > 0");
    const int chunks = row / 8;
    const int64_t pool_slots = (int64_t)cache.num_blocks * cache.block_size;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    // one launch per 65535 tokens (the grid's y extent), in stream order
    for (int t0 = 0; t0 < n_tokens; t0 += kMaxGridY) {
        const int n = std::min(kMaxGridY, n_tokens - t0);
        const dim3 grid((chunks + 127) / 128, n);
        const __half *k = static_cast<const __half *>(key) + (size_t)t0 * key_stride;
        const __half *v = static_cast<const __half *>(value) + (size_t)t0 * value_stride;
        if (cache.dtype == PA_F16)
            pa::kv_cache_write_kernel<false><<<grid, 128, 0, st>>>(
                k, v, key_stride, value_stride, key_cache, value_cache, slot_mapping + t0, row, pool_slots,
                1.0f, 1.0f);
        else
            pa::kv_cache_write_kernel<true><<<grid, 128, 0, st>>>(
                k, v, key_stride, value_stride, key_cache, value_cache, slot_mapping + t0, row, pool_slots,
                k_scale, v_scale);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "kv_cache_write_kernel launch");
    }
    return ok();
}

int pa_copy_blocks(void *key_cache, void *value_cache, pa_cache_desc cache,
                   const int32_t *src_dst_pairs, int n_pairs, void *stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (n_pairs < 0) return fail(PA_ERR_INVALID, "n_pairs %d < 0", n_pairs);
    if (n_pairs == 0) return ok();
    if (!key_cache || !value_cache || !src_dst_pairs)
        return fail(PA_ERR_INVALID, "null pointer argument");
    if (!aligned16(key_cache) || !aligned16(value_cache))
        return fail(PA_ERR_INVALID, "caches must be 16-byte aligned");
    const int64_t block_vecs =
        (int64_t)cache.block_size * cache.num_heads * cache.head_size * elem_bytes(cache) / 16;
    const int64_t per_cta = (int64_t)pa::kCopyThreads * pa::kCopyVecs;
    for (int p0 = 0; p0 < n_pairs; p0 += kMaxGridY) {  // one launch per 65535 pairs
        const dim3 grid((unsigned)((block_vecs + per_cta - 1) / per_cta), std::min(kMaxGridY, n_pairs - p0), 2);
        pa::copy_blocks_kernel<<<grid, pa::kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
            key_cache, value_cache, src_dst_pairs + 2 * (size_t)p0, block_vecs, cache.num_blocks);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "copy_blocks_kernel launch");
    }
    return ok();
}

int pa_swap_blocks(void *dst_key_cache, void *dst_value_cache, int dst_num_blocks,
                   const void *src_key_cache, const void *src_value_cache, int src_num_blocks,
                   pa_cache_desc cache, const int32_t *src_dst_pairs, int n_pairs, void *stream) {
    pa_cache_desc c = cache;
    c.num_blocks = std::max(1, std::max(dst_num_blocks, src_num_blocks));
    int rc = check_cache(c);
    if (rc) return rc;
    if (dst_num_blocks < 1 || src_num_blocks < 1)
        return fail(PA_ERR_INVALID, "dst_num_blocks (%d) and src_num_blocks (%d) must be >= 1",
                    dst_num_blocks, src_num_blocks);
    if (n_pairs < 0) return fail(PA_ERR_INVALID, "n_pairs %d < 0", n_pairs);
    if (n_pairs == 0) return ok();
    if (!dst_key_cache || !dst_value_cache || !src_key_cache || !src_value_cache || !src_dst_pairs)
        return fail(PA_ERR_INVALID, "null pointer argument");
    if (!aligned16(dst_key_cache) || !aligned16(dst_value_cache) || !aligned16(src_key_cache) ||
        !aligned16(src_value_cache))
        return fail(PA_ERR_INVALID, "caches must be 16-byte aligned");
    const int64_t block_vecs =
        (int64_t)c.block_size * c.num_heads * c.head_size * elem_bytes(c) / 16;
    const int64_t per_cta = (int64_t)pa::kCopyThreads * pa::kCopyVecs;
    for (int p0 = 0; p0 < n_pairs; p0 += kMaxGridY) {  // one launch per 65535 pairs
        const dim3 grid((unsigned)((block_vecs + per_cta - 1) / per_cta), std::min(kMaxGridY, n_pairs - p0), 2);
        pa::swap_blocks_kernel<<<grid, pa::kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
            dst_key_cache, dst_value_cache, src_key_cache, src_value_cache, src_dst_pairs + 2 * (size_t)p0,
            block_vecs, src_num_blocks, dst_num_blocks);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "swap_blocks_kernel launch");
    }
    return ok();
}

int pa_decode_choose_config(pa_cache_desc cache, int num_seqs, int max_context_len,
                            pa_decode_config *cfg) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (!cfg) return fail(PA_ERR_INVALID, "cfg is null");
    if (num_seqs < 0 || max_context_len < 0)
        return fail(PA_ERR_INVALID, "num_seqs and max_context_len must be >= 0");
    rc = fill_config(cache, num_seqs, max_context_len, cfg);
    if (rc) return rc;
    return ok();
}

size_t pa_decode_workspace_size(pa_cache_desc cache, int num_seqs, int max_context_len,
                                const pa_decode_config *cfg) {
    if (check_cache(cache) || num_seqs <= 0 || max_context_len < 0) return 0;
    pa_decode_config r = cfg ? *cfg : pa_decode_config{0, 0, 0, 0, 0};
    if (fill_config(cache, num_seqs, max_context_len, &r)) return 0;
    return ws_bytes(cache, num_seqs, max_context_len, r);
}

int pa_paged_attention_decode(void *out, const void *query, const void *key_cache,
                              const void *value_cache, pa_cache_desc cache,
                              const int32_t *block_tables, int max_blocks_per_seq,
                              const int32_t *context_lens, int num_seqs, int max_context_len,
                              float scale, float k_scale, float v_scale, void *stream) {
    int rc = check_decode_args(out, query, key_cache, value_cache, cache, block_tables,
                               max_blocks_per_seq, context_lens, num_seqs, max_context_len, scale,
                               k_scale, v_scale);
    if (rc) return rc;
    if (num_seqs == 0) return ok();
    const int bound = (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * cache.block_size);
    pa_decode_config cfg{0, 0, 0, 0, 0};
    rc = fill_config(cache, num_seqs, bound, &cfg);
    if (rc) return rc;
    int dev = 0;
    rc = current_device(&dev);
    if (rc) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *ws = nullptr;
    const size_t need = ws_bytes(cache, num_seqs, bound, cfg);
    if (need) {
        rc = internal_workspace(need, st, dev, &ws);
        if (rc) return rc;
    }
    return launch_decode(out, query, key_cache, value_cache, cache, block_tables,
                         max_blocks_per_seq, context_lens, num_seqs, bound, scale, k_scale,
                         v_scale, cfg, ws, st, dev);
}

int pa_paged_attention_decode_ws(void *out, const void *query, const void *key_cache,
                                 const void *value_cache, pa_cache_desc cache,
                                 const int32_t *block_tables, int max_blocks_per_seq,
                                 const int32_t *context_lens, int num_seqs, int max_context_len,
                                 float scale, float k_scale, float v_scale,
                                 const pa_decode_config *cfg, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    int rc = check_decode_args(out, query, key_cache, value_cache, cache, block_tables,
                               max_blocks_per_seq, context_lens, num_seqs, max_context_len, scale,
                               k_scale, v_scale);
    if (rc) return rc;
    if (num_seqs == 0) return ok();
    const int bound = (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * cache.block_size);
    pa_decode_config r = cfg ? *cfg : pa_decode_config{0, 0, 0, 0, 0};
    rc = fill_config(cache, num_seqs, bound, &r);
    if (rc) return rc;
    const size_t need = ws_bytes(cache, num_seqs, bound, r);
    if (need && (!workspace || workspace_bytes < need ||
                 (reinterpret_cast<uintptr_t>(workspace) & 255u)))
        return fail(PA_ERR_WORKSPACE,
                    "workspace of %zu bytes at %p: need %zu bytes, 256-byte aligned",
                    workspace_bytes, workspace, need);
    int dev = 0;
    rc = current_device(&dev);
    if (rc) return rc;
    return launch_decode(out, query, key_cache, value_cache, cache, block_tables,
                         max_blocks_per_seq, context_lens, num_seqs, bound, scale, k_scale,
                         v_scale, r, workspace, static_cast<cudaStream_t>(stream), dev);
}

}  // extern "C"

extern "C" int pa_paged_attention_decode_append(
    void *out, const void *query, const void *new_key, const void *new_value, int64_t key_stride,
    int64_t value_stride, void *key_cache, void *value_cache, pa_cache_desc cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
    int num_seqs, int max_context_len, float scale, float k_scale, float v_scale,
    int32_t *slot_mapping_out, const pa_decode_config *cfg, void *workspace,
    size_t workspace_bytes, void *stream) {
    int rc = check_decode_args(out, query, key_cache, value_cache, cache, block_tables,
                               max_blocks_per_seq, context_lens, num_seqs, max_context_len, scale,
                               k_scale, v_scale);
    if (rc) return rc;
    if (num_seqs == 0) return ok();
    if (!new_key || !new_value) return fail(PA_ERR_INVALID, "null new_key/new_value");
    if (!aligned16(new_key) || !aligned16(new_value))
        return fail(PA_ERR_INVALID, "new_key and new_value must be 16-byte aligned");
    const int row = cache.num_heads * cache.head_size;
    if (key_stride < row || value_stride < row || key_stride % 8 || value_stride % 8)
        return fail(PA_ERR_INVALID,
                    "key_stride/value_stride (%lld/%lld) must be >= %d and multiples of 8",
                    (long long)key_stride, (long long)value_stride, row);
    const int bound =
        (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * cache.block_size);
    pa_decode_config r = cfg ? *cfg : pa_decode_config{0, 0, 0, 0, 0};
    rc = fill_config(cache, num_seqs, bound, &r);
    if (rc) return rc;
    const size_t need = ws_bytes(cache, num_seqs, bound, r);
    int dev = 0;
    rc = current_device(&dev);
    if (rc) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *ws = workspace;
    if (need && workspace) {
        if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return fail(PA_ERR_WORKSPACE,
                        "workspace of %zu bytes at %p: need %zu bytes, 256-byte aligned",
                        workspace_bytes, workspace, need);
    } else if (need) {
        rc = internal_workspace(need, st, dev, &ws);
        if (rc) return rc;
    }
    const AppendArgs app{new_key, new_value, key_stride, value_stride, slot_mapping_out};
    return launch_decode(out, query, key_cache, value_cache, cache, block_tables,
                         max_blocks_per_seq, context_lens, num_seqs, bound, scale, k_scale,
                         v_scale, r, ws, st, dev, &app);
}

namespace {

// Shared-prefix plan and the suffix config; returns the workspace bytes.
int plan_shared_prefix(const pa_cache_desc &c, int S, int bound, int prefix_blocks,
                       const pa_decode_config *cfg, pa_decode_config *suffix, PrefixPlan *pre,
                       size_t *ws) {
    const int B = c.block_size;
    if (prefix_blocks < 1) return fail(PA_ERR_INVALID, "shared_prefix_blocks %d < 1", prefix_blocks);
    if ((int64_t)prefix_blocks * B > bound)  // 64-bit: the size query has no table width to bound it
        return fail(PA_ERR_INVALID, "shared prefix (%lld tokens) beyond the context bound %d",
                    (long long)prefix_blocks * B, bound);
    pre->prefix_tokens = prefix_blocks * B;
    pre->heads = 1;
    pre->mma = c.dtype == PA_F16;
    pre->queries = pre->mma ? pa::kPrefixMmaQueries : std::min(S, pa::kMaxConsumerWarps);
    // prefix partitions of 512 tokens, halved (down to 4 blocks) while the
    // prefix grid has fewer than two CTAs per SM
    const int64_t n_qb = (S + pre->queries - 1) / pre->queries;
    pre->partition = std::max(B, 512 / B * B);
    while (pre->partition > 4 * B &&
           (int64_t)c.num_heads * n_qb * ((pre->prefix_tokens + pre->partition - 1) / pre->partition) <
               2 * kNumSMs)
        pre->partition /= 2;
    pre->parts = (pre->prefix_tokens + pre->partition - 1) / pre->partition;
    const size_t sb = pa::SmemLayout(B, 1, c.head_size, elem_bytes(c), 1, 1, 1).stage_bytes;
    pre->stages = (int)std::max<size_t>(2, std::min<size_t>(8, (96 * 1024) / sb));
    pa_decode_config r = cfg ? *cfg : pa_decode_config{0, 0, 0, 0, 0};
    const int suffix_bound = std::max(bound - pre->prefix_tokens, B);
    const int64_t prefix_ctas = (int64_t)(c.num_heads / pre->heads) * n_qb * pre->parts;
    int rc = fill_config(c, S, suffix_bound, &r, prefix_ctas);
    if (rc) return rc;
    *suffix = r;
    const int ws_parts = max_parts_of(suffix_bound, r.partition_size) + pre->parts;
    *ws = ws_lse_bytes(c, S, ws_parts) + (size_t)S * c.num_heads * ws_parts * c.head_size * sizeof(float);
    return PA_OK;
}

}  // namespace

extern "C" size_t pa_shared_prefix_workspace_size(pa_cache_desc cache, int num_seqs,
                                                  int max_context_len, int shared_prefix_blocks,
                                                  const pa_decode_config *cfg) {
    if (check_cache(cache) || num_seqs <= 0 || max_context_len < 0) return 0;
    pa_decode_config r;
    PrefixPlan pre;
    size_t ws = 0;
    if (plan_shared_prefix(cache, num_seqs, max_context_len, shared_prefix_blocks, cfg, &r, &pre, &ws))
        return 0;
    return ws;
}

extern "C" int pa_paged_attention_decode_shared_prefix(
    void *out, const void *query, const void *new_key, const void *new_value, int64_t key_stride,
    int64_t value_stride, void *key_cache, void *value_cache, pa_cache_desc cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
    int num_seqs, int max_context_len, int shared_prefix_blocks, float scale, float k_scale,
    float v_scale, int32_t *slot_mapping_out, const pa_decode_config *cfg, void *workspace,
    size_t workspace_bytes, void *stream) {
    int rc = check_decode_args(out, query, key_cache, value_cache, cache, block_tables,
                               max_blocks_per_seq, context_lens, num_seqs, max_context_len, scale,
                               k_scale, v_scale);
    if (rc) return rc;
    if (num_seqs == 0) return ok();
    if ((new_key == nullptr) != (new_value == nullptr))
        return fail(PA_ERR_INVALID, "new_key and new_value must both be given or both be NULL");
    if (new_key) {
        if (!aligned16(new_key) || !aligned16(new_value))
            return fail(PA_ERR_INVALID, "new_key and new_value must be 16-byte aligned");
        const int row = cache.num_heads * cache.head_size;
        if (key_stride < row || value_stride < row || key_stride % 8 || value_stride % 8)
            return fail(PA_ERR_INVALID,
                        "key_stride/value_stride (%lld/%lld) must be >= %d and multiples of 8",
                        (long long)key_stride, (long long)value_stride, row);
    }
    if (shared_prefix_blocks > max_blocks_per_seq)
        return fail(PA_ERR_INVALID, "shared_prefix_blocks %d > max_blocks_per_seq %d",
                    shared_prefix_blocks, max_blocks_per_seq);
    const int bound =
        (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * cache.block_size);
    pa_decode_config r;
    PrefixPlan pre;
    size_t need = 0;
    rc = plan_shared_prefix(cache, num_seqs, bound, shared_prefix_blocks, cfg, &r, &pre, &need);
    if (rc) return rc;
    int dev = 0;
    rc = current_device(&dev);
    if (rc) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *ws = workspace;
    if (workspace) {
        if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return fail(PA_ERR_WORKSPACE,
                        "workspace of %zu bytes at %p: need %zu bytes, 256-byte aligned",
                        workspace_bytes, workspace, need);
    } else {
        rc = internal_workspace(need, st, dev, &ws);
        if (rc) return rc;
    }
    const AppendArgs app{new_key, new_value, key_stride, value_stride, slot_mapping_out};
    return launch_decode(out, query, key_cache, value_cache, cache, block_tables,
                         max_blocks_per_seq, context_lens, num_seqs, bound, scale, k_scale,
                         v_scale, r, ws, st, dev, new_key ? &app : nullptr, &pre);
}

// ---------------------------------------------------------------------------
// Decode for callers that may not allocate device memory at all.
//
// Some callers cannot call cudaMalloc (or any allocator) on the path that
// runs the decode: engine plugins whose host framework owns every device
// buffer and forbids allocation during execution, code that runs while a
// CUDA graph is being captured (an allocation there becomes part of the
// graph), and real-time loops with a fixed, pre-planned memory budget. The
// split-context partials of such a call live in the file-scope array below
// instead of a workspace. The array is part of the library's device image:
// every GPU that loads the library holds its kDecodeScratchBytes until the
// process exits.
namespace {

constexpr size_t kDecodeScratchBytes = size_t(16) << 20;  // 16 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

std::mutex g_scratch_mu;
constexpr int kMaxDevices = 128;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so its address is looked up once
// per device with cudaGetSymbolAddress and cached.
int scratch_address(int device, void **out) {
    if (device < 0 || device >= kMaxDevices)
        return fail(PA_ERR_INVALID, "device ordinal %d out of range", device);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[device]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress (static decode scratch)");
        g_scratch_addr[device] = p;
    }
    *out = g_scratch_addr[device];
    return PA_OK;
}

}  // namespace

extern "C" int pa_paged_attention_decode_noalloc(
    void *out, const void *query, const void *key_cache, const void *value_cache,
    pa_cache_desc cache, const int32_t *block_tables, int max_blocks_per_seq,
    const int32_t *context_lens, int num_seqs, int max_context_len, float scale, float k_scale,
    float v_scale, void *stream) {
    int rc = check_decode_args(out, query, key_cache, value_cache, cache, block_tables,
                               max_blocks_per_seq, context_lens, num_seqs, max_context_len, scale,
                               k_scale, v_scale);
    if (rc) return rc;
    if (num_seqs == 0) return ok();
    const int bound =
        (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * cache.block_size);
    pa_decode_config cfg{0, 0, 0, 0, 0};
    rc = fill_config(cache, num_seqs, bound, &cfg);
    if (rc) return rc;
    const size_t need = ws_bytes(cache, num_seqs, bound, cfg);
    if (need > kDecodeScratchBytes)
        return fail(PA_ERR_WORKSPACE,
                    "this decode needs %zu bytes of split scratch but the static scratch of "
                    "pa_paged_attention_decode_noalloc holds %zu; lower num_seqs or "
                    "max_context_len, or call pa_paged_attention_decode_ws",
                    need, kDecodeScratchBytes);
    int dev = 0;
    rc = current_device(&dev);
    if (rc) return rc;
    void *scratch = nullptr;
    rc = scratch_address(dev, &scratch);  // first call on a device: symbol lookup
    if (rc) return rc;
    return launch_decode(out, query, key_cache, value_cache, cache, block_tables,
                         max_blocks_per_seq, context_lens, num_seqs, bound, scale, k_scale,
                         v_scale, cfg, need ? scratch : nullptr, static_cast<cudaStream_t>(stream),
                         dev);
}

// ------------------------------------------------------------ paged prefill

namespace {

using PrefillKernel = void (*)(const CUtensorMap, const CUtensorMap, const pa::PrefillParams);

PrefillKernel pick_prefill(int D, int B) {
    if (D == 64 && B == 16) return pa::paged_prefill_kernel<64, 16>;
    if (D == 64 && B == 32) return pa::paged_prefill_kernel<64, 32>;
    if (D == 128 && B == 16) return pa::paged_prefill_kernel<128, 16>;
    if (D == 128 && B == 32) return pa::paged_prefill_kernel<128, 32>;
    return nullptr;
}

PrefillKernel pick_prefill_tc(int D, int B) {
    if (D == 64 && B == 16) return pa::paged_prefill_tc_kernel<64, 16>;
    if (D == 64 && B == 32) return pa::paged_prefill_tc_kernel<64, 32>;
    if (D == 128 && B == 16) return pa::paged_prefill_tc_kernel<128, 16>;
    if (D == 128 && B == 32) return pa::paged_prefill_tc_kernel<128, 32>;
    return nullptr;
}

// Ring of the prefill kernel: about 96 KiB of K/V tiles, so that two CTAs
// (160 threads, under 200 registers each) share an SM.
int prefill_stages(const pa_cache_desc &c) {
    const int stage = 4 * c.block_size * c.head_size;  // K + V tiles, fp16
    return std::max(2, std::min(8, (96 * 1024) / stage));
}

}  // namespace

extern "C" int pa_prefill_slot_mapping(int32_t *slot_mapping, const int32_t *query_start,
                                       const int32_t *block_tables, int max_blocks_per_seq,
                                       const int32_t *context_lens, int num_seqs, int total_q,
                                       int max_query_len, pa_cache_desc cache, void *stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (num_seqs < 0 || num_seqs > 65535) return fail(PA_ERR_INVALID, "num_seqs %d not in [0, 65535]", num_seqs);
    if (total_q < 0) return fail(PA_ERR_INVALID, "total_q %d < 0", total_q);
    if (max_query_len < 0) return fail(PA_ERR_INVALID, "max_query_len %d < 0", max_query_len);
    if (num_seqs == 0 || total_q == 0) return ok();
    if (!slot_mapping || !query_start || !block_tables || !context_lens)
        return fail(PA_ERR_INVALID, "null pointer argument");
    if (max_blocks_per_seq < 1) return fail(PA_ERR_INVALID, "max_blocks_per_seq < 1");
    const int threads = 256;
    const int gx = (int)std::max<int64_t>(1, std::min<int64_t>(((int64_t)max_query_len + threads - 1) / threads, 1024));
    pa::prefill_slot_mapping_kernel<<<dim3(gx, num_seqs), threads, 0, static_cast<cudaStream_t>(stream)>>>(
        slot_mapping, total_q, query_start, block_tables, max_blocks_per_seq, context_lens, cache.block_size,
        cache.num_blocks);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prefill_slot_mapping_kernel launch");
    return ok();
}

extern "C" int pa_paged_prefill(void *out, const void *query, const int32_t *query_start,
                                const void *key_cache, const void *value_cache, pa_cache_desc cache,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *context_lens, int num_seqs, int total_q, int max_query_len,
                                float scale, void *stream) {
    int rc = check_cache(cache);
    if (rc) return rc;
    if (cache.dtype != PA_F16) return fail(PA_ERR_DTYPE, "paged prefill supports fp16 caches only");
    if (num_seqs < 0 || num_seqs > 65535) return fail(PA_ERR_INVALID, "num_seqs %d not in [0, 65535]", num_seqs);
    if (total_q < 0) return fail(PA_ERR_INVALID, "total_q %d < 0", total_q);
    if (max_query_len < 0) return fail(PA_ERR_INVALID, "max_query_len %d < 0", max_query_len);
    if (num_seqs == 0 || total_q == 0 || max_query_len == 0) return ok();
    if (!out || !query || !query_start || !key_cache || !value_cache || !block_tables || !context_lens)
        return fail(PA_ERR_INVALID, "null pointer argument");
    if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
        return fail(PA_ERR_INVALID, "out, query and caches must be 16-byte aligned");
    if (max_blocks_per_seq < 1) return fail(PA_ERR_INVALID, "max_blocks_per_seq %d < 1", max_blocks_per_seq);
    if ((int64_t)max_blocks_per_seq * cache.block_size >= (int64_t(1) << 31))
        return fail(PA_ERR_OVERFLOW, "max_blocks_per_seq * block_size overflows int32");
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID, "scale is not finite");
    // head_size 64 or 128 with a positive scale: the tcgen05 kernel (128-row
    // tiles, S and O in tensor memory); otherwise the mma.sync kernel (64-row
    // tiles).
    const bool tc = (cache.head_size == 64 || cache.head_size == 128) && scale > 0.f;
    const int rows_per_cta = tc ? pa::kTcRows : pa::kPrefillRows;
    const int64_t row_tiles = ((int64_t)max_query_len + rows_per_cta - 1) / rows_per_cta;
    const int64_t n_ctas = row_tiles * num_seqs * cache.num_heads;
    if (n_ctas > 0x7fffffff) return fail(PA_ERR_INVALID, "too many prefill tiles (%lld)", (long long)n_ctas);
    int dev = 0;
    rc = current_device(&dev);
    if (rc) return rc;
    PrefillKernel kern = tc ? pick_prefill_tc(cache.head_size, cache.block_size)
                            : pick_prefill(cache.head_size, cache.block_size);
    rc = ensure_smem_attr(reinterpret_cast<const void *>(kern), dev);
    if (rc) return rc;
    CUtensorMap mk, mv;
    rc = cache_tensor_map(key_cache, cache, 1, &mk, 1);
    if (rc) return rc;
    rc = cache_tensor_map(value_cache, cache, 1, &mv, 1);
    if (rc) return rc;
    pa::PrefillParams p{};
    p.out = static_cast<__half *>(out);
    p.query = static_cast<const __half *>(query);
    p.query_start = query_start;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.num_seqs = num_seqs;
    p.total_q = total_q;
    p.num_heads = cache.num_heads;
    p.num_blocks = cache.num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_query_len = max_query_len;
    p.row_tiles = (int)row_tiles;
    p.stages = prefill_stages(cache);
    p.qk_scale_log2 = scale * pa::kLog2e;
    // ring (or tcgen05 tiles) + barriers + 1 KiB to align to 1024 bytes in the kernel
    const size_t smem = tc ? (size_t)(cache.head_size == 64 ? pa::TcLayout<64>::kBytes : pa::TcLayout<128>::kBytes) + 1024
                           : (size_t)p.stages * 4 * cache.block_size * cache.head_size + 16 * (size_t)p.stages + 1024;
    kern<<<dim3((unsigned)n_ctas), dim3(tc ? pa::kTcThreads : 32 * 5), smem, static_cast<cudaStream_t>(stream)>>>(
        mk, mv, p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "paged_prefill_kernel launch");
    return ok();
}
