// pa_api.cpp — the C ABI declared in include/pa.h: argument validation,
// partition policy, workspace carving and dispatch to the kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "pa.h"
#include "pa_internal.h"
#include "pa_test.h"

namespace {

thread_local std::string t_last_error;
thread_local int t_last_kernel = -1;  // PA_KERNEL_* of the last decode enqueued here
int g_test_skip_position = -1;  // set only by pa_test_skip_load

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return code;
}

int fail_cuda(cudaError_t e, const char* what) {
    return fail(PA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ilog2_exact(int x) {
    int l = 0;
    while ((1 << l) < x) ++l;
    return (1 << l) == x ? l : -1;
}

int elem_bytes(int dtype) { return dtype == PA_F32 ? 4 : dtype == PA_BF16 ? 2 : 1; }

bool quantised(int dtype) { return dtype == PA_FP8_E4M3 || dtype == PA_INT8; }

// Shape checks shared by every call.
int check_cache(const pa_cache_desc* c) {
    if (!c) return fail(PA_ERR_INVALID_ARG, "cache descriptor is NULL");
    if (c->dtype != PA_F32 && c->dtype != PA_BF16 && !quantised(c->dtype))
        return fail(PA_ERR_DTYPE, "dtype %d is not PA_F32, PA_BF16, PA_FP8_E4M3 or PA_INT8",
                    c->dtype);
    if (c->num_blocks <= 0 || c->num_kv_heads <= 0)
        return fail(PA_ERR_INVALID_ARG, "num_blocks (%d) and num_kv_heads (%d) must be positive",
                    c->num_blocks, c->num_kv_heads);
    if (c->head_dim != 64 && c->head_dim != 128)
        return fail(PA_ERR_UNSUPPORTED, "head_dim %d not compiled (64 or 128)", c->head_dim);
    const int lg = ilog2_exact(c->block_size);
    if (c->block_size < 16 || c->block_size > 256 || lg < 0)
        return fail(PA_ERR_UNSUPPORTED, "block_size %d must be a power of two in [16, 256]",
                    c->block_size);
    if ((int64_t)c->num_blocks * c->num_kv_heads * c->block_size > (int64_t)INT32_MAX)
        return fail(PA_ERR_UNSUPPORTED, "pool of %d blocks x %d kv heads x %d slots exceeds 2^31 "
                    "rows", c->num_blocks, c->num_kv_heads, c->block_size);
    return PA_OK;
}

pa::CopyParams copy_params(const pa_cache_desc* c) {
    pa::CopyParams cp;
    cp.num_blocks = c->num_blocks;
    cp.num_kv_heads = c->num_kv_heads;
    cp.block_size = c->block_size;
    cp.log2_block_size = ilog2_exact(c->block_size);
    cp.row_vecs = c->head_dim * elem_bytes(c->dtype) / 16;
    return cp;
}

int sm_count() {
    static int cache[128];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// ---- TMA tensor maps -------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// The pool as a 2-D tensor [num_blocks * num_kv_heads * block_size rows][head_dim],
// loaded in boxes of 16 rows x 128 bytes with the 128-byte swizzle. A head_dim 64
// pool of one-byte codes has 64-byte rows: its box still spans 128 codes, the TMA
// fills the 64 past the row's end with zero codes without reading memory, and
// the consumers over codes (built for 128-code rows) take the padding as zeros.
int make_cache_map(CUtensorMap* map, const void* base, const pa_cache_desc* c) {
    auto fn = encode_fn();
    if (!fn) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    const int e = elem_bytes(c->dtype);
    cuuint64_t dims[2] = {(cuuint64_t)c->head_dim,
                          (cuuint64_t)c->num_blocks * c->num_kv_heads * c->block_size};
    cuuint64_t strides[1] = {(cuuint64_t)c->head_dim * e};
    cuuint32_t box[2] = {(cuuint32_t)(128 / e), 16u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, c->dtype == PA_BF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                         : c->dtype == PA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                              : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                    2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PA_OK;
}

constexpr int kMaxPartitions = 4096;
constexpr int kAutoPartition = 512;    // CUDA-core kernel: partition when splitting
constexpr double kMmaItemOverhead = 8.0; // tensor-core kernel: per-item cost, in 16-token sub-tiles
constexpr int kMinPartition = 256;       // tensor-core kernel: smallest partition

struct Plan {
    bool use_mma;
    bool grouped;       // the grouped kernel (group_size > 1 and supported, or multi-token)
    bool multi;         // several query tokens per sequence (pa_decode_multi)
    int group_size;     // members per grouped item: sequences, or query tokens of one sequence
    int q_chunks;       // multi: items per (sequence, kv head, partition) = ceil(max_query_len / gs)
    int partition_size;
    int num_partitions;
    size_t ws_bytes;      // partial results: the least workspace the call accepts
    size_t ws_ml_offset;
    size_t sched_offset;  // persistent kernels: the dynamic schedule's counter
    size_t ws_full;       // the workspace size reported: partials + schedule
};

int round_up16(int x) { return (x + 15) / 16 * 16; }

// Partition policy: split the context only when the (sequence, head) work
// units alone cannot fill the GPU, then into 512-token partitions.
// num_query_tokens >= 0 selects the multi-token mode (pa_decode_multi): query
// tokens of one sequence are grouped (at most 8, at most 64 query columns).
int plan_decode(int32_t num_seqs, int32_t num_heads, int32_t max_ctx, const pa_cache_desc* c,
                int32_t partition_size, Plan* plan, int32_t group_size = 1,
                int32_t num_query_tokens = -1, int32_t max_query_len = 0) {
    int rc = check_cache(c);
    if (rc != PA_OK) return rc;
    if (num_seqs < 0 || num_seqs > 65535)
        return fail(PA_ERR_INVALID_ARG, "num_seqs %d outside [0, 65535]", num_seqs);
    if (num_heads <= 0 || num_heads > 65535 || num_heads % c->num_kv_heads != 0)
        return fail(PA_ERR_INVALID_ARG, "num_heads %d must be positive and a multiple of "
                    "num_kv_heads %d", num_heads, c->num_kv_heads);
    if (max_ctx < 0) return fail(PA_ERR_INVALID_ARG, "max_context_len %d is negative", max_ctx);
    const int group = num_heads / c->num_kv_heads;
    if (group_size < 1 || group_size > 8)
        return fail(PA_ERR_INVALID_ARG, "group_size %d outside [1, 8]", group_size);
    plan->multi = num_query_tokens >= 0;
    plan->q_chunks = 1;
    if (plan->multi) {
        if (max_query_len < 1 || max_query_len > num_query_tokens + (num_query_tokens == 0))
            return fail(PA_ERR_INVALID_ARG, "max_query_len %d must be in [1, num_query_tokens %d]",
                        max_query_len, num_query_tokens);
        int gs = max_query_len < 8 ? max_query_len : 8;
        const int max_cols = pa::grouped_max_cols(c->dtype, c->head_dim, group);
        while (gs > 1 && gs * group > max_cols) --gs;
        if (pa::grouped_supported(c->dtype, c->head_dim, group, gs)) {
            group_size = gs;
            plan->q_chunks = (max_query_len + gs - 1) / gs;
            plan->grouped = true;
        } else {
            // fp32 caches, or query groups above 64 columns: one query token per
            // row of the CUDA-core consumer, which reads its sequence's blocks
            group_size = 1;
            plan->grouped = false;
        }
    } else {
        plan->grouped =
            group_size > 1 && pa::grouped_supported(c->dtype, c->head_dim, group, group_size);
    }
    plan->group_size = group_size;
    if (plan->grouped && max_ctx > (1 << 27))
        return fail(PA_ERR_INVALID_ARG, "max_context_len %d above 2^27 on the grouped kernel", max_ctx);
    // the tensor-core GQA consumer takes one query row per sequence
    plan->use_mma = !plan->multi && pa::mma_supported(c->dtype, c->head_dim, group);
    const int whole = round_up16(max_ctx > 16 ? max_ctx : 16);
    int ps = whole, np = 1;
    if (partition_size > 0) {
        if (partition_size % 16 != 0)
            return fail(PA_ERR_INVALID_ARG, "partition_size %d is not a multiple of 16",
                        partition_size);
        ps = partition_size;
        np = (max_ctx + ps - 1) / ps;
        if (np < 1) np = 1;
        if (np > kMaxPartitions)
            return fail(PA_ERR_INVALID_ARG, "partition_size %d gives %d partitions (max %d)",
                        partition_size, np, kMaxPartitions);
    } else if (partition_size == 0) {
        if (plan->use_mma || plan->grouped) {
            // The persistent tensor-core kernel hands items to its CTA slots statically
            // (item u to CTA u mod slots), so its time is about
            //   waves * (sub-tiles per item + per-item overhead),  waves = ceil(items / slots),
            // the overhead being the item's merge, partial write and share of the reduce.
            // Pick the partition count with the smallest such cost (ties: fewer partitions),
            // partitions cut equal and at least kMinPartition tokens long.
            // The grouped kernel is persistent the same way; its unit is a group.
            const long units =
                plan->multi     ? (long)num_seqs * plan->q_chunks * c->num_kv_heads
                : plan->grouped ? (long)((num_seqs + group_size - 1) / group_size) * c->num_kv_heads
                                : (long)num_seqs * c->num_kv_heads;
            const long slots =
                (long)sm_count() * (plan->grouped ? pa::grouped_ctas_per_sm(c->dtype, c->head_dim, group_size, group)
                                                  : pa::mma_ctas_per_sm());
            long most = (max_ctx + kMinPartition - 1) / kMinPartition;
            if (most > kMaxPartitions) most = kMaxPartitions;
            if (most < 1) most = 1;
            long best_np = 1, best_ps = whole;
            double best_cost = -1.0;
            // (Also under the GQA kernel's dynamic schedule: a model of balanced
            // items, items x (sub-tiles + overhead) / slots + a tail, ranked the
            // 70B-GQA sweep well for bf16 (16 partitions 168.4 us vs 9: 170.4) but
            // not over codes (fp8: 9 partitions 98.8 us, 16: 106.9), and a few
            // items more than slots leave CTAs running a second item alone at the
            // end; the waves model picks 9 for both.)
            for (long n = 1; n <= most; ++n) {
                const int cand_ps = round_up16((int)((max_ctx + n - 1) / n));
                const long cand_np = (max_ctx + cand_ps - 1) / cand_ps;
                if (cand_np != n) continue;  // rounding merged two cuts: seen already
                const long items = units * cand_np;
                const long waves = (items + slots - 1) / slots;
                const double cost =
                    (double)waves * ((double)(cand_np == 1 ? whole : cand_ps) / 16.0 +
                                     (cand_np == 1 ? 0.0 : kMmaItemOverhead));
                if (best_cost < 0.0 || cost < best_cost) {
                    best_cost = cost;
                    best_np = cand_np;
                    best_ps = cand_ps;
                }
            }
            np = (int)best_np;
            ps = np == 1 ? whole : (int)best_ps;
        } else {
            // The CUDA-core kernel is not persistent: split only when the
            // (row, head) units alone cannot fill the GPU.
            const long units = (long)(plan->multi ? num_query_tokens : num_seqs) * num_heads;
            if (units < 4L * sm_count() && max_ctx > kAutoPartition) {
                ps = kAutoPartition;
                np = (max_ctx + ps - 1) / ps;
                while (np > kMaxPartitions) {
                    ps *= 2;
                    np = (max_ctx + ps - 1) / ps;
                }
            }
        }
    } else if (partition_size != -1) {
        return fail(PA_ERR_INVALID_ARG, "partition_size %d: use 0 (policy), -1 (no split) or a "
                    "positive multiple of 16", partition_size);
    }
    plan->partition_size = np == 1 ? whole : ps;
    plan->num_partitions = np;
    if (np == 1) {
        plan->ws_bytes = 0;
        plan->ws_ml_offset = 0;
    } else {
        const size_t rows =
            (size_t)(plan->multi ? num_query_tokens : num_seqs) * num_heads * np;
        const size_t o_bytes = rows * c->head_dim * sizeof(float);
        plan->ws_ml_offset = (o_bytes + 255) / 256 * 256;
        plan->ws_bytes = plan->ws_ml_offset + rows * 2 * sizeof(float);
    }
    // The persistent tensor-core GQA kernel claims its work items from a counter
    // in the 256 bytes after the partials (zeroed by the call before it
    // launches); a workspace without them runs the static schedule. (The
    // grouped kernel keeps its static schedule: its items are few and long, one
    // or two per CTA at the measured workloads, so a claim's latency at each
    // item start cost more than balancing gained: 4-beam CoW 94.9 vs 90.2 us,
    // 4-token verification 214.5 vs 212 us.)
    plan->sched_offset = (plan->ws_bytes + 255) / 256 * 256;
    plan->ws_full = plan->use_mma && !plan->grouped ? plan->sched_offset + 256 : plan->ws_bytes;
    return PA_OK;
}

}  // namespace

int pa::report_error(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return code;
}

// num_query_tokens >= 0: multi-token queries (query_start [num_seqs + 1]).
static int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, int32_t block_table_stride,
                       const int32_t* context_lens, int32_t max_context_len, int32_t num_seqs,
                       int32_t num_heads, float scale, const pa_cache_desc* cache,
                       int32_t group_size, int32_t partition_size, void* workspace,
                       size_t workspace_bytes, void* stream, const int32_t* query_start = nullptr,
                       int32_t num_query_tokens = -1, int32_t max_query_len = 0,
                       const float* k_scale = nullptr, const float* v_scale = nullptr) {
    Plan plan;
    if (cache && quantised(cache->dtype) != (k_scale != nullptr || v_scale != nullptr))
        return fail(PA_ERR_DTYPE, quantised(cache->dtype)
                                      ? "a quantised cache decodes through pa_decode_quant"
                                      : "pa_decode_quant needs a PA_FP8_E4M3 or PA_INT8 cache");
    if (cache && quantised(cache->dtype)) {
        if (!k_scale || !v_scale ||
            (reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u))
            return fail(PA_ERR_INVALID_ARG, "pa_decode_quant: k_scale and v_scale must be 4-byte "
                        "aligned device arrays of num_kv_heads floats");
    }
    if (num_query_tokens > 65535)
        return fail(PA_ERR_INVALID_ARG, "num_query_tokens %d above 65535", num_query_tokens);
    int rc = plan_decode(num_seqs, num_heads, max_context_len, cache, partition_size, &plan,
                         group_size, num_query_tokens, max_query_len);
    if (rc != PA_OK) return rc;
    if (num_seqs == 0 || num_query_tokens == 0) return PA_OK;
    if (plan.multi && (!query_start || (reinterpret_cast<uintptr_t>(query_start) & 3u) != 0))
        return fail(PA_ERR_INVALID_ARG, "pa_decode_multi: query_start must be a 4-byte aligned "
                    "device array of num_seqs + 1 entries");
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return fail(PA_ERR_INVALID_ARG, "pa_decode: NULL pointer argument");
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_ALIGN, "pa_decode: out, q and the caches must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(block_tables) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(context_lens) & 3u) != 0)
        return fail(PA_ERR_ALIGN, "pa_decode: block_tables / context_lens must be 4-byte aligned");
    if (block_table_stride < 0 ||
        (int64_t)block_table_stride * cache->block_size < (int64_t)max_context_len)
        return fail(PA_ERR_INVALID_ARG, "max_context_len %d exceeds block_table_stride %d * "
                    "block_size %d", max_context_len, block_table_stride, cache->block_size);
    if (!std::isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "scale is not finite");
    const bool ws_aligned = (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0;
    if (plan.ws_bytes > 0) {
        if (!workspace || workspace_bytes < plan.ws_bytes)
            return fail(PA_ERR_WORKSPACE, "pa_decode needs %zu workspace bytes, got %zu at %p",
                        plan.ws_bytes, workspace_bytes, workspace);
        if (!ws_aligned) return fail(PA_ERR_ALIGN, "pa_decode: workspace must be 256-byte aligned");
    }
    // the dynamic schedule when the workspace holds its counter and there are
    // at least two items per CTA slot: with fewer there is little to balance and
    // a claim only adds its latency (measured, claimed vs static: 70B-GQA at 9
    // partitions, one item per slot, 172.6 vs 170.5-171.6 us; 4-beam CoW per
    // sequence, 1.7 per slot, 111.0 vs 108.8; 256 x 1K, 3.5 per slot, 163.9 vs
    // 172.5; 70B at 512-token partitions, 6.9 per slot, 178.6 vs 186.7). The
    // results are the same bit for bit either way: an item's arithmetic does not
    // depend on the CTA that runs it.
    const long mma_items = (long)plan.num_partitions * cache->num_kv_heads * num_seqs;
    const bool dyn_sched = plan.ws_full > plan.ws_bytes && workspace && ws_aligned &&
                           workspace_bytes >= plan.ws_full &&
                           mma_items >= 2L * sm_count() * pa::mma_ctas_per_sm();
    pa::DecodeParams p;
    p.out = out;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.ws_o = plan.ws_bytes ? static_cast<float*>(workspace) : nullptr;
    p.ws_ml = plan.ws_bytes
                  ? reinterpret_cast<float*>(static_cast<char*>(workspace) + plan.ws_ml_offset)
                  : nullptr;
    p.table_stride = block_table_stride;
    p.max_context_len = max_context_len;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = cache->num_kv_heads;
    p.num_blocks = cache->num_blocks;
    p.block_size = cache->block_size;
    p.log2_block_size = ilog2_exact(cache->block_size);
    p.partition_size = plan.partition_size;
    p.num_partitions = plan.num_partitions;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.test_skip_position = g_test_skip_position;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.head_dim = cache->head_dim;
    p.query_start = plan.multi ? query_start : nullptr;
    p.q_chunks = plan.q_chunks;
    p.num_rows = plan.multi ? num_query_tokens : num_seqs;
    p.sched = dyn_sched ? reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) +
                                                          plan.sched_offset)
                        : nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (p.sched) {
        const cudaError_t me = cudaMemsetAsync(p.sched, 0, sizeof(unsigned int), st);
        if (me != cudaSuccess) return fail_cuda(me, "pa_decode schedule reset");
    }
    CUtensorMap kmap, vmap;
    if ((rc = make_cache_map(&kmap, k_cache, cache)) != PA_OK) return rc;
    if ((rc = make_cache_map(&vmap, v_cache, cache)) != PA_OK) return rc;
    cudaError_t e =
        plan.grouped
            ? pa::launch_decode_grouped(p, cache->dtype, cache->head_dim, plan.group_size, kmap, vmap, st)
            : pa::launch_decode_tma(p, cache->dtype, cache->head_dim, plan.use_mma, kmap, vmap, st);
    if (e != cudaSuccess) return fail_cuda(e, "pa_decode launch");
    t_last_kernel = !plan.grouped ? (plan.use_mma ? PA_KERNEL_MMA : PA_KERNEL_SIMT)
                    : pa::grouped_is_tcgen05(cache->dtype, cache->head_dim, plan.group_size,
                                             num_heads / cache->num_kv_heads)
                        ? PA_KERNEL_GROUPED_TCGEN05
                        : PA_KERNEL_GROUPED;
    if (plan.num_partitions > 1) {
        e = pa::launch_partition_reduce(p, cache->dtype, cache->head_dim, st);
        if (e != cudaSuccess) return fail_cuda(e, "pa_decode reduce launch");
    }
    return PA_OK;
}

extern "C" {

int pa_kv_append(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                 void* k_cache, void* v_cache, const pa_cache_desc* cache, void* stream) {
    int rc = check_cache(cache);
    if (rc != PA_OK) return rc;
    if (quantised(cache->dtype))
        return fail(PA_ERR_DTYPE, "a quantised cache is written through pa_kv_append_quant");
    if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens %d is negative", num_tokens);
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache)
        return fail(PA_ERR_INVALID_ARG, "pa_kv_append: NULL pointer argument");
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_ALIGN, "pa_kv_append: k, v and the caches must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(slot_mapping) & 7u) != 0)
        return fail(PA_ERR_ALIGN, "pa_kv_append: slot_mapping must be 8-byte aligned");
    cudaError_t e = pa::launch_kv_append(k, v, slot_mapping, num_tokens, k_cache, v_cache,
                                         copy_params(cache), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e, "pa_kv_append launch");
}

int pa_kv_append_quant(const void* k, const void* v, const int64_t* slot_mapping,
                       int32_t num_tokens, void* k_cache, void* v_cache, const float* k_scale,
                       const float* v_scale, const pa_cache_desc* cache, void* stream) {
    int rc = check_cache(cache);
    if (rc != PA_OK) return rc;
    if (!quantised(cache->dtype))
        return fail(PA_ERR_DTYPE, "pa_kv_append_quant needs a PA_FP8_E4M3 or PA_INT8 cache");
    if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "num_tokens %d is negative", num_tokens);
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale)
        return fail(PA_ERR_INVALID_ARG, "pa_kv_append_quant: NULL pointer argument");
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_ALIGN, "pa_kv_append_quant: k, v and the caches must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(slot_mapping) & 7u) != 0 ||
        (reinterpret_cast<uintptr_t>(k_scale) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(v_scale) & 3u) != 0)
        return fail(PA_ERR_ALIGN, "pa_kv_append_quant: slot_mapping 8-byte, scales 4-byte aligned");
    cudaError_t e = pa::launch_kv_append_quant(k, v, slot_mapping, num_tokens, k_cache, v_cache,
                                               k_scale, v_scale, cache->dtype, copy_params(cache),
                                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e, "pa_kv_append_quant launch");
}

int pa_decode_quant(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const float* k_scale, const float* v_scale, const int32_t* block_tables,
                    int32_t block_table_stride, const int32_t* context_lens,
                    int32_t max_context_len, int32_t num_seqs, int32_t num_heads, float scale,
                    const pa_cache_desc* cache, int32_t partition_size, void* workspace,
                    size_t workspace_bytes, void* stream) {
    if (!k_scale || !v_scale)
        return fail(PA_ERR_INVALID_ARG, "pa_decode_quant: k_scale and v_scale are required");
    return decode_impl(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                       max_context_len, num_seqs, num_heads, scale, cache, 1, partition_size,
                       workspace, workspace_bytes, stream, nullptr, -1, 0, k_scale, v_scale);
}

int pa_block_copy(const int64_t* src_dst_pairs, int32_t num_pairs, void* k_cache, void* v_cache,
                  const pa_cache_desc* cache, void* stream) {
    int rc = check_cache(cache);
    if (rc != PA_OK) return rc;
    if (num_pairs < 0) return fail(PA_ERR_INVALID_ARG, "num_pairs %d is negative", num_pairs);
    if (num_pairs == 0) return PA_OK;
    if (!src_dst_pairs || !k_cache || !v_cache)
        return fail(PA_ERR_INVALID_ARG, "pa_block_copy: NULL pointer argument");
    if (!aligned16(k_cache) || !aligned16(v_cache))
        return fail(PA_ERR_ALIGN, "pa_block_copy: caches must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(src_dst_pairs) & 7u) != 0)
        return fail(PA_ERR_ALIGN, "pa_block_copy: src_dst_pairs must be 8-byte aligned");
    cudaError_t e = pa::launch_block_copy(src_dst_pairs, num_pairs, k_cache, v_cache,
                                          copy_params(cache), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e, "pa_block_copy launch");
}

int pa_block_swap(const int64_t* src_dst_pairs, int32_t num_pairs, const void* src_k,
                  const void* src_v, const pa_cache_desc* src, void* dst_k, void* dst_v,
                  const pa_cache_desc* dst, void* stream) {
    int rc = check_cache(src);
    if (rc != PA_OK) return rc;
    if ((rc = check_cache(dst)) != PA_OK) return rc;
    if (src->num_kv_heads != dst->num_kv_heads || src->block_size != dst->block_size ||
        src->head_dim != dst->head_dim || src->dtype != dst->dtype)
        return fail(PA_ERR_INVALID_ARG, "pa_block_swap: the two pools differ in block shape or dtype");
    if (num_pairs < 0) return fail(PA_ERR_INVALID_ARG, "num_pairs %d is negative", num_pairs);
    if (num_pairs == 0) return PA_OK;
    if (!src_dst_pairs || !src_k || !src_v || !dst_k || !dst_v)
        return fail(PA_ERR_INVALID_ARG, "pa_block_swap: NULL pointer argument");
    if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v))
        return fail(PA_ERR_ALIGN, "pa_block_swap: the pools must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(src_dst_pairs) & 7u) != 0)
        return fail(PA_ERR_ALIGN, "pa_block_swap: src_dst_pairs must be 8-byte aligned");
    const size_t block_bytes =
        (size_t)src->num_kv_heads * src->block_size * src->head_dim * elem_bytes(src->dtype);
    const char* sk = static_cast<const char*>(src_k);
    const char* dk = static_cast<const char*>(dst_k);
    const size_t sbytes = block_bytes * (size_t)src->num_blocks;
    const size_t dbytes = block_bytes * (size_t)dst->num_blocks;
    const char* sv = static_cast<const char*>(src_v);
    const char* dv = static_cast<const char*>(dst_v);
    auto overlap = [](const char* a, size_t na, const char* b, size_t nb) {
        return a < b + nb && b < a + na;
    };
    if (overlap(sk, sbytes, dk, dbytes) || overlap(sk, sbytes, dv, dbytes) ||
        overlap(sv, sbytes, dk, dbytes) || overlap(sv, sbytes, dv, dbytes) ||
        overlap(dk, dbytes, dv, dbytes))
        return fail(PA_ERR_INVALID_ARG, "pa_block_swap: destination caches overlap each other "
                    "or the source pool");
    // every pointer must be addressable by the device: device, managed or pinned host memory
    const void* ptrs[5] = {src_dst_pairs, src_k, src_v, dst_k, dst_v};
    const void* dev[5];
    const char* names[5] = {"src_dst_pairs", "src_k", "src_v", "dst_k", "dst_v"};
    for (int i = 0; i < 5; ++i) {
        cudaPointerAttributes a;
        cudaError_t e = cudaPointerGetAttributes(&a, ptrs[i]);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return fail(PA_ERR_INVALID_ARG, "pa_block_swap: %s is not CUDA-visible memory", names[i]);
        }
        if (a.type == cudaMemoryTypeUnregistered || a.devicePointer == nullptr)
            return fail(PA_ERR_INVALID_ARG, "pa_block_swap: %s is pageable host memory; pin it "
                        "(cudaHostAlloc / cudaHostRegister)", names[i]);
        dev[i] = a.devicePointer;
    }
    cudaError_t e = pa::launch_block_swap(static_cast<const int64_t*>(dev[0]), num_pairs, dev[1],
                                          dev[2], src->num_blocks, const_cast<void*>(dev[3]),
                                          const_cast<void*>(dev[4]), dst->num_blocks,
                                          copy_params(src), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : fail_cuda(e, "pa_block_swap launch");
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t max_context_len,
                                const pa_cache_desc* cache, int32_t partition_size) {
    Plan plan;
    if (plan_decode(num_seqs, num_heads, max_context_len, cache, partition_size, &plan) != PA_OK)
        return 0;
    return plan.ws_full;
}

int pa_decode_num_partitions(int32_t num_seqs, int32_t num_heads, int32_t max_context_len,
                             const pa_cache_desc* cache, int32_t partition_size) {
    Plan plan;
    int rc = plan_decode(num_seqs, num_heads, max_context_len, cache, partition_size, &plan);
    return rc != PA_OK ? rc : plan.num_partitions;
}

int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, int32_t block_table_stride,
              const int32_t* context_lens, int32_t max_context_len, int32_t num_seqs,
              int32_t num_heads, float scale, const pa_cache_desc* cache,
              int32_t partition_size, void* workspace, size_t workspace_bytes, void* stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                       max_context_len, num_seqs, num_heads, scale, cache, 1, partition_size,
                       workspace, workspace_bytes, stream);
}

int pa_decode_grouped(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int32_t block_table_stride,
                      const int32_t* context_lens, int32_t max_context_len, int32_t num_seqs,
                      int32_t num_heads, float scale, const pa_cache_desc* cache,
                      int32_t group_size, int32_t partition_size, void* workspace,
                      size_t workspace_bytes, void* stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                       max_context_len, num_seqs, num_heads, scale, cache, group_size,
                       partition_size, workspace, workspace_bytes, stream);
}

int pa_decode_multi(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t block_table_stride,
                    const int32_t* context_lens, const int32_t* query_start,
                    int32_t max_context_len, int32_t num_seqs, int32_t num_query_tokens,
                    int32_t max_query_len, int32_t num_heads, float scale,
                    const pa_cache_desc* cache, int32_t partition_size, void* workspace,
                    size_t workspace_bytes, void* stream) {
    if (num_query_tokens < 0)
        return fail(PA_ERR_INVALID_ARG, "num_query_tokens %d is negative", num_query_tokens);
    return decode_impl(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                       max_context_len, num_seqs, num_heads, scale, cache, 1, partition_size,
                       workspace, workspace_bytes, stream, query_start, num_query_tokens,
                       max_query_len);
}

int pa_decode_grouped_quant(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const float* k_scale, const float* v_scale,
                            const int32_t* block_tables, int32_t block_table_stride,
                            const int32_t* context_lens, int32_t max_context_len,
                            int32_t num_seqs, int32_t num_heads, float scale,
                            const pa_cache_desc* cache, int32_t group_size,
                            int32_t partition_size, void* workspace, size_t workspace_bytes,
                            void* stream) {
    if (!k_scale || !v_scale)
        return fail(PA_ERR_INVALID_ARG, "pa_decode_grouped_quant: k_scale and v_scale are required");
    return decode_impl(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                       max_context_len, num_seqs, num_heads, scale, cache, group_size,
                       partition_size, workspace, workspace_bytes, stream, nullptr, -1, 0, k_scale,
                       v_scale);
}

int pa_decode_multi_quant(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const float* k_scale, const float* v_scale, const int32_t* block_tables,
                          int32_t block_table_stride, const int32_t* context_lens,
                          const int32_t* query_start, int32_t max_context_len, int32_t num_seqs,
                          int32_t num_query_tokens, int32_t max_query_len, int32_t num_heads,
                          float scale, const pa_cache_desc* cache, int32_t partition_size,
                          void* workspace, size_t workspace_bytes, void* stream) {
    if (!k_scale || !v_scale)
        return fail(PA_ERR_INVALID_ARG, "pa_decode_multi_quant: k_scale and v_scale are required");
    if (num_query_tokens < 0)
        return fail(PA_ERR_INVALID_ARG, "num_query_tokens %d is negative", num_query_tokens);
    return decode_impl(out, q, k_cache, v_cache, block_tables, block_table_stride, context_lens,
                       max_context_len, num_seqs, num_heads, scale, cache, 1, partition_size,
                       workspace, workspace_bytes, stream, query_start, num_query_tokens,
                       max_query_len, k_scale, v_scale);
}

size_t pa_decode_multi_workspace_size(int32_t num_seqs, int32_t num_query_tokens,
                                      int32_t max_query_len, int32_t num_heads,
                                      int32_t max_context_len, const pa_cache_desc* cache,
                                      int32_t partition_size) {
    Plan plan;
    if (num_query_tokens < 0 ||
        plan_decode(num_seqs, num_heads, max_context_len, cache, partition_size, &plan, 1,
                    num_query_tokens, max_query_len) != PA_OK)
        return 0;
    return plan.ws_full;
}

int pa_decode_multi_num_partitions(int32_t num_seqs, int32_t num_query_tokens,
                                   int32_t max_query_len, int32_t num_heads,
                                   int32_t max_context_len, const pa_cache_desc* cache,
                                   int32_t partition_size) {
    if (num_query_tokens < 0)
        return fail(PA_ERR_INVALID_ARG, "num_query_tokens %d is negative", num_query_tokens);
    Plan plan;
    int rc = plan_decode(num_seqs, num_heads, max_context_len, cache, partition_size, &plan, 1,
                         num_query_tokens, max_query_len);
    return rc != PA_OK ? rc : plan.num_partitions;
}

size_t pa_decode_grouped_workspace_size(int32_t num_seqs, int32_t num_heads,
                                        int32_t max_context_len, const pa_cache_desc* cache,
                                        int32_t group_size, int32_t partition_size) {
    Plan plan;
    if (plan_decode(num_seqs, num_heads, max_context_len, cache, partition_size, &plan,
                    group_size) != PA_OK)
        return 0;
    return plan.ws_full;
}

int pa_decode_grouped_num_partitions(int32_t num_seqs, int32_t num_heads,
                                     int32_t max_context_len, const pa_cache_desc* cache,
                                     int32_t group_size, int32_t partition_size) {
    Plan plan;
    int rc = plan_decode(num_seqs, num_heads, max_context_len, cache, partition_size, &plan,
                         group_size);
    return rc != PA_OK ? rc : plan.num_partitions;
}

int pa_set_grouped_consumer(int consumer) {
    if (consumer != PA_GROUPED_MMA_SYNC && consumer != PA_GROUPED_TCGEN05)
        return fail(PA_ERR_INVALID_ARG, "unknown grouped consumer %d", consumer);
    return pa::set_grouped_consumer(consumer);
}

int pa_sync_check(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, "pa_sync_check: stream");
    unsigned a = 0, b = 0;
    if ((e = pa::read_status_copy(&a, true)) != cudaSuccess ||
        (e = pa::read_status_tma(&b, true)) != cudaSuccess)
        return fail_cuda(e, "pa_sync_check: status word");
    if ((a | b) & pa::kStatusSmemAlign)
        return fail(PA_ERR_CUDA, "a decode kernel found its shared memory misaligned and did not run");
    if ((a | b) & pa::kStatusTimeout)
        return fail(PA_ERR_TIMEOUT, "a bounded pipeline wait gave up (bits copy=%u decode=%u)", a, b);
    if ((a | b) & pa::kStatusBadIndex)
        return fail(PA_ERR_BAD_INDEX, "a kernel met a block id, slot or context length outside "
                    "its bounds (bits copy=%u decode=%u)", a, b);
    return PA_OK;
}

const char* pa_get_last_error(void) { return t_last_error.c_str(); }

void pa_test_skip_load(int32_t position) { g_test_skip_position = position < 0 ? -1 : position; }

int pa_test_last_decode_kernel(void) { return t_last_kernel; }

const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_DTYPE: return "PA_ERR_DTYPE";
        case PA_ERR_ALIGN: return "PA_ERR_ALIGN";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_BAD_INDEX: return "PA_ERR_BAD_INDEX";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
        case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT";
        default: return "PA_ERR_UNKNOWN";
    }
}

}  // extern "C"
