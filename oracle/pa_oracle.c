/*
 * pa_oracle.c — plain, slow, fp64 CPU oracle for the paged KV-cache decode
 * path. TEST INFRASTRUCTURE: only the tests, the smoke check and the bench's
 * CPU-baseline / reference arm load it; the product library never does, and
 * this file shares no code, header or table with the CUDA sources.
 *
 * Every function is the plain definition of its operation, written from the
 * pages (page title, section):
 *   [P1] "PagedAttention：大模型推理性能优化的核心技术解析", § 核心工作机制与创新
 *   [P2] "AI 推理系列（十六）：PagedAttention——为什么 vLLM 能把 GPU 显存
 *        “像操作系统一样”管理？", § PagedAttention 如何把连续序列映射到离散显存块
 *        (block table example, flowchart), § Copy-on-Write、并行采样与 Prefix
 *        Caching 不是同一件事, § 非连续 KV 为什么需要专门的 Attention Kernel
 *   [P3] "PagedAttention原理详解：GPU显存优化与模型路由技术", § 显存消耗的三大来源,
 *        § PagedAttention的三大核心优势
 *
 * Cache layout, re-derived here from its written definition (not from the
 * CUDA sources): cache[num_blocks][num_kv_heads][block_size][head_dim]; token
 * position t of a sequence lives in block table[t / block_size], slot
 * t % block_size. Element types: 0 = binary32, 1 = bfloat16 (the upper half
 * of a binary32). All arithmetic is double precision, in one pass, with no
 * partitioning, blocking or reordering.
 *
 * Pins (what checks this file against something other than itself) live in
 * tests/test_oracle_pins.py: contiguous attention through a library routine,
 * golden layout fixtures, placement invariance, prefix sharing, closed forms.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_OK 0
#define OR_ERR_ARG (-1)
#define OR_ERR_INDEX (-2)
#define OR_ERR_NOMEM (-3)

static size_t elem_bytes(int32_t dtype) { return dtype == 0 ? 4u : 2u; }

/* Widen one stored element to double. bfloat16 -> binary32 is exact: the 16
 * stored bits become the high half of the binary32 pattern. */
static double load_elem(const void* base, int64_t idx, int32_t dtype) {
    float f;
    if (dtype == 0) {
        memcpy(&f, (const char*)base + 4 * idx, 4);
    } else {
        uint16_t h;
        uint32_t u;
        memcpy(&h, (const char*)base + 2 * idx, 2);
        u = ((uint32_t)h) << 16;
        memcpy(&f, &u, 4);
    }
    return (double)f;
}

static int shape_ok(int32_t num_blocks, int32_t num_kv_heads, int32_t block_size,
                    int32_t head_dim, int32_t dtype) {
    return num_blocks > 0 && num_kv_heads > 0 && block_size > 0 && head_dim > 0 &&
           (dtype == 0 || dtype == 1);
}

/*
 * Append ("追加 KV", [P2] flowchart): tokens in order i = 0..num_tokens-1; a
 * negative slot is padding and is skipped; otherwise (block, offset) =
 * (slot / block_size, slot % block_size) and the token's vector for every kv
 * head is copied bit for bit into that slot.
 */
int oracle_kv_append(const void* k, const void* v, const int64_t* slot_mapping,
                     int32_t num_tokens, void* k_cache, void* v_cache,
                     int32_t num_blocks, int32_t num_kv_heads, int32_t block_size,
                     int32_t head_dim, int32_t dtype) {
    if (num_tokens < 0 || !shape_ok(num_blocks, num_kv_heads, block_size, head_dim, dtype))
        return OR_ERR_ARG;
    const size_t e = elem_bytes(dtype);
    const size_t vec = (size_t)head_dim * e;
    for (int32_t i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        if (block >= num_blocks) return OR_ERR_INDEX;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            size_t src = ((size_t)i * num_kv_heads + h) * vec;
            size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) * vec;
            memcpy((char*)k_cache + dst, (const char*)k + src, vec);
            memcpy((char*)v_cache + dst, (const char*)v + src, vec);
        }
    }
    return OR_OK;
}

/*
 * Copy-on-write block copy ([P1] § 2 写入时拷贝, [P2] § Copy-on-Write, [P3]
 * § 三大核心优势): every pair (src, dst) gives dst the full contents of src —
 * all slots, all kv heads, K and V. Sources are read before any destination
 * is written, which is the meaning of a set of simultaneous copies.
 */
int oracle_block_copy(const int64_t* pairs, int32_t num_pairs, void* k_cache,
                      void* v_cache, int32_t num_blocks, int32_t num_kv_heads,
                      int32_t block_size, int32_t head_dim, int32_t dtype) {
    if (num_pairs < 0 || !shape_ok(num_blocks, num_kv_heads, block_size, head_dim, dtype))
        return OR_ERR_ARG;
    if (num_pairs == 0) return OR_OK;
    const size_t block_bytes =
        (size_t)num_kv_heads * block_size * head_dim * elem_bytes(dtype);
    for (int32_t p = 0; p < num_pairs; ++p) {
        if (pairs[2 * p] < 0 || pairs[2 * p] >= num_blocks || pairs[2 * p + 1] < 0 ||
            pairs[2 * p + 1] >= num_blocks)
            return OR_ERR_INDEX;
    }
    char* snap = (char*)malloc(2 * block_bytes * (size_t)num_pairs);
    if (!snap) return OR_ERR_NOMEM;
    for (int32_t p = 0; p < num_pairs; ++p) {
        size_t src = (size_t)pairs[2 * p] * block_bytes;
        memcpy(snap + (2 * (size_t)p) * block_bytes, (const char*)k_cache + src, block_bytes);
        memcpy(snap + (2 * (size_t)p + 1) * block_bytes, (const char*)v_cache + src, block_bytes);
    }
    for (int32_t p = 0; p < num_pairs; ++p) {
        size_t dst = (size_t)pairs[2 * p + 1] * block_bytes;
        memcpy((char*)k_cache + dst, snap + (2 * (size_t)p) * block_bytes, block_bytes);
        memcpy((char*)v_cache + dst, snap + (2 * (size_t)p + 1) * block_bytes, block_bytes);
    }
    free(snap);
    return OR_OK;
}

/*
 * Swap of whole blocks between two pools of one block shape ([P2] § 生产环境
 * monitoring list: CPU offload / swap of KV blocks): every pair (src, dst)
 * gives block dst of the destination pool the full contents of block src of
 * the source pool, K and V. The pools are distinct memory, so the pairs are
 * independent copies.
 */
int oracle_block_swap(const int64_t* pairs, int32_t num_pairs, const void* src_k,
                      const void* src_v, int32_t src_blocks, void* dst_k, void* dst_v,
                      int32_t dst_blocks, int32_t num_kv_heads, int32_t block_size,
                      int32_t head_dim, int32_t dtype) {
    if (num_pairs < 0 || !shape_ok(src_blocks, num_kv_heads, block_size, head_dim, dtype) ||
        !shape_ok(dst_blocks, num_kv_heads, block_size, head_dim, dtype))
        return OR_ERR_ARG;
    const size_t block_bytes =
        (size_t)num_kv_heads * block_size * head_dim * elem_bytes(dtype);
    for (int32_t p = 0; p < num_pairs; ++p) {
        if (pairs[2 * p] < 0 || pairs[2 * p] >= src_blocks || pairs[2 * p + 1] < 0 ||
            pairs[2 * p + 1] >= dst_blocks)
            return OR_ERR_INDEX;
    }
    for (int32_t p = 0; p < num_pairs; ++p) {
        const size_t from = (size_t)pairs[2 * p] * block_bytes;
        const size_t to = (size_t)pairs[2 * p + 1] * block_bytes;
        memcpy((char*)dst_k + to, (const char*)src_k + from, block_bytes);
        memcpy((char*)dst_v + to, (const char*)src_v + from, block_bytes);
    }
    return OR_OK;
}

/*
 * Decode attention for one (sequence, query head), straight from the
 * definition: gather the n logical K and V vectors through the block table
 * ([P2] block-table example: logical block j -> physical table[j]), then
 *   s_t = scale * sum_i q_i K_t,i          (one query, n cached keys, [P3])
 *   w_t = exp(s_t - max_u s_u)
 *   out = sum_t w_t V_t / sum_t w_t
 * The attention formula is the ordinary one ([P2]: paging is a storage and
 * access scheme, not a new attention formula). Query head h reads kv head
 * h / (num_heads / num_kv_heads) (contiguous groups). n == 0 gives zeros.
 */
static int decode_one(double* out, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* table_row, int32_t n,
                      int32_t s, int32_t h, int32_t num_heads, int32_t num_kv_heads,
                      int32_t num_blocks, int32_t block_size, int32_t head_dim,
                      int32_t dtype, double scale) {
    /* s: the row of q and out (the sequence, or the query token) */
    double* o = out + ((size_t)s * num_heads + h) * head_dim;
    for (int32_t i = 0; i < head_dim; ++i) o[i] = 0.0;
    if (n == 0) return OR_OK;
    const int32_t group = num_heads / num_kv_heads;
    const int32_t kh = h / group;
    double* K = (double*)malloc(sizeof(double) * (size_t)n * head_dim);
    double* V = (double*)malloc(sizeof(double) * (size_t)n * head_dim);
    double* w = (double*)malloc(sizeof(double) * (size_t)n);
    double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
    if (!K || !V || !w || !qd) {
        free(K); free(V); free(w); free(qd);
        return OR_ERR_NOMEM;
    }
    int rc = OR_OK;
    for (int32_t t = 0; t < n && rc == OR_OK; ++t) {
        int32_t phys = table_row[t / block_size];
        if (phys < 0 || phys >= num_blocks) {
            rc = OR_ERR_INDEX;
            break;
        }
        int64_t base = (((int64_t)phys * num_kv_heads + kh) * block_size + t % block_size) *
                       (int64_t)head_dim;
        for (int32_t i = 0; i < head_dim; ++i) {
            K[(size_t)t * head_dim + i] = load_elem(k_cache, base + i, dtype);
            V[(size_t)t * head_dim + i] = load_elem(v_cache, base + i, dtype);
        }
    }
    if (rc == OR_OK) {
        for (int32_t i = 0; i < head_dim; ++i)
            qd[i] = load_elem(q, ((int64_t)s * num_heads + h) * head_dim + i, dtype);
        double m = -INFINITY;
        for (int32_t t = 0; t < n; ++t) {
            double dot = 0.0;
            for (int32_t i = 0; i < head_dim; ++i) dot += qd[i] * K[(size_t)t * head_dim + i];
            w[t] = scale * dot;
            if (w[t] > m) m = w[t];
        }
        double l = 0.0;
        for (int32_t t = 0; t < n; ++t) {
            w[t] = exp(w[t] - m);
            l += w[t];
        }
        for (int32_t t = 0; t < n; ++t)
            for (int32_t i = 0; i < head_dim; ++i) o[i] += w[t] * V[(size_t)t * head_dim + i];
        for (int32_t i = 0; i < head_dim; ++i) o[i] /= l;
    }
    free(K); free(V); free(w); free(qd);
    return rc;
}

/*
 * out: double [num_seqs][num_heads][head_dim]. `scale` is the binary32 value
 * the GPU path receives, widened to double. Pairs (s, h) are independent, so
 * the thread count changes the run time and nothing else.
 */
int oracle_decode(double* out, const void* q, const void* k_cache, const void* v_cache,
                  const int32_t* block_tables, int32_t block_table_stride,
                  const int32_t* context_lens, int32_t num_seqs, int32_t num_heads,
                  int32_t num_kv_heads, int32_t num_blocks, int32_t block_size,
                  int32_t head_dim, int32_t dtype, float scale, int32_t num_threads) {
    if (num_seqs < 0 || num_heads <= 0 ||
        !shape_ok(num_blocks, num_kv_heads, block_size, head_dim, dtype) ||
        num_heads % num_kv_heads != 0 || block_table_stride < 0)
        return OR_ERR_ARG;
    for (int32_t s = 0; s < num_seqs; ++s) {
        int32_t n = context_lens[s];
        if (n < 0 || (int64_t)n > (int64_t)block_table_stride * block_size) return OR_ERR_ARG;
    }
    const int64_t pairs = (int64_t)num_seqs * num_heads;
    int rc = OR_OK;
    if (num_threads < 1) num_threads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads)
#endif
    for (int64_t idx = 0; idx < pairs; ++idx) {
        int32_t s = (int32_t)(idx / num_heads);
        int32_t h = (int32_t)(idx % num_heads);
        int r = decode_one(out, q, k_cache, v_cache,
                           block_tables + (size_t)s * block_table_stride, context_lens[s], s, h,
                           num_heads, num_kv_heads, num_blocks, block_size, head_dim, dtype,
                           (double)scale);
        if (r != OR_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
            rc = r;
        }
    }
    return rc;
}

/*
 * Several new query tokens per sequence (chunked prefill / verification of
 * draft tokens, [P2] § 如何判断服务瓶颈是否真的来自 PagedAttention names chunked
 * prefill): sequence s owns q / out rows query_start[s] .. query_start[s+1]-1;
 * those n tokens are the last n of its context_lens[s] positions, so row
 * query_start[s] + j is the query at position p = ctx - n + j and sees keys
 * 0 .. p (causal), i.e. exactly the single-query decode above with the
 * context cut at p + 1. p < 0 (more query tokens than context) is an error.
 */
int oracle_decode_multi(double* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int32_t block_table_stride,
                        const int32_t* context_lens, const int32_t* query_start,
                        int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                        int32_t num_blocks, int32_t block_size, int32_t head_dim, int32_t dtype,
                        float scale, int32_t num_threads) {
    if (num_seqs < 0 || num_heads <= 0 ||
        !shape_ok(num_blocks, num_kv_heads, block_size, head_dim, dtype) ||
        num_heads % num_kv_heads != 0 || block_table_stride < 0 || query_start[0] != 0)
        return OR_ERR_ARG;
    for (int32_t s = 0; s < num_seqs; ++s) {
        int32_t n = query_start[s + 1] - query_start[s];
        if (n < 0 || n > context_lens[s] ||
            (int64_t)context_lens[s] > (int64_t)block_table_stride * block_size)
            return OR_ERR_ARG;
    }
    const int64_t rows = query_start[num_seqs];
    const int64_t pairs = rows * num_heads;
    int rc = OR_OK;
    if (num_threads < 1) num_threads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads)
#endif
    for (int64_t idx = 0; idx < pairs; ++idx) {
        int32_t row = (int32_t)(idx / num_heads);
        int32_t h = (int32_t)(idx % num_heads);
        int32_t s = 0;
        while (query_start[s + 1] <= row) ++s;          /* the sequence holding this row */
        int32_t n = query_start[s + 1] - query_start[s];
        int32_t pos = context_lens[s] - n + (row - query_start[s]);
        int r = decode_one(out, q, k_cache, v_cache,
                           block_tables + (size_t)s * block_table_stride, pos + 1, row, h,
                           num_heads, num_kv_heads, num_blocks, block_size, head_dim, dtype,
                           (double)scale);
        if (r != OR_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
            rc = r;
        }
    }
    return rc;
}

/* Threads OpenMP would use by default (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
