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
 * of a binary32), 2 = FP8 E4M3 code, 3 = int8 code (quantised caches, one
 * scale per kv head). All attention arithmetic is double precision, in one
 * pass, with no partitioning, blocking or reordering; a quantiser takes its
 * decision in binary32, the precision the stored code is defined in.
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

/* Element types: 0 binary32, 1 bfloat16, 2 FP8 E4M3 code, 3 int8 code. */
static size_t elem_bytes(int32_t dtype) { return dtype == 0 ? 4u : dtype == 1 ? 2u : 1u; }

/*
 * KV-cache quantisation ([P2] mechanisms table: KV cache quantisation lowers
 * the bits per cached element at the cost of quantisation error and
 * conversion; [P3] § 量化技术: INT8 KV halves KV memory, orthogonal to paging).
 * The pages give no format details; the reading used: one binary32 scale per
 * kv head for K and one for V, supplied by the caller; a stored code c stands
 * for value(c) * scale; a value x is stored as the code of y = x / scale (the
 * division in binary32, as a GPU does it).
 *
 * FP8 E4M3 (the OCP 8-bit format with 4 exponent bits, bias 7, 3 mantissa
 * bits, no infinities; S.1111.111 is NaN): value = (-1)^S 2^(E-7) (1 + M/8)
 * for E > 0, (-1)^S 2^-6 (M/8) for E = 0.
 */
static double e4m3_value(uint8_t c) {
    const int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* y -> E4M3 code: round to nearest, ties to the even code; magnitudes of 448
 * (the largest finite value) and above, infinities included, saturate to
 * +-448; NaN gives the NaN code 0x7F. Plain search over the 127 finite
 * magnitudes. */
static uint8_t e4m3_code(float y) {
    if (isnan(y)) return 0x7F;
    const uint8_t sgn = signbit(y) ? 0x80 : 0x00;
    const double a = fabs((double)y);
    if (a >= 448.0) return sgn | 0x7E;
    uint8_t best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        const double err = fabs(a - e4m3_value((uint8_t)c));
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = (uint8_t)c;
            best_err = err;
        }
    }
    return sgn | best;
}

/* y -> int8 code: clamp to [-127, 127] (fmaxf / fminf: a NaN operand yields
 * the other one), then round to nearest, ties to even. */
static int8_t int8_code(float y) {
    const float c = fminf(fmaxf(y, -127.0f), 127.0f);
    return (int8_t)lrintf(c);
}

/* The stored code of element x (a binary32 value) under `scale`. */
static uint8_t quantize(float x, float scale, int32_t fmt) {
    const float y = x / scale;
    if (fmt == 2) return e4m3_code(y);
    const int8_t q = int8_code(y);
    uint8_t u;
    memcpy(&u, &q, 1);
    return u;
}

/* Widen one stored element to double. bfloat16 -> binary32 is exact: the 16
 * stored bits become the high half of the binary32 pattern. */
static double load_elem(const void* base, int64_t idx, int32_t dtype) {
    float f;
    if (dtype == 2) return e4m3_value(((const uint8_t*)base)[idx]);
    if (dtype == 3) return (double)((const int8_t*)base)[idx];
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
           dtype >= 0 && dtype <= 3;
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
static int decode_one_q(double* out, const void* q, int32_t q_dtype, const void* k_cache,
                        const void* v_cache, const float* k_scale, const float* v_scale,
                        const int32_t* table_row, int32_t n,
                        int32_t s, int32_t h, int32_t num_heads, int32_t num_kv_heads,
                        int32_t num_blocks, int32_t block_size, int32_t head_dim,
                        int32_t dtype, double scale) {
    /* s: the row of q and out (the sequence, or the query token); k_scale /
     * v_scale (per kv head) multiply the stored codes of a quantised cache */
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
        const double ks = k_scale ? (double)k_scale[kh] : 1.0;
        const double vs = v_scale ? (double)v_scale[kh] : 1.0;
        for (int32_t i = 0; i < head_dim; ++i) {
            K[(size_t)t * head_dim + i] = load_elem(k_cache, base + i, dtype) * ks;
            V[(size_t)t * head_dim + i] = load_elem(v_cache, base + i, dtype) * vs;
        }
    }
    if (rc == OR_OK) {
        for (int32_t i = 0; i < head_dim; ++i)
            qd[i] = load_elem(q, ((int64_t)s * num_heads + h) * head_dim + i, q_dtype);
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

static int decode_one(double* out, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* table_row, int32_t n,
                      int32_t s, int32_t h, int32_t num_heads, int32_t num_kv_heads,
                      int32_t num_blocks, int32_t block_size, int32_t head_dim,
                      int32_t dtype, double scale) {
    return decode_one_q(out, q, dtype, k_cache, v_cache, NULL, NULL, table_row, n, s, h,
                        num_heads, num_kv_heads, num_blocks, block_size, head_dim, dtype, scale);
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

/*
 * Quantising append: as oracle_kv_append, but k and v are bfloat16 vectors
 * and each element is stored as its code under the kv head's scale (fmt 2 =
 * FP8 E4M3, 3 = int8).
 */
int oracle_kv_append_quant(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                           int32_t num_tokens, uint8_t* k_cache, uint8_t* v_cache,
                           const float* k_scale, const float* v_scale, int32_t num_blocks,
                           int32_t num_kv_heads, int32_t block_size, int32_t head_dim,
                           int32_t fmt) {
    if (num_tokens < 0 || (fmt != 2 && fmt != 3) ||
        !shape_ok(num_blocks, num_kv_heads, block_size, head_dim, fmt))
        return OR_ERR_ARG;
    for (int32_t i = 0; i < num_tokens; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot <= -1) continue; /* padding token */
        if (slot >= (int64_t)num_blocks * block_size) return OR_ERR_INDEX;
        const int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            const int64_t src = ((int64_t)i * num_kv_heads + h) * head_dim;
            const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
            for (int32_t d = 0; d < head_dim; ++d) {
                k_cache[dst + d] = quantize((float)load_elem(k, src + d, 1), k_scale[h], fmt);
                v_cache[dst + d] = quantize((float)load_elem(v, src + d, 1), v_scale[h], fmt);
            }
        }
    }
    return OR_OK;
}

/* Codes of an array of binary32 values (for the quantiser's own pins). */
int oracle_quantize(const float* x, int64_t n, float scale, int32_t fmt, uint8_t* codes) {
    if (fmt != 2 && fmt != 3) return OR_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) codes[i] = quantize(x[i], scale, fmt);
    return OR_OK;
}

/* Values of an array of codes (fmt 2 or 3), unscaled. */
int oracle_code_values(const uint8_t* codes, int64_t n, int32_t fmt, double* out) {
    if (fmt != 2 && fmt != 3) return OR_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) out[i] = load_elem(codes, i, fmt);
    return OR_OK;
}

/*
 * Decode over a quantised cache: the plain attention of oracle_decode with
 * K_t = value(code) * k_scale[kh], V_t = value(code) * v_scale[kh]; q is
 * bfloat16.
 */
int oracle_decode_quant(double* out, const uint16_t* q, const uint8_t* k_cache,
                        const uint8_t* v_cache, const float* k_scale, const float* v_scale,
                        const int32_t* block_tables, int32_t block_table_stride,
                        const int32_t* context_lens, int32_t num_seqs, int32_t num_heads,
                        int32_t num_kv_heads, int32_t num_blocks, int32_t block_size,
                        int32_t head_dim, int32_t fmt, float scale, int32_t num_threads) {
    if (num_seqs < 0 || num_heads <= 0 || (fmt != 2 && fmt != 3) ||
        !shape_ok(num_blocks, num_kv_heads, block_size, head_dim, fmt) ||
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
        const int32_t n_ctx = context_lens[s];
        int r = decode_one_q(out, q, 1, k_cache, v_cache, k_scale, v_scale,
                             block_tables + (size_t)s * block_table_stride, n_ctx, s, h,
                             num_heads, num_kv_heads, num_blocks, block_size, head_dim, fmt,
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
