/*
 * pa.h — C ABI of the paged KV-cache decode library (sm_100a, one GPU).
 *
 * Three operations make up the decode hot path of PagedAttention:
 *
 *   pa_kv_append   scatter each step's new K/V vectors into their cache slots
 *   pa_decode      single-query attention over K/V that a per-sequence block
 *                  table gathers from fixed-size physical blocks
 *   pa_block_copy  copy whole physical blocks (copy-on-write at a fork)
 *
 * plus pa_block_swap (blocks between a device pool and a pinned host pool),
 * pa_kv_append_quant / pa_decode_quant (FP8 E4M3 or int8 caches with per-head
 * scales),
 * pa_decode_multi (several query tokens per sequence: chunked prefill,
 * speculative verification), and pa_decode_grouped, pa_decode for groups of sequences that share blocks
 * (beams, parallel samples), which reads each shared block once per group.
 *
 * Sources for what each call computes (page title, section):
 *   [P1] "PagedAttention：大模型推理性能优化的核心技术解析" (bmjup.com),
 *        § "PagedAttention 的核心工作机制与创新" (1 页表式管理, 2 写入时拷贝).
 *   [P2] "AI 推理系列（十六）：PagedAttention——为什么 vLLM 能把 GPU 显存
 *        “像操作系统一样”管理？" (wiblog.cn), § "PagedAttention 如何把连续
 *        序列映射到离散显存块" (block table, flowchart), § "Copy-on-Write、
 *        并行采样与 Prefix Caching 不是同一件事", § "非连续 KV 为什么需要
 *        专门的 Attention Kernel".
 *   [P3] "PagedAttention原理详解：GPU显存优化与模型路由技术" (kongchang.com),
 *        § "显存消耗的三大来源" (single-query attention over cached K/V),
 *        § "PagedAttention的三大核心优势" (reference counts, copy-on-write).
 *   [P4] "vLLM的Paged Attention技术：高效注意力机制解析" (intelliparadigm.com),
 *        § 2.2 内存布局优化, § 3.1 核函数签名解析, § 3.2 执行层次结构.
 *
 * ---------------------------------------------------------------------------
 * Conventions shared by every call
 * ---------------------------------------------------------------------------
 * Memory.  Every tensor pointer is a DEVICE pointer owned by the caller. The
 *   library never allocates, frees or retains caller memory; it keeps only a
 *   per-device 4-byte status word (see pa_sync_check) and the fixed scratch
 *   buffer of pa_decode_noalloc.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *   default stream). Every call only enqueues work on that stream and returns;
 *   results are ready when the stream reaches that point.
 * Status.  Every int-returning call returns PA_OK (0) or a negative PA_ERR_*
 *   code. Argument errors are detected on the host before anything is
 *   enqueued; pa_get_last_error() then returns a message for the calling
 *   thread. Data-dependent errors (a block id or slot outside the pool, a
 *   context longer than its block-table row) are detected by the kernels,
 *   which skip the offending access, never fault, and record PA_ERR_BAD_INDEX
 *   in the device status word that pa_sync_check reads.
 * Element type.  PA_F32 (IEEE binary32) or PA_BF16 (bfloat16). q, out, k, v
 *   and both caches of one call share that type (quantised caches: see
 *   pa_decode_quant). Attention arithmetic is
 *   fp32 internally; outputs are rounded to nearest-even into the type.
 *
 * Cache layout (identical for k_cache and v_cache):
 *
 *   cache[num_blocks][num_kv_heads][block_size][head_dim], head_dim fastest.
 *
 *   Element (block b, kv head h, slot o, dim i) sits at linear index
 *   ((b * num_kv_heads + h) * block_size + o) * head_dim + i.
 *   Token position t of a sequence whose block table row is `tbl` lives in
 *   block tbl[t / block_size], slot t % block_size [P2 block-table example:
 *   logical blocks 0,1,2 -> physical 17,4,29]. Only the last block of a
 *   sequence is partly filled [P2 same section, closing paragraph].
 *   A slot index encodes (block, offset) as block * block_size + offset.
 *   This replaces the 5-D [blocks, kv_heads, head_dim/x, block_size, x] key
 *   layout of [P4 § 2.2]: here each (block, kv head) tile of one cache is one
 *   contiguous, 16-byte aligned span of block_size * head_dim elements.
 *
 * Supported shapes: head_dim in {64, 128}; block_size a power of two in
 *   [16, 256]; num_heads % num_kv_heads == 0 (query head h reads kv head
 *   h / (num_heads / num_kv_heads), contiguous groups). All pointers must be
 *   16-byte aligned.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define PA_OK               0
#define PA_ERR_INVALID_ARG (-1) /* null pointer, negative size, bad shape     */
#define PA_ERR_DTYPE       (-2) /* dtype unknown, or wrong for this call        */
#define PA_ERR_ALIGN       (-3) /* a pointer is not 16-byte aligned           */
#define PA_ERR_UNSUPPORTED (-4) /* head_dim / block_size not compiled         */
#define PA_ERR_CUDA        (-5) /* a CUDA runtime call or launch failed       */
#define PA_ERR_BAD_INDEX   (-6) /* a kernel met an out-of-range index         */
#define PA_ERR_WORKSPACE   (-7) /* workspace missing or smaller than needed   */
#define PA_ERR_TIMEOUT     (-8) /* a bounded in-kernel pipeline wait gave up  */

/* ---- element types ------------------------------------------------------ */
#define PA_F32  0
#define PA_BF16 1
#define PA_FP8_E4M3 2  /* quantised cache: one-byte OCP FP8 E4M3 codes (pa_*_quant calls) */
#define PA_INT8 3      /* quantised cache: one-byte signed int8 codes (pa_*_quant calls)  */

/* Shape of one physical KV pool (both k_cache and v_cache). */
typedef struct pa_cache_desc {
    int32_t num_blocks;   /* physical blocks in the pool                    */
    int32_t num_kv_heads; /* KV heads stored per block                      */
    int32_t block_size;   /* token slots per block                          */
    int32_t head_dim;     /* elements per K or V vector                     */
    int32_t dtype;        /* PA_F32, PA_BF16, PA_FP8_E4M3 or PA_INT8        */
} pa_cache_desc;

/*
 * pa_kv_append — write this step's new K/V vectors into their slots.
 *
 * Computes the flowchart node "追加 KV" of [P2 § PagedAttention 如何把连续序列
 * 映射到离散显存块]: for every token i in [0, num_tokens) with
 * slot_mapping[i] >= 0, and every kv head h,
 *     k_cache[slot / block_size][h][slot % block_size][:] = k[i][h][:]
 *     v_cache[slot / block_size][h][slot % block_size][:] = v[i][h][:]
 * as a bit-exact copy. slot_mapping[i] < 0 marks a padding token: skipped.
 * Allocating a new block when the current one is full is the caller's job.
 *
 *   k, v          device, [num_tokens][num_kv_heads][head_dim], contiguous.
 *   slot_mapping  device, int64 [num_tokens].
 *   k_cache, v_cache  device pools in the layout above.
 *   cache         host pointer to the pool's shape.
 * Non-negative slots within one call must be distinct (otherwise which token
 * lands in a slot is unspecified). A slot >= num_blocks * block_size is
 * skipped and recorded as PA_ERR_BAD_INDEX. num_tokens == 0 is a no-op.
 */
int pa_kv_append(const void* k, const void* v, const int64_t* slot_mapping,
                 int32_t num_tokens, void* k_cache, void* v_cache,
                 const pa_cache_desc* cache, void* stream);

/*
 * pa_decode — single-query paged attention for one decode step.
 *
 * For every sequence s, query head h (kh = h / (num_heads / num_kv_heads)):
 *     n      = context_lens[s]
 *     K_t    = k_cache[block_tables[s][t / block_size]][kh][t % block_size]
 *     V_t    = v_cache[ ... same ... ],                  t = 0 .. n-1
 *     out[s][h] = softmax_t(scale * q[s][h] . K_t) . V
 * i.e. the unchanged attention of [P2 § 非连续 KV 为什么需要专门的 Attention
 * Kernel] and [P3 § 显存消耗的三大来源] (one query against all cached K/V),
 * read through the block table. n == 0 gives out[s][h] = 0.
 * Long contexts are split into partitions of `partition_size` tokens, each
 * producing (running max, running sum, normalised partial output) in the
 * workspace, then merged by a log-sum-exp reduction (grid dimension
 * "分区" of [P4 § 3.2]; the merge itself is not on the pages).
 *
 *   out           device, [num_seqs][num_heads][head_dim], type of the cache.
 *   q             device, [num_seqs][num_heads][head_dim], type of the cache.
 *   block_tables  device, int32 [num_seqs][block_table_stride]; entries past
 *                 ceil(n / block_size) are never read.
 *   context_lens  device, int32 [num_seqs], each in [0, max_context_len].
 *   max_context_len  host bound on context_lens; must not exceed
 *                 block_table_stride * block_size. A larger context is
 *                 clipped to the bound and recorded as PA_ERR_BAD_INDEX.
 *   scale         softmax scale (commonly 1/sqrt(head_dim)).
 *   cache         host pointer; cache->num_kv_heads is the kv-head count.
 *   partition_size  0 = library policy; -1 = never split; otherwise the
 *                 tokens per partition, a positive multiple of 16.
 *   workspace     device scratch of pa_decode_workspace_size(...) bytes (same
 *                 arguments), 256-byte aligned; may be NULL when that size is 0.
 *                 For grouped-query heads (2..8 query heads per kv head) the
 *                 size includes 256 bytes after the partial results for the
 *                 tensor-core kernel's work-item counter, which the call zeroes
 *                 (cudaMemsetAsync on `stream`) before the kernel: with at least
 *                 two work items per CTA slot, the CTAs claim items from it so
 *                 that those streaming faster take more. A workspace that holds
 *                 only the partial results (or none when the call does not
 *                 split) is accepted and runs the static schedule instead
 *                 (item u to CTA u mod grid); the results are the same bit for
 *                 bit. A workspace must not be used by two calls at once.
 * The result does not depend on the physical placement of blocks: the
 * arithmetic order depends only on logical token positions.
 */
int pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, int32_t block_table_stride,
              const int32_t* context_lens, int32_t max_context_len,
              int32_t num_seqs, int32_t num_heads, float scale,
              const pa_cache_desc* cache, int32_t partition_size,
              void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_decode_workspace_size — bytes of device scratch pa_decode takes for the
 * same (num_seqs, num_heads, max_context_len, cache, partition_size): the
 * partial results of a split context, plus 256 bytes for the tensor-core
 * kernel's work-item counter when the heads are grouped-query (so 256 for an
 * unsplit grouped-query call, 0 for an unsplit call on the CUDA-core kernel).
 * Returns 0 and sets the last error on bad arguments. Queries the current
 * device's SM count (cached per device).
 */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads,
                                int32_t max_context_len,
                                const pa_cache_desc* cache,
                                int32_t partition_size);

/*
 * pa_decode_num_partitions — number of context partitions pa_decode will use
 * for these arguments (1 = no split); negative PA_ERR_* on bad arguments.
 */
int pa_decode_num_partitions(int32_t num_seqs, int32_t num_heads,
                             int32_t max_context_len,
                             const pa_cache_desc* cache,
                             int32_t partition_size);

/*
 * pa_decode_grouped — pa_decode for batches whose sequences come in groups
 * that share blocks: the beams of a beam search or the parallel samples of
 * one prompt, which after a fork hold the prompt's blocks through reference
 * counts ([P2 § Copy-on-Write、并行采样与 Prefix Caching 不是同一件事]: several
 * logical sequences point at one physical block; [P3 § PagedAttention的三大
 * 核心优势], point 2 and the beam-search paragraph).
 *
 * Computes exactly what pa_decode computes, for every sequence and head, with
 * the same arguments and conventions. Sequences k*group_size ..
 * (k+1)*group_size - 1 form group k (the last group may be shorter); the
 * sequences of a group are decoded together, so a block that several of them
 * reference, at the same logical position, is read from memory once for all
 * of them. Grouping never changes a result: any sequences may be grouped,
 * sharing or not, and each sequence's output is bit-identical to the one it
 * gets when its blocks are private copies (for the same group_size and
 * partitioning). The result can differ from pa_decode's in the last bits
 * (another summation order), within the same tolerance of the exact value.
 *
 *   group_size    1 .. 8. The grouped kernel runs for bf16, head_dim 64/128
 *                 and group_size * (num_heads / num_kv_heads) <= 64; other
 *                 calls, and group_size 1, run pa_decode's kernels.
 *   workspace     at least pa_decode_grouped_workspace_size(...) bytes with
 *                 the same arguments.
 * Returns PA_ERR_INVALID_ARG for group_size outside [1, 8] or a
 * max_context_len above 2^27 on the grouped kernel.
 */
int pa_decode_grouped(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int32_t block_table_stride,
                      const int32_t* context_lens, int32_t max_context_len,
                      int32_t num_seqs, int32_t num_heads, float scale,
                      const pa_cache_desc* cache, int32_t group_size,
                      int32_t partition_size, void* workspace, size_t workspace_bytes,
                      void* stream);

/* Workspace bytes and partition count of pa_decode_grouped (see
 * pa_decode_workspace_size / pa_decode_num_partitions). */
size_t pa_decode_grouped_workspace_size(int32_t num_seqs, int32_t num_heads,
                                        int32_t max_context_len,
                                        const pa_cache_desc* cache, int32_t group_size,
                                        int32_t partition_size);
int pa_decode_grouped_num_partitions(int32_t num_seqs, int32_t num_heads,
                                     int32_t max_context_len,
                                     const pa_cache_desc* cache, int32_t group_size,
                                     int32_t partition_size);

/*
 * pa_decode_multi — attention of several new query tokens per sequence over
 * the paged cache: a chunk of a prompt processed against the cache (chunked
 * prefill, which [P2 § 如何判断服务瓶颈是否真的来自 PagedAttention] names
 * among the things to check when prefill dominates), or the draft tokens of a
 * speculative step being verified. Same block tables, same cache.
 *
 * Sequence s has n_s = query_start[s+1] - query_start[s] new tokens, whose K/V
 * have already been appended: they are the last n_s of its context_lens[s]
 * positions. Query token j (0 <= j < n_s, row query_start[s] + j of q and out)
 * sits at position p = context_lens[s] - n_s + j and attends causally to
 * positions 0 .. p:
 *     out[row][h] = softmax_{t <= p}(scale q[row][h] . K_t) . V
 * with K_t, V_t read through block_tables[s] exactly as in pa_decode.
 *
 *   q, out        device, [num_query_tokens][num_heads][head_dim], the cache's
 *                 dtype (bf16 or fp32).
 *   query_start   device int32 [num_seqs + 1], non-decreasing, query_start[0]
 *                 = 0, query_start[num_seqs] = num_query_tokens (<= 65535).
 *   max_query_len host bound on n_s (>= 1). Over bf16 caches the tokens of one
 *                 sequence are decoded together in groups of up to 8 (at most
 *                 64 query columns per group), so each block is read once per
 *                 group; over fp32 caches (and for query groups above 64
 *                 columns) each token is a row of its own on the CUDA-core
 *                 consumer, which keeps the fp32 accuracy of pa_decode.
 *   workspace     at least pa_decode_multi_workspace_size(...) bytes.
 * Needs a bf16 or fp32 cache with head_dim 64 or 128 (PA_ERR_UNSUPPORTED
 * otherwise).
 * n_s > context_lens[s] is recorded as PA_ERR_BAD_INDEX (those rows get 0).
 * A query token's result does not depend on the other tokens in the call (it
 * is bit-identical to a call holding only that token with the context cut at
 * its position, for the same partition size).
 */
int pa_decode_multi(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t block_table_stride,
                    const int32_t* context_lens, const int32_t* query_start,
                    int32_t max_context_len, int32_t num_seqs, int32_t num_query_tokens,
                    int32_t max_query_len, int32_t num_heads, float scale,
                    const pa_cache_desc* cache, int32_t partition_size, void* workspace,
                    size_t workspace_bytes, void* stream);

/* Workspace bytes and partition count of pa_decode_multi. */
size_t pa_decode_multi_workspace_size(int32_t num_seqs, int32_t num_query_tokens,
                                      int32_t max_query_len, int32_t num_heads,
                                      int32_t max_context_len, const pa_cache_desc* cache,
                                      int32_t partition_size);
int pa_decode_multi_num_partitions(int32_t num_seqs, int32_t num_query_tokens,
                                   int32_t max_query_len, int32_t num_heads,
                                   int32_t max_context_len, const pa_cache_desc* cache,
                                   int32_t partition_size);

/*
 * Quantised KV cache ([P2] mechanisms table: KV cache quantisation lowers
 * the bits stored per cached element, at the price of quantisation error and
 * conversion work; [P3] § 量化技术: INT8 KV cache quantisation halves KV
 * memory without touching the weights and composes with paging). The pages
 * fix no format; this library stores one byte per element, a PA_FP8_E4M3 or
 * PA_INT8 code, with one binary32 scale per kv head for K and one for V:
 *     stored code  c = Q(x / scale[kv head])      (division in binary32)
 *     cached value   = value(c) * scale[kv head]
 * Q for PA_FP8_E4M3: round to nearest even, magnitudes >= 448 (infinities
 * too) saturate to +-448, NaN gives the NaN code 0x7F. Q for PA_INT8: clamp
 * to [-127, 127] (a NaN becomes -127), then round to nearest even. Scales are
 * the caller's (calibrated, or from the data); they must be positive and
 * finite for the codes to mean anything. The cache layout is unchanged with
 * one-byte elements; pa_block_copy and pa_block_swap move quantised pools as
 * they are. q and out stay bf16.
 *
 * pa_kv_append_quant — pa_kv_append for a quantised cache: k, v are bf16
 * [num_tokens][num_kv_heads][head_dim] (device); each element is stored as
 * its code. k_scale, v_scale: device float [num_kv_heads]. head_dim 64 or 128.
 *
 * pa_decode_quant — pa_decode over a quantised cache: the same attention with
 * K_t and V_t the cached values above (the K scale folds into the scores, the
 * V scale into the output). Arguments as pa_decode plus the two scale arrays;
 * head_dim 64 or 128; workspace sized by pa_decode_workspace_size with the
 * quantised descriptor. Precision: the products run with q rounded to f16
 * after a power-of-two shift that puts the largest |q| of the q values a warp
 * holds in [2^14, 2^15) (the scores are shifted back after the products; both
 * exact, so any bf16 q within 2^29 of that largest one is rounded exactly,
 * whatever its magnitude) and the softmax weights rounded to f16, accumulated
 * in fp32; results meet the bf16 bars of pa_decode. pa_decode,
 * pa_kv_append and the other decode calls refuse a quantised descriptor
 * (PA_ERR_DTYPE), and these two refuse an unquantised one.
 */
int pa_kv_append_quant(const void* k, const void* v, const int64_t* slot_mapping,
                       int32_t num_tokens, void* k_cache, void* v_cache,
                       const float* k_scale, const float* v_scale,
                       const pa_cache_desc* cache, void* stream);

int pa_decode_quant(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const float* k_scale, const float* v_scale,
                    const int32_t* block_tables, int32_t block_table_stride,
                    const int32_t* context_lens, int32_t max_context_len,
                    int32_t num_seqs, int32_t num_heads, float scale,
                    const pa_cache_desc* cache, int32_t partition_size,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_decode_grouped_quant / pa_decode_multi_quant — pa_decode_grouped and
 * pa_decode_multi over a quantised cache (the two compositions of the calls
 * above): arguments as those calls plus k_scale, v_scale after v_cache; the
 * precision of pa_decode_quant; head_dim 64 or 128. Workspace and partitions as
 * pa_decode_grouped_workspace_size / pa_decode_multi_workspace_size (and the
 * _num_partitions queries) with the quantised descriptor. Grouped and
 * multi-token decode are the same computation as pa_decode_quant: a group's
 * members, and each query token, get exactly the result pa_decode_quant
 * gives them alone up to rounding (grouping never changes a result beyond
 * that; within one call it changes no bit).
 */
int pa_decode_grouped_quant(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const float* k_scale, const float* v_scale,
                            const int32_t* block_tables, int32_t block_table_stride,
                            const int32_t* context_lens, int32_t max_context_len,
                            int32_t num_seqs, int32_t num_heads, float scale,
                            const pa_cache_desc* cache, int32_t group_size,
                            int32_t partition_size, void* workspace, size_t workspace_bytes,
                            void* stream);
int pa_decode_multi_quant(void* out, const void* q, const void* k_cache, const void* v_cache,
                          const float* k_scale, const float* v_scale, const int32_t* block_tables,
                          int32_t block_table_stride, const int32_t* context_lens,
                          const int32_t* query_start, int32_t max_context_len, int32_t num_seqs,
                          int32_t num_query_tokens, int32_t max_query_len, int32_t num_heads,
                          float scale, const pa_cache_desc* cache, int32_t partition_size,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_set_grouped_consumer — which consumer pa_decode_grouped and pa_decode_multi
 * use for bf16 head_dim 128 with 8..32 query columns (sequences or query
 * tokens x query heads per kv head):
 *   PA_GROUPED_MMA_SYNC: one warp per 8 query columns, m16n8k16 MMAs from
 *     registers;
 *   PA_GROUPED_TCGEN05: one thread issues tcgen05.mma (S = Q K^T and O += P V,
 *     S and O in tensor memory, P in shared memory) for four softmax warps
 *     that split each 64-token unit.
 * Both compute the same attention within the same tolerance of the exact
 * value, and both keep a sequence's result independent of which blocks it
 * shares; they round differently from each other. Other shapes always take
 * the mma.sync consumer. The setting belongs to the calling host thread (each
 * thread starts with the default). Returns the previous consumer, or
 * PA_ERR_INVALID_ARG for an unknown value.
 */
#define PA_GROUPED_MMA_SYNC 0
#define PA_GROUPED_TCGEN05 1
int pa_set_grouped_consumer(int consumer);

/*
 * pa_block_copy — copy whole physical blocks, the copy-on-write step that
 * [P1 § 2 写入时拷贝], [P2 § Copy-on-Write、并行采样与 Prefix Caching] and
 * [P3 § PagedAttention的三大核心优势] describe: when a sequence is about to
 * write into a block that other sequences still share, the block is first
 * copied to a private one.
 *
 * For every pair p: block dst = src_dst_pairs[2p+1] receives all slots of all
 * kv heads of block src = src_dst_pairs[2p], in both k_cache and v_cache, as
 * a bit-exact copy.
 *   src_dst_pairs  device, int64 [num_pairs][2] = (src, dst).
 * Within one call the dst ids must be distinct and no dst may also appear as
 * a src (the result is then independent of copy order). Ids outside
 * [0, num_blocks) are skipped and recorded as PA_ERR_BAD_INDEX. Deciding WHICH
 * blocks to copy (reference counts) is the caller's host-side job.
 */
int pa_block_copy(const int64_t* src_dst_pairs, int32_t num_pairs,
                  void* k_cache, void* v_cache, const pa_cache_desc* cache,
                  void* stream);

/*
 * pa_block_swap — copy whole blocks from one pool into another pool of the
 * same block shape, where either pool may live in pinned host memory: the
 * swap-out of a preempted request's blocks to host memory and their swap-in
 * when it resumes ([P2 § 生产环境 monitoring list]: the frequency and latency
 * of CPU offload or swap are among the signals a deployment watches; the
 * pages give no more).
 *
 * For every pair p: block dst = src_dst_pairs[2p+1] of the destination pool
 * receives all slots of all kv heads of block src = src_dst_pairs[2p] of the
 * source pool, in both caches, bit for bit.
 *   src_dst_pairs  device (or mapped pinned host) int64 [num_pairs][2].
 *   src_k, src_v   the source pool, `src` its shape; dst_k, dst_v and `dst`
 *                  the destination. num_kv_heads, block_size, head_dim and
 *                  dtype must agree; num_blocks may differ. Each pointer is
 *                  device memory or pinned host memory (cudaHostAlloc, or
 *                  cudaHostRegister'ed) that the device can address; pageable
 *                  host memory returns PA_ERR_INVALID_ARG.
 * The two pools must not overlap (within one pool use pa_block_copy), and dst
 * ids must be distinct within a call. Ids outside their pool are skipped and
 * recorded as PA_ERR_BAD_INDEX. The copy runs on the SMs (one launch for any
 * number of scattered blocks), reading and writing host memory over the host
 * link; the host pool must not be touched by the CPU until the stream passes
 * the call.
 */
int pa_block_swap(const int64_t* src_dst_pairs, int32_t num_pairs,
                  const void* src_k, const void* src_v, const pa_cache_desc* src,
                  void* dst_k, void* dst_v, const pa_cache_desc* dst, void* stream);

/*
 * PA_NOALLOC_SCRATCH_BYTES — size of the device buffer inside the library that
 * pa_decode_noalloc uses as its workspace (32 MiB per GPU that loads the
 * library, held until the process exits).
 */
#define PA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * pa_decode_noalloc — pa_decode for callers that cannot allocate device memory.
 *
 * The pages have no counterpart: this is an interface convenience. Some callers
 * cannot call cudaMalloc where they decode (code inside a memory arena sized up
 * front, plug-ins of an engine that owns all device allocations, loops that
 * must never enter an allocator). This entry point computes exactly what
 * pa_decode computes, with the same arguments minus the workspace: the
 * workspace pa_decode_workspace_size asks for (the partial results of a split
 * context, the work-item counter of grouped-query heads) is a buffer of
 * PA_NOALLOC_SCRATCH_BYTES inside the library. It allocates nothing.
 *
 * The first call on a device looks up that buffer's device address
 * (cudaGetSymbolAddress) with the device current and keeps it with the CUDA
 * context it belongs to; a later call that finds another context current (a
 * cudaDeviceReset makes the runtime create a new one, and the buffer may then
 * move) looks it up again. Make the first call on a device, and the first
 * after a reset, before any stream capture. A call whose workspace need (pa_decode_workspace_size
 * with the same arguments) exceeds PA_NOALLOC_SCRATCH_BYTES returns
 * PA_ERR_WORKSPACE and enqueues nothing. All calls on one device share the
 * buffer, which keeps the last call's contents: calls whose kernels may overlap
 * on the GPU (different streams without ordering) race on it and must not be
 * issued. The buffer needs no clearing between calls.
 */
int pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int32_t block_table_stride,
                      const int32_t* context_lens, int32_t max_context_len,
                      int32_t num_seqs, int32_t num_heads, float scale,
                      const pa_cache_desc* cache, int32_t partition_size, void* stream);

/*
 * pa_sync_check — wait for `stream`, then read and clear the current device's
 * status word. Returns PA_OK, PA_ERR_BAD_INDEX if any kernel since the last
 * check met an out-of-range index, PA_ERR_TIMEOUT if a kernel's bounded wait
 * on its shared-memory pipeline gave up (its results are then invalid; the
 * kernel still terminated), or PA_ERR_CUDA if the stream reported an error.
 */
int pa_sync_check(void* stream);

/* Message describing the last failed call on this host thread ("" if none). */
const char* pa_get_last_error(void);

/* Constant name of a status code, e.g. "PA_ERR_ALIGN". */
const char* pa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
