// pa_internal.h — host-side interface between the C ABI (pa_api.cpp) and the
// kernel translation units. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pa {

// Bit of the per-translation-unit status word a kernel sets when it meets an
// out-of-range block id, slot or context length (and skips the access).
constexpr unsigned kStatusBadIndex = 1u;
// Bit set when a bounded wait on a shared-memory pipeline barrier gave up.
constexpr unsigned kStatusTimeout = 2u;
// Bit set when a kernel found its dynamic shared memory not 1024-byte aligned
// (it then returns without running; the outputs are not written).
constexpr unsigned kStatusSmemAlign = 4u;

// Everything one decode launch needs. Offsets are in elements unless noted.
struct DecodeParams {
    void* out;                  // [S][H][D], cache dtype
    const void* q;              // [S][H][D]
    const void* k_cache;        // [NB][Hkv][BS][D]
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_o;                // [S][H][P][D] normalised partial outputs (P > 1)
    float* ws_ml;               // [S][H][P][2]  (running max in log2 units, running sum)
    int64_t table_stride;
    int32_t max_context_len;
    int32_t num_seqs;
    int32_t num_heads;
    int32_t num_kv_heads;
    int32_t num_blocks;
    int32_t block_size;
    int32_t log2_block_size;
    int32_t partition_size;     // tokens per partition (whole context when P == 1)
    int32_t num_partitions;     // P
    float scale_log2;           // softmax scale * log2(e)
    int32_t test_skip_position; // -1; >= 0 only under pa_test_skip_load (timeout test)
    // Multi-token queries (pa_decode_multi), else query_start == nullptr: q / out
    // rows of sequence s are query_start[s] .. query_start[s+1]-1 of num_rows;
    // grouped items take q_chunks chunks of <= gs query tokens per sequence.
    const int32_t* query_start;
    int32_t q_chunks;
    int32_t num_rows;           // rows of q / out: num_seqs, or the query tokens
    // Quantised caches (codes): per-kv-head scales, K_t = value(code) * k_scale[kh];
    // nullptr for bf16 / f32 caches.
    const float* k_scale;
    const float* v_scale;
    // head_dim of q / out / the workspace rows. The consumers over codes are
    // built for 128-code rows and take head_dim 64 pools as rows whose upper
    // half the TMA fills with zero codes (q zero there too, outputs not stored).
    int32_t head_dim;
    // Dynamic item schedule of the persistent kernels: a counter zeroed before
    // the launch, from which CTAs claim work items in order (nullptr: static
    // schedule, item u to CTA u mod grid).
    unsigned int* sched;
};

struct CopyParams {
    int32_t num_blocks;
    int32_t num_kv_heads;
    int32_t block_size;
    int32_t log2_block_size;
    int32_t row_vecs;           // 16-byte chunks per K/V vector = head_dim * elem / 16
};

// Launchers: return cudaSuccess or the launch error. dtype: 0 = f32, 1 = bf16.
cudaError_t launch_kv_append(const void* k, const void* v, const int64_t* slot_mapping,
                             int32_t num_tokens, void* k_cache, void* v_cache,
                             const CopyParams& cp, cudaStream_t stream);
// Quantising append: bf16 k, v [T][Hkv][D] -> codes (fmt 2 = FP8 E4M3, 3 = int8)
// of x / scale[kv head].
cudaError_t launch_kv_append_quant(const void* k, const void* v, const int64_t* slot_mapping,
                                   int32_t num_tokens, void* k_cache, void* v_cache,
                                   const float* k_scale, const float* v_scale, int fmt,
                                   const CopyParams& cp, cudaStream_t stream);
cudaError_t launch_block_copy(const int64_t* pairs, int32_t num_pairs, void* k_cache,
                              void* v_cache, const CopyParams& cp, cudaStream_t stream);
// Blocks of one pool into another of the same block shape (either may be
// mapped pinned host memory); block ids checked against each pool's size.
cudaError_t launch_block_swap(const int64_t* pairs, int32_t num_pairs, const void* src_k,
                              const void* src_v, int32_t src_blocks, void* dst_k, void* dst_v,
                              int32_t dst_blocks, const CopyParams& cp, cudaStream_t stream);

// Which decode kernel a call uses: the tensor-core GQA consumer for bf16 with
// a query group of 2..8, the CUDA-core consumer otherwise.
bool mma_supported(int dtype, int head_dim, int group);
// CTA slots per SM the persistent tensor-core kernel is built for (its grid is
// at most this many CTAs per SM; the partition policy sizes items for it).
int mma_ctas_per_sm();

// Decode with K/V staged through shared memory by TMA (producer warp +
// consumer warps); `mma` selects the tensor-core GQA consumer. The tensor maps
// describe k_cache / v_cache as [num_blocks * num_kv_heads * block_size rows]
// x [head_dim], boxes of 16 rows x 128 bytes, 128-byte swizzle.
cudaError_t launch_decode_tma(const DecodeParams& p, int dtype, int head_dim, bool mma,
                              const CUtensorMap& kmap, const CUtensorMap& vmap,
                              cudaStream_t stream);
// Grouped decode: sequences [k gs, (k + 1) gs) form group k and run in one CTA,
// so blocks they share are read once; with p.query_start set, the members of an
// item are up to gs query tokens of one sequence instead. bf16, head_dim
// 64 / 128, 1 <= gs <= 8, gs * (H / Hkv) <= 64 query columns.
bool grouped_supported(int dtype, int head_dim, int group, int gs);
// Select the grouped consumer (PA_GROUPED_MMA_SYNC / PA_GROUPED_TCGEN05);
// returns the previous one.
int set_grouped_consumer(int consumer);
// Most query columns (tokens x heads per kv head) one multi-token item may hold.
int grouped_max_cols(int dtype, int head_dim, int group);
// Whether the grouped kernel for (dtype, head_dim, gs, H / Hkv) is the tcgen05 consumer.
bool grouped_is_tcgen05(int dtype, int head_dim, int gs, int group);
// CTA slots per SM of the grouped kernel chosen for (dtype, head_dim, gs, H / Hkv).
int grouped_ctas_per_sm(int dtype, int head_dim, int gs, int group);
cudaError_t launch_decode_grouped(const DecodeParams& p, int dtype, int head_dim, int gs,
                                  const CUtensorMap& kmap, const CUtensorMap& vmap,
                                  cudaStream_t stream);
// Log-sum-exp merge of the P partial results into out.
cudaError_t launch_partition_reduce(const DecodeParams& p, int dtype, int head_dim,
                                    cudaStream_t stream);

// Record `fmt` as this host thread's last error (read by pa_get_last_error)
// and return `code`.
int report_error(int code, const char* fmt, ...);

// Status words of the kernel translation units: OR of kStatus* bits since the
// last clear. Return cudaSuccess or the copy error.
cudaError_t read_status_copy(unsigned* bits, bool clear);
cudaError_t read_status_tma(unsigned* bits, bool clear);

}  // namespace pa
