// pa_copy.cu — the two data-movement kernels of the hot path.
//
// kv_append_kernel: the flowchart step "追加 KV" of "AI 推理系列（十六）：
//   PagedAttention——…", § PagedAttention 如何把连续序列映射到离散显存块: each new
//   token's K and V vectors go to slot (block, offset) of the paged pool.
// block_copy_kernel: the copy-on-write step of "PagedAttention：大模型推理性能优化的
//   核心技术解析", § 核心工作机制与创新 / 2 写入时拷贝 — a shared block is duplicated
//   into a private one before a sharer writes to it.
//
// Both are pure 16-byte moves (bit-exact). One (block, kv head) tile of the pool
// is block_size * head_dim contiguous elements, and a whole block (all kv heads)
// is contiguous too, so the copy streams num_kv_heads * block_size * head_dim
// elements per cache per pair.
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

static __device__ unsigned int s_status_copy;

namespace {

constexpr int kThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kThreads)
kv_append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                 const int64_t* __restrict__ slot_mapping, int64_t total_vecs,
                 uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, CopyParams cp,
                 int64_t num_slots) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total_vecs;
         idx += stride) {
        const int64_t row = idx / cp.row_vecs;          // token * num_kv_heads + head
        const int32_t c = (int32_t)(idx - row * cp.row_vecs);
        const int64_t token = row / cp.num_kv_heads;
        const int32_t h = (int32_t)(row - token * cp.num_kv_heads);
        const int64_t slot = __ldg(slot_mapping + token);
        if (slot < 0) continue;                         // padding token
        if (slot >= num_slots) {
            atomicOr(&s_status_copy, kStatusBadIndex);
            continue;
        }
        const int64_t blk = slot >> cp.log2_block_size;
        const int64_t off = slot & (cp.block_size - 1);
        const int64_t dst = ((blk * cp.num_kv_heads + h) * cp.block_size + off) * cp.row_vecs + c;
        const uint4 kv = ld_stream(k + idx);
        const uint4 vv = ld_stream(v + idx);
        k_cache[dst] = kv;
        v_cache[dst] = vv;
    }
}

// grid = (chunks of one block, pairs, 2 = {K, V}); each CTA moves up to
// kThreads * kCopyUnroll 16-byte vectors of one block of one cache.
__global__ void __launch_bounds__(kThreads)
block_copy_kernel(const int64_t* __restrict__ pairs, uint4* __restrict__ k_cache,
                  uint4* __restrict__ v_cache, int64_t vecs_per_block, int32_t num_blocks) {
    const int64_t src = __ldg(pairs + 2 * (int64_t)blockIdx.y);
    const int64_t dst = __ldg(pairs + 2 * (int64_t)blockIdx.y + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0) atomicOr(&s_status_copy, kStatusBadIndex);
        return;
    }
    uint4* cache = blockIdx.z ? v_cache : k_cache;
    const uint4* s = cache + src * vecs_per_block;
    uint4* d = cache + dst * vecs_per_block;
    const int64_t start = (int64_t)blockIdx.x * (kThreads * kCopyUnroll) + threadIdx.x;
    uint4 tmp[kCopyUnroll];
#pragma unroll
    for (int i = 0; i < kCopyUnroll; ++i) {
        const int64_t idx = start + i * kThreads;
        if (idx < vecs_per_block) tmp[i] = ld_stream(s + idx);
    }
#pragma unroll
    for (int i = 0; i < kCopyUnroll; ++i) {
        const int64_t idx = start + i * kThreads;
        if (idx < vecs_per_block) d[idx] = tmp[i];
    }
}

// Quantising append (KV cache quantisation, "AI 推理系列（十六）：PagedAttention——…",
// mechanisms table; "PagedAttention原理详解…", § 量化技术): each thread turns
// 16 bf16 elements of one (token, kv head) row into 16 one-byte codes of
// y = x / scale[head] (binary32 division): FP8 E4M3 rounded to nearest even
// and saturated to +-448, or int8 clamped to +-127 then rounded to nearest
// even. The slot is checked as in kv_append_kernel.
__device__ __forceinline__ uint32_t e4m3x2_code(float lo, float hi) {
    uint32_t d;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

__device__ __forceinline__ uint32_t int8_code(float y) {
    return (uint32_t)(__float2int_rn(fminf(fmaxf(y, -127.f), 127.f)) & 0xff);
}

template <int FMT>
__global__ void __launch_bounds__(kThreads)
kv_append_quant_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                       const int64_t* __restrict__ slot_mapping, int64_t total_chunks,
                       uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                       const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                       CopyParams cp, int64_t num_slots) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total_chunks;
         idx += stride) {
        const int64_t row = idx / cp.row_vecs;          // token * num_kv_heads + head
        const int32_t c = (int32_t)(idx - row * cp.row_vecs);
        const int64_t token = row / cp.num_kv_heads;
        const int32_t h = (int32_t)(row - token * cp.num_kv_heads);
        const int64_t slot = __ldg(slot_mapping + token);
        if (slot < 0) continue;                         // padding token
        if (slot >= num_slots) {
            atomicOr(&s_status_copy, kStatusBadIndex);
            continue;
        }
        const int64_t blk = slot >> cp.log2_block_size;
        const int64_t off = slot & (cp.block_size - 1);
        const int64_t dst = ((blk * cp.num_kv_heads + h) * cp.block_size + off) * cp.row_vecs + c;
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
            const uint4* src = (kv ? v : k) + 2 * idx;  // 16 bf16 = two 16-byte chunks
            const float sc = __ldg((kv ? v_scale : k_scale) + h);
            const uint4 a = ld_stream(src), b = ld_stream(src + 1);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t out[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float y[4] = {__fdiv_rn(bf16_lo(w[2 * i]), sc), __fdiv_rn(bf16_hi(w[2 * i]), sc),
                              __fdiv_rn(bf16_lo(w[2 * i + 1]), sc),
                              __fdiv_rn(bf16_hi(w[2 * i + 1]), sc)};
                if (FMT == 2)
                    out[i] = e4m3x2_code(y[0], y[1]) | (e4m3x2_code(y[2], y[3]) << 16);
                else
                    out[i] = int8_code(y[0]) | (int8_code(y[1]) << 8) | (int8_code(y[2]) << 16) |
                             (int8_code(y[3]) << 24);
            }
            (kv ? v_cache : k_cache)[dst] = make_uint4(out[0], out[1], out[2], out[3]);
        }
    }
}

// Swap between two pools of the same block shape, either of which may be
// pinned host memory mapped into the device address space (swap-out to host
// when a request is preempted, swap-in when it resumes; "AI 推理系列（十六）：
// PagedAttention——…", § 生产环境 signals: CPU offload / swap frequency and
// latency). grid = (chunks of one block, pairs, 2 = {K, V}); the SMs move the
// data over the host link with plain 16-byte loads and stores, many in flight
// per thread, so one launch carries any number of scattered blocks.
constexpr int kSwapUnroll = 8;

__global__ void __launch_bounds__(kThreads)
block_swap_kernel(const int64_t* __restrict__ pairs, const uint4* __restrict__ src_k,
                  const uint4* __restrict__ src_v, uint4* __restrict__ dst_k,
                  uint4* __restrict__ dst_v, int64_t vecs_per_block, int32_t src_blocks,
                  int32_t dst_blocks) {
    const int64_t src = __ldg(pairs + 2 * (int64_t)blockIdx.y);
    const int64_t dst = __ldg(pairs + 2 * (int64_t)blockIdx.y + 1);
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (threadIdx.x == 0) atomicOr(&s_status_copy, kStatusBadIndex);
        return;
    }
    const uint4* s = (blockIdx.z ? src_v : src_k) + src * vecs_per_block;
    uint4* d = (blockIdx.z ? dst_v : dst_k) + dst * vecs_per_block;
    const int64_t start = (int64_t)blockIdx.x * (kThreads * kSwapUnroll) + threadIdx.x;
    uint4 tmp[kSwapUnroll];
#pragma unroll
    for (int i = 0; i < kSwapUnroll; ++i) {
        const int64_t idx = start + i * kThreads;
        if (idx < vecs_per_block) tmp[i] = ld_v4(s + idx);
    }
#pragma unroll
    for (int i = 0; i < kSwapUnroll; ++i) {
        const int64_t idx = start + i * kThreads;
        if (idx < vecs_per_block) d[idx] = tmp[i];
    }
}

}  // namespace

cudaError_t launch_block_swap(const int64_t* pairs, int32_t num_pairs, const void* src_k,
                              const void* src_v, int32_t src_blocks, void* dst_k, void* dst_v,
                              int32_t dst_blocks, const CopyParams& cp, cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const int64_t vecs = (int64_t)cp.num_kv_heads * cp.block_size * cp.row_vecs;
    const int64_t chunks = (vecs + kThreads * kSwapUnroll - 1) / (kThreads * kSwapUnroll);
    constexpr int32_t kMaxGridY = 65535;
    for (int32_t first = 0; first < num_pairs; first += kMaxGridY) {
        const int32_t n = num_pairs - first < kMaxGridY ? num_pairs - first : kMaxGridY;
        dim3 grid((unsigned)chunks, (unsigned)n, 2);
        block_swap_kernel<<<grid, kThreads, 0, stream>>>(
            pairs + 2 * (int64_t)first, static_cast<const uint4*>(src_k),
            static_cast<const uint4*>(src_v), static_cast<uint4*>(dst_k),
            static_cast<uint4*>(dst_v), vecs, src_blocks, dst_blocks);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_kv_append(const void* k, const void* v, const int64_t* slot_mapping,
                             int32_t num_tokens, void* k_cache, void* v_cache,
                             const CopyParams& cp, cudaStream_t stream) {
    const int64_t total = (int64_t)num_tokens * cp.num_kv_heads * cp.row_vecs;
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + kThreads - 1) / kThreads;
    if (blocks > 148 * 32) blocks = 148 * 32;          // grid-stride beyond this
    const int64_t num_slots = (int64_t)cp.num_blocks * cp.block_size;
    kv_append_kernel<<<(unsigned)blocks, kThreads, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, total,
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), cp, num_slots);
    return cudaGetLastError();
}

cudaError_t launch_kv_append_quant(const void* k, const void* v, const int64_t* slot_mapping,
                                   int32_t num_tokens, void* k_cache, void* v_cache,
                                   const float* k_scale, const float* v_scale, int fmt,
                                   const CopyParams& cp, cudaStream_t stream) {
    const int64_t total = (int64_t)num_tokens * cp.num_kv_heads * cp.row_vecs;
    if (total == 0) return cudaSuccess;
    int64_t blocks = (total + kThreads - 1) / kThreads;
    if (blocks > 148 * 32) blocks = 148 * 32;
    const int64_t num_slots = (int64_t)cp.num_blocks * cp.block_size;
    auto kern = fmt == 2 ? kv_append_quant_kernel<2> : kv_append_quant_kernel<3>;
    kern<<<(unsigned)blocks, kThreads, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, total,
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), k_scale, v_scale, cp,
        num_slots);
    return cudaGetLastError();
}

cudaError_t launch_block_copy(const int64_t* pairs, int32_t num_pairs, void* k_cache,
                              void* v_cache, const CopyParams& cp, cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const int64_t vecs = (int64_t)cp.num_kv_heads * cp.block_size * cp.row_vecs;
    const int64_t chunks = (vecs + kThreads * kCopyUnroll - 1) / (kThreads * kCopyUnroll);
    constexpr int32_t kMaxGridY = 65535;
    for (int32_t first = 0; first < num_pairs; first += kMaxGridY) {
        const int32_t n = num_pairs - first < kMaxGridY ? num_pairs - first : kMaxGridY;
        dim3 grid((unsigned)chunks, (unsigned)n, 2);
        block_copy_kernel<<<grid, kThreads, 0, stream>>>(pairs + 2 * (int64_t)first,
                                                         static_cast<uint4*>(k_cache),
                                                         static_cast<uint4*>(v_cache), vecs,
                                                         cp.num_blocks);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t read_status_copy(unsigned* bits, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(bits, s_status_copy, sizeof(unsigned));
    if (e != cudaSuccess || !clear) return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(s_status_copy, &zero, sizeof(unsigned));
}

}  // namespace pa
