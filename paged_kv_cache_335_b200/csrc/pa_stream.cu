// pa_stream.cu — a read-only streaming kernel that measures the HBM read
// bandwidth this GPU can actually sustain: the reference a read-dominated
// kernel such as decode attention is compared with, next to the copy
// bandwidth (read + write) the roofline uses.
//
// It reads the way the decode kernels do: one lane of a producer warp issues
// bulk asynchronous copies (cp.async.bulk, global -> shared, no multicast) of
// 16 KiB chunks into a ring of shared-memory stages guarded by mbarriers, and
// a consumer warp waits for each chunk, folds one 16-byte word per lane into a
// checksum and releases the stage. CTA c reads chunks c, c + G, c + 2G, ...
// (G = CTAs), so at any moment the grid reads one contiguous window of HBM.
// Every wait is bounded; the producer drains its copies before the CTA exits.
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_stream.h"
#include "pa_tma.cuh"

namespace pa {
namespace {

constexpr int kChunk = 16384;   // bytes per bulk copy (a multiple of 16)
constexpr int kStages = 6;      // 96 KiB ring: two CTAs per SM
constexpr int kThreads = 64;    // producer warp + consumer warp
constexpr size_t kSmem = (size_t)kStages * kChunk + 2 * kStages * 8;

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

__global__ void __launch_bounds__(kThreads)
stream_read_kernel(const uint8_t* __restrict__ src, int64_t bytes, uint32_t* __restrict__ partial) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t ring = smem_u32(smem);
    const uint32_t full = ring + kStages * kChunk, empty = full + 8 * kStages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + 8 * s, 1);
            mbar_init(empty + 8 * s, 1);
        }
        fence_barrier_init();
    }
    __syncthreads();
    const int64_t nchunks = (bytes + kChunk - 1) / kChunk;
    const int64_t mine = nchunks > blockIdx.x ? (nchunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    if (warp == 0) {  // producer
        int64_t issued = 0;
        if (lane == 0) {
            for (int64_t k = 0; k < mine; ++k) {
                const int st = (int)(k % kStages);
                if (!mbar_wait_bounded(empty + 8 * st, ((uint32_t)(k / kStages) & 1u) ^ 1u)) break;
                const int64_t off = (blockIdx.x + k * gridDim.x) * (int64_t)kChunk;
                const uint32_t n = (uint32_t)min((int64_t)kChunk, bytes - off);
                mbar_arrive_expect_tx(full + 8 * st, n);
                bulk_load(ring + st * kChunk, src + off, n, full + 8 * st);
                issued = k + 1;
            }
            // drain: the last copy into every stage has landed
            for (int64_t k = issued > kStages ? issued - kStages : 0; k < issued; ++k)
                mbar_wait_bounded(full + 8 * (int)(k % kStages), (uint32_t)(k / kStages) & 1u);
        }
        return;
    }
    uint32_t acc = 0;
    for (int64_t k = 0; k < mine; ++k) {  // consumer
        const int st = (int)(k % kStages);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(full + 8 * st, (uint32_t)(k / kStages) & 1u)))
            break;
        const int64_t off = (blockIdx.x + k * gridDim.x) * (int64_t)kChunk;
        const int n16 = (int)(min((int64_t)kChunk, bytes - off) / 16);
        if (lane < n16) {
            const uint4 v = lds128(ring + st * kChunk + 16 * lane);
            acc += v.x ^ v.y ^ v.z ^ v.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + 8 * st);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) partial[blockIdx.x] = acc;
}

}  // namespace
}  // namespace pa

extern "C" int pa_stream_read(const void* src, size_t bytes, uint32_t* partial, int32_t num_ctas,
                              void* stream) {
    if (!src || !partial || num_ctas <= 0 || (bytes & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(src) & 15u) != 0)
        return -1;
    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(pa::stream_read_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)pa::kSmem) != cudaSuccess)
            return -5;
        attr_set = true;
    }
    pa::stream_read_kernel<<<num_ctas, pa::kThreads, pa::kSmem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(src), (int64_t)bytes, partial);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}
