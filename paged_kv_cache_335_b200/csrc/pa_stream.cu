// pa_stream.cu — a read-only streaming kernel that measures the HBM read
// bandwidth this GPU can actually sustain: the reference a read-dominated
// kernel such as decode attention is compared with, next to the copy
// bandwidth (read + write) the roofline uses.
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_stream.h"

namespace pa {
namespace {

constexpr int kThreads = 512;
constexpr int kUnroll = 8;

// Each thread sums its 16-byte words (as 32-bit integers, so nothing can be
// folded away) and the CTA writes one partial: the output is tiny, the reads
// are every byte of `src`.
__global__ void __launch_bounds__(kThreads)
stream_read_kernel(const uint4* __restrict__ src, int64_t n16, uint32_t* __restrict__ partial) {
    uint32_t acc = 0;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    for (; i + (kUnroll - 1) * stride < n16; i += kUnroll * stride) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) v[u] = ld_stream(src + i + u * stride);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) acc += v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
    }
    for (; i < n16; i += stride) {
        const uint4 v = ld_stream(src + i);
        acc += v.x ^ v.y ^ v.z ^ v.w;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    __shared__ uint32_t sm[kThreads / 32];
    if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = 0;
        for (int w = 0; w < kThreads / 32; ++w) t += sm[w];
        partial[blockIdx.x] = t;
    }
}

}  // namespace
}  // namespace pa

extern "C" int pa_stream_read(const void* src, size_t bytes, uint32_t* partial, int32_t num_ctas,
                              void* stream) {
    if (!src || !partial || num_ctas <= 0 || (bytes & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(src) & 15u) != 0)
        return -1;
    pa::stream_read_kernel<<<num_ctas, pa::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(src), (int64_t)(bytes / 16), partial);
    return cudaGetLastError() == cudaSuccess ? 0 : -5;
}
