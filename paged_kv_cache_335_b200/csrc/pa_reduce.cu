// pa_reduce.cu — log-sum-exp merge of the context partitions of pa_decode.
//
// When a long context is split into partitions ("vLLM的Paged Attention技术：高效
// 注意力机制解析", § 3.2: the grid's 分区 dimension), each partition j of a
// (sequence, query head) leaves its running max m_j (log2 units), running sum
// l_j and normalised partial output o_j in the workspace. The pages do not
// describe the merge; the one that reproduces the exact softmax over the union
// of the partitions is the log-sum-exp merge below.
#include <math.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ int clamp_context(int ctx, int max_ctx) {
    return ctx < 0 ? 0 : (ctx > max_ctx ? max_ctx : ctx);
}

// Merge of partitions j = 0 .. ceil(n / partition_size) - 1 of one (s, h):
//   M = max_j m_j,  w_j = l_j * 2^(m_j - M),  out = sum_j w_j o_j / sum_j w_j,
// where o_j is partition j's normalised output. This is the exact softmax over
// the union of the partitions. grid = (num_heads, rows of out). Launched as a
// programmatic dependent of the decode kernel: it may start while the decode
// drains and waits (griddepcontrol.wait) for all of its results.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
partition_reduce_kernel(const DecodeParams p) {
    extern __shared__ float sm_w[];  // [num_partitions] weights
    __shared__ float sm_L;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int h = blockIdx.x;
    const int row = blockIdx.y;  // sequence, or query token with multi-token queries
    int ctx;
    if (p.query_start == nullptr) {
        ctx = clamp_context(__ldg(p.context_lens + row), p.max_context_len);
    } else {
        // the sequence holding query token `row`: query_start[s] <= row < query_start[s+1]
        int lo = 0, hi = p.num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(p.query_start + mid) <= row) lo = mid; else hi = mid - 1;
        }
        const int q0 = __ldg(p.query_start + lo), n_new = __ldg(p.query_start + lo + 1) - q0;
        const int lim = clamp_context(__ldg(p.context_lens + lo), p.max_context_len) - n_new +
                        (row - q0) + 1;  // causal end of this query token
        ctx = lim < 0 ? 0 : lim;
    }
    const int n = (ctx + p.partition_size - 1) / p.partition_size;
    const int64_t out_row = (int64_t)row * p.num_heads + h;
    const float* ml = p.ws_ml + out_row * p.num_partitions * 2;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        float M = -INFINITY;
        for (int j = lane; j < n; j += 32) M = fmaxf(M, ml[2 * j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float L = 0.f;
        for (int j = lane; j < n; j += 32) {
            const float mj = ml[2 * j];
            const float w = mj == -INFINITY ? 0.f : ml[2 * j + 1] * exp2f(mj - M);
            sm_w[j] = w;
            L += w;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        if (lane == 0) sm_L = L;
    }
    __syncthreads();
    const float L = sm_L;
    const float* o = p.ws_o + out_row * p.num_partitions * D;
    for (int d = threadIdx.x; d < D; d += kThreads) {
        float acc = 0.f;
#pragma unroll 8
        for (int j = 0; j < n; ++j) acc = fmaf(sm_w[j], o[(int64_t)j * D + d], acc);
        Elem<T>::store(p.out, out_row * D + d, L > 0.f ? acc / L : 0.f);
    }
}

template <typename T, int D>
cudaError_t launch_reduce_t(const DecodeParams& p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_heads, (unsigned)p.num_rows);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)p.num_partitions * sizeof(float);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, partition_reduce_kernel<T, D>, p);
}

}  // namespace

cudaError_t launch_partition_reduce(const DecodeParams& p, int dtype, int head_dim,
                                    cudaStream_t stream) {
    if (dtype == 0) {
        return head_dim == 64 ? launch_reduce_t<float, 64>(p, stream)
                              : launch_reduce_t<float, 128>(p, stream);
    }
    return head_dim == 64 ? launch_reduce_t<__nv_bfloat16, 64>(p, stream)
                          : launch_reduce_t<__nv_bfloat16, 128>(p, stream);
}

}  // namespace pa
