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
//
// Warp w takes partitions w, w + 4, ...; each lane holds D / 32 consecutive
// elements of a partial output, and a warp issues the loads of up to kBatch
// partitions (with the (m, l) loads of the maximum) before it uses any of
// them, so one round trip to memory covers the typical partition count. The
// warps' sums meet in shared memory.
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 16;

template <int V>
struct VecF;
template <>
struct VecF<2> {
    using type = float2;
};
template <>
struct VecF<4> {
    using type = float4;
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
partition_reduce_kernel(const DecodeParams p) {
    constexpr int V = D / 32;  // elements per lane
    using Vec = typename VecF<V>::type;
    __shared__ float sm_acc[kWarps][D];
    __shared__ float sm_l[kWarps];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int h = blockIdx.x;
    const int row = blockIdx.y;  // sequence, or query token with multi-token queries
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    const float2* ml = reinterpret_cast<const float2*>(p.ws_ml + out_row * p.num_partitions * 2);
    const float* o = p.ws_o + out_row * p.num_partitions * D;
    // A warp's batch of partials (output rows and their (m, l)) is requested
    // before the maximum over all partitions is formed, so the first batch and
    // the maxima share one round trip to memory.
    Vec ov[kBatch];
    float2 mlv[kBatch];
    auto load_batch = [&](int j0) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = j0 + u * kWarps;
            if (j < n) {
                ov[u] = *reinterpret_cast<const Vec*>(o + (int64_t)j * D + lane * V);
                mlv[u] = ml[j];
            }
        }
    };
    load_batch(warp);
    // M over all partitions, by every warp (no block barrier needed for it)
    float M = -INFINITY;
    for (int j = lane; j < n; j += 32) M = fmaxf(M, ml[j].x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float acc[V];
#pragma unroll
    for (int k = 0; k < V; ++k) acc[k] = 0.f;
    float L = 0.f;
    for (int j0 = warp; j0 < n; j0 += kWarps * kBatch) {
        if (j0 != warp) load_batch(j0);
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = j0 + u * kWarps;
            if (j < n) {
                const float w = mlv[u].x == -INFINITY ? 0.f : mlv[u].y * exp2f(mlv[u].x - M);
                const float* x = reinterpret_cast<const float*>(&ov[u]);
#pragma unroll
                for (int k = 0; k < V; ++k) acc[k] = fmaf(w, x[k], acc[k]);
                L += w;
            }
        }
    }
#pragma unroll
    for (int k = 0; k < V; ++k) sm_acc[warp][lane * V + k] = acc[k];
    if (lane == 0) sm_l[warp] = L;
    __syncthreads();
    float Lt = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) Lt += sm_l[w];
    for (int d = threadIdx.x; d < D; d += kThreads) {
        float a = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) a += sm_acc[w][d];
        Elem<T>::store(p.out, out_row * D + d, Lt > 0.f ? a / Lt : 0.f);
    }
}

template <typename T, int D>
cudaError_t launch_reduce_t(const DecodeParams& p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_heads, (unsigned)p.num_rows);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
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
