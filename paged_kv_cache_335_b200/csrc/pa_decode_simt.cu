// pa_decode_simt.cu — single-query paged decode attention on the CUDA cores,
// and the log-sum-exp merge of context partitions.
//
// What it computes: for sequence s and query head h, softmax(scale q . K_t) V_t
// over the n = context_lens[s] cached tokens, K_t / V_t read from physical
// block block_tables[s][t / block_size], slot t % block_size ("AI 推理系列
// （十六）：PagedAttention——…", § PagedAttention 如何把连续序列映射到离散显存块 and
// § 非连续 KV 为什么需要专门的 Attention Kernel; the attention itself is the usual
// one, "PagedAttention原理详解：GPU显存优化与模型路由技术", § 显存消耗的三大来源).
//
// How (sm_100a, HBM-bound work, so no tensor cores here):
// * Grid = (partition, query head, sequence), the three grid dimensions of
//   "vLLM的Paged Attention技术：高效注意力机制解析", § 3.2 执行层次结构. A partition is
//   a range of logical tokens; with one partition the CTA covers the context.
// * The CTA's 4 warps take 16-token sub-tiles round robin (warp w: sub-tiles
//   w, w+4, ...), the balancing scheme of § 4.2 动态负载均衡 of the same page.
//   Each warp keeps its own running max / sum / accumulator.
// * Loads are 16-byte, coalesced along head_dim: a warp-wide load covers whole
//   rows of the (block, kv head) tile, which is one contiguous span in this
//   layout (the role of the x-split 5-D layout of § 2.2 on older GPUs).
// * q stays in registers, pre-scaled by scale * log2(e) so the softmax uses exp2.
// * The arithmetic order depends only on logical token positions (never on
//   physical block ids), so any placement of blocks gives identical bits.
#include <math.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

static __device__ unsigned int s_status_simt;

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

template <typename T, int D>
struct SimtShape {
    static constexpr int VEC = Elem<T>::kVec;              // elements per 16-byte chunk
    static constexpr int CPR = D / VEC;                    // chunks per K/V row
    static constexpr int RPL = 32 / CPR;                   // rows per warp-wide load
    static constexpr int SUB = (8 * RPL < 16) ? 8 * RPL : 16;  // rows per sub-tile
    static constexpr int ITER = SUB / RPL;                 // loads per lane per sub-tile
    static_assert(CPR <= 32 && 32 % CPR == 0, "row must map onto a warp");
    static_assert(16 % SUB == 0, "sub-tiles must not straddle a 16-slot boundary");
};

__device__ __forceinline__ int clamp_context(int ctx, int max_ctx, unsigned* status, bool report) {
    if (ctx < 0 || ctx > max_ctx) {
        if (report) atomicOr(status, kStatusBadIndex);
        ctx = ctx < 0 ? 0 : max_ctx;
    }
    return ctx;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
decode_simt_kernel(const DecodeParams p) {
    using S = SimtShape<T, D>;
    const int part = blockIdx.x;
    const int h = blockIdx.y;
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int c = lane % S::CPR;   // chunk of the row this lane reads
    const int rs = lane / S::CPR;  // row offset within a warp-wide load

    const int ctx = clamp_context(__ldg(p.context_lens + s), p.max_context_len, &s_status_simt,
                                  threadIdx.x == 0 && part == 0);
    const int t0 = part * p.partition_size;
    const int t1 = min(ctx, t0 + p.partition_size);
    const int64_t out_row = (int64_t)s * p.num_heads + h;
    if (t0 >= t1) {
        // Empty partition. With a single partition this is ctx == 0: out = 0.
        if (p.num_partitions == 1)
            for (int d = threadIdx.x; d < D; d += kThreads) Elem<T>::store(p.out, out_row * D + d, 0.f);
        return;
    }
    const int kh = h / (p.num_heads / p.num_kv_heads);

    float qf[S::VEC];
    {
        const uint4 raw = ld_v4(static_cast<const T*>(p.q) + out_row * D + c * S::VEC);
        Elem<T>::widen(raw, qf);
#pragma unroll
        for (int j = 0; j < S::VEC; ++j) qf[j] *= p.scale_log2;
    }

    float m = -INFINITY;  // running max of the scores (log2 units)
    float l = 0.f;        // running sum of exp2(score - m) over this lane's rows
    float acc[S::VEC];
#pragma unroll
    for (int j = 0; j < S::VEC; ++j) acc[j] = 0.f;

    const int32_t* table = p.block_tables + (int64_t)s * p.table_stride;
    const uint4* kbase = static_cast<const uint4*>(p.k_cache);
    const uint4* vbase = static_cast<const uint4*>(p.v_cache);
    const int n_sub = (t1 - t0 + S::SUB - 1) / S::SUB;

    for (int i = warp; i < n_sub; i += kWarps) {
        const int tok0 = t0 + i * S::SUB;
        const int phys = __ldg(table + (tok0 >> p.log2_block_size));
        if ((unsigned)phys >= (unsigned)p.num_blocks) {
            if (lane == 0) atomicOr(&s_status_simt, kStatusBadIndex);
            continue;
        }
        const int64_t row0 = ((int64_t)phys * p.num_kv_heads + kh) * p.block_size +
                             (tok0 & (p.block_size - 1));
        const uint4* kp = kbase + row0 * S::CPR + c;
        const uint4* vp = vbase + row0 * S::CPR + c;
        uint4 kr[S::ITER], vr[S::ITER];
#pragma unroll
        for (int it = 0; it < S::ITER; ++it) kr[it] = ld_stream(kp + (it * S::RPL + rs) * S::CPR);
#pragma unroll
        for (int it = 0; it < S::ITER; ++it) vr[it] = ld_stream(vp + (it * S::RPL + rs) * S::CPR);

        float sc[S::ITER];
#pragma unroll
        for (int it = 0; it < S::ITER; ++it) {
            float kf[S::VEC];
            Elem<T>::widen(kr[it], kf);
            float dot = 0.f;
#pragma unroll
            for (int j = 0; j < S::VEC; ++j) dot = fmaf(qf[j], kf[j], dot);
#pragma unroll
            for (int off = 1; off < S::CPR; off <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            const int tok = tok0 + it * S::RPL + rs;
            sc[it] = tok < t1 ? dot : -INFINITY;
        }
        float mt = sc[0];
#pragma unroll
        for (int it = 1; it < S::ITER; ++it) mt = fmaxf(mt, sc[it]);
#pragma unroll
        for (int off = S::CPR; off < 32; off <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float m_new = fmaxf(m, mt);  // finite: every sub-tile holds a valid token
        const float alpha = exp2f(m - m_new);
        l *= alpha;
#pragma unroll
        for (int j = 0; j < S::VEC; ++j) acc[j] *= alpha;
#pragma unroll
        for (int it = 0; it < S::ITER; ++it) {
            const float pr = exp2f(sc[it] - m_new);
            l += pr;
            const int tok = tok0 + it * S::RPL + rs;
            if (tok < t1) {  // slots past the context may hold anything, even NaN
                float vf[S::VEC];
                Elem<T>::widen(vr[it], vf);
#pragma unroll
                for (int j = 0; j < S::VEC; ++j) acc[j] = fmaf(pr, vf[j], acc[j]);
            }
        }
        m = m_new;
    }

    // Lanes with the same chunk c hold partial sums over different rows.
#pragma unroll
    for (int off = S::CPR; off < 32; off <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
        for (int j = 0; j < S::VEC; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    }

    __shared__ float sm_o[kWarps][D];
    __shared__ float sm_m[kWarps];
    __shared__ float sm_l[kWarps];
    if (rs == 0) {
#pragma unroll
        for (int j = 0; j < S::VEC; ++j) sm_o[warp][c * S::VEC + j] = acc[j];
    }
    if (lane == 0) {
        sm_m[warp] = m;
        sm_l[warp] = l;
    }
    __syncthreads();

    // Merge the warps in fixed order.
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w]);
    float wgt[kWarps];
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        wgt[w] = sm_m[w] == -INFINITY ? 0.f : exp2f(sm_m[w] - M);
        L = fmaf(sm_l[w], wgt[w], L);
    }
    for (int d = threadIdx.x; d < D; d += kThreads) {
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) o = fmaf(sm_o[w][d], wgt[w], o);
        const float val = L > 0.f ? o / L : 0.f;
        if (p.num_partitions == 1) {
            Elem<T>::store(p.out, out_row * D + d, val);
        } else {
            p.ws_o[(out_row * p.num_partitions + part) * D + d] = val;
        }
    }
    if (p.num_partitions > 1 && threadIdx.x == 0) {
        float* ml = p.ws_ml + (out_row * p.num_partitions + part) * 2;
        ml[0] = L > 0.f ? M : -INFINITY;
        ml[1] = L;
    }
}

// Merge of partitions j = 0 .. ceil(n / partition_size) - 1 of one (s, h):
//   M = max_j m_j,  w_j = l_j * 2^(m_j - M),  out = sum_j w_j o_j / sum_j w_j,
// where o_j is partition j's normalised output. This is the exact softmax over
// the union of the partitions. grid = (num_heads, num_seqs). Launched as a
// programmatic dependent of the decode kernel: it may start while the decode
// drains and waits (griddepcontrol.wait) for all of its results.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
partition_reduce_kernel(const DecodeParams p) {
    extern __shared__ float sm_w[];  // [num_partitions] weights
    __shared__ float sm_L;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int h = blockIdx.x;
    const int s = blockIdx.y;
    const int ctx = clamp_context(__ldg(p.context_lens + s), p.max_context_len, &s_status_simt, false);
    const int n = (ctx + p.partition_size - 1) / p.partition_size;
    const int64_t out_row = (int64_t)s * p.num_heads + h;
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
cudaError_t launch_simt_t(const DecodeParams& p, cudaStream_t stream) {
    dim3 grid((unsigned)p.num_partitions, (unsigned)p.num_heads, (unsigned)p.num_seqs);
    decode_simt_kernel<T, D><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_reduce_t(const DecodeParams& p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_heads, (unsigned)p.num_seqs);
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

bool simt_supported(int dtype, int head_dim) {
    return (dtype == 0 || dtype == 1) && (head_dim == 64 || head_dim == 128);
}

cudaError_t launch_decode_simt(const DecodeParams& p, int dtype, int head_dim, cudaStream_t stream) {
    if (dtype == 0) {
        return head_dim == 64 ? launch_simt_t<float, 64>(p, stream) : launch_simt_t<float, 128>(p, stream);
    }
    return head_dim == 64 ? launch_simt_t<__nv_bfloat16, 64>(p, stream)
                          : launch_simt_t<__nv_bfloat16, 128>(p, stream);
}

cudaError_t launch_partition_reduce(const DecodeParams& p, int dtype, int head_dim,
                                    cudaStream_t stream) {
    if (dtype == 0) {
        return head_dim == 64 ? launch_reduce_t<float, 64>(p, stream)
                              : launch_reduce_t<float, 128>(p, stream);
    }
    return head_dim == 64 ? launch_reduce_t<__nv_bfloat16, 64>(p, stream)
                          : launch_reduce_t<__nv_bfloat16, 128>(p, stream);
}

cudaError_t read_status_simt(unsigned* bits, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(bits, s_status_simt, sizeof(unsigned));
    if (e != cudaSuccess || !clear) return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(s_status_simt, &zero, sizeof(unsigned));
}

}  // namespace pa
