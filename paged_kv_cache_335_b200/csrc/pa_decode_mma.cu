// pa_decode_mma.cu — paged decode attention for grouped-query attention on the
// tensor cores (bf16 in, fp32 accumulate).
//
// Same result as the CUDA-core kernel (softmax(scale q . K_t) V_t over the
// block-table-gathered context, "AI 推理系列（十六）：PagedAttention——…",
// § 非连续 KV 为什么需要专门的 Attention Kernel), for query groups of
// g = num_heads / num_kv_heads in [2, 8] (GQA, named in the same page's table
// of mechanisms). With g query rows per KV row the step costs g flop per byte
// of K/V: at g = 8 that is more than the CUDA cores sustain at HBM speed, so
// the two contractions of a 16-token sub-tile run as m16n8k16 MMAs:
//
//   S^T[16 tok][8 heads] = K[16 tok][D] . Q^T[D][8 heads]      (D/16 MMAs)
//   O^T[D][8 heads]     += V^T[D][16 tok] . P^T[16 tok][8 heads] (D/16 MMAs)
//
// Token rows are the MMA's M dimension and the query group its N dimension, so
// no MMA lane is wasted at g = 8. Operands come straight from HBM into
// registers with 16-byte loads: the order of head_dim inside each QK k-step is
// permuted identically for K and Q (a sum does not care), and the rows of each
// PV m-tile are mapped to head_dim so that a thread's V elements are 16
// contiguous bytes. P^T is made from the S^T accumulator with one
// movmatrix.trans per 8x8 half, without shared memory.
//
// Grid = (partition, kv head, sequence); 4 warps take 16-token sub-tiles round
// robin ("vLLM的Paged Attention技术：高效注意力机制解析", § 3.2 and § 4.2). The
// arithmetic order depends only on logical positions.
#include <math.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

static __device__ unsigned int s_status_mma;

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kGroupMax = 8;

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

// Two floats -> bf16x2 (round to nearest even), `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

template <int D>
__global__ void __launch_bounds__(kThreads)
decode_mma_kernel(const DecodeParams p) {
    constexpr int KSTEPS = D / 16;  // k-steps of the QK product
    constexpr int KCH = D / 32;     // 16-byte K chunks per row per thread
    constexpr int VCH = D / 64;     // 16-byte V chunks per token per thread
    constexpr int MT = D / 16;      // m-tiles of the PV product
    const int part = blockIdx.x;
    const int kh = blockIdx.y;
    const int s = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int r = lane >> 2;  // MMA group id
    const int c = lane & 3;   // thread in group
    const int group = p.num_heads / p.num_kv_heads;

    int ctx = __ldg(p.context_lens + s);
    if (ctx < 0 || ctx > p.max_context_len) {
        if (threadIdx.x == 0 && part == 0) atomicOr(&s_status_mma, kStatusBadIndex);
        ctx = ctx < 0 ? 0 : p.max_context_len;
    }
    const int t0 = part * p.partition_size;
    const int t1 = min(ctx, t0 + p.partition_size);
    const int64_t head0 = (int64_t)s * p.num_heads + (int64_t)kh * group;  // first q row
    if (t0 >= t1) {
        if (p.num_partitions == 1)
            for (int idx = threadIdx.x; idx < group * D; idx += kThreads)
                Elem<__nv_bfloat16>::store(p.out, head0 * D + idx, 0.f);
        return;
    }

    // Q^T fragments (B operand of the QK MMA): thread (r, c) holds query row r.
    // k-step j uses head_dim {32*(j/2) + 8c + 4*(j%2) + 0..3} for this thread.
    uint32_t qb[KSTEPS][2];
    if (r < group) {
        const uint16_t* qrow = static_cast<const uint16_t*>(p.q) + (head0 + r) * D;
#pragma unroll
        for (int jp = 0; jp < KCH; ++jp) {
            const uint4 w = ld_v4(qrow + jp * 32 + c * 8);
            qb[2 * jp][0] = w.x;
            qb[2 * jp][1] = w.y;
            qb[2 * jp + 1][0] = w.z;
            qb[2 * jp + 1][1] = w.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j) qb[j][0] = qb[j][1] = 0u;
    }

    float acc[MT][4];  // O^T fragments: rows = head_dim (mapped), cols = heads 2c, 2c+1
#pragma unroll
    for (int i = 0; i < MT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;  // running max of heads 2c, 2c+1 (log2 units)
    float l0 = 0.f, l1 = 0.f;              // this thread's share of the running sums

    const int32_t* table = p.block_tables + (int64_t)s * p.table_stride;
    const uint16_t* kbase = static_cast<const uint16_t*>(p.k_cache);
    const uint16_t* vbase = static_cast<const uint16_t*>(p.v_cache);
    const int n_sub = (t1 - t0 + 15) >> 4;
    // tokens of the sub-tile whose V elements this thread feeds to the PV MMA
    const int tv0 = 2 * c, tv1 = 2 * c + 1, tv2 = 2 * c + 8, tv3 = 2 * c + 9;

    for (int i = warp; i < n_sub; i += kWarps) {
        const int tok0 = t0 + (i << 4);
        const int phys = __ldg(table + (tok0 >> p.log2_block_size));
        if ((unsigned)phys >= (unsigned)p.num_blocks) {
            if (lane == 0) atomicOr(&s_status_mma, kStatusBadIndex);
            continue;
        }
        const int64_t row0 = ((int64_t)phys * p.num_kv_heads + kh) * p.block_size +
                             (tok0 & (p.block_size - 1));
        const uint16_t* kt = kbase + row0 * D;
        const uint16_t* vt = vbase + row0 * D;
        uint4 kr[2][KCH];
        uint4 vr[4][VCH];
#pragma unroll
        for (int jp = 0; jp < KCH; ++jp) {
            kr[0][jp] = ld_stream(kt + r * D + jp * 32 + c * 8);
            kr[1][jp] = ld_stream(kt + (r + 8) * D + jp * 32 + c * 8);
        }
#pragma unroll
        for (int hh = 0; hh < VCH; ++hh) {
            vr[0][hh] = ld_stream(vt + tv0 * D + hh * 64 + r * 8);
            vr[1][hh] = ld_stream(vt + tv1 * D + hh * 64 + r * 8);
            vr[2][hh] = ld_stream(vt + tv2 * D + hh * 64 + r * 8);
            vr[3][hh] = ld_stream(vt + tv3 * D + hh * 64 + r * 8);
        }

        // S^T = K . Q^T
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j) {
            const int jp = j >> 1;
            const bool odd = j & 1;
            mma_16816(sc, odd ? kr[0][jp].z : kr[0][jp].x, odd ? kr[1][jp].z : kr[1][jp].x,
                      odd ? kr[0][jp].w : kr[0][jp].y, odd ? kr[1][jp].w : kr[1][jp].y,
                      qb[j][0], qb[j][1]);
        }
        const int nvalid = t1 - tok0;  // >= 1
        const bool lo_ok = r < nvalid, hi_ok = r + 8 < nvalid;
        const float s0 = lo_ok ? sc[0] * p.scale_log2 : -INFINITY;  // token r,   head 2c
        const float s1 = lo_ok ? sc[1] * p.scale_log2 : -INFINITY;  // token r,   head 2c+1
        const float s2 = hi_ok ? sc[2] * p.scale_log2 : -INFINITY;  // token r+8, head 2c
        const float s3 = hi_ok ? sc[3] * p.scale_log2 : -INFINITY;  // token r+8, head 2c+1

        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
        const uint32_t x0 = pack_bf16x2(exp2f(s0 - mn0), exp2f(s1 - mn1));
        const uint32_t x1 = pack_bf16x2(exp2f(s2 - mn0), exp2f(s3 - mn1));
        // the sums use the same rounded weights the PV product sees
        l0 = fmaf(l0, al0, bf16_lo(x0) + bf16_lo(x1));
        l1 = fmaf(l1, al1, bf16_hi(x0) + bf16_hi(x1));
        m0 = mn0;
        m1 = mn1;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            acc[t][0] *= al0;
            acc[t][1] *= al1;
            acc[t][2] *= al0;
            acc[t][3] *= al1;
        }
        const uint32_t pb0 = movmatrix_trans(x0);  // P^T rows (tokens) 2c, 2c+1; col head r
        const uint32_t pb1 = movmatrix_trans(x1);  // tokens 2c+8, 2c+9
        if (nvalid < 16) {  // slots past the context may hold anything, even NaN
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int hh = 0; hh < VCH; ++hh) {
                if (tv0 >= nvalid) vr[0][hh] = z;
                if (tv1 >= nvalid) vr[1][hh] = z;
                if (tv2 >= nvalid) vr[2][hh] = z;
                if (tv3 >= nvalid) vr[3][hh] = z;
            }
        }
        // O^T += V^T . P^T ; m-tile t covers head_dim 64*(t/4) + 8r + 2*(t%4) (+1 for row r+8)
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            const int hh = t >> 2, w = t & 3;
            const uint32_t xa = word(vr[0][hh], w), xb = word(vr[1][hh], w);
            const uint32_t ya = word(vr[2][hh], w), yb = word(vr[3][hh], w);
            mma_16816(acc[t], __byte_perm(xa, xb, 0x5410), __byte_perm(xa, xb, 0x7632),
                      __byte_perm(ya, yb, 0x5410), __byte_perm(ya, yb, 0x7632), pb0, pb1);
        }
    }

#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }

    __shared__ float sm_o[kWarps][kGroupMax][D];
    __shared__ float sm_m[kWarps][kGroupMax];
    __shared__ float sm_l[kWarps][kGroupMax];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        const int d0 = (t >> 2) * 64 + r * 8 + 2 * (t & 3);
        sm_o[warp][2 * c][d0] = acc[t][0];
        sm_o[warp][2 * c + 1][d0] = acc[t][1];
        sm_o[warp][2 * c][d0 + 1] = acc[t][2];
        sm_o[warp][2 * c + 1][d0 + 1] = acc[t][3];
    }
    if (r == 0) {
        sm_m[warp][2 * c] = m0;
        sm_m[warp][2 * c + 1] = m1;
        sm_l[warp][2 * c] = l0;
        sm_l[warp][2 * c + 1] = l1;
    }
    __syncthreads();

    for (int idx = threadIdx.x; idx < group * D; idx += kThreads) {
        const int n = idx / D;
        const int d = idx - n * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][n]);
        float L = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float wg = sm_m[w][n] == -INFINITY ? 0.f : exp2f(sm_m[w][n] - M);
            L = fmaf(sm_l[w][n], wg, L);
            o = fmaf(sm_o[w][n][d], wg, o);
        }
        const float val = L > 0.f ? o / L : 0.f;
        const int64_t row = head0 + n;
        if (p.num_partitions == 1) {
            Elem<__nv_bfloat16>::store(p.out, row * D + d, val);
        } else {
            p.ws_o[(row * p.num_partitions + part) * D + d] = val;
            if (d == 0) {
                float* ml = p.ws_ml + (row * p.num_partitions + part) * 2;
                ml[0] = L > 0.f ? M : -INFINITY;
                ml[1] = L;
            }
        }
    }
}

}  // namespace

bool mma_supported(int dtype, int head_dim, int group) {
    return dtype == 1 && (head_dim == 64 || head_dim == 128) && group >= 2 && group <= kGroupMax;
}

cudaError_t launch_decode_mma(const DecodeParams& p, int head_dim, cudaStream_t stream) {
    dim3 grid((unsigned)p.num_partitions, (unsigned)p.num_kv_heads, (unsigned)p.num_seqs);
    if (head_dim == 64)
        decode_mma_kernel<64><<<grid, kThreads, 0, stream>>>(p);
    else
        decode_mma_kernel<128><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t read_status_mma(unsigned* bits, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(bits, s_status_mma, sizeof(unsigned));
    if (e != cudaSuccess || !clear) return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(s_status_mma, &zero, sizeof(unsigned));
}

}  // namespace pa
