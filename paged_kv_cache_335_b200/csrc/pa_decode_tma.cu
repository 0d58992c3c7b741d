// pa_decode_tma.cu — paged decode attention with K/V staged through shared
// memory by the Tensor Memory Accelerator (sm_100a).
//
// What it computes is unchanged: for sequence s and query head h,
// softmax(scale q . K_t) V_t over the n = context_lens[s] cached tokens, K_t and
// V_t taken from physical block block_tables[s][t / block_size], slot
// t % block_size ("AI 推理系列（十六）：PagedAttention——…", § PagedAttention 如何
// 把连续序列映射到离散显存块 and § 非连续 KV 为什么需要专门的 Attention Kernel).
//
// How. One CTA = (partition, head or kv head, sequence), the three grid
// dimensions of "vLLM的Paged Attention技术：高效注意力机制解析", § 3.2. Inside it:
// * a producer warp reads the block-table entries of the partition 32 at a
//   time and, for every 16-token sub-tile, issues tiled TMA loads of the K and
//   V rows (boxes of 16 rows x 128 bytes, 128-byte swizzle, no multicast) into
//   a ring of shared-memory stages guarded by mbarriers (full: data landed;
//   empty: stage released);
// * consumer warps take sub-tiles round robin (warp w: w, w+4, ...; § 4.2 of
//   the same page), copy their fragments out of the stage, release it, and
//   update a running max / sum / accumulator (online softmax in exp2).
// Four consumers share this pipeline: the CUDA-core one (one query head per
// CTA; any dtype, quantised codes through a mixed-precision fma), the
// tensor-core one for grouped-query attention (bf16 or codes, group 2..8:
// S^T = K Q^T and O^T += V^T P^T as m16n8k16 MMAs, tokens as M, the query
// group as N), the grouped one (several sequences or query tokens that share
// blocks, one CTA per group, units of several sub-tiles per softmax step) and
// an opt-in tcgen05 variant of the grouped one. The swizzle makes every
// consumer fragment load bank-conflict free. Every wait is bounded: after
// kWaitLimitNs the waiter records PA_ERR_TIMEOUT and carries on, so the kernel
// always terminates. The arithmetic order depends only on logical token
// positions.
#include <math.h>

#include <type_traits>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tma.cuh"

namespace pa {

static __device__ unsigned int s_status_tma;

namespace {

// Tunables (compile-time; the defaults are the measured choice, see the
// variant sweeps recorded with the profiles). Consumer warps per CTA, ring
// bytes, and for the persistent tensor-core kernel the CTAs per SM it is
// compiled (and its grid sized) for.
#ifndef PA_SIMT_CONSUMER_WARPS
#define PA_SIMT_CONSUMER_WARPS 4
#endif
#ifndef PA_SIMT_RING_BYTES
#define PA_SIMT_RING_BYTES 65536
#endif
#ifndef PA_MMA_CONSUMER_WARPS
#define PA_MMA_CONSUMER_WARPS 2
#endif
#ifndef PA_MMA_RING_BYTES
#define PA_MMA_RING_BYTES 49152
#endif
#ifndef PA_MMA_MIN_BLOCKS
#define PA_MMA_MIN_BLOCKS 4
#endif
#ifndef PA_MMA_SPLIT_QK
#define PA_MMA_SPLIT_QK 0
#endif


constexpr int kBoxBytes = 16 * 128;  // 16 rows x 128 bytes
constexpr int kGroupMax = 8;

// Geometry of one pipeline: element type, head_dim, consumer warps, ring bytes.
template <typename T_, int D_, int CW_, int RING_>
struct Geom {
    using T = T_;
    static constexpr int D = D_;
    static constexpr int kCW = CW_;                              // consumer warps
    static constexpr int kThreads = (CW_ + 1) * 32;              // + one producer warp
    static constexpr int kBoxes = D_ * (int)sizeof(T_) / 128;    // boxes per K (or V) row set
    static constexpr int kBoxElems = 128 / (int)sizeof(T_);      // elements per box row
    static constexpr int kStageBytes = 2 * kBoxes * kBoxBytes;   // K + V of one sub-tile
    // Stages: as many as fit in RING_ bytes, rounded DOWN to a multiple of the
    // consumer warps. Consumers take sub-tiles round robin, so with a multiple
    // every stage always belongs to the same warp and no warp can wait on a
    // stage more than one phase ahead of its data; otherwise a warp can test
    // a phase parity two phases early, see it as already complete, read a
    // stage before its load lands and release it twice.
    static constexpr int kFit = RING_ / kStageBytes;
    static constexpr int kStages = kFit < CW_ ? CW_ : (kFit / CW_) * CW_;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static_assert(kStages % CW_ == 0, "stage count must be a multiple of the consumer warps");
};

struct Ring {
    uint32_t stages;  // shared address of stage 0 (1024-byte aligned)
    uint32_t full;    // shared address of full[0]; full[i] at + 8 i
    uint32_t empty;
    int* valid;       // per stage: 1 = data loaded, 0 = skipped (bad block id)
};

// Issue of one sub-tile by one producer lane: wait until its stage is free,
// then load K and V rows [row, row + 16) of kv head `kh` into it (or, for a
// block id outside the pool, mark the stage empty-handed and complete it).
// A stage may carry a header word (`hdr`, one per stage), written before the
// stage is completed. Returns false if the wait timed out (nothing was issued).
template <class G>
__device__ __forceinline__ bool issue_subtile(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                              const DecodeParams& p, const Ring& ring, int gi,
                                              int phys, int kh, int tok0,
                                              uint32_t* hdr = nullptr, uint32_t hval = 0,
                                              uint32_t* hdr2 = nullptr, uint32_t hval2 = 0) {
    const int st = gi % G::kStages;
    const uint32_t round = (uint32_t)(gi / G::kStages);
    if (!mbar_wait_bounded(ring.empty + 8 * st, (round & 1u) ^ 1u)) {
        atomicOr(&s_status_tma, kStatusTimeout);
        return false;
    }
    if (gi == p.test_skip_position) return true;  // test hook: leave this stage unloaded
    if (hdr != nullptr) hdr[st] = hval;
    if (hdr2 != nullptr) hdr2[st] = hval2;
    if ((unsigned)phys < (unsigned)p.num_blocks) {
        ring.valid[st] = 1;
        const uint32_t full = ring.full + 8 * st;
        mbar_arrive_expect_tx(full, G::kStageBytes);
        const int32_t row = (phys * p.num_kv_heads + kh) * p.block_size + (tok0 & (p.block_size - 1));
        const uint32_t sb = ring.stages + st * G::kStageBytes;
#pragma unroll
        for (int b = 0; b < G::kBoxes; ++b)
            tma_load_2d(sb + b * kBoxBytes, kmap, b * G::kBoxElems, row, full);
#pragma unroll
        for (int b = 0; b < G::kBoxes; ++b)
            tma_load_2d(sb + (G::kBoxes + b) * kBoxBytes, vmap, b * G::kBoxElems, row, full);
    } else {
        atomicOr(&s_status_tma, kStatusBadIndex);
        ring.valid[st] = 0;
        mbar_arrive(ring.full + 8 * st);
    }
    return true;
}

// Issue a batch of `cnt` <= 32 consecutive sub-tiles (ring positions g .. g+cnt-1)
// of one item; lane l owns sub-tile l (`phys` = its block id). Lanes issue in
// sub-rounds of kStages, so each sub-round touches every stage at most once and
// a stage's rounds are issued in order. `issued` tracks 1 + the last position
// issued; `dead` becomes warp-wide once any wait timed out.
template <class G>
__device__ __forceinline__ void issue_batch(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                            const DecodeParams& p, const Ring& ring, int g, int cnt,
                                            int phys, int kh, int tok0_lane, int lane, int& issued,
                                            bool& dead) {
    for (int k0 = 0; k0 < cnt && !dead; k0 += G::kStages) {
        bool ok = true;
        if (lane >= k0 && lane < k0 + G::kStages && lane < cnt) {
            ok = issue_subtile<G>(kmap, vmap, p, ring, g + lane, phys, kh, tok0_lane);
            if (ok) issued = g + lane + 1;
        }
        dead = __any_sync(0xffffffffu, !ok);
    }
    issued = __reduce_max_sync(0xffffffffu, issued);
}

// Producer of one item: all lanes fetch block-table entries, 32 sub-tiles at a
// time, and issue them. Returns the ring position after the item.
template <class G>
__device__ __forceinline__ int produce_item(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                            const DecodeParams& p, const Ring& ring, int s, int kh,
                                            int t0, int n_sub, int lane, int g, int& issued,
                                            bool& dead) {
    const int32_t* table = p.block_tables + (int64_t)s * p.table_stride;
    for (int base = 0; base < n_sub && !dead; base += 32) {
        const int i = base + lane;
        const int tok0 = t0 + (i << 4);
        int phys = -1;
        if (i < n_sub) phys = __ldg(table + (tok0 >> p.log2_block_size));
        issue_batch<G>(kmap, vmap, p, ring, g + base, min(32, n_sub - base), phys, kh, tok0,
                          lane, issued, dead);
    }
    return g + n_sub;
}

// Drain: the last load of every stage has landed before the CTA reuses or
// releases shared memory (immediate unless a consumer gave up waiting).
template <class G>
__device__ __forceinline__ void drain_ring(const Ring& ring, int issued, int lane) {
    if (lane != 0 || issued <= 0) return;
    const int last = min(issued, G::kStages);
    for (int st = 0; st < last; ++st) {
        const int it = issued - 1 - ((issued - 1 - st) % G::kStages);
        const uint32_t round = (uint32_t)(it / G::kStages);
        if (!mbar_wait_bounded(ring.full + 8 * st, round & 1u)) atomicOr(&s_status_tma, kStatusTimeout);
    }
}

// Shared memory: [ring] [extra_bytes] [full bars] [empty bars] [valid]. The
// dynamic shared memory is declared 1024-byte aligned (the 128-byte swizzle
// repeats every 1024 bytes and the fragment addressing assumes box bases on
// that boundary); setup_ring returns nullptr if it is not, and the kernel then
// records kStatusSmemAlign and returns before touching shared memory.
// `releases`: arrivals that free a stage (the consumer warps that read every
// stage; 1 when each stage has a single reader).
template <class G>
__device__ __forceinline__ uint8_t* setup_ring(uint8_t* smem_raw, Ring& ring, int extra_bytes = 0,
                                               int releases = 1) {
    const uint32_t raw = smem_u32(smem_raw);
    if (raw & 1023u) return nullptr;
    uint8_t* base = smem_raw;
    ring.stages = raw;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + G::kRingBytes + ((extra_bytes + 7) & ~7));
    ring.full = smem_u32(bars);
    ring.empty = smem_u32(bars + G::kStages);
    ring.valid = reinterpret_cast<int*>(bars + 2 * G::kStages);
    if (threadIdx.x == 0) {
        for (int st = 0; st < G::kStages; ++st) {
            mbar_init(ring.full + 8 * st, 1);
            mbar_init(ring.empty + 8 * st, releases);
        }
        fence_barrier_init();
    }
    return base;
}

template <class G>
constexpr size_t smem_bytes(int extra_bytes = 0) {
    return G::kRingBytes + ((extra_bytes + 7) & ~7) + 2 * G::kStages * 8 + G::kStages * 4 + 64;
}

__device__ __forceinline__ int clamp_ctx(int ctx, int max_ctx, bool report) {
    if (ctx < 0 || ctx > max_ctx) {
        if (report) atomicOr(&s_status_tma, kStatusBadIndex);
        ctx = ctx < 0 ? 0 : max_ctx;
    }
    return ctx;
}

// 2^x by the hardware approximation (ex2.approx.ftz: relative error about
// 2^-22; results below 2^-126 flush to 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// q on the paths over codes is rounded to f16 (the MMA operand type beside the
// codes). To keep that rounding exact whatever q's magnitude, q is scaled by
// 2^-sh first, sh chosen so that the largest |q| a warp holds lands in
// [2^14, 2^15), and the scores are scaled by 2^sh after the products. Both
// scalings are by powers of two: every bf16 q within 2^29 of that largest one
// becomes an f16 exactly (f16: 11 significant bits from 2^-14 up to 65504),
// and the fp32 products and sums are the unshifted ones times 2^-sh exactly,
// so the scores do not depend on sh. (Rounding q to f16 unshifted would turn
// |q| > 65504 into infinity and drop bits below 2^-14.)
__device__ __forceinline__ int q_shift_warp(float amax_lane) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(amax_lane));
    if (m == 0u) return 0;
    const int e = (int)((m >> 23) & 0xFFu) - 127;  // floor(log2 of the largest |q|)
    return max(-112, min(113, e - 14));
}
// 2^e for -126 <= e <= 127
__device__ __forceinline__ float pow2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// Softmax weights of the CUDA-core consumer over quantised codes by
// ex2_approx rather than exp2f: that consumer is bound by instruction issue
// (one widening per code), bf16 and fp32 caches are bound by HBM.
#ifndef PA_SIMT_CODES_FAST_EXP
#define PA_SIMT_CODES_FAST_EXP 1
#endif
// Int8 codes widened with a bias of 1152 (one byte permute per two codes, no
// per-code subtraction); the bias leaves the scores as 1152 x the sum of the
// lane's q elements and the output as 1152 x the sum of the weights. The
// biased terms are ~10x the true ones, so the fp32 sums carry ~10x the rounding
// of exactly widened codes (still far inside the bf16 bars). Off: the codes
// are widened exactly (one f16 subtraction per two codes; 13B int8 step 502 vs
// 485 us on a B200).
#ifndef PA_SIMT_INT8_BIASED
#define PA_SIMT_INT8_BIASED 1
#endif
// Codes as f16 operands of the mixed-precision fma (f16 x f16 + f32 -> f32,
// one instruction per code, no widening to f32): q is rounded to f16 (exact
// for bf16 values of magnitude 2^-14 .. 65504, as on the tensor-core path
// over codes) and scaled after the dot product; the weights are rounded to
// f16 and their sum is kept over the rounded values.
#ifndef PA_SIMT_CODES_MIXED_FMA
#define PA_SIMT_CODES_MIXED_FMA 1
#endif

// d = a * b + c for the two f16 halves of a and b (low with c0, high with c1),
// products exact, one rounding to f32 each.
__device__ __forceinline__ void fma2_f16_f32(uint32_t a, uint32_t b, float& c0, float& c1) {
    asm("{\n .reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %2;\n mov.b32 {bl, bh}, %3;\n"
        " fma.rn.f32.f16 %0, al, bl, %0;\n fma.rn.f32.f16 %1, ah, bh, %1;\n}"
        : "+f"(c0), "+f"(c1) : "r"(a), "r"(b));
}
// d = p * (both halves of b) + c, p one f16 value (the low half of pp).
__device__ __forceinline__ void fma2_f16s_f32(uint32_t pp, uint32_t b, float& c0, float& c1) {
    asm("{\n .reg .b16 pl, ph, bl, bh;\n mov.b32 {pl, ph}, %2;\n mov.b32 {bl, bh}, %3;\n"
        " fma.rn.f32.f16 %0, pl, bl, %0;\n fma.rn.f32.f16 %1, pl, bh, %1;\n}"
        : "+f"(c0), "+f"(c1) : "r"(pp), "r"(b));
}

// 16 codes -> 8 f16x2 words in order: E4M3 exactly; int8 as 1152 + code
// (exact), or with kExactInt8 the code itself (one exact f16 subtraction of
// 1152 per two codes).
template <typename TC, bool kExactInt8 = false>
__device__ __forceinline__ void codes_to_f16x2(const uint4& c, uint32_t (&h)[8]) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (std::is_same<TC, E4M3Code>::value) {
            asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %2;\n"
                " cvt.rn.f16x2.e4m3x2 %0, lo;\n cvt.rn.f16x2.e4m3x2 %1, hi;\n}"
                : "=r"(h[2 * i]), "=r"(h[2 * i + 1]) : "r"(w[i]));
        } else {
            const uint32_t u = w[i] ^ 0x80808080u;
            h[2 * i] = __byte_perm(u, 0x64646464u, 0x5140);
            h[2 * i + 1] = __byte_perm(u, 0x64646464u, 0x5342);
            if constexpr (kExactInt8) {
                const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
                __half2 a = __hsub2(*reinterpret_cast<__half2*>(&h[2 * i]), bias);
                __half2 b = __hsub2(*reinterpret_cast<__half2*>(&h[2 * i + 1]), bias);
                h[2 * i] = *reinterpret_cast<uint32_t*>(&a);
                h[2 * i + 1] = *reinterpret_cast<uint32_t*>(&b);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// CUDA-core consumer: one query head per CTA.
// ---------------------------------------------------------------------------
// Ring bytes of the consumer over one-byte codes (a 16-token K+V sub-tile is
// 4 KiB there, half the bf16 one): 48 KiB lets 4 CTAs share an SM (13B on a
// B200: int8 508 -> 494 us, fp8 493 -> 484 us against 64 KiB; 32 KiB 498 / 488).
#ifndef PA_SIMT_CODES_RING_BYTES
#define PA_SIMT_CODES_RING_BYTES 49152
#endif
template <typename T>
constexpr bool is_code_type() {
    return std::is_same<T, E4M3Code>::value || std::is_same<T, Int8Code>::value;
}
template <typename T, int D>
using SimtGeom = Geom<T, D, PA_SIMT_CONSUMER_WARPS,
                      is_code_type<T>() ? PA_SIMT_CODES_RING_BYTES : PA_SIMT_RING_BYTES>;

template <typename T, int D>
__global__ void __launch_bounds__(SimtGeom<T, D>::kThreads)
decode_tma_simt_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const DecodeParams p) {
    using G = SimtGeom<T, D>;
    using TQ = typename QType<T>::type;         // q / out element type
    constexpr int kConsumerWarps = G::kCW;
    constexpr int kThreads = G::kThreads;
    constexpr int VEC = Elem<T>::kVec;          // cache elements per 16-byte chunk
    constexpr int QV = Elem<TQ>::kVec;          // q elements per 16-byte chunk
    constexpr int CPR = D / VEC;                // chunks per row
    constexpr int RPL = 32 / CPR;               // rows per warp-wide pass
    constexpr int ITER = 16 / RPL;              // passes per 16-row sub-tile
    constexpr int IPP = ITER < 8 ? ITER : 8;    // passes held in registers at once
    constexpr bool kFastExp = PA_SIMT_CODES_FAST_EXP && (std::is_same<T, E4M3Code>::value ||
                                                         std::is_same<T, Int8Code>::value);
    constexpr bool kCodes = std::is_same<T, E4M3Code>::value || std::is_same<T, Int8Code>::value;
    constexpr bool kMixed = PA_SIMT_CODES_MIXED_FMA && kCodes;
    constexpr bool kBiased = PA_SIMT_INT8_BIASED && std::is_same<T, Int8Code>::value;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    asm volatile("griddepcontrol.launch_dependents;");

    // grid z = rows of q / out: sequences, or with multi-token queries the query
    // tokens, each of which reads its sequence's blocks up to its causal end
    const int part = blockIdx.x, h = blockIdx.y, row = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int s = row, ctx;
    if (p.query_start == nullptr) {
        ctx = clamp_ctx(__ldg(p.context_lens + s), p.max_context_len, threadIdx.x == 0 && part == 0);
    } else {
        // the sequence holding query token `row`: query_start[s] <= row < query_start[s + 1]
        int lo = 0, hi = p.num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(p.query_start + mid) <= row) lo = mid; else hi = mid - 1;
        }
        s = lo;
        const int q0 = __ldg(p.query_start + s), n_new = __ldg(p.query_start + s + 1) - q0;
        const bool report = threadIdx.x == 0 && part == 0 && h == 0;
        const int lim = clamp_ctx(__ldg(p.context_lens + s), p.max_context_len, report && row == q0) -
                        n_new + (row - q0) + 1;  // causal end of this query token
        if (lim < 1 && report) atomicOr(&s_status_tma, kStatusBadIndex);  // more queries than context
        ctx = lim < 1 ? 0 : lim;
    }
    const int t0 = part * p.partition_size;
    const int t1 = min(ctx, t0 + p.partition_size);
    const int64_t out_row = (int64_t)row * p.num_heads + h;
    const int DQ = kCodes ? p.head_dim : D;  // q / out head_dim (codes: 64 or 128)
    if (t0 >= t1) {
        if (p.num_partitions == 1)
            for (int d = threadIdx.x; d < DQ; d += kThreads) Elem<TQ>::store(p.out, out_row * DQ + d, 0.f);
        return;
    }
    const int kh = h / (p.num_heads / p.num_kv_heads);
    const int n_sub = (t1 - t0 + 15) >> 4;
    Ring ring;
    uint8_t* base = setup_ring<G>(smem_raw, ring);
    if (base == nullptr) {
        if (threadIdx.x == 0) atomicOr(&s_status_tma, kStatusSmemAlign);
        return;
    }
    __syncthreads();

    float m = -INFINITY, l = 0.f;
    float acc[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] = 0.f;

    if (warp == kConsumerWarps) {
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        bool dead = false;
        int issued = 0;
        produce_item<G>(&kmap, &vmap, p, ring, s, kh, t0, n_sub, lane, 0, issued, dead);
        drain_ring<G>(ring, issued, lane);
    } else {
        const int c = lane % CPR, rs = lane / CPR;
        const uint32_t coff = (uint32_t)(c / 8) * kBoxBytes;  // box of this lane's chunk
        const uint32_t cx = (uint32_t)(c % 8);
        float qf[VEC];
        uint32_t qh[VEC / 2];  // mixed-precision path: q as unscaled f16 pairs
        // the K scale of a quantised cache folds into q (exactly 1 otherwise); the
        // mixed-precision path applies it to the dot product instead
        const float qs = p.scale_log2 * (p.k_scale != nullptr ? __ldg(p.k_scale + kh) : 1.f);
#pragma unroll
        for (int u = 0; u < VEC / QV; ++u) {
            float f[QV];
            const int d0 = c * VEC + u * QV;
            Elem<TQ>::widen(d0 < DQ ? ld_v4(static_cast<const TQ*>(p.q) + out_row * DQ + d0)
                                    : make_uint4(0u, 0u, 0u, 0u), f);
#pragma unroll
            for (int j = 0; j < QV; ++j) qf[u * QV + j] = kMixed ? f[j] : f[j] * qs;
        }
        float qsc = qs;  // score scale applied to the dot product
        if constexpr (kMixed) {
            // q to f16 with the power-of-two shift of q_shift_warp (every lane
            // holds a part of this head's q row)
            float am = 0.f;
#pragma unroll
            for (int j = 0; j < VEC; ++j) am = fmaxf(am, fabsf(qf[j]));
            const int sh = q_shift_warp(am);
            const float mul = pow2i(-sh);
            qsc = qs * pow2i(sh);
#pragma unroll
            for (int j = 0; j < VEC; ++j) qf[j] *= mul;
#pragma unroll
            for (int j = 0; j < VEC / 2; ++j) {
                const __half2 h2 = __floats2half2_rn(qf[2 * j], qf[2 * j + 1]);
                qh[j] = *reinterpret_cast<const uint32_t*>(&h2);
                qf[2 * j] = __low2float(h2);  // the values the products use
                qf[2 * j + 1] = __high2float(h2);
            }
        }
        float qsum = 0.f;  // biased int8 widening: what the bias adds to this lane's dot products
        if constexpr (kBiased) {
#pragma unroll
            for (int j = 0; j < VEC; ++j) qsum += qf[j];
        }
        bool dead = false;
        for (int i = warp; i < n_sub && !dead; i += kConsumerWarps) {
            const int st = i % G::kStages;
            const uint32_t round = (uint32_t)(i / G::kStages);
            // warp-uniform outcome: lanes must not split on a wait that ran out
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(ring.full + 8 * st, round & 1u))) {
                if (lane == 0) atomicOr(&s_status_tma, kStatusTimeout);
                dead = true;
                break;
            }
            const bool valid = ring.valid[st] != 0;
            const uint32_t kb = ring.stages + st * G::kStageBytes + coff;
            const uint32_t vb = kb + G::kBoxes * kBoxBytes;
            const int tok0 = t0 + (i << 4);
#pragma unroll
            for (int pass = 0; pass < ITER; pass += IPP) {
                uint4 kr[IPP], vr[IPP];
#pragma unroll
                for (int it = 0; it < IPP; ++it) {
                    const uint32_t row = (uint32_t)((pass + it) * RPL + rs);
                    kr[it] = lds128(kb + swz(row, cx));
                    vr[it] = lds128(vb + swz(row, cx));
                }
                if (pass + IPP >= ITER) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ring.empty + 8 * st);
                }
                if (!valid) continue;
                float sc[IPP];
#pragma unroll
                for (int it = 0; it < IPP; ++it) {
                    float dot = 0.f;
                    if constexpr (kMixed) {
                        uint32_t kh2[VEC / 2];
                        codes_to_f16x2<T, !kBiased>(kr[it], kh2);
                        float d1 = 0.f;
#pragma unroll
                        for (int j = 0; j < VEC / 2; ++j) fma2_f16_f32(qh[j], kh2[j], dot, d1);
                        dot += d1;
                        if constexpr (kBiased) dot = fmaf(-kInt8WidenBias, qsum, dot);
                        dot *= qsc;
                    } else {
                        float kf[VEC];
                        if constexpr (kBiased) int8_widen_biased(kr[it], kf);
                        else Elem<T>::widen(kr[it], kf);
#pragma unroll
                        for (int j = 0; j < VEC; ++j) dot = fmaf(qf[j], kf[j], dot);
                        if constexpr (kBiased) dot = fmaf(-kInt8WidenBias, qsum, dot);
                    }
#pragma unroll
                    for (int off = 1; off < CPR; off <<= 1)
                        dot += __shfl_xor_sync(0xffffffffu, dot, off);
                    const int tok = tok0 + (pass + it) * RPL + rs;
                    sc[it] = tok < t1 ? dot : -INFINITY;
                }
                float mt = sc[0];
#pragma unroll
                for (int it = 1; it < IPP; ++it) mt = fmaxf(mt, sc[it]);
#pragma unroll
                for (int off = CPR; off < 32; off <<= 1)
                    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
                if (mt == -INFINITY) continue;  // only masked rows in this pass
                const float m_new = fmaxf(m, mt);
                if (m_new != m) {  // warp-uniform; a factor of exactly 1 changes no bit
                    const float alpha = kFastExp ? ex2_approx(m - m_new) : exp2f(m - m_new);
                    l *= alpha;
#pragma unroll
                    for (int j = 0; j < VEC; ++j) acc[j] *= alpha;
                }
#pragma unroll
                for (int it = 0; it < IPP; ++it) {
                    const float pr = kFastExp ? ex2_approx(sc[it] - m_new) : exp2f(sc[it] - m_new);
                    const int tok = tok0 + (pass + it) * RPL + rs;
                    if constexpr (kMixed) {
                        const __half ph = __float2half_rn(pr);  // the weight the products use
                        l += __half2float(ph);
                        if (tok < t1) {  // slots past the context may hold anything, even NaN
                            uint32_t vh2[VEC / 2];
                            codes_to_f16x2<T, !kBiased>(vr[it], vh2);
                            const uint32_t pp = (uint32_t)__half_as_ushort(ph);
#pragma unroll
                            for (int j = 0; j < VEC / 2; ++j)
                                fma2_f16s_f32(pp, vh2[j], acc[2 * j], acc[2 * j + 1]);
                        }
                    } else {
                        l += pr;
                        if (tok < t1) {  // slots past the context may hold anything, even NaN
                            float vf[VEC];
                            if constexpr (kBiased) int8_widen_biased(vr[it], vf);
                            else Elem<T>::widen(vr[it], vf);
#pragma unroll
                            for (int j = 0; j < VEC; ++j) acc[j] = fmaf(pr, vf[j], acc[j]);
                        }
                    }
                }
                m = m_new;
            }
        }
        if constexpr (kBiased) {  // the bias's share of the weighted sum: 1152 x the weights
#pragma unroll
            for (int j = 0; j < VEC; ++j) acc[j] = fmaf(-kInt8WidenBias, l, acc[j]);
        }
#pragma unroll
        for (int off = CPR; off < 32; off <<= 1) {
            l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
            for (int j = 0; j < VEC; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
        }
    }
    __syncthreads();  // all loads landed and consumed: the ring is free

    float* sm_o = reinterpret_cast<float*>(base);            // [warps][D]
    float* sm_m = sm_o + kConsumerWarps * D;                 // [warps]
    float* sm_l = sm_m + kConsumerWarps;
    if (warp < kConsumerWarps) {
        const int c = lane % CPR, rs = lane / CPR;
        if (rs == 0) {
#pragma unroll
            for (int j = 0; j < VEC; ++j) sm_o[warp * D + c * VEC + j] = acc[j];
        }
        if (lane == 0) {
            sm_m[warp] = m;
            sm_l[warp] = l;
        }
    }
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w]);
    float wgt[kConsumerWarps];
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
        wgt[w] = sm_m[w] == -INFINITY ? 0.f : exp2f(sm_m[w] - M);
        L = fmaf(sm_l[w], wgt[w], L);
    }
    const float vs = p.v_scale != nullptr ? __ldg(p.v_scale + kh) : 1.f;
    for (int d = threadIdx.x; d < DQ; d += kThreads) {
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) o = fmaf(sm_o[w * D + d], wgt[w], o);
        float val = L > 0.f ? o / L : 0.f;
        if (p.v_scale != nullptr) val *= vs;  // V scale of a quantised cache
        if (p.num_partitions == 1)
            Elem<TQ>::store(p.out, out_row * DQ + d, val);
        else
            p.ws_o[(out_row * p.num_partitions + part) * DQ + d] = val;
    }
    if (p.num_partitions > 1 && threadIdx.x == 0) {
        float* ml = p.ws_ml + (out_row * p.num_partitions + part) * 2;
        ml[0] = L > 0.f ? M : -INFINITY;
        ml[1] = L;
    }
}

// ---------------------------------------------------------------------------
// Tensor-core consumer: the whole query group of one kv head per CTA.
// ---------------------------------------------------------------------------
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Merge buffer of the tensor-core consumer: per warp and query row, the
// running max, sum and head_dim accumulators (rows padded to D + 1 floats so
// the fragment stores hit at most two banks per word).
// ---------------------------------------------------------------------------
// The tensor-core step on one 16-token sub-tile in shared memory (shared by the
// grouped and ungrouped GQA kernels). Thread (r, c) = (lane / 4, lane % 4).
// ---------------------------------------------------------------------------

// S^T[16 tokens][8 heads] = K . Q^T. For chunk step jp (k-steps 2jp, 2jp+1) the
// thread reads 16-byte chunk x = 2c + (jp & 1) of box jp / 2 of rows r and r+8;
// q holds the same head_dim positions of query row r.
template <int D>
__device__ __forceinline__ void mma_qk(uint32_t kb, const uint4 (&q)[D / 32], int r, int c,
                                       float (&sc)[4]) {
    constexpr int KCH = D / 32;
    sc[0] = sc[1] = sc[2] = sc[3] = 0.f;
    uint4 kr[2][KCH];
#pragma unroll
    for (int jp = 0; jp < KCH; ++jp) {
        const uint32_t bx = kb + (jp >> 1) * kBoxBytes;
        const uint32_t x = (uint32_t)(2 * c + (jp & 1));
        kr[0][jp] = lds128(bx + swz(r, x));
        kr[1][jp] = lds128(bx + swz(r + 8, x));
    }
#if PA_MMA_SPLIT_QK
    float sd[4] = {0.f, 0.f, 0.f, 0.f};  // second chain: shorter MMA dependency
#pragma unroll
    for (int jp = 0; jp < KCH; ++jp) {
        mma_16816(sc, kr[0][jp].x, kr[1][jp].x, kr[0][jp].y, kr[1][jp].y, q[jp].x, q[jp].y);
        mma_16816(sd, kr[0][jp].z, kr[1][jp].z, kr[0][jp].w, kr[1][jp].w, q[jp].z, q[jp].w);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[e] += sd[e];
#else
#pragma unroll
    for (int jp = 0; jp < KCH; ++jp) {
        mma_16816(sc, kr[0][jp].x, kr[1][jp].x, kr[0][jp].y, kr[1][jp].y, q[jp].x, q[jp].y);
        mma_16816(sc, kr[0][jp].z, kr[1][jp].z, kr[0][jp].w, kr[1][jp].w, q[jp].z, q[jp].w);
    }
#endif
}

// V fragments: tokens 2c, 2c+1, 2c+8, 2c+9; 16-byte chunk r of each box.
template <int D>
__device__ __forceinline__ void mma_load_v(uint32_t vb, int r, int c, uint4 (&vr)[4][D / 64]) {
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
        const uint32_t bx = vb + hh * kBoxBytes;
        vr[0][hh] = lds128(bx + swz(2 * c, r));
        vr[1][hh] = lds128(bx + swz(2 * c + 1, r));
        vr[2][hh] = lds128(bx + swz(2 * c + 8, r));
        vr[3][hh] = lds128(bx + swz(2 * c + 9, r));
    }
}

// Online-softmax update with the sub-tile's scores and O^T += V^T . P^T.
// nvalid = tokens of the sub-tile inside the context (>= 1). State: acc = O^T
// fragments (rows head_dim 64*(t/4) + 8r + 2*(t%4) (+1), cols heads 2c, 2c+1),
// m0/m1 running max (log2 units), l0/l1 this thread's share of the sums.
template <int D>
__device__ __forceinline__ void mma_softmax_pv(const float (&sc)[4], uint4 (&vr)[4][D / 64],
                                               int nvalid, float scale_log2, int r, int c,
                                               float (&acc)[D / 16][4], float& m0, float& m1,
                                               float& l0, float& l1) {
    constexpr int VCH = D / 64;
    constexpr int MT = D / 16;
    const bool lo_ok = r < nvalid, hi_ok = r + 8 < nvalid;
    const float s0 = lo_ok ? sc[0] * scale_log2 : -INFINITY;  // token r,   head 2c
    const float s1 = lo_ok ? sc[1] * scale_log2 : -INFINITY;  // token r,   head 2c+1
    const float s2 = hi_ok ? sc[2] * scale_log2 : -INFINITY;  // token r+8, head 2c
    const float s3 = hi_ok ? sc[3] * scale_log2 : -INFINITY;  // token r+8, head 2c+1
    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    // The accumulator is rescaled only when some running max moved; a factor of
    // exactly 1 would leave every bit unchanged anyway.
    const bool moved = __any_sync(0xffffffffu, mn0 != m0 || mn1 != m1);
    const float al0 = moved ? exp2f(m0 - mn0) : 1.f;
    const float al1 = moved ? exp2f(m1 - mn1) : 1.f;
    const uint32_t x0 = pack_bf16x2(exp2f(s0 - mn0), exp2f(s1 - mn1));
    const uint32_t x1 = pack_bf16x2(exp2f(s2 - mn0), exp2f(s3 - mn1));
    // the sums use the same rounded weights the PV product sees
    l0 = fmaf(l0, al0, bf16_lo(x0) + bf16_lo(x1));
    l1 = fmaf(l1, al1, bf16_hi(x0) + bf16_hi(x1));
    m0 = mn0;
    m1 = mn1;
    if (moved) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            acc[t][0] *= al0;
            acc[t][1] *= al1;
            acc[t][2] *= al0;
            acc[t][3] *= al1;
        }
    }
    const uint32_t pb0 = movmatrix_trans(x0);  // P^T rows (tokens) 2c, 2c+1; col head r
    const uint32_t pb1 = movmatrix_trans(x1);  // tokens 2c+8, 2c+9
    if (nvalid < 16) {  // slots past the context may hold anything, even NaN
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        const int tv0 = 2 * c, tv1 = 2 * c + 1, tv2 = 2 * c + 8, tv3 = 2 * c + 9;
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

// ---------------------------------------------------------------------------
// The tensor-core step over quantised codes (FP8 E4M3 / int8, head_dim 128):
// codes become f16 exactly (every E4M3 value and every integer up to 2048 is
// an f16), q becomes f16 exactly within f16 range, and the MMAs run in f16
// with fp32 accumulation. K fragments: thread (r, c) reads 16-byte chunks
// 2c, 2c+1 of rows r, r+8; k-step ks takes word ks & 3 of chunk 2c + ks / 4,
// so its head_dim positions are 32c + 4 ks + {0,1} (A cols 2c, 2c+1) and
// + {2,3} (cols 2c+8, 2c+9); q uses the same positions. V fragments: chunk r
// of tokens 2c, 2c+1, 2c+8, 2c+9; m-tile t rows r / r+8 are head_dim
// 16 r + 2t / + 1.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float f16_lo(uint32_t w) {
    return __low2float(*reinterpret_cast<const __half2*>(&w));
}
__device__ __forceinline__ float f16_hi(uint32_t w) {
    return __high2float(*reinterpret_cast<const __half2*>(&w));
}

// Word t = [x0, y0, x1, y1] (bytes, low first) of codes -> f16x2 (x0, y0) and
// (x1, y1). Int8 words arrive with their sign bits flipped (byte = code + 128):
// 0x64uu as an f16 is 1024 + u, and subtracting 1152 leaves the code.
template <typename TC>
__device__ __forceinline__ void code_pairs_f16(uint32_t t, uint32_t& p0, uint32_t& p1) {
    if constexpr (std::is_same<TC, E4M3Code>::value) {
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
            "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
            : "=r"(p0), "=r"(p1) : "r"(t));
    } else {
        // int8 (bytes already offset by 128 in code_word): 1024 + byte = code + 1152,
        // exact in f16; the consumers take the 1152 out once per sum (kInt8Bias)
        p0 = __byte_perm(t, 0x64646464u, 0x5140);
        p1 = __byte_perm(t, 0x64646464u, 0x7362);
    }
}

// The offset the tensor-core consumers' int8 operands carry (code + 1152): a
// score over such a K row exceeds the true one by 1152 x the sum of q, an
// output over such V rows by 1152 (times the V scale) once normalised.
constexpr float kInt8Bias = 1152.f;

// 1152 x the sum of q over head_dim for query rows 2c and 2c + 1 (b0, b1), from
// the f16 q fragments thread (r, c) holds for row r (code consumers' B operand):
// a fixed-order sum over the thread's 32 elements, then over the four threads of
// the row.
__device__ __forceinline__ void int8_qk_bias(const uint4 (&q)[4], int c, float& b0, float& b1) {
    float sum = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) sum += f16_lo(w[i]) + f16_hi(w[i]);
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    b0 = kInt8Bias * __shfl_sync(0xffffffffu, sum, 4 * (2 * c));
    b1 = kInt8Bias * __shfl_sync(0xffffffffu, sum, 4 * (2 * c + 1));
}

template <typename TC>
__device__ __forceinline__ uint32_t code_word(uint32_t w) {
    return std::is_same<TC, Int8Code>::value ? w ^ 0x80808080u : w;
}

// q row of the B operand for codes: head_dim 32c .. 32c+31 as raw bf16 words
// (zeros without a row), their largest magnitude, and their conversion to 16
// f16x2 words of q * mul (mul a signed power of two: exact).
// (head_dim positions at or past dq, the padding of a head_dim 64 pool, are zero).
__device__ __forceinline__ void load_q_raw(const uint16_t* qrow, int c, uint4 (&raw)[4], int dq) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
        raw[u] = qrow != nullptr && 32 * c + 8 * u < dq ? ld_v4(qrow + 32 * c + 8 * u)
                                                        : make_uint4(0u, 0u, 0u, 0u);
}
__device__ __forceinline__ float q_raw_amax(const uint4 (&raw)[4]) {
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, max((w[i] << 16) & 0x7fffffffu, w[i] & 0x7fff0000u));
    }
    return __uint_as_float(m);
}
__device__ __forceinline__ void q_raw_to_f16(const uint4 (&raw)[4], float mul, uint4 (&q)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
        q[u] = make_uint4(pack_f16x2(bf16_lo(raw[u].x) * mul, bf16_hi(raw[u].x) * mul),
                          pack_f16x2(bf16_lo(raw[u].y) * mul, bf16_hi(raw[u].y) * mul),
                          pack_f16x2(bf16_lo(raw[u].z) * mul, bf16_hi(raw[u].z) * mul),
                          pack_f16x2(bf16_lo(raw[u].w) * mul, bf16_hi(raw[u].w) * mul));
}

template <typename TC>
__device__ __forceinline__ void codes_qk(uint32_t kb, const uint4 (&q)[4], int r, int c,
                                         float (&sc)[4]) {
    uint4 kr[2][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        kr[0][h] = lds128(kb + swz(r, 2 * c + h));
        kr[1][h] = lds128(kb + swz(r + 8, 2 * c + h));
    }
    float sd[4] = {0.f, 0.f, 0.f, 0.f};
    sc[0] = sc[1] = sc[2] = sc[3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        const uint32_t wa = code_word<TC>(word(kr[0][ks >> 2], ks & 3));
        const uint32_t wb = code_word<TC>(word(kr[1][ks >> 2], ks & 3));
        uint32_t a0, a1, a2, a3;
        code_pairs_f16<TC>(wa, a0, a2);
        code_pairs_f16<TC>(wb, a1, a3);
        const uint32_t b0 = word(q[ks >> 1], 2 * (ks & 1)), b1 = word(q[ks >> 1], 2 * (ks & 1) + 1);
        if (ks & 1)
            mma_16816_f16(sd, a0, a1, a2, a3, b0, b1);
        else
            mma_16816_f16(sc, a0, a1, a2, a3, b0, b1);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[e] += sd[e];
}

__device__ __forceinline__ void codes_load_v(uint32_t vb, int r, int c, uint4 (&vr)[4]) {
    vr[0] = lds128(vb + swz(2 * c, r));
    vr[1] = lds128(vb + swz(2 * c + 1, r));
    vr[2] = lds128(vb + swz(2 * c + 8, r));
    vr[3] = lds128(vb + swz(2 * c + 9, r));
}

// As mma_softmax_pv, over codes: scores scaled by scale_log2 x k_scale (sl),
// weights packed as f16, V^T fragments built from the code chunks.
template <typename TC>
__device__ __forceinline__ void codes_softmax_pv(const float (&sc)[4], uint4 (&vr)[4], int nvalid,
                                                 float sl, int r, int c, float (&acc)[8][4],
                                                 float& m0, float& m1, float& l0, float& l1) {
    const bool lo_ok = r < nvalid, hi_ok = r + 8 < nvalid;
    const float s0 = lo_ok ? sc[0] * sl : -INFINITY;
    const float s1 = lo_ok ? sc[1] * sl : -INFINITY;
    const float s2 = hi_ok ? sc[2] * sl : -INFINITY;
    const float s3 = hi_ok ? sc[3] * sl : -INFINITY;
    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const bool moved = __any_sync(0xffffffffu, mn0 != m0 || mn1 != m1);
    const float al0 = moved ? exp2f(m0 - mn0) : 1.f;
    const float al1 = moved ? exp2f(m1 - mn1) : 1.f;
    const uint32_t x0 = pack_f16x2(exp2f(s0 - mn0), exp2f(s1 - mn1));
    const uint32_t x1 = pack_f16x2(exp2f(s2 - mn0), exp2f(s3 - mn1));
    l0 = fmaf(l0, al0, f16_lo(x0) + f16_lo(x1));
    l1 = fmaf(l1, al1, f16_hi(x0) + f16_hi(x1));
    m0 = mn0;
    m1 = mn1;
    if (moved) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            acc[t][0] *= al0;
            acc[t][1] *= al1;
            acc[t][2] *= al0;
            acc[t][3] *= al1;
        }
    }
    const uint32_t pb0 = movmatrix_trans(x0);
    const uint32_t pb1 = movmatrix_trans(x1);
    if (nvalid < 16) {  // a zero code is the value 0 in both formats
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        if (2 * c >= nvalid) vr[0] = z;
        if (2 * c + 1 >= nvalid) vr[1] = z;
        if (2 * c + 8 >= nvalid) vr[2] = z;
        if (2 * c + 9 >= nvalid) vr[3] = z;
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t va = code_word<TC>(word(vr[0], w)), vb = code_word<TC>(word(vr[1], w));
        const uint32_t vc = code_word<TC>(word(vr[2], w)), vd = code_word<TC>(word(vr[3], w));
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // m-tile t = 2w + h: bytes 2h, 2h+1 of word w
            const uint32_t sel = h ? 0x7362u : 0x5140u;
            uint32_t a0, a1, a2, a3;
            code_pairs_f16<TC>(__byte_perm(va, vb, sel), a0, a1);
            code_pairs_f16<TC>(__byte_perm(vc, vd, sel), a2, a3);
            mma_16816_f16(acc[2 * w + h], a0, a1, a2, a3, pb0, pb1);
        }
    }
}

// Store one warp's item result (heads 2c, 2c+1 of query rows head0 + n) from its
// registers: bf16 output when P == 1, else the normalised partial and (m, l).
// kCodes: the m-tile rows of the code consumer (head_dim 16 r + 2t, + 1) and
// the V scale `vs` of a quantised cache.
template <int D, bool kCodes = false>
__device__ __forceinline__ void mma_store_item(const DecodeParams& p, int64_t head0, int group,
                                               int part, int r, int c, const float (&acc)[D / 16][4],
                                               float m0, float m1, float l0, float l1,
                                               float vs = 1.f, float obias = 0.f) {
    constexpr int MT = D / 16;
    const int P = p.num_partitions;
    const int DQ = kCodes ? p.head_dim : D;  // out / workspace row length
    float inv0 = l0 > 0.f ? 1.f / l0 : 0.f;
    float inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
    if constexpr (kCodes) {
        inv0 *= vs;
        inv1 *= vs;
    }
    // int8 codes: the accumulator carries 1152 x the weights (obias = 1152 x the
    // V scale), taken out after the normalisation
    const float ob0 = l0 > 0.f ? obias : 0.f, ob1 = l1 > 0.f ? obias : 0.f;
    auto nv = [&](float a, float inv, float ob) { return obias != 0.f ? fmaf(a, inv, -ob) : a * inv; };
    const int n0 = 2 * c, n1 = 2 * c + 1;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        const int d0 = kCodes ? 16 * r + 2 * t : (t >> 2) * 64 + r * 8 + 2 * (t & 3);
        if (d0 >= DQ) continue;  // padding of a head_dim 64 pool of codes
        if (P == 1) {
            if (n0 < group)
                *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.out) + (head0 + n0) * DQ + d0) =
                    pack_bf16x2(nv(acc[t][0], inv0, ob0), nv(acc[t][2], inv0, ob0));
            if (n1 < group)
                *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.out) + (head0 + n1) * DQ + d0) =
                    pack_bf16x2(nv(acc[t][1], inv1, ob1), nv(acc[t][3], inv1, ob1));
        } else {
            if (n0 < group)
                *reinterpret_cast<float2*>(p.ws_o + ((head0 + n0) * P + part) * DQ + d0) =
                    make_float2(nv(acc[t][0], inv0, ob0), nv(acc[t][2], inv0, ob0));
            if (n1 < group)
                *reinterpret_cast<float2*>(p.ws_o + ((head0 + n1) * P + part) * DQ + d0) =
                    make_float2(nv(acc[t][1], inv1, ob1), nv(acc[t][3], inv1, ob1));
        }
    }
    if (P > 1 && r == 0) {
        if (n0 < group) {
            float* ml = p.ws_ml + ((head0 + n0) * P + part) * 2;
            ml[0] = l0 > 0.f ? m0 : -INFINITY;
            ml[1] = l0;
        }
        if (n1 < group) {
            float* ml = p.ws_ml + ((head0 + n1) * P + part) * 2;
            ml[0] = l1 > 0.f ? m1 : -INFINITY;
            ml[1] = l1;
        }
    }
}

template <int D, typename TC = __nv_bfloat16>
using MmaGeom = Geom<TC, D, PA_MMA_CONSUMER_WARPS, PA_MMA_RING_BYTES>;

template <int D>
constexpr int merge_floats() {
    // o[warps][8][D + 1], m[warps][8], l[warps][8], w[warps][8] (normalised weights)
    return PA_MMA_CONSUMER_WARPS * kGroupMax * (D + 1) + 3 * PA_MMA_CONSUMER_WARPS * kGroupMax;
}
template <int D>
constexpr int merge_bytes() {
    // one warp: none; two warps: warp 1's registers, in register order, for warp 0
    // ((D/16 * 4 accumulators + m0, m1, l0, l1) x 32 lanes); more warps: a
    // double-buffered [warps][8][D + 1] buffer (item k uses buffer k % 2)
    return PA_MMA_CONSUMER_WARPS == 1   ? 0
           : PA_MMA_CONSUMER_WARPS == 2 ? (D / 16 * 4 + 4) * 32 * 4
                                        : 2 * merge_floats<D>() * 4;
}

// The work items of one persistent CTA, in order: u = blockIdx.x + k * gridDim.x,
// item u = (partition u % P, kv head, sequence). Every warp walks them itself;
// the context lengths of 32 upcoming items are held one per lane, so a warp
// pays one load latency per 32 items, not per item.
struct ItemWalk {
    int k;        // ordinal of the current item within this CTA
    int kbase;    // ordinal of the item whose context length lane 0 holds
    int ctx_lane; // context length of item kbase + lane (clamped), -1 past the end
};

struct Item {
    bool valid;   // false: no items left
    int s, kh, part, t0, t1;
};

__device__ __forceinline__ int item_ctx_load(const DecodeParams& p, int num_items, int kbase,
                                             int lane, bool report) {
    const int u = blockIdx.x + (kbase + lane) * gridDim.x;
    if (u >= num_items) return -1;
    const int s = (u / p.num_partitions) / p.num_kv_heads;
    const int part = u % p.num_partitions;
    return clamp_ctx(__ldg(p.context_lens + s), p.max_context_len, report && part == 0);
}

// Next non-empty item (t0 < t1) or !valid. Items that are empty are returned
// too when `want_empty` (consumers write zeros for them when P == 1).
__device__ __forceinline__ Item item_next(ItemWalk& w, const DecodeParams& p, int num_items,
                                          int lane, bool report, bool want_empty) {
    for (;;) {
        const int u = blockIdx.x + w.k * gridDim.x;
        Item it;
        it.valid = u < num_items;
        if (!it.valid) return it;
        if (w.k - w.kbase >= 32) {
            w.kbase = w.k;
            w.ctx_lane = item_ctx_load(p, num_items, w.kbase, lane, report);
        }
        const int ctx = __shfl_sync(0xffffffffu, w.ctx_lane, w.k - w.kbase);
        it.part = u % p.num_partitions;
        const int rest = u / p.num_partitions;
        it.kh = rest % p.num_kv_heads;
        it.s = rest / p.num_kv_heads;
        it.t0 = it.part * p.partition_size;
        it.t1 = min(ctx, it.t0 + p.partition_size);
        ++w.k;
        if (it.t0 < it.t1 || want_empty) return it;
    }
}

// Dynamic schedule of a persistent CTA: the producer claims work items from
// the launch's counter in order (so CTAs that stream faster take more items,
// and every CTA ends within about one item of the others) and hands them to
// the consumer warps through kItemQ slots with a full / empty mbarrier pair
// each. The producer keeps one claimed item ahead of the one it issues, so an
// item is in the queue before any of the previous item's loads wait for ring
// space: the consumers, which take the next item when they start one (to
// fetch its q early), never wait for an item the producer cannot yet claim.
// Slot value -1 ends the stream. Empty items (a partition past the context)
// are skipped by the producer, except with one partition, where their heads
// get a zero output from the consumers.
constexpr int kItemQ = 4;
constexpr int kItemQBytes = 2 * kItemQ * 8 + 2 * kItemQ * 4;

struct ItemQueue {
    uint32_t full, empty;  // shared addresses of the barriers, slot i at + 8 i
    int* u;                // [kItemQ] item index, -1: no more items
    int* t1;               // [kItemQ] end of the item's tokens
};

__device__ __forceinline__ ItemQueue item_queue_setup(uint8_t* at, int consumers) {
    ItemQueue q;
    q.full = smem_u32(at);
    q.empty = q.full + 8 * kItemQ;
    q.u = reinterpret_cast<int*>(at + 16 * kItemQ);
    q.t1 = q.u + kItemQ;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kItemQ; ++i) {
            mbar_init(q.full + 8 * i, 1);
            mbar_init(q.empty + 8 * i, consumers);
        }
        fence_barrier_init();
    }
    return q;
}

__device__ __forceinline__ Item item_of(const DecodeParams& p, int u, int t1) {
    Item it;
    it.valid = u >= 0;
    it.part = it.valid ? u % p.num_partitions : 0;
    const int rest = it.valid ? u / p.num_partitions : 0;
    it.kh = rest % p.num_kv_heads;
    it.s = rest / p.num_kv_heads;
    it.t0 = it.part * p.partition_size;
    it.t1 = t1;
    return it;
}

// Producer side, whole warp: finish a claim whose counter value lane 0 holds
// in `ticket` (claiming again past empty items). Lane 0 reports context
// lengths out of range, once per sequence (its first partition).
__device__ __forceinline__ Item item_claim_finish(const DecodeParams& p, int num_items,
                                                  unsigned ticket, int lane) {
    for (;;) {
        const unsigned u = __shfl_sync(0xffffffffu, ticket, 0);
        if (u >= (unsigned)num_items) {
            Item none;
            none.valid = false;
            return none;
        }
        Item it = item_of(p, (int)u, 0);
        int ctx = 0;
        if (lane == 0)
            ctx = clamp_ctx(__ldg(p.context_lens + it.s), p.max_context_len, it.part == 0);
        ctx = __shfl_sync(0xffffffffu, ctx, 0);
        it.t1 = min(ctx, it.t0 + p.partition_size);
        if (it.t0 < it.t1 || p.num_partitions == 1) return it;
        if (lane == 0) ticket = atomicAdd(p.sched, 1u);
    }
}

// Producer: put the k-th item (or the end of the stream) in its slot. False if
// the wait for the slot ran out.
__device__ __forceinline__ bool item_push(const DecodeParams& p, const ItemQueue& q, int k,
                                          const Item& it, int lane) {
    const int slot = k % kItemQ;
    const uint32_t round = (uint32_t)(k / kItemQ);
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(q.empty + 8 * slot, (round & 1u) ^ 1u))) {
        if (lane == 0) atomicOr(&s_status_tma, kStatusTimeout);
        return false;
    }
    if (lane == 0) {
        q.u[slot] = it.valid ? it.part + p.num_partitions * (it.kh + p.num_kv_heads * it.s) : -1;
        q.t1[slot] = it.valid ? it.t1 : 0;
        mbar_arrive(q.full + 8 * slot);  // release: the slot's words are visible to its readers
    }
    __syncwarp();
    return true;
}

// Consumer warp: take the k-th item (the end of the stream if `dead` or the
// wait ran out, which also sets `dead`).
__device__ __forceinline__ Item item_pop(const DecodeParams& p, const ItemQueue& q, int k,
                                         int lane, bool& dead) {
    Item it;
    it.valid = false;
    if (dead) return it;
    const int slot = k % kItemQ;
    const uint32_t round = (uint32_t)(k / kItemQ);
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(q.full + 8 * slot, round & 1u))) {
        if (lane == 0) atomicOr(&s_status_tma, kStatusTimeout);
        dead = true;
        return it;
    }
    const int u = q.u[slot], t1 = q.t1[slot];
    __syncwarp();
    if (lane == 0) mbar_arrive(q.empty + 8 * slot);
    return item_of(p, u, t1);
}

// AND of `pred` over the first `threads` threads of the CTA (named barrier 2).
__device__ __forceinline__ bool consumers_all(bool pred, int threads) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n"
                 " bar.red.and.pred p, 2, %2, q;\n selp.u32 %0, 1, 0, p;\n}"
                 : "=r"(r) : "r"((uint32_t)pred), "r"(threads) : "memory");
    return r != 0;
}

// Persistent: each CTA walks its work items. The producer streams the items'
// sub-tiles through the ring without a break between items (block-table
// entries fetched one 32-sub-tile batch ahead), while the consumers finish one
// item (cross-warp merge, store) and start the next (q fragments fetched one
// item ahead).
template <int D, typename TC = __nv_bfloat16>
__global__ void __launch_bounds__(MmaGeom<D, TC>::kThreads, PA_MMA_MIN_BLOCKS)
decode_tma_mma_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const DecodeParams p,
                      int num_items) {
    using T = __nv_bfloat16;
    using G = MmaGeom<D, TC>;
    constexpr bool kCodes = !std::is_same<TC, __nv_bfloat16>::value;
    static_assert(!kCodes || D == 128, "quantised codes: head_dim 128");
    static_assert(!kCodes || G::kCW <= 2, "the code consumer's head_dim order needs the register merge");
    constexpr int kConsumerWarps = G::kCW;
    constexpr int KCH = D / 32;  // 16-byte K chunks per row per thread (2 k-steps each)
    constexpr int VCH = D / 64;  // V boxes
    constexpr int MT = D / 16;   // PV m-tiles
    constexpr int OS = D + 1;    // merge-buffer row stride (floats)
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    asm volatile("griddepcontrol.launch_dependents;");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.num_partitions;
    const int group = p.num_heads / p.num_kv_heads;
    Ring ring;
    uint8_t* base = setup_ring<G>(smem_raw, ring, merge_bytes<D>() + kItemQBytes);
    if (base == nullptr) {
        if (threadIdx.x == 0) atomicOr(&s_status_tma, kStatusSmemAlign);
        return;
    }
    float* merge_buf = reinterpret_cast<float*>(base + G::kRingBytes);
    int merge_sel = 0;  // which half of the double-buffered merge area this item uses
    const bool dyn = p.sched != nullptr;  // dynamic schedule (else item u to CTA u mod grid)
    const ItemQueue iq = item_queue_setup(base + G::kRingBytes + merge_bytes<D>(), kConsumerWarps);
    ItemWalk walk;
    walk.k = 0;
    walk.kbase = 0;
    walk.ctx_lane = dyn ? -1 : item_ctx_load(p, num_items, 0, lane, warp == 0);
    __syncthreads();

    if (warp == kConsumerWarps) {  // producer
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        bool dead = false;
        int g = 0, issued = 0, kq = 0;
        // Batches of up to 32 sub-tiles, the next batch's table entries in flight.
        // Dynamic schedule: an item is claimed (and queued for the consumers) once
        // every sub-tile of the previous one is issued, so a CTA holds at most the
        // ring's worth of work ahead of its consumers when the items run out.
        auto claim = [&]() -> Item {
            unsigned ticket = 0;
            if (lane == 0) ticket = atomicAdd(p.sched, 1u);
            const Item it = item_claim_finish(p, num_items, ticket, lane);
            if (!item_push(p, iq, kq++, it, lane)) dead = true;
            return it;
        };
        Item cur = dyn ? claim() : item_next(walk, p, num_items, lane, false, false);
        int cur_base = 0;
        int phys_cur = -1;
        if (cur.valid && lane < ((cur.t1 - cur.t0 + 15) >> 4))
            phys_cur = __ldg(p.block_tables + (int64_t)cur.s * p.table_stride +
                             ((cur.t0 + (lane << 4)) >> p.log2_block_size));
        while (cur.valid && !dead) {
            const int n_sub = (cur.t1 - cur.t0 + 15) >> 4;
            const bool last = cur_base + 32 >= n_sub;
            Item nxt = cur;
            int nxt_base = cur_base + 32;
            if (last) {
                if (!dyn) nxt = item_next(walk, p, num_items, lane, false, false);
                nxt_base = 0;
            }
            int phys_nxt = -1;
            if (!(dyn && last) && nxt.valid && nxt_base + lane < ((nxt.t1 - nxt.t0 + 15) >> 4))
                phys_nxt = __ldg(p.block_tables + (int64_t)nxt.s * p.table_stride +
                                 ((nxt.t0 + ((nxt_base + lane) << 4)) >> p.log2_block_size));
            const int cnt = min(32, n_sub - cur_base);
            issue_batch<G>(&kmap, &vmap, p, ring, g, cnt, phys_cur, cur.kh,
                              cur.t0 + ((cur_base + lane) << 4), lane, issued, dead);
            g += cnt;
            if (dyn && last && !dead) {
                nxt = claim();
                if (nxt.valid && lane < ((nxt.t1 - nxt.t0 + 15) >> 4))
                    phys_nxt = __ldg(p.block_tables + (int64_t)nxt.s * p.table_stride +
                                     ((nxt.t0 + (lane << 4)) >> p.log2_block_size));
            }
            cur = nxt;
            cur_base = nxt_base;
            phys_cur = phys_nxt;
        }
        drain_ring<G>(ring, issued, lane);
        return;
    }

    // consumers (threads 0 .. 127)
    const int r = lane >> 2, c = lane & 3;
    bool dead = false;
    int g = 0;
    // Q^T (B operand of QK): thread (r, c) holds query row r. For chunk step jp
    // (k-steps 2jp, 2jp+1) it reads 16-byte chunk x = 2c + (jp & 1) of box jp / 2,
    // the same head_dim positions its K fragments come from.
    // Over codes q stays raw bf16 here; it becomes f16 with its power-of-two
    // shift when the item starts (q_shift_warp).
    auto load_q = [&](const Item& it, uint4 (&q)[KCH]) {
        const int64_t head0 = (int64_t)it.s * p.num_heads + (int64_t)it.kh * group;
        if (it.valid && it.t0 < it.t1 && r < group) {
            if constexpr (kCodes) {
                load_q_raw(static_cast<const uint16_t*>(p.q) + (head0 + r) * p.head_dim, c, q,
                           p.head_dim);
            } else {
                const uint16_t* qrow = static_cast<const uint16_t*>(p.q) + (head0 + r) * D;
#pragma unroll
                for (int jp = 0; jp < KCH; ++jp)
                    q[jp] = ld_v4(qrow + (jp >> 1) * 64 + (2 * c + (jp & 1)) * 8);
            }
        } else {
#pragma unroll
            for (int jp = 0; jp < KCH; ++jp) q[jp] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    // Dynamic schedule: the k-th queued item; the consumer warps take an item
    // only if every one of them got it (a wait that ran out in one warp ends
    // the stream for all, so they never split on the merge barriers).
    int kq = 0;
    auto next_item = [&]() -> Item {
        if (!dyn) return item_next(walk, p, num_items, lane, warp == 0, true);
        Item it = item_pop(p, iq, kq++, lane, dead);
        if constexpr (kConsumerWarps > 1) {
            if (!consumers_all(it.valid, kConsumerWarps * 32)) it.valid = false;
        }
        return it;
    };
    Item cur = next_item();
    uint4 qcur[KCH];
    load_q(cur, qcur);
    while (cur.valid) {
        Item nxt;
        uint4 qnxt[KCH];
        if (!dyn) {
            // static schedule: the next item is known, its q in flight meanwhile
            nxt = next_item();
            load_q(nxt, qnxt);
        }
        int qsh = 0;  // over codes: this item's q to f16, scaled by 2^-qsh
        float qb0 = 0.f, qb1 = 0.f;  // int8: 1152 x sum of q of query rows 2c, 2c + 1
        if constexpr (kCodes) {
            qsh = q_shift_warp(q_raw_amax(qcur));
            q_raw_to_f16(qcur, pow2i(-qsh), qcur);
            if constexpr (std::is_same<TC, Int8Code>::value) int8_qk_bias(qcur, c, qb0, qb1);
        }
        const int64_t head0 = (int64_t)cur.s * p.num_heads + (int64_t)cur.kh * group;
        if (cur.t0 >= cur.t1) {
            const int DQ = kCodes ? p.head_dim : D;
            if (P == 1)
                for (int idx = threadIdx.x; idx < group * DQ; idx += kConsumerWarps * 32)
                    Elem<T>::store(p.out, head0 * DQ + idx, 0.f);
            if (dyn) {
                nxt = next_item();
                load_q(nxt, qnxt);
            }
        } else {
            const int t0 = cur.t0, t1 = cur.t1;
            const int n_sub = (t1 - t0 + 15) >> 4;
            // score scale (the K scale of a quantised cache and q's shift fold in)
            const float sl =
                kCodes ? p.scale_log2 * __ldg(p.k_scale + cur.kh) * pow2i(qsh) : p.scale_log2;
            float acc[MT][4];
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
            float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

            for (int i = warp; i < n_sub && !dead; i += kConsumerWarps) {
                const int gi = g + i;
                const int st = gi % G::kStages;
                const uint32_t round = (uint32_t)(gi / G::kStages);
                // warp-uniform outcome: lanes must not split on a wait that ran out
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(ring.full + 8 * st, round & 1u))) {
                    if (lane == 0) atomicOr(&s_status_tma, kStatusTimeout);
                    dead = true;
                    break;
                }
                const bool valid = ring.valid[st] != 0;
                const uint32_t kb = ring.stages + st * G::kStageBytes;
                const uint32_t vb = kb + G::kBoxes * kBoxBytes;
                float sc[4];
                if constexpr (kCodes) {
                    codes_qk<TC>(kb, qcur, r, c, sc);
                    if constexpr (std::is_same<TC, Int8Code>::value) {
                        sc[0] -= qb0;
                        sc[1] -= qb1;
                        sc[2] -= qb0;
                        sc[3] -= qb1;
                    }
                    uint4 vr[4];
                    codes_load_v(vb, r, c, vr);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ring.empty + 8 * st);  // stage released
                    if (!valid) continue;
                    codes_softmax_pv<TC>(sc, vr, t1 - (t0 + (i << 4)), sl, r, c, acc, m0, m1, l0, l1);
                } else {
                    mma_qk<D>(kb, qcur, r, c, sc);
                    uint4 vr[4][VCH];
                    mma_load_v<D>(vb, r, c, vr);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ring.empty + 8 * st);  // stage released
                    if (!valid) continue;
                    mma_softmax_pv<D>(sc, vr, t1 - (t0 + (i << 4)), sl, r, c, acc, m0, m1, l0, l1);
                }
            }
            g += n_sub;
            if (dyn) {
                // the next item is queued by now (its loads follow this item's);
                // its q is in flight during this item's merge and store
                nxt = next_item();
                load_q(nxt, qnxt);
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, off);
                l1 += __shfl_xor_sync(0xffffffffu, l1, off);
            }
            if constexpr (kConsumerWarps == 2) {
                // Warp 1 hands its state to warp 0 in register order (conflict-free);
                // warp 0 merges it into its own registers, in fixed order.
                float* xb = merge_buf;
                if (warp == 1) {
#pragma unroll
                    for (int t = 0; t < MT; ++t)
#pragma unroll
                        for (int e = 0; e < 4; ++e) xb[(t * 4 + e) * 32 + lane] = acc[t][e];
                    xb[(MT * 4 + 0) * 32 + lane] = m0;
                    xb[(MT * 4 + 1) * 32 + lane] = m1;
                    xb[(MT * 4 + 2) * 32 + lane] = l0;
                    xb[(MT * 4 + 3) * 32 + lane] = l1;
                }
                named_barrier(1, 64);
                if (warp == 0) {
                    const float mb0 = xb[(MT * 4 + 0) * 32 + lane], mb1 = xb[(MT * 4 + 1) * 32 + lane];
                    const float lb0 = xb[(MT * 4 + 2) * 32 + lane], lb1 = xb[(MT * 4 + 3) * 32 + lane];
                    const float M0 = fmaxf(m0, mb0), M1 = fmaxf(m1, mb1);
                    const float wa0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M0);
                    const float wb0 = mb0 == -INFINITY ? 0.f : exp2f(mb0 - M0);
                    const float wa1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M1);
                    const float wb1 = mb1 == -INFINITY ? 0.f : exp2f(mb1 - M1);
#pragma unroll
                    for (int t = 0; t < MT; ++t) {
                        acc[t][0] = fmaf(xb[(t * 4 + 0) * 32 + lane], wb0, acc[t][0] * wa0);
                        acc[t][1] = fmaf(xb[(t * 4 + 1) * 32 + lane], wb1, acc[t][1] * wa1);
                        acc[t][2] = fmaf(xb[(t * 4 + 2) * 32 + lane], wb0, acc[t][2] * wa0);
                        acc[t][3] = fmaf(xb[(t * 4 + 3) * 32 + lane], wb1, acc[t][3] * wa1);
                    }
                    l0 = fmaf(lb0, wb0, l0 * wa0);
                    l1 = fmaf(lb1, wb1, l1 * wa1);
                    m0 = M0;
                    m1 = M1;
                }
            }
            if constexpr (kConsumerWarps <= 2) {
                // One warp holds the whole item: normalise and store from registers.
                if (warp == 0)
                    mma_store_item<D, kCodes>(p, head0, group, cur.part, r, c, acc, m0, m1, l0, l1,
                                              kCodes ? __ldg(p.v_scale + cur.kh) : 1.f,
                                              std::is_same<TC, Int8Code>::value
                                                  ? kInt8Bias * __ldg(p.v_scale + cur.kh) : 0.f);
                if constexpr (kConsumerWarps == 2) named_barrier(1, 64);  // buffer free again
            } else {
                // Cross-warp merge of this item, in fixed warp order. Buffers alternate
                // between items, so a warp that races ahead to the next item's merge
                // cannot overwrite what a slower warp still reads here.
                float* sm_o = merge_buf + merge_sel * merge_floats<D>();  // [warps][8][OS]
                float* sm_m = sm_o + kConsumerWarps * kGroupMax * OS;     // [warps][8]
                float* sm_l = sm_m + kConsumerWarps * kGroupMax;
                float* sm_w = sm_l + kConsumerWarps * kGroupMax;          // weight / L
                merge_sel ^= 1;
    #pragma unroll
                for (int t = 0; t < MT; ++t) {
                    const int d0 = (t >> 2) * 64 + r * 8 + 2 * (t & 3);
                    float* o = sm_o + (warp * kGroupMax + 2 * c) * OS;
                    o[d0] = acc[t][0];
                    o[OS + d0] = acc[t][1];
                    o[d0 + 1] = acc[t][2];
                    o[OS + d0 + 1] = acc[t][3];
                }
                if (r == 0) {
                    sm_m[warp * kGroupMax + 2 * c] = m0;
                    sm_m[warp * kGroupMax + 2 * c + 1] = m1;
                    sm_l[warp * kGroupMax + 2 * c] = l0;
                    sm_l[warp * kGroupMax + 2 * c + 1] = l1;
                }
                named_barrier(1, kConsumerWarps * 32);
                if (threadIdx.x < group) {  // one thread per query row: the warps' weights
                    const int n = threadIdx.x;
                    float M = -INFINITY;
    #pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w * kGroupMax + n]);
                    float wg[kConsumerWarps];
                    float L = 0.f;
    #pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        const float mw = sm_m[w * kGroupMax + n];
                        wg[w] = mw == -INFINITY ? 0.f : exp2f(mw - M);
                        L = fmaf(sm_l[w * kGroupMax + n], wg[w], L);
                    }
    #pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w)
                        sm_w[w * kGroupMax + n] = L > 0.f ? wg[w] / L : 0.f;
                    if (P > 1) {
                        float* ml = p.ws_ml + ((head0 + n) * P + cur.part) * 2;
                        ml[0] = L > 0.f ? M : -INFINITY;
                        ml[1] = L;
                    }
                }
                named_barrier(1, kConsumerWarps * 32);
                for (int idx = threadIdx.x; idx < group * D; idx += kConsumerWarps * 32) {
                    const int n = idx / D;
                    const int d = idx - n * D;
                    float val = 0.f;
    #pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w)
                        val = fmaf(sm_o[(w * kGroupMax + n) * OS + d], sm_w[w * kGroupMax + n], val);
                    const int64_t row = head0 + n;
                    if (P == 1)
                        Elem<T>::store(p.out, row * D + d, val);
                    else
                        p.ws_o[(row * P + cur.part) * D + d] = val;
                }
            }
        }
        cur = nxt;
#pragma unroll
        for (int jp = 0; jp < KCH; ++jp) qcur[jp] = qnxt[jp];
    }
}

// ---------------------------------------------------------------------------
// Grouped decode: the sequences of one group (beams or parallel samples of
// one prompt, which hold its blocks through reference counts) run in one CTA,
// so a block they share crosses HBM once and feeds all of them.
//
// The CTA's query columns are (member, head) pairs, column = member * g + head
// for g = H / Hkv; consumer warp w owns n-tiles NT w .. NT w + NT - 1 of 8
// columns. Work item = (partition, kv head, group). The item's logical tokens
// are cut into units of SUB 16-token sub-tiles; for every unit the producer
// reads each active member's block ids and issues one ring position per
// distinct block sequence, tagged in a per-stage header with the mask of
// members that use it, the unit index and an end-of-item flag. Every consumer
// warp walks every position (the empty barrier counts all consumer warps),
// computes only when one of its members is in the mask (one online-softmax
// step per unit), and keeps its members' running state in registers to the
// end of the item; unit boundaries are logical positions, so each member's
// arithmetic is the same whichever blocks it shares. Sharing of prefix blocks among parallel samples and beams:
// "AI 推理系列（十六）：PagedAttention——…", § Copy-on-Write、并行采样与
// Prefix Caching 不是同一件事; "PagedAttention原理详解：GPU显存优化与模型路由
// 技术", § PagedAttention的三大核心优势 (point 2 and the beam-search paragraph).
// ---------------------------------------------------------------------------

// V fragments by ldmatrix.trans (head_dim in natural order in the
// accumulator). QK accumulation chains per sub-tile (1: a unit of several
// sub-tiles already gives independent chains).
#ifndef PA_GROUPED_QK_CHAINS
#define PA_GROUPED_QK_CHAINS 1
#endif
// Softmax weights by the hardware 2^x approximation (ex2.approx.ftz: relative
// error ~2^-22, far below the bf16 rounding the weights then take) on
// fma(score, scale, -max) instead of exp2f on separately scaled scores.
#ifndef PA_GROUPED_FAST_EXP
#define PA_GROUPED_FAST_EXP 1
#endif
// Column sums of the softmax weights by the tensor core: one more MMA per
// sub-tile with an all-ones A operand (each row of the result is the column's
// sum over the sub-tile's tokens), kept and rescaled like the accumulator,
// instead of unpacking and adding the weights on the CUDA cores.
#ifndef PA_GROUPED_MMA_SUM
#define PA_GROUPED_MMA_SUM 1
#endif

constexpr int kMaxGroupSeqs = 8;            // members per group (header mask bits 0..7)
constexpr int kGroupedMaxCols = 64;         // query columns (member, head) per CTA
constexpr uint32_t kUnitLast = 1u << 31;    // header: last unit of the item
constexpr int kUnitSubShift = 8;            // header bits 8..30: unit index in the item
constexpr uint32_t kUnitSubMask = 0x7fffffu;


// Ring bytes and CTAs per SM of each grouped variant (consumer warps CW,
// n-tiles per warp NT), the measured best of ring / occupancy sweeps on the
// beam and verification workloads: the kernel is latency-bound per warp, so
// each variant runs as many warps per SM as its ~168 registers allow, and
// four consumer warps take a deeper ring. Two n-tiles per warp need about 240
// registers at head_dim 128. Overridable for sweeps.
#ifndef PA_GROUPED_ONE_TILE_WARPS
#define PA_GROUPED_ONE_TILE_WARPS 4
#endif
#ifndef PA_G_RING1
#define PA_G_RING1 49152
#endif
#ifndef PA_G_BLK1
#define PA_G_BLK1 4
#endif
#ifndef PA_G_RING2
#define PA_G_RING2 49152
#endif
#ifndef PA_G_BLK2
#define PA_G_BLK2 4
#endif
#ifndef PA_G_RING3
#define PA_G_RING3 49152
#endif
#ifndef PA_G_BLK3
#define PA_G_BLK3 3
#endif
#ifndef PA_G_RING4
#define PA_G_RING4 65536
#endif
#ifndef PA_G_BLK4
#define PA_G_BLK4 2
#endif
// Sub-tiles per unit: a unit is SUB consecutive 16-token sub-tiles of one
// distinct block sequence, consumed in one online-softmax step, so the
// per-step work (barrier waits, the cross-lane max, rescaling) is paid once
// per 16 SUB tokens. SUB and the ring bytes of each variant (a stage holds
// 2 SUB sub-tiles of K and V) are the measured best; at least two stages.
#ifndef PA_G_SUB1
#define PA_G_SUB1 2
#endif
#ifndef PA_G_SUB2
#define PA_G_SUB2 2
#endif
#ifndef PA_G_SUB3
#define PA_G_SUB3 2
#endif
#ifndef PA_G_SUB4
#define PA_G_SUB4 4
#endif
#ifndef PA_G_SUB_NT2
#define PA_G_SUB_NT2 2
#endif
#ifndef PA_G_SRING4
#define PA_G_SRING4 98304
#endif
__host__ __device__ constexpr int grouped_sub(int cw, int nt) {
    return nt != 1 ? PA_G_SUB_NT2 : cw == 1 ? PA_G_SUB1 : cw == 2 ? PA_G_SUB2 : cw == 3 ? PA_G_SUB3 : PA_G_SUB4;
}
__host__ __device__ constexpr int grouped_ring_bytes(int cw, int nt) {
    return nt != 1 ? 49152
                   : cw == 1 ? PA_G_RING1
                   : cw == 2 ? PA_G_RING2
                   : cw == 3 ? PA_G_RING3
                   : grouped_sub(cw, nt) > 2 ? PA_G_SRING4 : PA_G_RING4;
}
__host__ __device__ constexpr int grouped_min_blocks(int d, int cw, int nt) {
    return nt == 1 ? (cw == 1 ? PA_G_BLK1 : cw == 2 ? PA_G_BLK2 : cw == 3 ? PA_G_BLK3 : PA_G_BLK4)
                   : d == 64 ? (cw <= 1 ? 4 : cw == 2 ? 3 : 2) : (cw <= 1 ? 4 : cw <= 3 ? 2 : 1);
}

// Ring of the grouped kernel: stage = K of the unit's SUB sub-tiles, then
// their V (kSubBytes each). Every consumer warp reads every stage.
template <typename TC, int D, int SUB, int RING>
struct GroupedRing {
    using T = TC;
    static constexpr bool kU2 = false;  // stage layout: [K sub-tiles][V sub-tiles]
    static constexpr int kSub = SUB;
    static constexpr int kBoxes = D * (int)sizeof(TC) / 128;
    static constexpr int kBoxElems = 128 / (int)sizeof(TC);
    static constexpr int kSubBytes = kBoxes * kBoxBytes;
    static constexpr int kStageBytes = 2 * SUB * kSubBytes;
    static constexpr int kStages = RING / kStageBytes;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static_assert(kStages >= 2, "grouped ring: at least two stages");
};
template <int D, int CW, int NT, typename TC = __nv_bfloat16>
using GroupedGeom = GroupedRing<TC, D, grouped_sub(CW, NT), grouped_ring_bytes(CW, NT)>;

// Walk over a grouped CTA's items, u = blockIdx.x + k * gridDim.x, item u =
// (partition u % P, kv head, group u / (P Hkv)). Lane l holds the context
// length of member l % gs of item kbase + l / gs (32 / gs items per load).
struct GWalk {
    int k, kbase, ctx_lane;
};

// Members of an item: sequences grp * gs + m (beams, samples), or, with
// multi-token queries, query tokens c * gs + m of sequence grp / q_chunks
// (c = grp % q_chunks), which all read that sequence's blocks.
struct GItem {
    bool valid;
    int grp, kh, part, t0;
    int tmax;     // end of the item's tokens over its members (== t0: nothing to read)
    int t1_lane;  // end of member (lane & 7)'s tokens in the item (t0 if none)
    int row0;     // q / out row of member 0 (member m: row0 + m)
    int nmem;     // members that exist (rows to write); <= 0: none
    int tab0;     // block-table row of member 0 (member m: tab0 + m * tab_step)
    int tab_step;
};

// Member m's token limit: its context length, or for query token j of a
// sequence with n new tokens (the last n of its context_len positions), the
// causal end ctx - n + j + 1. 0 for members that do not exist.
// Token limit of member m of grouped item u (0 when the member does not exist
// or reads nothing); `report`: record context lengths out of range (once per
// member: at its first partition).
__device__ __forceinline__ int gmember_limit(const DecodeParams& p, int u, int m, int gs,
                                             bool report) {
    const int part = u % p.num_partitions;
    const int grp = u / p.num_partitions / p.num_kv_heads;
    if (p.query_start == nullptr) {
        const int s = grp * gs + m;
        if (s >= p.num_seqs) return 0;
        return clamp_ctx(__ldg(p.context_lens + s), p.max_context_len, report && part == 0);
    }
    const int s = grp / p.q_chunks, j = (grp % p.q_chunks) * gs + m;
    const int q0 = __ldg(p.query_start + s), n = __ldg(p.query_start + s + 1) - q0;
    if (j >= n) return 0;
    const int ctx = clamp_ctx(__ldg(p.context_lens + s), p.max_context_len, report && part == 0);
    const int lim = ctx - n + j + 1;
    if (lim < 1) {  // more new query tokens than context: not a valid step
        if (report && part == 0) atomicOr(&s_status_tma, kStatusBadIndex);
        return 0;
    }
    return lim;
}

__device__ __forceinline__ int gwalk_load(const DecodeParams& p, int num_items, int kbase, int lane,
                                          int gs, int ipb, bool report) {
    if (lane >= ipb * gs) return 0;
    const int u = blockIdx.x + (kbase + lane / gs) * gridDim.x;
    if (u >= num_items) return 0;
    return gmember_limit(p, u, lane % gs, gs, report);
}

// Item u with member limit `lim` on lane l for member l & 7 (any value on lanes
// whose member does not exist): its fields, tmax included.
__device__ __forceinline__ GItem gitem_of(const DecodeParams& p, int u, int lim, int gs, int lane) {
    GItem it;
    it.valid = u >= 0;
    it.grp = it.kh = it.part = it.t0 = it.tmax = it.t1_lane = 0;
    it.row0 = it.nmem = it.tab0 = it.tab_step = 0;
    if (!it.valid) return it;
    const int m = lane & (kMaxGroupSeqs - 1);
    it.part = u % p.num_partitions;
    const int rest = u / p.num_partitions;
    it.kh = rest % p.num_kv_heads;
    it.grp = rest / p.num_kv_heads;
    it.t0 = it.part * p.partition_size;
    it.t1_lane = m < gs ? max(it.t0, min(lim, it.t0 + p.partition_size)) : it.t0;
    it.tmax = __reduce_max_sync(0xffffffffu, it.t1_lane);
    return it;
}

// Rows and block-table rows of an item's members.
__device__ __forceinline__ void gitem_rows(const DecodeParams& p, GItem& it, int gs) {
    if (p.query_start == nullptr) {
        it.row0 = it.tab0 = it.grp * gs;
        it.tab_step = 1;
        it.nmem = min(gs, p.num_seqs - it.row0);
    } else {
        const int sq = it.grp / p.q_chunks, c = it.grp % p.q_chunks;
        const int q0 = __ldg(p.query_start + sq);
        it.row0 = q0 + c * gs;
        it.nmem = min(gs, __ldg(p.query_start + sq + 1) - it.row0);
        it.tab0 = sq;
        it.tab_step = 0;
    }
}

__device__ __forceinline__ GItem gitem_next(GWalk& w, const DecodeParams& p, int num_items, int gs,
                                            int ipb, int lane, bool report, bool want_empty) {
    for (;;) {
        const int u = blockIdx.x + w.k * gridDim.x;
        if (u >= num_items) return gitem_of(p, -1, 0, gs, lane);
        if (w.k - w.kbase >= ipb) {
            w.kbase = w.k;
            w.ctx_lane = gwalk_load(p, num_items, w.kbase, lane, gs, ipb, report);
        }
        const int m = lane & (kMaxGroupSeqs - 1);
        const int ctx = __shfl_sync(0xffffffffu, w.ctx_lane, (w.k - w.kbase) * gs + (m < gs ? m : 0));
        GItem it = gitem_of(p, u, ctx, gs, lane);
        ++w.k;
        if (it.tmax > it.t0 || want_empty) {
            gitem_rows(p, it, gs);
            return it;
        }
    }
}

// Block ids of sub-tile base + lane for every member whose tokens reach it
// (bit m of `act`).
__device__ __forceinline__ void gload_phys(const DecodeParams& p, const GItem& it, int base, int gs,
                                           int lane, uint32_t& act, int (&phys)[kMaxGroupSeqs]) {
    act = 0;
    const int tok0 = it.t0 + ((base + lane) << 4);
#pragma unroll
    for (int m = 0; m < kMaxGroupSeqs; ++m) {
        const int t1 = __shfl_sync(0xffffffffu, it.t1_lane, m);
        phys[m] = -1;
        if (it.valid && m < gs && tok0 < t1) {
            act |= 1u << m;
            phys[m] = __ldg(p.block_tables + (int64_t)(it.tab0 + m * it.tab_step) * p.table_stride +
                            (tok0 >> p.log2_block_size));
        }
    }
}

// Issue the units of a batch of up to 32 sub-tiles (lane l: sub-tile base + l).
// Each lane finds the distinct block ids among its active members (the first
// member holding an id leads its unit); units take ring positions g + exclusive
// prefix sum, in sub-tile order and, within a sub-tile, in leader order. Lanes
// issue in sub-rounds of kStages positions, so a sub-round touches each stage
// at most once and a stage's rounds are issued in order.
template <class G>
// hdr2 (optional): per stage, the unit's largest valid token count over the
// members that use it (1..16).
__device__ __forceinline__ void issue_units(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                            const DecodeParams& p, const Ring& ring, uint32_t* hdr,
                                            const GItem& it, int base, int n_sub, uint32_t act,
                                            const int (&phys)[kMaxGroupSeqs], int lane, int& g,
                                            int& issued, bool& dead, uint32_t* hdr2 = nullptr) {
    int t1m[kMaxGroupSeqs];
#pragma unroll
    for (int m = 0; m < kMaxGroupSeqs; ++m) t1m[m] = __shfl_sync(0xffffffffu, it.t1_lane, m);
    uint32_t lead = 0;
    int nu = 0;
#pragma unroll
    for (int m = 0; m < kMaxGroupSeqs; ++m) {
        bool first = ((act >> m) & 1u) != 0;
#pragma unroll
        for (int m2 = 0; m2 < m; ++m2)
            if (((act >> m2) & 1u) && phys[m2] == phys[m]) first = false;
        if (first) {
            lead |= 1u << m;
            ++nu;
        }
    }
    int incl = nu;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    const int first_pos = incl - nu;
    const bool last_batch = base + 32 >= n_sub;
    const int i = base + lane;
    const int tok0 = it.t0 + (i << 4);
    for (int k0 = 0; k0 < total && !dead; k0 += G::kStages) {
        bool ok = true;
        int pos = first_pos;
#pragma unroll
        for (int m = 0; m < kMaxGroupSeqs; ++m) {
            if ((lead >> m) & 1u) {
                if (ok && pos >= k0 && pos < k0 + G::kStages) {
                    uint32_t mask = 0;
#pragma unroll
                    for (int m2 = m; m2 < kMaxGroupSeqs; ++m2)
                        if (((act >> m2) & 1u) && phys[m2] == phys[m]) mask |= 1u << m2;
                    const uint32_t h = mask | ((uint32_t)i << kUnitSubShift) |
                                       (last_batch && pos == total - 1 ? kUnitLast : 0u);
                    int nv = 0;
#pragma unroll
                    for (int m2 = 0; m2 < kMaxGroupSeqs; ++m2)
                        if ((mask >> m2) & 1u) nv = max(nv, min(16, t1m[m2] - tok0));
                    ok = issue_subtile<G>(kmap, vmap, p, ring, g + pos, phys[m], it.kh, tok0, hdr, h,
                                          hdr2, (uint32_t)nv);
                    if (ok) issued = g + pos + 1;
                }
                ++pos;
            }
        }
        dead = __any_sync(0xffffffffu, !ok);
    }
    issued = __reduce_max_sync(0xffffffffu, issued);
    g += total;
}

// Units of SUB sub-tiles. Lane l of a batch holds unit ubase + l, logical
// tokens tok0 .. tok0 + 16 SUB - 1 (tok0 = t0 + 16 SUB (ubase + l)), and for
// every member whose tokens reach the unit (bit m of `act`) the block ids of
// the sub-tiles it uses (-1 past its last token).
template <int SUB>
__device__ __forceinline__ void gload_units(const DecodeParams& p, const GItem& it, int ubase, int gs,
                                            int lane, uint32_t& act, int (&phys)[kMaxGroupSeqs][SUB]) {
    act = 0;
    const int tok0 = it.t0 + (ubase + lane) * (16 * SUB);
#pragma unroll
    for (int m = 0; m < kMaxGroupSeqs; ++m) {
        const int t1 = __shfl_sync(0xffffffffu, it.t1_lane, m);
        const bool on = it.valid && m < gs && tok0 < t1;
        if (on) act |= 1u << m;
        const int32_t* row = p.block_tables + (int64_t)(it.tab0 + m * it.tab_step) * p.table_stride;
#pragma unroll
        for (int s = 0; s < SUB; ++s) {
            const int tk = tok0 + 16 * s;
            phys[m][s] = on && tk < t1 ? __ldg(row + (tk >> p.log2_block_size)) : -1;
        }
    }
}

// Issue of one unit by one producer lane: wait until its stage is free, write
// the header, then load K and V of its first `nsub` sub-tiles (block ids ph)
// of kv head kh; the full barrier expects exactly those bytes. A block id
// outside the pool marks the stage empty-handed (nothing loaded) and records
// PA_ERR_BAD_INDEX. Returns false if the wait timed out.
// With G::kU2 (the tcgen05 consumer's ring) a stage holds K as two d-halves of
// kSub * 16 rows x 128 bytes, then V the same way (one canonical operand tile
// per half), K completing on ring.full[st] and V on the barrier kStages
// entries after it; hdr2 (if given) receives the unit's largest valid token
// count over the members that use it.
template <class G>
__device__ __forceinline__ bool issue_unit(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                           const DecodeParams& p, const Ring& ring, int gi,
                                           const int (&ph)[G::kSub], int nsub, int kh, int tok0,
                                           uint32_t* hdr, uint32_t hval, uint32_t* hdr2 = nullptr,
                                           uint32_t hval2 = 0) {
    const int st = gi % G::kStages;
    const uint32_t round = (uint32_t)(gi / G::kStages);
    if (!mbar_wait_bounded(ring.empty + 8 * st, (round & 1u) ^ 1u)) {
        atomicOr(&s_status_tma, kStatusTimeout);
        return false;
    }
    if (gi == p.test_skip_position) return true;  // test hook: leave this stage unloaded
    hdr[st] = hval;
    if (hdr2 != nullptr) hdr2[st] = hval2;
    bool ok = true;
#pragma unroll
    for (int s = 0; s < G::kSub; ++s)
        if (s < nsub && (unsigned)ph[s] >= (unsigned)p.num_blocks) ok = false;
    if constexpr (G::kU2) {
        const uint32_t full_k = ring.full + 8 * st, full_v = ring.full + 8 * (G::kStages + st);
        if (ok) {
            ring.valid[st] = 1;
            const uint32_t bytes = (uint32_t)(nsub * G::kBoxes * kBoxBytes);
            mbar_arrive_expect_tx(full_k, bytes);
            mbar_arrive_expect_tx(full_v, bytes);
            const uint32_t sb = ring.stages + st * G::kStageBytes;
#pragma unroll
            for (int s = 0; s < G::kSub; ++s) {
                if (s < nsub) {
                    const int32_t row = (ph[s] * p.num_kv_heads + kh) * p.block_size +
                                        ((tok0 + 16 * s) & (p.block_size - 1));
#pragma unroll
                    for (int b = 0; b < G::kBoxes; ++b)
                        tma_load_2d(sb + b * G::kHalfBytes + s * kBoxBytes, kmap, b * G::kBoxElems, row,
                                    full_k);
#pragma unroll
                    for (int b = 0; b < G::kBoxes; ++b)
                        tma_load_2d(sb + (G::kBoxes + b) * G::kHalfBytes + s * kBoxBytes, vmap,
                                    b * G::kBoxElems, row, full_v);
                }
            }
        } else {
            atomicOr(&s_status_tma, kStatusBadIndex);
            ring.valid[st] = 0;
            mbar_arrive(full_k);
            mbar_arrive(full_v);
        }
        return true;
    }
    if (ok) {
        ring.valid[st] = 1;
        const uint32_t full = ring.full + 8 * st;
        mbar_arrive_expect_tx(full, (uint32_t)(nsub * 2 * G::kSubBytes));
        const uint32_t sb = ring.stages + st * G::kStageBytes;
#pragma unroll
        for (int s = 0; s < G::kSub; ++s) {
            if (s < nsub) {
                const int32_t row = (ph[s] * p.num_kv_heads + kh) * p.block_size +
                                    ((tok0 + 16 * s) & (p.block_size - 1));
#pragma unroll
                for (int b = 0; b < G::kBoxes; ++b)
                    tma_load_2d(sb + s * G::kSubBytes + b * kBoxBytes, kmap, b * G::kBoxElems, row, full);
#pragma unroll
                for (int b = 0; b < G::kBoxes; ++b)
                    tma_load_2d(sb + (G::kSub + s) * G::kSubBytes + b * kBoxBytes, vmap, b * G::kBoxElems,
                                row, full);
            }
        }
    } else {
        atomicOr(&s_status_tma, kStatusBadIndex);
        ring.valid[st] = 0;
        mbar_arrive(ring.full + 8 * st);
    }
    return true;
}

// Issue the units of a batch of up to 32 (lane l: unit ubase + l). Members
// whose block ids and sub-tile counts agree share one ring position, led by
// the first of them; positions follow the same prefix-sum and sub-round order
// as issue_units.
template <class G>
__device__ __forceinline__ void issue_units_sub(const CUtensorMap* kmap, const CUtensorMap* vmap,
                                                const DecodeParams& p, const Ring& ring, uint32_t* hdr,
                                                const GItem& it, int ubase, int n_units, uint32_t act,
                                                const int (&phys)[kMaxGroupSeqs][G::kSub], int lane,
                                                int& g, int& issued, bool& dead,
                                                uint32_t* hdr2 = nullptr) {
    constexpr int SUB = G::kSub;
    const int i = ubase + lane;
    const int tok0 = it.t0 + i * (16 * SUB);
    int nsub[kMaxGroupSeqs], nvm[kMaxGroupSeqs];
#pragma unroll
    for (int m = 0; m < kMaxGroupSeqs; ++m) {
        const int t1 = __shfl_sync(0xffffffffu, it.t1_lane, m);
        nsub[m] = ((act >> m) & 1u) ? min(SUB, (t1 - tok0 + 15) >> 4) : 0;
        nvm[m] = ((act >> m) & 1u) ? min(16 * SUB, t1 - tok0) : 0;
    }
    auto same = [&](int a, int b) {
        bool eq = nsub[a] == nsub[b];
#pragma unroll
        for (int s = 0; s < SUB; ++s) eq = eq && phys[a][s] == phys[b][s];
        return eq;
    };
    uint32_t lead = 0;
    int nu = 0;
#pragma unroll
    for (int m = 0; m < kMaxGroupSeqs; ++m) {
        bool first = ((act >> m) & 1u) != 0;
#pragma unroll
        for (int m2 = 0; m2 < m; ++m2)
            if (((act >> m2) & 1u) && same(m2, m)) first = false;
        if (first) {
            lead |= 1u << m;
            ++nu;
        }
    }
    int incl = nu;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    const int first_pos = incl - nu;
    const bool last_batch = ubase + 32 >= n_units;
    for (int k0 = 0; k0 < total && !dead; k0 += G::kStages) {
        bool ok = true;
        int pos = first_pos;
#pragma unroll
        for (int m = 0; m < kMaxGroupSeqs; ++m) {
            if ((lead >> m) & 1u) {
                if (ok && pos >= k0 && pos < k0 + G::kStages) {
                    uint32_t mask = 0;
#pragma unroll
                    for (int m2 = m; m2 < kMaxGroupSeqs; ++m2)
                        if (((act >> m2) & 1u) && same(m, m2)) mask |= 1u << m2;
                    const uint32_t h = mask | ((uint32_t)i << kUnitSubShift) |
                                       (last_batch && pos == total - 1 ? kUnitLast : 0u);
                    int nv = 0;
#pragma unroll
                    for (int m2 = 0; m2 < kMaxGroupSeqs; ++m2)
                        if ((mask >> m2) & 1u) nv = max(nv, nvm[m2]);
                    ok = issue_unit<G>(kmap, vmap, p, ring, g + pos, phys[m], nsub[m], it.kh, tok0, hdr, h,
                                       hdr2, (uint32_t)nv);
                    if (ok) issued = g + pos + 1;
                }
                ++pos;
            }
        }
        dead = __any_sync(0xffffffffu, !ok);
    }
    issued = __reduce_max_sync(0xffffffffu, issued);
    g += total;
}

// S^T for NT n-tiles from one set of K fragments (see mma_qk).
template <int D, int NT>
__device__ __forceinline__ void mma_qk_n(uint32_t kb, const uint4 (&q)[NT][D / 32], int r, int c,
                                         float (&sc)[NT][4]) {
    constexpr int KCH = D / 32;
    uint4 kr[2][KCH];
#pragma unroll
    for (int jp = 0; jp < KCH; ++jp) {
        const uint32_t bx = kb + (jp >> 1) * kBoxBytes;
        const uint32_t x = (uint32_t)(2 * c + (jp & 1));
        kr[0][jp] = lds128(bx + swz(r, x));
        kr[1][jp] = lds128(bx + swz(r + 8, x));
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#if PA_GROUPED_QK_CHAINS == 2
        float sd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int jp = 0; jp < KCH; ++jp) {
            mma_16816(sc[j], kr[0][jp].x, kr[1][jp].x, kr[0][jp].y, kr[1][jp].y, q[j][jp].x, q[j][jp].y);
            mma_16816(sd, kr[0][jp].z, kr[1][jp].z, kr[0][jp].w, kr[1][jp].w, q[j][jp].z, q[j][jp].w);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[j][e] += sd[e];
#else
#pragma unroll
        for (int jp = 0; jp < KCH; ++jp) {
            mma_16816(sc[j], kr[0][jp].x, kr[1][jp].x, kr[0][jp].y, kr[1][jp].y, q[j][jp].x, q[j][jp].y);
            mma_16816(sc[j], kr[0][jp].z, kr[1][jp].z, kr[0][jp].w, kr[1][jp].w, q[j][jp].z, q[j][jp].w);
        }
#endif
    }
}

// V^T A-fragments of m-tile t (head_dim 16t .. 16t+15, natural order) by
// ldmatrix.trans: lane l addresses row l % 8 of matrix l / 8, i.e. token
// 8 (i / 2) + l % 8, head_dim 16t + 8 (i % 2) .. + 7. Thread (r, c) then holds
// A[r (+8)][tokens 2c, 2c+1 (+8)] as the m16n8k16 A operand wants.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&a)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

// Online-softmax update over a unit of SUB sub-tiles for NT n-tiles whose
// columns may each see a different number of valid tokens: nva / nvb = valid
// tokens (from the unit's first) of this thread's columns 2c and 2c + 1 of
// n-tile j, 0 for a column whose member does not use the unit. sc[s][j]: the
// S^T fragment of sub-tile s (tokens 16 s + r, 16 s + r + 8). A column that
// has seen no valid token keeps max -inf and weight 0. Leaves the P^T
// B-fragments of sub-tile s in pb0[s] / pb1[s] and returns the largest valid
// count of the warp's columns (V rows from there on must be zeroed).
template <int D, int NT, int SUB, bool kF16 = false>
__device__ __forceinline__ int softmax_update_n(const float (&sc)[SUB][NT][4], const int (&nva)[NT],
                                                const int (&nvb)[NT], float scale_log2, int r,
                                                float (&acc)[NT][D / 16][4], float (&ma)[NT],
                                                float (&mb)[NT], float (&la)[NT], float (&lb)[NT],
                                                float (&ls)[NT][4], uint32_t (&pb0)[SUB][NT],
                                                uint32_t (&pb1)[SUB][NT]) {
    constexpr int MT = D / 16;
    constexpr bool kMmaSum = PA_GROUPED_MMA_SUM != 0;
    // kFast: masked raw scores, max scaled once, weights 2^fma(s, scale, -max)
    constexpr bool kFast = PA_GROUPED_FAST_EXP != 0;
    const float mul = kFast ? 1.f : scale_log2;
    float sv[SUB][NT][4], mxa[NT], mxb[NT];
    int nvmax = 0, nvmin = 16 * SUB;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        nvmax = max(nvmax, max(nva[j], nvb[j]));
        nvmin = min(nvmin, min(nva[j], nvb[j]));
    }
    // every column of the warp uses every token of the unit (the common case):
    // no masking
    const bool full = __all_sync(0xffffffffu, nvmin >= 16 * SUB);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        mxa[j] = mxb[j] = -INFINITY;
#pragma unroll
        for (int s = 0; s < SUB; ++s) {
            const int t0 = 16 * s + r, t1 = t0 + 8;
            if (full) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sv[s][j][e] = sc[s][j][e] * mul;
            } else {
                sv[s][j][0] = t0 < nva[j] ? sc[s][j][0] * mul : -INFINITY;  // token t0, column 2c
                sv[s][j][1] = t0 < nvb[j] ? sc[s][j][1] * mul : -INFINITY;  // token t0, column 2c+1
                sv[s][j][2] = t1 < nva[j] ? sc[s][j][2] * mul : -INFINITY;  // token t1, column 2c
                sv[s][j][3] = t1 < nvb[j] ? sc[s][j][3] * mul : -INFINITY;  // token t1, column 2c+1
            }
            mxa[j] = fmaxf(mxa[j], fmaxf(sv[s][j][0], sv[s][j][2]));
            mxb[j] = fmaxf(mxb[j], fmaxf(sv[s][j][1], sv[s][j][3]));
        }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            mxa[j] = fmaxf(mxa[j], __shfl_xor_sync(0xffffffffu, mxa[j], off));
            mxb[j] = fmaxf(mxb[j], __shfl_xor_sync(0xffffffffu, mxb[j], off));
        }
    }
    bool mv = false;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        if (kFast) {  // the scaled max: scaling by a positive factor keeps the order
            mxa[j] *= scale_log2;
            mxb[j] *= scale_log2;
        }
        mxa[j] = fmaxf(ma[j], mxa[j]);  // new running max
        mxb[j] = fmaxf(mb[j], mxb[j]);
        mv = mv || mxa[j] != ma[j] || mxb[j] != mb[j];
    }
    const bool moved = __any_sync(0xffffffffu, mv);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        const float ba = mxa[j] == -INFINITY ? 0.f : mxa[j];
        const float bb = mxb[j] == -INFINITY ? 0.f : mxb[j];
        float ala = 1.f, alb = 1.f;
        if (moved) {
            if (kFast) {  // a max that did not move rescales by exactly 1
                ala = ma[j] == mxa[j] ? 1.f : ex2_approx(ma[j] - ba);
                alb = mb[j] == mxb[j] ? 1.f : ex2_approx(mb[j] - bb);
            } else {
                ala = exp2f(ma[j] - ba);
                alb = exp2f(mb[j] - bb);
            }
        }
        auto wt = [&](float x, float b) {
            return kFast ? ex2_approx(fmaf(x, scale_log2, -b)) : exp2f(x - b);
        };
        float suma = 0.f, sumb = 0.f;
#pragma unroll
        for (int s = 0; s < SUB; ++s) {
            // weights as the PV operand type: bf16, or f16 beside codes
            const uint32_t x0 = kF16 ? pack_f16x2(wt(sv[s][j][0], ba), wt(sv[s][j][1], bb))
                                     : pack_bf16x2(wt(sv[s][j][0], ba), wt(sv[s][j][1], bb));
            const uint32_t x1 = kF16 ? pack_f16x2(wt(sv[s][j][2], ba), wt(sv[s][j][3], bb))
                                     : pack_bf16x2(wt(sv[s][j][2], ba), wt(sv[s][j][3], bb));
            if (!kMmaSum) {
                suma += kF16 ? f16_lo(x0) + f16_lo(x1) : bf16_lo(x0) + bf16_lo(x1);
                sumb += kF16 ? f16_hi(x0) + f16_hi(x1) : bf16_hi(x0) + bf16_hi(x1);
            }
            pb0[s][j] = movmatrix_trans(x0);  // P^T rows (tokens) 16s + 2c, 2c+1; column r
            pb1[s][j] = movmatrix_trans(x1);  // tokens 16s + 2c+8, 2c+9
        }
        if (!kMmaSum) {
            la[j] = fmaf(la[j], ala, suma);
            lb[j] = fmaf(lb[j], alb, sumb);
        }
        ma[j] = mxa[j];
        mb[j] = mxb[j];
        if (moved) {
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                acc[j][t][0] *= ala;
                acc[j][t][1] *= alb;
                acc[j][t][2] *= ala;
                acc[j][t][3] *= alb;
            }
            if (kMmaSum) {
                ls[j][0] *= ala;
                ls[j][1] *= alb;
                ls[j][2] *= ala;
                ls[j][3] *= alb;
            }
        }
    }
    return __reduce_max_sync(0xffffffffu, nvmax);
}

// O^T += V^T . P^T over the unit's SUB sub-tiles, V^T fragments by
// ldmatrix.trans from the stage (vb: V of sub-tile 0, sub-tile s at
// vb + s * sub_bytes; natural head_dim order): a0 / a1 hold tokens 2c, 2c+1,
// a2 / a3 tokens 2c+8, 2c+9 of the sub-tile. Rows at or past nvmax (past every
// column's tokens: they may hold anything) are zeroed first; rows before that
// belong to some member's context. The stage is released (`release`: its
// empty barrier) as soon as the last fragments are in registers.
template <int D, int NT, int SUB>
__device__ __forceinline__ void pv_ldsm(uint32_t vb, int sub_bytes, int lane, int nvmax, int c,
                                        const uint32_t (&pb0)[SUB][NT], const uint32_t (&pb1)[SUB][NT],
                                        float (&acc)[NT][D / 16][4], float (&ls)[NT][4],
                                        uint32_t release) {
    constexpr int MT = D / 16;
    const int i = lane >> 3, row = 8 * (i >> 1) + (lane & 7);
    // sub-tiles that hold a token of some column (nvmax >= 1 for a unit in use)
    const int nsub = max(1, min(SUB, (nvmax + 15) >> 4));
#pragma unroll
    for (int s = 0; s < SUB; ++s) {
        if (s >= nsub) break;
        uint32_t va[MT][4];
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            const int d0 = 16 * t + 8 * (i & 1);
            ldsm_x4_trans(vb + s * sub_bytes + (d0 >> 6) * kBoxBytes + swz(row, (d0 & 63) >> 3), va[t]);
        }
        if (s == nsub - 1) {
            __syncwarp();
            if (lane == 0) mbar_arrive(release);
        }
        const int k0 = 16 * s;
        if (k0 + 16 > nvmax) {
            const uint32_t m01 = (k0 + 2 * c < nvmax ? 0x0000ffffu : 0u) |
                                 (k0 + 2 * c + 1 < nvmax ? 0xffff0000u : 0u);
            const uint32_t m89 = (k0 + 2 * c + 8 < nvmax ? 0x0000ffffu : 0u) |
                                 (k0 + 2 * c + 9 < nvmax ? 0xffff0000u : 0u);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                va[t][0] &= m01;
                va[t][1] &= m01;
                va[t][2] &= m89;
                va[t][3] &= m89;
            }
        }
#pragma unroll
        for (int t = 0; t < MT; ++t)
#pragma unroll
            for (int j = 0; j < NT; ++j)
                mma_16816(acc[j][t], va[t][0], va[t][1], va[t][2], va[t][3], pb0[s][j], pb1[s][j]);
        if (PA_GROUPED_MMA_SUM) {
            constexpr uint32_t kOnes = 0x3F803F80u;  // bf16 1.0, 1.0
#pragma unroll
            for (int j = 0; j < NT; ++j) mma_16816(ls[j], kOnes, kOnes, kOnes, kOnes, pb0[s][j], pb1[s][j]);
        }
    }
}

// O^T += V^T . P^T over the unit's SUB sub-tiles of codes (f16 MMAs; V^T
// fragments built from 16-byte chunks as in codes_softmax_pv: m-tile t rows r
// and r + 8 are head_dim 16 r + 2t and + 1). Tokens at or past nvmax are
// zeroed (a zero code is the value 0); the stage is released once the last
// chunks are in registers.
template <typename TC, int NT, int SUB>
__device__ __forceinline__ void pv_codes(uint32_t vb, int sub_bytes, int lane, int nvmax, int r,
                                         int c, const uint32_t (&pb0)[SUB][NT],
                                         const uint32_t (&pb1)[SUB][NT], float (&acc)[NT][8][4],
                                         float (&ls)[NT][4], uint32_t release) {
    const int nsub = max(1, min(SUB, (nvmax + 15) >> 4));
#pragma unroll
    for (int s = 0; s < SUB; ++s) {
        if (s >= nsub) break;
        uint4 vr[4];
        codes_load_v(vb + s * sub_bytes, r, c, vr);
        if (s == nsub - 1) {
            __syncwarp();
            if (lane == 0) mbar_arrive(release);
        }
        const int k0 = 16 * s;
        if (k0 + 16 > nvmax) {
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            if (k0 + 2 * c >= nvmax) vr[0] = z;
            if (k0 + 2 * c + 1 >= nvmax) vr[1] = z;
            if (k0 + 2 * c + 8 >= nvmax) vr[2] = z;
            if (k0 + 2 * c + 9 >= nvmax) vr[3] = z;
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const uint32_t va = code_word<TC>(word(vr[0], w)), vbw = code_word<TC>(word(vr[1], w));
            const uint32_t vc = code_word<TC>(word(vr[2], w)), vd = code_word<TC>(word(vr[3], w));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t sel = h ? 0x7362u : 0x5140u;
                uint32_t a0, a1, a2, a3;
                code_pairs_f16<TC>(__byte_perm(va, vbw, sel), a0, a1);
                code_pairs_f16<TC>(__byte_perm(vc, vd, sel), a2, a3);
#pragma unroll
                for (int j = 0; j < NT; ++j)
                    mma_16816_f16(acc[j][2 * w + h], a0, a1, a2, a3, pb0[s][j], pb1[s][j]);
            }
        }
        if (PA_GROUPED_MMA_SUM) {
            constexpr uint32_t kOnes = 0x3C003C00u;  // f16 1.0, 1.0
#pragma unroll
            for (int j = 0; j < NT; ++j)
                mma_16816_f16(ls[j], kOnes, kOnes, kOnes, kOnes, pb0[s][j], pb1[s][j]);
        }
    }
}

// Store one column's result (m, l = its running max and summed weights): bf16
// output when P == 1, else the normalised partial and (m, l).
template <int D, bool kCodes = false>
__device__ __forceinline__ void grouped_store_col(const DecodeParams& p, int64_t row, int part, int r,
                                                  int c, int e, const float (&acc)[D / 16][4],
                                                  float m, float l, float vs = 1.f,
                                                  float obias = 0.f) {
    constexpr int MT = D / 16;
    const int P = p.num_partitions;
    const int DQ = kCodes ? p.head_dim : D;  // out / workspace row length
    const float inv = (l > 0.f ? 1.f / l : 0.f) * vs;  // vs: V scale of a quantised cache
    // int8 codes: 1152 x the weights in the accumulator (obias = 1152 x vs)
    const float ob = l > 0.f ? obias : 0.f;
    auto nv = [&](float a) { return obias != 0.f ? fmaf(a, inv, -ob) : a * inv; };
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        // rows r and r + 8 of m-tile t: head_dim 16t + r and 16t + 8 + r (codes:
        // 16r + 2t and 16r + 2t + 1; at or past DQ: padding, not stored)
        const int d0 = kCodes ? 16 * r + 2 * t : 16 * t + r, d1 = kCodes ? d0 + 1 : d0 + 8;
        if (kCodes && d0 >= DQ) continue;
        if (P == 1) {
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + row * DQ;
            o[d0] = __float2bfloat16_rn(nv(acc[t][e]));
            o[d1] = __float2bfloat16_rn(nv(acc[t][e + 2]));
        } else {
            float* o = p.ws_o + (row * P + part) * DQ;
            o[d0] = nv(acc[t][e]);
            o[d1] = nv(acc[t][e + 2]);
        }
    }
    if (P > 1 && r == 0) {
        float* ml = p.ws_ml + (row * P + part) * 2;
        ml[0] = l > 0.f ? m : -INFINITY;
        ml[1] = l;
    }
}

template <int D, int CW, int NT, typename TC = __nv_bfloat16>
__global__ void __launch_bounds__((CW + 1) * 32, grouped_min_blocks(D, CW, NT))
decode_tma_grouped_kernel(const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap, const DecodeParams p,
                          int num_items, int gs) {
    using G = GroupedGeom<D, CW, NT, TC>;
    // quantised codes: f16 MMAs on exactly converted codes (as the tensor-core
    // consumer over codes), q rounded to f16, the K scale in the score scale
    // and the V scale in the output
    constexpr bool kCodes = !std::is_same<TC, __nv_bfloat16>::value;
    static_assert(!kCodes || D == 128, "quantised codes: head_dim 128");
    constexpr int SUB = G::kSub;
    constexpr int KCH = D / 32;
    constexpr int MT = D / 16;
    constexpr int kUnitTokens = 16 * SUB;
    const int DQ = kCodes ? p.head_dim : D;  // q / out head_dim (codes: 64 or 128)
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    asm volatile("griddepcontrol.launch_dependents;");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.num_partitions;
    const int group = p.num_heads / p.num_kv_heads;
    const int ipb = 32 / gs;
    Ring ring;
    uint8_t* base = setup_ring<G>(smem_raw, ring, G::kStages * 4, CW);
    if (base == nullptr) {
        if (threadIdx.x == 0) atomicOr(&s_status_tma, kStatusSmemAlign);
        return;
    }
    uint32_t* hdr = reinterpret_cast<uint32_t*>(base + G::kRingBytes);
    GWalk walk;
    walk.k = 0;
    walk.kbase = 0;
    walk.ctx_lane = gwalk_load(p, num_items, 0, lane, gs, ipb, warp == 0);
    __syncthreads();

    if (warp == CW) {  // producer
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        bool dead = false;
        int g = 0, issued = 0;
        GItem cur = gitem_next(walk, p, num_items, gs, ipb, lane, false, false);
        int cur_base = 0;
        uint32_t act_cur;
        int phys_cur[kMaxGroupSeqs][SUB];
        gload_units<SUB>(p, cur, cur_base, gs, lane, act_cur, phys_cur);
        while (cur.valid && !dead) {
            const int n_units = (cur.tmax - cur.t0 + kUnitTokens - 1) / kUnitTokens;
            GItem nxt = cur;
            int nxt_base = cur_base + 32;
            if (nxt_base >= n_units) {
                nxt = gitem_next(walk, p, num_items, gs, ipb, lane, false, false);
                nxt_base = 0;
            }
            uint32_t act_nxt;
            int phys_nxt[kMaxGroupSeqs][SUB];
            gload_units<SUB>(p, nxt, nxt_base, gs, lane, act_nxt, phys_nxt);  // in flight meanwhile
            issue_units_sub<G>(&kmap, &vmap, p, ring, hdr, cur, cur_base, n_units, act_cur, phys_cur,
                               lane, g, issued, dead);
            cur = nxt;
            cur_base = nxt_base;
            act_cur = act_nxt;
#pragma unroll
            for (int m = 0; m < kMaxGroupSeqs; ++m)
#pragma unroll
                for (int u = 0; u < SUB; ++u) phys_cur[m][u] = phys_nxt[m][u];
        }
        drain_ring<G>(ring, issued, lane);
        return;
    }

    // consumers: thread (r, c) holds q column 8 (NT warp + j) + r of n-tile j as
    // the B operand, and C-fragment columns 8 (NT warp + j) + 2c, + 2c + 1
    const int r = lane >> 2, c = lane & 3;
    const int col0 = 8 * NT * warp;
    uint32_t bita[NT], bitb[NT];  // mask bit of this thread's columns' members (0: none)
    uint32_t wbits = 0;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        const int ma = (col0 + 8 * j + 2 * c) / group, mb = (col0 + 8 * j + 2 * c + 1) / group;
        bita[j] = ma < gs ? 1u << ma : 0u;
        bitb[j] = mb < gs ? 1u << mb : 0u;
        wbits |= bita[j] | bitb[j];
    }
    wbits = __reduce_or_sync(0xffffffffu, wbits);
    // q of the item's columns (zero for columns without a member, sequence or
    // tokens). The softmax below takes the max of unscaled scores, so the sign
    // of the score scale goes into q (an exact negation) and the scale used is
    // its magnitude; over codes q is rounded to f16 with a power-of-two shift
    // (q_shift_warp) that the returned score scale undoes.
    auto load_q = [&](const GItem& it, uint4 (&q)[NT][KCH]) -> float {
        const float sl0 = kCodes && it.valid ? p.scale_log2 * __ldg(p.k_scale + it.kh) : p.scale_log2;
        const bool neg = sl0 < 0.f;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int col = col0 + 8 * j + r;
            const int m = col / group, hd = col - m * group;
            const int t1 = __shfl_sync(0xffffffffu, it.t1_lane, m & (kMaxGroupSeqs - 1));
            const uint16_t* qrow = nullptr;
            if (it.valid && m < gs && m < it.nmem && t1 > it.t0)
                qrow = static_cast<const uint16_t*>(p.q) +
                       ((int64_t)(it.row0 + m) * p.num_heads + (int64_t)it.kh * group + hd) * DQ;
            if constexpr (kCodes) {
                load_q_raw(qrow, c, q[j], DQ);
            } else {
                const uint32_t sg = neg ? 0x80008000u : 0u;
#pragma unroll
                for (int jp = 0; jp < KCH; ++jp) {
                    uint4 v = qrow != nullptr ? ld_v4(qrow + (jp >> 1) * 64 + (2 * c + (jp & 1)) * 8)
                                              : make_uint4(0u, 0u, 0u, 0u);
                    q[j][jp] = make_uint4(v.x ^ sg, v.y ^ sg, v.z ^ sg, v.w ^ sg);
                }
            }
        }
        if constexpr (kCodes) {
            float am = 0.f;
#pragma unroll
            for (int j = 0; j < NT; ++j) am = fmaxf(am, q_raw_amax(q[j]));
            const int sh = q_shift_warp(am);
            const float mul = neg ? -pow2i(-sh) : pow2i(-sh);
#pragma unroll
            for (int j = 0; j < NT; ++j) q_raw_to_f16(q[j], mul, q[j]);
            return fabsf(sl0) * pow2i(sh);
        }
        return fabsf(sl0);
    };
    bool dead = false;
    int g = 0;
    GItem cur = gitem_next(walk, p, num_items, gs, ipb, lane, warp == 0, P == 1);
    uint4 q[NT][KCH];
    float sl = load_q(cur, q);  // the item's score scale (log2 units, positive)
    // int8 codes: 1152 x the sum of q of the thread's score columns 8j + 2c, + 1
    constexpr bool kInt8 = std::is_same<TC, Int8Code>::value;
    float qb[NT][2];
    auto q_bias = [&]() {
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            qb[j][0] = qb[j][1] = 0.f;
            if constexpr (kInt8) int8_qk_bias(q[j], c, qb[j][0], qb[j][1]);
        }
    };
    q_bias();
    while (cur.valid && !dead) {
        GItem nxt = gitem_next(walk, p, num_items, gs, ipb, lane, warp == 0, P == 1);
        int t1a[NT], t1b[NT];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int ma = (col0 + 8 * j + 2 * c) / group, mb = (col0 + 8 * j + 2 * c + 1) / group;
            t1a[j] = __shfl_sync(0xffffffffu, cur.t1_lane, ma & (kMaxGroupSeqs - 1));
            t1b[j] = __shfl_sync(0xffffffffu, cur.t1_lane, mb & (kMaxGroupSeqs - 1));
        }
        float acc[NT][MT][4], ls[NT][4];
        float ma[NT], mb[NT], la[NT], lb[NT];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[j][t][0] = acc[j][t][1] = acc[j][t][2] = acc[j][t][3] = 0.f;
            ls[j][0] = ls[j][1] = ls[j][2] = ls[j][3] = 0.f;
            ma[j] = mb[j] = -INFINITY;
            la[j] = lb[j] = 0.f;
        }
        if (cur.tmax > cur.t0) {
            for (;;) {
                const int st = g % G::kStages;
                const uint32_t round = (uint32_t)(g / G::kStages);
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(ring.full + 8 * st, round & 1u))) {
                    if (lane == 0) atomicOr(&s_status_tma, kStatusTimeout);
                    dead = true;
                    break;
                }
                const uint32_t h = hdr[st];
                const bool mine = ring.valid[st] != 0 && (h & wbits) != 0;
                if (mine) {
                    const int tok0 = cur.t0 + (int)((h >> kUnitSubShift) & kUnitSubMask) * kUnitTokens;
                    const uint32_t kb = ring.stages + st * G::kStageBytes;
                    float sc[SUB][NT][4];
#pragma unroll
                    for (int u = 0; u < SUB; ++u) {
                        if constexpr (kCodes) {
#pragma unroll
                            for (int j = 0; j < NT; ++j) {
                                codes_qk<TC>(kb + u * G::kSubBytes, q[j], r, c, sc[u][j]);
                                if constexpr (kInt8) {
                                    sc[u][j][0] -= qb[j][0];
                                    sc[u][j][1] -= qb[j][1];
                                    sc[u][j][2] -= qb[j][0];
                                    sc[u][j][3] -= qb[j][1];
                                }
                            }
                        } else {
                            mma_qk_n<D, NT>(kb + u * G::kSubBytes, q, r, c, sc[u]);
                        }
                    }
                    int nva[NT], nvb[NT];
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        nva[j] = (h & bita[j]) ? min(kUnitTokens, t1a[j] - tok0) : 0;
                        nvb[j] = (h & bitb[j]) ? min(kUnitTokens, t1b[j] - tok0) : 0;
                    }
                    uint32_t pb0[SUB][NT], pb1[SUB][NT];
                    const int nvmax = softmax_update_n<D, NT, SUB, kCodes>(sc, nva, nvb, sl, r, acc, ma,
                                                                           mb, la, lb, ls, pb0, pb1);
                    if constexpr (kCodes)
                        pv_codes<TC, NT, SUB>(kb + SUB * G::kSubBytes, G::kSubBytes, lane, nvmax, r, c,
                                              pb0, pb1, acc, ls, ring.empty + 8 * st);
                    else
                        pv_ldsm<D, NT, SUB>(kb + SUB * G::kSubBytes, G::kSubBytes, lane, nvmax, c, pb0,
                                            pb1, acc, ls, ring.empty + 8 * st);  // releases the stage
                } else {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(ring.empty + 8 * st);  // stage released
                }
                ++g;
                if (h & kUnitLast) break;
            }
        }
        if (dead) break;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            if (PA_GROUPED_MMA_SUM) {  // every row of the sums tile holds the column sums
                la[j] = ls[j][0];
                lb[j] = ls[j][1];
            } else {
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    la[j] += __shfl_xor_sync(0xffffffffu, la[j], off);
                    lb[j] += __shfl_xor_sync(0xffffffffu, lb[j], off);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < NT; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int col = col0 + 8 * j + 2 * c + e;
                const int m = col / group, hd = col - m * group;
                const int t1 = e == 0 ? t1a[j] : t1b[j];
                if (m < gs && m < cur.nmem && (P == 1 || t1 > cur.t0)) {
                    const int64_t row =
                        (int64_t)(cur.row0 + m) * p.num_heads + (int64_t)cur.kh * group + hd;
                    grouped_store_col<D, kCodes>(p, row, cur.part, r, c, e, acc[j],
                                                 e == 0 ? ma[j] : mb[j], e == 0 ? la[j] : lb[j],
                                                 kCodes ? __ldg(p.v_scale + cur.kh) : 1.f,
                                                 kInt8 ? kInt8Bias * __ldg(p.v_scale + cur.kh) : 0.f);
                }
            }
        }
        cur = nxt;
        sl = load_q(cur, q);
        q_bias();
    }
}

// ---------------------------------------------------------------------------
// 5th-generation tensor-core (tcgen05) helpers.
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor: start address, leading / stride byte
// offsets (16-byte units), descriptor version 1, layout 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor for kind::f16: fp32 accumulator, bf16 (or, with
// f16, f16) A and B, A K-major, B K-major or MN-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc(int m, int n, bool b_mn_major, bool f16 = false,
                                                  bool a_mn_major = false) {
    return (1u << 4) | ((f16 ? 0u : 1u) << 7) | ((f16 ? 0u : 1u) << 10) |
           ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}
// D (TMEM) (+)= A (shared) . B (shared)^T, issued by one thread.
__device__ __forceinline__ void umma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        bool acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)acc) : "memory");
}
// D (TMEM) (+)= A (TMEM) . B (shared)^T.
__device__ __forceinline__ void umma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                        bool acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"((uint32_t)acc) : "memory");
}
// The mbarrier at `bar` gets one arrival once every tcgen05 operation this
// thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// generic-proxy shared-memory writes made visible to the tensor core's reads
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(slot), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(taddr), "r"(ncols) : "memory");
}
// Loads / stores of this warp's 32 TMEM lanes (32x32b): thread t reads or
// writes lane (lane of taddr) + t, consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]) : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
                 :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]) : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Grouped and multi-token decode on the 5th-generation tensor cores (head_dim
// 128, at most 32 query columns (member, head) per item; bf16 caches, or
// FP8 E4M3 / int8 codes converted to f16 in shared memory).
// Same work items as decode_tma_grouped_kernel, with 64-token units: four
// 16-token sub-tiles of one distinct block sequence, a header per stage
// (member mask, unit index, last-unit flag) and the unit's largest valid
// token count over its members. Roles:
//   warp 4: the producer. Over bf16 a stage holds the unit's K as two
//     d-halves of 64 rows x 128 bytes (128-byte swizzle), then its V the same
//     way, so each is one canonical operand tile; K and V complete on barriers
//     of their own, so S = Q K^T can start while V is still landing. Over
//     codes a stage holds the 64 rows of 128 codes of K, then of V;
//   warps 6 and 7 (codes only): the converters. They turn a unit's codes into
//     an f16 K tile and an f16 V tile laid out as the bf16 stage (exact: every
//     E4M3 and int8 value is an f16), V rows past every member's tokens as
//     zeros, copy the unit's header into one of four slots, and release the
//     stage; the K tile is rewritten once the previous unit's QK is done, the
//     V tile once its PV is;
//   warp 5, lane 0: per unit S = Q . K^T (M = 128 rows, N = 64 tokens,
//     K = 128: 8 tcgen05.mma kind::f16 steps, S in TMEM, double-buffered) and
//     O += P . V (A = P from shared memory, B = V read MN-major; M = 128,
//     N = 128, K = 64: 4 steps, O in TMEM); completions by tcgen05.commit;
//   warps 0..3 (TMEM lane quarters 0..3): softmax. The item's (up to) 32 query
//     columns are replicated into the four 32-row quarters of the 128-row Q
//     tile, so warp w finds every column's scores in its own TMEM lanes; it
//     takes tokens 16 w .. 16 w + 15 of each unit (thread = column x token
//     slice). The four warps share one reference max per column.
// A unit's weights are 2^(score - m) with m the column's reference max, moved
// only when a score exceeds it by more than kU2RescaleLog2 (log2 units);
// numerator and denominator share m, so the result is the exact softmax with
// weights below 2^kU2RescaleLog2. Whether any column must move is one
// bar.red.or over the softmax warps per unit; only then do they exchange their
// slice maxima through shared memory, and warp 0 (whose TMEM lanes hold O's
// rows) rescales O. A column's decisions depend only on its own scores in
// logical order, so its result is the same whichever blocks it shares and
// whichever members share its CTA. P (bf16, or f16 beside codes; row =
// column, 64 tokens) goes to a double-buffered shared tile that the PV MMA
// reads. Over codes q is rounded to f16 after a power-of-two shift of its own
// column (q_shift_warp's rule per row), undone in the column's score scale,
// and the K and V scales fold into the score scale and the output. Every wait
// is bounded; a give-up is agreed by the softmax warps at the next per-unit
// vote, and TMEM is freed after a final commit on every path.
// ---------------------------------------------------------------------------
constexpr int kU2Tokens = 64;                   // tokens per unit
constexpr int kU2Cols = 32;                     // query columns per item, at most
constexpr int kU2Slice = kU2Tokens / 4;         // tokens per softmax warp per unit
constexpr int kU2HalfBytes = kU2Tokens * 128;   // one d-half of a K or V tile: 8 KB
// Ring depth and CTAs per SM. A stage is busy for the TMA latency of its
// loads (~2 us for a unit's 16 boxes, measured by timestamps on a B200) plus
// its use (QK, softmax, PV: ~1.2-1.8 us), so an SM needs about five 32 KB stages
// in flight to read at HBM rate: one CTA per SM with five bf16 stages (eight
// 16 KB stages over codes), 200 KB of shared memory.
#ifndef PA_U2_STAGES
#define PA_U2_STAGES 3
#endif
#ifndef PA_U2_CODE_STAGES
#define PA_U2_CODE_STAGES 4
#endif
#ifndef PA_U2_CTAS
#define PA_U2_CTAS 2
#endif
constexpr int kU2PBytes = kU2Cols * 128;        // P tile: 32 rows x 64 16-bit tokens
constexpr int kU2RingOff = 2 * kU2PBytes;       // shared memory: [P0][P1][ring][...]
// TMEM columns: O^T (128 head_dim lanes x 32 query columns, fp32), then Q
// (128 rows x 128 16-bit values, two per column: the A operand of QK), then S
// (128 rows x 64 tokens, fp32) twice.
constexpr uint32_t kU2TmemCols = 256;
constexpr uint32_t kU2ColO = 0, kU2ColQ = 32, kU2ColS = 96;
constexpr float kU2RescaleLog2 = 8.f;

// Ring of the bf16 variant: box-major stages with K and V barriers of their own.
struct U2Geom {
    using T = __nv_bfloat16;
    static constexpr bool kU2 = true;
    static constexpr int kSub = kU2Tokens / 16;
    static constexpr int kStages = PA_U2_STAGES;
    static constexpr int kBoxes = 2;
    static constexpr int kBoxElems = 64;
    static constexpr int kHalfBytes = kU2HalfBytes;
    static constexpr int kSubBytes = kBoxes * kBoxBytes;
    static constexpr int kStageBytes = 4 * kU2HalfBytes;  // K halves, then V halves: 32 KB
    static constexpr int kRingBytes = kStages * kStageBytes;
};

// Layout of one variant: the ring the producer fills (over codes: stages of
// [K sub-tiles][V sub-tiles], 16 KB, one barrier), the f16 K and V tiles over
// codes, and after them [hdr S][hdr2 S][valid S][header slots 3 x 4], the
// barriers (full_k S, full_v S, empty S, s 2, pv 2, p 2, q, ofree, done, fin,
// kf_full 4, kf_free, vf_full, vf_free), the TMEM slot and the dead flag, the
// slice maxima [2][4][32], give-up flags [2][4] and slice sums [4][32].
template <typename TC>
struct U2Cfg {
    static constexpr bool kCodes = !std::is_same<TC, __nv_bfloat16>::value;
    using Ring = typename std::conditional<
        kCodes, GroupedRing<TC, 128, kU2Tokens / 16, PA_U2_CODE_STAGES * 2 * kU2HalfBytes>, U2Geom>::type;
    static constexpr int kStages = Ring::kStages;
    static constexpr int kThreads = kCodes ? 256 : 192;
    static constexpr int kKfOff = kU2RingOff + Ring::kRingBytes;   // f16 K tile (codes)
    static constexpr int kVfOff = kKfOff + 2 * kU2HalfBytes;       // f16 V tile (codes)
    static constexpr int kExtOff = kCodes ? kVfOff + 2 * kU2HalfBytes : kU2RingOff + Ring::kRingBytes;
    static constexpr int kHdr = 12 * kStages + 48;
    static constexpr int kBars = (kHdr + 7) & ~7;
    static constexpr int kNumBars = 3 * kStages + 17;
    static constexpr int kSlot = kBars + 8 * kNumBars;
    static constexpr int kXm = (kSlot + 8 + 15) & ~15;
    static constexpr int kXf = kXm + 2 * 4 * 32 * 4;
    static constexpr int kXl = kXf + 2 * 4 * 4;
    static constexpr int kExtBytes = kXl + 4 * 32 * 4;
    static constexpr size_t kSmem = (size_t)kExtOff + kExtBytes;
    // QK: A = Q from TMEM, B = K K-major; PV (transposed): A = V^T MN-major
    // (head_dim contiguous in the V tile), B = P K-major (tokens contiguous)
    static constexpr uint32_t kIdescQK = umma_idesc(128, 64, false, kCodes);
    static constexpr uint32_t kIdescPV = umma_idesc(128, kU2Cols, false, kCodes, true);
    static_assert(kU2RingOff % 1024 == 0 && kKfOff % 1024 == 0 && kVfOff % 1024 == 0,
                  "operand tiles on 1024-byte boundaries");
    static_assert(kSmem * PA_U2_CTAS + 1024 * PA_U2_CTAS <= 228 * 1024 && kSmem <= 227 * 1024,
                  "shared memory of PA_U2_CTAS CTAs per SM");
};

struct U2Bars {
    uint32_t full_k, full_v, empty, s, pv, p, q, ofree, done, fin;  // shared addresses
    uint32_t kf_full, kf_free, vf_full, vf_free;                    // codes: f16 tiles
    volatile int* dead;
};

// Bounded wait by a whole warp, warp-uniform outcome; gives up at once when
// another role already gave up (so timeouts do not chain).
__device__ __forceinline__ bool u2_wait(const U2Bars& b, uint32_t bar, uint32_t parity) {
    const bool ok = __all_sync(0xffffffffu, *b.dead == 0 && mbar_wait_bounded(bar, parity));
    if (!ok && (threadIdx.x & 31) == 0) {
        if (*b.dead == 0) atomicOr(&s_status_tma, kStatusTimeout);
        *b.dead = 1;
    }
    return ok;
}

// OR of `pred` over the 128 threads of the softmax warps (named barrier 1).
__device__ __forceinline__ bool softmax_any(bool pred) {
    uint32_t r;
    asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n"
                 " bar.red.or.pred p, 1, 128, q;\n selp.u32 %0, 1, 0, p;\n}"
                 : "=r"(r) : "r"((uint32_t)pred) : "memory");
    return r != 0;
}

// 16 codes (one 16-byte chunk, in order) -> 16 f16 values in order, exactly:
// E4M3 by the hardware conversion; int8 as (1024 + code + 128) - 1152 in f16
// (a byte permute under the exponent of 1024, then one exact subtraction).
template <typename TC>
__device__ __forceinline__ void codes_to_f16_exact(const uint4& c, uint4& lo, uint4& hi) {
    uint32_t h[8];
    codes_to_f16x2<TC, true>(c, h);
    lo = make_uint4(h[0], h[1], h[2], h[3]);
    hi = make_uint4(h[4], h[5], h[6], h[7]);
}

// 64 rows of 128 codes (rows 128 bytes apart, 128-byte swizzle) -> an f16 tile
// [2 halves][64 rows][128 B] (128-byte swizzle); rows at or past `zero_from`
// become zeros. 64 threads (t = 0..63), 8 chunks of 16 codes each.
template <typename TC>
__device__ __forceinline__ void convert_tile(uint32_t src, uint32_t dst, int t, int zero_from) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int i = t + 64 * k, r = i >> 3, x = i & 7;
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
        if (r < zero_from) codes_to_f16_exact<TC>(lds128(src + swz(r, x)), lo, hi);
        const uint32_t half = dst + (x >> 2) * kU2HalfBytes;
        const uint32_t c0 = 2 * (x & 3);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                     :: "r"(half + swz(r, c0)), "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w) : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                     :: "r"(half + swz(r, c0 + 1)), "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w) : "memory");
    }
}

template <typename TC>
__global__ void __launch_bounds__(U2Cfg<TC>::kThreads, PA_U2_CTAS)
decode_umma_grouped_kernel(const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap, const DecodeParams p,
                           int num_items, int gs) {
    using C = U2Cfg<TC>;
    using G = typename C::Ring;
    constexpr bool kCodes = C::kCodes;
    constexpr int S_ = C::kStages;
    constexpr int D = 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    asm volatile("griddepcontrol.launch_dependents;");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.num_partitions;
    const int group = p.num_heads / p.num_kv_heads;
    const int ncols = gs * group;
    const int ipb = 32 / gs;
    const int DQ = kCodes ? p.head_dim : D;  // q / out head_dim (codes: 64 or 128)
    const uint32_t raw = smem_u32(smem_raw);
    if (raw & 1023u) {
        if (threadIdx.x == 0) atomicOr(&s_status_tma, kStatusSmemAlign);
        return;
    }
    const uint32_t pbuf = raw;
    const uint32_t kfbuf = raw + C::kKfOff, vfbuf = raw + C::kVfOff;
    uint8_t* ext = smem_raw + C::kExtOff;
    uint32_t* hdr = reinterpret_cast<uint32_t*>(ext);
    uint32_t* hdr2 = hdr + S_;
    int* valid = reinterpret_cast<int*>(hdr2 + S_);
    uint32_t* hc = reinterpret_cast<uint32_t*>(valid + S_);  // codes: header slots [3][4]
    U2Bars B;
    B.full_k = smem_u32(ext + C::kBars);
    B.full_v = B.full_k + 8 * S_;
    B.empty = B.full_v + 8 * S_;
    B.s = B.empty + 8 * S_;  // [2]
    B.pv = B.s + 16;         // [2]
    B.p = B.pv + 16;         // [2]
    B.q = B.p + 16;
    B.ofree = B.q + 8;
    B.done = B.ofree + 8;
    B.fin = B.done + 8;
    B.kf_full = B.fin + 8;   // [4]
    B.kf_free = B.kf_full + 32;
    B.vf_full = B.kf_free + 8;
    B.vf_free = B.vf_full + 8;
    uint32_t* tslot = reinterpret_cast<uint32_t*>(ext + C::kSlot);
    B.dead = reinterpret_cast<volatile int*>(tslot + 1);
    float* xm = reinterpret_cast<float*>(ext + C::kXm);  // [2][4][32] slice maxima
    volatile int* xf = reinterpret_cast<volatile int*>(ext + C::kXf);  // [2][4] give-ups
    float* xl = reinterpret_cast<float*>(ext + C::kXl);  // [4][32] slice sums
    Ring ring;
    ring.stages = raw + kU2RingOff;
    ring.full = B.full_k;
    ring.empty = B.empty;
    ring.valid = valid;
    if (threadIdx.x == 0) {
        for (int st = 0; st < S_; ++st) {
            mbar_init(B.full_k + 8 * st, 1);
            mbar_init(B.full_v + 8 * st, 1);
            // released by the MMA thread's commit after the unit's PV, or over
            // codes by the two converter warps once they converted it
            mbar_init(B.empty + 8 * st, kCodes ? 2 : 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(B.s + 8 * i, 1);
            mbar_init(B.pv + 8 * i, 1);
            mbar_init(B.p + 8 * i, 4);
        }
        mbar_init(B.q, 4);
        mbar_init(B.ofree, 1);  // warp 0's final commit: every PV it issued is complete
        mbar_init(B.done, 4);
        mbar_init(B.fin, 1);
        for (int i = 0; i < 4; ++i) mbar_init(B.kf_full + 8 * i, 2);
        mbar_init(B.kf_free, 1);
        mbar_init(B.vf_full, 2);
        mbar_init(B.vf_free, 1);
        *B.dead = 0;
        fence_barrier_init();
    }
    if (warp == 5) tmem_alloc(smem_u32(tslot), kU2TmemCols);
    GWalk walk;
    walk.k = 0;
    walk.kbase = 0;
    walk.ctx_lane = gwalk_load(p, num_items, 0, lane, gs, ipb, warp == 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tslot;

    if (warp == 4) {  // producer
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        constexpr int SUB = G::kSub;
        bool dead = false;
        int g = 0, issued = 0;
        GItem cur = gitem_next(walk, p, num_items, gs, ipb, lane, false, false);
        int cur_base = 0;
        uint32_t act_cur;
        int phys_cur[kMaxGroupSeqs][SUB];
        gload_units<SUB>(p, cur, cur_base, gs, lane, act_cur, phys_cur);
        while (cur.valid && !dead) {
            const int n_units = (cur.tmax - cur.t0 + kU2Tokens - 1) / kU2Tokens;
            GItem nxt = cur;
            int nxt_base = cur_base + 32;
            if (nxt_base >= n_units) {
                nxt = gitem_next(walk, p, num_items, gs, ipb, lane, false, false);
                nxt_base = 0;
            }
            uint32_t act_nxt;
            int phys_nxt[kMaxGroupSeqs][SUB];
            gload_units<SUB>(p, nxt, nxt_base, gs, lane, act_nxt, phys_nxt);
            issue_units_sub<G>(&kmap, &vmap, p, ring, hdr, cur, cur_base, n_units, act_cur, phys_cur,
                               lane, g, issued, dead, hdr2);
            if (*B.dead) dead = true;
            cur = nxt;
            cur_base = nxt_base;
            act_cur = act_nxt;
#pragma unroll
            for (int m = 0; m < kMaxGroupSeqs; ++m)
#pragma unroll
                for (int u = 0; u < SUB; ++u) phys_cur[m][u] = phys_nxt[m][u];
        }
        if (dead) *B.dead = 1;
        // drain: the last loads of every stage have landed
        if (lane == 0 && issued > 0) {
            const int last = min(issued, S_);
            for (int st = 0; st < last; ++st) {
                const int it = issued - 1 - ((issued - 1 - st) % S_);
                const uint32_t par = (uint32_t)(it / S_) & 1u;
                if (!mbar_wait_bounded(B.full_k + 8 * st, par) ||
                    (!kCodes && !mbar_wait_bounded(B.full_v + 8 * st, par)))
                    atomicOr(&s_status_tma, kStatusTimeout);
            }
        }
        return;
    }

    if (kCodes && warp >= 6) {  // converters: codes -> f16 K and V tiles
        const int t = threadIdx.x - 192;
        int g = 0;
        bool ok = true;
        GItem cur = gitem_next(walk, p, num_items, gs, ipb, lane, false, false);
        while (cur.valid && ok) {
            for (;;) {
                const int st = g % S_;
                if (!u2_wait(B, ring.full + 8 * st, (uint32_t)(g / S_) & 1u)) { ok = false; break; }
                const uint32_t h = hdr[st], h2 = hdr2[st];
                const int v = valid[st];
                const uint32_t cb = ring.stages + st * G::kStageBytes;
                // the K tile is free once the previous unit's QK is done
                if (g >= 1 && !u2_wait(B, B.kf_free, (uint32_t)(g - 1) & 1u)) { ok = false; break; }
                if (v) convert_tile<TC>(cb, kfbuf, t, kU2Tokens);
                if (t == 0) {
                    hc[g & 3] = h;
                    hc[4 + (g & 3)] = h2;
                    hc[8 + (g & 3)] = (uint32_t)v;
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(B.kf_full + 8 * (g & 3));
                // the V tile is free once the previous unit's PV is done; rows
                // past every member's tokens become zeros
                if (g >= 1 && !u2_wait(B, B.vf_free, (uint32_t)(g - 1) & 1u)) { ok = false; break; }
                if (v) convert_tile<TC>(cb + G::kSub * G::kSubBytes, vfbuf, t, (int)h2);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(B.vf_full);
                    mbar_arrive(ring.empty + 8 * st);  // the codes are no longer needed
                }
                ++g;
                if (h & kUnitLast) break;
            }
            if (ok) cur = gitem_next(walk, p, num_items, gs, ipb, lane, false, false);
        }
        return;
    }

    if (warp == 5) {
        // QK issuer: lane 0 issues S = Q . K^T of each unit once the item's q is
        // in TMEM, the unit's K tile has landed and its S buffer is free (the
        // softmax of the unit two back has read it). The PVs are issued by the
        // softmax warps themselves, as soon as P is written.
        int g = 0, n = 0;
        bool ok = true;
        GItem cur = gitem_next(walk, p, num_items, gs, ipb, lane, false, false);
        while (cur.valid && ok) {
            if (!u2_wait(B, B.q, n & 1)) { ok = false; break; }
            for (;;) {
                const int st = g % S_;
                if (g >= 2 && !u2_wait(B, B.p + 8 * (g & 1), ((g - 2) >> 1) & 1)) { ok = false; break; }
                if (kCodes) {
                    if (!u2_wait(B, B.kf_full + 8 * (g & 3), (uint32_t)(g >> 2) & 1u)) { ok = false; break; }
                } else if (!u2_wait(B, B.full_k + 8 * st, (uint32_t)(g / S_) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t h = kCodes ? hc[g & 3] : hdr[st];
                const bool v = (kCodes ? hc[8 + (g & 3)] : (uint32_t)valid[st]) != 0;
                if (lane == 0) {
                    if (v) {
                        const uint32_t kb = kCodes ? kfbuf : ring.stages + st * G::kStageBytes;
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            umma_ts(tm + kU2ColS + 64 * (g & 1), tm + kU2ColQ + 8 * k,
                                    umma_desc(kb + (k >> 2) * kU2HalfBytes + (k & 3) * 32, 16, 1024),
                                    C::kIdescQK, k > 0);
                    }
                    umma_commit(B.s + 8 * (g & 1));
                    if (kCodes) umma_commit(B.kf_free);
                }
                __syncwarp();
                ++g;
                if (h & kUnitLast) break;
            }
            ++n;
            if (ok) cur = gitem_next(walk, p, num_items, gs, ipb, lane, false, false);
        }
        // wait for the softmax warps (even after a give-up: they stop touching
        // TMEM, and their PVs are complete, before they arrive), then for every
        // QK issued here, then free TMEM
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(B.done, 0)) && lane == 0)
            atomicOr(&s_status_tma, kStatusTimeout);
        if (lane == 0) umma_commit(B.fin);
        __syncwarp();
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(B.fin, 0)) && lane == 0)
            atomicOr(&s_status_tma, kStatusTimeout);
        tc_fence_after();
        tmem_dealloc(tm, kU2TmemCols);
        return;
    }

    // softmax warps: thread = query column `lane` (member, head) of the item,
    // tokens 16 warp .. 16 warp + 15 of every unit; Q row 32 warp + lane
    const int col = lane;
    const int mem = col / group, hd = col - mem * group;
    const bool colv = col < ncols;
    const uint32_t mybit = (colv && mem < gs) ? 1u << mem : 0u;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const int slice0 = kU2Slice * warp;
    const uint8_t* qsrc_base = static_cast<const uint8_t*>(p.q);
    int g = 0, n = 0;
    bool ok = true, healthy = true;
    // Next item with tokens; with one partition, the members of items without
    // any tokens get a zero output here.
    auto next_item = [&]() -> GItem {
        for (;;) {
            GItem it = gitem_next(walk, p, num_items, gs, ipb, lane, warp == 0, P == 1);
            if (!it.valid || it.tmax > it.t0) return it;
            if (warp == 0 && colv && mem < it.nmem) {
                uint16_t* o = static_cast<uint16_t*>(p.out) +
                              ((int64_t)(it.row0 + mem) * p.num_heads + (int64_t)it.kh * group + hd) * DQ;
                for (int c = 0; c < DQ / 8; ++c)
                    reinterpret_cast<uint4*>(o)[c] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    // This thread's Q row (32 warp + lane) := q of its column, 128-byte
    // swizzled. The softmax takes maxima of unscaled scores, so the sign of the
    // score scale goes into q (an exact negation) and its magnitude is used;
    // over codes q is rounded to f16 after its column's power-of-two shift.
    // Returns the column's score scale (log2 units, positive).
    auto stage_q = [&](const GItem& it) -> float {
        const int t1 = __shfl_sync(0xffffffffu, it.t1_lane, mem & (kMaxGroupSeqs - 1));
        const bool has = colv && mem < it.nmem && t1 > it.t0;
        const float sl0 = kCodes ? p.scale_log2 * __ldg(p.k_scale + it.kh) : p.scale_log2;
        const uint32_t sg = sl0 < 0.f ? 0x80008000u : 0u;
        const uint4* src = reinterpret_cast<const uint4*>(qsrc_base +
            ((int64_t)(it.row0 + mem) * p.num_heads + (int64_t)it.kh * group + hd) * DQ * 2);
        auto ldq = [&](int c) {
            const uint4 v = has && 8 * c < DQ ? ld_v4(src + c) : make_uint4(0u, 0u, 0u, 0u);
            return make_uint4(v.x ^ sg, v.y ^ sg, v.z ^ sg, v.w ^ sg);
        };
        float slc = fabsf(sl0);
        float mul = 1.f;
        if constexpr (kCodes) {
            uint32_t m = 0;  // largest |q| of the row (bits of a non-negative float)
#pragma unroll 4
            for (int c = 0; c < 16; ++c) {
                const uint4 v = ldq(c);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    m = max(m, max((w[i] << 16) & 0x7fffffffu, w[i] & 0x7fff0000u));
            }
            const int sh = m == 0u ? 0 : max(-112, min(113, (int)((m >> 23) & 0xFFu) - 127 - 14));
            mul = pow2i(-sh);
            slc *= pow2i(sh);
        }
        // the row in its TMEM lane: head_dim 2i, 2i + 1 in column i (two halves
        // of 32 columns)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            uint32_t w[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 v = ldq(8 * hf + c);  // (again: a cache hit)
                if constexpr (kCodes)
                    v = make_uint4(pack_f16x2(bf16_lo(v.x) * mul, bf16_hi(v.x) * mul),
                                   pack_f16x2(bf16_lo(v.y) * mul, bf16_hi(v.y) * mul),
                                   pack_f16x2(bf16_lo(v.z) * mul, bf16_hi(v.z) * mul),
                                   pack_f16x2(bf16_lo(v.w) * mul, bf16_hi(v.w) * mul));
                w[4 * c] = v.x;
                w[4 * c + 1] = v.y;
                w[4 * c + 2] = v.z;
                w[4 * c + 3] = v.w;
            }
            tmem_st32(tm + lane_off + kU2ColQ + 32 * hf, w);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B.q);
        return slc;
    };
    GItem cur = next_item();
    float sl_next = cur.valid ? stage_q(cur) : 0.f;
    while (cur.valid && ok) {
        const int t1 = __shfl_sync(0xffffffffu, cur.t1_lane, mem & (kMaxGroupSeqs - 1));
        const float sl = sl_next;
        float m_ref = -INFINITY, l = 0.f;
        bool o_started = false;  // warp 0: a PV of this item has written O^T
        for (;;) {
            const int b = g & 1, st = g % S_;
            // S of unit g (and with it every earlier MMA: the PV of unit g - 2
            // no longer reads P buffer b); the K barrier (bf16) or the header
            // slot's barrier (codes) orders the header reads
            if (healthy) healthy = u2_wait(B, B.s + 8 * b, (g >> 1) & 1);
            if (kCodes) {
                if (healthy) healthy = u2_wait(B, B.kf_full + 8 * (g & 3), (uint32_t)(g >> 2) & 1u);
            } else if (healthy) {
                healthy = u2_wait(B, B.full_k + 8 * st, (uint32_t)(g / S_) & 1u);
            }
            uint32_t h = 0;
            int nvmax = 0;
            bool v = false;
            float sv[kU2Slice];
            float mx = -INFINITY;
            if (healthy) {
                tc_fence_after();
                h = kCodes ? hc[g & 3] : hdr[st];
                v = (kCodes ? hc[8 + (g & 3)] : (uint32_t)valid[st]) != 0;
                nvmax = (int)(kCodes ? hc[4 + (g & 3)] : hdr2[st]);
                const int tok0 = cur.t0 + (int)((h >> kUnitSubShift) & kUnitSubMask) * kU2Tokens;
                uint32_t sr[kU2Slice];
                tmem_ld16(tm + lane_off + kU2ColS + 64 * b + slice0, sr);
                const int nv = (v && (h & mybit)) ? min(kU2Slice, t1 - tok0 - slice0) : 0;
#pragma unroll
                for (int j = 0; j < kU2Slice; ++j) sv[j] = j < nv ? __uint_as_float(sr[j]) : -INFINITY;
                float m4[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    m4[j] = fmaxf(fmaxf(sv[4 * j], sv[4 * j + 1]), fmaxf(sv[4 * j + 2], sv[4 * j + 3]));
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            } else {
#pragma unroll
                for (int j = 0; j < kU2Slice; ++j) sv[j] = -INFINITY;
            }
            // a column's reference max moves when a score exceeds it by more
            // than the threshold (or on its first scores)
            const bool exceed =
                mx != -INFINITY && (m_ref == -INFINITY || mx * sl > m_ref + kU2RescaleLog2);
            if (softmax_any(exceed || !healthy)) {
                xm[(b * 4 + warp) * 32 + lane] = mx;
                if (lane == 0) xf[b * 4 + warp] = healthy ? 0 : 1;
                named_barrier(1, 128);
                if (xf[b * 4] | xf[b * 4 + 1] | xf[b * 4 + 2] | xf[b * 4 + 3]) {
                    ok = false;
                    break;
                }
                float M = xm[(b * 4) * 32 + lane];
#pragma unroll
                for (int w = 1; w < 4; ++w) M = fmaxf(M, xm[(b * 4 + w) * 32 + lane]);
                float alpha = 1.f;
                bool resc = false;
                if (M != -INFINITY && (m_ref == -INFINITY || M * sl > m_ref + kU2RescaleLog2)) {
                    const float nm = M * sl;
                    if (m_ref != -INFINITY) {
                        alpha = exp2f(m_ref - nm);
                        l *= alpha;
                        resc = true;
                    }
                    m_ref = nm;
                }
                // O^T (lanes: head_dim 32 warp .. + 31, column j: query column j)
                // is rescaled column by column once the PV of the previous unit is
                // done; lane j holds column j's factor (every warp holds every
                // column's state, so all four take the same branch)
                if (__any_sync(0xffffffffu, resc)) {
                    healthy = u2_wait(B, B.pv + 8 * ((g - 1) & 1), ((g - 1) >> 1) & 1);
                    if (healthy) {
                        tc_fence_after();
                        uint32_t o[32];
                        tmem_ld32(tm + lane_off + kU2ColO, o);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            o[j] = __float_as_uint(__uint_as_float(o[j]) * __shfl_sync(0xffffffffu, alpha, j));
                        tmem_st32(tm + lane_off + kU2ColO, o);
                    }
                }
            }
            // weights of the slice (masked scores give 2^-inf = 0), bf16 (f16
            // beside codes), summed as rounded
            const float base = m_ref == -INFINITY ? 0.f : m_ref;
            uint32_t pk[kU2Slice / 2];
            float ps = 0.f;
#pragma unroll
            for (int j = 0; j < kU2Slice / 2; ++j) {
                const float w0 = ex2_approx(fmaf(sv[2 * j], sl, -base));
                const float w1 = ex2_approx(fmaf(sv[2 * j + 1], sl, -base));
                if constexpr (kCodes) {
                    pk[j] = pack_f16x2(w0, w1);
                    ps += f16_lo(pk[j]) + f16_hi(pk[j]);
                } else {
                    pk[j] = pack_bf16x2(w0, w1);
                    ps += bf16_lo(pk[j]) + bf16_hi(pk[j]);
                }
            }
            l += ps;
            // P buffer b is read by the PV of unit g - 2, issued by warp 0 at the
            // end of that unit: it must be complete before P is rewritten
            if (g >= 2 && healthy) healthy = u2_wait(B, B.pv + 8 * b, ((g - 2) >> 1) & 1);
            // P row `col`, tokens 16 warp .. + 15: 16-byte chunks 2 warp, 2 warp + 1
            const uint32_t prow = pbuf + b * kU2PBytes;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                         :: "r"(prow + swz(col, 2 * warp)), "r"(pk[0]), "r"(pk[1]), "r"(pk[2]),
                            "r"(pk[3]) : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                         :: "r"(prow + swz(col, 2 * warp + 1)), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]),
                            "r"(pk[7]) : "memory");
            // bf16: V rows of the slice at or past every member's tokens may hold
            // anything (NaN included): zero them once V has landed (over codes
            // the converters wrote those rows as zeros)
            if (!kCodes && healthy && v && nvmax < slice0 + kU2Slice) {
                healthy = u2_wait(B, B.full_v + 8 * st, (uint32_t)(g / S_) & 1u);
                if (healthy) {
                    const uint32_t vb = ring.stages + st * G::kStageBytes + 2 * kU2HalfBytes;
                    const int r0 = max(nvmax, slice0);
                    for (int i = lane; i < (slice0 + kU2Slice - r0) * 16; i += 32) {
                        const int row = r0 + (i >> 4), c16 = i & 15;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};"
                                     :: "r"(vb + (c16 >> 3) * kU2HalfBytes + row * 128 + (c16 & 7) * 16),
                                        "r"(0u) : "memory");
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            // S buffer b has been read (the QK issuer may overwrite it)
            if (lane == 0) mbar_arrive(B.p + 8 * b);
            // O^T += V^T . P^T by warp 0's lane 0 once every warp's P rows are
            // written (and, over bf16, V has landed); then the stage (bf16) or the
            // f16 V tile (codes) is released. The first unit of an item overwrites
            // O^T: the previous item's output was read before this item began.
            named_barrier(1, 128);
            if (warp == 0) {
                if (healthy) {
                    healthy = kCodes ? u2_wait(B, B.vf_full, (uint32_t)g & 1u)
                                     : u2_wait(B, B.full_v + 8 * st, (uint32_t)(g / S_) & 1u);
                }
                tc_fence_after();
                if (lane == 0 && healthy) {
                    if (v) {
                        const uint32_t vb =
                            kCodes ? vfbuf : ring.stages + st * G::kStageBytes + 2 * kU2HalfBytes;
#pragma unroll
                        for (int k = 0; k < kU2Tokens / 16; ++k)
                            umma_ss(tm + kU2ColO, umma_desc(vb + 2048 * k, kU2HalfBytes, 1024),
                                    umma_desc(prow + 32 * k, 16, 1024), C::kIdescPV,
                                    o_started || k > 0);
                    }
                    umma_commit(B.pv + 8 * b);
                    umma_commit(kCodes ? B.vf_free : B.empty + 8 * st);
                }
                if (v) o_started = true;
                __syncwarp();
            }
            ++g;
            if (h & kUnitLast) break;
        }
        if (!ok) break;
        // the column's weight sum over the four slices (fixed order)
        xl[warp * 32 + lane] = l;
        named_barrier(1, 128);
        const float lt = ((xl[lane] + xl[32 + lane]) + xl[64 + lane]) + xl[96 + lane];
        // the next item's q: every QK of this item is complete (its last S was read)
        const GItem nxt = next_item();
        if (nxt.valid) sl_next = stage_q(nxt);
        // O^T: thread (warp, lane) holds head_dim d = 32 warp + lane of every
        // column; column j's row, normaliser and flags come from lane j
        if (healthy) healthy = u2_wait(B, B.pv + 8 * ((g - 1) & 1), ((g - 1) >> 1) & 1);
        {
            const bool has = colv && mem < cur.nmem && t1 > cur.t0;
            const bool wr = colv && mem < cur.nmem;
            const int64_t row = (int64_t)(cur.row0 + mem) * p.num_heads + (int64_t)cur.kh * group + hd;
            const float inv = (lt > 0.f ? 1.f / lt : 0.f) * (kCodes ? __ldg(p.v_scale + cur.kh) : 1.f);
            const int d = 32 * warp + lane;
            if (healthy) {
                tc_fence_after();
                uint32_t o[32];
                tmem_ld32(tm + lane_off + kU2ColO, o);
#pragma unroll
                for (int j = 0; j < kU2Cols; ++j) {
                    const bool wr_j = __shfl_sync(0xffffffffu, wr, j);
                    const bool has_j = __shfl_sync(0xffffffffu, has, j);
                    const int64_t row_j = __shfl_sync(0xffffffffu, row, j);
                    const float val = __uint_as_float(o[j]) * __shfl_sync(0xffffffffu, inv, j);
                    if (d < DQ) {
                        if (P == 1) {
                            if (wr_j) static_cast<__nv_bfloat16*>(p.out)[row_j * DQ + d] = __float2bfloat16_rn(val);
                        } else if (has_j) {
                            p.ws_o[(row_j * P + cur.part) * DQ + d] = val;
                        }
                    }
                }
                if (warp == 0 && P > 1 && has) {
                    float* ml = p.ws_ml + (row * P + cur.part) * 2;
                    ml[0] = lt > 0.f ? m_ref : -INFINITY;
                    ml[1] = lt;
                }
            }
        }
        tc_fence_before();  // O^T reads done before the next item's first PV (after a barrier)
        __syncwarp();
        cur = nxt;
        ++n;
    }
    // warp 0 issued the PVs: all of them complete before TMEM may be freed
    if (warp == 0) {
        if (lane == 0) umma_commit(B.ofree);
        __syncwarp();
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(B.ofree, 0)) && lane == 0)
            atomicOr(&s_status_tma, kStatusTimeout);
        tc_fence_before();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(B.done);
}

template <typename T, int D>
cudaError_t launch_simt_t(const DecodeParams& p, const CUtensorMap& km, const CUtensorMap& vm,
                          cudaStream_t stream) {
    using G = SimtGeom<T, D>;
    constexpr size_t smem = smem_bytes<G>();
    cudaError_t e = cudaFuncSetAttribute(decode_tma_simt_kernel<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(decode_tma_simt_kernel<T, D>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)p.num_partitions, (unsigned)p.num_heads, (unsigned)p.num_rows);
    decode_tma_simt_kernel<T, D><<<grid, G::kThreads, smem, stream>>>(km, vm, p);
    return cudaGetLastError();
}

template <int D, typename TC = __nv_bfloat16>
cudaError_t launch_mma_t(const DecodeParams& p, const CUtensorMap& km, const CUtensorMap& vm,
                         cudaStream_t stream) {
    using G = MmaGeom<D, TC>;
    constexpr size_t smem = smem_bytes<G>(merge_bytes<D>() + kItemQBytes);
    auto kernel = decode_tma_mma_kernel<D, TC>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    // persistent grid: every CTA slot of the GPU, or fewer if there are fewer items
    static int per_sm[128] = {0};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
    if (per_sm[dev] == 0) {
        int n = 0;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, G::kThreads, smem)) != cudaSuccess)
            return e;
        per_sm[dev] = n > 0 ? n : 1;
    }
    int sms = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long items = (long)p.num_partitions * p.num_kv_heads * p.num_seqs;
    const long slots = (long)per_sm[dev] * sms;
    const unsigned grid = (unsigned)(items < slots ? items : slots);
    kernel<<<grid, G::kThreads, smem, stream>>>(km, vm, p, (int)items);
    return cudaGetLastError();
}

template <typename TC>
cudaError_t launch_umma_grouped(const DecodeParams& p, const CUtensorMap& km,
                                const CUtensorMap& vm, int gs, cudaStream_t stream) {
    using C = U2Cfg<TC>;
    constexpr size_t smem = C::kSmem;
    auto kernel = decode_umma_grouped_kernel<TC>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long groups = p.query_start != nullptr ? (long)p.num_seqs * p.q_chunks
                                                 : (long)(p.num_seqs + gs - 1) / gs;
    const long items = (long)p.num_partitions * p.num_kv_heads * groups;
    const long slots = (long)PA_U2_CTAS * sms;
    const unsigned grid = (unsigned)(items < slots ? items : slots);
    kernel<<<grid, C::kThreads, smem, stream>>>(km, vm, p, (int)items, gs);
    return cudaGetLastError();
}

template <int D, int CW, int NT, typename TC = __nv_bfloat16>
cudaError_t launch_grouped_t(const DecodeParams& p, const CUtensorMap& km, const CUtensorMap& vm,
                             int gs, cudaStream_t stream) {
    using G = GroupedGeom<D, CW, NT, TC>;
    constexpr size_t smem = smem_bytes<G>(G::kStages * 4);
    constexpr int kThreads = (CW + 1) * 32;
    auto kernel = decode_tma_grouped_kernel<D, CW, NT, TC>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    static int per_sm[128] = {0};
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 128) return cudaErrorInvalidDevice;
    if (per_sm[dev] == 0) {
        int n = 0;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, smem)) != cudaSuccess)
            return e;
        per_sm[dev] = n > 0 ? n : 1;
    }
    int sms = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long groups = p.query_start != nullptr ? (long)p.num_seqs * p.q_chunks
                                                 : (long)(p.num_seqs + gs - 1) / gs;
    const long items = (long)p.num_partitions * p.num_kv_heads * groups;
    const long slots = (long)per_sm[dev] * sms;
    const unsigned grid = (unsigned)(items < slots ? items : slots);
    kernel<<<grid, kThreads, smem, stream>>>(km, vm, p, (int)items, gs);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_tma(const DecodeParams& p, int dtype, int head_dim, bool mma,
                              const CUtensorMap& kmap, const CUtensorMap& vmap,
                              cudaStream_t stream) {
    if (mma) {
        if (dtype == 2) return launch_mma_t<128, E4M3Code>(p, kmap, vmap, stream);
        if (dtype == 3) return launch_mma_t<128, Int8Code>(p, kmap, vmap, stream);
        return head_dim == 64 ? launch_mma_t<64>(p, kmap, vmap, stream)
                              : launch_mma_t<128>(p, kmap, vmap, stream);
    }
    if (dtype == 0) {
        return head_dim == 64 ? launch_simt_t<float, 64>(p, kmap, vmap, stream)
                              : launch_simt_t<float, 128>(p, kmap, vmap, stream);
    }
    if (dtype == 2) return launch_simt_t<E4M3Code, 128>(p, kmap, vmap, stream);
    if (dtype == 3) return launch_simt_t<Int8Code, 128>(p, kmap, vmap, stream);
    return head_dim == 64 ? launch_simt_t<__nv_bfloat16, 64>(p, kmap, vmap, stream)
                          : launch_simt_t<__nv_bfloat16, 128>(p, kmap, vmap, stream);
}

int mma_ctas_per_sm() { return PA_MMA_MIN_BLOCKS; }

// The tensor-core consumer takes grouped-query heads (g = 2..8) over bf16 or
// codes. One query head per kv head stays on the CUDA-core consumer: over
// codes the tensor-core one with one MMA column of eight measured slower on
// B200 (13B MHA: fp8 564 vs 536 us, int8 661 vs 622 us; 7B fp8 173 vs 125 us).
bool mma_supported(int dtype, int head_dim, int group) {
    const bool codes = (dtype == 2 || dtype == 3) && (head_dim == 64 || head_dim == 128);
    return (codes || (dtype == 1 && (head_dim == 64 || head_dim == 128))) && group >= 2 &&
           group <= kGroupMax;
}

// Grouped consumer selected by pa_set_grouped_consumer (process-wide). The
// tcgen05 consumer takes head_dim 128 with 8..32 query columns (its 128-row
// MMAs hold four copies of up to 32 columns; with fewer than 8 they would mostly
// idle); other shapes stay on mma.sync.
static thread_local int g_grouped_consumer = PA_GROUPED_MMA_SYNC;  // per host thread

static bool use_umma(int head_dim, int gs, int group) {
    return g_grouped_consumer == PA_GROUPED_TCGEN05 && head_dim == 128 && gs * group >= 8 &&
           gs * group <= kU2Cols;
}

// Query columns (member, head) -> n-tiles of 8 -> consumer warps: one n-tile
// per warp when a single tile holds them all, else two per warp.
static void grouped_shape(int gs, int group, int* cw, int* nt) {
    const int tiles = (gs * group + 7) / 8;
    *nt = tiles <= PA_GROUPED_ONE_TILE_WARPS ? 1 : 2;
    *cw = (tiles + *nt - 1) / *nt;
}

// bf16 or quantised codes (PA_FP8_E4M3, PA_INT8) at head_dim 64 or 128 (codes
// at 64 on the 128-code consumer, rows zero-filled past 64).
bool grouped_supported(int dtype, int head_dim, int group, int gs) {
    const bool shape = (dtype == 1 || dtype == 2 || dtype == 3) && (head_dim == 64 || head_dim == 128);
    return shape && gs >= 1 && gs <= kMaxGroupSeqs && group >= 1 && gs * group <= kGroupedMaxCols;
}

// Query columns a multi-token item may hold: with the tcgen05 consumer selected
// and a shape it takes, at most its 32, so every call of that shape runs on it
// (a token's result is then the same whichever other tokens share the call).
int grouped_max_cols(int dtype, int head_dim, int group) {
    const bool capable = (dtype == 1 && head_dim == 128) || dtype == 2 || dtype == 3;
    return g_grouped_consumer == PA_GROUPED_TCGEN05 && capable && group <= kU2Cols ? kU2Cols
                                                                                 : kGroupedMaxCols;
}

// The tcgen05 consumer takes bf16 at head_dim 128 and codes at 64 or 128.
bool grouped_is_tcgen05(int dtype, int head_dim, int gs, int group) {
    return (dtype == 1 || dtype == 2 || dtype == 3) && use_umma(dtype == 1 ? head_dim : 128, gs, group);
}

int grouped_ctas_per_sm(int dtype, int head_dim, int gs, int group) {
    if (grouped_is_tcgen05(dtype, head_dim, gs, group)) return PA_U2_CTAS;
    int cw = 1, nt = 1;
    grouped_shape(gs, group, &cw, &nt);
    return grouped_min_blocks(head_dim, cw, nt);
}

template <int D, typename TC = __nv_bfloat16>
static cudaError_t launch_grouped_d(const DecodeParams& p, int cw, int nt, int gs,
                                   const CUtensorMap& kmap, const CUtensorMap& vmap,
                                   cudaStream_t stream) {
    static_assert(PA_GROUPED_ONE_TILE_WARPS >= 1 && PA_GROUPED_ONE_TILE_WARPS <= 4,
                  "one-tile warps: 1 .. 4");
    if (nt == 1) {
        switch (cw) {
            case 1: return launch_grouped_t<D, 1, 1, TC>(p, kmap, vmap, gs, stream);
#if PA_GROUPED_ONE_TILE_WARPS >= 2
            case 2: return launch_grouped_t<D, 2, 1, TC>(p, kmap, vmap, gs, stream);
#endif
#if PA_GROUPED_ONE_TILE_WARPS >= 3
            case 3: return launch_grouped_t<D, 3, 1, TC>(p, kmap, vmap, gs, stream);
#endif
#if PA_GROUPED_ONE_TILE_WARPS >= 4
            case 4: return launch_grouped_t<D, 4, 1, TC>(p, kmap, vmap, gs, stream);
#endif
            default: return cudaErrorInvalidValue;
        }
    }
    switch (cw) {
        case 1: return launch_grouped_t<D, 1, 2, TC>(p, kmap, vmap, gs, stream);
        case 2: return launch_grouped_t<D, 2, 2, TC>(p, kmap, vmap, gs, stream);
        case 3: return launch_grouped_t<D, 3, 2, TC>(p, kmap, vmap, gs, stream);
        case 4: return launch_grouped_t<D, 4, 2, TC>(p, kmap, vmap, gs, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_grouped(const DecodeParams& p, int dtype, int head_dim, int gs,
                                  const CUtensorMap& kmap, const CUtensorMap& vmap,
                                  cudaStream_t stream) {
    if (grouped_is_tcgen05(dtype, head_dim, gs, p.num_heads / p.num_kv_heads)) {
        if (dtype == 2) return launch_umma_grouped<E4M3Code>(p, kmap, vmap, gs, stream);
        if (dtype == 3) return launch_umma_grouped<Int8Code>(p, kmap, vmap, gs, stream);
        return launch_umma_grouped<__nv_bfloat16>(p, kmap, vmap, gs, stream);
    }
    int cw = 1, nt = 1;
    grouped_shape(gs, p.num_heads / p.num_kv_heads, &cw, &nt);
    if (dtype == 2) return launch_grouped_d<128, E4M3Code>(p, cw, nt, gs, kmap, vmap, stream);
    if (dtype == 3) return launch_grouped_d<128, Int8Code>(p, cw, nt, gs, kmap, vmap, stream);
    return head_dim == 64 ? launch_grouped_d<64>(p, cw, nt, gs, kmap, vmap, stream)
                          : launch_grouped_d<128>(p, cw, nt, gs, kmap, vmap, stream);
}



int set_grouped_consumer(int consumer) {
    const int prev = g_grouped_consumer;
    g_grouped_consumer = consumer;
    return prev;
}

cudaError_t read_status_tma(unsigned* bits, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(bits, s_status_tma, sizeof(unsigned));
    if (e != cudaSuccess || !clear) return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(s_status_tma, &zero, sizeof(unsigned));
}

}  // namespace pa
