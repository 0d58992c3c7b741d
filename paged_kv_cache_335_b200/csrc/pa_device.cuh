// pa_device.cuh — device helpers shared by the paged-attention kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_internal.h"

namespace pa {

// 16-byte streaming load from global memory: read-only path, no L1 allocation
// (every K/V byte is read exactly once per call).
__device__ __forceinline__ uint4 ld_stream(const void* ptr) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(ptr));
    return r;
}

// Plain 16-byte load (may be cached in L1).
__device__ __forceinline__ uint4 ld_v4(const void* ptr) {
    return *reinterpret_cast<const uint4*>(ptr);
}

__device__ __forceinline__ void st_v4(void* ptr, uint4 v) {
    *reinterpret_cast<uint4*>(ptr) = v;
}

// bf16 pair in one 32-bit word -> two floats (exact: bf16 is the upper half of binary32).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}

// Element traits: how many elements one 16-byte chunk holds and how to widen them.
template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kVec = 4;
    __device__ __forceinline__ static void widen(const uint4& c, float (&f)[4]) {
        f[0] = __uint_as_float(c.x);
        f[1] = __uint_as_float(c.y);
        f[2] = __uint_as_float(c.z);
        f[3] = __uint_as_float(c.w);
    }
    __device__ __forceinline__ static void store(void* base, int64_t idx, float v) {
        reinterpret_cast<float*>(base)[idx] = v;
    }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void widen(const uint4& c, float (&f)[8]) {
        f[0] = bf16_lo(c.x); f[1] = bf16_hi(c.x);
        f[2] = bf16_lo(c.y); f[3] = bf16_hi(c.y);
        f[4] = bf16_lo(c.z); f[5] = bf16_hi(c.z);
        f[6] = bf16_lo(c.w); f[7] = bf16_hi(c.w);
    }
    __device__ __forceinline__ static void store(void* base, int64_t idx, float v) {
        reinterpret_cast<uint16_t*>(base)[idx] = float_to_bf16_bits(v);
    }
};

// Quantised cache codes (one byte per element; the value is code value x the
// kv head's scale, applied by the caller of widen): tag types for Elem.
struct E4M3Code {};
struct Int8Code {};

// Two FP8 E4M3 codes (low byte first) -> two floats, by the hardware
// conversion to f16x2 (exact: every E4M3 value, NaN included, is an f16).
__device__ __forceinline__ void e4m3x2_to_float2(uint32_t two, float& lo, float& hi) {
    uint32_t h2;
    asm("{\n\t.reg .b16 t;\n\tmov.b16 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h2) : "h"((unsigned short)two));
    const __half2 v = *reinterpret_cast<const __half2*>(&h2);
    lo = __low2float(v);
    hi = __high2float(v);
}

template <>
struct Elem<E4M3Code> {
    static constexpr int kVec = 16;
    __device__ __forceinline__ static void widen(const uint4& c, float (&f)[16]) {
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            e4m3x2_to_float2(w[i] & 0xffffu, f[4 * i], f[4 * i + 1]);
            e4m3x2_to_float2(w[i] >> 16, f[4 * i + 2], f[4 * i + 3]);
        }
    }
};

// Int8 codes -> floats without an integer conversion: with the sign bit
// flipped, byte b is u = code + 128 in [0, 255]; one byte permute places it
// as the low mantissa byte of 2^23 (bits 0x4B0000uu = 2^23 + u exactly) and
// one subtraction of 2^23 + 128 leaves the code, exactly.
template <>
struct Elem<Int8Code> {
    static constexpr int kVec = 16;
    __device__ __forceinline__ static void widen(const uint4& c, float (&f)[16]) {
        const uint32_t w[4] = {c.x ^ 0x80808080u, c.y ^ 0x80808080u, c.z ^ 0x80808080u,
                               c.w ^ 0x80808080u};
        constexpr float kBias = 8388736.0f;  // 2^23 + 128
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[4 * i + 0] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540)) - kBias;
            f[4 * i + 1] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7541)) - kBias;
            f[4 * i + 2] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7542)) - kBias;
            f[4 * i + 3] = __uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7543)) - kBias;
        }
    }
};

// Int8 codes -> floats biased by 1152: with the sign bit flipped, byte b is
// u = code + 128; one byte permute per two codes places u under the f16
// exponent of 1024 (f16 bits 0x64uu = 1024 + u exactly), and the f16 -> f32
// widening gives 1152 + code, exactly. The caller removes the bias once per
// sum (bias x the sum of the weights) instead of once per code.
constexpr float kInt8WidenBias = 1152.0f;
__device__ __forceinline__ void int8_widen_biased(const uint4& c, float (&f)[16]) {
    const uint32_t w[4] = {c.x ^ 0x80808080u, c.y ^ 0x80808080u, c.z ^ 0x80808080u,
                           c.w ^ 0x80808080u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t h01 = __byte_perm(w[i], 0x64646464u, 0x5140);  // f16x2 (1024 + u0, 1024 + u1)
        const uint32_t h23 = __byte_perm(w[i], 0x64646464u, 0x5342);
        const __half2 a = *reinterpret_cast<const __half2*>(&h01);
        const __half2 b = *reinterpret_cast<const __half2*>(&h23);
        f[4 * i + 0] = __low2float(a);
        f[4 * i + 1] = __high2float(a);
        f[4 * i + 2] = __low2float(b);
        f[4 * i + 3] = __high2float(b);
    }
}

// q / out element type for a cache element type (quantised caches: bf16).
template <typename TC> struct QType { using type = TC; };
template <> struct QType<E4M3Code> { using type = __nv_bfloat16; };
template <> struct QType<Int8Code> { using type = __nv_bfloat16; };

}  // namespace pa
