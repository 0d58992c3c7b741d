// pa_device.cuh — device helpers shared by the paged-attention kernels.
#pragma once

#include <cuda_bf16.h>
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

}  // namespace pa
