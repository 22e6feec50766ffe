// Device-side helpers shared by the kernels: vector loads with explicit
// cache hints and fp16 bit handling.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace wq {

// 16-byte streaming load that bypasses L1 (data read exactly once).
__device__ __forceinline__ uint4 ld_stream_u4(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// 16-byte read-only load through L1 (data shared by many warps of an SM).
__device__ __forceinline__ uint4 ld_shared_ro_u4(const void *p) {
    uint4 r;
    asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream_u4(void *p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
    return __half2float(__ushort_as_half(b));
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t b) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&b));
}

__device__ __forceinline__ uint16_t float_to_half_bits_rn(float f) {
    return __half_as_ushort(__float2half_rn(f));
}

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return min(max(v, lo), hi); }

}  // namespace wq
