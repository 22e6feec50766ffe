// Device-side helpers shared by the kernels: vector loads with explicit
// cache hints and fp16 bit handling.
#pragma once

#include <cuda_bf16.h>
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

__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
    return __half2float(__ushort_as_half(b));
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t b) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&b));
}

__device__ __forceinline__ uint16_t float_to_half_bits_rn(float f) {
    return __half_as_ushort(__float2half_rn(f));
}

__device__ __forceinline__ uint16_t float_to_bf16_bits_rn(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return min(max(v, lo), hi); }

// rne(fl(a / b)) -- the integer that rounding the IEEE fp32 quotient to the
// nearest (ties to even) gives -- for |a / b| < 2^(E+1), with y = RN(1/b).
// q = RN(a * y) has relative error below 2^-23 + 2^-48, so |q - a/b| <
// 2^(E-22) and |fl(a/b) - a/b| <= 2^(E-24); both lie on the same side of every
// half-integer that q is more than `guard` = 2^(E-21) away from, and then
// round to the same integer.  Otherwise (a near-tie, rare) the correctly
// rounded quotient decides.  q - rint(q) and its distance to 0.5 are exact
// (Sterbenz), so the test itself does not round.
template <int E>
__device__ __forceinline__ int rne_quotient(float a, float b, float y) {
    constexpr float guard = E >= 21 ? 1.0f : 1.0f / (float)(1u << (21 - E));
    const float q = __fmul_rn(a, y);
    const float n = rintf(q);
    if (fabsf(fabsf(__fsub_rn(q, n)) - 0.5f) <= guard) return __float2int_rn(__fdiv_rn(a, b));
    return __float2int_rn(n);
}

}  // namespace wq
