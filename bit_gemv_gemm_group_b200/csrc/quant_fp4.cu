// Block-scaled FP4 quantizers: MXFP4 (E2M1, blocks of 32 sharing an E8M0
// power-of-two scale) and NVFP4 (E2M1, blocks of 16 with an E4M3 scale per
// block over one fp32 scale per tensor).
//
// Source: "Quantization: Smaller Weights, Same Answers (Mostly)", "What about
// FP8, MXFP4, NVFP4 and GGUF?" (MXFP4: blocks of 32 four-bit floats sharing
// one 8-bit power-of-two scale; NVFP4: blocks of 16, an FP8 scale per block
// plus one FP32 scale per tensor); "Quantization from Scratch", Formats (MX
// formats: blocks of 32 share one 8-bit power-of-two scale); "How
// quantization works", Mainstream schemes (FP4 on Blackwell).
//
//   MXFP4: e = floor(log2 max|v|) - 2 (E8M0 code e + 127; 0 for an all-zero
//          block), q = e2m1_rn(v * 2^-e) -- an exact scaling, then one
//          rounding (cvt ... e2m1x2, saturating at +-6).
//   NVFP4: S = max(max|v| over the tensor, 1e-8) / 2688 (= 6 * 448);
//          per block b = e4m3_rn((max|v| / 6) / S), d = e4m3(b) * S,
//          q = e2m1_rn(fl(v / d)) (all zero when b == 0).
//
// One thread per block: 64 (MX) or 32 (NV) bytes in, 16 or 8 bytes of packed
// codes (element 2i in the low nibble of byte i) and one scale byte out; HBM
// traffic is 2 B in + 0.5 B + one scale byte per block out, per element.
//
// The scale bytes are written in the layout the tensor cores read them in
// (tcgen05.cp of 512-byte atoms into tensor memory for the block-scaled MMA):
// rows in blocks of 128, a row's factors in groups of 4, one atom per (row
// block, group), atoms in row-block-major order; factor f of row r is byte
// 16 (r % 32) + 4 ((r / 32) % 4) + f % 4 of atom (r / 128, f / 4).  A GEMM
// stage then fetches its factors with one contiguous bulk copy per operand.
#include "wq_device.cuh"
#include "wq_host.h"

#include <algorithm>

namespace wq {
namespace {

constexpr int kThreads = 256;

// Byte offset of factor f of row r in the atom layout; fg = groups of 4 factors per row.
__device__ __forceinline__ size_t sf_offset(int r, int f, int fg) {
    return ((size_t)(r >> 7) * fg + (f >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (f & 3);
}

// (row, factor) of block b = r F + f along a grid-stride loop, without a division per step.
struct BlockPos {
    int r, f, dr, df, F;
    __device__ BlockPos(size_t b0, size_t stride, int F_)
        : r((int)(b0 / F_)), f((int)(b0 % F_)), dr((int)(stride / F_)), df((int)(stride % F_)), F(F_) {}
    __device__ void advance() {
        r += dr;
        f += df;
        if (f >= F) {
            f -= F;
            ++r;
        }
    }
};

// Eight fp32 values to eight E2M1 codes (round to nearest even, saturating at +-6), element 0 in
// the low nibble.  cvt ... e2m1x2 puts its first operand in the high nibble of the byte.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

__device__ __forceinline__ void load8h(const uint16_t *p, float (&v)[8]) {
    const uint4 r = ld_stream_u4(p);
    const float2 a = half2_bits_to_float2(r.x), b = half2_bits_to_float2(r.y);
    const float2 c = half2_bits_to_float2(r.z), d = half2_bits_to_float2(r.w);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    v[4] = c.x; v[5] = c.y; v[6] = d.x; v[7] = d.y;
}

__device__ __forceinline__ float amax8(const float (&v)[8], float m) {
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
    return m;
}

__global__ void __launch_bounds__(kThreads) quant_mxfp4_kernel(const uint16_t *__restrict__ x, size_t nblocks, int F,
                                                               uint8_t *__restrict__ q, uint8_t *__restrict__ scales) {
    const int fg = (F + 3) / 4;
    const size_t stride = (size_t)gridDim.x * kThreads;
    BlockPos pos((size_t)blockIdx.x * kThreads + threadIdx.x, stride, F);
    for (size_t b = (size_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride, pos.advance()) {
        float v[4][8];
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            load8h(x + 32 * b + 8 * i, v[i]);
            a = amax8(v[i], a);
        }
        // floor(log2 a) is the unbiased exponent of a (a >= 2^-24 is a normal fp32 when nonzero)
        const int e = a > 0.0f ? (int)((__float_as_uint(a) >> 23) & 0xFF) - 127 - 2 : -127;
        const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, e in [-26, 13] here
        uint32_t c[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float t[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) t[k] = a > 0.0f ? v[i][k] * inv : 0.0f;  // exact
            c[i] = cvt_e2m1x8(t);
        }
        *reinterpret_cast<uint4 *>(q + 16 * b) = make_uint4(c[0], c[1], c[2], c[3]);
        scales[sf_offset(pos.r, pos.f, fg)] = (uint8_t)(e + 127);
    }
}

// Tensor max |x| into the tensor-scale word (float bits; cleared by the call first).
__global__ void __launch_bounds__(kThreads) tensor_absmax_fp4_kernel(const uint16_t *__restrict__ x, size_t n8,
                                                                     unsigned int *__restrict__ amax) {
    __shared__ float red[kThreads / 32];
    float m = 0.0f;
    for (size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x; i < n8; i += (size_t)gridDim.x * kThreads) {
        float v[8];
        load8h(x + 8 * i, v);
        m = amax8(v, m);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = red[0];
#pragma unroll
        for (int i = 1; i < kThreads / 32; ++i) t = fmaxf(t, red[i]);
        atomicMax(amax, __float_as_uint(t));
    }
}

// E4M3 byte to float (exact); the byte is placed in both lanes of the pair conversion.
__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}"
        : "=r"(h)
        : "r"(code * 0x101u));
    return half_bits_to_float((uint16_t)(h & 0xFFFFu));
}

// Float to E4M3 (round to nearest even, saturating at +-448); both lanes convert v.
__device__ __forceinline__ uint32_t float_to_e4m3(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(v), "f"(v));
    return r & 0xFFu;
}

// RN(a / 6) for an fp16 value a >= 0 (a block's max |v|): a = m 2^e with an 11-bit integer m,
// and m / 3 is either exact or k + r / 3 (r = 1, 2), whose binary tail repeats 01 or 10, so the
// quotient never lies within an fp32 ulp / 6 of a rounding boundary; the fp64 product with
// RN64(1/6) is within 2^-52 relative of it and rounds to the same fp32 value.
__device__ __forceinline__ float div6_rn(float a) {
    return __double2float_rn(__dmul_rn((double)a, 0x1.5555555555555p-3));
}

__global__ void __launch_bounds__(kThreads) quant_nvfp4_kernel(const uint16_t *__restrict__ x, size_t nblocks, int F,
                                                               const unsigned int *__restrict__ tensor_amax,
                                                               uint8_t *__restrict__ q, uint8_t *__restrict__ scales) {
    const int fg = (F + 3) / 4;
    const float S = __fdiv_rn(fmaxf(__uint_as_float(*tensor_amax), 1e-8f), 2688.0f);
    const float rS = __frcp_rn(S);
    constexpr float kDown = 1.0f - 0x1p-20f, kUp = 1.0f + 0x1p-20f;
    const size_t stride = (size_t)gridDim.x * kThreads;
    BlockPos pos((size_t)blockIdx.x * kThreads + threadIdx.x, stride, F);
    for (size_t b = (size_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride, pos.advance()) {
        const uint4 r0 = ld_stream_u4(x + 16 * b), r1 = ld_stream_u4(x + 16 * b + 8);
        // max |v| on the fp16 bits (non-negative fp16 order like their bit patterns)
        uint32_t m = __vmaxu2(__vmaxu2(r0.x & 0x7fff7fffu, r0.y & 0x7fff7fffu),
                              __vmaxu2(r0.z & 0x7fff7fffu, r0.w & 0x7fff7fffu));
        m = __vmaxu2(m, __vmaxu2(__vmaxu2(r1.x & 0x7fff7fffu, r1.y & 0x7fff7fffu),
                                 __vmaxu2(r1.z & 0x7fff7fffu, r1.w & 0x7fff7fffu)));
        const float a = half_bits_to_float((uint16_t)max(m & 0xffffu, m >> 16));
        // b = e4m3_rn(fl(fl(a / 6) / S)): t = RN(fl(a / 6) RN(1/S)) is within 1.5 2^-23 |t| of the
        // quotient, so fl(quotient) lies between t (1 -+ 2^-20); E4M3 rounding is monotone, so
        // where both ends give one code it is the code, else the IEEE quotient decides.
        const float a6 = div6_rn(a);
        const float t = __fmul_rn(a6, rS);
        uint32_t sb = float_to_e4m3(__fmul_rn(t, kDown));
        if (sb != float_to_e4m3(__fmul_rn(t, kUp))) sb = float_to_e4m3(__fdiv_rn(a6, S));
        const float d = __fmul_rn(e4m3_to_float(sb), S);
        uint32_t c[2] = {0u, 0u};
        if (sb != 0u) {
            // e2m1_rn(fl(v / d)): t = RN(v * RN(1/d)) and both t (1 -+ 2^-20) round to the same code
            // unless fl(v / d) sits next to an E2M1 midpoint; then the IEEE quotient decides.
            const float rd = __frcp_rn(d);
            const float2 rd2 = make_float2(rd, rd), dn = make_float2(kDown, kDown), up = make_float2(kUp, kUp);
            const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
            uint32_t bad = 0;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float lo[8], hi[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 tv = __fmul2_rn(half2_bits_to_float2(w[4 * i + k]), rd2);
                    const float2 l = __fmul2_rn(tv, dn), h = __fmul2_rn(tv, up);
                    lo[2 * k] = l.x;
                    lo[2 * k + 1] = l.y;
                    hi[2 * k] = h.x;
                    hi[2 * k + 1] = h.y;
                }
                c[i] = cvt_e2m1x8(lo);
                bad |= c[i] ^ cvt_e2m1x8(hi);
            }
            if (bad) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float tq[8];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 v = half2_bits_to_float2(w[4 * i + k]);
                        tq[2 * k] = __fdiv_rn(v.x, d);
                        tq[2 * k + 1] = __fdiv_rn(v.y, d);
                    }
                    c[i] = cvt_e2m1x8(tq);
                }
            }
        }
        *reinterpret_cast<uint2 *>(q + 8 * b) = make_uint2(c[0], c[1]);
        scales[sf_offset(pos.r, pos.f, fg)] = (uint8_t)sb;
    }
}

__global__ void finish_nvfp4_scale_kernel(float *tensor_scale) {
    *tensor_scale = __fdiv_rn(fmaxf(*tensor_scale, 1e-8f), 2688.0f);
}

int grid_for(size_t items) {
    return (int)std::max<size_t>(1, std::min<size_t>((items + kThreads - 1) / kThreads, (size_t)num_sms() * 8));
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_quantize_mxfp4(const uint16_t *x, int R, int K, uint8_t *q, uint8_t *scales, void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(q, "q");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE(R > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_quantize_mxfp4: sizes must be positive (rows=%d K=%d)", R, K);
    WQ_REQUIRE(K % 32 == 0, WQ_ERR_UNSUPPORTED, "wq_quantize_mxfp4: K (%d) must be a multiple of 32", K);
    WQ_REQUIRE(R < (1 << 30), WQ_ERR_UNSUPPORTED, "wq_quantize_mxfp4: too many rows");
    const size_t nblocks = (size_t)R * (K / 32);
    quant_mxfp4_kernel<<<grid_for(nblocks), kThreads, 0, as_stream(stream)>>>(x, nblocks, K / 32, q, scales);
    return check_launch("wq_quantize_mxfp4");
}

extern "C" wq_status wq_quantize_nvfp4(const uint16_t *x, int R, int K, uint8_t *q, uint8_t *scales,
                                       float *tensor_scale, void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(q, "q");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE_PTR(tensor_scale, "tensor_scale");
    WQ_REQUIRE(R > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_quantize_nvfp4: sizes must be positive (rows=%d K=%d)", R, K);
    WQ_REQUIRE(K % 16 == 0, WQ_ERR_UNSUPPORTED, "wq_quantize_nvfp4: K (%d) must be a multiple of 16", K);
    WQ_REQUIRE(R < (1 << 30), WQ_ERR_UNSUPPORTED, "wq_quantize_nvfp4: too many rows");
    cudaStream_t st = as_stream(stream);
    unsigned int *amax = reinterpret_cast<unsigned int *>(tensor_scale);
    cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), st);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_quantize_nvfp4: clearing the tensor scale failed");
    const size_t n8 = (size_t)R * K / 8, nblocks = (size_t)R * (K / 16);
    tensor_absmax_fp4_kernel<<<grid_for(n8), kThreads, 0, st>>>(x, n8, amax);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return fail(WQ_ERR_CUDA, "wq_quantize_nvfp4: launch failed: %s", cudaGetErrorString(e));
    quant_nvfp4_kernel<<<grid_for(nblocks), kThreads, 0, st>>>(x, nblocks, K / 16, amax, q, scales);
    if ((e = cudaGetLastError()) != cudaSuccess)
        return fail(WQ_ERR_CUDA, "wq_quantize_nvfp4: launch failed: %s", cudaGetErrorString(e));
    finish_nvfp4_scale_kernel<<<1, 1, 0, st>>>(tensor_scale);
    return check_launch("wq_quantize_nvfp4");
}

extern "C" size_t wq_fp4_scale_bytes(int R, int K, int nvfp4) {
    if (R <= 0 || K <= 0) return 0;
    const long long F = K / (nvfp4 ? 16 : 32);
    return (size_t)((R + 127) / 128) * (size_t)((F + 3) / 4) * 512;
}
