// Symmetric INT8 row quantizers: per output channel (weights, optional
// SmoothQuant W * s) and per token (activations, optional X / s); and the FP8
// E4M3 quantizer per row or per tensor, which shares their row machinery.
//
// Source: "How quantization works", sections "The math of quantization"
// (s = max|x| / (2^(b-1) - 1), q = clamp(round(x/s), -2^(b-1), 2^(b-1)-1)),
// the quant.py listing (absmax clamped at 1e-8), q8_per_row and SmoothQuant's
// "Xs, Ws = X / s, W * s" in "Activation quantization and outliers";
// "Quantization: Smaller Weights, Same Answers (Mostly)", Quick Reference
// (per-token dynamic activation scales).  FP8: "How quantization works",
// quant.py fake_quant_fp8 (scale = max|w| / 448, then the cast to E4M3);
// "Quantization from Scratch", Formats, and "Quantization: Smaller Weights,
// Same Answers (Mostly)", "What about FP8, MXFP4, NVFP4 and GGUF?" (E4M3
// reaches +-448).
//
// One CTA of 256 threads per row.  Each thread owns 16-byte chunks of 8 fp16
// values; for K <= 16384 the (smoothed) row stays in registers between the
// absmax pass and the quantize pass, so HBM sees 2 B read + 1 B written per
// element.  Rows of 8192 < K <= 16384 are split over a cluster of two CTAs
// (the partial maxima meet in distributed shared memory); longer rows are read
// twice (the second read hits L2).
#include "sm100.cuh"
#include "wq_device.cuh"
#include "wq_host.h"

#include <algorithm>

namespace wq {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 8;                         // fp16 elements per 16-byte chunk
constexpr int kRowStep = kThreads * kChunk;       // elements per pass over the CTA

enum Mode { kPlain = 0, kMul = 1, kDiv = 2 };

template <int MODE>
__device__ __forceinline__ void smooth8(float (&v)[8], const float *__restrict__ smooth, int k) {
    if (MODE == kPlain) return;
    const float4 a = __ldg(reinterpret_cast<const float4 *>(smooth + k));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(smooth + k + 4));
    const float s[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    if (MODE == kMul) {
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const float2 p = __fmul2_rn(make_float2(v[e], v[e + 1]), make_float2(s[e], s[e + 1]));
            v[e] = p.x;
            v[e + 1] = p.y;
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = __fdiv_rn(v[e], s[e]);
    }
}

__device__ __forceinline__ void unpack8(const uint4 r, float (&v)[8]) {
    const float2 a = half2_bits_to_float2(r.x), b = half2_bits_to_float2(r.y);
    const float2 c = half2_bits_to_float2(r.z), d = half2_bits_to_float2(r.w);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    v[4] = c.x; v[5] = c.y; v[6] = d.x; v[7] = d.y;
}

__device__ __forceinline__ void load8(const uint16_t *p, float (&v)[8]) {
    const uint4 r = ld_stream_u4(p);
    const float2 a = half2_bits_to_float2(r.x), b = half2_bits_to_float2(r.y);
    const float2 c = half2_bits_to_float2(r.z), d = half2_bits_to_float2(r.w);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    v[4] = c.x; v[5] = c.y; v[6] = d.x; v[7] = d.y;
}

// |v / s| <= 127 (1 + 2^-23) < 2^8 (E = 7): the codes equal rne(fl(v / s)).  Pairs are
// decided with f32x2 fused arithmetic on the exact product t = v * RN(1/s):
// r = RN(t + 1.5*2^23) (rne(t) lands in r's low mantissa bits), d = RN(t - (r - 1.5*2^23)).
// rne(t) is rne(v / s) unless |d| comes within the guard band of 1/2 (t is within 2^(E-23)
// of v / s, so a band of 2^-13 suffices); a chunk with such a near-tie is redone with
// rne_quotient (IEEE quotient).  No clamp is needed: s = RN(a / 127) with a = max |v| over
// the same values, so |v| * RN(1/s) <= 127 (1 + 2^-22) and every code lies in [-127, 127].
__device__ __forceinline__ uint32_t pair_rne8(float a, float b, float rs, uint32_t &bad) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    constexpr float kGuardSq = (0.5f - 0x1p-13f) * (0.5f - 0x1p-13f);
    const float2 v = make_float2(a, b), r2 = make_float2(rs, rs);
    const float2 r = __ffma2_rn(v, r2, make_float2(kMagic, kMagic));
    const float2 n = __fadd2_rn(r, make_float2(-kMagic, -kMagic));
    const float2 d = __ffma2_rn(v, r2, make_float2(-n.x, -n.y));
    const float2 e = __ffma2_rn(d, make_float2(-d.x, -d.y), make_float2(kGuardSq, kGuardSq));
    bad |= __float_as_uint(e.x) | __float_as_uint(e.y);
    return __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x5410);  // int16x2 rne(t)
}

__device__ __forceinline__ uint2 quant8(const float (&v)[8], float s, float rs) {
    uint32_t bad = 0;
    uint32_t p0 = pair_rne8(v[0], v[1], rs, bad), p1 = pair_rne8(v[2], v[3], rs, bad);
    uint32_t p2 = pair_rne8(v[4], v[5], rs, bad), p3 = pair_rne8(v[6], v[7], rs, bad);
    if (bad >> 31) {  // a near-tie: the IEEE quotient decides every code of this chunk
        uint32_t c[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) c[e] = (uint32_t)rne_quotient<7>(v[e], s, rs) & 0xFFFFu;
        p0 = c[0] | (c[1] << 16); p1 = c[2] | (c[3] << 16); p2 = c[4] | (c[5] << 16); p3 = c[6] | (c[7] << 16);
    }
    // low byte of every 16-bit lane, in element order
    return make_uint2(__byte_perm(p0, p1, 0x6420), __byte_perm(p2, p3, 0x6420));
}

enum Format { kInt8 = 0, kE4M3 = 1 };

// Two fp32 values to E4M3 (round to nearest even, saturating at +-448); `lo` lands in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// E4M3 codes of v / s for one chunk: e4m3_rn(fl(v / s)).  t = RN(v * RN(1/s)) is within
// 1.5 * 2^-23 |t| of v / s and fl(v / s) within 2^-24 of v / s, so fl(v / s) lies in
// [t (1 - 2^-21), t (1 + 2^-21)], which the two products t (1 -+ 2^-20) enclose even after
// their own rounding.  Rounding to E4M3 is monotone: when both ends give the same code, so
// does fl(v / s).  Otherwise (v / s next to an E4M3 midpoint, rare) the chunk is redone from
// the IEEE quotient.  Saturation never applies: |v / s| <= 448 (1 + 2^-22) rounds to 448.
__device__ __forceinline__ uint2 quant8_e4m3(const float (&v)[8], float s, float rs) {
    constexpr float kDown = 1.0f - 0x1p-20f, kUp = 1.0f + 0x1p-20f;
    uint32_t c[4], bad = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float2 t = __fmul2_rn(make_float2(v[2 * p], v[2 * p + 1]), make_float2(rs, rs));
        const float2 a = __fmul2_rn(t, make_float2(kDown, kDown));
        const float2 b = __fmul2_rn(t, make_float2(kUp, kUp));
        c[p] = cvt_e4m3x2(a.x, a.y);
        bad |= c[p] ^ cvt_e4m3x2(b.x, b.y);
    }
    if (bad) {
#pragma unroll
        for (int p = 0; p < 4; ++p) c[p] = cvt_e4m3x2(__fdiv_rn(v[2 * p], s), __fdiv_rn(v[2 * p + 1], s));
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

template <int FMT>
struct FormatTraits;
template <>
struct FormatTraits<kInt8> {
    static constexpr float kMax = 127.0f;  // 2^(b-1) - 1
    __device__ static uint2 chunk(const float (&v)[8], float s, float rs) { return quant8(v, s, rs); }
};
template <>
struct FormatTraits<kE4M3> {
    static constexpr float kMax = 448.0f;  // largest finite E4M3 value
    __device__ static uint2 chunk(const float (&v)[8], float s, float rs) { return quant8_e4m3(v, s, rs); }
};

template <int T = kThreads>
__device__ __forceinline__ float block_max(float a, float *red) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[warp] = a;
    __syncthreads();
    float m = red[0];
#pragma unroll
    for (int i = 1; i < T / 32; ++i) m = fmaxf(m, red[i]);
    return m;
}

// NCH > 0: the row is kept in registers (K <= NCH * 2048).  NCH == 0: two passes.
// tensor_amax (FP8 per tensor): the tensor's max |x| (float bits), used instead of the
// row's; the scale is then written by finish_tensor_scale_kernel, not here.
// T threads per row (256, or 512 for the X / s rows of 4096 < K <= 8192: measured on B200,
// twice the threads per row hide the IEEE division better there and nowhere else).
template <int NCH, int MODE, int FMT = kInt8, int T = kThreads>
__global__ void __launch_bounds__(T) quant_int8_rows_kernel(const uint16_t *__restrict__ x, int K,
                                                                   const float *__restrict__ smooth,
                                                                   int8_t *__restrict__ q,
                                                                   float *__restrict__ scales,
                                                                   const unsigned int *__restrict__ tensor_amax = nullptr) {
    using F = FormatTraits<FMT>;
    constexpr int kRowStep = T * kChunk;
    __shared__ float red[T / 32];
    const size_t row = blockIdx.x;
    const uint16_t *xr = x + row * K;
    int8_t *qr = q + row * K;
    const int t0 = threadIdx.x * kChunk;
    float amax = 0.0f;
    if (NCH > 0 && MODE != kDiv) {
        // The row stays in registers as fp16 (half the registers of fp32, so more rows are in
        // flight per SM); the conversion (and W * s) is redone in the second pass.
        uint4 raw[NCH > 0 ? NCH : 1];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = c * kRowStep + t0;
            raw[c] = k < K ? ld_stream_u4(xr + k) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = c * kRowStep + t0;
            if (k < K) {
                float v[8];
                unpack8(raw[c], v);
                smooth8<MODE>(v, smooth, k);
#pragma unroll
                for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
            }
        }
        const float a = fmaxf(tensor_amax ? __uint_as_float(*tensor_amax) : block_max<T>(amax, red), 1e-8f);
        const float s = __fdiv_rn(a, F::kMax);
        const float rs = __frcp_rn(s);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = c * kRowStep + t0;
            if (k < K) {
                float v[8];
                unpack8(raw[c], v);
                smooth8<MODE>(v, smooth, k);
                *reinterpret_cast<uint2 *>(qr + k) = F::chunk(v, s, rs);
            }
        }
        if (threadIdx.x == 0 && !tensor_amax) scales[row] = s;
    } else if (NCH > 0) {
        float v[NCH > 0 ? NCH : 1][8];
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = c * kRowStep + t0;
            if (k < K) {
                load8(xr + k, v[c]);
                smooth8<MODE>(v[c], smooth, k);
#pragma unroll
                for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[c][e]));
            }
        }
        const float a = fmaxf(tensor_amax ? __uint_as_float(*tensor_amax) : block_max<T>(amax, red), 1e-8f);
        const float s = __fdiv_rn(a, F::kMax);
        const float rs = __frcp_rn(s);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = c * kRowStep + t0;
            if (k < K) *reinterpret_cast<uint2 *>(qr + k) = F::chunk(v[c], s, rs);
        }
        if (threadIdx.x == 0 && !tensor_amax) scales[row] = s;
    } else {
        // Two passes over the row: the first pass keeps its lines in L2 (evict-last policy)
        // so that the second pass, the lines' last use (evict-first), hits L2.  Without the
        // hint most second-pass reads went back to DRAM (ncu: 1.9x the algorithmic bytes).
        uint64_t keep, drop;
        asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
        asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(drop));
        // W * s rows take four 16-byte loads per thread and step (each chunk also loads its
        // smoothing factors, so a step costs one round trip, not four: 8192x28672 on B200
        // 180.7 -> 164.3 us); the other modes keep one load per step, which measured faster
        // there (more CTAs per SM at fewer registers).
        auto load_hint = [&](int k, uint64_t pol) {
            uint4 r;
            asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                         : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(xr + k), "l"(pol));
            return r;
        };
        constexpr int U = MODE == kMul ? 4 : 1;
        for (int k0 = t0; k0 < K; k0 += U * kRowStep) {
            uint4 r[U];
#pragma unroll
            for (int u = 0; u < U; ++u) r[u] = k0 + u * kRowStep < K ? load_hint(k0 + u * kRowStep, keep) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = k0 + u * kRowStep;
                if (k < K) {
                    float v[8];
                    unpack8(r[u], v);
                    smooth8<MODE>(v, smooth, k);
#pragma unroll
                    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
                }
            }
        }
        const float a = fmaxf(tensor_amax ? __uint_as_float(*tensor_amax) : block_max<T>(amax, red), 1e-8f);
        const float s = __fdiv_rn(a, F::kMax);
        const float rs = __frcp_rn(s);
        for (int k0 = t0; k0 < K; k0 += U * kRowStep) {
            uint4 r[U];  // L2-resident re-reads, last use
#pragma unroll
            for (int u = 0; u < U; ++u) r[u] = k0 + u * kRowStep < K ? load_hint(k0 + u * kRowStep, drop) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = k0 + u * kRowStep;
                if (k < K) {
                    float v[8];
                    unpack8(r[u], v);
                    smooth8<MODE>(v, smooth, k);
                    *reinterpret_cast<uint2 *>(qr + k) = F::chunk(v, s, rs);
                }
            }
        }
        if (threadIdx.x == 0 && !tensor_amax) scales[row] = s;
    }
}

// 8192 < K <= 16384: a row is split over a cluster of C = 2 CTAs (at most 8192
// columns each), each keeping its part in registers with at most 4 chunks per thread (as fp16
// bits, converted and smoothed again for the codes; fp32 for X / s, whose division is not worth
// doing twice); the partial maxima are exchanged through distributed shared memory, so HBM
// sees each element once.  Every CTA signals the cluster barrier on entry and waits on it
// before its first store into a peer's shared memory, so no store reaches a CTA that has not
// started.
template <int C, int MODE, int FMT = kInt8>
__global__ void __launch_bounds__(kThreads) quant_int8_rows_cluster_kernel(const uint16_t *__restrict__ x, int K,
                                                                           const float *__restrict__ smooth,
                                                                           int8_t *__restrict__ q,
                                                                           float *__restrict__ scales) {
    constexpr int NCH = 4;
    constexpr bool RAW = MODE != kDiv;
    __shared__ float red[kThreads / 32];
    __shared__ float part_max[C];
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    const size_t row = blockIdx.y;
    const uint32_t rank = sm100::cluster_ctarank();  // cluster (C, 1, 1) along x
    const int part = K / C;                          // K % (8 C) == 0: whole chunks per CTA
    const int kb = (int)rank * part;
    const uint16_t *xr = x + row * K + kb;
    int8_t *qr = q + row * K + kb;
    const int t0 = threadIdx.x * kChunk;
    float amax = 0.0f;
    uint4 raw[RAW ? NCH : 1];
    float v[RAW ? 1 : NCH][8];
    if (RAW) {
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = c * kRowStep + t0;
            raw[c] = k < part ? ld_stream_u4(xr + k) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = c * kRowStep + t0;
            if (k < part) {
                float w[8];
                unpack8(raw[c], w);
                smooth8<MODE>(w, smooth, kb + k);
#pragma unroll
                for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(w[e]));
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int k = c * kRowStep + t0;
            if (k < part) {
                load8(xr + k, v[c]);
                smooth8<MODE>(v[c], smooth, kb + k);
#pragma unroll
                for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[c][e]));
            }
        }
    }
    const float mine = block_max(amax, red);
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // every CTA of the cluster has started
    if (threadIdx.x < C) {  // this CTA's maximum into slot `rank` of every CTA of the cluster
        const uint32_t slot = sm100::smem_u32(&part_max[rank]);
        asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(sm100::mapa_shared(slot, threadIdx.x)), "f"(mine)
                     : "memory");
    }
    sm100::cluster_sync();
    float a = part_max[0];
#pragma unroll
    for (int c = 1; c < C; ++c) a = fmaxf(a, part_max[c]);
    a = fmaxf(a, 1e-8f);
    const float s = __fdiv_rn(a, FormatTraits<FMT>::kMax);
    const float rs = __frcp_rn(s);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int k = c * kRowStep + t0;
        if (k < part) {
            if (RAW) {
                float w[8];
                unpack8(raw[c], w);
                smooth8<MODE>(w, smooth, kb + k);
                *reinterpret_cast<uint2 *>(qr + k) = FormatTraits<FMT>::chunk(w, s, rs);
            } else {
                *reinterpret_cast<uint2 *>(qr + k) = FormatTraits<FMT>::chunk(v[RAW ? 0 : c], s, rs);
            }
        }
    }
    if (threadIdx.x == 0 && rank == 0) scales[row] = s;
}

template <int C, int MODE, int FMT = kInt8>
cudaError_t launch_cluster(const uint16_t *x, int R, int K, const float *smooth, int8_t *q, float *scales,
                           cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, R, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, quant_int8_rows_cluster_kernel<C, MODE, FMT>, x, K, smooth, q, scales);
}

template <int MODE, int FMT = kInt8>
cudaError_t launch_mode(const uint16_t *x, int R, int K, const float *smooth, int8_t *q, float *scales,
                        cudaStream_t st, const unsigned int *tensor_amax = nullptr) {
    const int nch = (K + kRowStep - 1) / kRowStep;
    // Measured on B200: pairs beat the 8-chunk single CTA (4096x16384: 59.7 -> 45.6 us with the
    // pair's rows kept as fp16); for longer rows the two-pass kernel (second read from L2) beats
    // clusters of 4 (8192x28672: 129.5 against 155.9 us) or 8.
    if (!tensor_amax && nch > 4 && nch <= 8 && R < 65536 && K % 16 == 0)
        return launch_cluster<2, MODE, FMT>(x, R, K, smooth, q, scales, st);
    dim3 grid(R), block(kThreads);
    if (MODE == kDiv && !tensor_amax && K > 4096 && K <= 8192) {
        quant_int8_rows_kernel<2, MODE, FMT, 512><<<grid, dim3(512), 0, st>>>(x, K, smooth, q, scales, tensor_amax);
        return cudaGetLastError();
    }
    if (nch <= 1)
        quant_int8_rows_kernel<1, MODE, FMT><<<grid, block, 0, st>>>(x, K, smooth, q, scales, tensor_amax);
    else if (nch <= 2)
        quant_int8_rows_kernel<2, MODE, FMT><<<grid, block, 0, st>>>(x, K, smooth, q, scales, tensor_amax);
    else if (nch <= 4)
        quant_int8_rows_kernel<4, MODE, FMT><<<grid, block, 0, st>>>(x, K, smooth, q, scales, tensor_amax);
    else if (nch <= 8)
        quant_int8_rows_kernel<8, MODE, FMT><<<grid, block, 0, st>>>(x, K, smooth, q, scales, tensor_amax);
    else
        quant_int8_rows_kernel<0, MODE, FMT><<<grid, block, 0, st>>>(x, K, smooth, q, scales, tensor_amax);
    return cudaGetLastError();
}

// Per-tensor FP8: the tensor's max |x| by atomicMax on the float bits (non-negative floats
// order like their bit patterns) into the scale slot, which the call clears first.
__global__ void __launch_bounds__(kThreads) tensor_absmax_kernel(const uint16_t *__restrict__ x, size_t n8,
                                                                 unsigned int *__restrict__ amax) {
    __shared__ float red[kThreads / 32];
    float m = 0.0f;
    for (size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x; i < n8; i += (size_t)gridDim.x * kThreads) {
        float v[8];
        load8(x + 8 * i, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
    }
    m = block_max(m, red);
    if (threadIdx.x == 0) atomicMax(amax, __float_as_uint(m));
}

// Turns the tensor's max |x| into its scale once every row has been quantized with it.
__global__ void finish_tensor_scale_kernel(float *scale) {
    *scale = __fdiv_rn(fmaxf(*scale, 1e-8f), 448.0f);
}

wq_status quantize_rows(const char *name, const uint16_t *x, int R, int K, const float *smooth, int mode,
                        int8_t *q, float *scales, void *stream) {
    WQ_REQUIRE_PTR(x, "input");
    WQ_REQUIRE_PTR(q, "q");
    WQ_REQUIRE_PTR(scales, "scales");
    if (smooth) WQ_REQUIRE(aligned16(smooth), WQ_ERR_ALIGNMENT, "smooth is not 16-byte aligned");
    WQ_REQUIRE(R > 0 && K > 0, WQ_ERR_INVALID_ARG, "%s: sizes must be positive (rows=%d K=%d)", name, R, K);
    WQ_REQUIRE(K % 16 == 0, WQ_ERR_UNSUPPORTED, "%s: K (%d) must be a multiple of 16", name, K);
    WQ_REQUIRE(R < (1 << 30), WQ_ERR_UNSUPPORTED, "%s: too many rows", name);
    cudaStream_t st = as_stream(stream);
    cudaError_t e;
    if (!smooth)
        e = launch_mode<kPlain>(x, R, K, nullptr, q, scales, st);
    else if (mode == kMul)
        e = launch_mode<kMul>(x, R, K, smooth, q, scales, st);
    else
        e = launch_mode<kDiv>(x, R, K, smooth, q, scales, st);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: launch failed: %s", name, cudaGetErrorString(e));
    return WQ_OK;
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_quantize_int8_per_channel(const uint16_t *w, int N, int K, const float *smooth,
                                                  int8_t *q, float *scales, void *stream) {
    return wq::quantize_rows("wq_quantize_int8_per_channel", w, N, K, smooth, wq::kMul, q, scales, stream);
}

extern "C" wq_status wq_quantize_int8_per_token(const uint16_t *x, int M, int K, const float *smooth,
                                                int8_t *q, float *scales, void *stream) {
    return wq::quantize_rows("wq_quantize_int8_per_token", x, M, K, smooth, wq::kDiv, q, scales, stream);
}

extern "C" wq_status wq_quantize_fp8_e4m3(const uint16_t *x, int R, int K, int per_row, uint8_t *q, float *scales,
                                          void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(x, "input");
    WQ_REQUIRE_PTR(q, "q");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE(R > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_quantize_fp8_e4m3: sizes must be positive (rows=%d K=%d)",
               R, K);
    WQ_REQUIRE(K % 16 == 0, WQ_ERR_UNSUPPORTED, "wq_quantize_fp8_e4m3: K (%d) must be a multiple of 16", K);
    WQ_REQUIRE(R < (1 << 30), WQ_ERR_UNSUPPORTED, "wq_quantize_fp8_e4m3: too many rows");
    cudaStream_t st = as_stream(stream);
    int8_t *q8 = reinterpret_cast<int8_t *>(q);
    cudaError_t e;
    if (per_row) {
        e = launch_mode<kPlain, kE4M3>(x, R, K, nullptr, q8, scales, st);
    } else {
        unsigned int *amax = reinterpret_cast<unsigned int *>(scales);
        e = cudaMemsetAsync(amax, 0, sizeof(unsigned int), st);
        if (e == cudaSuccess) {
            const size_t n8 = (size_t)R * K / 8;
            const size_t want = (n8 + kThreads - 1) / kThreads;
            const int grid = (int)std::min<size_t>(want, (size_t)num_sms() * 8);
            tensor_absmax_kernel<<<grid, kThreads, 0, st>>>(x, n8, amax);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = launch_mode<kPlain, kE4M3>(x, R, K, nullptr, q8, scales, st, amax);
        if (e == cudaSuccess) {
            finish_tensor_scale_kernel<<<1, 1, 0, st>>>(scales);
            e = cudaGetLastError();
        }
    }
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_quantize_fp8_e4m3: launch failed: %s", cudaGetErrorString(e));
    return WQ_OK;
}
