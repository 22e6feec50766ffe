// Asymmetric INT4 per-group quantizer: per-group min/max reduction with warp
// shuffles -> fp16 scale and 4-bit zero point -> round/clamp -> 8 codes per
// uint32.
//
// Source: "Quantization Explained: INT8, INT4, GPTQ and AWQ for LLMs",
// sections "Uniform Affine Quantization", "Scale and Zero-Point" and "Manual
// Group-Wise Quantizer"; "Quantization from Scratch", section "Scale and
// zero-point" and its round-to-nearest quantize() (zero scale -> 1); "How
// quantization works", section "Granularity" and exercise 2 (fp16 scale and
// 4-bit zero point per 128 weights).
//
// Work decomposition: one warp per (row, zero word) = 8 consecutive groups of
// one row.  Each lane owns 8 consecutive elements (one 16-byte load for fp16),
// so a group of G elements is handled by G/8 lanes and a warp covers 256/G
// groups per iteration.  All of a warp's loads are issued before any
// arithmetic (G/32 x 16 B in flight per lane) to keep HBM busy.  HBM bytes per
// weight: 2 (fp16 in) + 0.5 + 2.5/G (out).  The codes rne(w / s) are decided
// from w * RN(1/s) with an exact near-tie fallback (rne_quotient), which gives
// the same integers as the IEEE division at a third of its instructions.
#include <type_traits>

#include "wq_device.cuh"
#include "wq_host.h"

namespace wq {
namespace {

template <typename TIn>
struct Loader;

template <>
struct Loader<__half> {
    // 8 fp16 elements -> 8 floats
    static __device__ __forceinline__ void load8(const __half *p, float (&v)[8]) {
        uint4 r = ld_stream_u4(p);
        float2 a = half2_bits_to_float2(r.x), b = half2_bits_to_float2(r.y);
        float2 c = half2_bits_to_float2(r.z), d = half2_bits_to_float2(r.w);
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
        v[4] = c.x; v[5] = c.y; v[6] = d.x; v[7] = d.y;
    }
};

template <>
struct Loader<float> {
    static __device__ __forceinline__ void load8(const float *p, float (&v)[8]) {
        uint4 r0 = ld_stream_u4(p), r1 = ld_stream_u4(p + 4);
        v[0] = __uint_as_float(r0.x); v[1] = __uint_as_float(r0.y);
        v[2] = __uint_as_float(r0.z); v[3] = __uint_as_float(r0.w);
        v[4] = __uint_as_float(r1.x); v[5] = __uint_as_float(r1.y);
        v[6] = __uint_as_float(r1.z); v[7] = __uint_as_float(r1.w);
    }
};

template <typename TIn, int G>
__global__ void __launch_bounds__(256) quant_int4_group_kernel(const TIn *__restrict__ w, int N, int K,
                                                                uint32_t *__restrict__ qweight,
                                                                uint16_t *__restrict__ scales,
                                                                uint32_t *__restrict__ qzeros) {
    constexpr int LPG = G / 8;       // lanes per group
    constexpr int GPI = 32 / LPG;    // groups per warp iteration
    constexpr int ITERS = 8 / GPI;   // iterations per zero word (8 groups)
    const int groups = K / G;
    const int zwords = (groups + 7) / 8;
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (unit >= (long long)N * zwords) return;
    const int n = (int)(unit / zwords);
    const int zw = (int)(unit % zwords);
    const int sub = lane / LPG;  // group slot within an iteration
    const int li = lane % LPG;   // lane within the group

    // Issue every load of this warp first.
    float v[ITERS][8];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const int j = zw * 8 + it * GPI + sub;
        if (j < groups) {
            Loader<TIn>::load8(w + (size_t)n * K + (size_t)j * G + li * 8, v[it]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[it][e] = 0.0f;
        }
    }

    uint32_t zacc = 0;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const int j = zw * 8 + it * GPI + sub;
        // Range of the group, widened to contain 0.
        float lo = 0.0f, hi = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            lo = fminf(lo, v[it][e]);
            hi = fmaxf(hi, v[it][e]);
        }
#pragma unroll
        for (int off = LPG / 2; off >= 1; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        // s = fp16((hi - lo) / 15); a zero scale becomes 1.
        uint16_t s16 = float_to_half_bits_rn(__fdiv_rn(hi - lo, 15.0f));
        if (s16 == 0) s16 = 0x3c00;
        const float s = half_bits_to_float(s16);
        const float rs = __frcp_rn(s);
        // z = round(-lo / s) in [0, 15]; |-lo / s| and |w / s| stay below 32 (E = 4)
        const int z = clampi(rne_quotient<4>(-lo, s, rs), 0, 15);
        if (j < groups) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int q = clampi(rne_quotient<4>(v[it][e], s, rs) + z, 0, 15);
                word |= (uint32_t)q << (4 * e);
            }
            qweight[(size_t)n * (K / 8) + (size_t)j * (G / 8) + li] = word;
            if (li == 0) {
                scales[(size_t)n * groups + j] = s16;
                zacc |= (uint32_t)z << (4 * (j & 7));
            }
        }
    }
    const uint32_t zword = __reduce_or_sync(0xffffffffu, zacc);
    if (lane == 0) qzeros[(size_t)n * zwords + zw] = zword;
}

// ---------------------------------------------------------------------------
// fp16 input: the same decomposition with packed arithmetic.  The range comes
// from fp16x2 min/max on the raw bits (exact); a pair of codes is decided with
// f32x2 fused operations on the exact product w * RN(1/s):
//   r = RN(w * RN(1/s) + (1.5*2^23 + z))   (rne + z lands in r's low mantissa bits),
//   d = RN(w * RN(1/s) - (r - (1.5*2^23 + z)))   (within 2^-25 of the true remainder).
// w * RN(1/s) is within 2^-19 of w/s (|w/s| < 32), so the pair is exact unless
// |d| comes within 2^-16 of 1/2, in which case the lane recomputes its codes
// with the IEEE quotient.  Clamping (one min.relu.s16x2 per pair) and nibble
// packing run on 16-bit SIMD lanes.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t hmin2_bits(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hmax2_bits(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// rne(w * rs) + z of an fp16 pair as int16x2, with magic = 1.5 * 2^23 + z: one fused
// multiply-add rounds w * rs + magic to an integer, which is magic + rne(w * rs) away from a
// tie (at a tie the parity of z decides, and the guard band below catches it); `bad`
// collects the sign bit of (1/2 - 2^-16)^2 - d^2 (set when a lane lies in the guard band).
__device__ __forceinline__ uint32_t pair_rne(uint32_t h2, float rs, float magic, uint32_t &bad) {
    constexpr float kGuardSq = (0.5f - 0x1p-16f) * (0.5f - 0x1p-16f);
    const float2 f = half2_bits_to_float2(h2);
    const float2 r = __ffma2_rn(f, make_float2(rs, rs), make_float2(magic, magic));
    const float2 n = __fadd2_rn(r, make_float2(-magic, -magic));
    const float2 d = __ffma2_rn(f, make_float2(rs, rs), make_float2(-n.x, -n.y));
    const float2 e = __ffma2_rn(d, make_float2(-d.x, -d.y), make_float2(kGuardSq, kGuardSq));
    bad |= __float_as_uint(e.x) | __float_as_uint(e.y);
    return __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x5410);  // low 16 bits: rne(t) + z
}

// int16x2 -> each half clamped to [0, 15] in one instruction
__device__ __forceinline__ uint32_t clamp15x2(uint32_t p) {
    uint32_t d;
    asm("min.relu.s16x2 %0, %1, %2;" : "=r"(d) : "r"(p), "r"(0x000F000Fu));
    return d;
}

// codes c_e in [0, 15] (int16x2 pairs (c0,c1), (c2,c3), ...) -> one word, code e at bits 4e
__device__ __forceinline__ uint32_t pack8(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t p3) {
    const uint32_t x0 = p0 + (p1 << 8), x1 = p2 + (p3 << 8);  // c0 | c2 << 8 | c1 << 16 | c3 << 24
    return __byte_perm(x0 | (x0 >> 12), x1 | (x1 >> 12), 0x5410);
}

template <int G>
__global__ void __launch_bounds__(256) quant_int4_group_f16_kernel(const uint16_t *__restrict__ w, int N, int K,
                                                                    uint32_t *__restrict__ qweight,
                                                                    uint16_t *__restrict__ scales,
                                                                    uint32_t *__restrict__ qzeros) {
    constexpr int LPG = G / 8;       // lanes per group
    constexpr int GPI = 32 / LPG;    // groups per warp iteration
    constexpr int ITERS = 8 / GPI;   // iterations per zero word (8 groups)
    const int groups = K / G;
    const int zwords = (groups + 7) / 8;
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (unit >= (long long)N * zwords) return;
    const int n = (int)(unit / zwords);
    const int zw = (int)(unit % zwords);
    const int sub = lane / LPG;  // group slot within an iteration
    const int li = lane % LPG;   // lane within the group

    // Issue every load of this warp first.
    uint4 raw[ITERS];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const int j = zw * 8 + it * GPI + sub;
        raw[it] = j < groups ? ld_stream_u4(w + (size_t)n * K + (size_t)j * G + li * 8) : make_uint4(0u, 0u, 0u, 0u);
    }

    uint32_t zacc = 0;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const int j = zw * 8 + it * GPI + sub;
        const uint4 c = raw[it];
        // Range of the group, widened to contain 0.
        const uint32_t mn = hmin2_bits(hmin2_bits(c.x, c.y), hmin2_bits(c.z, c.w));
        const uint32_t mx = hmax2_bits(hmax2_bits(c.x, c.y), hmax2_bits(c.z, c.w));
        const float2 mnf = half2_bits_to_float2(mn), mxf = half2_bits_to_float2(mx);
        float lo = fminf(0.0f, fminf(mnf.x, mnf.y));
        float hi = fmaxf(0.0f, fmaxf(mxf.x, mxf.y));
#pragma unroll
        for (int off = LPG / 2; off >= 1; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        // s = fp16((hi - lo) / 15); a zero scale becomes 1.
        uint16_t s16 = float_to_half_bits_rn(__fdiv_rn(hi - lo, 15.0f));
        if (s16 == 0) s16 = 0x3c00;
        const float s = half_bits_to_float(s16);
        const float rs = __frcp_rn(s);
        // z = round(-lo / s) in [0, 15]; |-lo / s| and |w / s| stay below 32 (E = 4)
        const int z = clampi(rne_quotient<4>(-lo, s, rs), 0, 15);
        if (j < groups) {
            uint32_t bad = 0;
            const float magic = 12582912.0f + (float)z;  // 1.5 * 2^23 + z
            uint32_t p0 = pair_rne(c.x, rs, magic, bad), p1 = pair_rne(c.y, rs, magic, bad);
            uint32_t p2 = pair_rne(c.z, rs, magic, bad), p3 = pair_rne(c.w, rs, magic, bad);
            if (bad >> 31) {  // a near-tie: the IEEE quotient decides every code of this lane
                const uint32_t h[4] = {c.x, c.y, c.z, c.w};
                uint32_t pp[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = half2_bits_to_float2(h[e]);
                    const uint32_t a = (uint32_t)(__float2int_rn(__fdiv_rn(f.x, s)) + z) & 0xFFFFu;
                    const uint32_t b = (uint32_t)(__float2int_rn(__fdiv_rn(f.y, s)) + z) & 0xFFFFu;
                    pp[e] = a | (b << 16);
                }
                p0 = pp[0]; p1 = pp[1]; p2 = pp[2]; p3 = pp[3];
            }
            p0 = clamp15x2(p0);
            p1 = clamp15x2(p1);
            p2 = clamp15x2(p2);
            p3 = clamp15x2(p3);
            qweight[(size_t)n * (K / 8) + (size_t)j * (G / 8) + li] = pack8(p0, p1, p2, p3);
            if (li == 0) {
                scales[(size_t)n * groups + j] = s16;
                zacc |= (uint32_t)z << (4 * (j & 7));
            }
        }
    }
    const uint32_t zword = __reduce_or_sync(0xffffffffu, zacc);
    if (lane == 0) qzeros[(size_t)n * zwords + zw] = zword;
}

// G >= 64: 16 elements (two 16-byte loads) per lane, so the range butterfly,
// which a warp pays once for all its lanes, is spread over twice the elements;
// the range travels as one fp16x2 value (-lo, hi) (negation and max are exact
// in fp16), one shuffle and one max per butterfly step.  The scale and zero
// point of the warp's 8 groups are then computed once, on lanes 0..7 (one
// group each), and shuffled to the group's lanes: measured 5% faster on B200
// than every lane computing its own group's values in each iteration.
template <int G>
__global__ void __launch_bounds__(256) quant_int4_group_f16x16_kernel(const uint16_t *__restrict__ w, int N, int K,
                                                                      uint32_t *__restrict__ qweight,
                                                                      uint16_t *__restrict__ scales,
                                                                      uint32_t *__restrict__ qzeros) {
    constexpr int LPG = G / 16;      // lanes per group
    constexpr int GPI = 32 / LPG;    // groups per warp iteration
    constexpr int ITERS = 8 / GPI;   // iterations per zero word (8 groups)
    static_assert(ITERS >= 1, "G >= 64");
    const int groups = K / G;
    const int zwords = (groups + 7) / 8;
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (unit >= (long long)N * zwords) return;
    const int n = (int)(unit / zwords);
    const int zw = (int)(unit % zwords);
    const int sub = lane / LPG;  // group slot within an iteration
    const int li = lane % LPG;   // lane within the group

    // Issue every load of this warp first.
    uint4 raw[ITERS][2];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const int j = zw * 8 + it * GPI + sub;
        const uint16_t *p = w + (size_t)n * K + (size_t)j * G + li * 16;
        raw[it][0] = j < groups ? ld_stream_u4(p) : make_uint4(0u, 0u, 0u, 0u);
        raw[it][1] = j < groups ? ld_stream_u4(p + 8) : make_uint4(0u, 0u, 0u, 0u);
    }

    // Range of every group: (-lo, hi) with lo = min(0, min w), hi = max(0, max w), as fp16x2.
    uint32_t rr[ITERS];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const uint4 c0 = raw[it][0], c1 = raw[it][1];
        const uint32_t mn = hmin2_bits(hmin2_bits(hmin2_bits(c0.x, c0.y), hmin2_bits(c0.z, c0.w)),
                                       hmin2_bits(hmin2_bits(c1.x, c1.y), hmin2_bits(c1.z, c1.w)));
        const uint32_t mx = hmax2_bits(hmax2_bits(hmax2_bits(c0.x, c0.y), hmax2_bits(c0.z, c0.w)),
                                       hmax2_bits(hmax2_bits(c1.x, c1.y), hmax2_bits(c1.z, c1.w)));
        uint32_t r = hmax2_bits(__byte_perm(mn, mx, 0x5410) ^ 0x00008000u, __byte_perm(mn, mx, 0x7632) ^ 0x00008000u);
        r = hmax2_bits(r, 0u);
#pragma unroll
        for (int off = LPG / 2; off >= 1; off >>= 1) r = hmax2_bits(r, __shfl_xor_sync(0xffffffffu, r, off));
        rr[it] = r;
    }
    // Scale and zero point once per group: lane g (and its copies g + 8, g + 16, g + 24)
    // takes group g of the zero word, so the scalar work runs once, not once per iteration.
    const int gl = lane & 7;
    uint32_t mine = 0;
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const uint32_t t = __shfl_sync(0xffffffffu, rr[it], (gl % GPI) * LPG);
        if (gl / GPI == it) mine = t;
    }
    const float2 rf = half2_bits_to_float2(mine);
    const float lo = -rf.x, hi = rf.y;
    // s = fp16((hi - lo) / 15); a zero scale becomes 1.
    uint16_t s16 = float_to_half_bits_rn(__fdiv_rn(hi - lo, 15.0f));
    if (s16 == 0) s16 = 0x3c00;
    const float s = half_bits_to_float(s16);
    const float rs = __frcp_rn(s);
    // z = round(-lo / s) in [0, 15]; |-lo / s| and |w / s| stay below 32 (E = 4)
    const int z = clampi(rne_quotient<4>(-lo, s, rs), 0, 15);
    const float magic_g = 12582912.0f + (float)z;  // 1.5 * 2^23 + z
    // groups past the end have w = 0: s = 1, z = 0, nothing stored
    if (lane < 8 && zw * 8 + lane < groups) scales[(size_t)n * groups + zw * 8 + lane] = s16;
    const uint32_t zword = __reduce_or_sync(0xffffffffu, lane < 8 ? (uint32_t)z << (4 * lane) : 0u);

#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
        const int j = zw * 8 + it * GPI + sub;
        const int owner = it * GPI + sub;  // lane holding this group's scale and zero point
        const float rs_g = __shfl_sync(0xffffffffu, rs, owner);
        const float mg = __shfl_sync(0xffffffffu, magic_g, owner);
        const float s_g = __shfl_sync(0xffffffffu, s, owner);
        if (j < groups) {
            const uint4 c0 = raw[it][0], c1 = raw[it][1];
            const uint32_t h[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t p[8];
            uint32_t bad = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) p[e] = pair_rne(h[e], rs_g, mg, bad);
            if (bad >> 31) {  // a near-tie: the IEEE quotient decides every code of this lane
                const int zg = (int)(mg - 12582912.0f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float2 f = half2_bits_to_float2(h[e]);
                    const uint32_t a = (uint32_t)(__float2int_rn(__fdiv_rn(f.x, s_g)) + zg) & 0xFFFFu;
                    const uint32_t b = (uint32_t)(__float2int_rn(__fdiv_rn(f.y, s_g)) + zg) & 0xFFFFu;
                    p[e] = a | (b << 16);
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) p[e] = clamp15x2(p[e]);
            *reinterpret_cast<uint2 *>(qweight + (size_t)n * (K / 8) + (size_t)j * (G / 8) + li * 2) =
                make_uint2(pack8(p[0], p[1], p[2], p[3]), pack8(p[4], p[5], p[6], p[7]));
        }
    }
    if (lane == 0) qzeros[(size_t)n * zwords + zw] = zword;
}

template <typename TIn, int G>
cudaError_t launch(const void *w, int N, int K, uint32_t *qweight, uint16_t *scales, uint32_t *qzeros,
                   cudaStream_t stream) {
    const int zwords = (K / G + 7) / 8;
    const long long units = (long long)N * zwords;
    const int warps_per_block = 8;
    const long long blocks = (units + warps_per_block - 1) / warps_per_block;
    if (std::is_same<TIn, __half>::value && G >= 64)
        quant_int4_group_f16x16_kernel<G < 64 ? 64 : G><<<(unsigned)blocks, warps_per_block * 32, 0, stream>>>(
            static_cast<const uint16_t *>(w), N, K, qweight, scales, qzeros);
    else if (std::is_same<TIn, __half>::value)
        quant_int4_group_f16_kernel<G><<<(unsigned)blocks, warps_per_block * 32, 0, stream>>>(
            static_cast<const uint16_t *>(w), N, K, qweight, scales, qzeros);
    else
        quant_int4_group_kernel<TIn, G><<<(unsigned)blocks, warps_per_block * 32, 0, stream>>>(
            static_cast<const TIn *>(w), N, K, qweight, scales, qzeros);
    return cudaGetLastError();
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_quantize_group_int4(const void *w, wq_dtype w_dtype, int N, int K, int group_size,
                                            uint32_t *qweight, uint16_t *scales, uint32_t *qzeros,
                                            void *stream) {
    WQ_REQUIRE_PTR(w, "w");
    WQ_REQUIRE_PTR(qweight, "qweight");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE_PTR(qzeros, "qzeros");
    WQ_REQUIRE(N > 0 && K > 0, WQ_ERR_INVALID_ARG, "N and K must be positive (N=%d K=%d)", N, K);
    WQ_REQUIRE(w_dtype == WQ_F32 || w_dtype == WQ_F16, WQ_ERR_INVALID_ARG, "unknown w_dtype %d",
               (int)w_dtype);
    WQ_REQUIRE(group_size == 32 || group_size == 64 || group_size == 128 || group_size == 256,
               WQ_ERR_UNSUPPORTED, "group_size must be 32, 64, 128 or 256 (got %d)", group_size);
    WQ_REQUIRE(K % group_size == 0, WQ_ERR_INVALID_ARG, "K (%d) must be a multiple of group_size (%d)", K,
               group_size);
    const long long units = (long long)N * ((K / group_size + 7) / 8);
    WQ_REQUIRE(units / 8 < (1ll << 31), WQ_ERR_UNSUPPORTED, "matrix too large");
    cudaStream_t st = wq::as_stream(stream);
    cudaError_t e;
    const bool f16 = w_dtype == WQ_F16;
    switch (group_size) {
        case 32: e = f16 ? wq::launch<__half, 32>(w, N, K, qweight, scales, qzeros, st)
                         : wq::launch<float, 32>(w, N, K, qweight, scales, qzeros, st); break;
        case 64: e = f16 ? wq::launch<__half, 64>(w, N, K, qweight, scales, qzeros, st)
                         : wq::launch<float, 64>(w, N, K, qweight, scales, qzeros, st); break;
        case 128: e = f16 ? wq::launch<__half, 128>(w, N, K, qweight, scales, qzeros, st)
                          : wq::launch<float, 128>(w, N, K, qweight, scales, qzeros, st); break;
        default: e = f16 ? wq::launch<__half, 256>(w, N, K, qweight, scales, qzeros, st)
                         : wq::launch<float, 256>(w, N, K, qweight, scales, qzeros, st); break;
    }
    if (e != cudaSuccess)
        return wq::fail(WQ_ERR_CUDA, "wq_quantize_group_int4: launch failed: %s", cudaGetErrorString(e));
    return WQ_OK;
}
