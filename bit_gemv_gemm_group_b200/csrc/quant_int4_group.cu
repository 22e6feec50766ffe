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
#include <algorithm>
#include <type_traits>

#include "sm100.cuh"
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
// f32x2 fused operations on the products of w with RN(1/s) one ulp down and
// one ulp up (pair_code below: exact without a division, ties to even).
// Clamping (one min.relu.s16x2 per pair) and nibble packing run on 16-bit SIMD
// lanes.
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

// rne(w / s) + z of an fp16 pair as int16x2, exactly, without a division: rs_lo and rs_hi are
// RN(1/s) one ulp down and one ulp up (so rs_lo < 1/s < rs_hi).
//  - For fp16 w and s with |w / s| < 32, w / s is either exactly a half-integer or at least
//    2^-13 away from every half-integer (w / s = M_w 2^c / M_s with 11-bit M_w, M_s; a
//    nonzero distance is at least 1 / (2 M_s 2^max(-c, 0)) >= 1/8190).  w rs_lo and w rs_hi
//    are within 1.5 2^-23 |w / s| < 2^-17 of w / s, so off a tie both round (one fused
//    multiply-add each, rounding w rs + M, M = 1.5 * 2^23, to an integer) to rne(w / s),
//    which is also rne(fl(w / s)) (fl(w / s) is within 2^-19).
//  - At an exact tie k + 1/2 the two products lie strictly on either side of it (rs_lo <
//    1/s < rs_hi), so one gives M + k and the other M + k + 1; fl(w / s) = k + 1/2 exactly
//    and rounds to the even of k, k + 1.  The mean of the two candidates, rounded once
//    (a fused multiply-add), is M + k + 1/2 there and rounds to the even one (M is even,
//    the ulp is 1, ties go to even); off a tie it is the common candidate itself.
//  - The fused sums never sit exactly on a half-integer themselves: that would need rs_lo or
//    rs_hi to have at most 6 significant bits, and a float within 1.5 ulp of 1/s has that few
//    only if s is a power of two, whose RN(1/s) -+ 1 ulp have 24.
// Adding z (an integer below 16) is exact; the low 16 bits of M + j are j as an int16.
// All of it runs on the fp32 pipe (f32x2); the one integer instruction gathers the halves.
__device__ __forceinline__ uint32_t pair_code(uint32_t h2, float rs_lo, float rs_hi, float zf) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const float2 f = half2_bits_to_float2(h2);
    const float2 rl = __ffma2_rn(f, make_float2(rs_lo, rs_lo), make_float2(kMagic, kMagic));
    const float2 rh = __ffma2_rn(f, make_float2(rs_hi, rs_hi), make_float2(kMagic, kMagic));
    const float2 half_rh = __fmul2_rn(rh, make_float2(0.5f, 0.5f));                   // exact
    const float2 mean = __ffma2_rn(rl, make_float2(0.5f, 0.5f), half_rh);             // M + rne(w / s)
    const float2 r = __fadd2_rn(mean, make_float2(zf, zf));                           // + z, exact
    return __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x5410);
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
            const float zf = (float)z;
            const float rs_lo = __uint_as_float(__float_as_uint(rs) - 1u);
            const float rs_hi = __uint_as_float(__float_as_uint(rs) + 1u);
            uint32_t p0 = pair_code(c.x, rs_lo, rs_hi, zf), p1 = pair_code(c.y, rs_lo, rs_hi, zf);
            uint32_t p2 = pair_code(c.z, rs_lo, rs_hi, zf), p3 = pair_code(c.w, rs_lo, rs_hi, zf);
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

// G >= 64: one warp per (row, unit of 32 E consecutive elements), E = 32
// elements per lane (E = 64 for G = 256), so a group spans LPG = G / E lanes
// (2 or 4) and a unit holds whole zero words (one, or two for G = 64).  Each
// lane loads its E elements with E / 8 16-byte loads issued before any
// arithmetic, and computes the scale and zero point of its own group itself:
// nothing is distributed by shuffles and no scalar step runs more than once
// per unit.  The range is one fp16x2 value (-lo, hi) (negation and max are
// exact in fp16), reduced over the group's lanes with one shuffle and one max
// per step.  The grid is (row blocks of 8, units), so no index is divided.
template <int G>
struct Wide {
    static constexpr int E = G >= 256 ? 64 : 32;  // elements per lane
    static constexpr int V = E / 8;               // 16-byte loads (and code words) per lane
    static constexpr int LPG = G / E;             // lanes per group
    static constexpr int UE = 32 * E;             // elements per unit
    static constexpr int ZPU = UE / (8 * G);      // zero words per unit
    static_assert(G >= 64 && LPG >= 2 && ZPU >= 1, "G in {64, 128, 256}");
};

// RN(d / 15) for a finite fp32 d >= 0 (the scale's quotient (hi - lo) / 15).
// With d = m 2^e (m a 24-bit integer), m / 15 is either exact or k + r / 15
// with r in 1..14, whose binary fraction repeats r's four bits forever; the
// part below an fp32 ulp is then c / 15 of an ulp with c in 1..14, so the
// quotient is never a tie and stays at least ulp / 30 away from one.  The
// fp64 product d * RN64(1/15) is within 2^-52 relative (well under 2^-28 ulp)
// of d / 15, so rounding it to fp32 gives the correctly rounded quotient.
__device__ __forceinline__ float div15_rn(float d) {
    return __double2float_rn(__dmul_rn((double)d, 0x1.1111111111111p-4));
}

// One lane's share of a unit: its E weights (raw fp16, zeros past the end) -> its V code
// words, and the scale and zero point of its group.  Every lane of the warp must call it
// (the range is reduced across the group's lanes).
template <int G>
__device__ __forceinline__ void quantize_lane(const uint4 (&raw)[Wide<G>::V], uint32_t (&words)[Wide<G>::V],
                                              uint16_t &s16_out, int &z_out) {
    using P = Wide<G>;
    // Range of the group, widened to contain 0, as fp16x2 (-lo, hi).
    uint32_t mn = hmin2_bits(hmin2_bits(raw[0].x, raw[0].y), hmin2_bits(raw[0].z, raw[0].w));
    uint32_t mx = hmax2_bits(hmax2_bits(raw[0].x, raw[0].y), hmax2_bits(raw[0].z, raw[0].w));
#pragma unroll
    for (int v = 1; v < P::V; ++v) {
        mn = hmin2_bits(mn, hmin2_bits(hmin2_bits(raw[v].x, raw[v].y), hmin2_bits(raw[v].z, raw[v].w)));
        mx = hmax2_bits(mx, hmax2_bits(hmax2_bits(raw[v].x, raw[v].y), hmax2_bits(raw[v].z, raw[v].w)));
    }
    uint32_t r = hmax2_bits(__byte_perm(mn, mx, 0x5410) ^ 0x00008000u, __byte_perm(mn, mx, 0x7632) ^ 0x00008000u);
    r = hmax2_bits(r, 0u);
#pragma unroll
    for (int off = 1; off < P::LPG; off <<= 1) r = hmax2_bits(r, __shfl_xor_sync(0xffffffffu, r, off));

    const float2 rf = half2_bits_to_float2(r);
    const float lo = -rf.x, hi = rf.y;
    // s = fp16((hi - lo) / 15); a zero scale becomes 1.
    uint16_t s16 = float_to_half_bits_rn(div15_rn(hi - lo));
    if (s16 == 0) s16 = 0x3c00;
    const float s = half_bits_to_float(s16);
    const float rs = __frcp_rn(s);
    // z = round(-lo / s) in [0, 15]; |-lo / s| and |w / s| stay below 32 (E = 4)
    const int z = clampi(rne_quotient<4>(-lo, s, rs), 0, 15);
    const float zf = (float)z;

    const float rs_lo = __uint_as_float(__float_as_uint(rs) - 1u), rs_hi = __uint_as_float(__float_as_uint(rs) + 1u);
#pragma unroll
    for (int v = 0; v < P::V; ++v)
        words[v] = pack8(clamp15x2(pair_code(raw[v].x, rs_lo, rs_hi, zf)),
                         clamp15x2(pair_code(raw[v].y, rs_lo, rs_hi, zf)),
                         clamp15x2(pair_code(raw[v].z, rs_lo, rs_hi, zf)),
                         clamp15x2(pair_code(raw[v].w, rs_lo, rs_hi, zf)));
    s16_out = s16;
    z_out = z;
}

// The unit's zero words (nibble j mod 8 of a word from each group's first lane, j the group's
// index in its row) -> zw(q, word) for each of the unit's ZPU words.
template <int G, typename Store>
__device__ __forceinline__ void store_zero_words(int lane, int j, int z, Store zw) {
    using P = Wide<G>;
    const uint32_t zbits = lane % P::LPG == 0 ? (uint32_t)z << (4 * (j & 7)) : 0u;
    constexpr int kLanesPerWord = 32 / P::ZPU;
#pragma unroll
    for (int q = 0; q < P::ZPU; ++q) {
        const uint32_t word = __reduce_or_sync(0xffffffffu, lane / kLanesPerWord == q ? zbits : 0u);
        if (lane == q * kLanesPerWord) zw(q, word);
    }
}

// Any K (a multiple of G): grid (row blocks of 8, units of a row), one warp per (row, unit).
template <int G>
__global__ void __launch_bounds__(256, G >= 256 ? 2 : 4) quant_int4_group_f16w_kernel(const uint16_t *__restrict__ w, int N, int K,
                                                                       uint32_t *__restrict__ qweight,
                                                                       uint16_t *__restrict__ scales,
                                                                       uint32_t *__restrict__ qzeros) {
    using P = Wide<G>;
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (n >= N) return;
    const int k0 = blockIdx.y * P::UE + lane * P::E;  // this lane's first element
    const bool in = k0 < K;                           // K % G == 0: a lane is wholly in or out
    const uint16_t *src = w + (size_t)n * K + k0;

    uint4 raw[P::V];
#pragma unroll
    for (int v = 0; v < P::V; ++v) raw[v] = in ? ld_stream_u4(src + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
    uint32_t words[P::V];
    uint16_t s16;
    int z;
    quantize_lane<G>(raw, words, s16, z);

    const int j = k0 / G;  // this lane's group
    if (in) {
        uint32_t *dst = qweight + (size_t)n * (K / 8) + k0 / 8;
#pragma unroll
        for (int v = 0; v < P::V; v += 4)
            *reinterpret_cast<uint4 *>(dst + v) = make_uint4(words[v], words[v + 1], words[v + 2], words[v + 3]);
        if (lane % P::LPG == 0) scales[(size_t)n * (K / G) + j] = s16;
    }
    const int zwords = (K / G + 7) / 8;
    store_zero_words<G>(lane, j, z, [&](int q, uint32_t word) {
        const int zw = blockIdx.y * P::ZPU + q;
        if (zw < zwords) qzeros[(size_t)n * zwords + zw] = word;
    });
}

// K a multiple of the unit (every decode shape): the matrix is one run of N K / UE units, and
// the codes, scales and zero words of unit u start at u's element offset divided by 8, G and
// 8 G.  A persistent CTA of 8 quantizing warps and one copy warp walks stages of 8
// consecutive units (16 KB of fp16; 32 KB for G = 256), stages blockIdx.x + i gridDim.x;
// the copy warp keeps the CTA's next S stages in flight in a ring of shared-memory slots, so
// the loads never wait for the arithmetic, and each quantizing warp takes one unit of a
// stage, frees the slot as soon as its data is in registers and writes its results straight
// to global memory.  A stage arrives by one 2-D TMA copy of the matrix seen as rows of 128
// bytes, with the 128-byte swizzle (16-byte chunk c of row r lands at chunk c ^ (r mod 8)):
// a lane's E contiguous weights start 64 or 128 bytes after its neighbour's, so unswizzled
// its 16-byte loads would meet on the same banks (16- or 32-way); swizzled, a warp's load
// spreads over all 32 banks.
constexpr unsigned kQ4RingSite = 0x2000;
// Waiting threads sleep inside mbarrier.try_wait (up to this long per test) instead of polling:
// the kernel is issue-bound, and the polling took issue slots (measured 2% faster).
constexpr uint32_t kQ4SleepNs = 20000;

template <int G>
struct Q4Ring {
    static constexpr uint32_t STAGE = 8u * Wide<G>::UE * 2u;  // bytes per stage
    static constexpr int S = G >= 256 ? 2 : 4;                // slots: three CTAs per SM
    static constexpr uint32_t ROWS = STAGE / 128;                // 128-byte rows per stage (TMA box)
    static constexpr uint32_t OFF_BAR = S * STAGE;
    static constexpr uint32_t SMEM = 1024 + OFF_BAR + 16u * S + 16u;  // slots 1024-byte aligned (swizzle)
    static_assert(ROWS <= 256, "TMA box height");
};

template <int G>
__global__ void __launch_bounds__(288, G >= 256 ? 2 : 3)
    quant_int4_group_ring_kernel(const __grid_constant__ CUtensorMap tmap_w, long long units,
                                 uint32_t *__restrict__ qweight,
                                 uint16_t *__restrict__ scales, uint32_t *__restrict__ qzeros, unsigned int *status,
                                 uint64_t limit_ns) {
    using namespace sm100;
    using P = Wide<G>;
    using RL = Q4Ring<G>;
    extern __shared__ uint8_t q4_ring_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(q4_ring_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(base + RL::OFF_BAR);
    uint64_t *empty = full + RL::S;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + RL::S);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long stages = (units + 7) / 8;
    const long long mine = (long long)blockIdx.x < stages ? (stages - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < RL::S; ++i) {
            mbar_init(smem_u32(&full[i]), 1);
            mbar_init(smem_u32(&empty[i]), 8);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const WaitCtl ctl{abort_flag, status, limit_ns};

    long long issued = 0;  // copy warp, lane 0: stages handed to the copy engine
    if (warp == 8) {
        // ------------------------------------------------------------ copy warp
        if (lane == 0) {
            prefetch_tmap(&tmap_w);
            for (; issued < mine; ++issued) {
                const int slot = (int)(issued % RL::S);
                const uint32_t u = (uint32_t)(issued / RL::S);
                if (!wait_parity(smem_u32(&empty[slot]), (u & 1u) ^ 1u, ctl, kQ4RingSite | 0x1, kQ4SleepNs)) break;
                const long long u0 = (blockIdx.x + issued * gridDim.x) * 8;
                const uint32_t fb = smem_u32(&full[slot]);
                // rows past the matrix (a last, partial stage) arrive as zeros and count in full
                mbar_arrive_expect_tx(fb, RL::STAGE);
                tma_load_2d(smem_u32(base + (uint32_t)slot * RL::STAGE), &tmap_w, fb, 0,
                            (int)(u0 * (P::UE * 2 / 128)));
            }
        }
    } else {
        // ------------------------------------------------------------ quantizing warps
        for (long long i = 0; i < mine; ++i) {
            const int slot = (int)(i % RL::S);
            const uint32_t u = (uint32_t)(i / RL::S);
            // warp-uniform: the lanes leave together (the shuffles below need the whole warp)
            if (!__all_sync(0xffffffffu, wait_parity(smem_u32(&full[slot]), u & 1u, ctl, kQ4RingSite, kQ4SleepNs))) break;
            const long long unit = (blockIdx.x + i * gridDim.x) * 8 + warp;
            uint4 raw[P::V];
            // this lane's E weights: row r of the stage, chunks c0 .. c0 + V - 1, stored swizzled
            const uint32_t pos = (uint32_t)warp * P::UE * 2 + (uint32_t)lane * P::E * 2;
            const uint32_t row = pos >> 7, c0 = (pos & 127u) >> 4;
            const uint8_t *rp = base + (uint32_t)slot * RL::STAGE + row * 128u;
#pragma unroll
            for (int v = 0; v < P::V; ++v)
                raw[v] = *reinterpret_cast<const uint4 *>(rp + (((c0 + (uint32_t)v) ^ (row & 7u)) << 4));
            // Every lane orders its reads of the slot before the copy engine's next write into it
            // (generic -> async proxy), then the warp releases the slot.
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&empty[slot]));
            if (unit >= units) continue;  // past the end of the last stage (warp-uniform)
            uint32_t words[P::V];
            uint16_t s16;
            int z;
            quantize_lane<G>(raw, words, s16, z);
            const size_t e0 = (size_t)unit * P::UE + (size_t)lane * P::E;  // this lane's first element
            uint32_t *dst = qweight + e0 / 8;
#pragma unroll
            for (int v = 0; v < P::V; v += 4)
                *reinterpret_cast<uint4 *>(dst + v) = make_uint4(words[v], words[v + 1], words[v + 2], words[v + 3]);
            if (lane % P::LPG == 0) scales[e0 / G] = s16;
            store_zero_words<G>(lane, (int)((e0 / G) & 7), z,
                                [&](int q, uint32_t word) { qzeros[(size_t)unit * P::ZPU + q] = word; });
        }
    }
    // Every warp is done with the ring.  After a timeout the copies still in flight (at most the
    // last S issued) land before the CTA exits.
    __syncthreads();
    if (warp == 8 && lane == 0 && *abort_flag) {
        for (long long j = issued > RL::S ? issued - RL::S : 0; j < issued; ++j)
            drain_parity(smem_u32(&full[j % RL::S]), (uint32_t)(j / RL::S) & 1u, 2000000000ull, status,
                         kQ4RingSite | 0x2);
    }
}

template <typename TIn, int G>
cudaError_t launch(const void *w, int N, int K, uint32_t *qweight, uint16_t *scales, uint32_t *qzeros,
                   cudaStream_t stream) {
    const int zwords = (K / G + 7) / 8;
    const long long units = (long long)N * zwords;
    const int warps_per_block = 8;
    if (std::is_same<TIn, __half>::value && G >= 64) {
        constexpr int GW = G < 64 ? 64 : G;
        if (K % Wide<GW>::UE == 0) {
            using RL = Q4Ring<GW>;
            unsigned int *status = device_status_word();
            if (!status) return cudaErrorUnknown;
            auto kern = quant_int4_group_ring_kernel<GW>;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RL::SMEM);
            if (e != cudaSuccess) return e;
            int per_sm = 0;
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 288, RL::SMEM);
            if (e != cudaSuccess) return e;
            const long long total = (long long)N * (K / Wide<GW>::UE);
            const long long stages = (total + 7) / 8;
            const int grid = (int)std::min<long long>(stages, (long long)num_sms() * std::max(per_sm, 1));
            CUtensorMap tmap;
            if (!encode_tmap_2d(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, w, 64, (uint64_t)total * (Wide<GW>::UE / 64),
                                128, 64, RL::ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
                return cudaErrorInvalidValue;
            kern<<<grid, 288, RL::SMEM, stream>>>(tmap, total, qweight, scales, qzeros, status, wait_limit());
            return cudaGetLastError();
        }
        const dim3 grid((unsigned)((N + 7) / 8), (unsigned)((K + Wide<GW>::UE - 1) / Wide<GW>::UE));
        quant_int4_group_f16w_kernel<GW><<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(w), N, K, qweight,
                                                                   scales, qzeros);
        return cudaGetLastError();
    }
    const long long blocks = (units + warps_per_block - 1) / warps_per_block;
    if (std::is_same<TIn, __half>::value)
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
    // fp16 with g >= 64: a grid of (ceil(N / 8), ceil(K / 1024)) blocks (K / 2048 for g = 256)
    WQ_REQUIRE(!(w_dtype == WQ_F16 && group_size >= 64) || (K + 1023) / 1024 <= 65535, WQ_ERR_UNSUPPORTED,
               "K (%d) too large for the fp16 quantizer (at most 65535 * 1024)", K);
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
