// Fused dequantize + GEMV for W4A16 decode, batch 1..8.
//
// Source: "How quantization works", section "Inference view" (quantized
// weights are unpacked in registers and multiplied by their scales inside the
// kernel); "Quantization from Scratch", section "Scale and zero-point"
// (w^ = (q - z) s) and "What it buys at decode" (a decode step streams every
// weight once); "Quantization Explained", "Why It Is Faster".
//
//   y[b][n] = fp16_rn( sum_j s[n][j] * sum_{k in group j} (q[n][k] - z[n][j]) * x[b][k] )
//
// Three kernels, chosen by wq_gemv_w4a16:
//   - group size 128, K % 256 == 0 (every decode shape): the streaming
//     tensor-core kernel further below (TMA ring, producer-built B fragments,
//     codes fed to mma.sync as fp16 subnormals); it also serves wq_gemm_w4a16
//     for up to 32 rows in passes of up to 16;
//   - group size 128, other K: a register-prefetch mma.sync kernel;
//   - other group sizes: the CUDA-core kernel that follows.
//
// CUDA-core kernel.  Work decomposition: a warp owns R weight rows and walks K in steps of 1024
// weights: lane l of step t reads the 16-byte chunk c = 32 t + l of each of
// its rows (32 consecutive codes, all in one group since g >= 32), so a warp
// load instruction covers 512 contiguous bytes of a row.  Loads bypass L1
// (each weight byte is read once); x is read through L1 (shared by every warp
// of the SM) and converted to fp32 once per step, then reused for the R rows.
//
// Dequantization is exact and needs no conversion instruction: OR-ing nibble
// i of a word into the mantissa of 2^23 gives the float 2^23 + 16^(i mod 5) q
// (one LOP3 per code), and one packed fma (f32x2) with the constants
// 16^-(i mod 5) and -(2^(23 - 4(i mod 5)) + z) turns it into the exact float
// q - z.  A second packed fma accumulates (q - z) x in fp32; the group scale
// multiplies the 32-code partial sum once.
#include "sm100.cuh"
#include "wq_device.cuh"
#include "wq_host.h"

#include <algorithm>
#include <cmath>

namespace wq {
namespace {

constexpr int kWarps = 8;

struct Unpacked {
    float2 d[4];  // (q - z) for codes (0,1) (2,3) (4,5) (6,7) of one word
};

// Per-row constants for one group: offsets 2^(23-4e) + z for e = 0..4.
struct ZeroOffsets {
    float o0, o4, o8, o12, o16;
};

__device__ __forceinline__ ZeroOffsets zero_offsets(int z) {
    ZeroOffsets r;
    r.o0 = __int_as_float(0x4B000000 + z);   // 2^23 + z
    r.o4 = __int_as_float(0x49000000 + (z << 4)) ;  // 2^19 + z  (mantissa step 2^-4 at 2^19)
    r.o8 = __int_as_float(0x47000000 + (z << 8));   // 2^15 + z
    r.o12 = __int_as_float(0x45000000 + (z << 12)); // 2^11 + z
    r.o16 = __int_as_float(0x43000000 + (z << 16)); // 2^7 + z
    return r;
}

__device__ __forceinline__ Unpacked unpack_word(uint32_t w, const ZeroOffsets &o) {
    const uint32_t u = w >> 12;
    const float t0 = __uint_as_float((w & 0x0000000Fu) | 0x4B000000u);  // 2^23 + q0
    const float t1 = __uint_as_float((w & 0x000000F0u) | 0x4B000000u);  // 2^23 + 16 q1
    const float t2 = __uint_as_float((w & 0x00000F00u) | 0x4B000000u);  // 2^23 + 256 q2
    const float t3 = __uint_as_float((w & 0x0000F000u) | 0x4B000000u);  // 2^23 + 4096 q3
    const float t4 = __uint_as_float((w & 0x000F0000u) | 0x4B000000u);  // 2^23 + 65536 q4
    const float t5 = __uint_as_float((u & 0x00000F00u) | 0x4B000000u);  // 2^23 + 256 q5
    const float t6 = __uint_as_float((u & 0x0000F000u) | 0x4B000000u);  // 2^23 + 4096 q6
    const float t7 = __uint_as_float((u & 0x000F0000u) | 0x4B000000u);  // 2^23 + 65536 q7
    Unpacked r;
    r.d[0] = __ffma2_rn(make_float2(t0, t1), make_float2(1.0f, 0x1p-4f), make_float2(-o.o0, -o.o4));
    r.d[1] = __ffma2_rn(make_float2(t2, t3), make_float2(0x1p-8f, 0x1p-12f), make_float2(-o.o8, -o.o12));
    r.d[2] = __ffma2_rn(make_float2(t4, t5), make_float2(0x1p-16f, 0x1p-8f), make_float2(-o.o16, -o.o8));
    r.d[3] = __ffma2_rn(make_float2(t6, t7), make_float2(0x1p-12f, 0x1p-16f), make_float2(-o.o12, -o.o16));
    return r;
}

// Activations and output in fp16, or in bf16 (BF: x = bits << 16 as fp32, exact; y rounded to bf16).
__device__ __forceinline__ float2 bf16x2_bits_to_float2(uint32_t b) {
    return make_float2(__uint_as_float(b << 16), __uint_as_float(b & 0xFFFF0000u));
}

template <int B, int R, bool BF = false>
__global__ void __launch_bounds__(kWarps * 32) gemv_w4a16_kernel(const uint16_t *__restrict__ x,
                                                                 const uint32_t *__restrict__ qweight,
                                                                 const uint16_t *__restrict__ scales,
                                                                 const uint32_t *__restrict__ qzeros, int N,
                                                                 int K, int g, uint16_t *__restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int row0 = (blockIdx.x * kWarps + (threadIdx.x >> 5)) * R;
    if (row0 >= N) return;
    const int chunks = K >> 5;          // 16-byte chunks per row
    const int groups = K / g;
    const int zwords = (groups + 7) >> 3;
    const int words = K >> 3;

    float acc[R][B];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) acc[r][b] = 0.0f;

    for (int c = lane; c < chunks; c += 32) {
        const int k0 = c << 5;
        const int j = k0 / g;
        uint4 wv[R];
        float sc[R];
        ZeroOffsets zo[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int n = min(row0 + r, N - 1);
            wv[r] = ld_stream_u4(qweight + (size_t)n * words + (c << 2));
            sc[r] = half_bits_to_float(__ldg(scales + (size_t)n * groups + j));
            const uint32_t zw = __ldg(qzeros + (size_t)n * zwords + (j >> 3));
            zo[r] = zero_offsets((int)((zw >> ((j & 7) << 2)) & 0xFu));
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const uint16_t *xp = x + (size_t)b * K + k0;
            float2 xf[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 xv = ld_shared_ro_u4(xp + 8 * v);
                xf[4 * v + 0] = BF ? bf16x2_bits_to_float2(xv.x) : half2_bits_to_float2(xv.x);
                xf[4 * v + 1] = BF ? bf16x2_bits_to_float2(xv.y) : half2_bits_to_float2(xv.y);
                xf[4 * v + 2] = BF ? bf16x2_bits_to_float2(xv.z) : half2_bits_to_float2(xv.z);
                xf[4 * v + 3] = BF ? bf16x2_bits_to_float2(xv.w) : half2_bits_to_float2(xv.w);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float2 p = make_float2(0.0f, 0.0f);
                const uint32_t wr[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const Unpacked u = unpack_word(wr[q], zo[r]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) p = __ffma2_rn(u.d[i], xf[4 * q + i], p);
                }
                acc[r][b] = fmaf(sc[r], p.x + p.y, acc[r][b]);
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) {
            float v = acc[r][b];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            acc[r][b] = v;
        }
    if (lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            if (row0 + r < N) {
#pragma unroll
                for (int b = 0; b < B; ++b)
                    y[(size_t)b * N + row0 + r] =
                        BF ? float_to_bf16_bits_rn(acc[r][b]) : float_to_half_bits_rn(acc[r][b]);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Group size 128: the dot products run on the warp-level tensor-core MMA
// (mma.sync m16n8k16, fp16 x fp16 -> fp32).  Dequantization stays in
// registers and exact: LOP3 with the fp16 exponent trick turns a word into
// four fp16 pairs (1024 + q) / (1024 + 16 q), and one fp16x2 add or fma per
// pair gives q - z exactly.  Those pairs are the MMA's A fragment directly
// (no shared-memory round trip), x is the B fragment (batch = the MMA's N,
// so batches 1..8 cost the same), and the group scale multiplies the fp32
// per-group result.  This takes about 1.7 issue slots per weight against
// 2.3+ for the fp32 FMA formulation, which keeps the kernel on the HBM side
// of the roofline.
//
// Layout of a group (128 codes of one row) in the MMA: thread t = lane % 4
// owns codes [32 t, 32 t + 32) of the group, i.e. one 16-byte load per row.
// Word j of that block feeds k-steps 2j and 2j+1; the MMA's logical k index is
// a fixed permutation of the real one, applied identically to the x fragment:
// (a0,a1) = (q[8j+2h], q[8j+2h+4]), (a4,a5) = (q[8j+2h+1], q[8j+2h+5]) for
// k-step 2j+h, and the matching x pairs are built with PRMT.
// Work split: a CTA owns RT*16 rows; its 8 warps take contiguous group ranges
// of K and reduce through shared memory at the end.
// ---------------------------------------------------------------------------
constexpr int kMmaWarps = 8;

__device__ __forceinline__ uint32_t lop3_or_and(uint32_t a, uint32_t mask, uint32_t magic) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(magic));  // (a & mask) | magic
    return d;
}

__device__ __forceinline__ uint32_t hadd2_u(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t prmt_u(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// (q0-z, q4-z), (q1-z, q5-z), (q2-z, q6-z), (q3-z, q7-z) as fp16x2, exact.
__device__ __forceinline__ void dequant_pairs(uint32_t w, uint32_t zlo, uint32_t zhi, uint32_t (&p)[4]) {
    const uint32_t w8 = w >> 8;
    p[0] = hadd2_u(lop3_or_and(w, 0x000F000Fu, 0x64006400u), zlo);                // 1024+q - (1024+z)
    p[1] = hfma2_u(lop3_or_and(w, 0x00F000F0u, 0x64006400u), 0x2C002C00u, zhi);   // (1024+16q)/16 - (64+z)
    p[2] = hadd2_u(lop3_or_and(w8, 0x000F000Fu, 0x64006400u), zlo);
    p[3] = hfma2_u(lop3_or_and(w8, 0x00F000F0u, 0x64006400u), 0x2C002C00u, zhi);
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

struct GroupData {
    uint4 w[2];        // rows r0 and r0 + 8: 32 codes each
    uint32_t s;        // fp16 scales of the two rows (lo: r0, hi: r0 + 8)
    uint32_t z;        // zero points of the two rows (bits 0..3: r0, 4..7: r0 + 8)
};

template <int RT>
__device__ __forceinline__ void load_group(GroupData (&gd)[RT], const uint32_t *__restrict__ qweight,
                                           const uint16_t *__restrict__ scales, const uint32_t *__restrict__ qzeros,
                                           const int (&rows)[RT][2], int g, int t, int words, int groups, int zwords) {
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        uint32_t s2 = 0, z2 = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int n = rows[i][h];
            gd[i].w[h] = ld_stream_u4(qweight + (size_t)n * words + g * 16 + t * 4);
            s2 |= (uint32_t)__ldg(scales + (size_t)n * groups + g) << (16 * h);
            z2 |= ((__ldg(qzeros + (size_t)n * zwords + (g >> 3)) >> ((g & 7) * 4)) & 0xFu) << (4 * h);
        }
        gd[i].s = s2;
        gd[i].z = z2;
    }
}

template <int RT>
__global__ void __launch_bounds__(kMmaWarps * 32) gemv_w4a16_mma_kernel(const uint16_t *__restrict__ x, int B,
                                                                        const uint32_t *__restrict__ qweight,
                                                                        const uint16_t *__restrict__ scales,
                                                                        const uint32_t *__restrict__ qzeros, int N,
                                                                        int K, uint16_t *__restrict__ y) {
    __shared__ float red[kMmaWarps][RT * 16][8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = lane & 3, r = lane >> 2;  // r: row in the 8-row half / batch column of the B fragment
    const int n_base = blockIdx.x * RT * 16;
    const int groups = K >> 7, zwords = (groups + 7) >> 3, words = K >> 3;
    const int g0 = (int)((long long)warp * groups / kMmaWarps);
    const int g1 = (int)((long long)(warp + 1) * groups / kMmaWarps);
    int rows[RT][2];
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        rows[i][0] = min(n_base + 16 * i + r, N - 1);
        rows[i][1] = min(n_base + 16 * i + r + 8, N - 1);
    }
    const bool xrow = r < B;
    const uint16_t *xp = x + (size_t)(xrow ? r : 0) * K + t * 32;

    float acc[RT][4];
#pragma unroll
    for (int i = 0; i < RT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

    GroupData cur[RT], nxt[RT];
    uint4 xc[4], xn[4];
    if (g0 < g1) {
        load_group<RT>(cur, qweight, scales, qzeros, rows, g0, t, words, groups, zwords);
#pragma unroll
        for (int v = 0; v < 4; ++v) xc[v] = xrow ? ld_shared_ro_u4(xp + (size_t)g0 * 128 + 8 * v) : make_uint4(0, 0, 0, 0);
    }
    for (int g = g0; g < g1; ++g) {
        if (g + 1 < g1) {
            load_group<RT>(nxt, qweight, scales, qzeros, rows, g + 1, t, words, groups, zwords);
#pragma unroll
            for (int v = 0; v < 4; ++v)
                xn[v] = xrow ? ld_shared_ro_u4(xp + (size_t)(g + 1) * 128 + 8 * v) : make_uint4(0, 0, 0, 0);
        }
        // B fragments for the 8 k-steps: word j of x (8 halves) -> pairs (x_a, x_a+4), (x_a+1, x_a+5)
        uint32_t bf[8][2];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t v01 = j == 0 ? xc[0].x : j == 1 ? xc[1].x : j == 2 ? xc[2].x : xc[3].x;
            const uint32_t v23 = j == 0 ? xc[0].y : j == 1 ? xc[1].y : j == 2 ? xc[2].y : xc[3].y;
            const uint32_t v45 = j == 0 ? xc[0].z : j == 1 ? xc[1].z : j == 2 ? xc[2].z : xc[3].z;
            const uint32_t v67 = j == 0 ? xc[0].w : j == 1 ? xc[1].w : j == 2 ? xc[2].w : xc[3].w;
            bf[2 * j][0] = prmt_u(v01, v45, 0x5410u);      // (x0, x4)
            bf[2 * j][1] = prmt_u(v01, v45, 0x7632u);      // (x1, x5)
            bf[2 * j + 1][0] = prmt_u(v23, v67, 0x5410u);  // (x2, x6)
            bf[2 * j + 1][1] = prmt_u(v23, v67, 0x7632u);  // (x3, x7)
        }
#pragma unroll
        for (int i = 0; i < RT; ++i) {
            const uint32_t z0 = cur[i].z & 0xFu, z1 = (cur[i].z >> 4) & 0xFu;
            const uint32_t zlo0 = 0xE400E400u + z0 * 0x00010001u, zhi0 = 0xD400D400u + z0 * 0x00100010u;
            const uint32_t zlo1 = 0xE400E400u + z1 * 0x00010001u, zhi1 = 0xD400D400u + z1 * 0x00100010u;
            float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            const uint32_t wa[4] = {cur[i].w[0].x, cur[i].w[0].y, cur[i].w[0].z, cur[i].w[0].w};
            const uint32_t wb[4] = {cur[i].w[1].x, cur[i].w[1].y, cur[i].w[1].z, cur[i].w[1].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t pa[4], pb[4];
                dequant_pairs(wa[j], zlo0, zhi0, pa);
                dequant_pairs(wb[j], zlo1, zhi1, pb);
                // k-step 2j: codes (0,4) and (1,5); k-step 2j+1: codes (2,6) and (3,7)
                const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
                const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
                mma_16816(c, a0, bf[2 * j][0], bf[2 * j][1]);
                mma_16816(c, a1, bf[2 * j + 1][0], bf[2 * j + 1][1]);
            }
            const float2 s = half2_bits_to_float2(cur[i].s);
            acc[i][0] = fmaf(s.x, c[0], acc[i][0]);
            acc[i][1] = fmaf(s.x, c[1], acc[i][1]);
            acc[i][2] = fmaf(s.y, c[2], acc[i][2]);
            acc[i][3] = fmaf(s.y, c[3], acc[i][3]);
        }
        if (g + 1 < g1) {
#pragma unroll
            for (int i = 0; i < RT; ++i) cur[i] = nxt[i];
#pragma unroll
            for (int v = 0; v < 4; ++v) xc[v] = xn[v];
        }
    }
    // C fragment: (row r, batch 2t / 2t+1) and (row r + 8, same batches)
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        red[warp][16 * i + r][2 * t] = acc[i][0];
        red[warp][16 * i + r][2 * t + 1] = acc[i][1];
        red[warp][16 * i + r + 8][2 * t] = acc[i][2];
        red[warp][16 * i + r + 8][2 * t + 1] = acc[i][3];
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < RT * 16 * 8; idx += blockDim.x) {
        const int row = idx >> 3, b = idx & 7;
        const int n = n_base + row;
        if (b < B && n < N) {
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < kMmaWarps; ++w) v += red[w][row][b];
            y[(size_t)b * N + n] = float_to_half_bits_rn(v);
        }
    }
}

// ---------------------------------------------------------------------------
// Streaming GEMV for K % 256 == 0 (the decode shapes), batch 1..8*NT.
//
// Memory side: one producer warp per CTA streams the CTA tile's codes through
// a shared-memory ring (2-D TMA, one ROWS x 64-byte plane per group, two
// groups per stage).  The same warp turns x into the MMA's B fragments once
// per CTA: each producer lane loads the 32 x values that consumer lane `lane`
// needs for a group (per n-tile of 8 batch rows), permutes them into fragment
// order and stores them lane-major (conflict-free 16-byte loads for every
// consumer warp), and adds them up into the group sum X_g of its batch row.
// The consumers fetch the fp16 scales and zero-point words of their own rows
// from global memory one block of 8 groups ahead; the CTA's shared memory is
// the ring alone, so two CTAs fit on an SM.
//
// Compute side (warp-level mma.sync m16n8k16, batch = N): the codes go into
// the A fragment as fp16 *subnormals*.  Masking a word with 0x000F000F leaves
// two nibbles in the mantissa bits of two fp16 lanes, i.e. exactly q * 2^-24
// (and 0x00F000F0 gives q * 2^-20), one LOP3 per pair and no conversion or
// subtraction; the MMA multiplies them exactly.  The x lanes that meet the
// 2^-20 codes are pre-scaled by 2^-4 (exact for |x| >= 2^-10, below that the
// rounding is far inside the tolerance), so one MMA chain accumulates
// D = 2^-24 sum_k q x in fp32.  With X'_g = 2^-24 X_g (scaled by the
// producer) a group adds s (D - z X'_g) to the accumulator, and the result is
// scaled by 2^24 once at the end: y = 2^24 sum_g s_g (D_g - z_g X'_g).
// Each consumer warp owns RT m-tiles and NT n-tiles (RT*NT independent MMA
// chains, interleaved).  K is split over a thread-block cluster (DSMEM
// reduction into the leading CTA) when the tiles alone would leave SMs idle.
// A consumer makes its shared-memory reads visible to the async proxy
// (fence.proxy.async) before releasing a stage for the next TMA write.
// ---------------------------------------------------------------------------
constexpr uint32_t kStreamRingBudget = 110 * 1024;  // two CTAs per SM (228 KB, 1 KB reserved per CTA)
constexpr int kGPS = 2;                              // groups per stage (scales fetched as one 32-bit pair)

template <int CW, int RT, int NT>
struct StreamLayout {
    static constexpr int ROWS = CW * RT * 16;          // <= 256 (TMA box)
    static constexpr uint32_t PLANE = ROWS * 64;       // codes of one group
    static constexpr uint32_t W_BYTES = PLANE * kGPS;
    static constexpr uint32_t XF_BYTES = NT * 32 * 64; // B fragments of one group: [NT][4][32 lanes][16 B]
    static constexpr uint32_t OFF_XF = W_BYTES;
    static constexpr uint32_t OFF_XS = OFF_XF + XF_BYTES * kGPS;  // X'_g: [kGPS][8 * NT] fp32
    static constexpr uint32_t OFF_FL = OFF_XS + 32 * NT * kGPS;   // per group: fp32 factor of its scales (1 or 1/16)
    static constexpr uint32_t STAGE = (OFF_FL + 4 * kGPS + 127) / 128 * 128;  // 128-byte aligned TMA
    static constexpr int RING = (kStreamRingBudget / STAGE) < 3 ? 3
                                : (kStreamRingBudget / STAGE) > 8 ? 8 : (kStreamRingBudget / STAGE);
    static constexpr uint32_t OFF_BAR = RING * STAGE;
    static constexpr size_t SMEM = 128 + OFF_BAR + 256;
    static constexpr int THREADS = (CW + 1) * 32;
    static constexpr int MAX_B = 8 * NT;
};

struct StreamBars {
    uint64_t full[8];
    uint64_t empty[8];
    int abort;
};

// Read-only global loads kept where they are written (volatile): a prefetch that the compiler
// sank next to its use would expose the full memory latency.
__device__ __forceinline__ uint32_t ldg_nc_u32(const void *p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_nc_u4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ float2 lds64f(uint32_t a) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

__device__ __forceinline__ void sts32f(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

__device__ __forceinline__ float lds32f(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <int CW, int RT, int NT>
__global__ void __launch_bounds__(StreamLayout<CW, RT, NT>::THREADS, 2)
    gemv_w4a16_stream_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t *__restrict__ x,
                             const uint16_t *__restrict__ scales, const uint32_t *__restrict__ qzeros, int N, int K,
                             int B, int splits, uint16_t *__restrict__ y, unsigned int *status, uint64_t limit_ns) {
    using namespace sm100;
    using L = StreamLayout<CW, RT, NT>;
    constexpr int GPS = kGPS;
    extern __shared__ uint8_t stream_smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(stream_smem_raw) + 127) & ~uintptr_t(127));
    StreamBars *bar = reinterpret_cast<StreamBars *>(base + L::OFF_BAR);
    const uint32_t sbase = smem_u32(base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)blockIdx.x;
    const int n0 = blockIdx.y * L::ROWS;
    const int groups = K >> 7, zwords = (groups + 7) >> 3;
    const int nst = groups / (splits * GPS);  // stages of this CTA
    const int g_begin = rank * nst * GPS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::RING; ++s) {
            mbar_init(smem_u32(&bar->full[s]), 1 + 32);  // TMA transaction + the producer lanes' fragment stores
            mbar_init(smem_u32(&bar->empty[s]), CW);
        }
        bar->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == CW * 32) prefetch_tmap(&tmap_w);
    __syncthreads();
    const WaitCtl ctl{&bar->abort, status, limit_ns};

    float acc[RT][NT][4];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[i][n][0] = acc[i][n][1] = acc[i][n][2] = acc[i][n][3] = 0.0f;
    const int t = lane & 3, r = lane >> 2;

    if (warp == CW) {
        // ------------------------------------------------------------------ producer warp
        // Lane (r, t) prepares consumer lane (r, t)'s fragments: batch rows r + 8n,
        // the 32 values k = 32t .. 32t+31 of each group (the codes of the same k
        // sit in that lane's 16 code bytes).
        const uint16_t *xrow = x + (size_t)r * K + 32 * t;
        // One n-tile: x of stage i lives in xa (even i) or xb (odd i); each buffer is
        // refilled for stage i + 2 right after stage i's fragments are stored, so the
        // loads have a whole stage to arrive.
        auto load_x = [&](int i, uint4 (&xr)[NT][GPS][4]) {
            const int g = g_begin + i * GPS;
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int q = 0; q < GPS; ++q)
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        xr[n][q][v] = r + 8 * n < B ? ldg_nc_u4(xrow + (size_t)(8 * n) * K + (size_t)(g + q) * 128 + 8 * v)
                                                    : make_uint4(0u, 0u, 0u, 0u);
        };
        int issued = 0;
        auto produce = [&](int i, const uint4 (&xr)[NT][GPS][4]) -> bool {
            const int s = i % L::RING, u = i / L::RING;
            if (!__all_sync(0xffffffffu, wait_parity(smem_u32(&bar->empty[s]), (u & 1) ^ 1, ctl, 0x402))) return false;
            const uint32_t fb = smem_u32(&bar->full[s]);
            const uint32_t st = sbase + s * L::STAGE;
            const int g = g_begin + i * GPS;
            if (lane == 0) {
                mbar_arrive_expect_tx(fb, L::W_BYTES);
                // one 64-byte-pitch plane per group keeps the consumers' 16-byte loads conflict-free
#pragma unroll
                for (int q = 0; q < GPS; ++q) tma_load_2d(st + q * L::PLANE, &tmap_w, fb, (g + q) * 64, n0);
            }
            ++issued;
#pragma unroll
            for (int q = 0; q < GPS; ++q) {
                // Fragment k-step 2j: (x0,x4) and 2^-4 (x1,x5) of chunk j; 2j+1: (x2,x6) and 2^-4 (x3,x7).
                // The 2^-4 pre-scaling of the high-nibble lanes is exact unless some |x| < 2^-10
                // loses bits in fp16 (the round trip x * 2^-4 * 16 then differs from x).  If that
                // happens anywhere in the group (any lane, any batch row) and no |x| in the
                // low-nibble lanes reaches 4096, the group's fragments carry 16 x in the low-nibble
                // lanes and x in the high-nibble lanes instead (both exact), and its flag word
                // tells the consumers that D and X'_g come out 16 times larger.
                uint32_t inexact = 0u;
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 c = xr[n][q][j];
                        const uint32_t h0 = prmt_u(c.x, c.z, 0x7632u), h1 = prmt_u(c.y, c.w, 0x7632u);
                        inexact |= (hmul2_u(hmul2_u(h0, 0x2C002C00u), 0x4C004C00u) ^ h0) |
                                   (hmul2_u(hmul2_u(h1, 0x2C002C00u), 0x4C004C00u) ^ h1);
                    }
                bool x16 = __any_sync(0xffffffffu, inexact != 0u);
                if (x16) {  // rare: is 16 x finite for every low-nibble lane of the group?
                    uint32_t big = 0u;
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint4 c = xr[n][q][j];
                            // |x| >= 4096 (0x6C00) sets bit 15 of (|x| + 0x1400) in each half
                            big |= ((prmt_u(c.x, c.z, 0x5410u) & 0x7FFF7FFFu) + 0x14001400u) |
                                   ((prmt_u(c.y, c.w, 0x5410u) & 0x7FFF7FFFu) + 0x14001400u);
                        }
                    x16 = !__any_sync(0xffffffffu, (big & 0x80008000u) != 0u);
                }
                const uint32_t lo_scale = x16 ? 0x4C004C00u : 0x3C003C00u;   // 16 or 1
                const uint32_t hi_scale = x16 ? 0x3C003C00u : 0x2C002C00u;   // 1 or 2^-4
                const float xs_scale = x16 ? -9.5367431640625e-7f : -5.9604644775390625e-8f;  // -2^-20 / -2^-24
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    float sum0 = 0.0f, sum1 = 0.0f;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 c = xr[n][q][j];
                        sts128(st + L::OFF_XF + q * L::XF_BYTES + (n * 4 + j) * 512 + lane * 16,
                               hmul2_u(prmt_u(c.x, c.z, 0x5410u), lo_scale), hmul2_u(prmt_u(c.x, c.z, 0x7632u), hi_scale),
                               hmul2_u(prmt_u(c.y, c.w, 0x5410u), lo_scale), hmul2_u(prmt_u(c.y, c.w, 0x7632u), hi_scale));
                        const float2 f0 = half2_bits_to_float2(c.x), f1 = half2_bits_to_float2(c.y);
                        const float2 f2 = half2_bits_to_float2(c.z), f3 = half2_bits_to_float2(c.w);
                        sum0 += (f0.x + f1.x) + (f2.x + f3.x);
                        sum1 += (f0.y + f1.y) + (f2.y + f3.y);
                    }
                    float xg = sum0 + sum1;
                    xg += __shfl_xor_sync(0xffffffffu, xg, 1);
                    xg += __shfl_xor_sync(0xffffffffu, xg, 2);
                    // -2^-24 X_g (or -2^-20 X_g) of batch row r + 8n (exact scaling)
                    if (t == 0) sts32f(st + L::OFF_XS + (q * NT + n) * 32 + r * 4, xg * xs_scale);
                }
                if (lane == 0) sts32f(st + L::OFF_FL + q * 4, x16 ? 0.0625f : 1.0f);
            }
            mbar_arrive(fb);  // release: the fragments are visible to the consumers' acquire
            return true;
        };
        if (NT == 1) {
            uint4 xa[NT][GPS][4], xb[NT][GPS][4];
            load_x(0, xa);
            if (nst > 1) load_x(1, xb);
            for (int i = 0; i < nst; i += 2) {
                if (!produce(i, xa)) break;
                if (i + 2 < nst) load_x(i + 2, xa);
                if (i + 1 >= nst) break;
                if (!produce(i + 1, xb)) break;
                if (i + 3 < nst) load_x(i + 3, xb);
            }
        } else {  // two n-tiles: one stage of x in registers (the two-stage prefetch would spill)
            uint4 xa[NT][GPS][4];
            load_x(0, xa);
            for (int i = 0; i < nst; ++i) {
                if (!produce(i, xa)) break;
                if (i + 1 < nst) load_x(i + 1, xa);
            }
        }
        if (lane == 0 && bar->abort) {
            for (int s = 0; s < L::RING; ++s) {
                const int uses = issued > s ? (issued - s - 1) / L::RING + 1 : 0;
                if (uses) drain_parity(smem_u32(&bar->full[s]), (uses - 1) & 1, 2000000000ull, status, 0x410);
            }
        }
    } else {
        // ------------------------------------------------------------------ consumer warps
        const int wrow = warp * RT * 16;
        // this lane's rows are nl + 8 (2i + h); rows past N read no scales and are never stored
        const int nl = n0 + wrow + r;
        const uint16_t *srow = scales + (size_t)min(nl, N - 1) * groups;
        const uint32_t *zrow = qzeros + (size_t)min(nl, N - 1) * zwords;
        const size_t sstep = (size_t)8 * groups, zstep = (size_t)8 * zwords;
        // Scales and zero-point words travel per block of 4 stages (8 groups, one
        // zero word per row): lane t of a row quad holds the scale pair of the
        // block's stage t and hands it to its quad by shuffle, so a warp reads each
        // row's 16 scale bytes with one sector request.  The next block's words are
        // in flight while the current block is processed.
        const int nblk = (nst + 3) >> 2;
        uint32_t sw[RT][2], zw[RT][2], swn[RT][2], zwn[RT][2];
        auto fetch = [&](int blk, uint32_t (&sv)[RT][2], uint32_t (&zv)[RT][2]) {
            const int g0 = g_begin + blk * 8;
            const int gs = min(g0 + 2 * t, g_begin + 2 * (nst - 1));  // stage t of the block, clamped
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const bool in = nl + 16 * i + 8 * h < N;
                    sv[i][h] = in ? ldg_nc_u32(srow + (2 * i + h) * sstep + gs) : 0u;
                    zv[i][h] = in ? ldg_nc_u32(zrow + (2 * i + h) * zstep + (g0 >> 3)) : 0u;
                }
        };
        fetch(0, sw, zw);
        bool ok = true;
#pragma unroll 1
        for (int blk = 0; blk < nblk && ok; ++blk) {
            fetch(blk + 1 < nblk ? blk + 1 : blk, swn, zwn);
#pragma unroll 1
            for (int gs = 0; gs < 4; ++gs) {
                const int it = blk * 4 + gs;
                if (it >= nst) break;
                const int s = it % L::RING, u = it / L::RING;
                const int g = g_begin + it * GPS;
                uint32_t scw[RT][2];
#pragma unroll
                for (int i = 0; i < RT; ++i)
#pragma unroll
                    for (int h = 0; h < 2; ++h) scw[i][h] = __shfl_sync(0xffffffffu, sw[i][h], (lane & ~3) | gs);
                if (!__all_sync(0xffffffffu, wait_parity(smem_u32(&bar->full[s]), u & 1, ctl, 0x408))) {
                    ok = false;
                    break;
                }
                const uint32_t st = sbase + s * L::STAGE;
                const int zsh = 4 * (g & 7);
                // one group at a time (half the live fragments); the stage is released
                // once the last group's operands are in registers
#pragma unroll
                for (int q = 0; q < GPS; ++q) {
                    uint4 xv[NT][4];
                    uint4 wv[RT][2];
                    float2 xg[NT];
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            xv[n][v] = lds128(st + L::OFF_XF + q * L::XF_BYTES + (n * 4 + v) * 512 + lane * 16);
                        xg[n] = lds64f(st + L::OFF_XS + (q * NT + n) * 32 + t * 8);  // -X'_g of batches 2t, 2t+1
                    }
#pragma unroll
                    for (int i = 0; i < RT; ++i)
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            wv[i][h] = lds128(st + q * L::PLANE + (wrow + 16 * i + r + 8 * h) * 64 + t * 16);
                    if (q == GPS - 1) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&bar->empty[s]));
                    }
                    // RT * NT independent accumulation chains, interleaved k-step by k-step
                    float d[RT][NT][4];
#pragma unroll
                    for (int i = 0; i < RT; ++i)
#pragma unroll
                        for (int n = 0; n < NT; ++n) d[i][n][0] = d[i][n][1] = d[i][n][2] = d[i][n][3] = 0.0f;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
#pragma unroll
                        for (int hn = 0; hn < 2; ++hn) {
#pragma unroll
                            for (int i = 0; i < RT; ++i) {
                                const uint32_t wa = j == 0 ? wv[i][0].x : j == 1 ? wv[i][0].y : j == 2 ? wv[i][0].z : wv[i][0].w;
                                const uint32_t wb = j == 0 ? wv[i][1].x : j == 1 ? wv[i][1].y : j == 2 ? wv[i][1].z : wv[i][1].w;
                                const uint32_t ua = hn ? wa >> 8 : wa, ub = hn ? wb >> 8 : wb;
                                const uint32_t af[4] = {ua & 0x000F000Fu, ub & 0x000F000Fu, ua & 0x00F000F0u,
                                                        ub & 0x00F000F0u};
#pragma unroll
                                for (int n = 0; n < NT; ++n) {
                                    if (hn == 0)
                                        mma_16816(d[i][n], af, xv[n][j].x, xv[n][j].y);
                                    else
                                        mma_16816(d[i][n], af, xv[n][j].z, xv[n][j].w);
                                }
                            }
                        }
                    }
                    // acc += s (D - z X'_g)  (rows r and r + 8 of each m-tile); a group whose fragments
                    // carry 16 x in the low-nibble lanes has D and X'_g 16 times larger
                    const float gf = lds32f(st + L::OFF_FL + q * 4);  // 1 or 1/16
#pragma unroll
                    for (int i = 0; i < RT; ++i) {
                        const float s0 = half_bits_to_float((uint16_t)(scw[i][0] >> (16 * q))) * gf;
                        const float s1 = half_bits_to_float((uint16_t)(scw[i][1] >> (16 * q))) * gf;
                        const float z0 = (float)((zw[i][0] >> (zsh + 4 * q)) & 0xFu);
                        const float z1 = (float)((zw[i][1] >> (zsh + 4 * q)) & 0xFu);
#pragma unroll
                        for (int n = 0; n < NT; ++n) {
                            acc[i][n][0] = fmaf(s0, fmaf(z0, xg[n].x, d[i][n][0]), acc[i][n][0]);
                            acc[i][n][1] = fmaf(s0, fmaf(z0, xg[n].y, d[i][n][1]), acc[i][n][1]);
                            acc[i][n][2] = fmaf(s1, fmaf(z1, xg[n].x, d[i][n][2]), acc[i][n][2]);
                            acc[i][n][3] = fmaf(s1, fmaf(z1, xg[n].y, d[i][n][3]), acc[i][n][3]);
                        }
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    sw[i][h] = swn[i][h];
                    zw[i][h] = zwn[i][h];
                }
        }
    }

    // ---------------------------------------------------------------------- results (times 2^24)
    constexpr float kUnscale = 16777216.0f;
    const bool cons = warp < CW;
    const int wrow = warp * RT * 16;
    if (splits == 1) {
        if (cons && !bar->abort) {
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = n0 + wrow + 16 * i + r + 8 * h;
                        const int b0 = 8 * n + 2 * t;
                        if (row < N) {
                            if (b0 < B) y[(size_t)b0 * N + row] = float_to_half_bits_rn(acc[i][n][2 * h] * kUnscale);
                            if (b0 + 1 < B)
                                y[(size_t)(b0 + 1) * N + row] = float_to_half_bits_rn(acc[i][n][2 * h + 1] * kUnscale);
                        }
                    }
        }
    } else {
        cluster_sync();  // every CTA of the cluster is done with its ring
        if (cons && rank != 0) {
            const uint32_t red = mapa_shared(sbase, 0);
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = wrow + 16 * i + r + 8 * h;
                        const uint32_t a = red + (uint32_t)((((rank - 1) * L::ROWS + row) * NT + n) * 8 + 2 * t) * 4;
                        asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(acc[i][n][2 * h]),
                                     "f"(acc[i][n][2 * h + 1])
                                     : "memory");
                    }
        }
        cluster_sync();  // partials landed in the leading CTA
        if (cons && rank == 0 && !bar->abort) {
            const float *red = reinterpret_cast<const float *>(base);
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = wrow + 16 * i + r + 8 * h;
                        float v0 = acc[i][n][2 * h], v1 = acc[i][n][2 * h + 1];
                        for (int sl = 0; sl < splits - 1; ++sl) {
                            v0 += red[((sl * L::ROWS + row) * NT + n) * 8 + 2 * t];
                            v1 += red[((sl * L::ROWS + row) * NT + n) * 8 + 2 * t + 1];
                        }
                        const int gr = n0 + row, b0 = 8 * n + 2 * t;
                        if (gr < N) {
                            if (b0 < B) y[(size_t)b0 * N + gr] = float_to_half_bits_rn(v0 * kUnscale);
                            if (b0 + 1 < B) y[(size_t)(b0 + 1) * N + gr] = float_to_half_bits_rn(v1 * kUnscale);
                        }
                    }
        }
    }
}

template <int CW, int RT, int NT>
wq_status launch_stream(const uint16_t *x, int B, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                        int K, int splits, uint16_t *y, cudaStream_t st, const char *who) {
    using L = StreamLayout<CW, RT, NT>;
    unsigned int *status = device_status_word();
    if (!status) return WQ_ERR_CUDA;
    CUtensorMap tw;
    if (!encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qw, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, 64,
                        L::ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        return WQ_ERR_CUDA;
    auto kern = gemv_w4a16_stream_kernel<CW, RT, NT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: cudaFuncSetAttribute: %s", who, cudaGetErrorString(e));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(splits, (N + L::ROWS - 1) / L::ROWS, 1);
    cfg.blockDim = dim3(L::THREADS);
    cfg.dynamicSmemBytes = L::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tw, x, sc, qz, N, K, B, splits, y, status, wait_limit());
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: launch failed: %s", who, cudaGetErrorString(e));
    return WQ_OK;
}

// Tile height and K split of the streaming GEMV.  Two CTAs are resident per
// SM; the split (cluster size, at most 8, keeping every CTA's start on a
// zero-point word, partials fitting the leading CTA's ring) is the smallest one
// that reaches the best fill of those slots over whole waves.  Measured on
// B200, for one and for two n-tiles: the 224-row tile (7 consumer warps x 2
// m-tiles, 8 warps and at most 128 registers per thread, so that 16 warps
// share an SM) is the fastest; the 128-row tile serves matrices with too few
// 224-row tiles.  (Unaligned splits that fill every slot, e.g. 8-CTA clusters
// on the 28672-wide down projection, measured slower.)
template <typename L>
int stream_splits(int N, int K, int sms) {
    const int tiles = (N + L::ROWS - 1) / L::ROWS;
    const long long slots = 2ll * sms;
    int best = 1;
    double best_fill = 0.0;
    for (int s = 1; s <= 8; ++s) {
        if (s > 1 && (K / 128) % (8 * s)) continue;  // every CTA starts on a zero-point word
        if ((size_t)(s - 1) * L::ROWS * L::MAX_B * 4 > L::OFF_BAR) continue;
        const long long ctas = (long long)tiles * s;
        const long long waves = (ctas + slots - 1) / slots;
        const double fill = (double)ctas / (double)(waves * slots);
        if (fill > best_fill + 1e-9) {
            best_fill = fill;
            best = s;
        }
    }
    return best;
}

template <int NT, int BCW, int BRT>
wq_status gemv_stream_nt(const uint16_t *x, int B, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                         int K, uint16_t *y, cudaStream_t st, const char *who) {
    const int sms = num_sms();
    using Big = StreamLayout<BCW, BRT, NT>;
    using Small = StreamLayout<4, 2, NT>;
    const int tiles_big = (N + Big::ROWS - 1) / Big::ROWS;
    if (tiles_big * 8 >= 2 * sms)
        return launch_stream<BCW, BRT, NT>(x, B, qw, sc, qz, N, K, stream_splits<Big>(N, K, sms), y, st, who);
    return launch_stream<4, 2, NT>(x, B, qw, sc, qz, N, K, stream_splits<Small>(N, K, sms), y, st, who);
}

}  // namespace

// Batch 1..16 with K % 256 == 0, group size 128 (also serves wq_gemm_w4a16 for up to 32 rows,
// in passes of up to 16).
wq_status gemv_stream(const uint16_t *x, int B, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                      int K, uint16_t *y, cudaStream_t st, const char *who) {
    if (B <= 8) return gemv_stream_nt<1, 7, 2>(x, B, qw, sc, qz, N, K, y, st, who);
    return gemv_stream_nt<2, 7, 2>(x, B, qw, sc, qz, N, K, y, st, who);
}

namespace {

template <int RT>
cudaError_t launch_mma(const uint16_t *x, int B, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                       int K, uint16_t *y, cudaStream_t st) {
    const int blocks = (N + RT * 16 - 1) / (RT * 16);
    gemv_w4a16_mma_kernel<RT><<<blocks, kMmaWarps * 32, 0, st>>>(x, B, qw, sc, qz, N, K, y);
    return cudaGetLastError();
}

template <int B, int R, bool BF>
cudaError_t launch_br(const uint16_t *x, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                      int K, int g, uint16_t *y, cudaStream_t st) {
    const int rows_per_block = kWarps * R;
    const int blocks = (N + rows_per_block - 1) / rows_per_block;
    gemv_w4a16_kernel<B, R, BF><<<blocks, kWarps * 32, 0, st>>>(x, qw, sc, qz, N, K, g, y);
    return cudaGetLastError();
}

template <int B, bool BF = false>
cudaError_t launch_b(const uint16_t *x, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                     int K, int g, uint16_t *y, cudaStream_t st) {
    // Two rows per warp when that still gives every SM several CTAs.
    const long long blocks2 = (N + kWarps * 2 - 1) / (kWarps * 2);
    if (blocks2 >= 6ll * num_sms()) return launch_br<B, 2, BF>(x, qw, sc, qz, N, K, g, y, st);
    return launch_br<B, 1, BF>(x, qw, sc, qz, N, K, g, y, st);
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_gemv_w4a16(const uint16_t *x, int B, const uint32_t *qweight, const uint16_t *scales,
                                   const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y,
                                   void *stream) {
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(qweight, "qweight");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE_PTR(qzeros, "qzeros");
    WQ_REQUIRE_PTR(y, "y");
    WQ_REQUIRE(N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_gemv_w4a16: N and K must be positive (N=%d K=%d)", N, K);
    WQ_REQUIRE(B >= 1 && B <= 8, WQ_ERR_UNSUPPORTED, "wq_gemv_w4a16: B must be 1..8 (got %d)", B);
    WQ_REQUIRE(group_size == 32 || group_size == 64 || group_size == 128 || group_size == 256,
               WQ_ERR_UNSUPPORTED, "wq_gemv_w4a16: group_size must be 32, 64, 128 or 256 (got %d)", group_size);
    WQ_REQUIRE(K % group_size == 0, WQ_ERR_INVALID_ARG,
               "wq_gemv_w4a16: K (%d) must be a multiple of group_size (%d)", K, group_size);
    cudaStream_t st = wq::as_stream(stream);
    cudaError_t e;
    if (group_size == 128 && K % 256 == 0) return wq::gemv_stream(x, B, qweight, scales, qzeros, N, K, y, st, "wq_gemv_w4a16");
    if (group_size == 128) {
        // Two 16-row MMA tiles per CTA when that still gives every SM several CTAs.
        const long long blocks2 = (N + 31) / 32;
        e = blocks2 >= 4ll * wq::num_sms() ? wq::launch_mma<2>(x, B, qweight, scales, qzeros, N, K, y, st)
                                           : wq::launch_mma<1>(x, B, qweight, scales, qzeros, N, K, y, st);
        if (e != cudaSuccess)
            return wq::fail(WQ_ERR_CUDA, "wq_gemv_w4a16: launch failed: %s", cudaGetErrorString(e));
        return WQ_OK;
    }
    switch (B) {
        case 1: e = wq::launch_b<1>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 2: e = wq::launch_b<2>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 3: e = wq::launch_b<3>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 4: e = wq::launch_b<4>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 5: e = wq::launch_b<5>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 6: e = wq::launch_b<6>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 7: e = wq::launch_b<7>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        default: e = wq::launch_b<8>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
    }
    if (e != cudaSuccess) return wq::fail(WQ_ERR_CUDA, "wq_gemv_w4a16: launch failed: %s", cudaGetErrorString(e));
    return WQ_OK;
}

// bf16 activations and output, any group size: the CUDA-core kernel (fp32 products of the exact
// q - z and the exactly converted x, group scale applied in fp32, one rounding to bf16 at the end).
extern "C" wq_status wq_gemv_w4a16_bf16(const uint16_t *x, int B, const uint32_t *qweight, const uint16_t *scales,
                                        const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y,
                                        void *stream) {
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(qweight, "qweight");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE_PTR(qzeros, "qzeros");
    WQ_REQUIRE_PTR(y, "y");
    WQ_REQUIRE(N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_gemv_w4a16_bf16: N and K must be positive (N=%d K=%d)", N, K);
    WQ_REQUIRE(B >= 1 && B <= 8, WQ_ERR_UNSUPPORTED, "wq_gemv_w4a16_bf16: B must be 1..8 (got %d)", B);
    WQ_REQUIRE(group_size == 32 || group_size == 64 || group_size == 128 || group_size == 256, WQ_ERR_UNSUPPORTED,
               "wq_gemv_w4a16_bf16: group_size must be 32, 64, 128 or 256 (got %d)", group_size);
    WQ_REQUIRE(K % group_size == 0, WQ_ERR_INVALID_ARG,
               "wq_gemv_w4a16_bf16: K (%d) must be a multiple of group_size (%d)", K, group_size);
    cudaStream_t st = wq::as_stream(stream);
    cudaError_t e;
    switch (B) {
        case 1: e = wq::launch_b<1, true>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 2: e = wq::launch_b<2, true>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 3: e = wq::launch_b<3, true>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 4: e = wq::launch_b<4, true>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 5: e = wq::launch_b<5, true>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 6: e = wq::launch_b<6, true>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        case 7: e = wq::launch_b<7, true>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
        default: e = wq::launch_b<8, true>(x, qweight, scales, qzeros, N, K, group_size, y, st); break;
    }
    if (e != cudaSuccess)
        return wq::fail(WQ_ERR_CUDA, "wq_gemv_w4a16_bf16: launch failed: %s", cudaGetErrorString(e));
    return WQ_OK;
}
