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
// Work decomposition: a warp owns R weight rows and walks K in steps of 1024
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

template <int B, int R>
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
                xf[4 * v + 0] = half2_bits_to_float2(xv.x);
                xf[4 * v + 1] = half2_bits_to_float2(xv.y);
                xf[4 * v + 2] = half2_bits_to_float2(xv.z);
                xf[4 * v + 3] = half2_bits_to_float2(xv.w);
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
                for (int b = 0; b < B; ++b) y[(size_t)b * N + row0 + r] = float_to_half_bits_rn(acc[r][b]);
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
// Streaming variant of the MMA GEMV for K % 1024 == 0 (the decode shapes).
// Small per-group loads of scales, zero points and x through L1 leave warps
// waiting on long scoreboards, and register prefetching keeps too few weight
// bytes in flight; here one producer warp per CTA streams everything through
// shared memory, so ~90 KB per CTA are in flight and the consumer warps only
// read shared memory:
//   - per group (128 codes): the CTA tile's codes (2-D TMA, ROWS x 64 B) and
//     x rows 0..7 (2-D TMA, 8 x 128 fp16; rows >= B arrive zero-filled, which
//     is exactly the MMA's padding), into a kGRing-deep ring;
//   - per block of 8 groups: the tile's fp16 scales (2-D TMA, ROWS x 16 B)
//     and zero-point words (cp.async, 4 B per row), double-buffered.
// All 8 consumer warps walk the same groups, each owning RT*16 rows, so no
// cross-warp reduction is needed.  When the tiles alone would leave SMs idle,
// K is split across the CTAs of a thread-block cluster and the fp32 partial
// results are summed in the leading CTA through distributed shared memory.
// A consumer makes its shared-memory reads visible to the async proxy
// (fence.proxy.async) before releasing a stage for the next TMA write.
// ---------------------------------------------------------------------------
constexpr int kConsumerWarps = 8;
constexpr int kGRing = 5;

template <int RT>
struct StreamLayout {
    static constexpr int ROWS = kConsumerWarps * RT * 16;
    static constexpr uint32_t W_BYTES = ROWS * 64;
    static constexpr uint32_t X_BYTES = 8 * 128 * 2;
    static constexpr uint32_t STAGE = W_BYTES + X_BYTES;
    static constexpr uint32_t S_BYTES = ROWS * 16;
    static constexpr uint32_t Z_BYTES = ROWS * 4;
    static constexpr uint32_t OFF_S = kGRing * STAGE;
    static constexpr uint32_t OFF_Z = OFF_S + 2 * S_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_Z + 2 * Z_BYTES;
    static constexpr size_t SMEM = 128 + OFF_BAR + 256;
};

struct StreamBars {
    uint64_t wfull[kGRing];
    uint64_t wempty[kGRing];
    uint64_t sfull[2];
    uint64_t sempty[2];
    int abort;
};

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

template <int RT>
__global__ void __launch_bounds__((kConsumerWarps + 1) * 32)
    gemv_w4a16_stream_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                             const __grid_constant__ CUtensorMap tmap_s, const uint32_t *__restrict__ qzeros, int N,
                             int K, int B, int splits, uint16_t *__restrict__ y, unsigned int *status,
                             uint64_t limit_ns) {
    using namespace sm100;
    using L = StreamLayout<RT>;
    extern __shared__ uint8_t stream_smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(stream_smem_raw) + 127) & ~uintptr_t(127));
    StreamBars *bar = reinterpret_cast<StreamBars *>(base + L::OFF_BAR);
    const uint32_t sbase = smem_u32(base);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)blockIdx.x;
    const int n0 = blockIdx.y * L::ROWS;
    const int groups = K >> 7, zwords = (groups + 7) >> 3;
    const int ng = groups / splits, g_begin = rank * ng, nsb = ng >> 3;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGRing; ++s) {
            mbar_init(smem_u32(&bar->wfull[s]), 1);
            mbar_init(smem_u32(&bar->wempty[s]), kConsumerWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&bar->sfull[b]), 1 + 32);
            mbar_init(smem_u32(&bar->sempty[b]), kConsumerWarps);
        }
        bar->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x == kConsumerWarps * 32) {
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_s);
    }
    __syncthreads();
    const WaitCtl ctl{&bar->abort, status, limit_ns};

    float acc[RT][4];
#pragma unroll
    for (int i = 0; i < RT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    const int t = lane & 3, r = lane >> 2;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------------ producer warp
        int issued = 0, sblocks = 0;
        bool ok = true;
        for (int sb = 0; sb < nsb && ok; ++sb) {
            const int b = sb & 1;
            ok = __all_sync(0xffffffffu, wait_parity(smem_u32(&bar->sempty[b]), ((sb >> 1) & 1) ^ 1, ctl, 0x401));
            if (!ok) break;
            const int blk = (g_begin >> 3) + sb;
            if (lane == 0) {
                mbar_arrive_expect_tx(smem_u32(&bar->sfull[b]), L::S_BYTES);
                tma_load_2d(sbase + L::OFF_S + b * L::S_BYTES, &tmap_s, smem_u32(&bar->sfull[b]), blk * 8, n0);
            }
            for (int row = lane; row < L::ROWS; row += 32)
                cp_async_4(sbase + L::OFF_Z + b * L::Z_BYTES + row * 4,
                           qzeros + (size_t)min(n0 + row, N - 1) * zwords + blk);
            cp_async_arrive_noinc(smem_u32(&bar->sfull[b]));
            ++sblocks;
            for (int gg = 0; gg < 8; ++gg) {
                const int i = sb * 8 + gg, s = i % kGRing, u = i / kGRing;
                if (lane == 0) {
                    if (!wait_parity(smem_u32(&bar->wempty[s]), (u & 1) ^ 1, ctl, 0x402)) {
                        ok = false;
                    } else {
                        const uint32_t fb = smem_u32(&bar->wfull[s]);
                        mbar_arrive_expect_tx(fb, L::STAGE);
                        tma_load_2d(sbase + s * L::STAGE, &tmap_w, fb, (g_begin + i) * 64, n0);
                        tma_load_2d(sbase + s * L::STAGE + L::W_BYTES, &tmap_x, fb, (g_begin + i) * 128, 0);
                        ++issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0 && bar->abort) {
            for (int s = 0; s < kGRing; ++s) {
                const int uses = issued > s ? (issued - s - 1) / kGRing + 1 : 0;
                if (uses) drain_parity(smem_u32(&bar->wfull[s]), (uses - 1) & 1, 2000000000ull, status, 0x410);
            }
            for (int b = 0; b < 2; ++b) {
                const int uses = sblocks > b ? (sblocks - b - 1) / 2 + 1 : 0;
                if (uses) drain_parity(smem_u32(&bar->sfull[b]), (uses - 1) & 1, 2000000000ull, status, 0x410);
            }
        }
    } else {
        // ------------------------------------------------------------------ consumer warps
        const int wrow = warp * RT * 16;
        bool ok = true;
        for (int sb = 0; sb < nsb && ok; ++sb) {
            const int b = sb & 1;
            ok = __all_sync(0xffffffffu, wait_parity(smem_u32(&bar->sfull[b]), (sb >> 1) & 1, ctl, 0x404));
            if (!ok) break;
            uint4 sreg[RT][2];
            uint32_t zreg[RT][2];
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = wrow + 16 * i + r + 8 * h;
                    sreg[i][h] = lds128(sbase + L::OFF_S + b * L::S_BYTES + row * 16);
                    zreg[i][h] = lds32(sbase + L::OFF_Z + b * L::Z_BYTES + row * 4);
                }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&bar->sempty[b]));
#pragma unroll
            for (int gg = 0; gg < 8; ++gg) {
                const int i_st = sb * 8 + gg, s = i_st % kGRing, u = i_st / kGRing;
                ok = __all_sync(0xffffffffu, wait_parity(smem_u32(&bar->wfull[s]), u & 1, ctl, 0x408));
                if (!ok) break;
                const uint32_t st = sbase + s * L::STAGE;
                uint4 xv[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) xv[v] = lds128(st + L::W_BYTES + r * 256 + t * 64 + v * 16);
                uint4 wv[RT][2];
#pragma unroll
                for (int i = 0; i < RT; ++i)
#pragma unroll
                    for (int h = 0; h < 2; ++h) wv[i][h] = lds128(st + (wrow + 16 * i + r + 8 * h) * 64 + t * 16);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&bar->wempty[s]));
                uint32_t bf[8][2];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    bf[2 * j][0] = prmt_u(xv[j].x, xv[j].z, 0x5410u);
                    bf[2 * j][1] = prmt_u(xv[j].x, xv[j].z, 0x7632u);
                    bf[2 * j + 1][0] = prmt_u(xv[j].y, xv[j].w, 0x5410u);
                    bf[2 * j + 1][1] = prmt_u(xv[j].y, xv[j].w, 0x7632u);
                }
#pragma unroll
                for (int i = 0; i < RT; ++i) {
                    const uint32_t z0 = (zreg[i][0] >> (4 * gg)) & 0xFu, z1 = (zreg[i][1] >> (4 * gg)) & 0xFu;
                    const uint32_t zlo0 = 0xE400E400u + z0 * 0x00010001u, zhi0 = 0xD400D400u + z0 * 0x00100010u;
                    const uint32_t zlo1 = 0xE400E400u + z1 * 0x00010001u, zhi1 = 0xD400D400u + z1 * 0x00100010u;
                    float ce[4] = {0.0f, 0.0f, 0.0f, 0.0f}, co[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    const uint32_t wa[4] = {wv[i][0].x, wv[i][0].y, wv[i][0].z, wv[i][0].w};
                    const uint32_t wb[4] = {wv[i][1].x, wv[i][1].y, wv[i][1].z, wv[i][1].w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t pa[4], pb[4];
                        dequant_pairs(wa[j], zlo0, zhi0, pa);
                        dequant_pairs(wb[j], zlo1, zhi1, pb);
                        const uint32_t a0[4] = {pa[0], pb[0], pa[1], pb[1]};
                        const uint32_t a1[4] = {pa[2], pb[2], pa[3], pb[3]};
                        mma_16816(ce, a0, bf[2 * j][0], bf[2 * j][1]);
                        mma_16816(co, a1, bf[2 * j + 1][0], bf[2 * j + 1][1]);
                    }
                    const uint32_t sw0 = gg < 2 ? sreg[i][0].x : gg < 4 ? sreg[i][0].y : gg < 6 ? sreg[i][0].z : sreg[i][0].w;
                    const uint32_t sw1 = gg < 2 ? sreg[i][1].x : gg < 4 ? sreg[i][1].y : gg < 6 ? sreg[i][1].z : sreg[i][1].w;
                    const float s0 = half_bits_to_float((uint16_t)((gg & 1) ? (sw0 >> 16) : (sw0 & 0xFFFFu)));
                    const float s1 = half_bits_to_float((uint16_t)((gg & 1) ? (sw1 >> 16) : (sw1 & 0xFFFFu)));
                    acc[i][0] = fmaf(s0, ce[0] + co[0], acc[i][0]);
                    acc[i][1] = fmaf(s0, ce[1] + co[1], acc[i][1]);
                    acc[i][2] = fmaf(s1, ce[2] + co[2], acc[i][2]);
                    acc[i][3] = fmaf(s1, ce[3] + co[3], acc[i][3]);
                }
            }
        }
    }

    // ---------------------------------------------------------------------- results
    const bool cons = warp < kConsumerWarps;
    const int wrow = warp * RT * 16;
    if (splits == 1) {
        if (cons && !bar->abort) {
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int n = n0 + wrow + 16 * i + r + 8 * h;
                    if (n < N) {
                        if (2 * t < B) y[(size_t)(2 * t) * N + n] = float_to_half_bits_rn(acc[i][2 * h]);
                        if (2 * t + 1 < B) y[(size_t)(2 * t + 1) * N + n] = float_to_half_bits_rn(acc[i][2 * h + 1]);
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
                for (int h = 0; h < 2; ++h) {
                    const int row = wrow + 16 * i + r + 8 * h;
                    const uint32_t a = red + (uint32_t)(((rank - 1) * L::ROWS + row) * 8 + 2 * t) * 4;
                    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(acc[i][2 * h]),
                                 "f"(acc[i][2 * h + 1])
                                 : "memory");
                }
        }
        cluster_sync();  // partials landed in the leading CTA
        if (cons && rank == 0 && !bar->abort) {
            const float *red = reinterpret_cast<const float *>(base);
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int row = wrow + 16 * i + r + 8 * h;
                    float v0 = acc[i][2 * h], v1 = acc[i][2 * h + 1];
                    for (int sl = 0; sl < splits - 1; ++sl) {
                        v0 += red[(sl * L::ROWS + row) * 8 + 2 * t];
                        v1 += red[(sl * L::ROWS + row) * 8 + 2 * t + 1];
                    }
                    const int n = n0 + row;
                    if (n < N) {
                        if (2 * t < B) y[(size_t)(2 * t) * N + n] = float_to_half_bits_rn(v0);
                        if (2 * t + 1 < B) y[(size_t)(2 * t + 1) * N + n] = float_to_half_bits_rn(v1);
                    }
                }
        }
    }
}

template <int RT>
wq_status launch_stream(const uint16_t *x, int B, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                        int K, int splits, uint16_t *y, cudaStream_t st) {
    using L = StreamLayout<RT>;
    unsigned int *status = device_status_word();
    if (!status) return WQ_ERR_CUDA;
    CUtensorMap tw, tx, ts;
    if (!encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qw, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, 64,
                        L::ROWS, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x, (uint64_t)K, (uint64_t)B, (uint64_t)K * 2, 128, 8,
                        CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tmap_2d(&ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, sc, (uint64_t)K / 128, (uint64_t)N,
                        (uint64_t)K / 64, 8, L::ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        return WQ_ERR_CUDA;
    auto kern = gemv_w4a16_stream_kernel<RT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_gemv_w4a16: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(splits, (N + L::ROWS - 1) / L::ROWS, 1);
    cfg.blockDim = dim3((kConsumerWarps + 1) * 32);
    cfg.dynamicSmemBytes = L::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tw, tx, ts, qz, N, K, B, splits, y, status, wait_limit());
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_gemv_w4a16: launch failed: %s", cudaGetErrorString(e));
    return WQ_OK;
}

// Tile height (RT) and K split of the streaming GEMV: the cluster size divides
// K/1024 (whole blocks of 8 groups per CTA), at most 8, and the partial results
// fit the leading CTA's ring; the choice fills the SMs' CTA slots in the fewest,
// fullest waves, preferring the taller tile (fewer x fragments per weight).
wq_status gemv_stream(const uint16_t *x, int B, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                      int K, uint16_t *y, cudaStream_t st) {
    const int blocks8 = K / 1024;
    const int sms = num_sms();
    int best_rt = 1, best_s = 1;
    double best = -1.0;
    for (int rt = 2; rt >= 1; --rt) {
        const int rows = kConsumerWarps * rt * 16;
        const size_t smem = rt == 2 ? StreamLayout<2>::SMEM : StreamLayout<1>::SMEM;
        const size_t ring = rt == 2 ? (size_t)StreamLayout<2>::OFF_S : (size_t)StreamLayout<1>::OFF_S;
        const int per_sm = (int)std::min<size_t>(2048 / ((kConsumerWarps + 1) * 32), 227 * 1024 / smem);
        const int tiles = (N + rows - 1) / rows;
        for (int s = 1; s <= 8; ++s) {
            if (blocks8 % s) continue;
            if ((size_t)(s - 1) * rows * 8 * 4 > ring) continue;
            const double waves = (double)tiles * s / ((double)sms * per_sm);
            double score = waves / std::ceil(waves) + (rt == 2 ? 0.03 : 0.0) - 0.002 * s;
            if (waves < 0.5) score -= 1.0;  // leaves most SMs idle
            if (score > best) {
                best = score;
                best_rt = rt;
                best_s = s;
            }
        }
    }
    return best_rt == 2 ? launch_stream<2>(x, B, qw, sc, qz, N, K, best_s, y, st)
                        : launch_stream<1>(x, B, qw, sc, qz, N, K, best_s, y, st);
}

template <int RT>
cudaError_t launch_mma(const uint16_t *x, int B, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                       int K, uint16_t *y, cudaStream_t st) {
    const int blocks = (N + RT * 16 - 1) / (RT * 16);
    gemv_w4a16_mma_kernel<RT><<<blocks, kMmaWarps * 32, 0, st>>>(x, B, qw, sc, qz, N, K, y);
    return cudaGetLastError();
}

template <int B, int R>
cudaError_t launch_br(const uint16_t *x, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                      int K, int g, uint16_t *y, cudaStream_t st) {
    const int rows_per_block = kWarps * R;
    const int blocks = (N + rows_per_block - 1) / rows_per_block;
    gemv_w4a16_kernel<B, R><<<blocks, kWarps * 32, 0, st>>>(x, qw, sc, qz, N, K, g, y);
    return cudaGetLastError();
}

template <int B>
cudaError_t launch_b(const uint16_t *x, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                     int K, int g, uint16_t *y, cudaStream_t st) {
    // Two rows per warp when that still gives every SM several CTAs.
    const long long blocks2 = (N + kWarps * 2 - 1) / (kWarps * 2);
    if (blocks2 >= 6ll * num_sms()) return launch_br<B, 2>(x, qw, sc, qz, N, K, g, y, st);
    return launch_br<B, 1>(x, qw, sc, qz, N, K, g, y, st);
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
    if (group_size == 128 && K % 1024 == 0) return wq::gemv_stream(x, B, qweight, scales, qzeros, N, K, y, st);
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
