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
#include "wq_device.cuh"
#include "wq_host.h"

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
