// W8A16 GEMV: INT8 per-channel weights, fp16 activations, batch 1..8.
//
// Source: "How quantization works", section "Mainstream schemes at a glance"
// (W8A16: INT8 weights, 16-bit activations, speeds up weight reads) and the
// per-channel INT8 of "The math of quantization" / q8_per_row.
//
//   y[b][n] = fp16_rn( sw[n] * sum_k q[n][k] * x[b][k] )     fp32 accumulation
//
// Same decomposition as the W4A16 GEMV: a warp owns R rows; lane l of step t
// reads 16 int8 codes (chunk 32 t + l) of each row with a 16-byte streaming
// load.  Codes become exact floats without a conversion instruction: flipping
// the sign bit gives the byte q + 128, a byte permute drops it into the
// mantissa of 2^23 (float 2^23 + q + 128) and a packed subtract of 2^23 + 128
// leaves q.
#include "wq_device.cuh"
#include "wq_host.h"

namespace wq {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float byte_as_float(uint32_t w, uint32_t sel) {
    // d = [byte sel of w, 0x00, 0x00, 0x4B]  ->  2^23 + byte
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(0x4B000000u), "r"(sel));
    return __uint_as_float(d);
}

template <int B, int R>
__global__ void __launch_bounds__(kWarps * 32) gemv_w8a16_kernel(const uint16_t *__restrict__ x,
                                                                 const int8_t *__restrict__ wq,
                                                                 const float *__restrict__ sw, int N, int K,
                                                                 uint16_t *__restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int row0 = (blockIdx.x * kWarps + (threadIdx.x >> 5)) * R;
    if (row0 >= N) return;
    const int chunks = K >> 4;  // 16-code chunks per row
    const float2 bias = make_float2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)

    float2 acc[R][B];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) acc[r][b] = make_float2(0.0f, 0.0f);

    // Two rows per warp: four chunk steps unrolled keep more 16-byte loads in flight per lane
    // (measured on B200: 28672x8192 batch 1 51.8 -> 49.6 us, batch 4 111 -> 99 us); one row per
    // warp (the shapes with few rows) measured slower unrolled.
#pragma unroll (R == 2 ? 4 : 1)
    for (int c = lane; c < chunks; c += 32) {
        const int k0 = c << 4;
        float2 wf[R][8];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int n = min(row0 + r, N - 1);
            const uint4 v = ld_stream_u4(wq + (size_t)n * K + k0);
            const uint32_t words[4] = {v.x ^ 0x80808080u, v.y ^ 0x80808080u, v.z ^ 0x80808080u,
                                       v.w ^ 0x80808080u};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 lo = make_float2(byte_as_float(words[q], 0x7650u), byte_as_float(words[q], 0x7651u));
                const float2 hi = make_float2(byte_as_float(words[q], 0x7652u), byte_as_float(words[q], 0x7653u));
                wf[r][2 * q] = __fadd2_rn(lo, bias);
                wf[r][2 * q + 1] = __fadd2_rn(hi, bias);
            }
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const uint16_t *xp = x + (size_t)b * K + k0;
            const uint4 x0 = ld_shared_ro_u4(xp), x1 = ld_shared_ro_u4(xp + 8);
            const float2 xf[8] = {half2_bits_to_float2(x0.x), half2_bits_to_float2(x0.y),
                                  half2_bits_to_float2(x0.z), half2_bits_to_float2(x0.w),
                                  half2_bits_to_float2(x1.x), half2_bits_to_float2(x1.y),
                                  half2_bits_to_float2(x1.z), half2_bits_to_float2(x1.w)};
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[r][b] = __ffma2_rn(wf[r][i], xf[i], acc[r][b]);
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const float s = __ldg(sw + min(row0 + r, N - 1));
#pragma unroll
        for (int b = 0; b < B; ++b) {
            float v = acc[r][b].x + acc[r][b].y;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            if (lane == 0 && row0 + r < N) y[(size_t)b * N + row0 + r] = float_to_half_bits_rn(s * v);
        }
    }
}

template <int B, int R>
cudaError_t launch_br(const uint16_t *x, const int8_t *wq, const float *sw, int N, int K, uint16_t *y,
                      cudaStream_t st) {
    const int rows_per_block = kWarps * R;
    gemv_w8a16_kernel<B, R><<<(N + rows_per_block - 1) / rows_per_block, kWarps * 32, 0, st>>>(x, wq, sw, N, K, y);
    return cudaGetLastError();
}

template <int B>
cudaError_t launch_b(const uint16_t *x, const int8_t *wq, const float *sw, int N, int K, uint16_t *y,
                     cudaStream_t st) {
    const long long blocks2 = (N + kWarps * 2 - 1) / (kWarps * 2);
    if (blocks2 >= 6ll * num_sms()) return launch_br<B, 2>(x, wq, sw, N, K, y, st);
    return launch_br<B, 1>(x, wq, sw, N, K, y, st);
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_gemv_w8a16(const uint16_t *x, int B, const int8_t *wq_, const float *sw, int N, int K,
                                   uint16_t *y, void *stream) {
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(wq_, "wq");
    WQ_REQUIRE_PTR(sw, "sw");
    WQ_REQUIRE_PTR(y, "y");
    WQ_REQUIRE(N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_gemv_w8a16: N and K must be positive (N=%d K=%d)", N, K);
    WQ_REQUIRE(B >= 1 && B <= 8, WQ_ERR_UNSUPPORTED, "wq_gemv_w8a16: B must be 1..8 (got %d)", B);
    WQ_REQUIRE(K % 16 == 0, WQ_ERR_UNSUPPORTED, "wq_gemv_w8a16: K (%d) must be a multiple of 16", K);
    cudaStream_t st = wq::as_stream(stream);
    cudaError_t e;
    switch (B) {
        case 1: e = wq::launch_b<1>(x, wq_, sw, N, K, y, st); break;
        case 2: e = wq::launch_b<2>(x, wq_, sw, N, K, y, st); break;
        case 3: e = wq::launch_b<3>(x, wq_, sw, N, K, y, st); break;
        case 4: e = wq::launch_b<4>(x, wq_, sw, N, K, y, st); break;
        case 5: e = wq::launch_b<5>(x, wq_, sw, N, K, y, st); break;
        case 6: e = wq::launch_b<6>(x, wq_, sw, N, K, y, st); break;
        case 7: e = wq::launch_b<7>(x, wq_, sw, N, K, y, st); break;
        default: e = wq::launch_b<8>(x, wq_, sw, N, K, y, st); break;
    }
    if (e != cudaSuccess) return wq::fail(WQ_ERR_CUDA, "wq_gemv_w8a16: launch failed: %s", cudaGetErrorString(e));
    return WQ_OK;
}
