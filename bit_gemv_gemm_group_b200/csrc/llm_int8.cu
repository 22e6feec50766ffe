// LLM.int8() mixed-precision decomposition: the steps before the GEMM.
//
// Source: "Quantization" (engine-room chapter 15), "The Breakthrough" and
// "The Mathematics" (C ~= S_out (.) (X_q W_q) + X_16 W_16: vector-wise INT8
// scales per row and per column; the outlier feature dimensions are removed
// from the integer path and multiplied in 16-bit, then added back);
// "Quantization: Smaller Weights, Same Answers (Mostly)", "How do
// LLM-specific quantization schemes protect against outliers?" (keep the
// outlier dimensions in FP16 and quantize the rest).
//
//   1. wq_outlier_columns: column maxima of |X| (one read of X, atomicMax on
//      the float bits), then one CTA compacts the columns whose maximum
//      reaches the threshold, lowest index first, at most `cap` of them, and
//      writes keep[j] = 0 for those and 1 elsewhere.  keep doubles as the
//      reduction buffer (the call clears it first).
//   2. X_q, s_x: wq_quantize_int8_per_channel(X, keep) -- per-row INT8 of
//      X * keep, i.e. with the carved columns zeroed (no new kernel).
//   3. wq_gather_outliers: X_16 [M][cap] = X[:, idx] and W_16 [N][cap] = the
//      INT8 weight codes of the same columns as fp16 (exact), zero beyond the
//      carved count.
//   4. wq_gemm_w8a8_outliers (gemm_w8a8.cu): the INT8 GEMM whose epilogue adds
//      X_16 W_16^T, scaled by s_w.
#include "wq_device.cuh"
#include "wq_host.h"

#include <algorithm>

namespace wq {
namespace {

constexpr int kThreads = 256;
constexpr int kTileCols = 256;  // 32 lanes x 8 columns
constexpr int kScanThreads = 1024;

// Column maxima of |x| for one 256-column tile over rows [r0, r1), folded into amax with
// atomicMax on the float bits (non-negative floats order like their bit patterns).
__global__ void __launch_bounds__(kThreads) column_absmax_kernel(const uint16_t *__restrict__ x, int M, int K,
                                                                 int rows_per_share, unsigned int *__restrict__ amax) {
    __shared__ uint32_t part[kThreads / 32][kTileCols / 2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int col = blockIdx.x * kTileCols + lane * 8;
    const int r0 = blockIdx.y * rows_per_share, r1 = min(M, r0 + rows_per_share);
    uint32_t m[4] = {0u, 0u, 0u, 0u};  // |x| as fp16 bit pairs
    if (col < K) {
        constexpr int W = kThreads / 32;
        int r = r0 + warp;
        for (; r + 3 * W < r1; r += 4 * W) {  // four rows per step: four loads in flight per lane
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = ld_stream_u4(x + (size_t)(r + u * W) * K + col);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                m[0] = __vmaxu2(m[0], v[u].x & 0x7fff7fffu);
                m[1] = __vmaxu2(m[1], v[u].y & 0x7fff7fffu);
                m[2] = __vmaxu2(m[2], v[u].z & 0x7fff7fffu);
                m[3] = __vmaxu2(m[3], v[u].w & 0x7fff7fffu);
            }
        }
        for (; r < r1; r += W) {
            const uint4 v = ld_stream_u4(x + (size_t)r * K + col);
            m[0] = __vmaxu2(m[0], v.x & 0x7fff7fffu);
            m[1] = __vmaxu2(m[1], v.y & 0x7fff7fffu);
            m[2] = __vmaxu2(m[2], v.z & 0x7fff7fffu);
            m[3] = __vmaxu2(m[3], v.w & 0x7fff7fffu);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) part[warp][lane * 4 + i] = m[i];
    __syncthreads();
    if (threadIdx.x < kTileCols / 2) {
        uint32_t v = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) v = __vmaxu2(v, part[w][threadIdx.x]);
        const int c = blockIdx.x * kTileCols + 2 * threadIdx.x;
        if (c < K) atomicMax(amax + c, __float_as_uint(half_bits_to_float((uint16_t)(v & 0xffffu))));
        if (c + 1 < K) atomicMax(amax + c + 1, __float_as_uint(half_bits_to_float((uint16_t)(v >> 16))));
    }
}

// One CTA: thread t owns columns [t*per, (t+1)*per), per a multiple of 4 (K is a multiple of
// 8), read and written as float4.  Flags (max >= threshold) are counted, exclusive-scanned over
// the CTA, and the first `cap` flagged columns (lowest index first) become the carved set: idx
// gets their indices (0 in its unused entries), keep gets 0 there and 1 elsewhere (in place of
// the maxima), count gets the number of flagged columns.
__global__ void __launch_bounds__(kScanThreads) compact_outliers_kernel(int K, float threshold, int cap,
                                                                        float *__restrict__ keep,
                                                                        int32_t *__restrict__ idx,
                                                                        int32_t *__restrict__ count) {
    __shared__ int warp_sum[kScanThreads / 32];
    const int per = (K + 4 * kScanThreads - 1) / (4 * kScanThreads) * 4;
    const int c0 = threadIdx.x * per, c1 = min(K, c0 + per);
    int n = 0;
    for (int c = c0; c < c1; c += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(keep + c);
        n += (v.x >= threshold) + (v.y >= threshold) + (v.z >= threshold) + (v.w >= threshold);
    }
    // inclusive scan of n over the CTA
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int s = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += v;
    }
    if (lane == 31) warp_sum[warp] = s;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kScanThreads / 32 ? warp_sum[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += v;
        }
        if (lane < kScanThreads / 32) warp_sum[lane] = w;  // inclusive per-warp totals
    }
    __syncthreads();
    int pos = s - n + (warp > 0 ? warp_sum[warp - 1] : 0);  // exclusive prefix of this thread
    for (int c = c0; c < c1; c += 4) {
        const float4 v = *reinterpret_cast<const float4 *>(keep + c);
        const float vv[4] = {v.x, v.y, v.z, v.w};
        float kv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool out = vv[e] >= threshold;
            if (out && pos < cap) idx[pos] = c + e;
            kv[e] = (out && pos < cap) ? 0.0f : 1.0f;
            pos += out;
        }
        *reinterpret_cast<float4 *>(keep + c) = make_float4(kv[0], kv[1], kv[2], kv[3]);
    }
    __shared__ int total;
    if (threadIdx.x == kScanThreads - 1) {
        *count = pos;
        total = pos;
    }
    __syncthreads();
    for (int j = min(total, cap) + threadIdx.x; j < cap; j += kScanThreads) idx[j] = 0;  // unused entries
}

// Row r < M: X_16[r][i] = x[r][idx[i]]; row r >= M: W_16[r - M][i] = (fp16) wq[r - M][idx[i]];
// zero for i >= min(count, cap).
__global__ void __launch_bounds__(kThreads) gather_outliers_kernel(const uint16_t *__restrict__ x, int M, int K,
                                                                   const int8_t *__restrict__ wq, int N,
                                                                   const int32_t *__restrict__ idx,
                                                                   const int32_t *__restrict__ count, int cap,
                                                                   uint16_t *__restrict__ x16,
                                                                   uint16_t *__restrict__ w16) {
    const int n_out = min(*count, cap);
    const size_t total = (size_t)(M + N) * cap;
    const size_t stride = (size_t)gridDim.x * kThreads;
    // four elements per thread and step, every load issued before the first store (the loads
    // are scattered single elements, so only their number in flight sets the speed)
    for (size_t e0 = (size_t)blockIdx.x * kThreads + threadIdx.x; e0 < total; e0 += 4 * stride) {
        uint32_t v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const size_t e = e0 + u * stride;
            v[u] = 0u;
            if (e < total) {
                const int r = (int)(e / cap), i = (int)(e % cap);
                if (i < n_out)
                    v[u] = r < M ? (uint32_t)x[(size_t)r * K + idx[i]]
                                 : (uint32_t)float_to_half_bits_rn((float)wq[(size_t)(r - M) * K + idx[i]]);
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const size_t e = e0 + u * stride;
            if (e < total) {
                // rows < M: X_16 (fp16 bits as read); rows >= M: W_16 (|code| <= 128 is exact in fp16)
                if (e < (size_t)M * cap) x16[e] = (uint16_t)v[u];
                else w16[e - (size_t)M * cap] = (uint16_t)v[u];
            }
        }
    }
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_outlier_columns(const uint16_t *x, int M, int K, float threshold, int cap, int32_t *idx,
                                        int32_t *count, float *keep, void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(idx, "idx");
    WQ_REQUIRE_PTR(count, "count");
    WQ_REQUIRE_PTR(keep, "keep");
    WQ_REQUIRE(M > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_outlier_columns: sizes must be positive (M=%d K=%d)", M, K);
    WQ_REQUIRE(K % 8 == 0, WQ_ERR_UNSUPPORTED, "wq_outlier_columns: K (%d) must be a multiple of 8", K);
    WQ_REQUIRE(cap >= 1 && cap <= K, WQ_ERR_INVALID_ARG, "wq_outlier_columns: cap (%d) must lie in [1, K]", cap);
    WQ_REQUIRE(threshold > 0.0f, WQ_ERR_INVALID_ARG, "wq_outlier_columns: threshold must be positive");
    cudaStream_t st = as_stream(stream);
    cudaError_t e = cudaMemsetAsync(keep, 0, sizeof(float) * (size_t)K, st);
    if (e != cudaSuccess)
        return fail(WQ_ERR_CUDA, "wq_outlier_columns: clearing keep failed: %s", cudaGetErrorString(e));
    const int tiles = (K + kTileCols - 1) / kTileCols;
    // row shares: about eight CTAs per SM over the whole grid, at least 8 rows each
    const int shares = std::max(1, std::min((M + 7) / 8, (8 * num_sms() + tiles - 1) / tiles));
    const int rows_per_share = (M + shares - 1) / shares;
    column_absmax_kernel<<<dim3(tiles, (M + rows_per_share - 1) / rows_per_share), kThreads, 0, st>>>(
        x, M, K, rows_per_share, reinterpret_cast<unsigned int *>(keep));
    if ((e = cudaGetLastError()) != cudaSuccess)
        return fail(WQ_ERR_CUDA, "wq_outlier_columns: launch failed: %s", cudaGetErrorString(e));
    compact_outliers_kernel<<<1, kScanThreads, 0, st>>>(K, threshold, cap, keep, idx, count);
    return check_launch("wq_outlier_columns");
}

extern "C" wq_status wq_gather_outliers(const uint16_t *x, int M, int K, const int8_t *wq_, int N, const int32_t *idx,
                                        const int32_t *count, int cap, uint16_t *x16, uint16_t *w16, void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(wq_, "wq");
    WQ_REQUIRE_PTR(idx, "idx");
    WQ_REQUIRE_PTR(count, "count");
    WQ_REQUIRE_PTR(x16, "x16");
    WQ_REQUIRE_PTR(w16, "w16");
    WQ_REQUIRE(M > 0 && N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_gather_outliers: sizes must be positive");
    WQ_REQUIRE(cap >= 16 && cap <= 256 && cap % 16 == 0, WQ_ERR_UNSUPPORTED,
               "wq_gather_outliers: cap (%d) must be a multiple of 16 in [16, 256]", cap);
    const size_t total = (size_t)(M + N) * cap;
    const int grid = (int)std::min<size_t>((total + kThreads - 1) / kThreads, (size_t)num_sms() * 8);
    gather_outliers_kernel<<<grid, kThreads, 0, as_stream(stream)>>>(x, M, K, wq_, N, idx, count, cap, x16, w16);
    return check_launch("wq_gather_outliers");
}
