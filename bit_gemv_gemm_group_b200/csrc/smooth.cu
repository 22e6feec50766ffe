// SmoothQuant smoothing factors s_j = max|X_j|^alpha / max|W_j|^(1-alpha).
//
// Source: "How quantization works", section "Activation quantization and
// outliers" (s = X.abs().amax(0).clamp(1e-5)**a / W.abs().amax(0).clamp(1e-5)**(1-a),
// alpha = 0.5); "Quantization" (engine-room chapter 15), section "The
// Mathematics" (s_j = max(|X_j|)^a / max(|W_j|)^(1-a), computed offline).
//
// Both operands are [rows][K] row-major, so the column maxima are reductions
// across rows.  One kernel covers X and W: each CTA owns a tile of 256
// columns x kTileRows rows, keeps 8 running maxima per thread (one 16-byte
// load per row), reduces its 8 warps through shared memory and folds the tile
// into the global maxima with atomicMax on the float bit patterns (exact: for
// non-negative floats the bit patterns order like the values).  The last CTA
// to finish (ticket counter) turns the two maxima into s.  HBM traffic is one
// read of X and W: 2 B per element.
//
// Workspace layout (bytes): ax float[Kp] | aw float[Kp] | ticket uint32,
// Kp = K rounded up to 4.
#include "wq_device.cuh"
#include "wq_host.h"

namespace wq {
namespace {

constexpr int kThreads = 256;
constexpr int kTileCols = 256;  // 32 lanes x 8 columns
constexpr int kTileRows = 256;

__host__ __device__ inline size_t padded(int K) { return ((size_t)K + 3) & ~(size_t)3; }

__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) { return __vmaxu2(a, b); }

__global__ void __launch_bounds__(kThreads) smooth_kernel(const uint16_t *__restrict__ x, int M,
                                                          const uint16_t *__restrict__ w, int N, int K,
                                                          float alpha, float *__restrict__ s,
                                                          unsigned int *__restrict__ ws, int tiles_x,
                                                          int col_tiles, unsigned int total_blocks) {
    __shared__ uint32_t part[kThreads / 32][kTileCols / 2];  // packed fp16 |max| pairs per warp
    __shared__ bool last;
    const size_t Kp = padded(K);
    unsigned int *ax = ws;
    unsigned int *aw = ws + Kp;
    unsigned int *ticket = ws + 2 * Kp;

    int tile = blockIdx.x;
    const bool is_x = tile < tiles_x;
    if (!is_x) tile -= tiles_x;
    const uint16_t *src = is_x ? x : w;
    const int rows = is_x ? M : N;
    unsigned int *dst = is_x ? ax : aw;
    const int ct = tile % col_tiles;
    const int rt = tile / col_tiles;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int col = ct * kTileCols + lane * 8;
    const int r0 = rt * kTileRows;
    const int r1 = min(rows, r0 + kTileRows);

    // |value| as fp16 bits; for non-negative fp16 the bit patterns order like the values.
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
    if (col < K) {
        int r = r0 + warp;
        for (; r + 3 * 8 < r1; r += 4 * 8) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = ld_stream_u4(src + (size_t)(r + 8 * u) * K + col);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                m0 = umax2(m0, v[u].x & 0x7fff7fffu);
                m1 = umax2(m1, v[u].y & 0x7fff7fffu);
                m2 = umax2(m2, v[u].z & 0x7fff7fffu);
                m3 = umax2(m3, v[u].w & 0x7fff7fffu);
            }
        }
        for (; r < r1; r += 8) {
            const uint4 v = ld_stream_u4(src + (size_t)r * K + col);
            m0 = umax2(m0, v.x & 0x7fff7fffu);
            m1 = umax2(m1, v.y & 0x7fff7fffu);
            m2 = umax2(m2, v.z & 0x7fff7fffu);
            m3 = umax2(m3, v.w & 0x7fff7fffu);
        }
    }
    part[warp][lane * 4 + 0] = m0;
    part[warp][lane * 4 + 1] = m1;
    part[warp][lane * 4 + 2] = m2;
    part[warp][lane * 4 + 3] = m3;
    __syncthreads();
    if (threadIdx.x < kTileCols / 2) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < kThreads / 32; ++i) m = umax2(m, part[i][threadIdx.x]);
        const int c = ct * kTileCols + 2 * threadIdx.x;
        if (c < K) atomicMax(dst + c, __float_as_uint(half_bits_to_float((uint16_t)(m & 0xffffu))));
        if (c + 1 < K) atomicMax(dst + c + 1, __float_as_uint(half_bits_to_float((uint16_t)(m >> 16))));
    }

    // The last CTA to arrive turns the maxima into smoothing factors.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(ticket, 1u) == total_blocks - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int j = threadIdx.x; j < K; j += kThreads) {
        const float a_x = fmaxf(__uint_as_float(__ldcg(ax + j)), 1e-5f);
        const float a_w = fmaxf(__uint_as_float(__ldcg(aw + j)), 1e-5f);
        float num, den;
        if (alpha == 0.5f) {
            num = __fsqrt_rn(a_x);
            den = __fsqrt_rn(a_w);
        } else {
            num = (float)pow((double)a_x, (double)alpha);
            den = (float)pow((double)a_w, 1.0 - (double)alpha);
        }
        s[j] = __fdiv_rn(num, den);
    }
}

}  // namespace
}  // namespace wq

extern "C" size_t wq_smooth_workspace_bytes(int K) {
    if (K <= 0) return 0;
    return (2 * wq::padded(K) + 4) * sizeof(unsigned int);
}

extern "C" wq_status wq_smooth(const uint16_t *x, int M, const uint16_t *w, int N, int K, float alpha, float *s,
                               void *workspace, void *stream) {
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(w, "w");
    WQ_REQUIRE_PTR(s, "s");
    WQ_REQUIRE_PTR(workspace, "workspace");
    WQ_REQUIRE(M > 0 && N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_smooth: sizes must be positive (M=%d N=%d K=%d)",
               M, N, K);
    WQ_REQUIRE(K % 8 == 0, WQ_ERR_UNSUPPORTED, "wq_smooth: K (%d) must be a multiple of 8", K);
    WQ_REQUIRE(alpha >= 0.0f && alpha <= 1.0f, WQ_ERR_INVALID_ARG, "wq_smooth: alpha must lie in [0, 1]");
    const int col_tiles = (K + wq::kTileCols - 1) / wq::kTileCols;
    const long long tx = (long long)col_tiles * ((M + wq::kTileRows - 1) / wq::kTileRows);
    const long long tw = (long long)col_tiles * ((N + wq::kTileRows - 1) / wq::kTileRows);
    WQ_REQUIRE(tx + tw < (1ll << 31), WQ_ERR_UNSUPPORTED, "wq_smooth: problem too large");
    cudaStream_t st = wq::as_stream(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, wq_smooth_workspace_bytes(K), st);
    if (e != cudaSuccess) return wq::fail(WQ_ERR_CUDA, "wq_smooth: clearing the workspace failed: %s",
                                          cudaGetErrorString(e));
    const unsigned int total = (unsigned int)(tx + tw);
    wq::smooth_kernel<<<total, wq::kThreads, 0, st>>>(x, M, w, N, K, alpha, s,
                                                      static_cast<unsigned int *>(workspace), (int)tx, col_tiles,
                                                      total);
    return wq::check_launch("wq_smooth");
}

// ---------------------------------------------------------------------------
// Allocation-free smoothing.
//
// Some callers cannot allocate device memory for the workspace: a plug-in that
// runs inside a host engine which owns all device memory and exposes no
// allocator, or a latency-critical path where cudaMalloc's implicit device
// synchronization is not allowed.  wq_smooth_noalloc gives them the same
// computation with the workspace in a fixed-size array that the library keeps
// in device memory (every GPU that loads the library holds it until the
// process exits).  Host code cannot use the array's name as a device address,
// so the device address is looked up once per device with cudaGetSymbolAddress
// (on the first call made while that device is current) and cached.
// ---------------------------------------------------------------------------
#include <mutex>

namespace wq {
namespace {

constexpr size_t kNoAllocWords = 2 * (size_t)WQ_SMOOTH_NOALLOC_MAX_K + 4;  // ax | aw | ticket, K padded to 4
static __device__ __align__(256) unsigned int g_smooth_scratch[kNoAllocWords];

constexpr int kScratchDevices = 64;
std::mutex g_scratch_mu;
unsigned int *g_scratch_ptr[kScratchDevices];

unsigned int *smooth_scratch() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kScratchDevices) {
        fail(WQ_ERR_CUDA, "wq_smooth_noalloc: cudaGetDevice failed");
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_smooth_scratch);
        if (e != cudaSuccess) {
            fail(WQ_ERR_CUDA, "wq_smooth_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
            return nullptr;
        }
        g_scratch_ptr[dev] = static_cast<unsigned int *>(p);
    }
    return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_smooth_noalloc(const uint16_t *x, int M, const uint16_t *w, int N, int K, float alpha,
                                       float *s, void *stream) {
    WQ_REQUIRE(K <= WQ_SMOOTH_NOALLOC_MAX_K, WQ_ERR_UNSUPPORTED,
               "wq_smooth_noalloc: K (%d) exceeds the built-in workspace (K <= %d); use wq_smooth with a "
               "caller-owned workspace",
               K, WQ_SMOOTH_NOALLOC_MAX_K);
    WQ_REQUIRE(K > 0, WQ_ERR_INVALID_ARG, "wq_smooth_noalloc: K must be positive (K=%d)", K);
    unsigned int *scratch = wq::smooth_scratch();
    if (!scratch) return WQ_ERR_CUDA;
    // wq_smooth clears the part of the workspace that must start at zero.
    return wq_smooth(x, M, w, N, K, alpha, s, scratch, stream);
}
