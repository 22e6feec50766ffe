// SmoothQuant smoothing factors s_j = max|X_j|^alpha / max|W_j|^(1-alpha).
//
// Source: "How quantization works", section "Activation quantization and
// outliers" (s = X.abs().amax(0).clamp(1e-5)**a / W.abs().amax(0).clamp(1e-5)**(1-a),
// alpha = 0.5); "Quantization" (engine-room chapter 15), section "The
// Mathematics" (s_j = max(|X_j|)^a / max(|W_j|)^(1-a), computed offline).
//
// Both operands are [rows][K] row-major, so the column maxima are reductions
// across rows.  One kernel covers X and W: CTA (ct, g) owns the 256-column
// tile ct and an equal share g of the rows of both matrices, with as many
// shares as make the grid fill every CTA slot of the GPU once (no partial
// second wave).  A thread keeps 8 running maxima (one 16-byte load per row, 8
// rows in flight), the CTA reduces its 8 warps through shared memory and folds
// its maxima into the global ones with atomicMax on the float bit patterns
// (exact: for non-negative floats the bit patterns order like the values).  The last CTA
// of a column tile's CTAs to finish (a ticket per tile) turns the tile's two
// maxima into s.  HBM traffic is one
// read of X and W: 2 B per element.
//
// Workspace layout (words): ax float[Kp] | aw float[Kp] | tickets uint32[ceil4(K/256)],
// Kp = K rounded up to 4.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "wq_device.cuh"
#include "wq_host.h"

namespace wq {
namespace {

constexpr int kThreads = 256;
constexpr int kTileCols = 256;  // 32 lanes x 8 columns

__host__ __device__ inline size_t padded(int K) { return ((size_t)K + 3) & ~(size_t)3; }

__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) { return __vmaxu2(a, b); }

// Column maxima of rows [r0, r1) of one 256-column tile, folded into `dst` with
// atomicMax on the float bit patterns.  All of the CTA's threads call it.
__device__ __forceinline__ void tile_column_max(const uint16_t *__restrict__ src, int K, int col, int r0, int r1,
                                                int ct, unsigned int *__restrict__ dst,
                                                uint32_t (*part)[kTileCols / 2]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // |value| as fp16 bits; for non-negative fp16 the bit patterns order like the values.
    uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
    if (col < K) {
        int r = r0 + warp;
        for (; r + 7 * 8 < r1; r += 8 * 8) {  // 8 rows of 16-byte loads in flight per thread
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = ld_stream_u4(src + (size_t)(r + 8 * u) * K + col);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
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
    __syncthreads();  // `part` is free (a previous call's readers are done)
    part[warp][lane * 4 + 0] = m0;
    part[warp][lane * 4 + 1] = m1;
    part[warp][lane * 4 + 2] = m2;
    part[warp][lane * 4 + 3] = m3;
    __syncthreads();
    if (threadIdx.x < kTileCols / 2 && r0 < r1) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < kThreads / 32; ++i) m = umax2(m, part[i][threadIdx.x]);
        const int c = ct * kTileCols + 2 * threadIdx.x;
        if (c < K) atomicMax(dst + c, __float_as_uint(half_bits_to_float((uint16_t)(m & 0xffffu))));
        if (c + 1 < K) atomicMax(dst + c + 1, __float_as_uint(half_bits_to_float((uint16_t)(m >> 16))));
    }
}

// CTA (ct, g): column tile ct of both matrices, row share g of `groups` (X and W
// rows split evenly), so that the grid fills the SMs' CTA slots exactly once.
__global__ void __launch_bounds__(kThreads) smooth_kernel(const uint16_t *__restrict__ x, int M,
                                                          const uint16_t *__restrict__ w, int N, int K,
                                                          float alpha, float *__restrict__ s,
                                                          unsigned int *__restrict__ ws, int col_tiles, int groups) {
    __shared__ uint32_t part[kThreads / 32][kTileCols / 2];  // packed fp16 |max| pairs per warp
    __shared__ bool last;
    const size_t Kp = padded(K);
    unsigned int *ax = ws;
    unsigned int *aw = ws + Kp;
    unsigned int *ticket = ws + 2 * Kp;  // one per column tile

    const int ct = blockIdx.x % col_tiles;
    const int g = blockIdx.x / col_tiles;
    const int lane = threadIdx.x & 31;
    const int col = ct * kTileCols + lane * 8;
    tile_column_max(x, K, col, (int)((long long)M * g / groups), (int)((long long)M * (g + 1) / groups), ct, ax, part);
    tile_column_max(w, K, col, (int)((long long)N * g / groups), (int)((long long)N * (g + 1) / groups), ct, aw, part);

    // The last of the column tile's CTAs to arrive turns its 256 maxima into smoothing factors.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(ticket + ct, 1u) == (unsigned int)groups - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    for (int j = ct * kTileCols + threadIdx.x; j < min(K, (ct + 1) * kTileCols); j += kThreads) {
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

// Resident CTAs of smooth_kernel on the current device (SMs x CTAs per SM), cached per
// device; host threads may race to fill an entry, and they all store the same value.
int smooth_slots() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148 * 8;
    int v = cached[dev].load(std::memory_order_relaxed);
    if (!v) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, smooth_kernel, kThreads, 0) != cudaSuccess ||
            per_sm <= 0)
            per_sm = 8;
        v = per_sm * num_sms();
        cached[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

}  // namespace
}  // namespace wq

extern "C" size_t wq_smooth_workspace_bytes(int K) {
    if (K <= 0) return 0;
    return (2 * wq::padded(K) + wq::padded((K + wq::kTileCols - 1) / wq::kTileCols)) * sizeof(unsigned int);
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
    // row shares per column tile: fill every CTA slot of the GPU exactly once
    const int slots = wq::smooth_slots();
    const int groups = std::max(1, std::min(std::max(M, N), slots / col_tiles));
    WQ_REQUIRE((long long)col_tiles * groups < (1ll << 31), WQ_ERR_UNSUPPORTED, "wq_smooth: problem too large");
    cudaStream_t st = wq::as_stream(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, wq_smooth_workspace_bytes(K), st);
    if (e != cudaSuccess) return wq::fail(WQ_ERR_CUDA, "wq_smooth: clearing the workspace failed: %s",
                                          cudaGetErrorString(e));
    const unsigned int total = (unsigned int)(col_tiles * groups);
    wq::smooth_kernel<<<total, wq::kThreads, 0, st>>>(x, M, w, N, K, alpha, s,
                                                      static_cast<unsigned int *>(workspace), col_tiles, groups);
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

namespace wq {
namespace {

// ax | aw | one ticket per 256-column tile, each padded to 4 words
constexpr size_t kNoAllocWords = 2 * (size_t)WQ_SMOOTH_NOALLOC_MAX_K + WQ_SMOOTH_NOALLOC_MAX_K / 256;
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
