// W8A8 INT8 GEMM on the 5th-generation tensor cores (tcgen05, kind::i8) with
// a fused per-token x per-channel dequantization epilogue.
//
// Source: "Quantization: Smaller Weights, Same Answers (Mostly)", section
// "How does quantized matrix multiplication actually run on the GPU?" (int8
// operands through the integer tensor cores, exact 32-bit accumulation; with
// symmetric scales the zero-point terms vanish); "How quantization works",
// "Mainstream schemes at a glance" (W8A8 INT8) and the SmoothQuant section
// (the operands arrive already smoothed and quantized).
//
//   acc[m][n] = sum_k xq[m][k] * wq[n][k]          (int32, exact)
//   y[m][n]   = fp16_rn( (float)acc * sx[m] * sw[n] )
//
// Persistent, warp-specialized CTA (one per SM, 192 threads):
//   warp 0      TMA producer: 128x128-byte tiles of xq and 256x128-byte
//               tiles of wq (128-byte swizzle) into a 4-stage ring (48 KB/stage)
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma (M=128,
//               N=256, K=32 per instruction, 4 per stage); tcgen05.commit frees
//               a stage when its MMAs finish and signals a full accumulator
//   warps 2-5   epilogue: tcgen05.ld of the 128x256 int32 accumulator (warp w
//               reads TMEM lanes 32*(w%4)..+31), scale, convert, store; two
//               accumulators in TMEM so the epilogue of tile i overlaps the
//               MMAs of tile i+1.
// Tiles are 128 (M) x 256 (N), visited M-fastest so CTAs running together
// share the same weight tile.  No multicast of any kind.
#include "sm100.cuh"
#include "wq_device.cuh"
#include "wq_host.h"

#include <algorithm>

namespace wq {
namespace {

using namespace sm100;

constexpr int BM = 128, BN = 256, BK = 128;  // BK in bytes (= int8 elements)
constexpr int STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK;        // 16 KB
constexpr uint32_t B_BYTES = BN * BK;        // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 512;          // two 256-column fp32/int32 accumulators
constexpr int THREADS = 192;
constexpr uint32_t IDESC = make_idesc(/*s32*/ 2, /*s8*/ 1, /*s8*/ 1, BM, BN);
constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + 256 /*barriers etc.*/;
constexpr uint64_t DRAIN_NS = 2000000000ull;

// Site codes recorded in the device status word when a wait runs out.
constexpr unsigned SITE_PRODUCER = 0x101, SITE_MMA = 0x102, SITE_EPILOGUE = 0x104, SITE_DRAIN = 0x108;

struct Smem {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void store_chunk(uint16_t *__restrict__ y, int32_t *__restrict__ acc_out, int m, int n0,
                                            int N, float sxm, const float *__restrict__ sw, const uint32_t (&r)[32],
                                            bool vec_ok) {
    float swv[32];
    if (vec_ok && n0 + 32 <= N) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(sw + n0) + j);
            swv[4 * j] = v.x; swv[4 * j + 1] = v.y; swv[4 * j + 2] = v.z; swv[4 * j + 3] = v.w;
        }
        uint32_t h[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float a = __fmul_rn(__fmul_rn((float)(int32_t)r[2 * j], sxm), swv[2 * j]);
            const float b = __fmul_rn(__fmul_rn((float)(int32_t)r[2 * j + 1], sxm), swv[2 * j + 1]);
            h[j] = (uint32_t)float_to_half_bits_rn(a) | ((uint32_t)float_to_half_bits_rn(b) << 16);
        }
        uint4 *yp = reinterpret_cast<uint4 *>(y + (size_t)m * N + n0);
#pragma unroll
        for (int j = 0; j < 4; ++j) yp[j] = make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
        if (acc_out) {
            uint4 *ap = reinterpret_cast<uint4 *>(acc_out + (size_t)m * N + n0);
#pragma unroll
            for (int j = 0; j < 8; ++j) ap[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int n = n0 + j;
            if (n < N) {
                const float v = __fmul_rn(__fmul_rn((float)(int32_t)r[j], sxm), __ldg(sw + n));
                y[(size_t)m * N + n] = float_to_half_bits_rn(v);
                if (acc_out) acc_out[(size_t)m * N + n] = (int32_t)r[j];
            }
        }
    }
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const float *__restrict__ sx, const float *__restrict__ sw, uint16_t *__restrict__ y,
                     int32_t *__restrict__ acc_out, int M, int N, int K, unsigned int *status, uint64_t limit_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = base + STAGES * A_BYTES;
    Smem *sm = reinterpret_cast<Smem *>(base + STAGES * STAGE_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = (M + BM - 1) / BM, nt = (N + BN - 1) / BN;
    const int tiles = mt * nt;
    const int kblocks = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&sm->full[s]), 1);
            mbar_init(smem_u32(&sm->empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&sm->tmem_full[a]), 1);
            mbar_init(smem_u32(&sm->tmem_empty[a]), 4 * 32);
        }
        mbar_init(smem_u32(&sm->drain), 1);
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_w);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = sm->tmem_base;
    const WaitCtl ctl{&sm->abort, status, limit_ns};

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
                const int m0 = (tile % mt) * BM, n0 = (tile / mt) * BN;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES, u = it / STAGES;
                    if (!wait_parity(smem_u32(&sm->empty[s]), (u & 1) ^ 1, ctl, SITE_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&sm->full[s]);
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(smem_u32(sA + s * A_BYTES), &tmap_x, fb, kb * BK, m0);
                    tma_load_2d(smem_u32(sB + s * B_BYTES), &tmap_w, fb, kb * BK, n0);
                }
            }
            // Every issued load must land before the CTA may exit.
            for (uint32_t s = 0; s < STAGES; ++s) {
                const uint32_t issued = it > s ? (it - s - 1) / STAGES + 1 : 0;
                if (issued) drain_parity(smem_u32(&sm->full[s]), (issued - 1) & 1, DRAIN_NS, status, SITE_DRAIN);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x, ++tcount) {
                const uint32_t a = tcount & 1, ua = tcount >> 1;
                if (!wait_parity(smem_u32(&sm->tmem_empty[a]), (ua & 1) ^ 1, ctl, SITE_MMA)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + a * BN;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES, u = it / STAGES;
                    if (!wait_parity(smem_u32(&sm->full[s]), u & 1, ctl, SITE_MMA)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + s * A_BYTES), b_addr = smem_u32(sB + s * B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        mma_i8(d, umma_desc_sw128_kmajor(a_addr + kk * 32), umma_desc_sw128_kmajor(b_addr + kk * 32),
                               IDESC, (kb | kk) != 0);
                    tc_commit(smem_u32(&sm->empty[s]));
                }
                if (ok) tc_commit(smem_u32(&sm->tmem_full[a]));
            }
            // Wait for every MMA this thread issued before TMEM is released.
            tc_commit(smem_u32(&sm->drain));
            drain_parity(smem_u32(&sm->drain), 0, DRAIN_NS, status, SITE_DRAIN);
        }
        __syncwarp();
    } else {
        // -------------------------------------------------------------------- epilogue
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;
        const bool vec_ok = (N % 8) == 0;
        uint32_t tcount = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tcount) {
            const uint32_t a = tcount & 1, ua = tcount >> 1;
            bool ok = wait_parity(smem_u32(&sm->tmem_full[a]), ua & 1, ctl, SITE_EPILOGUE);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const int m = (tile % mt) * BM + row;
            const int nb = (tile / mt) * BN;
            const float sxm = m < M ? __ldg(sx + m) : 0.0f;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + a * BN + c * 32, r);
                tmem_ld_wait();
                if (m < M && nb + c * 32 < N) store_chunk(y, acc_out, m, nb + c * 32, N, sxm, sw, r, vec_ok);
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sm->tmem_empty[a]));
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_gemm_w8a8(const int8_t *xq, const float *sx, const int8_t *wq_, const float *sw, int M, int N,
                                  int K, uint16_t *y, int32_t *acc_out, void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(xq, "xq");
    WQ_REQUIRE_PTR(sx, "sx");
    WQ_REQUIRE_PTR(wq_, "wq");
    WQ_REQUIRE_PTR(sw, "sw");
    WQ_REQUIRE_PTR(y, "y");
    if (acc_out) WQ_REQUIRE(aligned16(acc_out), WQ_ERR_ALIGNMENT, "acc_out is not 16-byte aligned");
    WQ_REQUIRE(M > 0 && N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_gemm_w8a8: sizes must be positive (M=%d N=%d K=%d)", M,
               N, K);
    WQ_REQUIRE(K % 16 == 0, WQ_ERR_UNSUPPORTED, "wq_gemm_w8a8: K (%d) must be a multiple of 16", K);
    // |acc| <= 128 * 128 * K must stay below 2^31 for any int8 codes: K <= 131071, and K % 16 == 0
    WQ_REQUIRE(K <= 131056, WQ_ERR_UNSUPPORTED, "wq_gemm_w8a8: K (%d) above 131056 could overflow int32", K);
    unsigned int *status = device_status_word();
    if (!status) return WQ_ERR_CUDA;
    CUtensorMap tx, tw;
    if (!encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return WQ_ERR_CUDA;
    if (!encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq_, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BN,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return WQ_ERR_CUDA;
    cudaError_t e = cudaFuncSetAttribute(gemm_w8a8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess)
        return fail(WQ_ERR_CUDA, "wq_gemm_w8a8: cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
    const long long tiles = (long long)((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    WQ_REQUIRE(tiles < (1ll << 31), WQ_ERR_UNSUPPORTED, "wq_gemm_w8a8: problem too large");
    const int grid = (int)std::min<long long>(tiles, num_sms());
    gemm_w8a8_kernel<<<grid, THREADS, SMEM_BYTES, as_stream(stream)>>>(tx, tw, sx, sw, y, acc_out, M, N, K, status,
                                                                        wait_limit());
    return check_launch("wq_gemm_w8a8");
}
