// W8A8 GEMMs on the 5th-generation tensor cores with a fused per-token x
// per-channel dequantization epilogue: INT8 (tcgen05 kind::i8, int32
// accumulators) and FP8 E4M3 (kind::f8f6f4, fp32 accumulators).
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
// FP8: "How quantization works", "Mainstream schemes at a glance" (FP8 W8A8:
// FP8 weights and activations on FP8 tensor cores); "Quantization:
// Smaller Weights, Same Answers (Mostly)", "What about FP8, MXFP4, NVFP4 and
// GGUF?".  Same data flow with E4M3 codes; acc is the tensor cores' fp32 sum
// and a scale vector may hold one per-tensor value (stride 0).
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
//
// LLM.int8() variant ("Quantization" (engine-room ch. 15), "The Mathematics":
// C ~= S_out (.) (X_q W_q) + X_16 W_16): the INT8 GEMM above, whose epilogue
// warps also multiply the carved-out outlier columns in 16-bit.  Per 32 x 32
// chunk of its accumulator a warp runs mma.sync m16n8k16 (fp16 x fp16 -> fp32)
// over X_16 [M][cap] and W_16 [N][cap] (the INT8 weight codes of those columns
// as fp16, exact), transposes the fragments to one row per lane through 4 KB
// of shared memory, and stores y = fp16((acc * s_x + X_16 W_16^T) * s_w).  The
// epilogue of tile i runs while the MMAs of tile i + 1 proceed, so for a few
// dozen outlier columns the 16-bit product costs no extra time.
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
constexpr uint32_t IDESC_I8 = make_idesc(/*s32*/ 2, /*s8*/ 1, /*s8*/ 1, BM, BN);
constexpr uint32_t IDESC_E4M3 = make_idesc(/*f32*/ 1, /*e4m3*/ 0, /*e4m3*/ 0, BM, BN);
constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES + 256 /*barriers etc.*/;
constexpr int TR_PITCH = 33;                                     // fp32 words per row of a transpose buffer
constexpr size_t TR_BYTES = 4 * 32 * TR_PITCH * sizeof(float);    // one 32 x 32 buffer per epilogue warp
constexpr size_t SMEM_BYTES_OUTL = SMEM_BYTES + TR_BYTES;

// The carved-out outlier columns of the LLM.int8() variant (cap == 0: none).
struct Outliers {
    const uint16_t *x16;  // fp16 [M][cap]
    const uint16_t *w16;  // fp16 [N][cap]
    int cap;              // multiple of 16
};
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

// Accumulator bits to float: int32 (INT8) or fp32 (FP8).
template <bool FP8>
__device__ __forceinline__ float acc_value(uint32_t r) {
    return FP8 ? __uint_as_float(r) : (float)(int32_t)r;
}

template <bool FP8>
__device__ __forceinline__ void store_chunk(uint16_t *__restrict__ y, int32_t *__restrict__ acc_out, int m, int n0,
                                            int N, float sxm, const float *__restrict__ sw, int sw_stride,
                                            const uint32_t (&r)[32], bool vec_ok) {
    float swv[32];
    if (vec_ok && n0 + 32 <= N) {
        if (sw_stride) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(sw + n0) + j);
                swv[4 * j] = v.x; swv[4 * j + 1] = v.y; swv[4 * j + 2] = v.z; swv[4 * j + 3] = v.w;
            }
        } else {
            const float v = __ldg(sw);
#pragma unroll
            for (int j = 0; j < 32; ++j) swv[j] = v;
        }
        uint32_t h[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float a = __fmul_rn(__fmul_rn(acc_value<FP8>(r[2 * j]), sxm), swv[2 * j]);
            const float b = __fmul_rn(__fmul_rn(acc_value<FP8>(r[2 * j + 1]), sxm), swv[2 * j + 1]);
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
                const float v = __fmul_rn(__fmul_rn(acc_value<FP8>(r[j]), sxm), __ldg(sw + n * sw_stride));
                y[(size_t)m * N + n] = float_to_half_bits_rn(v);
                if (acc_out) acc_out[(size_t)m * N + n] = (int32_t)r[j];
            }
        }
    }
}

__device__ __forceinline__ void mma_16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t ldg_u32(const uint16_t *p) { return __ldg(reinterpret_cast<const uint32_t *>(p)); }

// o[j] = sum_i X_16[r0 + lane][i] * W_16[n0 + j][i] for j < 32 (one row per lane), by the whole
// warp: 2 x 4 tiles of m16n8k16 over cap / 16 k-steps, then a transpose through `tr`.  Rows and
// columns past M and N read the last valid ones (their results are never stored).
__device__ __forceinline__ void outlier_chunk(const Outliers &ol, int M, int N, int r0, int n0, int lane,
                                              float *__restrict__ tr, float (&o)[32]) {
    const int g = lane >> 2, t = lane & 3;
    const uint16_t *xa[2][2], *wb[4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int h = 0; h < 2; ++h) xa[mt][h] = ol.x16 + (size_t)min(r0 + 16 * mt + 8 * h + g, M - 1) * ol.cap + 2 * t;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) wb[nt] = ol.w16 + (size_t)min(n0 + 8 * nt + g, N - 1) * ol.cap + 2 * t;
    float cf[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) cf[mt][nt][0] = cf[mt][nt][1] = cf[mt][nt][2] = cf[mt][nt][3] = 0.0f;
    // Four k-steps (64 carved columns) per round: all of the round's fragments are requested
    // before its MMAs, so a chunk waits for one L2 round trip per 64 columns, not one per 16.
    for (int k0 = 0; k0 < ol.cap; k0 += 64) {
        uint32_t a[4][2][4], b[4][4][2];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const int kk = k0 + 16 * ks;
            if (kk < ol.cap) {
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    a[ks][mt][0] = ldg_u32(xa[mt][0] + kk);
                    a[ks][mt][1] = ldg_u32(xa[mt][1] + kk);
                    a[ks][mt][2] = ldg_u32(xa[mt][0] + kk + 8);
                    a[ks][mt][3] = ldg_u32(xa[mt][1] + kk + 8);
                }
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    b[ks][nt][0] = ldg_u32(wb[nt] + kk);
                    b[ks][nt][1] = ldg_u32(wb[nt] + kk + 8);
                }
            }
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            if (k0 + 16 * ks < ol.cap) {
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) mma_16816_f16(cf[mt][nt], a[ks][mt], b[ks][nt][0], b[ks][nt][1]);
            }
        }
    }
    __syncwarp();  // the previous chunk's readers are done with tr
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            float *p = tr + (16 * mt + g) * TR_PITCH + 8 * nt + 2 * t;
            p[0] = cf[mt][nt][0];
            p[1] = cf[mt][nt][1];
            p[8 * TR_PITCH] = cf[mt][nt][2];
            p[8 * TR_PITCH + 1] = cf[mt][nt][3];
        }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = tr[lane * TR_PITCH + j];
}

// Up to 64 carved columns (four k-steps): the epilogue keeps a warp's X_16 fragments for the
// whole tile and fetches the W_16 fragments of the next 32-column chunk while the current one
// is multiplied, so the chunks no longer wait for an L2 round trip each.  Fragments of k-steps
// at or past cap are zero.
__device__ __forceinline__ void outlier_x_frags(const Outliers &ol, int M, int r0, int lane, uint32_t (&a)[4][2][4]) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        const uint16_t *p0 = ol.x16 + (size_t)min(r0 + 16 * mt + g, M - 1) * ol.cap + 2 * t;
        const uint16_t *p1 = ol.x16 + (size_t)min(r0 + 16 * mt + 8 + g, M - 1) * ol.cap + 2 * t;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const bool in = 16 * ks < ol.cap;
            a[ks][mt][0] = in ? ldg_u32(p0 + 16 * ks) : 0u;
            a[ks][mt][1] = in ? ldg_u32(p1 + 16 * ks) : 0u;
            a[ks][mt][2] = in ? ldg_u32(p0 + 16 * ks + 8) : 0u;
            a[ks][mt][3] = in ? ldg_u32(p1 + 16 * ks + 8) : 0u;
        }
    }
}

__device__ __forceinline__ void outlier_w_frags(const Outliers &ol, int N, int n0, int lane, uint32_t (&b)[4][4][2]) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const uint16_t *p = ol.w16 + (size_t)min(n0 + 8 * nt + g, N - 1) * ol.cap + 2 * t;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const bool in = 16 * ks < ol.cap;
            b[ks][nt][0] = in ? ldg_u32(p + 16 * ks) : 0u;
            b[ks][nt][1] = in ? ldg_u32(p + 16 * ks + 8) : 0u;
        }
    }
}

// o[j] = sum_i X_16[row of lane][i] W_16[chunk column j][i] from fragments already in registers
// (the same MMA tiling and transpose as outlier_chunk).
__device__ __forceinline__ void outlier_mma64(const uint32_t (&a)[4][2][4], const uint32_t (&b)[4][4][2], int lane,
                                              float *__restrict__ tr, float (&o)[32]) {
    const int g = lane >> 2, t = lane & 3;
    float cf[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) cf[mt][nt][0] = cf[mt][nt][1] = cf[mt][nt][2] = cf[mt][nt][3] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) mma_16816_f16(cf[mt][nt], a[ks][mt], b[ks][nt][0], b[ks][nt][1]);
    __syncwarp();  // the previous chunk's readers are done with tr
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            float *p = tr + (16 * mt + g) * TR_PITCH + 8 * nt + 2 * t;
            p[0] = cf[mt][nt][0];
            p[1] = cf[mt][nt][1];
            p[8 * TR_PITCH] = cf[mt][nt][2];
            p[8 * TR_PITCH + 1] = cf[mt][nt][3];
        }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = tr[lane * TR_PITCH + j];
}

// y = fp16((acc * s_x + o) * s_w) for one row's 32-column chunk (INT8 accumulators).
__device__ __forceinline__ void store_chunk_outliers(uint16_t *__restrict__ y, int m, int n0, int N, float sxm,
                                                     const float *__restrict__ sw, const uint32_t (&r)[32],
                                                     const float (&o)[32], bool vec_ok) {
    if (vec_ok && n0 + 32 <= N) {
        uint32_t h[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(sw + n0) + j);
            const float sv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
                const int c = 4 * j + e;
                const float a = __fmul_rn(__fmaf_rn((float)(int32_t)r[c], sxm, o[c]), sv[e]);
                const float b = __fmul_rn(__fmaf_rn((float)(int32_t)r[c + 1], sxm, o[c + 1]), sv[e + 1]);
                h[c / 2] = (uint32_t)float_to_half_bits_rn(a) | ((uint32_t)float_to_half_bits_rn(b) << 16);
            }
        }
        uint4 *yp = reinterpret_cast<uint4 *>(y + (size_t)m * N + n0);
#pragma unroll
        for (int j = 0; j < 4; ++j) yp[j] = make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int n = n0 + j;
            if (n < N)
                y[(size_t)m * N + n] =
                    float_to_half_bits_rn(__fmul_rn(__fmaf_rn((float)(int32_t)r[j], sxm, o[j]), __ldg(sw + n)));
        }
    }
}

// Work schedule of the persistent CTAs.  Plain: tile blockIdx.x + u * gridDim.x for u = 0, 1, ...
// Split (the grid is made of CTA pairs, thread-block clusters of 2): `full_rounds` rounds of whole
// tiles, then the `split_tiles` tiles left over are shared by the pairs, one per pair, each CTA
// taking one half of K; the pair sums its two partial accumulators through distributed shared
// memory at the end.  This turns a last round that would keep only part of the SMs busy for a
// whole tile into a half-length round.
struct Sched {
    int tiles, full_rounds, split_tiles;  // split_tiles == 0: plain schedule

    __device__ __forceinline__ bool unit(int u, int kblocks, int &tile, int &kb0, int &kb1, bool &half) const {
        half = false;
        kb0 = 0;
        kb1 = kblocks;
        if (split_tiles == 0 || u < full_rounds) {
            tile = (int)blockIdx.x + u * (int)gridDim.x;
            return split_tiles == 0 ? tile < tiles : true;
        }
        const int pair = (int)blockIdx.x >> 1;
        if (u != full_rounds || pair >= split_tiles) return false;
        tile = full_rounds * (int)gridDim.x + pair;
        half = true;
        const int h = kblocks / 2;
        if (blockIdx.x & 1) kb0 = h;
        else kb1 = h;
        return true;
    }
};

constexpr int PART_PITCH = BN + 4;  // 32-bit words per row of the pair's partial tile in shared memory

// D (+)= A * B^T for one 128 x 256 x 32 step: kind::i8 (int32) or kind::f8f6f4 E4M3 (fp32).
template <bool FP8>
__device__ __forceinline__ void mma_step(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    if (FP8)
        mma_f8f6f4(d, a, b, IDESC_E4M3, acc);
    else
        mma_i8(d, a, b, IDESC_I8, acc);
}

// sx_stride / sw_stride: 1 for one scale per row, 0 for one scale for the whole operand.
// OUTL (INT8 only): the epilogue adds the 16-bit product of the outlier columns `ol`.
// SPLIT: launched as clusters of 2 with the split schedule (see Sched).
template <bool FP8, bool OUTL = false, bool SPLIT = false>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const float *__restrict__ sx, int sx_stride, const float *__restrict__ sw, int sw_stride,
                     uint16_t *__restrict__ y, int32_t *__restrict__ acc_out, int M, int N, int K, Outliers ol,
                     Sched sched, unsigned int *status, uint64_t limit_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sB = base + STAGES * A_BYTES;
    Smem *sm = reinterpret_cast<Smem *>(base + STAGES * STAGE_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = (M + BM - 1) / BM, nt = (N + BN - 1) / BN;
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
    int split_acc = -1, split_tile = 0;  // epilogue: accumulator and tile of the pair's shared tile

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            uint32_t it = 0;
            bool ok = true;
            int tile, kbb, kbe;
            bool half;
            for (int u = 0; ok && sched.unit(u, kblocks, tile, kbb, kbe, half); ++u) {
                const int m0 = (tile % mt) * BM, n0 = (tile / mt) * BN;
                for (int kb = kbb; kb < kbe; ++kb, ++it) {
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
            int tile, kbb, kbe;
            bool half;
            for (int u = 0; ok && sched.unit(u, kblocks, tile, kbb, kbe, half); ++u, ++tcount) {
                const uint32_t a = tcount & 1, ua = tcount >> 1;
                if (!wait_parity(smem_u32(&sm->tmem_empty[a]), (ua & 1) ^ 1, ctl, SITE_MMA)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + a * BN;
                for (int kb = kbb; kb < kbe; ++kb, ++it) {
                    const uint32_t s = it % STAGES, u = it / STAGES;
                    if (!wait_parity(smem_u32(&sm->full[s]), u & 1, ctl, SITE_MMA)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + s * A_BYTES), b_addr = smem_u32(sB + s * B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk)
                        mma_step<FP8>(d, umma_desc_sw128_kmajor(a_addr + kk * 32),
                                      umma_desc_sw128_kmajor(b_addr + kk * 32), (kb != kbb) || kk != 0);
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
        int tile, kbb, kbe;
        bool half;
        for (int u = 0; sched.unit(u, kblocks, tile, kbb, kbe, half); ++u, ++tcount) {
            const uint32_t a = tcount & 1, ua = tcount >> 1;
            bool ok = wait_parity(smem_u32(&sm->tmem_full[a]), ua & 1, ctl, SITE_EPILOGUE);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            if (SPLIT && half) {  // the pair's shared tile: summed and stored after the loop
                split_acc = (int)a;
                split_tile = tile;
                break;
            }
            const int m = (tile % mt) * BM + row;
            const int nb = (tile / mt) * BN;
            const float sxm = m < M ? __ldg(sx + m * sx_stride) : 0.0f;
            if (OUTL && ol.cap <= 64) {
                float *tr = reinterpret_cast<float *>(base + STAGES * STAGE_BYTES + 256) + (warp - 2) * 32 * TR_PITCH;
                const int r0 = m - row + q * 32;
                uint32_t xa[4][2][4], wb0[4][4][2], wb1[4][4][2];
                outlier_x_frags(ol, M, r0, lane, xa);
                outlier_w_frags(ol, N, nb, lane, wb0);
                // chunks in pairs so that each W_16 buffer has a fixed register home
#pragma unroll 1
                for (int c = 0; c < BN / 32; c += 2) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int cc = c + h;
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + a * BN + cc * 32, r);
                        if (cc + 1 < BN / 32) outlier_w_frags(ol, N, nb + (cc + 1) * 32, lane, h ? wb0 : wb1);
                        tmem_ld_wait();
                        if (nb + cc * 32 < N) {  // warp-uniform: the whole warp runs the outlier MMAs
                            float o[32];
                            outlier_mma64(xa, h ? wb1 : wb0, lane, tr, o);
                            if (m < M) store_chunk_outliers(y, m, nb + cc * 32, N, sxm, sw, r, o, vec_ok);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(smem_u32(&sm->tmem_empty[a]));
                continue;
            }
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + a * BN + c * 32, r);
                tmem_ld_wait();
                if (OUTL) {
                    if (nb + c * 32 < N) {  // warp-uniform: the whole warp runs the outlier MMAs
                        float o[32];
                        float *tr = reinterpret_cast<float *>(base + STAGES * STAGE_BYTES + 256) +
                                    (warp - 2) * 32 * TR_PITCH;
                        outlier_chunk(ol, M, N, m - row + q * 32, nb + c * 32, lane, tr, o);
                        if (m < M) store_chunk_outliers(y, m, nb + c * 32, N, sxm, sw, r, o, vec_ok);
                    }
                } else if (m < M && nb + c * 32 < N) {
                    store_chunk<FP8>(y, acc_out, m, nb + c * 32, N, sxm, sw, sw_stride, r, vec_ok);
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&sm->tmem_empty[a]));
        }
    }
    if (SPLIT) {
        // Every CTA of the pair is past its last wait: the MMAs of the shared tile are complete
        // (the epilogue warps waited for them) and every TMA load has landed, so both CTAs'
        // pipeline buffers are free.  The leading CTA stores the shared tile's columns 0..127 and
        // the second CTA columns 128..255: each first sends the other, through distributed shared
        // memory, the half of its partial accumulator that the other stores, so the two halves of
        // this last, unhidden epilogue run side by side.
        cluster_sync();
        const bool epi = warp >= 2;
        const int q = warp & 3, row = q * 32 + lane;
        const uint32_t second = blockIdx.x & 1;
        constexpr int HALF = BN / 64;                 // 32-column chunks per half
        const int c_mine = second ? HALF : 0, c_send = second ? 0 : HALF;
        uint32_t *part = reinterpret_cast<uint32_t *>(base);  // [BM][PART_PITCH] in each CTA of the pair
        if (epi && split_acc >= 0) {
            const uint32_t dst = mapa_shared(smem_u32(part + row * PART_PITCH), second ^ 1u);
#pragma unroll 1
            for (int c = c_send; c < c_send + HALF; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + split_acc * BN + c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    asm volatile("st.shared::cluster.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst + (c * 32 + j) * 4),
                                 "r"(r[j]), "r"(r[j + 1]), "r"(r[j + 2]), "r"(r[j + 3])
                                 : "memory");
            }
        }
        cluster_sync();
        if (epi && split_acc >= 0 && !sm->abort) {
            const int m = (split_tile % mt) * BM + row;
            const int nb = (split_tile / mt) * BN;
            const float sxm = m < M ? __ldg(sx + m * sx_stride) : 0.0f;
            const bool vec_ok = (N % 8) == 0;
            const uint32_t src = smem_u32(part + row * PART_PITCH);
            float *tr = reinterpret_cast<float *>(base + STAGES * STAGE_BYTES + 256) + (warp - 2) * 32 * TR_PITCH;
            // this CTA's partial of chunk c plus the other CTA's, which arrived in `part`
            auto summed = [&](int c, uint32_t (&r)[32]) {
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + split_acc * BN + c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    uint4 v;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                 : "r"(src + (c * 32 + j) * 4));
                    const uint32_t o[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)  // int32 sums are exact; fp32 sums of two terms commute
                        r[j + e] = FP8 ? __float_as_uint(__uint_as_float(r[j + e]) + __uint_as_float(o[e]))
                                       : r[j + e] + o[e];
                }
            };
            if (OUTL && ol.cap <= 64) {
                uint32_t xa[4][2][4], wb0[4][4][2], wb1[4][4][2];
                outlier_x_frags(ol, M, m - row + q * 32, lane, xa);
                outlier_w_frags(ol, N, nb + c_mine * 32, lane, wb0);
#pragma unroll 1
                for (int c = c_mine; c < c_mine + HALF; c += 2) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int cc = c + h;
                        if (cc + 1 < c_mine + HALF) outlier_w_frags(ol, N, nb + (cc + 1) * 32, lane, h ? wb0 : wb1);
                        uint32_t r[32];
                        summed(cc, r);
                        if (nb + cc * 32 < N) {  // warp-uniform
                            float o16[32];
                            outlier_mma64(xa, h ? wb1 : wb0, lane, tr, o16);
                            if (m < M) store_chunk_outliers(y, m, nb + cc * 32, N, sxm, sw, r, o16, vec_ok);
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int c = c_mine; c < c_mine + HALF; ++c) {
                    uint32_t r[32];
                    summed(c, r);
                    if (OUTL) {
                        if (nb + c * 32 < N) {  // warp-uniform: the whole warp runs the outlier MMAs
                            float o16[32];
                            outlier_chunk(ol, M, N, m - row + q * 32, nb + c * 32, lane, tr, o16);
                            if (m < M) store_chunk_outliers(y, m, nb + c * 32, N, sxm, sw, r, o16, vec_ok);
                        }
                    } else if (m < M && nb + c * 32 < N) {
                        store_chunk<FP8>(y, acc_out, m, nb + c * 32, N, sxm, sw, sw_stride, r, vec_ok);
                    }
                }
            }
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

namespace wq {
namespace {

// CTA pairs (clusters of 2, one CTA per SM) that can be resident at once, at most half the SMs;
// 0 if the query fails.  Cached per device.
int split_pairs(const void *kern, size_t smem, int sms) {
    static int cached[64][2] = {};  // per device, per shared-memory size (plain / LLM.int8())
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    int &slot = cached[dev][smem > SMEM_BYTES ? 1 : 0];
    if (slot) return slot > 0 ? slot : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sms / 2));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        clusters = -1;
    }
    const int pairs = clusters > 0 ? std::min(clusters, sms / 2) : -1;
    slot = pairs;
    return pairs > 0 ? pairs : 0;
}

// Shared launch path of the INT8, FP8 and LLM.int8() GEMMs (arguments already validated).
template <bool FP8, bool OUTL = false>
wq_status launch_gemm(const void *xq, const float *sx, int sx_stride, const void *wq_, const float *sw, int sw_stride,
                      int M, int N, int K, uint16_t *y, void *acc_out, void *stream, const char *who,
                      Outliers ol = Outliers{nullptr, nullptr, 0}) {
    unsigned int *status = device_status_word();
    if (!status) return WQ_ERR_CUDA;
    CUtensorMap tx, tw;
    if (!encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return WQ_ERR_CUDA;
    if (!encode_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, wq_, (uint64_t)K, (uint64_t)N, (uint64_t)K, BK, BN,
                        CU_TENSOR_MAP_SWIZZLE_128B))
        return WQ_ERR_CUDA;
    constexpr size_t smem = OUTL ? SMEM_BYTES_OUTL : SMEM_BYTES;
    cudaError_t e = cudaFuncSetAttribute(gemm_w8a8_kernel<FP8, OUTL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: cudaFuncSetAttribute failed: %s", who, cudaGetErrorString(e));
    const long long tiles = (long long)((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    WQ_REQUIRE(tiles < (1ll << 31), WQ_ERR_UNSUPPORTED, "%s: problem too large", who);
    const int sms = num_sms();
    const int kblocks = (K + BK - 1) / BK;
    // Split schedule when the tiles left after whole rounds fit one per CTA pair: the last
    // round then takes half a tile's time instead of a whole one.
    if (kblocks >= 2 && tiles > sms) {
        auto kern = gemm_w8a8_kernel<FP8, OUTL, true>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return fail(WQ_ERR_CUDA, "%s: cudaFuncSetAttribute failed: %s", who, cudaGetErrorString(e));
        const int pairs = split_pairs(reinterpret_cast<const void *>(kern), smem, sms);
        const int grid = 2 * pairs;
        const int full_rounds = grid > 0 ? (int)(tiles / grid) : 0;
        const int left = (int)(tiles - (long long)full_rounds * grid);
        // estimated time in tiles: full_rounds + 1/2 against ceil(tiles / sms) for the plain grid
        if (pairs > 0 && left > 0 && left <= pairs && full_rounds + 0.5 < (double)((tiles + sms - 1) / sms)) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(grid);
            cfg.blockDim = dim3(THREADS);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = as_stream(stream);
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            e = cudaLaunchKernelEx(&cfg, kern, tx, tw, sx, sx_stride, sw, sw_stride, y,
                                   reinterpret_cast<int32_t *>(acc_out), M, N, K, ol,
                                   Sched{(int)tiles, full_rounds, left}, status, wait_limit());
            if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: launch failed: %s", who, cudaGetErrorString(e));
            return WQ_OK;
        }
    }
    const int grid = (int)std::min<long long>(tiles, sms);
    gemm_w8a8_kernel<FP8, OUTL><<<grid, THREADS, smem, as_stream(stream)>>>(
        tx, tw, sx, sx_stride, sw, sw_stride, y, reinterpret_cast<int32_t *>(acc_out), M, N, K, ol,
        Sched{(int)tiles, 0, 0}, status, wait_limit());
    return check_launch(who);
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
    return launch_gemm<false>(xq, sx, 1, wq_, sw, 1, M, N, K, y, acc_out, stream, "wq_gemm_w8a8");
}

extern "C" wq_status wq_gemm_fp8(const uint8_t *xq, const float *sx, int sx_per_row, const uint8_t *wq_,
                                 const float *sw, int sw_per_row, int M, int N, int K, uint16_t *y, float *acc_out,
                                 void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(xq, "xq");
    WQ_REQUIRE_PTR(sx, "sx");
    WQ_REQUIRE_PTR(wq_, "wq");
    WQ_REQUIRE_PTR(sw, "sw");
    WQ_REQUIRE_PTR(y, "y");
    if (acc_out) WQ_REQUIRE(aligned16(acc_out), WQ_ERR_ALIGNMENT, "acc_out is not 16-byte aligned");
    WQ_REQUIRE(M > 0 && N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_gemm_fp8: sizes must be positive (M=%d N=%d K=%d)", M,
               N, K);
    WQ_REQUIRE(K % 16 == 0, WQ_ERR_UNSUPPORTED, "wq_gemm_fp8: K (%d) must be a multiple of 16", K);
    return launch_gemm<true>(xq, sx, sx_per_row ? 1 : 0, wq_, sw, sw_per_row ? 1 : 0, M, N, K, y, acc_out, stream,
                             "wq_gemm_fp8");
}

extern "C" wq_status wq_gemm_w8a8_outliers(const int8_t *xq, const float *sx, const int8_t *wq_, const float *sw,
                                           const uint16_t *x16, const uint16_t *w16, int cap, int M, int N, int K,
                                           uint16_t *y, void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(xq, "xq");
    WQ_REQUIRE_PTR(sx, "sx");
    WQ_REQUIRE_PTR(wq_, "wq");
    WQ_REQUIRE_PTR(sw, "sw");
    WQ_REQUIRE_PTR(x16, "x16");
    WQ_REQUIRE_PTR(w16, "w16");
    WQ_REQUIRE_PTR(y, "y");
    WQ_REQUIRE(M > 0 && N > 0 && K > 0, WQ_ERR_INVALID_ARG,
               "wq_gemm_w8a8_outliers: sizes must be positive (M=%d N=%d K=%d)", M, N, K);
    WQ_REQUIRE(K % 16 == 0, WQ_ERR_UNSUPPORTED, "wq_gemm_w8a8_outliers: K (%d) must be a multiple of 16", K);
    WQ_REQUIRE(K <= 131056, WQ_ERR_UNSUPPORTED, "wq_gemm_w8a8_outliers: K (%d) above 131056 could overflow int32", K);
    WQ_REQUIRE(cap >= 16 && cap <= 256 && cap % 16 == 0, WQ_ERR_UNSUPPORTED,
               "wq_gemm_w8a8_outliers: cap (%d) must be a multiple of 16 in [16, 256]", cap);
    return launch_gemm<false, true>(xq, sx, 1, wq_, sw, 1, M, N, K, y, nullptr, stream, "wq_gemm_w8a8_outliers",
                                    Outliers{x16, w16, cap});
}
