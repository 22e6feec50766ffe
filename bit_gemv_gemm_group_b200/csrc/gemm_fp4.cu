// Block-scaled FP4 GEMM (W4A4) on the 5th-generation tensor cores:
// tcgen05 kind::mxf4 (MXFP4: E2M1 x E2M1, E8M0 scales per 32) and
// kind::mxf4nvf4 (NVFP4: E2M1 x E2M1, E4M3 scales per 16, times the two fp32
// tensor scales in the epilogue), fp32 accumulators in tensor memory.
//
// Source: "Quantization: Smaller Weights, Same Answers (Mostly)", "What about
// FP8, MXFP4, NVFP4 and GGUF?" (block formats give every small block its own
// scale); "Quantization from Scratch", Formats ("a block scale in hardware is
// what group-wise quantization does in software"); "How quantization works",
// Mainstream schemes (FP4 on Blackwell).
//
//   y[m][n] = fp16_rn( ta * tb * sum_k e2m1(a[m][k]) sa[m][k/bs] e2m1(b[n][k]) sb[n][k/bs] )
//
// Persistent, warp-specialized CTA (one per SM, 192 threads), 128 x 128 tiles,
// 256 K (128 bytes of codes per row) per stage:
//   warp 0   lane 0 loads the A and B code tiles with TMA (128-byte swizzle) and
//            the stage's scale factors with two 1-D bulk copies: the quantizers
//            store them in the 512-byte atoms tcgen05.cp expects (row r of a
//            128-row block at byte 16 (r % 32) + 4 (r / 32) + j for its j-th
//            factor of a group of four, atoms row-block-major), so a tile's
//            factors for one stage are G contiguous atoms per operand
//   warp 1   allocates 512 TMEM columns (two 128-column accumulators and a
//            ring of scale-factor slots), copies a stage's factors into its
//            slot with tcgen05.cp (each 512-byte atom fills 4 columns, one
//            row per lane, replicated in the four subpartitions) and issues the
//            stage's four K = 64 MMAs, each naming its factors by column and
//            byte; tcgen05.commit frees the stage and signals the accumulator
//   warps 2-5 epilogue: tcgen05.ld, scale, convert, store, overlapping the
//            next tile's MMAs (two accumulators).
// Copies and MMAs issued by one thread execute in order, and a slot is only
// refilled once the MMAs that read it have completed (the ring has as many
// slots as the shared-memory ring has stages).  No multicast of any kind.
#include "sm100.cuh"
#include "wq_device.cuh"
#include "wq_host.h"

#include <algorithm>

namespace wq {
namespace {

using namespace sm100;

constexpr int BM = 128, BN = 128, BKB = 128;    // BKB: bytes of codes per row per stage (256 values)
constexpr int STAGES = 5;
constexpr uint32_t A_BYTES = BM * BKB;          // 16 KB
constexpr uint32_t B_BYTES = BN * BKB;          // 16 KB
constexpr uint32_t ATOM = 512;                  // 128 rows x 4 scale factors
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_TMEM0 = 2 * BN;           // first scale-factor column (after two accumulators)
constexpr int THREADS = 192;
constexpr uint64_t DRAIN_NS = 2000000000ull;
constexpr unsigned SITE_PRODUCER = 0x201, SITE_MMA = 0x202, SITE_EPILOGUE = 0x204, SITE_DRAIN = 0x208;

// Per-format constants: block size, scale groups of four per stage, E8M0 flag.
template <bool NV>
struct Fmt {
    static constexpr int BS = NV ? 16 : 32;           // values per scale factor
    static constexpr int G = 256 / BS / 4;            // groups of four factors per row per stage (4 or 2)
    static constexpr uint32_t SF_BYTES = 2 * G * ATOM;  // A and B atoms of one stage
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SF_BYTES;
    static constexpr uint32_t SF_COLS = 2 * G * 4;    // TMEM columns of one stage's factors
    static constexpr uint32_t IDESC = make_idesc_fp4(NV ? 0u : 1u, BM, BN);
    static constexpr size_t SMEM = 1024 + STAGES * STAGE_BYTES + 256;
    static_assert(SF_TMEM0 + STAGES * SF_COLS <= TMEM_COLS, "scale-factor slots fit in tensor memory");
    static_assert(SMEM <= 232448, "fits the 227 KB of shared memory a CTA may use");
};

struct Smem {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

template <bool NV>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const uint8_t *__restrict__ sfa, const uint8_t *__restrict__ sfb, const float *__restrict__ ta,
                    const float *__restrict__ tb, uint16_t *__restrict__ y, float *__restrict__ acc_out, int M, int N,
                    int K, unsigned int *status, uint64_t limit_ns) {
    using F = Fmt<NV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Smem *sm = reinterpret_cast<Smem *>(base + STAGES * F::STAGE_BYTES);
    const uint32_t sbase = smem_u32(base);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = (M + BM - 1) / BM, nt = (N + BN - 1) / BN;
    const int tiles = mt * nt;
    const int kblocks = K / 256;

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
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
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
            const int fg = K / F::BS / 4;  // atoms per 128-row block
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
                const int m0 = (tile % mt) * BM, n0 = (tile / mt) * BN;
                const uint8_t *sfa_t = sfa + ((size_t)(m0 / BM) * fg) * ATOM;
                const uint8_t *sfb_t = sfb + ((size_t)(n0 / BN) * fg) * ATOM;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const uint32_t s = it % STAGES, u = it / STAGES;
                    if (!wait_parity(smem_u32(&sm->empty[s]), (u & 1) ^ 1, ctl, SITE_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&sm->full[s]);
                    const uint32_t st = sbase + s * F::STAGE_BYTES;
                    mbar_arrive_expect_tx(fb, F::STAGE_BYTES);
                    tma_load_2d(st, &tmap_a, fb, kb * BKB, m0);
                    tma_load_2d(st + A_BYTES, &tmap_b, fb, kb * BKB, n0);
                    bulk_load(st + A_BYTES + B_BYTES, sfa_t + (size_t)kb * F::G * ATOM, F::G * ATOM, fb);
                    bulk_load(st + A_BYTES + B_BYTES + F::G * ATOM, sfb_t + (size_t)kb * F::G * ATOM, F::G * ATOM, fb);
                }
            }
            // Every issued copy must land before the CTA may exit.
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
                    const uint32_t st = sbase + s * F::STAGE_BYTES;
                    const uint32_t sf_src = st + A_BYTES + B_BYTES;
                    const uint32_t sf_a = tmem_base + SF_TMEM0 + s * F::SF_COLS;  // this stage's slot
                    const uint32_t sf_b = sf_a + F::G * 4;
#pragma unroll
                    for (int g = 0; g < F::G; ++g) {
                        tmem_cp_32x128b_warpx4(sf_a + 4 * g, utccp_desc_32x16(sf_src + g * ATOM));
                        tmem_cp_32x128b_warpx4(sf_b + 4 * g, utccp_desc_32x16(sf_src + (F::G + g) * ATOM));
                    }
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = umma_desc_sw128_kmajor(st + kk * 32);
                        const uint64_t bd = umma_desc_sw128_kmajor(st + A_BYTES + kk * 32);
                        const uint32_t acc = (kb | kk) != 0;
                        if (NV) {  // four factors per MMA: one full group
                            mma_nvf4(d, ad, bd, F::IDESC, sf_a + 4 * kk, sf_b + 4 * kk, acc);
                        } else {   // two factors per MMA: bytes 0-1 or 2-3 of a group
                            const uint32_t byte = 2 * (kk & 1);
                            mma_mxf4(d, ad, bd, idesc_sf_bytes(F::IDESC, byte, byte), sf_a + 4 * (kk >> 1),
                                     sf_b + 4 * (kk >> 1), acc);
                        }
                    }
                    tc_commit(smem_u32(&sm->empty[s]));
                }
                if (ok) tc_commit(smem_u32(&sm->tmem_full[a]));
            }
            tc_commit(smem_u32(&sm->drain));
            drain_parity(smem_u32(&sm->drain), 0, DRAIN_NS, status, SITE_DRAIN);
        }
        __syncwarp();
    } else {
        // -------------------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const float alpha = NV ? __fmul_rn(__ldg(ta), __ldg(tb)) : 1.0f;
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
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + a * BN + c * 32, r);
                tmem_ld_wait();
                const int n0 = nb + c * 32;
                if (m < M && n0 < N) {
                    if (vec_ok && n0 + 32 <= N) {
                        uint32_t h[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            h[j] = (uint32_t)float_to_half_bits_rn(__fmul_rn(__uint_as_float(r[2 * j]), alpha)) |
                                   ((uint32_t)float_to_half_bits_rn(__fmul_rn(__uint_as_float(r[2 * j + 1]), alpha))
                                    << 16);
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
                            if (n0 + j < N) {
                                y[(size_t)m * N + n0 + j] =
                                    float_to_half_bits_rn(__fmul_rn(__uint_as_float(r[j]), alpha));
                                if (acc_out) acc_out[(size_t)m * N + n0 + j] = __uint_as_float(r[j]);
                            }
                        }
                    }
                }
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

template <bool NV>
wq_status launch_fp4(const uint8_t *a, const uint8_t *sa, const float *ta, const uint8_t *b, const uint8_t *sb,
                     const float *tb, int M, int N, int K, uint16_t *y, float *acc_out, cudaStream_t st) {
    using F = Fmt<NV>;
    unsigned int *status = device_status_word();
    if (!status) return WQ_ERR_CUDA;
    CUtensorMap tma, tmb;
    if (!encode_tmap_2d(&tma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, BKB,
                        BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return WQ_ERR_CUDA;
    if (!encode_tmap_2d(&tmb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, b, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, BKB,
                        BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return WQ_ERR_CUDA;
    cudaError_t e = cudaFuncSetAttribute(gemm_fp4_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)F::SMEM);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_gemm_fp4: cudaFuncSetAttribute failed: %s", cudaGetErrorString(e));
    const long long tiles = (long long)((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    WQ_REQUIRE(tiles < (1ll << 31), WQ_ERR_UNSUPPORTED, "wq_gemm_fp4: problem too large");
    const int grid = (int)std::min<long long>(tiles, num_sms());
    gemm_fp4_kernel<NV><<<grid, THREADS, F::SMEM, st>>>(tma, tmb, sa, sb, ta, tb, y, acc_out, M, N, K, status,
                                                         wait_limit());
    return check_launch("wq_gemm_fp4");
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_gemm_fp4(int nvfp4, const uint8_t *a, const uint8_t *sfa, const float *ta, const uint8_t *b,
                                 const uint8_t *sfb, const float *tb, int M, int N, int K, uint16_t *y, float *acc_out,
                                 void *stream) {
    using namespace wq;
    WQ_REQUIRE_PTR(a, "a");
    WQ_REQUIRE_PTR(sfa, "sfa");
    WQ_REQUIRE_PTR(b, "b");
    WQ_REQUIRE_PTR(sfb, "sfb");
    WQ_REQUIRE_PTR(y, "y");
    if (nvfp4) {
        WQ_REQUIRE(ta != nullptr && tb != nullptr, WQ_ERR_INVALID_ARG, "wq_gemm_fp4: NVFP4 needs both tensor scales");
    }
    if (acc_out) WQ_REQUIRE(aligned16(acc_out), WQ_ERR_ALIGNMENT, "acc_out is not 16-byte aligned");
    WQ_REQUIRE(M > 0 && N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_gemm_fp4: sizes must be positive (M=%d N=%d K=%d)", M, N,
               K);
    WQ_REQUIRE(K % 256 == 0, WQ_ERR_UNSUPPORTED, "wq_gemm_fp4: K (%d) must be a multiple of 256", K);
    return nvfp4 ? launch_fp4<true>(a, sfa, ta, b, sfb, tb, M, N, K, y, acc_out, as_stream(stream))
                 : launch_fp4<false>(a, sfa, ta, b, sfb, tb, M, N, K, y, acc_out, as_stream(stream));
}
