// W4A16 GEMM on the tensor cores (tcgen05, kind::f16) for M >= 16 activation
// rows: packed INT4 tiles are dequantized into shared memory and fed to MMAs
// with fp32 accumulation in tensor memory.
//
// Source: "How quantization works", section "Inference view" (quantized
// weights are unpacked, multiplied by their scales and fed to the Tensor Cores
// inside the kernel); "Quantization from Scratch", sections "Scale and
// zero-point" (w^ = (q - z) s) and "What it buys at decode" (a batch of B
// sequences reads every weight once and does 2 FLOPs per weight per sequence).
//
//   y[m][n] = fp16_rn( sum_k fp16_rn(s[n][k/g] * (q[n][k] - z[n][k/g])) * x[m][k] )
//
// Group size g = 128 runs the paths tuned for it (scales of 8 groups fetched
// ahead, split-K in 16-stage parts); g = 32, 64 and 256 fetch each stage's
// scale and zero point one stage ahead (a thread's 32 codes of a stage always
// lie in one group).
//
// Swap-AB: the MMA's M dimension is 128 weight rows (TMEM lanes) and its N
// dimension is the activation tile (16..128 rows of x), so small batches still
// use full 128-row MMAs.  The dequantized weight tile never touches shared
// memory: the dequantizers write it into tensor memory (tcgen05.st), and the
// MMAs read their A operand from there, so shared memory holds only the TMA
// rings and the packed-code ring can be deep enough to keep HBM busy.  Per CTA
// (512 threads):
//   warp 0      TMA: packed weight tiles (128 rows x 32 bytes = 64 codes) into
//               a 16- or 24-deep ring (two or one CTAs per SM, see Layout)
//   warp 1      TMA: x tiles (MT rows x 64 fp16, 128-byte swizzle)
//   warps 2, 15 tcgen05.mma issue (4 x K=16 per stage, A from tensor memory),
//               warp 2 for the even stages and warp 15 for the odd ones, each
//               into its own fp32 accumulator in TMEM (warp 2 also allocates
//               it); one thread issues a tcgen05.mma only every ~50 cycles, so
//               a second issuer measured 6% (64 rows) to 16% (100-128 rows)
//               faster on B200
//   warps 3-10  dequantize: thread (warp w, lane l) owns weight row
//               32 (w mod 4) + l (the TMEM lanes its warp may access) and one
//               half of each 64-code stage; it turns its 32 codes into fp16
//               with PRMT/LOP3 (code -> 1024 + q), one exact fp16x2 fma
//               (-> q - z) and one fp16x2 multiply by the scale, and writes
//               them to the stage's 16 TMEM columns of its lane
//   warps 11-14 epilogue: tcgen05.ld of the two 128 x MT fp32 accumulators,
//               summed
// K is split over the S CTAs of a thread-block cluster when the weight tiles
// alone would leave SMs idle; their fp32 partial tiles are summed in the
// leading CTA's shared memory through distributed shared memory, so the
// kernel needs no global scratch.  No multicast of any kind.
#include "sm100.cuh"
#include "wq_device.cuh"
#include "wq_host.h"

#include <algorithm>

namespace wq {
namespace {

using namespace sm100;

constexpr int BMW = 128;                    // weight rows per tile (MMA M)
constexpr int BK = 64;                      // k per stage: 32 TMEM columns of fp16 pairs
constexpr int MAX_STAGES = 8;               // dequantized A stages in TMEM (barrier arrays)
constexpr int MAX_PSTAGES = 24;             // packed-tile ring (barrier arrays)
constexpr uint32_t A_COLS = BK / 2;         // TMEM columns per A stage
constexpr uint32_t P_BYTES = BMW * BK / 2;  // 4 KB of packed codes
constexpr int THREADS = 512;
constexpr int DQ_THREADS = 256;
constexpr uint64_t DRAIN_NS = 2000000000ull;
constexpr unsigned SITE_PRODUCER = 0x201, SITE_MMA = 0x202, SITE_DEQUANT = 0x204, SITE_EPILOGUE = 0x208,
                   SITE_DRAIN = 0x210;

// Activation tiles of up to 64 rows run two CTAs per SM (each CTA half of tensor memory, at
// most 64 registers per thread): measured on B200 that halves the time of the 64-row GEMM on
// the 28672x8192 projection against one CTA per SM, because a CTA's stage loop is bound by
// handoff latency rather than by any unit's throughput.  128-row tiles keep one CTA per SM.
// Tensor memory: two MT-column accumulators, then the A stages (32 columns each).
template <int MT>
struct Layout {
    static constexpr int CTAS_PER_SM = MT <= 64 ? 2 : 1;
    static constexpr uint32_t TMEM_COLS = MT <= 64 ? 256 : 512;
    static constexpr int STAGES = (int)((TMEM_COLS - 2 * MT) / A_COLS) < MAX_STAGES
                                      ? (int)((TMEM_COLS - 2 * MT) / A_COLS) : MAX_STAGES;
    static constexpr int PSTAGES = MT <= 64 ? 16 : 24;
    static constexpr uint32_t B_BYTES = MT * 128;
    // activation tiles get their own ring, deep enough that a tile is requested
    // well before the MMA needs it (x comes from L2; its latency would otherwise
    // stall the MMA warp every few stages)
    static constexpr int XSTAGES = MT <= 32 ? 6 : 4;
    static constexpr uint32_t OFF_B = 0;
    static constexpr uint32_t OFF_P = OFF_B + XSTAGES * B_BYTES;
    static constexpr uint32_t PIPE_BYTES = OFF_P + PSTAGES * P_BYTES;  // reused for split-K partials
    static constexpr size_t SMEM = 1024 + PIPE_BYTES + 1024;  // alignment slack + barriers
    static_assert(STAGES >= 2, "tensor memory holds at least two A stages");
    static_assert(OFF_P % 256 == 0, "packed tiles keep the 32-byte swizzle's 256-byte period");
};

struct Bars {
    uint64_t pk_full[MAX_PSTAGES];
    uint64_t pk_empty[MAX_PSTAGES];
    uint64_t a_full[MAX_STAGES];   // dequantized weight stage written to TMEM (256 arrivals)
    uint64_t st_empty[MAX_STAGES]; // A stage consumed by the MMAs
    uint64_t x_full[12];       // activation tile landed (TMA transaction count)
    uint64_t x_empty[12];      // activation tile consumed by the MMAs
    uint64_t tmem_full;
    uint64_t drain;            // issuer 0's outstanding MMAs (exit drain)
    uint64_t drain2;           // issuer 1's
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// fp16x2 constant (-(1024 + z), -(64 + z)) for zero point z.
__device__ __forceinline__ uint32_t zero_consts(uint32_t z) { return 0xD400E400u + z * 0x00100001u; }

// One word of 8 codes (k .. k+7) -> 8 fp16 weights fp16_rn(s (q - z)) in k order.
// Byte i holds codes 2i (low nibble) and 2i+1 (high nibble); PRMT copies it into
// both halves, LOP3 keeps the low nibble in the low half (1024 + q) and the high
// nibble in bits 4..7 of the high half (1024 + 16 q); one fma with (1, 1/16) and
// (-(1024+z), -(64+z)) gives q - z exactly, one multiply applies the scale.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t zc, uint32_t s2) {
    const uint32_t c1 = 0x2C003C00u;  // (1.0, 0.0625)
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t y = prmt(w, 0u, 0x4040u + 0x0101u * i);
        const uint32_t h = (y & 0x00F0000Fu) | 0x64006400u;
        o[i] = hmul2(hfma2(h, c1, zc), s2);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// bf16 tiles: q - z exactly in fp16 as above, then the product with the fp32 scale rounded once to
// bf16 (bf16_rn(s (q - z)); s is the stored fp16 value, exact in fp32).
__device__ __forceinline__ uint4 dequant_word_bf16(uint32_t w, uint32_t zc, float s) {
    const uint32_t c1 = 0x2C003C00u;  // (1.0, 0.0625)
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t y = prmt(w, 0u, 0x4040u + 0x0101u * i);
        const uint32_t h = (y & 0x00F0000Fu) | 0x64006400u;
        const float2 d = half2_bits_to_float2(hfma2(h, c1, zc));
        uint32_t b;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(b) : "f"(__fmul_rn(d.y, s)), "f"(__fmul_rn(d.x, s)));
        o[i] = b;
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <bool BF>
__device__ __forceinline__ uint16_t store_bits(float v) {
    return BF ? float_to_bf16_bits_rn(v) : float_to_half_bits_rn(v);
}

// Columns [c, c + 16) of the tile's accumulator for this warp's 32 TMEM lanes:
// the even-stage accumulator, plus the odd-stage one (MT columns further) when
// the second issuer ran.
__device__ __forceinline__ void load_acc16(uint32_t t_row, int c, int mt, bool two, uint32_t (&r)[16]) {
    tmem_ld_32x32b_x16(t_row + c, r);
    tmem_ld_wait();
    if (two) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t r2[8];
            tmem_ld_32x32b_x8(t_row + mt + c + 8 * h, r2);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 8; ++k)
                r[8 * h + k] = __float_as_uint(__uint_as_float(r[8 * h + k]) + __uint_as_float(r2[k]));
        }
    }
}

// BF: bf16 activations, dequantized bf16 tiles (kind::f16 with bf16 operands) and bf16 output.
template <int MT, bool SB, bool BF = false>
__global__ void __launch_bounds__(THREADS, Layout<MT>::CTAS_PER_SM)
    gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_x,
                      const uint16_t *__restrict__ scales, const uint32_t *__restrict__ qzeros,
                      uint16_t *__restrict__ y, int M, int N, int K, int gs, int splits, unsigned int *status,
                      uint64_t limit_ns) {
    using L = Layout<MT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bar = reinterpret_cast<Bars *>(base + L::PIPE_BYTES);
    const uint32_t sB = smem_u32(base + L::OFF_B), sP = smem_u32(base + L::OFF_P);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)blockIdx.x;  // cluster dims (splits, 1, 1)
    const int n0 = blockIdx.y * BMW, m0 = blockIdx.z * MT;
    const int kb_total = K / BK;
    const int nkb = kb_total / splits;
    const int kb0 = rank * nkb;
    const int groups = K / gs, zwords = (groups + 7) / 8;
    constexpr uint32_t IDESC = make_idesc(/*f32*/ 1, /*f16 or bf16*/ BF ? 1 : 0, BF ? 1 : 0, BMW, MT);
    constexpr uint32_t TMEM_COLS = L::TMEM_COLS;
    constexpr uint32_t A_COL0 = 2 * MT;  // first A stage column, after the two accumulators

    if (threadIdx.x == 0) {
        for (int p = 0; p < L::PSTAGES; ++p) {
            mbar_init(smem_u32(&bar->pk_full[p]), 1);
            mbar_init(smem_u32(&bar->pk_empty[p]), DQ_THREADS);
        }
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(smem_u32(&bar->a_full[s]), DQ_THREADS);
            mbar_init(smem_u32(&bar->st_empty[s]), 1);
        }
        for (int s = 0; s < L::XSTAGES; ++s) {
            mbar_init(smem_u32(&bar->x_full[s]), 1);
            mbar_init(smem_u32(&bar->x_empty[s]), 1);
        }
        mbar_init(smem_u32(&bar->tmem_full), 2);  // one commit per issuer
        mbar_init(smem_u32(&bar->drain), 1);
        mbar_init(smem_u32(&bar->drain2), 1);
        bar->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(&tmap_x);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(&bar->tmem_base), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = bar->tmem_base;
    const WaitCtl ctl{&bar->abort, status, limit_ns};

    if (warp == 0) {
        if (lane == 0) {  // ------------------------------------------------ packed-code producer
            int i = 0;
            for (; i < nkb; ++i) {
                const int p = i % L::PSTAGES, up = i / L::PSTAGES;
                if (!wait_parity(smem_u32(&bar->pk_empty[p]), (up & 1) ^ 1, ctl, SITE_PRODUCER)) break;
                const uint32_t fb = smem_u32(&bar->pk_full[p]);
                mbar_arrive_expect_tx(fb, P_BYTES);
                tma_load_2d(sP + p * P_BYTES, &tmap_q, fb, (kb0 + i) * (BK / 2), n0);
            }
            for (int p = 0; p < L::PSTAGES; ++p) {
                const int issued = i > p ? (i - p - 1) / L::PSTAGES + 1 : 0;
                if (issued) drain_parity(smem_u32(&bar->pk_full[p]), (issued - 1) & 1, DRAIN_NS, status, SITE_DRAIN);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ------------------------------------------------ activation producer
            int i = 0;
            for (; i < nkb; ++i) {
                const int s = i % L::XSTAGES, u = i / L::XSTAGES;
                if (!wait_parity(smem_u32(&bar->x_empty[s]), (u & 1) ^ 1, ctl, SITE_PRODUCER)) break;
                const uint32_t fb = smem_u32(&bar->x_full[s]);
                mbar_arrive_expect_tx(fb, L::B_BYTES);
                tma_load_2d(sB + s * L::B_BYTES, &tmap_x, fb, (kb0 + i) * BK, m0);
            }
            for (int s = 0; s < L::XSTAGES; ++s) {
                const int issued = i > s ? (i - s - 1) / L::XSTAGES + 1 : 0;
                if (issued) drain_parity(smem_u32(&bar->x_full[s]), (issued - 1) & 1, DRAIN_NS, status, SITE_DRAIN);
            }
        }
    } else if (warp == 2 || warp == 15) {
        if (lane == 0) {  // ------------------------------------------------ MMA issuers
            // Issuer j takes stages j, j + 2, ...  A-stage and x slots pass between the two
            // issuers in stage order: slot reuse waits for the dequantizers / producer, which
            // wait for the previous user's commit, so each barrier's phases stay in order.
            const int j = warp == 2 ? 0 : 1;
            const uint32_t acc = tmem_base + (uint32_t)(j * MT);
            const uint32_t drb = smem_u32(j ? &bar->drain2 : &bar->drain);
            bool ok = true;
            for (int i = j; i < nkb; i += 2) {
                const int s = i % L::STAGES, u = i / L::STAGES;
                const int xs = i % L::XSTAGES, xu = i / L::XSTAGES;
                if (!wait_parity(smem_u32(&bar->x_full[xs]), xu & 1, ctl, SITE_MMA) ||
                    !wait_parity(smem_u32(&bar->a_full[s]), u & 1, ctl, SITE_MMA)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_tm = tmem_base + A_COL0 + (uint32_t)s * A_COLS, b_addr = sB + xs * L::B_BYTES;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    mma_f16_tmem_a(acc, a_tm + kk * 8, umma_desc_sw128_kmajor(b_addr + kk * 32), IDESC,
                                   i != j || kk != 0);
                tc_commit(smem_u32(&bar->st_empty[s]));
                tc_commit(smem_u32(&bar->x_empty[xs]));
            }
            if (ok) tc_commit(smem_u32(&bar->tmem_full));
            tc_commit(drb);
            drain_parity(drb, 0, DRAIN_NS, status, SITE_DRAIN);
        }
        __syncwarp();
    } else if (warp < 11) {
        // -------------------------------------------------------------------- dequantizers
        // Warp w may access TMEM lanes 32 (w mod 4) .. + 31: thread (w, l) owns weight row
        // 32 (w mod 4) + l and half (w - 3) / 4 of each stage's 64 codes.
        const int row = 32 * (warp & 3) + lane, half = (warp - 3) >> 2;
        const int n = min(n0 + row, N - 1);
        const uint32_t t_a = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + A_COL0 + (uint32_t)half * (A_COLS / 2);
        const uint16_t *srow = scales + (size_t)n * groups;
        const uint32_t *zrow = qzeros + (size_t)n * zwords;
        bool ok = true;
        auto stage = [&](int i, uint32_t zc, uint32_t s2) -> bool {
            const int p = i % L::PSTAGES, up = i / L::PSTAGES;
            const int s = i % L::STAGES, u = i / L::STAGES;
            // Waits are warp-uniform: tcgen05.st and tcgen05.wait are warp-collective.
            if (!__all_sync(0xffffffffu, wait_parity(smem_u32(&bar->pk_full[p]), up & 1, ctl, SITE_DEQUANT)))
                return false;
            uint4 w;
            asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(w.x), "=r"(w.y), "=r"(w.z), "=r"(w.w)
                         : "r"(sP + p * P_BYTES + row * 32 + ((half ^ ((row >> 2) & 1)) << 4)));
            // The codes are in registers: the packed slot goes back to the producer (the proxy
            // fence orders this read before the next TMA write into the slot).
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(&bar->pk_empty[p]));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
            uint32_t o[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = BF ? dequant_word_bf16(ws[j], zc, half_bits_to_float((uint16_t)(s2 & 0xFFFFu)))
                                   : dequant_word(ws[j], zc, s2);
                o[4 * j] = v.x;
                o[4 * j + 1] = v.y;
                o[4 * j + 2] = v.z;
                o[4 * j + 3] = v.w;
            }
            if (!__all_sync(0xffffffffu, wait_parity(smem_u32(&bar->st_empty[s]), (u & 1) ^ 1, ctl, SITE_DEQUANT)))
                return false;
            tc_fence_after();
            tmem_st_32x32b_x16(t_a + (uint32_t)s * A_COLS, o);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(smem_u32(&bar->a_full[s]));
            return true;
        };
        auto two_stages = [&](int i, uint32_t zc, uint32_t s2) -> bool {
            return stage(i, zc, s2) && (i + 1 >= nkb || stage(i + 1, zc, s2));
        };
        if (SB) {
            // Scales and zero points of 8 groups (1024 codes) at a time, fetched one
            // such block ahead so their latency hides behind 16 stages of work.
            const int sb0 = kb0 / 16, nsb = nkb / 16;
            uint4 cs = __ldg(reinterpret_cast<const uint4 *>(srow) + sb0);
            uint32_t cz = __ldg(zrow + sb0);
            for (int b = 0; b < nsb && ok; ++b) {
                uint4 ns = cs;
                uint32_t nz = cz;
                if (b + 1 < nsb) {
                    ns = __ldg(reinterpret_cast<const uint4 *>(srow) + sb0 + b + 1);
                    nz = __ldg(zrow + sb0 + b + 1);
                }
                const uint32_t sv[4] = {cs.x, cs.y, cs.z, cs.w};
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const uint32_t s2 = prmt(sv[g >> 1], 0u, (g & 1) ? 0x3232u : 0x1010u);
                    const uint32_t zc = zero_consts((cz >> (4 * g)) & 0xFu);
                    if (!two_stages(b * 16 + 2 * g, zc, s2)) {
                        ok = false;
                        break;
                    }
                }
                cs = ns;
                cz = nz;
            }
        } else if (gs == 128) {
            for (int i = 0; i < nkb && ok; i += 2) {
                const int g = (kb0 + i) >> 1;
                const uint32_t sh = __ldg(srow + g);
                const uint32_t s2 = sh | (sh << 16);
                const uint32_t zc = zero_consts((__ldg(zrow + (g >> 3)) >> (4 * (g & 7))) & 0xFu);
                ok = two_stages(i, zc, s2);
            }
        } else {
            // Group sizes 32, 64 and 256: a thread's 32 codes of a stage lie in one group (groups
            // start on multiples of 32), whose scale and zero point it fetches one stage ahead.
            auto fetch = [&](int i, uint32_t &zc, uint32_t &s2) {
                const int g = ((kb0 + i) * BK + half * 32) / gs;
                const uint32_t sh = __ldg(srow + g);
                s2 = sh | (sh << 16);
                zc = zero_consts((__ldg(zrow + (g >> 3)) >> (4 * (g & 7))) & 0xFu);
            };
            uint32_t zc, s2;
            fetch(0, zc, s2);
            for (int i = 0; i < nkb && ok; ++i) {
                uint32_t zn = zc, sn = s2;
                if (i + 1 < nkb) fetch(i + 1, zn, sn);
                ok = stage(i, zc, s2);
                zc = zn;
                s2 = sn;
            }
        }
    }

    // ------------------------------------------------------------------------ epilogue
    const bool epi = warp >= 11 && warp < 15;
    const bool two = nkb > 1;  // issuer 1 ran at least one stage
    const int q = warp & 3;
    const int erow = q * 32 + lane;
    const int n = n0 + erow;
    bool have_acc = false;
    if (epi) {
        have_acc = wait_parity(smem_u32(&bar->tmem_full), 0, ctl, SITE_EPILOGUE);
        have_acc = __all_sync(0xffffffffu, have_acc);
        tc_fence_after();
    }
    const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16);
    if (splits == 1) {
        if (epi && have_acc) {
#pragma unroll 1
            for (int c = 0; c < MT; c += 16) {
                uint32_t r[16];
                load_acc16(t_row, c, MT, two, r);
                if (n < N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (m0 + c + j < M)
                            y[(size_t)(m0 + c + j) * N + n] = store_bits<BF>(__uint_as_float(r[j]));
                }
            }
        }
    } else {
        // Split-K: partial tiles of CTAs 1..S-1 go to CTA 0's shared memory (the
        // pipeline buffers, idle by now), CTA 0 adds them in rank order.
        cluster_sync();  // every CTA of the cluster is past its main loop
        const uint32_t red = smem_u32(base);
        if (epi && rank != 0) {
            const uint32_t slot = mapa_shared(red, 0) + (uint32_t)((rank - 1) * BMW + erow) * MT * 4;
#pragma unroll 1
            for (int c = 0; c < MT; c += 16) {
                uint32_t r[16];
                load_acc16(t_row, c, MT, two, r);
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    st_cluster_v4(slot + (c + j) * 4, __uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                  __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
            }
        }
        cluster_sync();  // partials have landed
        if (epi && rank == 0) {
            const float *redp = reinterpret_cast<const float *>(base);
#pragma unroll 1
            for (int c = 0; c < MT; c += 16) {
                uint32_t r[16];
                load_acc16(t_row, c, MT, two, r);
                float acc[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] = __uint_as_float(r[j]);
                for (int sl = 0; sl < splits - 1; ++sl) {
                    const float *pp = redp + (size_t)(sl * BMW + erow) * MT + c;
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[j] += pp[j];
                }
                if (n < N && have_acc) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (m0 + c + j < M) y[(size_t)(m0 + c + j) * N + n] = store_bits<BF>(acc[j]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <int MT, bool SB, bool BF>
wq_status launch(const CUtensorMap &tq, const CUtensorMap &tx, const uint16_t *scales, const uint32_t *qzeros,
                 uint16_t *y, int M, int N, int K, int gs, int splits, unsigned int *status, cudaStream_t st) {
    auto kern = gemm_w4a16_kernel<MT, SB, BF>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Layout<MT>::SMEM);
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_gemm_w4a16: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(splits, (N + BMW - 1) / BMW, (M + MT - 1) / MT);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = Layout<MT>::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tq, tx, scales, qzeros, y, M, N, K, gs, splits, status, wait_limit());
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "wq_gemm_w4a16: launch failed: %s", cudaGetErrorString(e));
    return WQ_OK;
}

// Number of CTAs sharing one weight tile's K range: a divisor of the stage
// count (a multiple of 16 stages each on the fast path), at most 8, whose
// partial tiles fit the leading CTA's pipeline buffers, chosen to fill the
// SMs in as few, as full waves as possible.  The group-size-128 path without
// the fast path takes no split; the other group sizes take any divisor.
int choose_splits(int tiles, int K, int MT, bool fast, bool generic, size_t pipe_bytes, int sms) {
    const int kb = K / BK;
    int best = 1;
    double best_eff = -1.0;
    for (int s = 1; s <= 8; ++s) {
        if (kb % s) continue;
        if (fast && (kb / s) % 16) continue;
        if (!fast && !generic && s > 1) continue;
        if ((size_t)(s - 1) * BMW * MT * 4 > pipe_bytes) continue;
        const double waves = (double)tiles * s / sms;
        const double eff = waves / std::ceil(waves);
        if (eff > best_eff + 0.02) {
            best_eff = eff;
            best = s;
        }
    }
    return best;
}

template <int MT, bool BF>
wq_status dispatch(const CUtensorMap &tq, const CUtensorMap &tx, const uint16_t *scales, const uint32_t *qzeros,
                   uint16_t *y, int M, int N, int K, int gs, unsigned int *status, cudaStream_t st) {
    const bool fast = gs == 128 && (K % 1024) == 0;
    const int tiles = ((N + BMW - 1) / BMW) * ((M + MT - 1) / MT);
    const int splits = choose_splits(tiles, K, MT, fast, gs != 128, Layout<MT>::PIPE_BYTES,
                                     Layout<MT>::CTAS_PER_SM * num_sms());
    if (fast && (K / BK / splits) % 16 == 0)
        return launch<MT, true, BF>(tq, tx, scales, qzeros, y, M, N, K, gs, splits, status, st);
    return launch<MT, false, BF>(tq, tx, scales, qzeros, y, M, N, K, gs, splits, status, st);
}

}  // namespace
}  // namespace wq

namespace wq {
namespace {

template <bool BF>
wq_status gemm_w4a16_entry(const uint16_t *x, int M, const uint32_t *qweight, const uint16_t *scales,
                           const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y, void *stream,
                           const char *who) {
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(qweight, "qweight");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE_PTR(qzeros, "qzeros");
    WQ_REQUIRE_PTR(y, "y");
    WQ_REQUIRE(M > 0 && N > 0 && K > 0, WQ_ERR_INVALID_ARG, "%s: sizes must be positive (M=%d N=%d K=%d)", who, M, N,
               K);
    WQ_REQUIRE(group_size == 32 || group_size == 64 || group_size == 128 || group_size == 256, WQ_ERR_UNSUPPORTED,
               "%s: group_size must be 32, 64, 128 or 256 (got %d)", who, group_size);
    WQ_REQUIRE(K % group_size == 0, WQ_ERR_INVALID_ARG, "%s: K (%d) must be a multiple of group_size (%d)", who, K,
               group_size);
    WQ_REQUIRE(K % 128 == 0, WQ_ERR_INVALID_ARG, "%s: K (%d) must be a multiple of 128", who, K);
    const bool stream_ok = !BF && group_size == 128 && K % 256 == 0;  // the fp16 streaming kernel
    WQ_REQUIRE(M >= 16 || (M >= 9 && (K % 256 == 0 || group_size != 128 || BF)), WQ_ERR_UNSUPPORTED,
               "%s: M (%d) below 16 needs K %% 256 == 0 (K = %d); use the GEMV for M <= 8", who, M, K);
    // Below 16 rows without the streaming kernel: the CUDA-core GEMV in passes of up to 8 rows.
    if (M < 16 && !stream_ok) {
        for (int r0 = 0; r0 < M; r0 += 8) {
            const wq_status e = BF ? wq_gemv_w4a16_bf16(x + (size_t)r0 * K, std::min(8, M - r0), qweight, scales,
                                                        qzeros, N, K, group_size, y + (size_t)r0 * N, stream)
                                   : wq_gemv_w4a16(x + (size_t)r0 * K, std::min(8, M - r0), qweight, scales, qzeros,
                                                   N, K, group_size, y + (size_t)r0 * N, stream);
            if (e != WQ_OK) return e;
        }
        return WQ_OK;
    }
    // Up to 32 activation rows the byte stream dominates: the streaming mma.sync kernel (codes
    // dequantized in registers, no shared-memory fp16 tile) takes up to 16 rows per pass (it also
    // serves 9 <= M < 16, which the tensor-core kernel below does not take) and, measured
    // on B200, beats the tensor-core kernel below at M <= 32 (2 passes at M = 32 take 0.36x its
    // time on the 28672x8192 projection; at three passes the two are even).
    if (stream_ok && M <= 32) {
        for (int r0 = 0; r0 < M; r0 += 16) {
            const wq_status e = gemv_stream(x + (size_t)r0 * K, std::min(16, M - r0), qweight, scales, qzeros, N, K,
                                            y + (size_t)r0 * N, as_stream(stream), who);
            if (e != WQ_OK) return e;
        }
        return WQ_OK;
    }
    unsigned int *status = device_status_word();
    if (!status) return WQ_ERR_CUDA;
    const int MT = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
    CUtensorMap tq, tx;
    // 32-byte swizzle: half h of row r lands at h ^ ((r / 4) mod 2), so the dequantizers' 16-byte loads
    // (one row per lane, rows 32 bytes apart) spread over all 32 banks.
    if (!encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qweight, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2,
                        BK / 2, BMW, CU_TENSOR_MAP_SWIZZLE_32B))
        return WQ_ERR_CUDA;
    if (!encode_tmap_2d(&tx, BF ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, x, (uint64_t)K,
                        (uint64_t)M, (uint64_t)K * 2, BK, MT, CU_TENSOR_MAP_SWIZZLE_128B))
        return WQ_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    switch (MT) {
        case 16: return dispatch<16, BF>(tq, tx, scales, qzeros, y, M, N, K, group_size, status, st);
        case 32: return dispatch<32, BF>(tq, tx, scales, qzeros, y, M, N, K, group_size, status, st);
        case 64: return dispatch<64, BF>(tq, tx, scales, qzeros, y, M, N, K, group_size, status, st);
        default: return dispatch<128, BF>(tq, tx, scales, qzeros, y, M, N, K, group_size, status, st);
    }
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_gemm_w4a16(const uint16_t *x, int M, const uint32_t *qweight, const uint16_t *scales,
                                   const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y, void *stream) {
    return wq::gemm_w4a16_entry<false>(x, M, qweight, scales, qzeros, N, K, group_size, y, stream, "wq_gemm_w4a16");
}

extern "C" wq_status wq_gemm_w4a16_bf16(const uint16_t *x, int M, const uint32_t *qweight, const uint16_t *scales,
                                        const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y,
                                        void *stream) {
    return wq::gemm_w4a16_entry<true>(x, M, qweight, scales, qzeros, N, K, group_size, y, stream,
                                      "wq_gemm_w4a16_bf16");
}
