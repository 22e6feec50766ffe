// Calibration-driven INT4 quantization on the GPU: GPTQ and AWQ's scaling
// search, producing the stored INT4 format of wq_quantize_group_int4.
//
// Source: "Quantization from Scratch", sections "GPTQ: rounding with error
// compensation" (quantize one input column at a time, push each column's
// rounding error onto the columns not yet quantized through the Cholesky
// factor of the inverse Hessian H = 2 X^T X, in blocks of 128 columns) and
// "AWQ: protect the channels that matter" (scale input channel j of the
// weights by s_j = mean|x_j|^alpha, choose alpha on calibration data), and the
// gptq() / awq() routines of "Measured on two real layers"; "Quantization"
// (engine-room ch. 15), "The Mathematics" (GPTQ's objective and Hessian).
//
// Pieces, all fp32 on the CUDA cores (the work is K^3 / 3 for the factor and
// N K^2 for the compensation, small next to the matmuls it prepares):
//   gemm_nt_kernel    C = beta C + alpha sum_k A(m, k) B(n, k) over strided
//                     operands (64 x 64 tiles, 4 x 4 outputs per thread); it
//                     forms H = 2 X^T X and GPTQ's trailing updates.
//   Cholesky          right-looking in 64-column blocks: a one-CTA kernel
//                     factors the diagonal block and inverts its factor, a
//                     panel kernel applies that inverse to the blocks below,
//                     the GEMM updates the trailing lower triangle.
//   U = chol(H'^-1)   without forming H'^-1: with P the index reversal,
//                     chol(P H' P) = Lr gives U = P Lr^-1 P (upper, positive
//                     diagonal, U^T U = H'^-1); Lr^-1 comes block row by block
//                     row from the inverted diagonal blocks.
//   GPTQ block        one warp per weight row walks a block's 128 columns in
//                     order (4 per lane), U's diagonal block in shared memory;
//                     the errors E then update the later columns (GEMM).
//   AWQ               channel means of |x|, per alpha: scales, W * s, the INT4
//                     quantizer, and the objective 2 ||X D^T||^2 of the
//                     dequantized difference D, fused into one tiled kernel;
//                     the first smallest objective wins (device-side select).
#include "wq_device.cuh"
#include "wq_host.h"

#include <algorithm>
#include <cmath>

namespace wq {
namespace {

constexpr int TB = 64;     // tile / block size
constexpr int TK = 16;     // k per smem step
constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<uint16_t>(uint16_t v) { return half_bits_to_float(v); }

// C[m][n] = beta * C[m][n] + alpha * sum_k A(m, k) B(n, k) for m < M, n < N, with
// A(m, k) = A[m * sam + k * sak] and B(n, k) = B[n * sbn + k * sbk]; C has row pitch ldc.
// lower_only: tiles strictly above the diagonal (tile column > tile row) are skipped.
template <typename TA, typename TB_>
__global__ void __launch_bounds__(kThreads) gemm_nt_kernel(int M, int N, int Kd, const TA *__restrict__ A, long sam,
                                                           long sak, const TB_ *__restrict__ B, long sbn, long sbk,
                                                           float *__restrict__ C, long ldc, float alpha, float beta,
                                                           int lower_only) {
    if (lower_only && blockIdx.x > blockIdx.y) return;
    __shared__ float As[TK][TB + 4], Bs[TK][TB + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m0 = blockIdx.y * TB, n0 = blockIdx.x * TB;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < Kd; k0 += TK) {
        for (int e = threadIdx.x; e < TK * TB; e += kThreads) {
            const int kk = e / TB, r = e % TB;
            const int k = k0 + kk;
            As[kk][r] = (m0 + r < M && k < Kd) ? to_f(A[(long)(m0 + r) * sam + (long)k * sak]) : 0.0f;
            Bs[kk][r] = (n0 + r < N && k < Kd) ? to_f(B[(long)(n0 + r) * sbn + (long)k * sbk]) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[kk][ty * 4 + i];
                b[i] = Bs[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + j;
            if (m < M && n < N) {
                float *c = C + (long)m * ldc + n;
                *c = beta == 0.0f ? alpha * acc[i][j] : fmaf(alpha, acc[i][j], beta * *c);
            }
        }
}

template <typename TA, typename TB_>
cudaError_t gemm_nt(int M, int N, int Kd, const TA *A, long sam, long sak, const TB_ *B, long sbn, long sbk, float *C,
                    long ldc, float alpha, float beta, bool lower_only, cudaStream_t st) {
    if (M <= 0 || N <= 0) return cudaSuccess;
    dim3 grid((N + TB - 1) / TB, (M + TB - 1) / TB);
    gemm_nt_kernel<TA, TB_><<<grid, kThreads, 0, st>>>(M, N, Kd, A, sam, sak, B, sbn, sbk, C, ldc, alpha, beta,
                                                       lower_only ? 1 : 0);
    return cudaGetLastError();
}

// A' = P (A + damp * mean(diag A) I) P (P reverses the index order), one CTA per 64 x 64 tile
// after a one-CTA pass that computes the mean diagonal.
__global__ void __launch_bounds__(kThreads) mean_diag_kernel(const float *__restrict__ A, int K, float *out) {
    __shared__ float red[kThreads];
    float s = 0.0f;
    for (int i = threadIdx.x; i < K; i += kThreads) s += A[(long)i * K + i];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int off = kThreads / 2; off > 0; off >>= 1) {
        if (threadIdx.x < off) red[threadIdx.x] += red[threadIdx.x + off];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = red[0] / (float)K;
}

__global__ void __launch_bounds__(kThreads) damp_reverse_kernel(const float *__restrict__ H, int K, float damp,
                                                                const float *__restrict__ mean_diag,
                                                                float *__restrict__ A) {
    const float add = damp * *mean_diag;
    const long n = (long)K * K;
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < n; e += (long)gridDim.x * kThreads) {
        const int i = (int)(e / K), j = (int)(e % K);
        float v = H[(long)(K - 1 - i) * K + (K - 1 - j)];
        if (i == j) v += add;
        A[e] = v;
    }
}

// Factors the diagonal block [j0, j0 + 64) of A in place (lower Cholesky factor, fp32) and
// writes the inverse of that factor to Dinv (64 x 64, lower).  One CTA of 256 threads.
__global__ void __launch_bounds__(kThreads) potrf_diag_kernel(float *__restrict__ A, int K, int j0,
                                                              float *__restrict__ Dinv) {
    __shared__ float L[TB][TB + 1], Li[TB][TB + 1];
    for (int e = threadIdx.x; e < TB * TB; e += kThreads) {
        const int r = e / TB, c = e % TB;
        L[r][c] = A[(long)(j0 + r) * K + j0 + c];
        Li[r][c] = 0.0f;
    }
    __syncthreads();
    for (int j = 0; j < TB; ++j) {  // right-looking, column j
        if (threadIdx.x == 0) L[j][j] = sqrtf(fmaxf(L[j][j], 1e-30f));  // pivots are positive for SPD input
        __syncthreads();
        const float djj = L[j][j];
        for (int r = j + 1 + threadIdx.x; r < TB; r += kThreads) L[r][j] = __fdiv_rn(L[r][j], djj);
        __syncthreads();
        for (int e = threadIdx.x; e < TB * TB; e += kThreads) {
            const int r = e / TB, c = e % TB;
            if (c > j && r >= c) L[r][c] = fmaf(-L[r][j], L[c][j], L[r][c]);
        }
        __syncthreads();
    }
    // inverse of the lower factor, one column per thread (forward substitution)
    if (threadIdx.x < TB) {
        const int c = threadIdx.x;
        for (int i = c; i < TB; ++i) {
            float v = (i == c) ? 1.0f : 0.0f;
            for (int k = c; k < i; ++k) v = fmaf(-L[i][k], Li[k][c], v);
            Li[i][c] = __fdiv_rn(v, L[i][i]);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < TB * TB; e += kThreads) {
        const int r = e / TB, c = e % TB;
        A[(long)(j0 + r) * K + j0 + c] = c <= r ? L[r][c] : 0.0f;
        Dinv[e] = c <= r ? Li[r][c] : 0.0f;
    }
}

// Panel: block (ib, jb) for ib > jb becomes A[ib][jb] Dinv^T (one CTA per block, in place).
__global__ void __launch_bounds__(kThreads) panel_kernel(float *__restrict__ A, int K, int j0,
                                                         const float *__restrict__ Dinv) {
    __shared__ float P[TB][TB + 1], D[TB][TB + 1];
    const int r0 = j0 + TB * (1 + blockIdx.x);
    for (int e = threadIdx.x; e < TB * TB; e += kThreads) {
        const int r = e / TB, c = e % TB;
        P[r][c] = A[(long)(r0 + r) * K + j0 + c];
        D[r][c] = Dinv[e];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < TB * TB; e += kThreads) {
        const int r = e / TB, c = e % TB;
        float v = 0.0f;
        for (int k = 0; k <= c; ++k) v = fmaf(P[r][k], D[c][k], v);  // (P Dinv^T)[r][c], Dinv lower
        A[(long)(r0 + r) * K + j0 + c] = v;
    }
}

// Block row ib of the inverse of the lower factor L (stored in A's lower triangle):
// Linv[ib][jb] = -Dinv[ib] * sum_{kb = jb}^{ib - 1} L[ib][kb] Linv[kb][jb] for jb < ib, and
// Linv[ib][ib] = Dinv[ib].  One CTA per jb (blockIdx.x = jb; the last one copies Dinv[ib]).
__global__ void __launch_bounds__(kThreads) trinv_row_kernel(const float *__restrict__ A, int K, int ib,
                                                             const float *__restrict__ Dinv_all,
                                                             float *__restrict__ Linv) {
    __shared__ float Ls[TB][TB + 1], Xs[TB][TB + 1];
    const int jb = blockIdx.x;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    if (jb == ib) {
        for (int e = threadIdx.x; e < TB * TB; e += kThreads)
            Linv[(long)(ib * TB + e / TB) * K + ib * TB + e % TB] = Dinv_all[(long)ib * TB * TB + e];
        return;
    }
    float acc[4][4] = {};
    for (int kb = jb; kb < ib; ++kb) {
        for (int e = threadIdx.x; e < TB * TB; e += kThreads) {
            const int r = e / TB, c = e % TB;
            Ls[r][c] = A[(long)(ib * TB + r) * K + kb * TB + c];
            Xs[r][c] = Linv[(long)(kb * TB + r) * K + jb * TB + c];
        }
        __syncthreads();
        for (int k = 0; k < TB; ++k) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = Ls[ty * 4 + i][k];
                b[i] = Xs[k][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    // T = acc; Linv[ib][jb] = -Dinv[ib] T
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Xs[ty * 4 + i][tx * 4 + j] = acc[i][j];
    for (int e = threadIdx.x; e < TB * TB; e += kThreads) Ls[e / TB][e % TB] = Dinv_all[(long)ib * TB * TB + e];
    __syncthreads();
    for (int e = threadIdx.x; e < TB * TB; e += kThreads) {
        const int r = e / TB, c = e % TB;
        float v = 0.0f;
        for (int k = 0; k <= r; ++k) v = fmaf(Ls[r][k], Xs[k][c], v);
        Linv[(long)(ib * TB + r) * K + jb * TB + c] = -v;
    }
}

// U[i][j] = Linv[K-1-i][K-1-j] (upper triangular).
__global__ void __launch_bounds__(kThreads) reverse_kernel(const float *__restrict__ Linv, int K, float *__restrict__ U) {
    const long n = (long)K * K;
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < n; e += (long)gridDim.x * kThreads) {
        const int i = (int)(e / K), j = (int)(e % K);
        U[e] = j >= i ? Linv[(long)(K - 1 - i) * K + (K - 1 - j)] : 0.0f;
    }
}

// ---------------------------------------------------------------------------- GPTQ
// The stored-format grid of one group from the warp's values (4 per lane), exactly as the
// INT4 quantizer computes it: range widened to contain 0, s = fp16((hi - lo) / 15) (1 if 0),
// z = clamp(rne(-lo / s), 0, 15).
__device__ __forceinline__ void warp_grid(const float (&v)[4], uint16_t &s16, float &s, int &z) {
    float lo = 0.0f, hi = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        lo = fminf(lo, v[c]);
        hi = fmaxf(hi, v[c]);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    s16 = float_to_half_bits_rn(__fdiv_rn(hi - lo, 15.0f));
    if (s16 == 0) s16 = 0x3c00;
    s = half_bits_to_float(s16);
    z = clampi(__float2int_rn(__fdiv_rn(-lo, s)), 0, 15);
}

constexpr int GQ_ROWS = 8;  // weight rows (warps) per CTA

// One block of GPTQ (group b, 128 columns) for 8 rows per CTA.  W: fp32 working copy [N][K];
// U: [K][K]; E: out [N][128] scaled errors.  Codes, scale and zero point of the group are
// written in the stored format (qzeros cleared by the caller beforehand).
__global__ void __launch_bounds__(GQ_ROWS * 32) gptq_block_kernel(float *__restrict__ W, int N, int K, int b,
                                                                 const float *__restrict__ U, float *__restrict__ E,
                                                                 uint32_t *__restrict__ qweight,
                                                                 uint16_t *__restrict__ scales,
                                                                 uint32_t *__restrict__ qzeros) {
    constexpr int G = 128;
    extern __shared__ float gq_smem[];
    float *Ub = gq_smem;                                           // [128][128] diagonal block of U
    uint8_t *codes = reinterpret_cast<uint8_t *>(gq_smem + G * G);  // [8 warps][128]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i1 = b * G;
    for (int e = threadIdx.x; e < G * G; e += blockDim.x) Ub[e] = U[(long)(i1 + e / G) * K + i1 + e % G];
    __syncthreads();
    const int n = blockIdx.x * GQ_ROWS + warp;
    if (n >= N) return;
    float *row = W + (long)n * K + i1;
    float v[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) v[c] = row[32 * c + lane];
    uint16_t s16;
    float s;
    int z;
    warp_grid(v, s16, s, z);
    uint8_t *cw = codes + warp * G;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll 1
        for (int l = 0; l < 32; ++l) {
            const int i = 32 * c + l;
            const float wi = __shfl_sync(0xffffffffu, v[c], l);
            const int q = clampi(__float2int_rn(__fdiv_rn(wi, s)) + z, 0, 15);
            const float e = __fdiv_rn(wi - (float)(q - z) * s, Ub[i * G + i]);
#pragma unroll
            for (int c2 = c; c2 < 4; ++c2) {
                const int j = 32 * c2 + lane;
                if (j > i) v[c2] = fmaf(-e, Ub[i * G + j], v[c2]);
            }
            if (lane == l) {
                cw[i] = (uint8_t)q;
                E[(long)n * G + i] = e;
            }
        }
    }
    __syncwarp();
    if (lane < G / 8) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) word |= (uint32_t)cw[lane * 8 + e] << (4 * e);
        qweight[(long)n * (K / 8) + i1 / 8 + lane] = word;
    }
    if (lane == 0) {
        const int groups = K / G;
        scales[(long)n * groups + b] = s16;
        uint32_t *zp = qzeros + (long)n * ((groups + 7) / 8) + b / 8;
        *zp |= (uint32_t)z << (4 * (b % 8));
    }
}

__global__ void __launch_bounds__(kThreads) half_to_float_kernel(const uint16_t *__restrict__ w, long n,
                                                                 float *__restrict__ out) {
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < n; e += (long)gridDim.x * kThreads)
        out[e] = half_bits_to_float(w[e]);
}

int grid_for(long items) {
    return (int)std::max<long>(1, std::min<long>((items + kThreads - 1) / kThreads, (long)num_sms() * 8));
}

// ---------------------------------------------------------------------------- AWQ
// mag[j] = mean_t |x[t][j]| (fp64 sums).
__global__ void __launch_bounds__(kThreads) channel_mean_abs_kernel(const uint16_t *__restrict__ x, int T, int K,
                                                                    double *__restrict__ mag) {
    const int j = blockIdx.x * kThreads + threadIdx.x;
    if (j >= K) return;
    double s = 0.0;
    for (int t = 0; t < T; ++t) s += (double)fabsf(half_bits_to_float(x[(long)t * K + j]));
    mag[j] = s / (double)T;
}

// s_j = fp32(mag_j^alpha / sqrt(max * min)); one CTA.
__global__ void __launch_bounds__(1024) awq_scales_kernel(const double *__restrict__ mag, int K, double alpha,
                                                          float *__restrict__ s) {
    __shared__ double mx[1024], mn[1024];
    double a = 0.0, b = INFINITY;
    for (int j = threadIdx.x; j < K; j += 1024) {
        const double p = pow(mag[j], alpha);
        a = fmax(a, p);
        b = fmin(b, p);
    }
    mx[threadIdx.x] = a;
    mn[threadIdx.x] = b;
    __syncthreads();
    for (int off = 512; off > 0; off >>= 1) {
        if (threadIdx.x < off) {
            mx[threadIdx.x] = fmax(mx[threadIdx.x], mx[threadIdx.x + off]);
            mn[threadIdx.x] = fmin(mn[threadIdx.x], mn[threadIdx.x + off]);
        }
        __syncthreads();
    }
    const double norm = sqrt(mx[0] * mn[0]);
    for (int j = threadIdx.x; j < K; j += 1024) s[j] = (float)(pow(mag[j], alpha) / norm);
}

// ws[n][j] = fp32(w[n][j]) * s[j]
__global__ void __launch_bounds__(kThreads) scale_columns_kernel(const uint16_t *__restrict__ w, long N, int K,
                                                                 const float *__restrict__ s, float *__restrict__ ws) {
    const long n = N * K;
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < n; e += (long)gridDim.x * kThreads)
        ws[e] = __fmul_rn(half_bits_to_float(w[e]), s[e % K]);
}

// D[n][j] = w[n][j] - s16 (q - z) / s_j (fp32), for the objective.
__global__ void __launch_bounds__(kThreads) awq_diff_kernel(const uint16_t *__restrict__ w, long N, int K, int g,
                                                            const uint32_t *__restrict__ qw,
                                                            const uint16_t *__restrict__ sc,
                                                            const uint32_t *__restrict__ qz,
                                                            const float *__restrict__ s, float *__restrict__ D) {
    const long n_el = N * K;
    const int groups = K / g, zwords = (groups + 7) / 8;
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < n_el; e += (long)gridDim.x * kThreads) {
        const long n = e / K;
        const int k = (int)(e % K), j = k / g;
        const int q = (qw[n * (K / 8) + k / 8] >> (4 * (k % 8))) & 0xF;
        const int z = (qz[n * zwords + j / 8] >> (4 * (j % 8))) & 0xF;
        const float deq = half_bits_to_float(sc[n * groups + j]) * (float)(q - z);  // exact
        D[e] = half_bits_to_float(w[e]) - __fdiv_rn(deq, s[k]);
    }
}

// err += 2 * sum over tiles of (X D^T)^2: 64 x 64 tile per CTA of P = X D^T (T x N), squared and
// summed, one fp64 atomic per CTA.
__global__ void __launch_bounds__(kThreads) awq_objective_kernel(const uint16_t *__restrict__ X, int T, int K,
                                                                 const float *__restrict__ D, int N,
                                                                 double *__restrict__ err) {
    __shared__ float As[TK][TB + 4], Bs[TK][TB + 4];
    __shared__ double red[kThreads];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m0 = blockIdx.y * TB, n0 = blockIdx.x * TB;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += TK) {
        for (int e = threadIdx.x; e < TK * TB; e += kThreads) {
            const int kk = e % TK, r = e / TK;
            const int k = k0 + kk;
            As[kk][r] = (m0 + r < T && k < K) ? half_bits_to_float(X[(long)(m0 + r) * K + k]) : 0.0f;
            Bs[kk][r] = (n0 + r < N && k < K) ? D[(long)(n0 + r) * K + k] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[kk][ty * 4 + i];
                b[i] = Bs[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s += (double)acc[i][j] * (double)acc[i][j];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int off = kThreads / 2; off > 0; off >>= 1) {
        if (threadIdx.x < off) red[threadIdx.x] += red[threadIdx.x + off];
        __syncthreads();
    }
    if (threadIdx.x == 0) atomicAdd(err, 2.0 * red[0]);
}

// After alpha a: if err[a] < err[best] (or a == 0), the candidate becomes the result.
__global__ void __launch_bounds__(kThreads) awq_select_kernel(int a, const double *__restrict__ err, int *best,
                                                              long nq, long ns, long nz, int K,
                                                              const uint32_t *__restrict__ cqw,
                                                              const uint16_t *__restrict__ csc,
                                                              const uint32_t *__restrict__ cqz,
                                                              const float *__restrict__ cs, uint32_t *__restrict__ qw,
                                                              uint16_t *__restrict__ sc, uint32_t *__restrict__ qz,
                                                              float *__restrict__ s) {
    const int b = *best;
    if (!(a == 0 || err[a] < err[b])) return;
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < nq; e += (long)gridDim.x * kThreads) qw[e] = cqw[e];
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < ns; e += (long)gridDim.x * kThreads) sc[e] = csc[e];
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < nz; e += (long)gridDim.x * kThreads) qz[e] = cqz[e];
    for (long e = (long)blockIdx.x * kThreads + threadIdx.x; e < K; e += (long)gridDim.x * kThreads) s[e] = cs[e];
}

__global__ void set_best_kernel(int a, const double *__restrict__ err, int *best) {
    if (a == 0 || err[a] < err[*best]) *best = a;
}

#define WQ_TRY(call, what)                                                                                 \
    do {                                                                                                   \
        cudaError_t e_ = (call);                                                                           \
        if (e_ != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: %s failed: %s", who, what, cudaGetErrorString(e_)); \
    } while (0)

}  // namespace
}  // namespace wq

extern "C" size_t wq_gptq_workspace_bytes(int K) {
    if (K <= 0) return 0;
    return sizeof(float) * ((size_t)2 * K * K + (size_t)K * 64 + 64) + 64;
}

extern "C" wq_status wq_hessian(const uint16_t *x, int T, int K, float *H, void *stream) {
    using namespace wq;
    const char *who = "wq_hessian";
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE_PTR(H, "H");
    WQ_REQUIRE(T > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_hessian: sizes must be positive (T=%d K=%d)", T, K);
    // H[i][j] = 2 sum_t X[t][i] X[t][j]: A(m = i, k = t) = X[t][i]
    WQ_TRY((gemm_nt<uint16_t, uint16_t>(K, K, T, x, 1, K, x, 1, K, H, K, 2.0f, 0.0f, false, as_stream(stream))),
           "launch");
    return WQ_OK;
}

extern "C" wq_status wq_gptq_prepare(const float *H, int K, float damp, float *U, void *workspace, void *stream) {
    using namespace wq;
    const char *who = "wq_gptq_prepare";
    WQ_REQUIRE_PTR(H, "H");
    WQ_REQUIRE_PTR(U, "U");
    WQ_REQUIRE_PTR(workspace, "workspace");
    WQ_REQUIRE(K > 0 && K % TB == 0, WQ_ERR_UNSUPPORTED, "wq_gptq_prepare: K (%d) must be a positive multiple of 64", K);
    WQ_REQUIRE(damp >= 0.0f, WQ_ERR_INVALID_ARG, "wq_gptq_prepare: damp must be >= 0");
    cudaStream_t st = as_stream(stream);
    float *A = static_cast<float *>(workspace);                 // [K][K]  P H' P, then its factor
    float *Linv = A + (size_t)K * K;                            // [K][K]
    float *Dinv = Linv + (size_t)K * K;                         // [K/64][64][64]
    float *mean = Dinv + (size_t)K * 64;                        // [1]
    WQ_TRY(cudaMemsetAsync(Linv, 0, sizeof(float) * (size_t)K * K, st), "memset");
    mean_diag_kernel<<<1, kThreads, 0, st>>>(H, K, mean);
    damp_reverse_kernel<<<grid_for((long)K * K), kThreads, 0, st>>>(H, K, damp, mean, A);
    WQ_TRY(cudaGetLastError(), "launch");
    const int nb = K / TB;
    for (int jb = 0; jb < nb; ++jb) {
        const int j0 = jb * TB;
        potrf_diag_kernel<<<1, kThreads, 0, st>>>(A, K, j0, Dinv + (size_t)jb * TB * TB);
        if (jb + 1 < nb) {
            panel_kernel<<<nb - jb - 1, kThreads, 0, st>>>(A, K, j0, Dinv + (size_t)jb * TB * TB);
            const int r0 = j0 + TB, rem = K - r0;
            // trailing lower triangle: A[r][c] -= sum_k L[r][j0 + k] L[c][j0 + k]
            WQ_TRY((gemm_nt<float, float>(rem, rem, TB, A + (size_t)r0 * K + j0, K, 1, A + (size_t)r0 * K + j0, K, 1,
                                          A + (size_t)r0 * K + r0, K, -1.0f, 1.0f, true, st)),
                   "launch");
        }
        WQ_TRY(cudaGetLastError(), "launch");
    }
    for (int ib = 0; ib < nb; ++ib) trinv_row_kernel<<<ib + 1, kThreads, 0, st>>>(A, K, ib, Dinv, Linv);
    reverse_kernel<<<grid_for((long)K * K), kThreads, 0, st>>>(Linv, K, U);
    WQ_TRY(cudaGetLastError(), "launch");
    return WQ_OK;
}

extern "C" wq_status wq_gptq_quantize(const uint16_t *w, int N, int K, int group_size, const float *U, float *work,
                                      uint32_t *qweight, uint16_t *scales, uint32_t *qzeros, void *stream) {
    using namespace wq;
    const char *who = "wq_gptq_quantize";
    WQ_REQUIRE_PTR(w, "w");
    WQ_REQUIRE_PTR(U, "U");
    WQ_REQUIRE_PTR(work, "work");
    WQ_REQUIRE_PTR(qweight, "qweight");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE_PTR(qzeros, "qzeros");
    WQ_REQUIRE(N > 0 && K > 0, WQ_ERR_INVALID_ARG, "wq_gptq_quantize: sizes must be positive (N=%d K=%d)", N, K);
    WQ_REQUIRE(group_size == 128, WQ_ERR_UNSUPPORTED, "wq_gptq_quantize: group_size must be 128 (got %d)", group_size);
    WQ_REQUIRE(K % 128 == 0, WQ_ERR_UNSUPPORTED, "wq_gptq_quantize: K (%d) must be a multiple of 128", K);
    cudaStream_t st = as_stream(stream);
    float *Wf = work;                                // [N][K] compensated weights
    float *E = work + (size_t)N * K;                 // [N][128] scaled errors of the current block
    const int groups = K / 128;
    WQ_TRY(cudaMemsetAsync(qzeros, 0, sizeof(uint32_t) * (size_t)N * ((groups + 7) / 8), st), "memset");
    half_to_float_kernel<<<grid_for((long)N * K), kThreads, 0, st>>>(w, (long)N * K, Wf);
    const size_t smem = sizeof(float) * 128 * 128 + GQ_ROWS * 128;
    WQ_TRY(cudaFuncSetAttribute(gptq_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem),
           "cudaFuncSetAttribute");
    for (int b = 0; b < groups; ++b) {
        gptq_block_kernel<<<(N + GQ_ROWS - 1) / GQ_ROWS, GQ_ROWS * 32, smem, st>>>(Wf, N, K, b, U, E, qweight, scales,
                                                                                 qzeros);
        WQ_TRY(cudaGetLastError(), "launch");
        const int i2 = (b + 1) * 128;
        if (i2 < K)  // W[n][j] -= sum_i E[n][i] U[i1 + i][j] for j >= i2
            WQ_TRY((gemm_nt<float, float>(N, K - i2, 128, E, 128, 1, U + (size_t)(b * 128) * K + i2, 1, K, Wf + i2, K,
                                          -1.0f, 1.0f, false, st)),
                   "launch");
    }
    return WQ_OK;
}

namespace wq {
namespace {
// Byte offsets of the AWQ workspace regions (each 16-byte aligned): W * s (then D), candidate
// codes, scales, zero words, channel scales, channel means; the last value is the total.
struct AwqLayout {
    size_t ws, qw, sc, qz, s, mag, total;
    AwqLayout(int N, int K) {
        auto up = [](size_t v) { return (v + 15) / 16 * 16; };
        const size_t groups = (size_t)K / 128, zwords = (groups + 7) / 8;
        ws = 0;
        qw = up(ws + sizeof(float) * (size_t)N * K);
        sc = up(qw + sizeof(uint32_t) * (size_t)N * (K / 8));
        qz = up(sc + sizeof(uint16_t) * (size_t)N * groups);
        s = up(qz + sizeof(uint32_t) * (size_t)N * zwords);
        mag = up(s + sizeof(float) * (size_t)K);
        total = up(mag + sizeof(double) * (size_t)K);
    }
};
}  // namespace
}  // namespace wq

extern "C" size_t wq_awq_workspace_bytes(int N, int K) {
    if (N <= 0 || K <= 0) return 0;
    return wq::AwqLayout(N, K).total;
}

extern "C" wq_status wq_awq(const uint16_t *w, int N, int K, int group_size, const uint16_t *x, int T,
                            const double *grid, int ngrid, uint32_t *qweight, uint16_t *scales, uint32_t *qzeros,
                            float *s, double *err, int *best, void *workspace, void *stream) {
    using namespace wq;
    const char *who = "wq_awq";
    WQ_REQUIRE_PTR(w, "w");
    WQ_REQUIRE_PTR(x, "x");
    WQ_REQUIRE(grid != nullptr && ngrid > 0 && ngrid <= 64, WQ_ERR_INVALID_ARG, "wq_awq: grid must hold 1..64 values");
    WQ_REQUIRE_PTR(qweight, "qweight");
    WQ_REQUIRE_PTR(scales, "scales");
    WQ_REQUIRE_PTR(qzeros, "qzeros");
    WQ_REQUIRE_PTR(s, "s");
    WQ_REQUIRE_PTR(err, "err");
    WQ_REQUIRE_PTR(best, "best");
    WQ_REQUIRE_PTR(workspace, "workspace");
    WQ_REQUIRE(N > 0 && K > 0 && T > 0, WQ_ERR_INVALID_ARG, "wq_awq: sizes must be positive");
    WQ_REQUIRE(group_size == 128 && K % 128 == 0, WQ_ERR_UNSUPPORTED,
               "wq_awq: group_size must be 128 and K a multiple of 128");
    cudaStream_t st = as_stream(stream);
    const size_t groups = (size_t)K / 128, zwords = (groups + 7) / 8;
    const AwqLayout lay(N, K);
    uint8_t *p = static_cast<uint8_t *>(workspace);
    float *WS = reinterpret_cast<float *>(p + lay.ws);
    uint32_t *cqw = reinterpret_cast<uint32_t *>(p + lay.qw);
    uint16_t *csc = reinterpret_cast<uint16_t *>(p + lay.sc);
    uint32_t *cqz = reinterpret_cast<uint32_t *>(p + lay.qz);
    float *cs = reinterpret_cast<float *>(p + lay.s);
    double *mag = reinterpret_cast<double *>(p + lay.mag);
    WQ_TRY(cudaMemsetAsync(err, 0, sizeof(double) * ngrid, st), "memset");
    channel_mean_abs_kernel<<<(K + kThreads - 1) / kThreads, kThreads, 0, st>>>(x, T, K, mag);
    WQ_TRY(cudaGetLastError(), "launch");
    for (int a = 0; a < ngrid; ++a) {
        awq_scales_kernel<<<1, 1024, 0, st>>>(mag, K, grid[a], cs);
        scale_columns_kernel<<<grid_for((long)N * K), kThreads, 0, st>>>(w, N, K, cs, WS);
        WQ_TRY(cudaGetLastError(), "launch");
        const wq_status q = wq_quantize_group_int4(WS, WQ_F32, N, K, 128, cqw, csc, cqz, stream);
        if (q != WQ_OK) return q;
        awq_diff_kernel<<<grid_for((long)N * K), kThreads, 0, st>>>(w, N, K, 128, cqw, csc, cqz, cs, WS);
        awq_objective_kernel<<<dim3((N + TB - 1) / TB, (T + TB - 1) / TB), kThreads, 0, st>>>(x, T, K, WS, N, err + a);
        awq_select_kernel<<<grid_for((long)N * K / 8), kThreads, 0, st>>>(
            a, err, best, (long)N * (K / 8), (long)N * groups, (long)N * zwords, K, cqw, csc, cqz, cs, qweight, scales,
            qzeros, s);
        set_best_kernel<<<1, 1, 0, st>>>(a, err, best);
        WQ_TRY(cudaGetLastError(), "launch");
    }
    return WQ_OK;
}
