/*
 * wq.h -- C ABI of the B200 (sm_100a) weight/activation quantization library.
 *
 * The library implements the data-parallel hot path of LLM post-training
 * quantization as described in five web pages on the subject:
 *
 *   [P1] "How quantization works" (AI-infra handbook)
 *   [P2] "Quantization" (engine-room, chapter 15)
 *   [P3] "Quantization from Scratch: Scale, Zero-Point, GPTQ and AWQ"
 *   [P4] "Quantization: Smaller Weights, Same Answers (Mostly)"
 *   [P5] "Quantization Explained: INT8, INT4, GPTQ and AWQ for LLMs"
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is a DEVICE pointer to memory owned by the caller
 *    (allocate it however you like; the library never allocates, frees or
 *    keeps a pointer after the call returns).  Every base address must be
 *    16-byte aligned (WQ_ERR_ALIGNMENT otherwise).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Each call only validates its arguments on the host and
 *    enqueues kernels on `stream`; it never synchronizes the device.
 *  - Matrices are row-major.  Weights are [N out][K in] (nn.Linear layout),
 *    activations are [B or M][K], outputs are [B or M][N].
 *  - fp16 data is passed as uint16_t bit patterns (IEEE 754 binary16).
 *  - Rounding is round-half-to-even everywhere; every division is an IEEE
 *    fp32 division; the library is built without fast-math.
 *  - On a precondition violation the call returns an error status, launches
 *    nothing and records a message readable with wq_last_error() (per host
 *    thread).  Launch failures return WQ_ERR_CUDA.
 *  - Kernels that wait on asynchronous copies or tensor-core operations bound
 *    every wait; a wait that runs out records WQ_ERR_TIMEOUT in a device
 *    status word that wq_device_status() reads.
 *
 * Packed INT4 layout (written by wq_quantize_group_int4, read by the W4A16
 * matmuls):
 *  - qweight uint32 [N][K/8]: element k of row n is nibble (k mod 8), i.e.
 *    bits [4(k mod 8), 4(k mod 8)+4), of word k/8.
 *  - scales  fp16   [N][K/g]: the step of group j = k / g.
 *  - qzeros  uint32 [N][ceil((K/g)/8)]: the zero point of group j is nibble
 *    (j mod 8) of word j/8; unused nibbles of the last word are 0.
 *  Storage is 0.5 + 2.5/g bytes per weight: 0.15625 bit/weight of overhead
 *  at g = 128 ([P3] "Where to put the scales", [P1] exercise 2).
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    WQ_OK = 0,
    WQ_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, inconsistent sizes */
    WQ_ERR_ALIGNMENT = 2,   /* a base address is not 16-byte aligned */
    WQ_ERR_UNSUPPORTED = 3, /* a size outside what the kernels implement */
    WQ_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
    WQ_ERR_TIMEOUT = 5      /* a bounded wait inside a kernel ran out */
} wq_status;

typedef enum { WQ_F32 = 0, WQ_F16 = 1 } wq_dtype;

/*
 * Asymmetric INT4 per-group quantization.
 * Source: [P5] "Uniform Affine Quantization" and "Scale and Zero-Point"
 * (s = (max - min) / (2^b - 1), z = round(-min / s), x_q = round(x/s) + z,
 * clamp to [0, 15]); [P3] "Scale and zero-point" and its round-to-nearest
 * quantize() (a zero scale becomes 1); [P1] "Granularity" (one scale per g
 * consecutive weights of a row) and exercise 2 (fp16 scale, 4-bit zero).
 * Per (row n, group j), in fp32:
 *   lo = min(0, min w), hi = max(0, max w)      (range widened to contain 0)
 *   s  = fp16_rn((hi - lo) / 15); if s == 0 then s = 1
 *   z  = clamp(rne(-lo / s), 0, 15)
 *   q  = clamp(rne(w / s) + z, 0, 15)          (s is the stored fp16 value)
 * w:        [N][K], fp32 (w_dtype WQ_F32) or fp16 bits (WQ_F16).
 * qweight:  out, uint32 [N][K/8];  scales: out, fp16 [N][K/g];
 * qzeros:   out, uint32 [N][ceil(K/g/8)]  (layout above).
 * group_size in {32, 64, 128, 256}, K % group_size == 0.  Inputs must be
 * finite and (hi - lo)/15 must fit fp16 (|w| below ~4.9e5).
 */
wq_status wq_quantize_group_int4(const void *w, wq_dtype w_dtype, int N, int K, int group_size,
                                 uint32_t *qweight, uint16_t *scales, uint32_t *qzeros,
                                 void *stream);

/*
 * Symmetric INT8 per output channel (one fp32 scale per weight row).
 * Source: [P1] "The math of quantization" (s = max|x| / (2^(b-1) - 1),
 * q = clamp(round(x/s), -2^(b-1), 2^(b-1) - 1)), the quant.py listing
 * (absmax clamped at 1e-8), q8_per_row, and SmoothQuant's Ws = W * s in
 * "Activation quantization and outliers".  Per row n, in fp32:
 *   w'_k = smooth ? w_k * smooth[k] : w_k
 *   a = max(max_k |w'_k|, 1e-8);  scales[n] = a / 127
 *   q[n][k] = clamp(rne(w'_k / scales[n]), -128, 127)
 * w: fp16 [N][K];  smooth: nullable fp32 [K];  q: out int8 [N][K];
 * scales: out fp32 [N].  K % 16 == 0.
 */
wq_status wq_quantize_int8_per_channel(const uint16_t *w, int N, int K, const float *smooth,
                                       int8_t *q, float *scales, void *stream);

/*
 * Symmetric INT8 per token (one fp32 scale per activation row, computed at
 * run time).  Source: as above, with SmoothQuant's Xs = X / s ([P1]) and
 * per-token dynamic activation scales ([P4] "Quick Reference").  Per row m:
 *   x'_k = smooth ? x_k / smooth[k] : x_k       (IEEE fp32 division)
 *   a = max(max_k |x'_k|, 1e-8);  scales[m] = a / 127
 *   q[m][k] = clamp(rne(x'_k / scales[m]), -128, 127)
 * x: fp16 [M][K];  smooth: nullable fp32 [K];  q: out int8 [M][K];
 * scales: out fp32 [M].  K % 16 == 0.
 */
wq_status wq_quantize_int8_per_token(const uint16_t *x, int M, int K, const float *smooth,
                                     int8_t *q, float *scales, void *stream);

/*
 * SmoothQuant smoothing factors.  Source: [P1] "Activation quantization and
 * outliers" (s = X.abs().amax(0).clamp(1e-5)^a / W.abs().amax(0).clamp(1e-5)^(1-a))
 * and [P2] "The Mathematics" (s_j = max|X_j|^a / max|W_j|^(1-a)).
 *   ax_j = max(max_m |x[m][j]|, 1e-5),  aw_j = max(max_n |w[n][j]|, 1e-5)
 *   s[j] = alpha == 0.5 ? sqrt(ax_j) / sqrt(aw_j)          (correctly rounded)
 *                       : (float)pow(ax_j, alpha) / (float)pow(aw_j, 1 - alpha)
 *                         (pow in fp64)
 * x: fp16 [M][K] (calibration activations), w: fp16 [N][K];  s: out fp32 [K].
 * workspace: caller-owned scratch of wq_smooth_workspace_bytes(K) bytes,
 * 16-byte aligned; its contents on entry do not matter (the call clears
 * it) and calls that share one workspace must not overlap on the GPU.
 * K % 8 == 0.  0 <= alpha <= 1.
 */
size_t wq_smooth_workspace_bytes(int K);
wq_status wq_smooth(const uint16_t *x, int M, const uint16_t *w, int N, int K, float alpha,
                    float *s, void *workspace, void *stream);

/*
 * wq_smooth without a caller-provided workspace.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory themselves (a plug-in inside a host engine that owns all
 * device memory and offers no allocator, or a latency-critical path that may
 * not call cudaMalloc because of its implicit device synchronization).
 * Same arguments, result and restrictions as wq_smooth, plus K <=
 * WQ_SMOOTH_NOALLOC_MAX_K (larger K returns WQ_ERR_UNSUPPORTED and launches
 * nothing).
 * The workspace is a fixed array of 2 * WQ_SMOOTH_NOALLOC_MAX_K + 256 words
 * (513 KiB) held in the device memory of every GPU that loads the library,
 * until the process exits.  The call allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.  The first call on a device (made
 * while that device is current) looks up the array's device address with
 * cudaGetSymbolAddress and caches it; make that first call before any stream
 * capture.  Under CUDA's lazy module loading (the default) the first use of
 * the library on a device -- this look-up or the first launch of any entry
 * point -- loads the library's device code on that device, which allocates
 * device memory for the code and the array and may synchronize: make one
 * ordinary call during set-up, or load modules eagerly
 * (CUDA_MODULE_LOADING=EAGER), if later calls must not do either.  All
 * calls on a device share the one array, which keeps the last
 * call's contents (each call clears what must start at zero), so calls that
 * overlap on the GPU (concurrent streams, several host threads) race and
 * give wrong results: order them on one stream or with events.
 */
#define WQ_SMOOTH_NOALLOC_MAX_K 65536
wq_status wq_smooth_noalloc(const uint16_t *x, int M, const uint16_t *w, int N, int K, float alpha,
                            float *s, void *stream);

/*
 * Fused dequantize + GEMV, W4A16, for decode batches B = 1..8.  Source: [P1]
 * "Inference view" (weights unpacked in registers, multiplied by their
 * scales), [P3] "Scale and zero-point" (w^ = (q - z) s), [P5] "Why It Is
 * Faster" (decode streams the weights).
 *   y[b][n] = fp16_rn( sum_k s[n][k/g] * (q[n][k] - z[n][k/g]) * x[b][k] )
 * accumulated in fp32 (order unspecified).  Every product s * (q - z) * x
 * enters the accumulation exactly, for any finite fp16 x, with one
 * exception: with group size 128 and K % 256 == 0 the kernel pre-scales half
 * of a group's x by 2^-4 (or, when that would drop bits of some |x| < 2^-10,
 * the other half by 16); if one activation row's group holds both a value
 * of magnitude >= 4096 in the second half and such a small value in the
 * first, the small values keep the 2^-4 pre-scaling and each product with
 * them is off by at most 2^-21 * s * q.
 * x: fp16 [B][K];  qweight/scales/qzeros: the packed layout above;
 * y: out fp16 [B][N].  group_size in {32, 64, 128, 256}; K % group_size == 0;
 * K % 32 == 0.
 */
wq_status wq_gemv_w4a16(const uint16_t *x, int B, const uint32_t *qweight, const uint16_t *scales,
                        const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y,
                        void *stream);

/*
 * W4A16 GEMM for M >= 9 rows of activations ([P1] "Inference view"), same
 * arithmetic and layouts as wq_gemv_w4a16, for every group size the
 * quantizer writes.  Group size 128: M <= 32 with K % 256 == 0 runs the
 * streaming kernel of wq_gemv_w4a16 in passes of 16 rows (codes dequantized
 * in registers, exact products, two 8-row batch tiles per weight fragment).
 * Other group sizes below 16 rows run wq_gemv_w4a16 in passes of 8 rows.
 * Everything else runs on the tensor cores: tiles of packed weights are
 * dequantized into shared memory (each dequantized weight rounded to fp16)
 * and fed to tcgen05 MMAs with fp32 accumulation in tensor memory
 * (activation tiles of up to 128 rows; larger M is several tiles).
 * M >= 16, or 9 <= M < 16 with K % 256 == 0 or group_size != 128;
 * group_size in {32, 64, 128, 256}, K % group_size == 0; K % 128 == 0.
 */
wq_status wq_gemm_w4a16(const uint16_t *x, int M, const uint32_t *qweight, const uint16_t *scales,
                        const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y,
                        void *stream);

/*
 * bf16 activations (the variants bf16 models call): same packed weights,
 * arithmetic and arguments as wq_gemv_w4a16 / wq_gemm_w4a16, with x and y
 * bf16 bit patterns instead of fp16.  The GEMV (B = 1..8, any group size)
 * multiplies the exact q - z by the exactly converted x in fp32 and applies
 * each group's scale in fp32; the GEMM's tensor-core path rounds each
 * dequantized weight s (q - z) to bf16 (tcgen05 kind::f16 with bf16
 * operands).  y is rounded to bf16 once, so the error is within
 * 2^-8 * sum_k |w^ x| (bf16 output and, for the GEMM, bf16 weights) on top
 * of the fp32 accumulation.  Preconditions as for the fp16 functions (the
 * GEMM below 16 rows runs the bf16 GEMV in passes of 8 rows).
 */
wq_status wq_gemv_w4a16_bf16(const uint16_t *x, int B, const uint32_t *qweight, const uint16_t *scales,
                             const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y, void *stream);
wq_status wq_gemm_w4a16_bf16(const uint16_t *x, int M, const uint32_t *qweight, const uint16_t *scales,
                             const uint32_t *qzeros, int N, int K, int group_size, uint16_t *y, void *stream);

/*
 * W8A8 INT8 GEMM on the tensor cores with a fused dequantization epilogue.
 * Source: [P4] "How does quantized matrix multiplication actually run on the
 * GPU?" (int8 operands, exact 32-bit accumulation; symmetric scales make the
 * zero-point terms vanish) and [P1] "Mainstream schemes" (W8A8 INT8).
 *   acc[m][n] = sum_k xq[m][k] * wq[n][k]      (int32, exact)
 *   y[m][n]   = fp16_rn( (float)acc * sx[m] * sw[n] )     (fp32 products)
 * xq: int8 [M][K], sx: fp32 [M], wq: int8 [N][K], sw: fp32 [N];
 * y: out fp16 [M][N];  acc_out: nullable, out int32 [M][N] (raw accumulators).
 * K % 16 == 0, K <= 131056 (so |acc| <= 128 * 128 * K < 2^31 for any
 * int8 codes).
 */
wq_status wq_gemm_w8a8(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                       int M, int N, int K, uint16_t *y, int32_t *acc_out, void *stream);

/*
 * W8A16 GEMV (INT8 per-channel weights, fp16 activations), B = 1..8.
 * Source: [P1] "Mainstream schemes" (W8A16) and the per-channel INT8 above.
 *   y[b][n] = fp16_rn( sw[n] * sum_k q[n][k] * x[b][k] )   (fp32 accumulation)
 * x: fp16 [B][K];  wq: int8 [N][K];  sw: fp32 [N];  y: out fp16 [B][N].
 * K % 16 == 0.
 */
wq_status wq_gemv_w8a16(const uint16_t *x, int B, const int8_t *wq, const float *sw, int N, int K,
                        uint16_t *y, void *stream);

/*
 * FP8 E4M3 quantization, per row or per tensor.  Source: [P1] quant.py
 * fake_quant_fp8 (scale = max|w| / 448, then the cast to E4M3) and
 * "Mainstream schemes at a glance" (FP8 W8A8, dynamic or static scales);
 * [P3] "Formats" and [P4] "What about FP8, MXFP4, NVFP4 and GGUF?" (E4M3:
 * 4 exponent bits, 3 mantissa bits, up to +-448).  E4M3 here is the variant
 * without infinities (exponent bias 7; 0x7F/0xFF are NaN).
 *   a = max(max |x| over the row (per_row) or the tensor, 1e-8)
 *   s = a / 448                                    (fp32 IEEE division)
 *   q = e4m3_rn(x / s)       (fp32 IEEE division, then round to nearest even)
 * x: fp16 [R][K];  q: out E4M3 codes [R][K];  scales: out fp32, [R] when
 * per_row != 0 (per output channel for weights, per token for activations),
 * else [1] (one scale for the whole tensor; the call uses it as its
 * reduction word first).  K % 16 == 0.  Inputs must be finite.
 */
wq_status wq_quantize_fp8_e4m3(const uint16_t *x, int R, int K, int per_row, uint8_t *q, float *scales,
                               void *stream);

/*
 * FP8 E4M3 W8A8 GEMM on the tensor cores (tcgen05 kind::f8f6f4, fp32
 * accumulation) with the fused dequantization epilogue.  Source: [P1]
 * "Mainstream schemes at a glance" (FP8 weights and activations on FP8
 * tensor cores), [P4] FP8 section.
 *   acc[m][n] = sum_k e4m3(xq[m][k]) * e4m3(wq[n][k])    (fp32, order unspecified)
 *   y[m][n]   = fp16_rn( acc * sx[m or 0] * sw[n or 0] )   (fp32 products)
 * xq: E4M3 [M][K], wq: E4M3 [N][K];  sx: fp32 [M] if sx_per_row else [1];
 * sw: fp32 [N] if sw_per_row else [1];  y: out fp16 [M][N];  acc_out:
 * nullable, out fp32 [M][N] (raw accumulators).  K % 16 == 0.
 */
wq_status wq_gemm_fp8(const uint8_t *xq, const float *sx, int sx_per_row, const uint8_t *wq, const float *sw,
                      int sw_per_row, int M, int N, int K, uint16_t *y, float *acc_out, void *stream);

/*
 * LLM.int8() mixed-precision decomposition.  Source: [P2] "The Breakthrough"
 * and "The Mathematics" (C ~= S_out (.) (X_q W_q) + X_16 W_16: INT8 with a
 * scale per row of X and per column of the product, the outlier feature
 * dimensions removed from the integer path and multiplied in 16-bit); [P4]
 * "How do LLM-specific quantization schemes protect against outliers?".
 * The weights are stored once, as per-output-channel INT8 (codes wq, scales
 * sw from wq_quantize_int8_per_channel without smoothing), and the 16-bit
 * outlier slice of W is their dequantized columns.  The sequence is:
 *   wq_outlier_columns  -> idx, count, keep
 *   wq_quantize_int8_per_channel(x, keep)  -> X_q, s_x  (the carved columns
 *       of x multiplied by 0: per-token INT8 over the other columns)
 *   wq_gather_outliers  -> X_16, W_16
 *   wq_gemm_w8a8_outliers -> y
 *
 * wq_outlier_columns: an outlier column is a column j of x [M][K] (fp16) with
 * max_m |x[m][j]| >= threshold.  idx (int32 [cap]) receives the first
 * min(total, cap) of them in increasing order (the ones carved out) and 0 in
 * its remaining entries, *count
 * (int32, device) the total that qualify, keep (fp32 [K]) 0 for the carved
 * columns and 1 elsewhere (keep also serves as the call's reduction buffer).
 * K % 8 == 0; 1 <= cap <= K; threshold > 0.
 */
wq_status wq_outlier_columns(const uint16_t *x, int M, int K, float threshold, int cap, int32_t *idx,
                             int32_t *count, float *keep, void *stream);

/*
 * wq_gather_outliers: X_16 (fp16 [M][cap]) = x[:, idx[i]] and W_16 (fp16
 * [N][cap]) = (fp16) wq[:, idx[i]] (exact: |code| <= 128) for i <
 * min(*count, cap); zero for the other i.  idx/count as written by
 * wq_outlier_columns.  cap % 16 == 0, 16 <= cap <= 256.
 */
wq_status wq_gather_outliers(const uint16_t *x, int M, int K, const int8_t *wq, int N, const int32_t *idx,
                             const int32_t *count, int cap, uint16_t *x16, uint16_t *w16, void *stream);

/*
 * wq_gemm_w8a8_outliers: the INT8 tensor-core GEMM of wq_gemm_w8a8 whose
 * epilogue adds the 16-bit product of the carved columns:
 *   y[m][n] = fp16_rn( (acc[m][n] * sx[m] + sum_i x16[m][i] w16[n][i]) * sw[n] )
 * acc as in wq_gemm_w8a8 (int32, exact), the 16-bit sum in fp32 (order
 * unspecified).  xq: int8 [M][K] (carved columns zero), sx: fp32 [M],
 * wq: int8 [N][K], sw: fp32 [N], x16: fp16 [M][cap], w16: fp16 [N][cap],
 * y: out fp16 [M][N].  K % 16 == 0, K <= 131056; cap % 16 == 0,
 * 16 <= cap <= 256.
 */
wq_status wq_gemm_w8a8_outliers(const int8_t *xq, const float *sx, const int8_t *wq, const float *sw,
                                const uint16_t *x16, const uint16_t *w16, int cap, int M, int N, int K, uint16_t *y,
                                void *stream);

/*
 * Block-scaled FP4 quantization.  Source: [P4] "What about FP8, MXFP4, NVFP4
 * and GGUF?" (MXFP4: blocks of 32 four-bit floats (E2M1) sharing one 8-bit
 * power-of-two scale; NVFP4: blocks of 16 with an FP8 scale per block plus
 * one FP32 scale per tensor); [P3] "Formats"; [P1] "Mainstream schemes" (FP4
 * on Blackwell).  E2M1 values: 0, 0.5, 1, 1.5, 2, 3, 4, 6 and negatives;
 * codes are packed two per byte along K, element 2i in the low nibble.
 * MXFP4 (the microscaling rule): per block of 32 consecutive values of a row,
 *   e = floor(log2 max|v|) - 2,  scale byte = e + 127 (E8M0; 0 for an all-zero
 *   block),  q = e2m1_rn(v * 2^-e)  (exact scaling, round to nearest even,
 *   saturating at +-6).
 * NVFP4: S = max(max|v| over the tensor, 1e-8) / 2688  (6 * 448, fp32 division;
 *   written to *tensor_scale); per block of 16, scale byte
 *   b = e4m3_rn((max|v| / 6) / S) (two fp32 divisions), d = e4m3(b) * S,
 *   q = e2m1_rn(v / d) (fp32 IEEE division; all zero when b == 0).
 * x: fp16 [R][K];  q: out [R][K/2];  tensor_scale: out fp32 [1] (also the
 * call's reduction word);  scales: out, wq_fp4_scale_bytes(R, K, nvfp4) bytes
 * in the tensor-core atom layout: with F = K/32 (MX) or K/16 (NV) factors per
 * row, rows in blocks of 128 and factors in groups of 4, one 512-byte atom per
 * (row block, group), atoms ordered row block major; factor f of row r is
 *   byte ((r/128) * ceil(F/4) + f/4) * 512 + 16 (r % 32) + 4 ((r/32) % 4) + f % 4.
 * Bytes of rows past R (and of factors past F) are not written.
 * K % 32 == 0 (MX) or K % 16 == 0 (NV).  Inputs must be finite.
 */
wq_status wq_quantize_mxfp4(const uint16_t *x, int R, int K, uint8_t *q, uint8_t *scales, void *stream);
wq_status wq_quantize_nvfp4(const uint16_t *x, int R, int K, uint8_t *q, uint8_t *scales, float *tensor_scale,
                            void *stream);

/* Size in bytes of the scale-factor buffer of an R x K FP4 tensor (0 for non-positive sizes). */
size_t wq_fp4_scale_bytes(int R, int K, int nvfp4);

/*
 * Block-scaled FP4 GEMM on the tensor cores (tcgen05 kind::mxf4 for MXFP4,
 * kind::mxf4nvf4 for NVFP4; fp32 accumulation).  Source: as above; the
 * hardware block scale is what group-wise quantization does in software
 * ([P3] "Formats").
 *   y[m][n] = fp16_rn( ta * tb * sum_k e2m1(a[m][k]) sa(m, k/bs) e2m1(b[n][k]) sb(n, k/bs) )
 * nvfp4 = 0: MXFP4 (bs = 32, E8M0 scales, ta = tb = 1, both may be NULL);
 * nvfp4 = 1: NVFP4 (bs = 16, E4M3 scales, ta/tb: device fp32 [1] tensor
 * scales).  a: [M][K/2], b: [N][K/2] packed codes; sfa, sfb: the scale
 * factors of a and b in the atom layout above (wq_fp4_scale_bytes(M or N, K,
 * nvfp4) bytes each);  y: out fp16 [M][N];  acc_out: nullable, out fp32
 * [M][N] (the block-scaled sums before ta * tb).  K % 256 == 0.
 */
wq_status wq_gemm_fp4(int nvfp4, const uint8_t *a, const uint8_t *sfa, const float *ta, const uint8_t *b,
                      const uint8_t *sfb, const float *tb, int M, int N, int K, uint16_t *y, float *acc_out,
                      void *stream);

/*
 * Calibration-driven INT4 (GPTQ and AWQ), producing the stored INT4 format of
 * wq_quantize_group_int4 (group size 128).  Source: [P3] "GPTQ: rounding with
 * error compensation", "AWQ: protect the channels that matter" and the
 * gptq() / awq() routines of "Measured on two real layers"; [P2] "The
 * Mathematics" (H = 2 X^T X).  A group's grid is the stored-format rule of
 * wq_quantize_group_int4 applied to the fp32 values it quantizes.  These are
 * fp32 GPU computations: their codes follow the fp64 reference closely but
 * not bit for bit (compensation rounds differently), except where no
 * compensation happens (U = identity gives round-to-nearest exactly).
 *
 * wq_hessian: H = 2 X^T X, fp32 [K][K], from fp16 calibration activations
 * x [T][K].
 *
 * wq_gptq_prepare: U = upper Cholesky factor of (H + damp * mean(diag H) I)^-1,
 * fp32 [K][K] (U^T U = that inverse), via the Cholesky factor of the
 * index-reversed matrix and its inverse.  K % 64 == 0; damp >= 0 (the pages
 * use 0.01); H must be symmetric and H + damping positive definite.
 * workspace: wq_gptq_workspace_bytes(K) bytes, 16-byte aligned.
 *
 * wq_gptq_quantize: GPTQ of fp16 w [N][K] given U: one column at a time in
 * blocks of 128 columns (one group), each block's grid from its compensated
 * weights, each column's scaled error e = (w - (q - z) s) / U[i][i] pushed
 * onto the block's later columns and, after the block, onto the columns after
 * it.  work: fp32 scratch of N * K + N * 128 floats.  group_size == 128,
 * K % 128 == 0.
 *
 * wq_awq: AWQ's scaling search.  mag_j = mean_t |x[t][j]|; for each alpha of
 * the host array grid[0..ngrid): s_j = fp32(mag_j^alpha / sqrt(max * min))
 * (fp64 powers), codes = round-to-nearest of the fp32 products w[n][j] * s_j,
 * D = w - dequant / s, err[a] = 2 ||x D^T||^2 (the calibration objective
 * sum_n D H D^T); the first alpha with the smallest err wins.  Outputs (device):
 * qweight/scales/qzeros of W diag(s) for the winner (serve it with x / s),
 * s fp32 [K], err fp64 [ngrid], best int [1].  workspace:
 * wq_awq_workspace_bytes(N, K) bytes.  group_size == 128, K % 128 == 0,
 * 1 <= ngrid <= 64.
 */
wq_status wq_hessian(const uint16_t *x, int T, int K, float *H, void *stream);
size_t wq_gptq_workspace_bytes(int K);
wq_status wq_gptq_prepare(const float *H, int K, float damp, float *U, void *workspace, void *stream);
wq_status wq_gptq_quantize(const uint16_t *w, int N, int K, int group_size, const float *U, float *work,
                           uint32_t *qweight, uint16_t *scales, uint32_t *qzeros, void *stream);
size_t wq_awq_workspace_bytes(int N, int K);
wq_status wq_awq(const uint16_t *w, int N, int K, int group_size, const uint16_t *x, int T, const double *grid,
                 int ngrid, uint32_t *qweight, uint16_t *scales, uint32_t *qzeros, float *s, double *err, int *best,
                 void *workspace, void *stream);

/* Message describing the last error status returned on this host thread. */
const char *wq_last_error(void);

/*
 * Synchronizes `stream`, then reads and clears the library's device status
 * word: WQ_OK, or WQ_ERR_TIMEOUT if a bounded wait ran out in a kernel since
 * the last call (or WQ_ERR_CUDA if synchronization failed).
 */
wq_status wq_device_status(void *stream);

/*
 * Wall-clock limit, in nanoseconds, of each bounded wait inside the
 * tensor-core kernels (default 2e9, two seconds; 0 restores the default).
 * Applies to launches made after the call.  Small values exist so that tests
 * can make a wait run out on purpose; the kernel then stops, drains its own
 * in-flight copies and tensor-core operations, releases its tensor memory and
 * records WQ_ERR_TIMEOUT for wq_device_status().
 */
void wq_set_wait_limit(uint64_t nanoseconds);

/*
 * Self-test of the bounded waits (failure detection; the pages have no
 * counterpart): launches one thread that waits, through the same bounded-wait
 * code as the pipelined kernels, on a barrier that nothing completes.  After
 * the current wait limit (wq_set_wait_limit) it gives up, so the next
 * wq_device_status() returns WQ_ERR_TIMEOUT.  Set a short limit first: with
 * the default the wait lasts two seconds.
 */
wq_status wq_selftest_wait_timeout(void *stream);

#ifdef __cplusplus
}
#endif
#endif /* WQ_H */
