// Host-side plumbing shared by the library's translation units: error
// recording, argument checks and the device status word.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>

#include "wq.h"

namespace wq {

// Records a formatted message for wq_last_error() and returns `st`.
wq_status fail(wq_status st, const char *fmt, ...);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Pointer to the library's device status word on the current device
// (nullptr and a recorded message if it cannot be obtained).
unsigned int *device_status_word();

// Current limit for bounded waits in kernels (nanoseconds).
uint64_t wait_limit();

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Maps the result of a launch to a status.
inline wq_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(WQ_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return WQ_OK;
}

int num_sms();

// Encodes a 2-D tiled TMA descriptor over a row-major [outer][inner] array
// (element size `elem_bytes`, row pitch `row_bytes`) with box
// [box_outer][box_inner].  Returns false and records a message on failure.
// Streaming W4A16 matmul for 1..16 activation rows (K % 256 == 0, group size 128); defined in
// gemv_w4a16.cu and shared by wq_gemv_w4a16 and wq_gemm_w4a16.  `who` names the entry point in errors.
wq_status gemv_stream(const uint16_t *x, int B, const uint32_t *qw, const uint16_t *sc, const uint32_t *qz, int N,
                      int K, uint16_t *y, cudaStream_t st, const char *who);

bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, int elem_bytes, const void *base, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle);

}  // namespace wq

#define WQ_REQUIRE(cond, status, ...)                     \
    do {                                                  \
        if (!(cond)) return ::wq::fail((status), __VA_ARGS__); \
    } while (0)

#define WQ_REQUIRE_PTR(p, name)                                                        \
    do {                                                                               \
        if ((p) == nullptr) return ::wq::fail(WQ_ERR_INVALID_ARG, "%s is null", name); \
        if (!::wq::aligned16(p))                                                       \
            return ::wq::fail(WQ_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);   \
    } while (0)
