// W4A16 tensor-core GEMM (placeholder until the tcgen05 kernel lands).
#include "wq_host.h"

extern "C" wq_status wq_gemm_w4a16(const uint16_t *, int, const uint32_t *, const uint16_t *, const uint32_t *, int,
                                   int, int, uint16_t *, void *) {
    return wq::fail(WQ_ERR_UNSUPPORTED, "wq_gemm_w4a16: not built yet");
}
