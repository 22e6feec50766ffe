// Library-wide host state: the per-thread error message, the device status
// word written by bounded waits, and the wait limit.
#include <atomic>
#include <cstring>
#include <mutex>

#include <cudaTypedefs.h>

#include "wq_host.h"

namespace {

thread_local char g_last_error[512] = "no error";

// Written by kernels (through a pointer argument) when a bounded wait runs
// out; read and cleared by wq_device_status().
__device__ unsigned int g_device_status;

constexpr uint64_t kDefaultWaitLimit = 2000000000ull;  // ns
std::atomic<uint64_t> g_wait_limit{kDefaultWaitLimit};

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int *g_status_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};

}  // namespace

namespace wq {

wq_status fail(wq_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

unsigned int *device_status_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        fail(WQ_ERR_CUDA, "cudaGetDevice failed");
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_device_status);
        if (e != cudaSuccess) {
            fail(WQ_ERR_CUDA, "cudaGetSymbolAddress(status) failed: %s", cudaGetErrorString(e));
            return nullptr;
        }
        g_status_ptr[dev] = static_cast<unsigned int *>(p);
    }
    return g_status_ptr[dev];
}

uint64_t wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_sms[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        g_sms[dev] = v;
    }
    return g_sms[dev];
}

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, int elem_bytes, const void *base, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                    CUtensorMapSwizzle swizzle) {
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) {
        fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
        return false;
    }
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    (void)elem_bytes;
    CUresult r = g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        fail(WQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
        return false;
    }
    return true;
}

}  // namespace wq

extern "C" const char *wq_last_error(void) { return g_last_error; }

extern "C" void wq_set_wait_limit(uint64_t nanoseconds) {
    g_wait_limit.store(nanoseconds ? nanoseconds : kDefaultWaitLimit, std::memory_order_relaxed);
}

extern "C" wq_status wq_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(wq::as_stream(stream));
    if (e != cudaSuccess) return wq::fail(WQ_ERR_CUDA, "stream synchronize failed: %s", cudaGetErrorString(e));
    unsigned int *p = wq::device_status_word();
    if (!p) return WQ_ERR_CUDA;
    unsigned int v = 0;
    e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return wq::fail(WQ_ERR_CUDA, "reading the status word failed: %s", cudaGetErrorString(e));
    if (v != 0) {
        unsigned int zero = 0;
        e = cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return wq::fail(WQ_ERR_CUDA, "clearing the status word failed: %s", cudaGetErrorString(e));
        return wq::fail(WQ_ERR_TIMEOUT, "a bounded wait ran out in a kernel (site code 0x%x)", v);
    }
    return WQ_OK;
}

// ---------------------------------------------------------------------------
// Self-test of the bounded waits: one thread waits, through the same code the
// pipelined kernels use, on an mbarrier that nothing ever arrives on.  The wait
// must give up after the current limit and record its site code in the status
// word, which the next wq_device_status() reports as WQ_ERR_TIMEOUT.
// ---------------------------------------------------------------------------
#include "sm100.cuh"

namespace wq {
namespace {

constexpr unsigned kSelftestSite = 0x800;

__global__ void selftest_wait_kernel(unsigned int *status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(sm100::smem_u32(&bar), 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const sm100::WaitCtl ctl{&abort_flag, status, limit_ns};
        sm100::wait_parity(sm100::smem_u32(&bar), 0, ctl, kSelftestSite);  // phase 0 never completes
    }
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_selftest_wait_timeout(void *stream) {
    unsigned int *status = wq::device_status_word();
    if (!status) return WQ_ERR_CUDA;
    wq::selftest_wait_kernel<<<1, 32, 0, wq::as_stream(stream)>>>(status, wq::wait_limit());
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return wq::fail(WQ_ERR_CUDA, "wq_selftest_wait_timeout: launch failed: %s", cudaGetErrorString(e));
    return WQ_OK;
}
