// qga_abi.cu -- status codes, error text, version and the per-device caches
// behind every entry point of libqga.so.

#include <cuda_runtime.h>

#include <atomic>

#include "qga_common.cuh"

namespace qga {

namespace {
thread_local int g_last_cuda_error = 0;
std::atomic<int> g_sm_count[64];
} // namespace

int cuda_status(cudaError_t err)
{
    if (err == cudaSuccess)
        return QGA_OK;
    g_last_cuda_error = (int)err;
    return QGA_ERR_CUDA;
}

int sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        dev = 0;
    int c = g_sm_count[dev].load(std::memory_order_relaxed);
    if (c > 0)
        return c;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c < 1)
        c = 1;
    g_sm_count[dev].store(c, std::memory_order_relaxed);
    return c;
}

} // namespace qga

extern "C" const char *qga_strerror(int status)
{
    switch (status) {
    case QGA_OK:
        return "ok";
    case QGA_ERR_INVALID_ARG:
        return "invalid argument (null or misaligned pointer, negative size, non-finite threshold, "
               "worker count out of range)";
    case QGA_ERR_UNSUPPORTED:
        return "unsupported request (e.g. a bit width other than 2, 4 or 8)";
    case QGA_ERR_CUDA:
        return "CUDA runtime error (see qga_last_cuda_error)";
    default:
        return "unknown status";
    }
}

extern "C" int qga_last_cuda_error(void) { return qga::g_last_cuda_error; }

extern "C" int qga_version(void) { return 10000; }
