// Device error word. A kernel whose bounded wait gives up sets it (through the
// pointer device_error_word() returns) instead of trapping or hanging; the host
// reads and clears it in bitlinear_get_device_error.
#include <bitlinear.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace bl {

__device__ unsigned int g_device_error_word = 0;

cudaError_t device_error_word(unsigned int** ptr) {
    return cudaGetSymbolAddress(reinterpret_cast<void**>(ptr), g_device_error_word);
}

cudaError_t read_and_clear_device_error(unsigned int* value) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_device_error_word, &zero, sizeof(unsigned int));
}

namespace {

// One thread waits, with the same bounded wait the GEMV and GEMM kernels use,
// on an mbarrier that nothing arrives on; after `limit_ns` it records the
// timeout in the error word and returns.
__global__ void timeout_probe_kernel(unsigned int* err, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    const uint32_t b = tc::smem_u32(&bar);
    tc::mbar_init(b, 1);
    tc::fence_mbar_init();
    if (!tc::mbar_wait(b, 0, limit_ns)) atomicOr(err, 1u);
}

}  // namespace

}  // namespace bl

#define BL_API extern "C" __attribute__((visibility("default")))

BL_API bl_status bitlinear_selftest_timeout(int64_t limit_us, bl_stream_t stream) {
    if (limit_us < 1 || limit_us > 2000000) return BL_ERR_SHAPE;
    int dev = -1, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
        cudaGetLastError();
        return BL_ERR_UNSUPPORTED;
    }
    unsigned int* err = nullptr;
    if (bl::device_error_word(&err) != cudaSuccess) return BL_ERR_CUDA;
    bl::timeout_probe_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(err, (unsigned long long)limit_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}
