// Device error word. A kernel whose bounded wait gives up sets it (through the
// pointer device_error_word() returns) instead of trapping or hanging; the host
// reads and clears it in bitlinear_get_device_error.
#include <cuda_runtime.h>

#include "kernels.h"

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

}  // namespace bl
