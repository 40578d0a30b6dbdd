// kernels_mma.cu -- tcgen05/TMEM tensor-core kernel (placeholder until it lands).
#include <cuda_runtime.h>

#include "aq_internal.h"

namespace aq {

__device__ int g_device_error = 0;

bool mma_supported(const MmaProblem&, const char** why) {
    if (why) *why = "tensor-core kernel not available";
    return false;
}

cudaError_t launch_mma(const MmaProblem&, cudaStream_t) { return cudaErrorNotSupported; }

cudaError_t read_and_clear_device_error(int* value, cudaStream_t s) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
}

}  // namespace aq
