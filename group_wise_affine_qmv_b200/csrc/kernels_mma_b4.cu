// kernels_mma_b4.cu -- the tensor-core kernels (decode and prefill) instantiated for 4-bit codes (bf16 and f16
// activations, groups 32/64/128).
#include "mma_kernel.cuh"
#include "mma_prefill.cuh"

namespace aq {
namespace mma {
template cudaError_t launch<4>(bool, int, const Params&, int, size_t, cudaStream_t);
template cudaError_t launch_prefill<4>(bool, int, const Params&, int, size_t, cudaStream_t);
}  // namespace mma
}  // namespace aq
