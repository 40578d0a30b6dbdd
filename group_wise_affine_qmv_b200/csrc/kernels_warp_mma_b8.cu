// kernels_warp_mma_b8.cu -- the warp-level tensor-core kernel instantiated for 8-bit codes (bf16 and
// f16 activations, every supported group, 8/16-token tiles).
#include "warp_mma_kernel.cuh"

namespace aq {
namespace wm {
template cudaError_t launch<8>(bool, int, int, const WParams&, dim3, int, size_t, cudaStream_t);
}  // namespace wm
}  // namespace aq
