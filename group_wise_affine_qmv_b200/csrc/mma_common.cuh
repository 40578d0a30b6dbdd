// mma_common.cuh -- definitions shared by the host side of the tensor-core kernel
// (kernels_mma.cu) and its device code (mma_kernel.cuh, instantiated once per bit width in
// kernels_mma_b{2,4,6,8}.cu so that the four compile in parallel).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace aq {
namespace mma {

// ---- warp roles ----
constexpr int EXP_WARPS = 8;                              // warps 2..9: code expanders
constexpr int FOLD_WARPS = 8;                             // warps 10..17: s*D + b*X folds
constexpr int FOLD_THREADS = 32 * FOLD_WARPS;
constexpr int XPROD_WARP = 2 + EXP_WARPS + FOLD_WARPS;    // warp 18: x producer
constexpr int THREADS = 32 * (XPROD_WARP + 1);            // 608

// ---- tiling ----
constexpr int NT = 32;                    // tokens per tile (the MMA's N)
constexpr int KB = 64;                    // codes per MMA sub-step (4 tcgen05.mma of K = 16)
constexpr int SCW = 32;                   // groups per scale/bias chunk
constexpr int SCP = SCW + 2;              // padded row pitch (halves) of a chunk in shared memory
constexpr int MAX_STAGES = 12;            // W ring
constexpr int MAX_XST = 4;                // streamed x ring
constexpr int MAX_EXPERTS = 1024;
constexpr int XTAB_MAX_BYTES = 32 * 1024; // sums of x per group and token of one token tile
constexpr int XV = 2;                     // 16-byte loads in flight per thread while summing x
constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait on a copy or on the tensor core
// waits on another role get twice as long, so that a stall is reported by the wait on the copy
// or MMA that did not complete rather than by the roles queued behind it
constexpr uint64_t WAIT_ROLE_NS = 2 * WAIT_NS;
constexpr int ERR_TIMEOUT = 1;

// W stage geometry.  A stage is 128 rows x WSC codes: at most 4 groups (so that two A blocks
// of WSC/2 columns and two sets of 4 group accumulators of NT columns fit the 512 tensor-memory
// columns) and a row of at most one 128-byte swizzle atom (96 bytes for 6-bit codes).
__host__ __device__ constexpr int stage_codes(int bits, int group) {
    return bits == 6 ? 128 : (1024 / bits < 256 ? (1024 / bits < 4 * group ? 1024 / bits : 4 * group)
                                                : (256 < 4 * group ? 256 : 4 * group));
}
__host__ __device__ constexpr int stage_rowb(int bits, int group) { return stage_codes(bits, group) * bits / 8; }
// XOR mask of the TMA swizzle on byte-address bits [4..6] from bits [7..9]
__host__ __device__ constexpr uint32_t stage_swz(int rowb) {
    return rowb == 128 ? 7u : rowb == 64 ? 3u : rowb == 32 ? 1u : 0u;
}

struct Params {
    CUtensorMap tx;  // x: 4D {K, rows, nb1, nb0} u16, box {64, NT, 1, 1}, 128-byte swizzle
    CUtensorMap tw;  // W: 2D {K*bits/32, rows} u32, box {rowb/4, 128}, swizzle by row bytes
    CUtensorMap ty;  // y (ytma): 4D {N, M, nb1, nb0} u16, box {128, NT, 1, 1}, no swizzle
    const void* x;
    void* y;
    const uint16_t* scales;
    const uint16_t* biases;
    int64_t M, N, K;
    int64_t x_row, y_row;
    int64_t xb[2], yb[2];
    int64_t nb1;
    int n_wtiles, n_ttiles, nbatch;
    int kg;              // groups per row = K / group
    int ydt;             // DT of y
    int n_wstages;       // W stages per tile
    int stages;          // W ring depth
    int xres;            // 1: the CTA's single x tile stays resident in shared memory
    int xst;             // streamed x ring depth (x stages of SUB boxes) when not resident
    uint32_t tmem_cols;
    uint32_t idesc;
    const int64_t* offsets;  // grouped mode when non-null
    int n_experts;
    int ksplit;                  // CTAs per cluster splitting each tile's K (1: no split)
    int ytma;                    // 1: each tile's y goes out as one TMA store of a shared-memory tile
    int* err;                    // device error word (set on a timed-out wait)
};

// W stages [w0, w1) of the tile handled by rank `rank` of `cs` CTAs splitting K.  Ranges
// start at an even group (4-byte scale/bias copies), so with one group per stage they move
// in units of two stages.
__host__ __device__ inline void split_range(int nws, int gps, int cs, int rank, int* w0, int* w1) {
    const int u = gps == 1 ? 2 : 1;
    const int nu = (nws + u - 1) / u;
    const int a = u * (nu * rank / cs), b = u * (nu * (rank + 1) / cs);
    *w0 = a < nws ? a : nws;
    *w1 = b < nws ? b : nws;
}
// the most W stages any rank gets
__host__ __device__ inline int split_max_stages(int nws, int gps, int cs) {
    const int u = gps == 1 ? 2 : 1;
    const int nu = (nws + u - 1) / u;
    const int m = u * ((nu + cs - 1) / cs);
    return m < nws ? m : nws;
}
constexpr int RED_BYTES = FOLD_THREADS * (NT / 2) * 4;  // one CTA's partial y tile (fp32)
constexpr int YSTG_BYTES = NT * 128 * 2;                 // a tile of y (16-bit) staged for its TMA store

// shared memory besides the x buffer, the W ring and the sum-of-x table
__host__ __device__ constexpr size_t smem_fixed_bytes() {
    return 2 * 2 * 128 * SCP * 2                                  // scale/bias chunk slots
           + (2 * MAX_STAGES + 2 * MAX_XST + 2 * 4 + 5) * 8 + 8  // mbarriers, TMEM base, abort flag
           + (MAX_EXPERTS + 1) * 4                               // grouped tile prefix sums
           + 2 * 1024;                                           // alignment
}

// ---- prefill kernel (mma_prefill.cuh): tiles of 128 W rows x 128 tokens, one group per stage
namespace pf {
constexpr int NTP = 128;                                  // tokens per tile
constexpr int P_EXP = 4;                                  // warps 2..5: code expanders
constexpr int P_FOLD = 8;                                 // warps 6..13: folds
constexpr int P_FOLD_THREADS = 32 * P_FOLD;
constexpr int P_XPROD = 2 + P_EXP + P_FOLD;               // warp 14: x producer
constexpr int P_THREADS = 32 * (P_XPROD + 1);             // 480
constexpr int P_MAX_STAGES = 12;
constexpr int P_YSTG_BYTES = NTP * 128 * 2;               // a tile of y (16-bit) staged for its TMA store
constexpr int P_MAX_XST = 4;
// scale/bias slots, the two sums-of-x rows, mbarriers, TMEM base, abort flag, alignment
__host__ __device__ constexpr size_t p_fixed_bytes() {
    return 2 * 2 * 128 * SCP * 2 + 2 * NTP * 4 + (2 * P_MAX_STAGES + 2 * P_MAX_XST + 2 * 6 + 2) * 8 + 8 + 2 * 1024;
}
}  // namespace pf

// defined in mma_kernel.cuh / mma_prefill.cuh, instantiated in kernels_mma_b<BITS>.cu
template <int BITS>
cudaError_t launch_prefill(bool bf16, int group, const Params& prm, int grid, size_t smem, cudaStream_t stream);
extern template cudaError_t launch_prefill<2>(bool, int, const Params&, int, size_t, cudaStream_t);
extern template cudaError_t launch_prefill<4>(bool, int, const Params&, int, size_t, cudaStream_t);
extern template cudaError_t launch_prefill<6>(bool, int, const Params&, int, size_t, cudaStream_t);
extern template cudaError_t launch_prefill<8>(bool, int, const Params&, int, size_t, cudaStream_t);

template <int BITS>
cudaError_t launch(bool bf16, int group, const Params& prm, int grid, size_t smem, cudaStream_t stream);
extern template cudaError_t launch<2>(bool, int, const Params&, int, size_t, cudaStream_t);
extern template cudaError_t launch<4>(bool, int, const Params&, int, size_t, cudaStream_t);
extern template cudaError_t launch<6>(bool, int, const Params&, int, size_t, cudaStream_t);
extern template cudaError_t launch<8>(bool, int, const Params&, int, size_t, cudaStream_t);

}  // namespace mma
}  // namespace aq
