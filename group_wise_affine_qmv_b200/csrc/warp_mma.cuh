// warp_mma.cuh -- definitions shared by the host side of the warp-level tensor-core kernel
// (kernels_warp_mma.cu) and its device code (warp_mma_kernel.cuh, instantiated once per bit
// width in kernels_warp_mma_b{2,4,8}.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace aq {
namespace wm {

constexpr int ROWS = 32;             // W rows per warp: two m16 tiles of mma.sync
constexpr int MAX_WARPS = 8;         // warps per CTA
constexpr int MAX_CLUSTER = 4;       // CTAs of a cluster splitting K
constexpr int MAX_TOKENS = 32;       // rows of x (in total) the kernel is chosen for
constexpr int TILE_TOKENS = 16;      // x rows per token tile: up to two n8 tiles (two CTAs fit an SM)
constexpr int RING_BYTES = 8192;     // most bytes of a warp's ring of W sub-blocks in shared memory
constexpr int RED_PITCH = ROWS + 4;  // floats per token of a warp's partial y tile (bank spread)
constexpr int MAX_XTAB_BYTES = 48 * 1024;
constexpr uint64_t WAIT_NS = 2000000000ull;   // budget of every bounded wait (2 s)

constexpr int MAX_SEGS = 3;          // W matrices sharing one x in one launch

// One W matrix of a launch, with its scales, biases and output.  A launch's W rows form one
// "logical" row space cut into blocks of ROWS rows (one block per warp): segment s owns blocks
// [rb0, rb0 + ceil(N / ROWS)) in the plain and fused-projection layouts.
struct WSeg {
    const uint32_t* wq;      // [N, w_row] packed codes
    const uint16_t* scales;  // [N, kg]
    const uint16_t* biases;  // [N, kg]
    void* y;                 // [nb0, nb1, M, N] through the launch's yb and this y_row
    int64_t N;
    int64_t w_row;           // words between W rows
    int64_t y_row;           // elements between rows of y
    int64_t rb0;             // first row block of the segment
    const void* r;           // optional residual, y's dtype and layout: y = r + x . W^T (null: none)
    int64_t r_row;           // elements between rows of r
};

struct WParams {
    CUtensorMap tw[MAX_SEGS];  // W of each segment: 2D {K*bits/32 words, N rows}, box {sub-block words,
                               // 32 rows (16 in the gate/up layout)}, no swizzle
    const uint16_t* x;       // [nb0, nb1, M, K] through xb / x_row
    WSeg seg[MAX_SEGS];
    int nseg;                // segments (1: a plain call)
    int glu;                 // 1: segments 0 (gate) and 1 (up) share every row block, 16 rows
                             //    each; the output is silu(gate) * up into segment 0's y
    int64_t nrb;             // row blocks of the launch
    int64_t M, K;
    int64_t x_row;
    int64_t xb[2], yb[2];
    int64_t nb1;
    int kg;                  // groups per row (K / group)
    int cs;                  // CTAs of a cluster splitting K (1: no split)
    int kgc;                 // groups per CTA of a cluster (kg when cs == 1)
    int gpw;                 // groups per warp
    int wr, wk;              // warps of a CTA along W rows / along K
    int ydt;                 // DT of y
    int yvec;                // 1: pairs of adjacent y elements may be stored as one vector
    int xsm;                 // 1: the CTA's x tile is staged in shared memory
    int x_pitch;             // bytes per staged x row (2 K + 16: spreads the lanes over the banks)
    int sb16;                // 1: each row block's scales and biases are copied as one bulk copy per
                             //    segment part (K/group a multiple of 8, 16-byte aligned); else 4-byte
                             //    cp.async copies
    int* err;                // device error word (DEVERR_TIMEOUT when a bounded wait expires)
    int rd;                  // ring slots per warp (a warp's sub-blocks, at most the ring's depth)
    int ring_bytes;          // bytes of a warp's ring (also holds its partial y tile at the end)
    int rms;                 // 1: the outputs are scaled by 1 / sqrt(mean_k x[t,k]^2 + rms_eps) per token
    float rms_eps;
};

constexpr size_t SMEM_LIMIT = 227 * 1024;

// Dynamic shared memory of a launch: the warps' W rings, the scales and biases of the CTA's rows,
// the CTA's partial tile when a cluster splits K, the sums of squares of x (per K-slice warp and
// token, then per token) when the inputs are RMS-normalised, and, when staged, the x tile.
constexpr int MAX_RD = 16;           // ring slots per warp (one mbarrier each)
constexpr size_t BAR_BYTES = (2 + MAX_WARPS * MAX_RD) * 8 + 16 + 128;   // staging + ring mbarriers, abort
                                                                       // flag, base alignment

inline size_t smem_bytes(int warps, int ring_bytes, int wr, int kg, int cs, int nt, int x_pitch, bool xsm, bool rms) {
    return (size_t)warps * ring_bytes + (size_t)wr * ROWS * kg * 2 * 2 +
           (cs > 1 ? (size_t)nt * wr * ROWS * sizeof(float) : 0) + (rms ? (size_t)(MAX_WARPS + 1) * nt * sizeof(float) : 0) +
           (xsm ? (size_t)nt * x_pitch : 0) + BAR_BYTES;
}

// defined in warp_mma_kernel.cuh, instantiated in kernels_warp_mma_b<BITS>.cu
template <int BITS>
cudaError_t launch(bool bf16, int group, int ntl, const WParams& p, dim3 grid, int warps, size_t smem,
                   cudaStream_t stream);
extern template cudaError_t launch<2>(bool, int, int, const WParams&, dim3, int, size_t, cudaStream_t);
extern template cudaError_t launch<4>(bool, int, int, const WParams&, dim3, int, size_t, cudaStream_t);
extern template cudaError_t launch<8>(bool, int, int, const WParams&, dim3, int, size_t, cudaStream_t);

}  // namespace wm
}  // namespace aq
