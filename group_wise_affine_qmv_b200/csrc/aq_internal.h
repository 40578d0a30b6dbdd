// aq_internal.h -- shared declarations between the host dispatcher and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "aq.h"

namespace aq {

// Element types of x / scales / biases (16-bit) and of y.
enum class DT : int { F32 = AQ_F32, BF16 = AQ_BF16, F16 = AQ_F16 };

// ---------------------------------------------------------------------------
// CUDA-core GEMV (qmv) arguments.  One launch batch per blockIdx.y; inside a
// launch batch, M rows of x (row stride x_row) against N rows of W.
// ---------------------------------------------------------------------------
struct QmvArgs {
    const void* x;
    const uint32_t* wq;
    const void* scales;
    const void* biases;
    void* y;
    int64_t x_row, y_row;          // elements between consecutive rows of x / y
    int64_t w_row, s_row, b_row;   // row strides of W (words), scales, biases (elements)
    int64_t M, N, K;
    int log2g;                     // log2(group)
    int xvec;                      // 1: x rows 16-byte aligned (vector loads allowed)
    int64_t bshape1;               // size of the inner launch-batch dim (1 if none)
    int64_t xb[2], yb[2], wb[2], sb[2], bb[2];  // launch-batch strides (outer, inner)
    // gathered rows (x_ids != nullptr): launch batch i is row i of y, computed from x row x_ids[i]
    // and W bank entry w_ids[i] (xb[0] / wb[0] / sb[0] / bb[0] are the per-row / per-entry strides,
    // yb[0] the row stride of y); ids outside [0, x_rows) / [0, w_entries) give a row of zeros
    // and set DEVERR_INDEX in *err
    const int64_t* x_ids;
    const int64_t* w_ids;
    int64_t x_rows, w_entries;
    int* err;
};

// Launches the GEMV kernel for `nbatch` launch batches.  Returns cudaSuccess or the launch error.
cudaError_t launch_qmv(const QmvArgs& a, int bits, DT xdt, DT ydt, int64_t nbatch, cudaStream_t s);

// ---------------------------------------------------------------------------
// Quantize / dequantize.
// ---------------------------------------------------------------------------
struct QuantArgs {
    const void* w;        // [N, K] (quantize input / dequantize output)
    uint32_t* wq;         // [N, K*bits/32]
    void* scales;         // [N, K/G]
    void* biases;
    int64_t w_row, wq_row, s_row, b_row;
    int64_t N, K;
    int group, bits;
    // dequantize only: row t of the output is row ids[t] of W (ids on the device, V rows of W);
    // an id outside [0, V) gives a row of zeros and sets DEVERR_INDEX in *err
    const int64_t* ids;
    int64_t V;
    int* err;
};
cudaError_t launch_quantize(const QuantArgs& a, DT wdt, DT sdt, cudaStream_t s);
cudaError_t launch_dequantize(const QuantArgs& a, DT wdt, DT sdt, cudaStream_t s);

// ---------------------------------------------------------------------------
// tcgen05 tensor-core kernel (A = dequantized W in TMEM, B = x tile in SMEM).
// ---------------------------------------------------------------------------
struct MmaProblem {
    // x viewed as [nb0, nb1, M, K] (strides in elements); y likewise with N.
    const void* x;
    void* y;
    const uint32_t* wq;
    const void* scales;
    const void* biases;
    int64_t M, N, K;
    int64_t x_row, y_row;
    int64_t nb[2];              // launch batch dims (outer, inner), 1 if absent
    int64_t xb[2], yb[2];
    int64_t w_row;              // words
    int group, bits;
    DT xdt, ydt;
    // grouped (mixture-of-experts) mode: offsets != nullptr
    const int64_t* offsets;     // device, n_experts + 1
    int n_experts;
    int64_t w_expert, s_expert, b_expert;  // per-expert strides (words / elements)
    // fused calls (warp-level kernel only): nseg > 1 W matrices share x in one launch; entry 0
    // repeats wq/scales/biases/y/N/w_row/y_row above.  glu: two segments (gate, up) whose
    // output is silu(gate) * up, written to seg_y[0].
    int nseg;
    int glu;
    const uint32_t* seg_wq[3];
    const void* seg_scales[3];
    const void* seg_biases[3];
    void* seg_y[3];
    int64_t seg_N[3], seg_w_row[3], seg_y_row[3];
    // optional residual of the plain call (warp-level kernel only): y = r + x . W^T
    const void* r;
    int64_t r_row;
    // fused calls: rms_eps > 0 scales every output of token t by 1 / sqrt(mean_k x[t,k]^2 + rms_eps)
    // (an RMS-normalised input, the norm's weight folded into W)
    float rms_eps;
};

// Whether the tensor-core kernel can run this problem (alignment, bits, K), and why not.
bool mma_supported(const MmaProblem& p, const char** why);
cudaError_t launch_mma(const MmaProblem& p, cudaStream_t s);

// Which tensor-core kernel launch_mma runs for a supported problem.
enum class MmaKernel : int { WARP = AQ_KERNEL_WARP_MMA, SMALL_M = AQ_KERNEL_TC_SMALL_M, PREFILL = AQ_KERNEL_TC_PREFILL };
MmaKernel mma_kernel_for(const MmaProblem& p);
// whether the tcgen05 kernel chosen for p writes each tile of y with one bulk tensor store
bool mma_y_tiles(const MmaProblem& p);

// Warp-level (mma.sync) kernel for up to 32 rows per launch batch: whether it takes the problem
// (given that mma_supported accepted it) and its launch.
bool warp_mma_supported(const MmaProblem& p);
bool warp_mma_preferred(const MmaProblem& p);
cudaError_t launch_warp_mma(const MmaProblem& p, cudaStream_t s);

// A 2D tensor map over packed W rows ({words, rows} uint32, row stride in words), box
// {box_words, box_rows}, no swizzle; false if the driver rejects it.
bool encode_w_rows(void* map, const uint32_t* wq, int64_t words, int64_t rows, int64_t row_stride_words,
                   int box_words, int box_rows);

// Device-side error word: bits set by kernels (a bounded wait expired; an index out of range).
constexpr int DEVERR_TIMEOUT = 1;
constexpr int DEVERR_INDEX = 2;
// Where a bounded wait expired (set with DEVERR_TIMEOUT by the wait that ran out first, not by the
// waits that returned because the CTA was already aborting); aq_device_error names them.
constexpr int DEVERR_AT_WARP_X = 1 << 8;      // warp-level kernel: the x tile's staging copies
constexpr int DEVERR_AT_WARP_SB = 1 << 9;     //   the scale/bias staging copies
constexpr int DEVERR_AT_WARP_W = 1 << 10;     //   a W box of a warp's ring
constexpr int DEVERR_AT_TC_WFREE = 1 << 11;   // tcgen05 small-M kernel: W producer waiting for the expanders
constexpr int DEVERR_AT_TC_XFREE = 1 << 12;   //   x producer waiting for the MMAs to release an x stage
constexpr int DEVERR_AT_TC_XFULL = 1 << 13;   //   MMA issuer waiting for an x copy
constexpr int DEVERR_AT_TC_AFULL = 1 << 14;   //   MMA issuer waiting for the expanders
constexpr int DEVERR_AT_TC_DFREE = 1 << 15;   //   MMA issuer waiting for the folds
constexpr int DEVERR_AT_TC_WFULL = 1 << 16;   //   expanders waiting for a W copy
constexpr int DEVERR_AT_TC_SDONE_E = 1 << 17; //   expanders waiting for MMAs to complete
constexpr int DEVERR_AT_TC_SDONE_F = 1 << 18; //   folds waiting for MMAs to complete
constexpr int DEVERR_AT_TC_FOLD = 1 << 19;    //   folds waiting for the other folds, x or the cluster
constexpr int DEVERR_AT_PF_W = 1 << 20;       // prefill kernel: W producer
constexpr int DEVERR_AT_PF_X = 1 << 21;       //   x producer
constexpr int DEVERR_AT_PF_MMA = 1 << 22;     //   MMA issuer
constexpr int DEVERR_AT_PF_EXP = 1 << 23;     //   code expanders
constexpr int DEVERR_AT_PF_FOLD = 1 << 24;    //   folds
constexpr int DEVERR_AT_CHECK = 1 << 25;      // the bounded-wait self-check
cudaError_t read_and_clear_device_error(int* value, cudaStream_t s);
// its device address on the current device
cudaError_t device_error_ptr(int** p);
// one warp's bounded wait on a barrier nothing completes (budget in ns)
cudaError_t launch_bounded_wait_check(uint64_t budget_ns, cudaStream_t s);

}  // namespace aq
