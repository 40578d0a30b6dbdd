/*
 * aq.h -- C ABI of libaq: affine group-quantized linear layers on B200 (sm_100a).
 *
 *     y = x . dequant(W)^T,   dequant(W)[n, k] = scale[n, k/G] * q[n, k] + bias[n, k/G]
 *
 * The operation, as the pages define it:
 *  - "MetalConfig quantization: batched generate silently corrupts all rows
 *    after the first" (transformers issue #47331), probe script and shape
 *    table: affine_qmm_t(x, w_packed, scales, biases, group, bits) must equal
 *    x @ dequant(W)^T row by row for every input shape -- [B, K], [1, S, K],
 *    [B, 1, K], [2, 4, K] -- i.e. leading batch dims are real batch dims.
 *  - "Metal Kernel Bits=8 Final Report", section 3.1: W [outDim, inDim*bits/32]
 *    uint32 with 32/bits codes per word, code inG of group g at word
 *    g*(G/(32/bits)) + inG/(32/bits), shift (inG % (32/bits))*bits; scales
 *    [outDim, inDim/G] (and G is inDim / scales.shape[-1]).
 *  - 3/5/6-bit codes: a dense little-endian bitstream per row, code i at bit
 *    i*bits of the row's uint32 words (the same rule the power-of-two formula
 *    is a special case of).
 *  - "mlx PR #4516": the bias term bias * sum(x) is formed from inputs widened
 *    to fp32 before they are added; rows past the end of the last row tile
 *    cost no per-row check inside the reduction loop.
 *  - candle "Metal batched matmul" pitfall page: strided batch views (narrowed
 *    Q/K heads, narrowed Linear inputs) are handled from EVERY batch stride,
 *    never from stride[-3] alone; uniform batch strides fold into rows.
 *
 * Conventions for every entry point:
 *  - All tensor arguments are aq_view descriptors of DEVICE memory owned by
 *    the caller.  The library allocates no memory, never synchronizes the
 *    stream, and keeps no pointer after the call returns.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream) of the current
 *    device; work is enqueued on it and runs asynchronously.
 *  - Strides are in ELEMENTS, may be any non-negative value, and the innermost
 *    stride of every view must be 1.
 *  - Arguments are validated on the host before any launch; on error nothing
 *    is launched and a status != AQ_OK is returned (never an abort).
 *    aq_status_string() names the status; aq_last_error_message() gives a
 *    one-line detail of the most recent failure on the calling thread.
 *  - Kernels never trap.  A kernel whose internal pipeline wait exceeds its
 *    bound records a device-side error instead; aq_device_error() reads and
 *    clears it (this one call synchronizes the stream).
 *  - Weights are constant operands.  The tensor-core kernels may start while
 *    the kernel before them in the stream still runs, and may read wq, scales
 *    and biases before that kernel has completed (the activations x and r only
 *    after it).  So the kernel immediately before a matrix call in its stream
 *    must not write that call's weights, unless it is aq_quantize (whose
 *    kernel lets no dependent start early and completes its writes before it
 *    exits).  Weights written earlier in the stream, by a copy, or on another
 *    stream and ordered by an event, are read correctly.
 */
#ifndef AQ_H
#define AQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum aq_status {
    AQ_OK = 0,
    AQ_ERR_NULL = 1,         /* a required pointer (view or data) is NULL            */
    AQ_ERR_DTYPE = 2,        /* dtype not allowed or dtypes disagree                 */
    AQ_ERR_RANK = 3,         /* view rank outside the allowed range                  */
    AQ_ERR_SHAPE = 4,        /* shapes inconsistent with each other / K, N, G, bits  */
    AQ_ERR_STRIDE = 5,       /* innermost stride != 1, or a negative stride          */
    AQ_ERR_BITS = 6,         /* bits not in {2, 3, 4, 5, 6, 8}                       */
    AQ_ERR_GROUP = 7,        /* group not in {32, 64, 128}, or K % group != 0        */
    AQ_ERR_ALIGN = 8,        /* a data pointer is not 16-byte aligned                */
    AQ_ERR_UNSUPPORTED = 9,  /* valid request the library does not implement         */
    AQ_ERR_OVERLAP = 10,     /* the output overlaps an input or itself               */
    AQ_ERR_CUDA = 11,        /* a CUDA runtime/driver call or a launch failed        */
    AQ_ERR_DEVICE = 12,      /* current device is not an sm_100 (B200-class) GPU     */
    AQ_ERR_TIMEOUT = 13,     /* a kernel's bounded pipeline wait expired (device)    */
    AQ_ERR_INDEX = 14        /* a row id on the device was out of range (device)     */
} aq_status;

typedef enum aq_dtype {
    AQ_F32 = 0,
    AQ_BF16 = 1,
    AQ_F16 = 2,
    AQ_U32 = 3
} aq_dtype;

/* A strided view of device memory: element (i0, .., i{rank-1}) lives at
 * data + sum_j i_j * stride[j] elements.  Entries past `rank` are ignored. */
typedef struct aq_view {
    void* data;
    int32_t dtype;      /* aq_dtype */
    int32_t rank;
    int64_t shape[4];
    int64_t stride[4];  /* in elements */
} aq_view;

/*
 * aq_quantize -- group-wise affine quantization of W.
 *   For each row n and group g of `group` consecutive K elements, in IEEE
 *   fp32: scale = (max - min) / (2^bits - 1), bias = min,
 *   q = clamp(rint((w - bias) / scale), 0, 2^bits - 1) (ties to even; a
 *   constant group has scale 0 and every q = 0); the stored scale and bias are
 *   then rounded to nearest-even in the dtype of `scales`/`biases`.
 *   (transformers issue #47331 probe script: quantize the fp32 W, then convert
 *   scales/biases to bf16.)
 * w:      [N, K] AQ_F32, AQ_BF16 or AQ_F16 (rank 2; rows may be strided).
 * wq:     [N, K*bits/32] AQ_U32 out, packed as described at the top.
 * scales: [N, K/group] AQ_BF16 or AQ_F16 out; biases: same shape and dtype.
 * The outputs must not overlap the input, each other, or themselves.
 * W must be finite; NaN/Inf inputs give unspecified codes.
 */
aq_status aq_quantize(const aq_view* w, int group, int bits, const aq_view* wq,
                      const aq_view* scales, const aq_view* biases, void* stream);

/*
 * aq_dequantize -- w_out[n, k] = scale[n, k/G] * q[n, k] + bias[n, k/G],
 *   evaluated in fp32 and rounded once to the dtype of w_out.
 * wq [N, K*bits/32] AQ_U32; scales/biases [N, K/group] AQ_BF16|AQ_F16;
 * w_out [N, K] AQ_F32, AQ_BF16 or AQ_F16.  All rank 2.
 */
aq_status aq_dequantize(const aq_view* wq, const aq_view* scales, const aq_view* biases,
                        int group, int bits, const aq_view* w_out, void* stream);

/*
 * aq_dequantize_rows -- embedding lookup on a quantized table, one row per id:
 *     out[t, k] = scale[ids[t], k/G] * q[ids[t], k] + bias[ids[t], k/G],   t < n_ids
 *   evaluated in fp32 and rounded once to out's dtype (the values aq_dequantize gives).
 *   ("Metal Kernel Bits=8 Final Report", sections 3.1-3.2 and 5.1: dequantize_row and
 *   dequantize_row_8bit turn the row of one token id into activations, called from
 *   dequantizeRow(weight:tokenId:output:); its embedding table is [262144, 352] uint32,
 *   scales [262144, 44].)
 * wq [V, K*bits/32] AQ_U32; scales/biases [V, K/group] AQ_BF16|AQ_F16 (rank 2).
 * ids: DEVICE pointer to n_ids int64 row ids (not readable on the host).  An id outside
 *   [0, V) gives a row of zeros and sets a device error that aq_device_error() returns as
 *   AQ_ERR_INDEX.
 * out [n_ids, K] AQ_F32, AQ_BF16 or AQ_F16, must not overlap the table.
 */
aq_status aq_dequantize_rows(const aq_view* wq, const aq_view* scales, const aq_view* biases,
                             int group, int bits, const int64_t* ids, int64_t n_ids,
                             const aq_view* out, void* stream);

/*
 * aq_qmm_t -- y = x . dequant(W)^T for any number of rows.
 * x:      rank 1..4, [..., M, K], AQ_BF16 or AQ_F16, any batch/row strides.
 *         Batch dims whose strides are uniform (stride[i] == stride[i+1] *
 *         shape[i+1] for x and y) fold into rows; the others are real batch
 *         dims whose offsets come from every one of their strides.
 * wq:     [..., N, K*bits/32] AQ_U32 with 0..2 batch dims that are 1
 *         (shared weight) or equal to x's corresponding batch dims
 *         (right-aligned, as in broadcasting).
 * scales, biases: [..., N, K/group], same dtype as x, same batch dims as wq.
 * y:      x.shape[:-1] + [N], dtype of x or AQ_F32, must not overlap inputs, and no two
 *         of its elements may share an address (a zero stride on a dimension of extent
 *         > 1 is AQ_ERR_OVERLAP).
 * bits in {2,3,4,5,6,8}; group in {32,64,128}; K % group == 0.
 * Rows per launch batch decide the kernel (aq_plan_linear reports it): up to 4
 * rows (or a batched W), a CUDA-core GEMV; 5..32 rows in total with 2/4/8-bit
 * codes (2-bit codes need groups of 64/128), where measured faster (always up
 * to 8 rows; up to 16 rows unless N is so large that a CTA holds many row
 * blocks and a warp more than eight 64-code pieces of K (lm_head); at 32 rows unless N is so large that
 * a CTA holds many row blocks, or K per warp is long), a warp-level mma.sync kernel that expands W
 * in registers, K split over a thread-block cluster when row blocks are few;
 * other cases below 64 rows, a tcgen05/TMEM kernel on tiles
 * of 128 W rows x 32 tokens (K split over the CTAs of a thread-block cluster
 * when the tiles alone would leave most SMs idle); 64 rows and more with
 * groups of 64/128, a tcgen05 kernel on 128 x 128 tiles.  3/5-bit codes, K
 * not a multiple of 64, an odd or very large K/group, or unaligned rows take
 * the GEMV.
 * Every kernel keeps W exact (integer codes, scale and bias in fp32).  The
 * tensor-core kernels are launched as programmatic dependents of the previous
 * kernel in the stream: their set-up and (warp-level kernel) the staging of
 * the weights overlap it, x is read only after it completed (see "Weights are
 * constant operands" above).  Where y has x's dtype, N is a multiple of 8 and
 * y's rows and batch strides are 16-byte aligned, the tcgen05 kernels write
 * each tile of y as one bulk tensor copy from shared memory (nothing outside
 * y's [.., M, N] is written); elsewhere they store y element by element.
 * Data pointers must be 16-byte aligned.
 */
aq_status aq_qmm_t(const aq_view* x, const aq_view* wq, const aq_view* scales,
                   const aq_view* biases, int group, int bits, const aq_view* y, void* stream);

/*
 * aq_qmv -- same contract as aq_qmm_t, but always runs the CUDA-core GEMV
 * kernel (128-bit weight loads, in-register unpack, fp32 s*sum(q*x) +
 * b*sum(x) with inputs widened before every sum, warp-shuffle reduction,
 * partial-rows tail without per-row checks in the loop).  Rows are processed
 * a few at a time, so large M re-reads W.
 */
aq_status aq_qmv(const aq_view* x, const aq_view* wq, const aq_view* scales,
                 const aq_view* biases, int group, int bits, const aq_view* y, void* stream);

/*
 * aq_qmm_t_grouped -- mixture-of-experts bank:
 *   y_sorted[t] = x_sorted[t] . dequant(W_e)^T  for offsets[e] <= t < offsets[e+1].
 * x_sorted: [T, K] AQ_BF16|AQ_F16 (rows grouped by expert, row stride free).
 * offsets:  DEVICE pointer to n_experts+1 int64, non-decreasing, offsets[0] = 0,
 *           offsets[n_experts] = T.  The host cannot check it (it lives on the device);
 *           the kernel clamps every expert's range into [0, T) (an end below its start is
 *           an empty expert), so a malformed array gives wrong rows but never an access
 *           outside x_sorted / y_sorted.
 * wq_bank [E, N, K*bits/32] AQ_U32; s_bank, b_bank [E, N, K/group].
 * y_sorted: [T, N], dtype of x or AQ_F32.
 * (Prior art: the gathered QMV of "mlx PR #4516"; expert shapes from "Metal
 * Kernel Bits=8 Final Report", section 4.3.)
 */
aq_status aq_qmm_t_grouped(const aq_view* x_sorted, const int64_t* offsets, int n_experts,
                           const aq_view* wq_bank, const aq_view* s_bank, const aq_view* b_bank,
                           int group, int bits, const aq_view* y_sorted, void* stream);

/*
 * aq_qmv_gathered -- mixture-of-experts rows without a host-side sort (the "gathered QMV" that
 * "mlx PR #4516" names next to its affine qmv kernels): for i < n_rows,
 *     y[i] = x[x_ids[i]] . dequant(W_{w_ids[i]})^T
 * so a decode step can route each token to its experts straight from the router's output.
 * x [T, K] AQ_BF16|AQ_F16 (row stride free); wq_bank [E, N, K*bits/32] AQ_U32; s_bank,
 * b_bank [E, N, K/group] in x's dtype (any row/entry strides that keep W rows aligned as for
 * aq_qmm_t); x_ids, w_ids: DEVICE pointers to n_rows int64 ids (n_rows <= 65535);
 * y [n_rows, N], x's dtype or AQ_F32.  Runs the CUDA-core GEMV, one row per id pair (each row
 * streams its expert's weights: meant for decode, where rows are few).  An id outside
 * [0, T) or [0, E) gives a row of zeros and a device error that aq_device_error() returns
 * as AQ_ERR_INDEX.
 */
aq_status aq_qmv_gathered(const aq_view* x, const int64_t* x_ids, const int64_t* w_ids, int64_t n_rows,
                          const aq_view* wq_bank, const aq_view* s_bank, const aq_view* b_bank,
                          int group, int bits, const aq_view* y, void* stream);

/* ---------------------------------------------------------------------- */
/* Fused calls of a decoder layer's decode step (warp-level kernel).       */
/*                                                                        */
/* The decode step the pages' bug reports run (transformers issue #47331, */
/* reproduction: a Qwen3-0.6B decoder under generate(), every projection  */
/* an affine_qmm_t on x [B, 1, hidden]; "mlx PR #4516": the narrow decode */
/* projections dominate decode time) makes seven small calls per layer.   */
/* These entry points do the same arithmetic as aq_qmm_t -- W exact,      */
/* factored s*sum(q*x) + b*sum(x) with x widened to fp32 before it is     */
/* summed -- in fewer launches.  x and every output must fold into one 2D */
/* problem (no launch batch dims) and W is unbatched.                     */
/* ---------------------------------------------------------------------- */

/*
 * Optional RMS-normalised input (rms_eps > 0) of aq_qmm_t_multi and aq_qmm_t_swiglu: the block
 * inputs of the decoder are normalised per token (RMSNorm), and since the contraction is linear
 * in x the kernel applies the norm to its result instead:
 *     x . W^T  ->  (x . W^T) / sqrt(mean_k x[t, k]^2 + rms_eps)
 * with the sum of squares of the widened x formed in fp32 next to sum(x); the norm's weight
 * vector is taken as folded into W (the decoder's RMSNorm is not on the pages; it keeps a chain
 * of layers at unit scale).  rms_eps = 0: no normalisation.
 */

/*
 * aq_qmm_t_multi -- n (1..3) matrices that share one input, in one launch:
 *     y[j] = x . dequant(W_j)^T,  j < n       (e.g. the q, k and v projections)
 * wq[j], scales[j], biases[j], y[j] as for aq_qmm_t, each W_j with its own N_j and
 * the same K; no output may overlap another output or any input.
 * One launch of the warp-level kernel when it takes every matrix (up to 32 rows in
 * total, 2/4/8-bit codes, 16-byte aligned rows); otherwise, without rms_eps, one
 * aq_qmm_t per matrix, in order, on the same stream (same results to the same bar),
 * and with rms_eps > 0, AQ_ERR_UNSUPPORTED.
 */
aq_status aq_qmm_t_multi(const aq_view* x, int n, const aq_view* const* wq, const aq_view* const* scales,
                         const aq_view* const* biases, int group, int bits, float rms_eps,
                         const aq_view* const* y, void* stream);

/*
 * aq_qmm_t_swiglu -- the gated MLP input of the decoder layer, in one launch:
 *     y = silu(x . dequant(W_gate)^T) * (x . dequant(W_up)^T),  silu(v) = v / (1 + exp(-v))
 * Both contractions are complete fp32 sums (each scaled by the RMS norm when rms_eps > 0)
 * before the activation; y is rounded once.
 * W_gate and W_up: [N, K*bits/32] with their scales and biases; y: x.shape[:-1] + [N].
 * (The activation is a reading: the issue names the model, whose MLP is
 * down(silu(gate(h)) * up(h)); the pages do not spell it out.)
 * Warp-level kernel only; AQ_ERR_UNSUPPORTED where it does not take the problem.
 */
aq_status aq_qmm_t_swiglu(const aq_view* x, const aq_view* wq_gate, const aq_view* s_gate,
                          const aq_view* b_gate, const aq_view* wq_up, const aq_view* s_up,
                          const aq_view* b_up, int group, int bits, float rms_eps, const aq_view* y,
                          void* stream);

/*
 * aq_qmm_t_residual -- a projection that adds into the residual stream, in one launch:
 *     y = r + x . dequant(W)^T
 * r has y's shape and dtype; the sum is formed in fp32 and rounded once.  r may be y
 * itself (the same view: an in-place update) but must not overlap it otherwise.
 * Warp-level kernel only; AQ_ERR_UNSUPPORTED where it does not take the problem.
 */
aq_status aq_qmm_t_residual(const aq_view* x, const aq_view* wq, const aq_view* scales,
                            const aq_view* biases, int group, int bits, const aq_view* r,
                            const aq_view* y, void* stream);

/* ---------------------------------------------------------------------- */
/* Introspection (host only, no GPU work).                                 */
/* ---------------------------------------------------------------------- */

typedef enum aq_regime {
    AQ_REGIME_QMV = 0,   /* CUDA-core GEMV                      */
    AQ_REGIME_MMA = 1    /* a tensor-core kernel (aq_kernel)    */
} aq_regime;

/* The kernel a call runs (aq_plan.kernel). */
typedef enum aq_kernel {
    AQ_KERNEL_GEMV = 0,        /* CUDA-core GEMV, 128-bit loads, warp-shuffle sums        */
    AQ_KERNEL_WARP_MMA = 1,    /* mma.sync, W expanded in registers, up to 32 rows        */
    AQ_KERNEL_TC_SMALL_M = 2,  /* tcgen05/TMEM, 128 W rows x 32 tokens, split-K clusters  */
    AQ_KERNEL_TC_PREFILL = 3   /* tcgen05/TMEM, 128 x 128 tiles, >= 64 rows, groups 64/128 */
} aq_kernel;

/* How a call will be executed: the result of view resolution and batch folding. */
typedef struct aq_plan {
    int32_t regime;            /* aq_regime                                            */
    int32_t w_batched;         /* 1 if W has a non-broadcast batch dim                 */
    int64_t M;                 /* rows per launch batch after folding                  */
    int64_t N, K;
    int32_t nbatch_dims;       /* launch batch dims left after folding (0..2)         */
    int32_t kernel;            /* aq_kernel                                            */
    int64_t batch_shape[2];    /* outer first                                          */
    int64_t x_batch_stride[2];
    int64_t y_batch_stride[2];
    int64_t w_batch_stride[2]; /* 0 where W broadcasts                                 */
    int64_t s_batch_stride[2];
    int64_t b_batch_stride[2];
    int64_t x_row_stride;      /* elements between folded rows                         */
    int64_t y_row_stride;
    int64_t total_rows;        /* product of batch_shape * M                           */
    int32_t y_tiles;           /* 1: a tcgen05 kernel writes each tile of y with one   */
                               /*    bulk tensor store from shared memory              */
} aq_plan;

/*
 * Resolve views, fold batch dims and pick the kernel exactly as aq_qmm_t
 * (force_qmv = 0) or aq_qmv (force_qmv = 1) would, without launching
 * anything.  Data pointers are checked for NULL and alignment only.
 */
aq_status aq_plan_linear(const aq_view* x, const aq_view* wq, const aq_view* scales,
                         const aq_view* biases, int group, int bits, const aq_view* y,
                         int force_qmv, aq_plan* out);

const char* aq_status_string(aq_status status);

/* One-line description of the last error returned on the calling thread ("" if none). */
const char* aq_last_error_message(void);

/*
 * Reads and clears the device-side error word of the current device after
 * synchronizing `stream`.  Returns AQ_OK if no kernel recorded an error,
 * AQ_ERR_TIMEOUT if a bounded wait expired, AQ_ERR_INDEX if a row gather met an
 * id outside its table, AQ_ERR_CUDA if the read failed.  For AQ_ERR_TIMEOUT,
 * aq_last_error_message() names the kernel and the wait that gave up first (a
 * copy, the tensor core, or another role of the kernel).
 */
aq_status aq_device_error(void* stream);

/*
 * aq_check_bounded_wait -- exercises the bounded wait of the pipeline kernels without any
 * fault: one warp waits, with the same bounded wait, on a barrier that nothing completes, gives
 * up after budget_ns (0 < budget_ns <= 1e9) and records the timeout in the device error word,
 * so that the next aq_device_error() returns AQ_ERR_TIMEOUT and clears it.  Nothing is in flight
 * when it gives up: the context stays usable.  (No counterpart on the pages: a self-check of
 * this library's failure reporting.)
 */
aq_status aq_check_bounded_wait(uint64_t budget_ns, void* stream);

/* Library version: major*10000 + minor*100 + patch. */
int aq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* AQ_H */
