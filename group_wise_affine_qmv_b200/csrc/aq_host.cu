// aq_host.cu -- the C ABI of libaq: argument validation, view resolution,
// batch folding, kernel selection.  No device code lives here.
//
// Batch folding follows the candle "Metal batched matmul" pitfall page
// (section "how to check"): a batch dim folds into rows only when
// stride[i] == stride[i+1] * dims[i+1] holds for it (size-1 dims exempt);
// every other batch dim stays a real batch dim whose offset is computed from
// its own stride -- never from stride[-3] alone, and never by treating a 3D
// input as 2D [shape[-2], K] (transformers issue #47331, root cause).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "aq_internal.h"

#define AQ_API extern "C" __attribute__((visibility("default")))

namespace {

thread_local char g_msg[512] = "";

aq_status fail(aq_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

int elem_size(int dt) {
    switch (dt) {
        case AQ_F32: return 4;
        case AQ_BF16: return 2;
        case AQ_F16: return 2;
        case AQ_U32: return 4;
        default: return 0;
    }
}

bool is_half(int dt) { return dt == AQ_BF16 || dt == AQ_F16; }

aq_status check_view(const aq_view* v, const char* name, int min_rank, int max_rank) {
    if (!v) return fail(AQ_ERR_NULL, "%s: view is NULL", name);
    if (v->rank < min_rank || v->rank > max_rank)
        return fail(AQ_ERR_RANK, "%s: rank %d outside [%d, %d]", name, v->rank, min_rank, max_rank);
    if (elem_size(v->dtype) == 0) return fail(AQ_ERR_DTYPE, "%s: unknown dtype %d", name, v->dtype);
    bool empty = false;
    for (int i = 0; i < v->rank; ++i) {
        if (v->shape[i] < 0) return fail(AQ_ERR_SHAPE, "%s: negative extent", name);
        if (v->stride[i] < 0) return fail(AQ_ERR_STRIDE, "%s: negative stride", name);
        if (v->shape[i] == 0) empty = true;
    }
    if (!empty && v->shape[v->rank - 1] > 1 && v->stride[v->rank - 1] != 1)
        return fail(AQ_ERR_STRIDE, "%s: innermost stride must be 1", name);
    if (!empty && !v->data) return fail(AQ_ERR_NULL, "%s: data is NULL", name);
    return AQ_OK;
}

int64_t numel(const aq_view* v) {
    int64_t n = 1;
    for (int i = 0; i < v->rank; ++i) n *= v->shape[i];
    return n;
}

// byte span [lo, hi) touched by a view (0,0 if empty)
void span(const aq_view* v, uintptr_t* lo, uintptr_t* hi) {
    if (numel(v) == 0) { *lo = *hi = 0; return; }
    int64_t last = 0;
    for (int i = 0; i < v->rank; ++i) last += (v->shape[i] - 1) * v->stride[i];
    *lo = (uintptr_t)v->data;
    *hi = *lo + (uintptr_t)((last + 1) * elem_size(v->dtype));
}

bool overlaps(const aq_view* a, const aq_view* b) {
    uintptr_t alo, ahi, blo, bhi;
    span(a, &alo, &ahi);
    span(b, &blo, &bhi);
    if (alo == ahi || blo == bhi) return false;
    return alo < bhi && blo < ahi;
}

// Whether two different indices of an output view reach the same element (a zero stride on a
// dimension of extent > 1, as an expand()ed tensor has, or strides too small for the extents
// inside them): several threads would then race on one element.  Dimensions are visited from the
// smallest stride up; each stride must exceed the largest offset the dimensions below it reach.
bool self_overlapping(const aq_view* v) {
    int idx[4];
    int n = 0;
    for (int i = 0; i < v->rank && i < 4; ++i)   // (ranks above 4 are rejected before)
        if (v->shape[i] > 1) idx[n++] = i;
    for (int j = 1; j < n; ++j)                   // by stride, ascending (at most 4 entries)
        for (int k = j; k > 0 && v->stride[idx[k]] < v->stride[idx[k - 1]]; --k) std::swap(idx[k], idx[k - 1]);
    int64_t reach = 0;
    for (int j = 0; j < n; ++j) {
        const int i = idx[j];
        if (v->stride[i] <= reach) return true;
        reach += (v->shape[i] - 1) * v->stride[i];
    }
    return false;
}

aq_status check_output(const aq_view* v, const char* name) {
    if (numel(v) > 0 && self_overlapping(v))
        return fail(AQ_ERR_OVERLAP, "%s: elements overlap (zero or too small stride)", name);
    return AQ_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

aq_status check_bits_group(int bits, int group) {
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 5 || bits == 6 || bits == 8))
        return fail(AQ_ERR_BITS, "bits=%d not in {2,3,4,5,6,8}", bits);
    if (!(group == 32 || group == 64 || group == 128))
        return fail(AQ_ERR_GROUP, "group=%d not in {32,64,128}", group);
    return AQ_OK;
}

int log2i(int v) { int r = 0; while ((1 << r) < v) ++r; return r; }

aq_status cuda_fail(cudaError_t e, const char* what) {
    return fail(AQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// The kernels are built for sm_100a only.
aq_status check_device() {
    static std::mutex mu;
    static int checked[64] = {0};  // 0 unknown, 1 ok, 2 bad
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(AQ_ERR_DEVICE, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lk(mu);
    if (checked[dev] == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return fail(AQ_ERR_CUDA, "cannot query device %d", dev);
        checked[dev] = (major == 10 && minor == 0) ? 1 : 2;
    }
    if (checked[dev] != 1) return fail(AQ_ERR_DEVICE, "device %d is not sm_100", dev);
    return AQ_OK;
}

// ---------------------------------------------------------------------------
// view resolution for the linear entry points
// ---------------------------------------------------------------------------

struct Resolved {
    aq_plan plan;
    int64_t w_row, s_row, b_row;
    int xvec;
    bool mma_ok;
    const char* mma_why;
    aq::MmaProblem mp;
};

void fill_mma_problem(const aq_view* x, const aq_view* wq, const aq_view* sc, const aq_view* bi, int group,
                      int bits, const aq_view* y, Resolved* R);

aq_status resolve_linear(const aq_view* x, const aq_view* wq, const aq_view* sc, const aq_view* bi,
                         int group, int bits, const aq_view* y, int force_qmv, Resolved* R) {
    aq_status st;
    if ((st = check_view(x, "x", 1, 4)) != AQ_OK) return st;
    if ((st = check_view(wq, "wq", 2, 4)) != AQ_OK) return st;
    if ((st = check_view(sc, "scales", 2, 4)) != AQ_OK) return st;
    if ((st = check_view(bi, "biases", 2, 4)) != AQ_OK) return st;
    if ((st = check_view(y, "y", 1, 4)) != AQ_OK) return st;
    if ((st = check_output(y, "y")) != AQ_OK) return st;
    if ((st = check_bits_group(bits, group)) != AQ_OK) return st;
    if (!is_half(x->dtype)) return fail(AQ_ERR_DTYPE, "x must be bf16 or f16");
    if (wq->dtype != AQ_U32) return fail(AQ_ERR_DTYPE, "wq must be u32");
    if (sc->dtype != x->dtype || bi->dtype != x->dtype)
        return fail(AQ_ERR_DTYPE, "scales/biases must have x's dtype");
    if (y->dtype != x->dtype && y->dtype != AQ_F32)
        return fail(AQ_ERR_DTYPE, "y must have x's dtype or f32");

    const int rx = x->rank, rw = wq->rank;
    const int64_t K = x->shape[rx - 1];
    const int64_t N = wq->shape[rw - 2];
    if (K % group != 0) return fail(AQ_ERR_GROUP, "K=%lld not a multiple of group=%d", (long long)K, group);
    if (wq->shape[rw - 1] != K * bits / 32)
        return fail(AQ_ERR_SHAPE, "wq last dim %lld != K*bits/32 = %lld", (long long)wq->shape[rw - 1],
                    (long long)(K * bits / 32));
    if (sc->rank != rw || bi->rank != rw) return fail(AQ_ERR_RANK, "scales/biases rank must equal wq rank");
    for (int i = 0; i < rw - 1; ++i)
        if (sc->shape[i] != wq->shape[i] || bi->shape[i] != wq->shape[i])
            return fail(AQ_ERR_SHAPE, "scales/biases leading dims must equal wq's");
    if (sc->shape[rw - 1] != K / group || bi->shape[rw - 1] != K / group)
        return fail(AQ_ERR_SHAPE, "scales/biases last dim must be K/group = %lld", (long long)(K / group));
    if (y->rank != rx) return fail(AQ_ERR_RANK, "y rank must equal x rank");
    for (int i = 0; i < rx - 1; ++i)
        if (y->shape[i] != x->shape[i]) return fail(AQ_ERR_SHAPE, "y.shape[:-1] must equal x.shape[:-1]");
    if (y->shape[rx - 1] != N) return fail(AQ_ERR_SHAPE, "y last dim must be N=%lld", (long long)N);

    const int nxb = rx >= 2 ? rx - 2 : 0;
    const int nwb = rw - 2;
    if (nwb > nxb && numel(wq) > 0) {
        for (int i = 0; i < nwb - nxb; ++i)
            if (wq->shape[i] != 1) return fail(AQ_ERR_SHAPE, "wq has more batch dims than x");
    }

    // alignment of weights (vector loads in every kernel)
    if (numel(wq) > 0) {
        if (!aligned16(wq->data)) return fail(AQ_ERR_ALIGN, "wq data must be 16-byte aligned");
        const int64_t need = (bits == 4 || bits == 8) ? 4 : (bits == 2 || bits == 6) ? 2 : 1;  // words
        if (N > 1 && wq->stride[rw - 2] % need != 0)
            return fail(AQ_ERR_ALIGN, "wq row stride must keep rows %lld-byte aligned", (long long)(need * 4));
    }

    if (numel(x) > 0 || numel(y) > 0) {
        if (overlaps(y, x) || overlaps(y, wq) || overlaps(y, sc) || overlaps(y, bi))
            return fail(AQ_ERR_OVERLAP, "y overlaps an input");
    }

    // ---- batch dims, outer to inner ----
    struct Dim { int64_t size, xs, ys, ws, ss, bs; bool wb; };
    Dim dims[2];
    int nd = 0;
    bool w_batched = false;
    for (int i = 0; i < nxb; ++i) {
        Dim d{};
        d.size = x->shape[i];
        d.xs = x->stride[i];
        d.ys = y->stride[i];
        int j = i - (nxb - nwb);
        if (j >= 0 && wq->shape[j] != 1) {
            if (wq->shape[j] != x->shape[i])
                return fail(AQ_ERR_SHAPE, "wq batch dim %d (%lld) does not match x (%lld)", j,
                            (long long)wq->shape[j], (long long)x->shape[i]);
            d.wb = true;
            d.ws = wq->stride[j];
            d.ss = sc->stride[j];
            d.bs = bi->stride[j];
            if (d.ws % 4 != 0 && bits != 3 && bits != 5)
                return fail(AQ_ERR_ALIGN, "wq batch stride must keep rows 16-byte aligned");
        }
        if (d.size == 1) continue;  // size-1 dims carry no offset
        if (d.wb) w_batched = true;
        dims[nd++] = d;
    }
    int64_t M = rx >= 2 ? x->shape[rx - 2] : 1;
    int64_t xrow = rx >= 2 ? x->stride[rx - 2] : K;
    int64_t yrow = y->rank >= 2 ? y->stride[rx - 2] : N;
    // fold from the innermost batch dim outwards
    int keep = nd;
    for (int i = nd - 1; i >= 0; --i) {
        const Dim& d = dims[i];
        if (d.wb) break;
        if (M == 1) {  // a single row has no row stride of its own: adopt this dim's
            M = d.size;
            xrow = d.xs;
            yrow = d.ys;
            keep = i;
            continue;
        }
        if (d.xs == xrow * M && d.ys == yrow * M) {
            M *= d.size;
            keep = i;
            continue;
        }
        break;
    }
    nd = keep;

    aq_plan& P = R->plan;
    memset(&P, 0, sizeof P);
    P.w_batched = w_batched ? 1 : 0;
    P.M = M;
    P.N = N;
    P.K = K;
    P.nbatch_dims = nd;
    P.batch_shape[0] = P.batch_shape[1] = 1;
    // right-align the remaining batch dims into slots [0,1]
    for (int i = 0; i < nd; ++i) {
        int s = 2 - nd + i;
        P.batch_shape[s] = dims[i].size;
        P.x_batch_stride[s] = dims[i].xs;
        P.y_batch_stride[s] = dims[i].ys;
        P.w_batch_stride[s] = dims[i].ws;
        P.s_batch_stride[s] = dims[i].ss;
        P.b_batch_stride[s] = dims[i].bs;
    }
    P.x_row_stride = xrow;
    P.y_row_stride = yrow;
    P.total_rows = P.batch_shape[0] * P.batch_shape[1] * M;

    R->w_row = wq->stride[rw - 2];
    R->s_row = sc->stride[rw - 2];
    R->b_row = bi->stride[rw - 2];
    // x rows usable with 16-byte vector loads?
    bool xv = aligned16(x->data) && (M <= 1 || xrow % 8 == 0);
    for (int s = 0; s < 2; ++s)
        if (P.batch_shape[s] > 1 && P.x_batch_stride[s] % 8 != 0) xv = false;
    R->xvec = xv ? 1 : 0;

    // ---- regime ----
    R->mma_ok = false;
    R->mma_why = "forced GEMV";
    if (!force_qmv) {
        if (w_batched) R->mma_why = "batched weights take the GEMV kernel";
        else if (M <= 4) R->mma_why = "few rows per launch: GEMV";
        else if (K == 0 || N == 0) R->mma_why = "empty contraction";
        else {
            fill_mma_problem(x, wq, sc, bi, group, bits, y, R);
            aq::MmaProblem& mp = R->mp;
            // scales/biases rows must be contiguous for the tile loads
            if (R->s_row != K / group || R->b_row != K / group) R->mma_why = "scales/biases rows not contiguous";
            else R->mma_ok = aq::mma_supported(mp, &R->mma_why);
        }
    }
    P.regime = R->mma_ok ? AQ_REGIME_MMA : AQ_REGIME_QMV;
    P.kernel = R->mma_ok ? (int32_t)aq::mma_kernel_for(R->mp) : AQ_KERNEL_GEMV;
    P.y_tiles = R->mma_ok && aq::mma_y_tiles(R->mp) ? 1 : 0;
    return AQ_OK;
}

// The tensor-core problem of a resolved call (its plan already filled in).
void fill_mma_problem(const aq_view* x, const aq_view* wq, const aq_view* sc, const aq_view* bi, int group,
                      int bits, const aq_view* y, Resolved* R) {
    const aq_plan& P = R->plan;
    aq::MmaProblem& mp = R->mp;
    memset(&mp, 0, sizeof mp);
    mp.x = x->data;
    mp.y = y->data;
    mp.wq = (const uint32_t*)wq->data;
    mp.scales = sc->data;
    mp.biases = bi->data;
    mp.M = P.M;
    mp.N = P.N;
    mp.K = P.K;
    mp.x_row = P.x_row_stride;
    mp.y_row = P.y_row_stride;
    mp.nb[0] = P.batch_shape[0];
    mp.nb[1] = P.batch_shape[1];
    for (int s = 0; s < 2; ++s) { mp.xb[s] = P.x_batch_stride[s]; mp.yb[s] = P.y_batch_stride[s]; }
    mp.w_row = R->w_row;
    mp.group = group;
    mp.bits = bits;
    mp.xdt = (aq::DT)x->dtype;
    mp.ydt = (aq::DT)y->dtype;
    mp.offsets = nullptr;
}

aq_status run_linear(const aq_view* x, const aq_view* wq, const aq_view* sc, const aq_view* bi, int group,
                     int bits, const aq_view* y, void* stream, int force_qmv) {
    Resolved R;
    aq_status st = resolve_linear(x, wq, sc, bi, group, bits, y, force_qmv, &R);
    if (st != AQ_OK) return st;
    const aq_plan& P = R.plan;
    if (P.total_rows == 0 || P.N == 0) return AQ_OK;  // nothing to write
    if ((st = check_device()) != AQ_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (P.regime == AQ_REGIME_MMA) {
        e = aq::launch_mma(R.mp, s);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core kernel launch");
        return AQ_OK;
    }
    aq::QmvArgs a;
    memset(&a, 0, sizeof a);
    a.x = x->data;
    a.wq = (const uint32_t*)wq->data;
    a.scales = sc->data;
    a.biases = bi->data;
    a.y = y->data;
    a.x_row = P.x_row_stride;
    a.y_row = P.y_row_stride;
    a.w_row = R.w_row;
    a.s_row = R.s_row;
    a.b_row = R.b_row;
    a.M = P.M;
    a.N = P.N;
    a.K = P.K;
    a.log2g = log2i(group);
    a.xvec = R.xvec;
    a.bshape1 = P.batch_shape[1];
    for (int i = 0; i < 2; ++i) {
        a.xb[i] = P.x_batch_stride[i];
        a.yb[i] = P.y_batch_stride[i];
        a.wb[i] = P.w_batch_stride[i];
        a.sb[i] = P.s_batch_stride[i];
        a.bb[i] = P.b_batch_stride[i];
    }
    const int64_t nbatch = P.batch_shape[0] * P.batch_shape[1];
    if (nbatch > 65535) return fail(AQ_ERR_UNSUPPORTED, "more than 65535 launch batches");
    e = aq::launch_qmv(a, bits, (aq::DT)x->dtype, (aq::DT)y->dtype, nbatch, s);
    if (e != cudaSuccess) return cuda_fail(e, "GEMV kernel launch");
    return AQ_OK;
}

// ---------------------------------------------------------------------------
// fused calls on the warp-level kernel: several W sharing x, gate/up with silu, a residual
// ---------------------------------------------------------------------------

// Resolves matrix j of a fused call as a plain call and checks that it folds to one 2D problem
// (no launch batch dims, unbatched W) the warp-level kernel can take.
aq_status resolve_fused_part(const aq_view* x, const aq_view* wq, const aq_view* sc, const aq_view* bi, int group,
                             int bits, const aq_view* y, const char* what, Resolved* R, bool* warp_ok) {
    aq_status st = resolve_linear(x, wq, sc, bi, group, bits, y, 0, R);
    if (st != AQ_OK) return st;
    if (R->plan.nbatch_dims != 0 || R->plan.w_batched)
        return fail(AQ_ERR_UNSUPPORTED, "%s: x and y must fold into one 2D problem, with an unbatched W", what);
    fill_mma_problem(x, wq, sc, bi, group, bits, y, R);
    const char* why = nullptr;
    *warp_ok = R->plan.total_rows > 0 && R->plan.N > 0 && R->s_row == R->plan.K / group &&
               R->b_row == R->plan.K / group && aq::mma_supported(R->mp, &why) && aq::warp_mma_supported(R->mp);
    return AQ_OK;
}

aq_status launch_fused(aq::MmaProblem& mp, void* stream) {
    aq_status st = check_device();
    if (st != AQ_OK) return st;
    cudaError_t e = aq::launch_warp_mma(mp, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "fused warp-level kernel launch");
    return AQ_OK;
}

aq_status check_quant_views(const aq_view* w, int group, int bits, const aq_view* wq, const aq_view* sc,
                            const aq_view* bi, bool w_is_output) {
    aq_status st;
    if ((st = check_view(w, w_is_output ? "w_out" : "w", 2, 2)) != AQ_OK) return st;
    if ((st = check_view(wq, "wq", 2, 2)) != AQ_OK) return st;
    if ((st = check_view(sc, "scales", 2, 2)) != AQ_OK) return st;
    if ((st = check_view(bi, "biases", 2, 2)) != AQ_OK) return st;
    if ((st = check_bits_group(bits, group)) != AQ_OK) return st;
    if (!(w->dtype == AQ_F32 || is_half(w->dtype))) return fail(AQ_ERR_DTYPE, "w must be f32, bf16 or f16");
    if (wq->dtype != AQ_U32) return fail(AQ_ERR_DTYPE, "wq must be u32");
    if (!is_half(sc->dtype) || bi->dtype != sc->dtype)
        return fail(AQ_ERR_DTYPE, "scales/biases must be bf16 or f16 (same dtype)");
    const int64_t N = w->shape[0], K = w->shape[1];
    if (K % group != 0) return fail(AQ_ERR_GROUP, "K=%lld not a multiple of group=%d", (long long)K, group);
    if (wq->shape[0] != N || wq->shape[1] != K * bits / 32) return fail(AQ_ERR_SHAPE, "wq must be [N, K*bits/32]");
    if (sc->shape[0] != N || sc->shape[1] != K / group || bi->shape[0] != N || bi->shape[1] != K / group)
        return fail(AQ_ERR_SHAPE, "scales/biases must be [N, K/group]");
    if (numel(wq) > 0 && !aligned16(wq->data)) return fail(AQ_ERR_ALIGN, "wq data must be 16-byte aligned");
    const aq_view* out = w_is_output ? w : wq;
    const aq_view* ins[3] = {w_is_output ? wq : w, sc, bi};
    if (w_is_output) {
        if ((st = check_output(w, "w_out")) != AQ_OK) return st;
    } else {
        if ((st = check_output(wq, "wq")) != AQ_OK) return st;
        if ((st = check_output(sc, "scales")) != AQ_OK) return st;
        if ((st = check_output(bi, "biases")) != AQ_OK) return st;
    }
    if (w_is_output) {
        for (const aq_view* v : ins)
            if (overlaps(out, v)) return fail(AQ_ERR_OVERLAP, "w_out overlaps an input");
    } else {
        if (overlaps(wq, w) || overlaps(sc, w) || overlaps(bi, w) || overlaps(wq, sc) || overlaps(wq, bi) ||
            overlaps(sc, bi))
            return fail(AQ_ERR_OVERLAP, "quantize outputs overlap each other or the input");
    }
    return AQ_OK;
}

}  // namespace

// ===========================================================================
// exported C ABI
// ===========================================================================

AQ_API const char* aq_status_string(aq_status s) {
    switch (s) {
        case AQ_OK: return "AQ_OK";
        case AQ_ERR_NULL: return "AQ_ERR_NULL";
        case AQ_ERR_DTYPE: return "AQ_ERR_DTYPE";
        case AQ_ERR_RANK: return "AQ_ERR_RANK";
        case AQ_ERR_SHAPE: return "AQ_ERR_SHAPE";
        case AQ_ERR_STRIDE: return "AQ_ERR_STRIDE";
        case AQ_ERR_BITS: return "AQ_ERR_BITS";
        case AQ_ERR_GROUP: return "AQ_ERR_GROUP";
        case AQ_ERR_ALIGN: return "AQ_ERR_ALIGN";
        case AQ_ERR_UNSUPPORTED: return "AQ_ERR_UNSUPPORTED";
        case AQ_ERR_OVERLAP: return "AQ_ERR_OVERLAP";
        case AQ_ERR_CUDA: return "AQ_ERR_CUDA";
        case AQ_ERR_DEVICE: return "AQ_ERR_DEVICE";
        case AQ_ERR_TIMEOUT: return "AQ_ERR_TIMEOUT";
        case AQ_ERR_INDEX: return "AQ_ERR_INDEX";
    }
    return "AQ_ERR_UNKNOWN";
}

AQ_API const char* aq_last_error_message(void) { return g_msg; }

AQ_API int aq_version(void) { return 100; }

AQ_API aq_status aq_plan_linear(const aq_view* x, const aq_view* wq, const aq_view* scales,
                                const aq_view* biases, int group, int bits, const aq_view* y, int force_qmv,
                                aq_plan* out) {
    g_msg[0] = 0;
    if (!out) return fail(AQ_ERR_NULL, "plan output is NULL");
    Resolved R;
    aq_status st = resolve_linear(x, wq, scales, biases, group, bits, y, force_qmv, &R);
    if (st != AQ_OK) return st;
    *out = R.plan;
    if (R.plan.regime == AQ_REGIME_QMV && R.mma_why) snprintf(g_msg, sizeof g_msg, "%s", R.mma_why);
    return AQ_OK;
}

AQ_API aq_status aq_qmm_t(const aq_view* x, const aq_view* wq, const aq_view* scales, const aq_view* biases,
                          int group, int bits, const aq_view* y, void* stream) {
    g_msg[0] = 0;
    return run_linear(x, wq, scales, biases, group, bits, y, stream, 0);
}

AQ_API aq_status aq_qmv(const aq_view* x, const aq_view* wq, const aq_view* scales, const aq_view* biases,
                        int group, int bits, const aq_view* y, void* stream) {
    g_msg[0] = 0;
    return run_linear(x, wq, scales, biases, group, bits, y, stream, 1);
}

AQ_API aq_status aq_quantize(const aq_view* w, int group, int bits, const aq_view* wq, const aq_view* scales,
                             const aq_view* biases, void* stream) {
    g_msg[0] = 0;
    aq_status st = check_quant_views(w, group, bits, wq, scales, biases, false);
    if (st != AQ_OK) return st;
    if (numel(w) == 0) return AQ_OK;
    if ((st = check_device()) != AQ_OK) return st;
    aq::QuantArgs a;
    memset(&a, 0, sizeof a);
    a.w = w->data;
    a.wq = (uint32_t*)wq->data;
    a.scales = scales->data;
    a.biases = biases->data;
    a.w_row = w->stride[0];
    a.wq_row = wq->stride[0];
    a.s_row = scales->stride[0];
    a.b_row = biases->stride[0];
    a.N = w->shape[0];
    a.K = w->shape[1];
    a.group = group;
    a.bits = bits;
    cudaError_t e = aq::launch_quantize(a, (aq::DT)w->dtype, (aq::DT)scales->dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    return AQ_OK;
}

AQ_API aq_status aq_dequantize(const aq_view* wq, const aq_view* scales, const aq_view* biases, int group,
                               int bits, const aq_view* w_out, void* stream) {
    g_msg[0] = 0;
    aq_status st = check_quant_views(w_out, group, bits, wq, scales, biases, true);
    if (st != AQ_OK) return st;
    if (numel(w_out) == 0) return AQ_OK;
    if ((st = check_device()) != AQ_OK) return st;
    aq::QuantArgs a;
    memset(&a, 0, sizeof a);
    a.w = w_out->data;
    a.wq = (uint32_t*)wq->data;
    a.scales = scales->data;
    a.biases = biases->data;
    a.w_row = w_out->stride[0];
    a.wq_row = wq->stride[0];
    a.s_row = scales->stride[0];
    a.b_row = biases->stride[0];
    a.N = w_out->shape[0];
    a.K = w_out->shape[1];
    a.group = group;
    a.bits = bits;
    cudaError_t e = aq::launch_dequantize(a, (aq::DT)w_out->dtype, (aq::DT)scales->dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
    return AQ_OK;
}

AQ_API aq_status aq_qmm_t_grouped(const aq_view* x_sorted, const int64_t* offsets, int n_experts,
                                  const aq_view* wq_bank, const aq_view* s_bank, const aq_view* b_bank, int group,
                                  int bits, const aq_view* y_sorted, void* stream) {
    g_msg[0] = 0;
    aq_status st;
    if ((st = check_view(x_sorted, "x_sorted", 2, 2)) != AQ_OK) return st;
    if ((st = check_view(wq_bank, "wq_bank", 3, 3)) != AQ_OK) return st;
    if ((st = check_view(s_bank, "s_bank", 3, 3)) != AQ_OK) return st;
    if ((st = check_view(b_bank, "b_bank", 3, 3)) != AQ_OK) return st;
    if ((st = check_view(y_sorted, "y_sorted", 2, 2)) != AQ_OK) return st;
    if ((st = check_output(y_sorted, "y_sorted")) != AQ_OK) return st;
    if ((st = check_bits_group(bits, group)) != AQ_OK) return st;
    if (!offsets) return fail(AQ_ERR_NULL, "offsets is NULL");
    if (n_experts <= 0 || wq_bank->shape[0] != n_experts || s_bank->shape[0] != n_experts ||
        b_bank->shape[0] != n_experts)
        return fail(AQ_ERR_SHAPE, "bank leading dim must equal n_experts");
    if (!is_half(x_sorted->dtype)) return fail(AQ_ERR_DTYPE, "x_sorted must be bf16 or f16");
    if (wq_bank->dtype != AQ_U32) return fail(AQ_ERR_DTYPE, "wq_bank must be u32");
    if (s_bank->dtype != x_sorted->dtype || b_bank->dtype != x_sorted->dtype)
        return fail(AQ_ERR_DTYPE, "scale/bias banks must have x's dtype");
    if (y_sorted->dtype != x_sorted->dtype && y_sorted->dtype != AQ_F32)
        return fail(AQ_ERR_DTYPE, "y_sorted must have x's dtype or f32");
    const int64_t T = x_sorted->shape[0], K = x_sorted->shape[1], N = wq_bank->shape[1];
    if (K % group != 0) return fail(AQ_ERR_GROUP, "K not a multiple of group");
    if (wq_bank->shape[2] != K * bits / 32) return fail(AQ_ERR_SHAPE, "wq_bank last dim must be K*bits/32");
    if (s_bank->shape[1] != N || b_bank->shape[1] != N || s_bank->shape[2] != K / group ||
        b_bank->shape[2] != K / group)
        return fail(AQ_ERR_SHAPE, "scale/bias banks must be [E, N, K/group]");
    if (y_sorted->shape[0] != T || y_sorted->shape[1] != N) return fail(AQ_ERR_SHAPE, "y_sorted must be [T, N]");
    if (numel(wq_bank) > 0 && !aligned16(wq_bank->data)) return fail(AQ_ERR_ALIGN, "wq_bank must be 16-byte aligned");
    if (overlaps(y_sorted, x_sorted) || overlaps(y_sorted, wq_bank) || overlaps(y_sorted, s_bank) ||
        overlaps(y_sorted, b_bank))
        return fail(AQ_ERR_OVERLAP, "y_sorted overlaps an input");
    if (T == 0 || N == 0) return AQ_OK;
    if ((st = check_device()) != AQ_OK) return st;
    aq::MmaProblem mp;
    memset(&mp, 0, sizeof mp);
    mp.x = x_sorted->data;
    mp.y = y_sorted->data;
    mp.wq = (const uint32_t*)wq_bank->data;
    mp.scales = s_bank->data;
    mp.biases = b_bank->data;
    mp.M = T;
    mp.N = N;
    mp.K = K;
    mp.x_row = x_sorted->stride[0];
    mp.y_row = y_sorted->stride[0];
    mp.nb[0] = mp.nb[1] = 1;
    mp.w_row = wq_bank->stride[1];
    mp.group = group;
    mp.bits = bits;
    mp.xdt = (aq::DT)x_sorted->dtype;
    mp.ydt = (aq::DT)y_sorted->dtype;
    mp.offsets = offsets;
    mp.n_experts = n_experts;
    mp.w_expert = wq_bank->stride[0];
    mp.s_expert = s_bank->stride[0];
    mp.b_expert = b_bank->stride[0];
    if (s_bank->stride[1] != K / group || b_bank->stride[1] != K / group)
        return fail(AQ_ERR_UNSUPPORTED, "scale/bias bank rows must be contiguous");
    const char* why = nullptr;
    if (!aq::mma_supported(mp, &why)) return fail(AQ_ERR_UNSUPPORTED, "grouped kernel: %s", why);
    cudaError_t e = aq::launch_mma(mp, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "grouped kernel launch");
    return AQ_OK;
}

AQ_API aq_status aq_device_error(void* stream) {
    g_msg[0] = 0;
    int v = 0;
    cudaError_t e = aq::read_and_clear_device_error(&v, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (v & aq::DEVERR_TIMEOUT) {
        static const struct { int bit; const char* name; } at[] = {
            {aq::DEVERR_AT_WARP_X, "warp-level kernel x staging"}, {aq::DEVERR_AT_WARP_SB, "warp-level kernel scale/bias staging"},
            {aq::DEVERR_AT_WARP_W, "warp-level kernel W ring"},
            {aq::DEVERR_AT_TC_WFREE, "small-M W producer (expanders)"}, {aq::DEVERR_AT_TC_XFREE, "small-M x producer (MMA commit)"},
            {aq::DEVERR_AT_TC_XFULL, "small-M MMA issuer (x copy)"}, {aq::DEVERR_AT_TC_AFULL, "small-M MMA issuer (expanders)"},
            {aq::DEVERR_AT_TC_DFREE, "small-M MMA issuer (folds)"}, {aq::DEVERR_AT_TC_WFULL, "small-M expanders (W copy)"},
            {aq::DEVERR_AT_TC_SDONE_E, "small-M expanders (MMA commit)"}, {aq::DEVERR_AT_TC_SDONE_F, "small-M folds (MMA commit)"},
            {aq::DEVERR_AT_TC_FOLD, "small-M folds (folds, x or cluster)"},
            {aq::DEVERR_AT_PF_W, "prefill W producer"}, {aq::DEVERR_AT_PF_X, "prefill x producer"},
            {aq::DEVERR_AT_PF_MMA, "prefill MMA issuer"}, {aq::DEVERR_AT_PF_EXP, "prefill expanders"},
            {aq::DEVERR_AT_PF_FOLD, "prefill folds"}, {aq::DEVERR_AT_CHECK, "bounded-wait self-check"}};
        char where[480];
        where[0] = 0;
        for (const auto& a : at)
            if (v & a.bit) {
                if (where[0]) strncat(where, ", ", sizeof where - strlen(where) - 1);
                strncat(where, a.name, sizeof where - strlen(where) - 1);
            }
        return fail(AQ_ERR_TIMEOUT, "a kernel's bounded wait expired (code %d; at: %s)", v, where[0] ? where : "unrecorded");
    }
    if (v & aq::DEVERR_INDEX) return fail(AQ_ERR_INDEX, "a row id was outside the table (code %d)", v);
    if (v != 0) return fail(AQ_ERR_CUDA, "unknown device error code %d", v);
    return AQ_OK;
}

AQ_API aq_status aq_qmm_t_multi(const aq_view* x, int n, const aq_view* const* wq, const aq_view* const* scales,
                                const aq_view* const* biases, int group, int bits, float rms_eps,
                                const aq_view* const* y, void* stream) {
    g_msg[0] = 0;
    if (n < 1 || n > 3) return fail(AQ_ERR_UNSUPPORTED, "n=%d matrices (1..3 supported)", n);
    if (!(rms_eps >= 0.0f)) return fail(AQ_ERR_SHAPE, "rms_eps must be >= 0");
    if (!wq || !scales || !biases || !y) return fail(AQ_ERR_NULL, "NULL array of views");
    Resolved R[3];
    bool all_warp = true;
    for (int j = 0; j < n; ++j) {
        aq_status st = resolve_linear(x, wq[j], scales[j], biases[j], group, bits, y[j], 0, &R[j]);
        if (st != AQ_OK) return st;
    }
    // no output may overlap another output or another matrix's inputs
    for (int j = 0; j < n; ++j)
        for (int k = 0; k < n; ++k) {
            if (j == k) continue;
            if (overlaps(y[j], y[k]) || overlaps(y[j], wq[k]) || overlaps(y[j], scales[k]) || overlaps(y[j], biases[k]))
                return fail(AQ_ERR_OVERLAP, "y[%d] overlaps an input or output of matrix %d", j, k);
        }
    if (R[0].plan.total_rows == 0) return AQ_OK;
    for (int j = 0; j < n && all_warp; ++j) {
        bool ok = false;
        aq_status st = resolve_fused_part(x, wq[j], scales[j], biases[j], group, bits, y[j], "aq_qmm_t_multi", &R[j],
                                          &ok);
        if (st != AQ_OK) ok = false;
        all_warp = ok && R[j].plan.M == R[0].plan.M && R[j].plan.x_row_stride == R[0].plan.x_row_stride;
    }
    if (rms_eps > 0.0f && !all_warp)
        return fail(AQ_ERR_UNSUPPORTED, "an RMS-normalised input needs the warp-level kernel (up to 32 rows, "
                                        "2/4/8-bit codes, 16-byte aligned rows)");
    if (!all_warp || (n == 1 && rms_eps == 0.0f)) {
        // one plain call per matrix, in order, on the same stream
        for (int j = 0; j < n; ++j) {
            aq_status st = run_linear(x, wq[j], scales[j], biases[j], group, bits, y[j], stream, 0);
            if (st != AQ_OK) return st;
        }
        return AQ_OK;
    }
    aq::MmaProblem mp = R[0].mp;
    mp.nseg = n;
    mp.rms_eps = rms_eps;
    for (int j = 0; j < n; ++j) {
        mp.seg_wq[j] = R[j].mp.wq;
        mp.seg_scales[j] = R[j].mp.scales;
        mp.seg_biases[j] = R[j].mp.biases;
        mp.seg_y[j] = R[j].mp.y;
        mp.seg_N[j] = R[j].mp.N;
        mp.seg_w_row[j] = R[j].mp.w_row;
        mp.seg_y_row[j] = R[j].mp.y_row;
    }
    if (!aq::warp_mma_supported(mp)) return fail(AQ_ERR_UNSUPPORTED, "fused projections: too many row blocks");
    return launch_fused(mp, stream);
}

AQ_API aq_status aq_qmm_t_swiglu(const aq_view* x, const aq_view* wq_gate, const aq_view* s_gate,
                                 const aq_view* b_gate, const aq_view* wq_up, const aq_view* s_up,
                                 const aq_view* b_up, int group, int bits, float rms_eps, const aq_view* y,
                                 void* stream) {
    g_msg[0] = 0;
    if (!(rms_eps >= 0.0f)) return fail(AQ_ERR_SHAPE, "rms_eps must be >= 0");
    Resolved Rg, Ru;
    bool okg = false, oku = false;
    aq_status st = resolve_fused_part(x, wq_gate, s_gate, b_gate, group, bits, y, "aq_qmm_t_swiglu", &Rg, &okg);
    if (st != AQ_OK) return st;
    st = resolve_fused_part(x, wq_up, s_up, b_up, group, bits, y, "aq_qmm_t_swiglu", &Ru, &oku);
    if (st != AQ_OK) return st;
    if (Ru.plan.N != Rg.plan.N) return fail(AQ_ERR_SHAPE, "gate and up matrices must have the same N");
    if (Rg.plan.total_rows == 0 || Rg.plan.N == 0) return AQ_OK;
    if (!okg || !oku)
        return fail(AQ_ERR_UNSUPPORTED,
                    "aq_qmm_t_swiglu runs on the warp-level kernel only (up to 32 rows, 2/4/8-bit codes, "
                    "16-byte aligned rows)");
    aq::MmaProblem mp = Rg.mp;
    mp.nseg = 2;
    mp.glu = 1;
    mp.rms_eps = rms_eps;
    const Resolved* parts[2] = {&Rg, &Ru};
    for (int j = 0; j < 2; ++j) {
        mp.seg_wq[j] = parts[j]->mp.wq;
        mp.seg_scales[j] = parts[j]->mp.scales;
        mp.seg_biases[j] = parts[j]->mp.biases;
        mp.seg_y[j] = Rg.mp.y;
        mp.seg_N[j] = parts[j]->mp.N;
        mp.seg_w_row[j] = parts[j]->mp.w_row;
        mp.seg_y_row[j] = Rg.mp.y_row;
    }
    if (!aq::warp_mma_supported(mp)) return fail(AQ_ERR_UNSUPPORTED, "gate/up: too many row blocks");
    return launch_fused(mp, stream);
}

AQ_API aq_status aq_qmm_t_residual(const aq_view* x, const aq_view* wq, const aq_view* scales,
                                   const aq_view* biases, int group, int bits, const aq_view* r, const aq_view* y,
                                   void* stream) {
    g_msg[0] = 0;
    Resolved R, Rr;
    bool ok = false, okr = false;
    aq_status st = resolve_fused_part(x, wq, scales, biases, group, bits, y, "aq_qmm_t_residual", &R, &ok);
    if (st != AQ_OK) return st;
    if ((st = check_view(r, "r", 1, 4)) != AQ_OK) return st;
    if (r->dtype != y->dtype) return fail(AQ_ERR_DTYPE, "r must have y's dtype");
    // r has y's shape and folds the same way; it is read as an input, so it may be y itself
    // (the same view: each element is read and then written by the same thread) but must not
    // overlap y otherwise, nor the other inputs
    const bool same = r->data == y->data && r->rank == y->rank &&
                      memcmp(r->shape, y->shape, sizeof(int64_t) * y->rank) == 0 &&
                      memcmp(r->stride, y->stride, sizeof(int64_t) * y->rank) == 0;
    if (!same) {
        st = resolve_fused_part(x, wq, scales, biases, group, bits, r, "aq_qmm_t_residual (r)", &Rr, &okr);
        if (st != AQ_OK) return st;
        if (overlaps(r, y)) return fail(AQ_ERR_OVERLAP, "r overlaps y (other than being the same view)");
    } else {
        Rr = R;
    }
    if (R.plan.total_rows == 0 || R.plan.N == 0) return AQ_OK;
    if (!ok)
        return fail(AQ_ERR_UNSUPPORTED,
                    "aq_qmm_t_residual runs on the warp-level kernel only (up to 32 rows, 2/4/8-bit codes, "
                    "16-byte aligned rows)");
    aq::MmaProblem mp = R.mp;
    mp.r = r->data;
    mp.r_row = Rr.plan.y_row_stride;
    return launch_fused(mp, stream);
}

AQ_API aq_status aq_dequantize_rows(const aq_view* wq, const aq_view* scales, const aq_view* biases, int group,
                                    int bits, const int64_t* ids, int64_t n_ids, const aq_view* out,
                                    void* stream) {
    g_msg[0] = 0;
    aq_status st;
    if ((st = check_view(out, "out", 2, 2)) != AQ_OK) return st;
    if (n_ids < 0) return fail(AQ_ERR_SHAPE, "n_ids < 0");
    if (out->shape[0] != n_ids) return fail(AQ_ERR_SHAPE, "out must have n_ids rows");
    if ((st = check_output(out, "out")) != AQ_OK) return st;
    if ((st = check_view(wq, "wq", 2, 2)) != AQ_OK) return st;
    if ((st = check_view(scales, "scales", 2, 2)) != AQ_OK) return st;
    if ((st = check_view(biases, "biases", 2, 2)) != AQ_OK) return st;
    if ((st = check_bits_group(bits, group)) != AQ_OK) return st;
    if (!(out->dtype == AQ_F32 || is_half(out->dtype))) return fail(AQ_ERR_DTYPE, "out must be f32, bf16 or f16");
    if (wq->dtype != AQ_U32) return fail(AQ_ERR_DTYPE, "wq must be u32");
    if (!is_half(scales->dtype) || biases->dtype != scales->dtype)
        return fail(AQ_ERR_DTYPE, "scales/biases must be bf16 or f16 (same dtype)");
    const int64_t V = wq->shape[0], K = out->shape[1];
    if (K % group != 0) return fail(AQ_ERR_GROUP, "K=%lld not a multiple of group=%d", (long long)K, group);
    if (wq->shape[1] != K * bits / 32) return fail(AQ_ERR_SHAPE, "wq must be [V, K*bits/32]");
    if (scales->shape[0] != V || scales->shape[1] != K / group || biases->shape[0] != V ||
        biases->shape[1] != K / group)
        return fail(AQ_ERR_SHAPE, "scales/biases must be [V, K/group]");
    if (numel(wq) > 0 && !aligned16(wq->data)) return fail(AQ_ERR_ALIGN, "wq data must be 16-byte aligned");
    if (overlaps(out, wq) || overlaps(out, scales) || overlaps(out, biases))
        return fail(AQ_ERR_OVERLAP, "out overlaps the table");
    if (n_ids == 0 || out->shape[1] == 0) return AQ_OK;
    if (!ids) return fail(AQ_ERR_NULL, "ids is NULL");
    if ((st = check_device()) != AQ_OK) return st;
    aq::QuantArgs a;
    memset(&a, 0, sizeof a);
    a.w = out->data;
    a.wq = (uint32_t*)wq->data;
    a.scales = scales->data;
    a.biases = biases->data;
    a.w_row = out->stride[0];
    a.wq_row = wq->stride[0];
    a.s_row = scales->stride[0];
    a.b_row = biases->stride[0];
    a.N = n_ids;
    a.K = out->shape[1];
    a.group = group;
    a.bits = bits;
    a.ids = ids;
    a.V = wq->shape[0];
    cudaError_t e = aq::device_error_ptr(&a.err);
    if (e != cudaSuccess) return cuda_fail(e, "device error word");
    e = aq::launch_dequantize(a, (aq::DT)out->dtype, (aq::DT)scales->dtype, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "row gather launch");
    return AQ_OK;
}

AQ_API aq_status aq_qmv_gathered(const aq_view* x, const int64_t* x_ids, const int64_t* w_ids, int64_t n_rows,
                                 const aq_view* wq_bank, const aq_view* s_bank, const aq_view* b_bank, int group,
                                 int bits, const aq_view* y, void* stream) {
    g_msg[0] = 0;
    aq_status st;
    if ((st = check_view(x, "x", 2, 2)) != AQ_OK) return st;
    if ((st = check_view(wq_bank, "wq_bank", 3, 3)) != AQ_OK) return st;
    if ((st = check_view(s_bank, "s_bank", 3, 3)) != AQ_OK) return st;
    if ((st = check_view(b_bank, "b_bank", 3, 3)) != AQ_OK) return st;
    if ((st = check_view(y, "y", 2, 2)) != AQ_OK) return st;
    if ((st = check_output(y, "y")) != AQ_OK) return st;
    if ((st = check_bits_group(bits, group)) != AQ_OK) return st;
    if (!is_half(x->dtype)) return fail(AQ_ERR_DTYPE, "x must be bf16 or f16");
    if (wq_bank->dtype != AQ_U32) return fail(AQ_ERR_DTYPE, "wq_bank must be u32");
    if (s_bank->dtype != x->dtype || b_bank->dtype != x->dtype)
        return fail(AQ_ERR_DTYPE, "scale/bias banks must have x's dtype");
    if (y->dtype != x->dtype && y->dtype != AQ_F32) return fail(AQ_ERR_DTYPE, "y must have x's dtype or f32");
    const int64_t T = x->shape[0], K = x->shape[1], E = wq_bank->shape[0], N = wq_bank->shape[1];
    if (n_rows < 0) return fail(AQ_ERR_SHAPE, "n_rows < 0");
    if (K % group != 0) return fail(AQ_ERR_GROUP, "K not a multiple of group");
    if (wq_bank->shape[2] != K * bits / 32) return fail(AQ_ERR_SHAPE, "wq_bank last dim must be K*bits/32");
    if (s_bank->shape[0] != E || b_bank->shape[0] != E || s_bank->shape[1] != N || b_bank->shape[1] != N ||
        s_bank->shape[2] != K / group || b_bank->shape[2] != K / group)
        return fail(AQ_ERR_SHAPE, "scale/bias banks must be [E, N, K/group]");
    if (y->shape[0] != n_rows || y->shape[1] != N) return fail(AQ_ERR_SHAPE, "y must be [n_rows, N]");
    if (numel(wq_bank) > 0) {
        const int64_t need = (bits == 4 || bits == 8) ? 4 : (bits == 2 || bits == 6) ? 2 : 1;  // words
        if (!aligned16(wq_bank->data) || wq_bank->stride[0] % need != 0 || (N > 1 && wq_bank->stride[1] % need != 0))
            return fail(AQ_ERR_ALIGN, "wq_bank rows must be %lld-byte aligned", (long long)(need * 4));
    }
    if (overlaps(y, x) || overlaps(y, wq_bank) || overlaps(y, s_bank) || overlaps(y, b_bank))
        return fail(AQ_ERR_OVERLAP, "y overlaps an input");
    if (n_rows == 0 || N == 0) return AQ_OK;
    if (!x_ids || !w_ids) return fail(AQ_ERR_NULL, "x_ids / w_ids is NULL");
    if (n_rows > 65535) return fail(AQ_ERR_UNSUPPORTED, "more than 65535 gathered rows per call");
    if ((st = check_device()) != AQ_OK) return st;
    aq::QmvArgs a;
    memset(&a, 0, sizeof a);
    a.x = x->data;
    a.wq = (const uint32_t*)wq_bank->data;
    a.scales = s_bank->data;
    a.biases = b_bank->data;
    a.y = y->data;
    a.x_row = x->stride[0];
    a.y_row = y->stride[0];
    a.w_row = wq_bank->stride[1];
    a.s_row = s_bank->stride[1];
    a.b_row = b_bank->stride[1];
    a.M = 1;
    a.N = N;
    a.K = K;
    a.log2g = log2i(group);
    a.xvec = (aligned16(x->data) && (T <= 1 || x->stride[0] % 8 == 0)) ? 1 : 0;
    a.bshape1 = 1;
    a.xb[0] = x->stride[0];
    a.yb[0] = y->stride[0];
    a.wb[0] = wq_bank->stride[0];
    a.sb[0] = s_bank->stride[0];
    a.bb[0] = b_bank->stride[0];
    a.x_ids = x_ids;
    a.w_ids = w_ids;
    a.x_rows = T;
    a.w_entries = E;
    cudaError_t e = aq::device_error_ptr(&a.err);
    if (e != cudaSuccess) return cuda_fail(e, "device error word");
    e = aq::launch_qmv(a, bits, (aq::DT)x->dtype, (aq::DT)y->dtype, n_rows, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gathered GEMV launch");
    return AQ_OK;
}

AQ_API aq_status aq_check_bounded_wait(uint64_t budget_ns, void* stream) {
    g_msg[0] = 0;
    if (budget_ns == 0 || budget_ns > 1000000000ull) return fail(AQ_ERR_SHAPE, "budget_ns must be in (0, 1e9]");
    aq_status st = check_device();
    if (st != AQ_OK) return st;
    cudaError_t e = aq::launch_bounded_wait_check(budget_ns, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "bounded-wait check launch");
    return AQ_OK;
}
