// kernels_qmv.cu -- CUDA-core GEMV for a handful of rows of x.
//
// What it computes (per output y[m, n]), in fp32:
//     y = sum_g  s[n,g] * sum_{k in g} q[n,k] * x[m,k]  +  b[n,g] * sum_{k in g} x[m,k]
// the factored form of x . (s*q + b)^T.  Following "mlx PR #4516"
// (load_vector fix) every x element is widened to fp32 BEFORE it enters any
// sum, so the bias term b * sum(x) is exact whenever the exact sum is
// representable in fp32.
//
// Layout of the work: a warp owns RPW (4, or 1 when N is so small that 4 would leave most SMs
// idle) consecutive rows of W; lane l walks
// the 32-code chunks l, l+32, l+64, ... of those rows (a chunk is `bits`
// consecutive uint32 words, read with the widest aligned vector load: 16-byte
// for 4/8-bit, 8-byte for 2/6-bit, 4-byte for 3/5-bit), reuses each x chunk
// for its 4 rows, and the partial sums meet in a warp-shuffle reduction.
//
// Partial-rows tail (mlx PR #4516, affine_qmv_fast_rows): rows of the last
// warp that fall past N are clamped to row N-1 for their loads and skip only
// the final store, so the reduction loop carries no per-row bounds check.
//
// Code-to-float trick: a code q (< 2^7, or < 2^8 for 8-bit) is OR-ed into the
// mantissa of the fp32 constant 128 (256), giving exactly 128+q (256+q) with
// one shift and one LOP3; the products (128+q)*x are exact in fp32 and the
// offset is removed once per chunk through (b - 128*s) * sum(x).
#include <cuda_runtime.h>

#include <type_traits>
#include <utility>

#include "aq_internal.h"
#include "device_common.cuh"

namespace aq {
namespace {

constexpr int QMV_THREADS = 256;
constexpr int QMV_WARPS = QMV_THREADS / 32;

// 128 + q  (bits <= 7) or 256 + q (bits == 8), as fp32 bit patterns
template <int BITS> struct Magic {
    static constexpr int POS = BITS == 8 ? 15 : 16;                 // mantissa bit that holds q's LSB
    static constexpr uint32_t BASEBITS = BITS == 8 ? 0x43800000u : 0x43000000u;
    static constexpr float BASE = BITS == 8 ? 256.0f : 128.0f;
    static constexpr uint32_t MASK = ((1u << BITS) - 1u) << POS;
};

// Code i (0..31) of a chunk held in `w[0..BITS)`, returned as the float (BASE + q).
template <int BITS, int I>
__device__ __forceinline__ float code_as_float(const uint32_t* w) {
    constexpr int P = I * BITS;          // stream bit of the code's LSB
    constexpr int WI = P / 32, SH = P % 32;
    constexpr int T = Magic<BITS>::POS;
    uint32_t t;
    if constexpr (SH + BITS > 32) {      // straddles two words
        t = __funnelshift_r(w[WI], w[WI + 1], SH - T);
    } else if constexpr (SH > T) {
        t = w[WI] >> (SH - T);
    } else if constexpr (SH < T) {
        t = w[WI] << (T - SH);
    } else {
        t = w[WI];
    }
    return __uint_as_float((t & Magic<BITS>::MASK) | Magic<BITS>::BASEBITS);
}

template <int BITS>
__device__ __forceinline__ void load_chunk(const uint32_t* p, uint32_t* w) {
    if constexpr (BITS % 4 == 0) {
#pragma unroll
        for (int i = 0; i < BITS / 4; ++i) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else if constexpr (BITS % 2 == 0) {
#pragma unroll
        for (int i = 0; i < BITS / 2; ++i) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(p) + i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = __ldg(p + i);
    }
}

template <typename XT>
__device__ __forceinline__ void load_x8(const XT* p, int vec, float* f) {
    if (vec) {
        unpack8(__ldg(reinterpret_cast<const uint4*>(p)), f, XT{});
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = to_float<XT>(p + j);
    }
}

// P[r][t] += (BASE + q[r][I0+J]) * x[t][J] for the 8 codes I0..I0+7 of every row r
template <int BITS, int TOK, int RPW, int I0, int... J>
__device__ __forceinline__ void fma_codes(const uint32_t (&wv)[RPW][BITS + 1], const float (&xf)[TOK][8],
                                          float (&P)[RPW][TOK], std::integer_sequence<int, J...>) {
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        (
            [&] {
                const float v = code_as_float<BITS, I0 + J>(wv[r]);
#pragma unroll
                for (int t = 0; t < TOK; ++t) P[r][t] = fmaf(v, xf[t][J], P[r][t]);
            }(),
            ...);
    }
}

template <int BITS, int TOK, int RPW, typename XT, typename YT>
__global__ void __launch_bounds__(QMV_THREADS) qmv_kernel(const __grid_constant__ QmvArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = ((int64_t)blockIdx.x * QMV_WARPS + warp) * RPW;
    if (n0 >= a.N) return;
    const int64_t bidx = blockIdx.y;
    int64_t b1 = bidx % a.bshape1, b0 = bidx / a.bshape1;
    int64_t xo = b0 * a.xb[0] + b1 * a.xb[1], wo = b0 * a.wb[0] + b1 * a.wb[1];
    int64_t so = b0 * a.sb[0] + b1 * a.sb[1], bo = b0 * a.bb[0] + b1 * a.bb[1];
    if (a.x_ids) {
        // gathered row bidx: x row and W bank entry from the device id arrays (read once per warp)
        const int64_t xi = a.x_ids[bidx], wi = a.w_ids[bidx];
        if (xi < 0 || xi >= a.x_rows || wi < 0 || wi >= a.w_entries) {
            if (lane < RPW && n0 + lane < a.N) store_out((YT*)a.y + bidx * a.yb[0] + n0 + lane, 0.0f);
            if (lane == 0 && n0 == 0) atomicOr(a.err, DEVERR_INDEX);
            return;
        }
        xo = xi * a.xb[0];
        wo = wi * a.wb[0];
        so = wi * a.sb[0];
        bo = wi * a.bb[0];
        b0 = bidx;
        b1 = 0;
    }

    const XT* xbase = (const XT*)a.x + xo;
    YT* ybase = (YT*)a.y + b0 * a.yb[0] + b1 * a.yb[1];
    const uint32_t* wbase = a.wq + wo;
    const XT* sbase = (const XT*)a.scales + so;
    const XT* bbase = (const XT*)a.biases + bo;

    int64_t nrow[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) nrow[r] = min(n0 + r, a.N - 1);  // partial-rows tail: clamp, store later

    const int nchunks = (int)(a.K >> 5);
    const int log2g = a.log2g;
    constexpr float BASE = Magic<BITS>::BASE;

    for (int64_t m0 = 0; m0 < a.M; m0 += TOK) {
        const XT* xrow[TOK];
#pragma unroll
        for (int t = 0; t < TOK; ++t) xrow[t] = xbase + min(m0 + t, a.M - 1) * a.x_row;

        float acc[RPW][TOK];
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int t = 0; t < TOK; ++t) acc[r][t] = 0.0f;

        for (int c = lane; c < nchunks; c += 32) {
            uint32_t wv[RPW][BITS + 1];
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
                load_chunk<BITS>(wbase + nrow[r] * a.w_row + (int64_t)c * BITS, wv[r]);
                wv[r][BITS] = 0;
            }
            const int g = (c << 5) >> log2g;
            float s[RPW], bb[RPW];
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
                s[r] = to_float<XT>(sbase + nrow[r] * a.s_row + g);
                const float b = to_float<XT>(bbase + nrow[r] * a.b_row + g);
                bb[r] = fmaf(-BASE, s[r], b);  // b - BASE*s: removes the code offset
            }
            float P[RPW][TOK], X[TOK];
#pragma unroll
            for (int t = 0; t < TOK; ++t) {
                X[t] = 0.0f;
#pragma unroll
                for (int r = 0; r < RPW; ++r) P[r][t] = 0.0f;
            }
            auto do_sub = [&](auto sub_c) {
                constexpr int SUB = decltype(sub_c)::value;
                float xf[TOK][8];
#pragma unroll
                for (int t = 0; t < TOK; ++t) {
                    load_x8<XT>(xrow[t] + (c << 5) + SUB * 8, a.xvec, xf[t]);
#pragma unroll
                    for (int j = 0; j < 8; ++j) X[t] += xf[t][j];  // widened before summing
                }
                fma_codes<BITS, TOK, RPW, SUB * 8>(wv, xf, P, std::make_integer_sequence<int, 8>{});
            };
            do_sub(std::integral_constant<int, 0>{});
            do_sub(std::integral_constant<int, 1>{});
            do_sub(std::integral_constant<int, 2>{});
            do_sub(std::integral_constant<int, 3>{});
#pragma unroll
            for (int r = 0; r < RPW; ++r)
#pragma unroll
                for (int t = 0; t < TOK; ++t) acc[r][t] = fmaf(s[r], P[r][t], fmaf(bb[r], X[t], acc[r][t]));
        }

#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int t = 0; t < TOK; ++t) acc[r][t] = warp_sum(acc[r][t]);

        // lane (r*TOK + t) stores y[m0+t, n0+r]
        float mine = 0.0f;
#pragma unroll
        for (int r = 0; r < RPW; ++r)
#pragma unroll
            for (int t = 0; t < TOK; ++t)
                if (lane == r * TOK + t) mine = acc[r][t];
        if (lane < RPW * TOK) {
            const int r = lane / TOK, t = lane % TOK;
            const int64_t n = n0 + r, m = m0 + t;
            if (n < a.N && m < a.M) store_out(ybase + m * a.y_row + n, mine);
        }
    }
}

template <int BITS, int TOK, int RPW, typename XT, typename YT>
cudaError_t launch_t(const QmvArgs& a, int64_t nbatch, cudaStream_t s) {
    const int64_t rows_per_cta = QMV_WARPS * RPW;
    const dim3 grid((unsigned)((a.N + rows_per_cta - 1) / rows_per_cta), (unsigned)nbatch);
    qmv_kernel<BITS, TOK, RPW, XT, YT><<<grid, QMV_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

// one W row per warp while 4 per warp would leave most SMs idle (under 64 CTAs); above that
// the four rows' reuse of each x chunk matters more than the extra warps
template <int BITS, int TOK, typename XT, typename YT>
cudaError_t launch_rpw(const QmvArgs& a, int64_t nbatch, cudaStream_t s) {
    if ((a.N + QMV_WARPS * 4 - 1) / (QMV_WARPS * 4) * nbatch < 64) return launch_t<BITS, TOK, 1, XT, YT>(a, nbatch, s);
    return launch_t<BITS, TOK, 4, XT, YT>(a, nbatch, s);
}

template <int BITS, typename XT, typename YT>
cudaError_t launch_tok(const QmvArgs& a, int64_t nbatch, cudaStream_t s) {
    if (a.M == 1) return launch_rpw<BITS, 1, XT, YT>(a, nbatch, s);
    if (a.M == 2) return launch_rpw<BITS, 2, XT, YT>(a, nbatch, s);
    return launch_rpw<BITS, 4, XT, YT>(a, nbatch, s);
}

template <typename XT, typename YT>
cudaError_t launch_bits(const QmvArgs& a, int bits, int64_t nbatch, cudaStream_t s) {
    switch (bits) {
        case 2: return launch_tok<2, XT, YT>(a, nbatch, s);
        case 3: return launch_tok<3, XT, YT>(a, nbatch, s);
        case 4: return launch_tok<4, XT, YT>(a, nbatch, s);
        case 5: return launch_tok<5, XT, YT>(a, nbatch, s);
        case 6: return launch_tok<6, XT, YT>(a, nbatch, s);
        case 8: return launch_tok<8, XT, YT>(a, nbatch, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_qmv(const QmvArgs& a, int bits, DT xdt, DT ydt, int64_t nbatch, cudaStream_t s) {
    if (xdt == DT::BF16) {
        return ydt == DT::F32 ? launch_bits<bf16_t, float>(a, bits, nbatch, s)
                              : launch_bits<bf16_t, bf16_t>(a, bits, nbatch, s);
    }
    return ydt == DT::F32 ? launch_bits<f16_t, float>(a, bits, nbatch, s)
                          : launch_bits<f16_t, f16_t>(a, bits, nbatch, s);
}

}  // namespace aq
