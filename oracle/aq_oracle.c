/*
 * aq_oracle.c -- plain, slow, obviously correct CPU oracle for the affine
 * group-quantized linear layer  y = x . dequant(W)^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only tests/, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or helper with the CUDA
 * library; both sides are written independently from the pages.
 *
 * Sources (page title + section), one per function below:
 *  - "MetalConfig quantization: batched generate silently corrupts all rows
 *    after the first" (transformers issue #47331), probe script: the
 *    quantizer is applied to an fp32 W on the CPU and the scales/biases are
 *    converted to bf16 *afterwards*; the reference is x @ dequant(W)^T, row by
 *    row, for every batch element.
 *  - "Metal Kernel Bits=8 Final Report", section 3.1 (quantization basics):
 *    4-bit: 8 codes per uint32, packedIdx = g*(groupSize/8) + inG/8,
 *    shift = (inG%8)*4, mask 0xF; 8-bit: 4 codes per uint32, /4, *8, 0xFF;
 *    W is [outDim, inDim*bits/32] uint32 and scales are [outDim, inDim/G].
 *  - The affine rule w = scale*q + bias with scale = (max-min)/(2^bits-1),
 *    bias = min, round to nearest, clamp; 3/5/6-bit codes form a dense
 *    little-endian bitstream (the method statement that accompanies the pages).
 *  - The gated MLP of the decoder that the decode workload is drawn from (transformers
 *    issue #47331, reproduction: a Qwen3-0.6B decoder layer, whose MLP is
 *    down(silu(gate(h)) * up(h))): silu(v) = v / (1 + exp(-v)), the one step of the
 *    fused gate/up call that is not a contraction (a reading: the page names the model,
 *    not its activation).
 *  - The same decoder normalises each block's input per token (RMSNorm,
 *    x / sqrt(mean(x^2) + eps), its weight folded into W): a reading too, used by
 *    the fused projections' optional normalised input.
 *  - "mlx PR #4516" (load_vector fix): the bias term bias*sum(x) must be formed
 *    from inputs widened before they are added; the oracle does every sum in
 *    fp64, which is the exact value that fix aims at.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - q is computed from the fp32 (unrounded) scale and bias, with IEEE fp32
 *    subtraction and true division, rounded half-to-even (rintf), clamped;
 *    the stored scale/bias are then rounded to bf16/fp16 (round to nearest even).
 *  - a constant group (max == min) has scale 0, every q = 0, bias = min.
 *  - dequantization uses the STORED (rounded) scale and bias, as a kernel sees
 *    them, and is evaluated in fp64: w' = fp64(s)*q + fp64(b).
 *  - the bitstream is LSB-first: code i of a row starts at bit i*bits of the
 *    row's little-endian uint32 words; for 2/4/8 bits this is the page's
 *    packedIdx/shift formula (checked by oracle_unpack_formula).
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -fopenmp -ffp-contract=off
 *        (no fast-math: fp32 steps of the quantizer must be IEEE-exact).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_BF16 1
#define ORACLE_F16 2

/* ------------------------------------------------------------------------ */
/* Half-precision conversions, written from the IEEE-754 / bfloat16 formats. */
/* ------------------------------------------------------------------------ */

static double bf16_bits_to_double(uint16_t h) {
    /* bfloat16 is the top 16 bits of an IEEE binary32. */
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double f16_bits_to_double(uint16_t h) {
    /* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
    } else if (e == 31) {
        v = m ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

double oracle_half_to_double(uint16_t h, int dtype) {
    return dtype == ORACLE_BF16 ? bf16_bits_to_double(h) : f16_bits_to_double(h);
}

static uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40); /* NaN */
    /* round to nearest, ties to even, on the 16 dropped bits */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static uint16_t float_to_f16_rne(float f) {
    /* Exact rounding of a binary32 to binary16 via fp64 arithmetic on the
     * exponent/fraction; ties to even. */
    double d = (double)f;
    uint16_t sign = 0;
    if (signbit(d)) { sign = 0x8000; d = -d; }
    if (isnan(d)) return 0x7e00;
    if (d >= 65520.0) return sign | 0x7c00; /* rounds to +inf (max finite 65504) */
    if (d < ldexp(1.0, -14)) {
        /* subnormal range: units of 2^-24 */
        double units = d * ldexp(1.0, 24);
        double r = nearbyint(units); /* default rounding mode: ties to even */
        return sign | (uint16_t)r;   /* r == 1024 carries into the exponent field correctly */
    }
    int e;
    double fr = frexp(d, &e);          /* d = fr * 2^e, fr in [0.5,1) */
    double units = ldexp(fr, 11);      /* in [1024, 2048) */
    double r = nearbyint(units);
    if (r == 2048.0) { r = 1024.0; e += 1; }
    int biased = e - 1 + 15;
    if (biased >= 31) return sign | 0x7c00;
    return sign | (uint16_t)((biased << 10) | ((int)r - 1024));
}

uint16_t oracle_float_to_half_rne(float f, int dtype) {
    return dtype == ORACLE_BF16 ? float_to_bf16_rne(f) : float_to_f16_rne(f);
}

/* ------------------------------------------------------------------------ */
/* Quantize: per (row n, group g) of G consecutive K elements.               */
/* ------------------------------------------------------------------------ */

/*
 * w:        [N, K] fp32, row-major contiguous.
 * codes:    [N, K] uint8 out, q in [0, 2^bits - 1].
 * scale32:  [N, K/G] fp32 out (the unrounded scale used to form q).
 * bias32:   [N, K/G] fp32 out (= group minimum).
 * scale_s:  [N, K/G] uint16 out, bf16/fp16 bits of the stored scale.
 * bias_s:   [N, K/G] uint16 out, bf16/fp16 bits of the stored bias.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_quantize(const float* w, int64_t N, int64_t K, int group, int bits, int sdtype,
                    uint8_t* codes, float* scale32, float* bias32,
                    uint16_t* scale_s, uint16_t* bias_s) {
    if (group <= 0 || K % group != 0 || bits < 1 || bits > 8) return -1;
    const int64_t ngroups = K / group;
    const float maxq = (float)((1 << bits) - 1);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < ngroups; ++g) {
            const float* wg = w + n * K + g * group;
            float mn = wg[0], mx = wg[0];
            for (int i = 1; i < group; ++i) {
                if (wg[i] < mn) mn = wg[i];
                if (wg[i] > mx) mx = wg[i];
            }
            volatile float range = mx - mn;       /* fp32 subtraction */
            volatile float scale = range / maxq;  /* fp32 true division */
            float bias = mn;
            for (int i = 0; i < group; ++i) {
                uint8_t q;
                if (scale == 0.0f) {
                    q = 0;
                } else {
                    volatile float d = wg[i] - bias;  /* fp32 */
                    volatile float t = d / scale;     /* fp32 true division */
                    float r = rintf(t);               /* nearest, ties to even */
                    if (r < 0.0f) r = 0.0f;
                    if (r > maxq) r = maxq;
                    q = (uint8_t)r;
                }
                codes[n * K + g * group + i] = q;
            }
            scale32[n * ngroups + g] = scale;
            bias32[n * ngroups + g] = bias;
            scale_s[n * ngroups + g] = oracle_float_to_half_rne(scale, sdtype);
            bias_s[n * ngroups + g] = oracle_float_to_half_rne(bias, sdtype);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Pack / unpack as an LSB-first little-endian bitstream per row.            */
/* ------------------------------------------------------------------------ */

/* codes [N, K] -> packed [N, K*bits/32]; requires K*bits % 32 == 0. */
int oracle_pack(const uint8_t* codes, int64_t N, int64_t K, int bits, uint32_t* packed) {
    if ((K * bits) % 32 != 0) return -1;
    const int64_t words = K * bits / 32;
    memset(packed, 0, (size_t)(N * words) * sizeof(uint32_t));
    for (int64_t n = 0; n < N; ++n) {
        uint32_t* row = packed + n * words;
        for (int64_t i = 0; i < K; ++i) {
            uint32_t q = codes[n * K + i];
            /* write code bit by bit: bit j of q goes to stream bit i*bits + j */
            for (int j = 0; j < bits; ++j) {
                int64_t pos = i * bits + j;
                if ((q >> j) & 1u) row[pos / 32] |= (1u << (pos % 32));
            }
        }
    }
    return 0;
}

/* packed [N, K*bits/32] -> codes [N, K], bit by bit. */
int oracle_unpack(const uint32_t* packed, int64_t N, int64_t K, int bits, uint8_t* codes) {
    if ((K * bits) % 32 != 0) return -1;
    const int64_t words = K * bits / 32;
    for (int64_t n = 0; n < N; ++n) {
        const uint32_t* row = packed + n * words;
        for (int64_t i = 0; i < K; ++i) {
            uint32_t q = 0;
            for (int j = 0; j < bits; ++j) {
                int64_t pos = i * bits + j;
                q |= ((row[pos / 32] >> (pos % 32)) & 1u) << j;
            }
            codes[n * K + i] = (uint8_t)q;
        }
    }
    return 0;
}

/*
 * The page's per-group index formula for the power-of-two widths
 * ("Metal Kernel Bits=8 Final Report", 3.1 / 3.2): with per = 32/bits codes
 * per word, element inG of group g sits in word g*(G/per) + inG/per at shift
 * (inG % per)*bits, masked with 2^bits - 1.  Only bits in {2, 4, 8}.
 */
int oracle_unpack_formula(const uint32_t* packed, int64_t N, int64_t K, int group, int bits,
                          uint8_t* codes) {
    if (bits != 2 && bits != 4 && bits != 8) return -1;
    if (K % group != 0) return -1;
    const int per = 32 / bits;
    if (group % per != 0) return -1;
    const int64_t words = K / per;
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < K / group; ++g) {
            for (int inG = 0; inG < group; ++inG) {
                int64_t packedIdx = g * (group / per) + inG / per;
                int shift = (inG % per) * bits;
                codes[n * K + g * group + inG] =
                    (uint8_t)((packed[n * words + packedIdx] >> shift) & mask);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Dequantize with the stored scale/bias, in fp64.                           */
/* ------------------------------------------------------------------------ */

/* codes [N,K], scale_s/bias_s [N,K/G] half bits -> wdq [N,K] fp64. */
void oracle_dequant(const uint8_t* codes, const uint16_t* scale_s, const uint16_t* bias_s,
                    int sdtype, int64_t N, int64_t K, int group, double* wdq) {
    const int64_t ngroups = K / group;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t g = k / group;
            double s = oracle_half_to_double(scale_s[n * ngroups + g], sdtype);
            double b = oracle_half_to_double(bias_s[n * ngroups + g], sdtype);
            wdq[n * K + k] = s * (double)codes[n * K + k] + b;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Linear: y[..., m, n] = sum_k x[..., m, k] * wdq[..., n, k]   (fp64)        */
/* ------------------------------------------------------------------------ */

/*
 * x is read element by element through its strided view (rank xr in 2..4,
 * strides in elements, half-precision bits of dtype xdtype) so that no batch
 * folding logic is involved.  wdq is an fp64 view of rank wr in 2..4 whose
 * leading (batch) dims are right-aligned against x's batch dims and either
 * equal them or are 1 (broadcast).  y is written contiguous with shape
 * x.shape[:-1] + [N].
 */
int oracle_linear(const uint16_t* x, int xdtype, int xr, const int64_t* xshape,
                  const int64_t* xstride, const double* wdq, int wr, const int64_t* wshape,
                  const int64_t* wstride, double* y) {
    if (xr < 2 || xr > 4 || wr < 2 || wr > 4) return -1;
    const int64_t K = xshape[xr - 1];
    const int64_t M = xshape[xr - 2];
    const int64_t N = wshape[wr - 2];
    if (wshape[wr - 1] != K) return -1;
    /* batch dims of x, padded to 2 on the left */
    int64_t xb[2] = {1, 1}, xbs[2] = {0, 0};
    int64_t wb[2] = {1, 1}, wbs[2] = {0, 0};
    for (int i = 0; i < xr - 2; ++i) { xb[2 - (xr - 2) + i] = xshape[i]; xbs[2 - (xr - 2) + i] = xstride[i]; }
    for (int i = 0; i < wr - 2; ++i) { wb[2 - (wr - 2) + i] = wshape[i]; wbs[2 - (wr - 2) + i] = wstride[i]; }
    for (int i = 0; i < 2; ++i)
        if (wb[i] != 1 && wb[i] != xb[i]) return -1;
    const int64_t total_rows = xb[0] * xb[1] * M;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < total_rows; ++r) {
        int64_t m = r % M;
        int64_t b1 = (r / M) % xb[1];
        int64_t b0 = r / (M * xb[1]);
        const int64_t xoff = b0 * xbs[0] + b1 * xbs[1] + m * xstride[xr - 2];
        const int64_t woff = (wb[0] == 1 ? 0 : b0 * wbs[0]) + (wb[1] == 1 ? 0 : b1 * wbs[1]);
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double xv = oracle_half_to_double(x[xoff + k * xstride[xr - 1]], xdtype);
                double wv = wdq[woff + n * wstride[wr - 2] + k * wstride[wr - 1]];
                acc += xv * wv;
            }
            y[r * N + n] = acc;
        }
    }
    return 0;
}

/*
 * Same contraction for a row sample: only the listed (row r, column n) pairs,
 * r indexing the flattened x.shape[:-1], for full-size checks.
 * x must be rank 2 [R, K] contiguous-rows view (stride given), wdq rank 2.
 */
void oracle_linear_sampled(const uint16_t* x, int xdtype, int64_t K, int64_t ldx,
                           const double* wdq, int64_t ldw, const int64_t* rows,
                           const int64_t* cols, int64_t count, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc += oracle_half_to_double(x[rows[i] * ldx + k], xdtype) * wdq[cols[i] * ldw + k];
        out[i] = acc;
    }
}

/*
 * Grouped (mixture-of-experts) contraction: x_sorted [T, K] rows grouped by
 * expert, expert e owning rows offsets[e] .. offsets[e+1]-1;
 * wdq_bank [E, N, K] fp64 contiguous.  y [T, N] fp64.
 */
int oracle_linear_grouped(const uint16_t* x, int xdtype, int64_t T, int64_t K,
                          const int64_t* offsets, int64_t E, const double* wdq_bank,
                          int64_t N, double* y) {
    if (offsets[0] != 0 || offsets[E] != T) return -1;
    for (int64_t e = 0; e < E; ++e)
        if (offsets[e + 1] < offsets[e]) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < T; ++t) {
        int64_t e = 0;
        while (!(t >= offsets[e] && t < offsets[e + 1])) ++e;
        const double* w = wdq_bank + e * N * K;
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += oracle_half_to_double(x[t * K + k], xdtype) * w[n * K + k];
            y[t * N + n] = acc;
        }
    }
    return 0;
}

/*
 * Factored form of one output, in fp64: sum over groups of
 * s_g * sum_{k in g} q_k x_k + b_g * sum_{k in g} x_k.  Used only by tests to
 * confirm the identity the kernels rely on.
 */
double oracle_factored_dot(const uint16_t* x, int xdtype, const uint8_t* codes,
                           const uint16_t* scale_s, const uint16_t* bias_s, int sdtype,
                           int64_t K, int group) {
    double total = 0.0;
    for (int64_t g = 0; g < K / group; ++g) {
        double sqx = 0.0, sx = 0.0;
        for (int64_t k = g * group; k < (g + 1) * group; ++k) {
            double xv = oracle_half_to_double(x[k], xdtype);
            sqx += (double)codes[k] * xv;
            sx += xv;
        }
        total += oracle_half_to_double(scale_s[g], sdtype) * sqx +
                 oracle_half_to_double(bias_s[g], sdtype) * sx;
    }
    return total;
}

/*
 * oracle_swiglu -- out[i] = silu(g[i]) * u[i], silu(v) = v / (1 + exp(-v)), all in fp64 (the
 * gated MLP of the Qwen3-0.6B decoder of transformers issue #47331's reproduction; the
 * activation is a reading, see the file header).  g and u are the fp64 results of the gate and
 * up contractions.
 */
double oracle_silu(double v) { return v / (1.0 + exp(-v)); }

void oracle_swiglu(const double* g, const double* u, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_silu(g[i]) * u[i];
}

/*
 * oracle_rms_inv -- per row t of x [rows, K] (half bits, contiguous), in fp64:
 *     out[t] = 1 / sqrt(sum_k x[t,k]^2 / K + eps)
 * the per-token factor of an RMS-normalised input (reading: the decoder's RMSNorm with its
 * weight folded into W).
 */
void oracle_rms_inv(const uint16_t* x, int xdtype, int64_t rows, int64_t K, double eps, double* out) {
    for (int64_t t = 0; t < rows; ++t) {
        double s2 = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double v = oracle_half_to_double(x[t * K + k], xdtype);
            s2 += v * v;
        }
        out[t] = 1.0 / sqrt(s2 / (double)K + eps);
    }
}
