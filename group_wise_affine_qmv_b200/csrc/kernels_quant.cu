// kernels_quant.cu -- group-wise affine quantization and dequantization.
//
// Quantizer (transformers issue #47331, probe script; the method statement):
// per (row, group of G consecutive K elements), in IEEE fp32,
//   scale = (max - min) / (2^bits - 1),  bias = min,
//   q = clamp(rint((w - bias) / scale), 0, 2^bits - 1)   (constant group: q = 0),
// then scale and bias are stored rounded to nearest-even in bf16/fp16.  The
// fp32 steps use explicit round-to-nearest subtraction and true division so
// every code is reproducible bit for bit.
//
// Packing ("Metal Kernel Bits=8 Final Report", section 3.1; the 3/5/6-bit
// bitstream of the method statement): code i of a row occupies stream bits
// [i*bits, (i+1)*bits) of the row's little-endian uint32 words.  A group of
// G >= 32 codes always starts on a word boundary (G*bits is a multiple of 32).
#include <cuda_runtime.h>

#include "aq_internal.h"
#include "device_common.cuh"

namespace aq {
namespace {

constexpr int QWARPS = 4;

template <typename WT, typename ST>
__global__ void __launch_bounds__(QWARPS * 32) quantize_kernel(const QuantArgs a) {
    __shared__ uint8_t codes_s[QWARPS][128];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gwarp = (int64_t)blockIdx.x * QWARPS + warp;
    const int64_t nwarps = (int64_t)gridDim.x * QWARPS;
    const int group = a.group, bits = a.bits;
    const int64_t ngroups = a.K / group;
    const int64_t total = a.N * ngroups;
    const int per_lane = group / 32;
    const float maxq = (float)((1 << bits) - 1);
    const int nwords = group * bits / 32;
    for (int64_t item = gwarp; item < total; item += nwarps) {
        const int64_t n = item / ngroups, g = item % ngroups;
        const WT* wg = (const WT*)a.w + n * a.w_row + g * group;
        float v[4];
        float mn = INFINITY, mx = -INFINITY;
        for (int i = 0; i < per_lane; ++i) {
            v[i] = to_float<WT>(wg + lane + 32 * i);
            mn = fminf(mn, v[i]);
            mx = fmaxf(mx, v[i]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const float scale = __fdiv_rn(__fsub_rn(mx, mn), maxq);
        for (int i = 0; i < per_lane; ++i) {
            float q = 0.0f;
            if (scale != 0.0f) {
                q = rintf(__fdiv_rn(__fsub_rn(v[i], mn), scale));
                q = fminf(fmaxf(q, 0.0f), maxq);
            }
            codes_s[warp][lane + 32 * i] = (uint8_t)q;
        }
        __syncwarp();
        if (lane < nwords) {
            // word `lane` of this group holds stream bits [32*lane, 32*lane + 32)
            uint32_t word = 0;
            const int first = (32 * lane) / bits;
            const int last = (32 * lane + 31) / bits;
            for (int i = first; i <= last; ++i) {
                const int pos = i * bits - 32 * lane;
                const uint32_t c = codes_s[warp][i];
                word |= pos >= 0 ? (c << pos) : (c >> (-pos));
            }
            a.wq[n * a.wq_row + g * nwords + lane] = word;
        }
        if (lane == 0) {
            store_out((ST*)a.scales + n * a.s_row + g, scale);
            store_out((ST*)a.biases + n * a.b_row + g, mn);
        }
        __syncwarp();
    }
    // The matrix kernels stage their weights before their wait on the kernel before them in the
    // stream.  This kernel never lets a dependent start early, and with every write performed
    // device-wide before its threads exit, a matrix call right after it reads the new weights.
    __threadfence();
}

// One thread per 32-code chunk of a row: out = fma(scale, q, bias) in fp32, rounded to WT.
// With a.ids (row gather, "Metal Kernel Bits=8 Final Report" section 3.2: dequantize_row for one
// token id) output row n reads W row ids[n]; an id outside [0, V) writes zeros and flags it.
template <typename WT, typename ST>
__global__ void __launch_bounds__(256) dequantize_kernel(const QuantArgs a) {
    const int64_t chunks = a.K / 32;
    const int64_t total = a.N * chunks;
    const int bits = a.bits;
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = t / chunks, c = t % chunks;
        int64_t n = row;
        if (a.ids) {
            n = a.ids[row];
            if (n < 0 || n >= a.V) {
                WT* out = (WT*)a.w + row * a.w_row + c * 32;
                for (int i = 0; i < 32; ++i) store_out(out + i, 0.0f);
                if (c == 0) atomicOr(a.err, DEVERR_INDEX);
                continue;
            }
        }
        const uint32_t* wp = a.wq + n * a.wq_row + c * bits;
        uint32_t w[9];
        for (int i = 0; i < bits; ++i) w[i] = __ldg(wp + i);
        w[bits] = 0;
        const int64_t g = (c * 32) / a.group;
        const float s = to_float<ST>((const ST*)a.scales + n * a.s_row + g);
        const float b = to_float<ST>((const ST*)a.biases + n * a.b_row + g);
        WT* out = (WT*)a.w + row * a.w_row + c * 32;
        for (int i = 0; i < 32; ++i) {
            const int pos = i * bits;
            const int wi = pos >> 5, sh = pos & 31;
            const uint32_t q = __funnelshift_r(w[wi], w[wi + 1], sh) & mask;
            store_out(out + i, fmaf(s, (float)q, b));
        }
    }
}

int grid_for(int64_t items, int per_block) {
    int64_t g = (items + per_block - 1) / per_block;
    if (g > 148 * 64) g = 148 * 64;
    if (g < 1) g = 1;
    return (int)g;
}

template <typename ST>
cudaError_t quantize_w(const QuantArgs& a, DT wdt, cudaStream_t s) {
    const int grid = grid_for(a.N * (a.K / a.group), QWARPS);
    switch (wdt) {
        case DT::F32: quantize_kernel<float, ST><<<grid, QWARPS * 32, 0, s>>>(a); break;
        case DT::BF16: quantize_kernel<bf16_t, ST><<<grid, QWARPS * 32, 0, s>>>(a); break;
        case DT::F16: quantize_kernel<f16_t, ST><<<grid, QWARPS * 32, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

template <typename ST>
cudaError_t dequantize_w(const QuantArgs& a, DT wdt, cudaStream_t s) {
    const int grid = grid_for(a.N * (a.K / 32), 256);
    switch (wdt) {
        case DT::F32: dequantize_kernel<float, ST><<<grid, 256, 0, s>>>(a); break;
        case DT::BF16: dequantize_kernel<bf16_t, ST><<<grid, 256, 0, s>>>(a); break;
        case DT::F16: dequantize_kernel<f16_t, ST><<<grid, 256, 0, s>>>(a); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const QuantArgs& a, DT wdt, DT sdt, cudaStream_t s) {
    return sdt == DT::BF16 ? quantize_w<bf16_t>(a, wdt, s) : quantize_w<f16_t>(a, wdt, s);
}

cudaError_t launch_dequantize(const QuantArgs& a, DT wdt, DT sdt, cudaStream_t s) {
    return sdt == DT::BF16 ? dequantize_w<bf16_t>(a, wdt, s) : dequantize_w<f16_t>(a, wdt, s);
}

}  // namespace aq
