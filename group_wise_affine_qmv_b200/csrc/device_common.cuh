// device_common.cuh -- small device helpers shared by the kernels of libaq.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace aq {

// 16-bit storage types of x / scales / biases
struct bf16_t { uint16_t v; };
struct f16_t { uint16_t v; };

__device__ __forceinline__ float half_bits_to_float(uint16_t h, bf16_t) {
    return __uint_as_float(((uint32_t)h) << 16);  // bf16 is the top half of an fp32
}
__device__ __forceinline__ float half_bits_to_float(uint16_t h, f16_t) {
    return __half2float(__ushort_as_half(h));
}
// fp32 -> the bits of the 16-bit type, round to nearest even (as the stores of y)
__device__ __forceinline__ uint16_t float_to_half_bits(float v, bf16_t) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
__device__ __forceinline__ uint16_t float_to_half_bits(float v, f16_t) { return __half_as_ushort(__float2half_rn(v)); }

template <typename T> __device__ __forceinline__ float to_float(const T* p);
template <> __device__ __forceinline__ float to_float<bf16_t>(const bf16_t* p) {
    return __uint_as_float(((uint32_t)__ldg((const unsigned short*)p)) << 16);
}
template <> __device__ __forceinline__ float to_float<f16_t>(const f16_t* p) {
    return __half2float(__ushort_as_half(__ldg((const unsigned short*)p)));
}
template <> __device__ __forceinline__ float to_float<float>(const float* p) { return __ldg(p); }

// round-to-nearest-even stores
__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_out(bf16_t* p, float v) {
    *(__nv_bfloat16*)p = __float2bfloat16_rn(v);
}
__device__ __forceinline__ void store_out(f16_t* p, float v) { *(__half*)p = __float2half_rn(v); }

// Unpack 8 packed 16-bit values (one 16-byte vector) into floats.
__device__ __forceinline__ void unpack8(const uint4& u, float* f, bf16_t) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack8(const uint4& u, float* f, f16_t) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace aq
