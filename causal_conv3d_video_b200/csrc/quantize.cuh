// quantize.cuh -- post-decode uint8 quantisation of decoded frames.
//
// The step after the decoder (FastVideo pull request "Quantize frames to
// uint8 on-device before the post-decode D->H copy", Summary): each value is
// multiplied by 255 in fp32, clamped to [0, 255] and truncated to uint8 on the
// device, so the device-to-host copy moves one byte per value instead of four
// (fp32) or two (bf16).  fmaxf returns its non-NaN operand, so a NaN maps to 0.
//
// HBM-bound: 4 + 1 (fp32) or 2 + 1 (bf16) bytes per value.  Each thread
// handles 16 consecutive values per step -- four (fp32) or two (bf16) 16-byte
// streaming loads in flight and one 16-byte streaming store -- over a
// grid-stride loop sized to the SM count; the last n % 16 values go through
// a scalar path.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

namespace ccv3d {

__device__ __forceinline__ uint32_t quant8(float v) {
    float y = v * 255.0f;
    y = fmaxf(y, 0.0f);
    y = fminf(y, 255.0f);
    return __float2uint_rz(y);
}

__device__ __forceinline__ uint32_t pack4(float a, float b, float c, float d) {
    return quant8(a) | (quant8(b) << 8) | (quant8(c) << 16) | (quant8(d) << 24);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// in: n fp32 values, out: n bytes; both 16-byte aligned.
__global__ void __launch_bounds__(256) quantize_u8_f32_kernel(const float* __restrict__ in,
                                                              uint8_t* __restrict__ out,
                                                              long long n) {
    const long long n16 = n / 16;
    const float4* src = reinterpret_cast<const float4*>(in);
    uint4* dst = reinterpret_cast<uint4*>(out);
    const long long step = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += step) {
        const float4 a = __ldcs(src + 4 * i);
        const float4 b = __ldcs(src + 4 * i + 1);
        const float4 c = __ldcs(src + 4 * i + 2);
        const float4 d = __ldcs(src + 4 * i + 3);
        __stcs(dst + i, make_uint4(pack4(a.x, a.y, a.z, a.w), pack4(b.x, b.y, b.z, b.w),
                                   pack4(c.x, c.y, c.z, c.w), pack4(d.x, d.y, d.z, d.w)));
    }
    if (blockIdx.x == 0)
        for (long long j = n16 * 16 + threadIdx.x; j < n; j += blockDim.x)
            out[j] = (uint8_t)quant8(in[j]);
}

// in: n bf16 values (raw bits), out: n bytes; both 16-byte aligned.
__global__ void __launch_bounds__(256) quantize_u8_bf16_kernel(const uint16_t* __restrict__ in,
                                                               uint8_t* __restrict__ out,
                                                               long long n) {
    const long long n16 = n / 16;
    const uint4* src = reinterpret_cast<const uint4*>(in);
    uint4* dst = reinterpret_cast<uint4*>(out);
    const long long step = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += step) {
        const uint4 a = __ldcs(src + 2 * i);
        const uint4 b = __ldcs(src + 2 * i + 1);
        __stcs(dst + i,
               make_uint4(pack4(bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y)),
                          pack4(bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w)),
                          pack4(bf16_lo(b.x), bf16_hi(b.x), bf16_lo(b.y), bf16_hi(b.y)),
                          pack4(bf16_lo(b.z), bf16_hi(b.z), bf16_lo(b.w), bf16_hi(b.w))));
    }
    if (blockIdx.x == 0)
        for (long long j = n16 * 16 + threadIdx.x; j < n; j += blockDim.x)
            out[j] = (uint8_t)quant8(__uint_as_float((uint32_t)in[j] << 16));
}

}  // namespace ccv3d
