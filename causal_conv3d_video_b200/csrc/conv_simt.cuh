// conv_simt.cuh -- cached causal Conv3D on the FP32 pipes: the FP32 contract
// (IEEE fp32 FMA, no TF32) and bf16 shapes too thin or too odd for the
// tensor-core tiles (Cin or Cout not a multiple of 16, large strides).
//
// Each thread owns one output pixel and CO_T consecutive output channels and
// walks the active taps only: for output frame o, tap k is skipped unless
// o_l[k] <= o < o_h[k] (paper, Sec. 4), and its source frame o*s_t + delta_k is
// read from the cache or the input by pointer select.  Blocks past
// conv_blocks write new_cache.
#pragma once
#include <cuda_bf16.h>

#include "cache_copy.cuh"
#include "params.h"

namespace ccv3d {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

constexpr int kSimtThreads = 128;
constexpr int kSimtCoT = 4;

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
conv_simt_kernel(const __grid_constant__ SimtParams p) {
    if ((int)blockIdx.x >= p.conv_blocks) {
        copy_new_cache(p.copy, blockIdx.x - p.conv_blocks, p.copy_blocks, threadIdx.x,
                       blockDim.x);
        return;
    }
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= p.conv_threads) return;
    const int cog = (int)(gid % p.co_groups);
    long long pix = gid / p.co_groups;
    const int xo = (int)(pix % p.W_o);
    pix /= p.W_o;
    const int yo = (int)(pix % p.H_o);
    pix /= p.H_o;
    const int o = (int)(pix % p.T_o);
    const int n = (int)(pix / p.T_o);
    const int co0 = cog * kSimtCoT;

    const T* x = static_cast<const T*>(p.x);
    const T* cache = static_cast<const T*>(p.cache);
    const T* w = static_cast<const T*>(p.w);
    const long long w_co_stride = (long long)p.taps.kt * p.kh * p.kw * p.Cin;

    float acc[kSimtCoT];
#pragma unroll
    for (int j = 0; j < kSimtCoT; ++j) acc[j] = 0.f;

    for (int k = 0; k < p.taps.kt; ++k) {
        if (!(o >= p.taps.o_l[k] && o < p.taps.o_h[k])) continue;
        const int t = o * p.taps.s_t + p.taps.delta[k];
        const T* frame = t < p.cache_len
                             ? cache + ((long long)n * p.cache_len + t) * p.H * p.W * p.Cin
                             : x + ((long long)n * p.T_x + (t - p.cache_len)) * p.H * p.W * p.Cin;
        for (int r = 0; r < p.kh; ++r) {
            const int yi = yo * p.s_h + r * p.d_h - p.p_h;
            if (yi < 0 || yi >= p.H) continue;
            for (int s = 0; s < p.kw; ++s) {
                const int xi = xo * p.s_w + s * p.d_w - p.p_w;
                if (xi < 0 || xi >= p.W) continue;
                const T* zrow = frame + ((long long)yi * p.W + xi) * p.Cin;
                const T* wrow = w + (((long long)co0 * p.taps.kt + k) * p.kh + r) * p.kw * p.Cin +
                                (long long)s * p.Cin;
                for (int ci = 0; ci < p.Cin; ++ci) {
                    const float z = to_f32<T>(zrow[ci]);
#pragma unroll
                    for (int j = 0; j < kSimtCoT; ++j)
                        if (co0 + j < p.Cout)
                            acc[j] = fmaf(z, to_f32<T>(wrow[j * w_co_stride + ci]), acc[j]);
                }
            }
        }
    }
    const T* bias = static_cast<const T*>(p.bias);
    T* out = static_cast<T*>(p.out) +
             ((((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo) * p.Cout;
#pragma unroll
    for (int j = 0; j < kSimtCoT; ++j) {
        if (co0 + j >= p.Cout) break;
        float v = acc[j];
        if (bias != nullptr) v += to_f32<T>(bias[co0 + j]);
        out[co0 + j] = from_f32<T>(v);
    }
}

// Small calls (too few (pixel, channel-group) units to fill the SMs with one
// thread each, e.g. the 16-channel fp32 contract call): one warp per unit.
// The lanes split the flattened reduction over (temporal tap, kernel row,
// kernel column, input channel) -- consecutive lanes take consecutive input
// channels, so their loads are contiguous -- and combine their partial sums
// with warp shuffles; lane 0 adds the bias and stores.  conv_threads counts
// units here.
template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
conv_simt_warp_kernel(const __grid_constant__ SimtParams p) {
    if ((int)blockIdx.x >= p.conv_blocks) {
        copy_new_cache(p.copy, blockIdx.x - p.conv_blocks, p.copy_blocks, threadIdx.x,
                       blockDim.x);
        return;
    }
    const long long unit = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (unit >= p.conv_threads) return;  // whole warps leave together
    const int cog = (int)(unit % p.co_groups);
    long long pix = unit / p.co_groups;
    const int xo = (int)(pix % p.W_o);
    pix /= p.W_o;
    const int yo = (int)(pix % p.H_o);
    pix /= p.H_o;
    const int o = (int)(pix % p.T_o);
    const int n = (int)(pix / p.T_o);
    const int co0 = cog * kSimtCoT;

    const T* x = static_cast<const T*>(p.x);
    const T* cache = static_cast<const T*>(p.cache);
    const T* w = static_cast<const T*>(p.w);
    const int taps2d = p.kh * p.kw;
    const long long w_co_stride = (long long)p.taps.kt * taps2d * p.Cin;
    const int K = p.taps.kt * taps2d * p.Cin;

    float acc[kSimtCoT];
#pragma unroll
    for (int j = 0; j < kSimtCoT; ++j) acc[j] = 0.f;
    // kU reduction steps per lane at a time: their (predicated) loads are
    // independent, so they are all in flight before the FMAs need them
    constexpr int kU = 4;
    for (int base = lane; base < K; base += 32 * kU) {
        float z[kU], wv[kU][kSimtCoT];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int idx = base + 32 * u;
            const int tap = idx / p.Cin;
            const int ci = idx - tap * p.Cin;
            const int k = tap / taps2d;
            const int rs = tap - k * taps2d;
            const int r = rs / p.kw;
            const int s = rs - r * p.kw;
            const int yi = yo * p.s_h + r * p.d_h - p.p_h;
            const int xi = xo * p.s_w + s * p.d_w - p.p_w;
            const bool live = idx < K && k < p.taps.kt && o >= p.taps.o_l[k] &&
                              o < p.taps.o_h[k] && yi >= 0 && yi < p.H && xi >= 0 && xi < p.W;
            z[u] = 0.f;
#pragma unroll
            for (int j = 0; j < kSimtCoT; ++j) wv[u][j] = 0.f;
            if (live) {
                const int t = o * p.taps.s_t + p.taps.delta[k];
                const T* frame =
                    t < p.cache_len
                        ? cache + ((long long)n * p.cache_len + t) * p.H * p.W * p.Cin
                        : x + ((long long)n * p.T_x + (t - p.cache_len)) * p.H * p.W * p.Cin;
                z[u] = to_f32<T>(frame[((long long)yi * p.W + xi) * p.Cin + ci]);
                const T* wcol = w + (long long)co0 * w_co_stride + (long long)tap * p.Cin + ci;
#pragma unroll
                for (int j = 0; j < kSimtCoT; ++j)
                    if (co0 + j < p.Cout) wv[u][j] = to_f32<T>(wcol[j * w_co_stride]);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u)
#pragma unroll
            for (int j = 0; j < kSimtCoT; ++j) acc[j] = fmaf(z[u], wv[u][j], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < kSimtCoT; ++j)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    if (lane != 0) return;
    const T* bias = static_cast<const T*>(p.bias);
    T* out = static_cast<T*>(p.out) +
             ((((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo) * p.Cout;
#pragma unroll
    for (int j = 0; j < kSimtCoT; ++j) {
        if (co0 + j >= p.Cout) break;
        float v = acc[j];
        if (bias != nullptr) v += to_f32<T>(bias[co0 + j]);
        out[co0 + j] = from_f32<T>(v);
    }
}

}  // namespace ccv3d
