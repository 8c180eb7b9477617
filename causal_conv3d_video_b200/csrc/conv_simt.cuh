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
#include "checked.cuh"
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

// The 16 bytes of one vector load as fp32 values (8 bf16 or 4 fp32).
template <typename T>
__device__ __forceinline__ void unpack16(uint4 v, float (&f)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void unpack16<float>(uint4 v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(uint4 v, float (&f)[8]) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // a bf16 is the high half of its fp32
        f[2 * j] = __uint_as_float(u[j] << 16);
        f[2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
    }
}

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
        const T* frame =
            t < p.cache_len
                ? cache + (long long)ring_frame(n, t, p.cache_slots, p.cache_head) * p.H * p.W * p.Cin
                : x + ((long long)n * p.T_x + (t - p.cache_len)) * p.H * p.W * p.Cin;
        const void* src_base = t < p.cache_len ? (const void*)cache : (const void*)x;
        const long long src_bytes = t < p.cache_len ? p.copy.cache_bytes : p.copy.x_bytes;
        for (int r = 0; r < p.kh; ++r) {
            const int yi = yo * p.s_h + r * p.d_h - p.p_h;
            if (yi < 0 || yi >= p.H) continue;
            for (int s = 0; s < p.kw; ++s) {
                const int xi = xo * p.s_w + s * p.d_w - p.p_w;
                if (xi < 0 || xi >= p.W) continue;
                const T* zrow = frame + ((long long)yi * p.W + xi) * p.Cin;
                const T* wrow = w + (((long long)co0 * p.taps.kt + k) * p.kh + r) * p.kw * p.Cin +
                                (long long)s * p.Cin;
                // checked build: the input pixel and the weight rows read below
                if (!in_bounds(p.status, zrow, (long long)p.Cin * sizeof(T), src_base, src_bytes))
                    continue;
                bool wok[kSimtCoT];
#pragma unroll
                for (int j = 0; j < kSimtCoT; ++j)
                    wok[j] = co0 + j < p.Cout &&
                             in_bounds(p.status, wrow + j * w_co_stride,
                                       (long long)p.Cin * sizeof(T), w,
                                       p.w_floats * (long long)sizeof(T));
                if (p.Cin % (16 / (int)sizeof(T)) == 0) {
                    // 16-byte loads: 8 bf16 or 4 fp32 channels of the pixel and
                    // of each weight row (both 16-byte aligned: their element
                    // offsets are multiples of Cin)
                    constexpr int V = 16 / sizeof(T);
                    for (int ci = 0; ci < p.Cin; ci += V) {
                        float z[V];
                        unpack16<T>(__ldg(reinterpret_cast<const uint4*>(zrow + ci)), z);
#pragma unroll
                        for (int j = 0; j < kSimtCoT; ++j) {
                            if (!wok[j]) continue;
                            float wv[V];
                            unpack16<T>(__ldg(reinterpret_cast<const uint4*>(
                                            wrow + j * w_co_stride + ci)), wv);
#pragma unroll
                            for (int e = 0; e < V; ++e) acc[j] = fmaf(z[e], wv[e], acc[j]);
                        }
                    }
                } else {
                    for (int ci = 0; ci < p.Cin; ++ci) {
                        const float z = to_f32<T>(zrow[ci]);
#pragma unroll
                        for (int j = 0; j < kSimtCoT; ++j)
                            if (wok[j])
                                acc[j] = fmaf(z, to_f32<T>(wrow[j * w_co_stride + ci]), acc[j]);
                    }
                }
            }
        }
    }
    const T* bias = static_cast<const T*>(p.bias);
    T* out = static_cast<T*>(p.out) +
             ((((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo) * p.Cout;
    const long long out_i = (((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo;
#pragma unroll
    for (int j = 0; j < kSimtCoT; ++j) {
        if (co0 + j >= p.Cout) break;
        if (!index_ok(p.status, out_i * p.Cout + co0 + j, p.out_elems)) break;
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
    // small calls only (fewer than 148 x 128 units): 32-bit unit decode
    const int unit = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (unit >= p.conv_threads) return;  // whole warps leave together
    const int cog = unit % p.co_groups;
    int pix = unit / p.co_groups;
    const int xo = pix % p.W_o;
    pix /= p.W_o;
    const int yo = pix % p.H_o;
    pix /= p.H_o;
    const int o = pix % p.T_o;
    const int n = pix / p.T_o;
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
    if (32 % p.Cin == 0) {
        // Cin divides 32 (the 16-channel contract call): lane = (tap offset,
        // channel); a lane walks the taps tpi = 32 / Cin apart with its
        // (k, r, s) position advanced step by step.  The temporal taps' frame
        // pointers and the weight base are fixed per warp, and offsets inside
        // a frame are 32-bit (a frame holds < 2^31 elements), so a reduction
        // step is a handful of integer ops, two loads and four FMAs.
        const int tpi = 32 / p.Cin, ci = lane % p.Cin;
        const int ntaps = p.taps.kt * taps2d;
        const T* fb[kMaxTaps];
        bool act[kMaxTaps];
#pragma unroll
        for (int k = 0; k < kMaxTaps; ++k) {
            act[k] = k < p.taps.kt && o >= p.taps.o_l[k] && o < p.taps.o_h[k];
            const int tf = o * p.taps.s_t + p.taps.delta[k];
            fb[k] = !act[k] ? x
                            : (tf < p.cache_len
                                   ? cache + (long long)ring_frame(n, tf, p.cache_slots,
                                                                   p.cache_head) *
                                                 p.H * p.W * p.Cin
                                   : x + ((long long)n * p.T_x + (tf - p.cache_len)) * p.H *
                                             p.W * p.Cin);
        }
        const int ybase = yo * p.s_h - p.p_h, xbase = xo * p.s_w - p.p_w;
        const T* wb = w + (long long)co0 * w_co_stride + ci;  // + j w_co_stride + t Cin
        const int jmax = min(kSimtCoT, p.Cout - co0);
        int t = lane / p.Cin;
        int k = t / taps2d, r = (t - k * taps2d) / p.kw, sx = t - k * taps2d - r * p.kw;
#pragma unroll 4
        for (; t < ntaps; t += tpi) {
            const int yi = ybase + r * p.d_h, xi = xbase + sx * p.d_w;
            const T* f = k == 0 ? fb[0] : (k == 1 ? fb[1] : fb[2]);
            const bool a = k == 0 ? act[0] : (k == 1 ? act[1] : act[2]);
            float z = 0.f;
            if (a && (unsigned)yi < (unsigned)p.H && (unsigned)xi < (unsigned)p.W) {
                const T* zp = f + (yi * p.W + xi) * p.Cin + ci;
                const int tf = o * p.taps.s_t + p.taps.delta[k];
                if (in_bounds(p.status, zp, sizeof(T),
                              tf < p.cache_len ? (const void*)cache : (const void*)x,
                              tf < p.cache_len ? p.copy.cache_bytes : p.copy.x_bytes))
                    z = to_f32<T>(__ldg(zp));
            }
            const T* wt = wb + t * p.Cin;
#pragma unroll
            for (int j = 0; j < kSimtCoT; ++j)
                if (j < jmax && in_bounds(p.status, wt + j * w_co_stride, sizeof(T), w,
                                          p.w_floats * (long long)sizeof(T)))
                    acc[j] = fmaf(z, to_f32<T>(__ldg(wt + j * w_co_stride)), acc[j]);
            for (int q = 0; q < tpi; ++q)  // next tap of this lane
                if (++sx == p.kw) {
                    sx = 0;
                    if (++r == p.kh) {
                        r = 0;
                        ++k;
                    }
                }
        }
    } else {
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
                        ? cache + (long long)ring_frame(n, t, p.cache_slots, p.cache_head) * p.H *
                                      p.W * p.Cin
                        : x + ((long long)n * p.T_x + (t - p.cache_len)) * p.H * p.W * p.Cin;
                const T* zp = frame + ((long long)yi * p.W + xi) * p.Cin + ci;
                if (in_bounds(p.status, zp, sizeof(T), t < p.cache_len ? (const void*)cache : (const void*)x,
                              t < p.cache_len ? p.copy.cache_bytes : p.copy.x_bytes))
                    z[u] = to_f32<T>(*zp);
                const T* wcol = w + (long long)co0 * w_co_stride + (long long)tap * p.Cin + ci;
#pragma unroll
                for (int j = 0; j < kSimtCoT; ++j)
                    if (co0 + j < p.Cout &&
                        in_bounds(p.status, wcol + j * w_co_stride, sizeof(T), w,
                                  p.w_floats * (long long)sizeof(T)))
                        wv[u][j] = to_f32<T>(wcol[j * w_co_stride]);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u)
#pragma unroll
            for (int j = 0; j < kSimtCoT; ++j) acc[j] = fmaf(z[u], wv[u][j], acc[j]);
    }
    }
#pragma unroll
    for (int j = 0; j < kSimtCoT; ++j)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
    if (lane != 0) return;
    const T* bias = static_cast<const T*>(p.bias);
    T* out = static_cast<T*>(p.out) +
             ((((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo) * p.Cout;
    const long long out_i = (((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo;
#pragma unroll
    for (int j = 0; j < kSimtCoT; ++j) {
        if (co0 + j >= p.Cout) break;
        if (!index_ok(p.status, out_i * p.Cout + co0 + j, p.out_elems)) break;
        float v = acc[j];
        if (bias != nullptr) v += to_f32<T>(bias[co0 + j]);
        out[co0 + j] = from_f32<T>(v);
    }
}

// Small calls whose Cin divides 32 and whose Cout <= 16 (the 16-channel fp32
// contract call): two warps per output pixel compute every output channel.
// A lane owns (tap offset, input channel): the 64 lanes of a pixel's two warps
// take taps 64 / Cin apart.  The block first stages, in shared memory, the
// weights as fp32 rows [(tap, ci)][co] of kW16Stride floats (16 channels,
// zero past Cout, and 4 floats of padding so that the 16-byte reads of the 8
// lanes of a phase fall in distinct banks) and a table of each tap's
// (temporal tap, row offset, column offset); a reduction step is then one
// table read, one input load, four 16-byte shared loads and 16 FMAs.  Each
// warp combines its lanes' 16 partial sums by recursive halving (each shuffle
// step hands the partner the half of the channels it keeps): 16 shuffles
// leave every even lane one channel's total; the second warp of a pixel hands
// its totals to the first through shared memory.  The first batch of input
// loads is issued before the staging, so both wait out one round of load
// latency together.  conv_threads counts pixels here.
constexpr int kW16Stride = 20;
constexpr int kW16Threads = 512;               // 8 pixels x 2 warps
constexpr int kW16Pixels = kW16Threads / 64;

__host__ __device__ constexpr size_t simt_warp16_smem_bytes(int taps, int cin) {
    return (size_t)taps * cin * kW16Stride * sizeof(float)  // weights
           + (size_t)taps * sizeof(int4)                      // tap table
           + (size_t)kW16Pixels * 16 * sizeof(float);         // second warps' totals
}

template <typename T>
__global__ void __launch_bounds__(kW16Threads)
conv_simt_warp16_kernel(const __grid_constant__ SimtParams p) {
    if ((int)blockIdx.x >= p.conv_blocks) {
        copy_new_cache(p.copy, blockIdx.x - p.conv_blocks, p.copy_blocks, threadIdx.x,
                       blockDim.x);
        return;
    }
    extern __shared__ float4 w16_smem[];
    const T* w = static_cast<const T*>(p.w);
    const int taps2d = p.kh * p.kw;
    const int ntaps = p.taps.kt * taps2d;
    const int K = ntaps * p.Cin;  // weight rows (tap, ci)
    float* ws = reinterpret_cast<float*>(w16_smem);
    int4* tap_tab = reinterpret_cast<int4*>(ws + (size_t)K * kW16Stride);
    float* red = reinterpret_cast<float*>(tap_tab + ntaps);

    // this warp's pixel and half (warps past the last pixel still help stage)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = warp & 1, pl = warp >> 1;  // pixel of the block
    const int unit = (int)blockIdx.x * kW16Pixels + pl;
    const bool live = unit < p.conv_threads;
    int pix = live ? unit : 0;
    const int xo = pix % p.W_o;
    pix /= p.W_o;
    const int yo = pix % p.H_o;
    pix /= p.H_o;
    const int o = pix % p.T_o;
    const int n = pix / p.T_o;

    const T* x = static_cast<const T*>(p.x);
    const T* cache = static_cast<const T*>(p.cache);
    const T* fb[kMaxTaps];
    bool act[kMaxTaps], fc[kMaxTaps];  // tap active; its frame is in the cache
#pragma unroll
    for (int k = 0; k < kMaxTaps; ++k) {
        act[k] = k < p.taps.kt && o >= p.taps.o_l[k] && o < p.taps.o_h[k];
        const int tf = o * p.taps.s_t + p.taps.delta[k];
        fc[k] = act[k] && tf < p.cache_len;
        fb[k] = !act[k] ? x
                        : (fc[k] ? cache + (long long)ring_frame(n, tf, p.cache_slots,
                                                                 p.cache_head) *
                                               p.H * p.W * p.Cin
                                 : x + ((long long)n * p.T_x + (tf - p.cache_len)) * p.H * p.W *
                                           p.Cin);
    }
    const long long cache_bytes = p.copy.cache_bytes, x_bytes = p.copy.x_bytes;
    const int tpi = 64 / p.Cin, ci = lane % p.Cin;
    const int ybase = yo * p.s_h - p.p_h, xbase = xo * p.s_w - p.p_w;
    // first tap of this lane, then every tpi-th; (k, r, s) of the first ones
    // by division here, of the rest from the table after the staging
    int t = live ? half * (32 / p.Cin) + lane / p.Cin : ntaps;
    constexpr int kZ = 8;
    float z[kZ];
    auto load_step = [&](int u, int tap, int k, int dy, int dx) {
        z[u] = 0.f;
        const int yi = ybase + dy, xi = xbase + dx;
        const T* f = k == 0 ? fb[0] : (k == 1 ? fb[1] : fb[2]);
        const bool a = k == 0 ? act[0] : (k == 1 ? act[1] : act[2]);
        if (tap < ntaps && a && (unsigned)yi < (unsigned)p.H && (unsigned)xi < (unsigned)p.W) {
            const T* zp = f + (yi * p.W + xi) * p.Cin + ci;
            const bool c = k == 0 ? fc[0] : (k == 1 ? fc[1] : fc[2]);
            if (in_bounds(p.status, zp, sizeof(T), c ? (const void*)cache : (const void*)x,
                          c ? cache_bytes : x_bytes))
                z[u] = to_f32<T>(__ldg(zp));
        }
    };
    {  // first batch: the first tap decoded by division, the next ones stepped
        int k = t / taps2d, rs = t - k * taps2d, r = rs / p.kw, sx = rs - r * p.kw;
#pragma unroll
        for (int u = 0; u < kZ; ++u) {
            load_step(u, t + u * tpi, k, r * p.d_h, sx * p.d_w);
            sx += tpi;  // advance (k, r, s) by tpi taps
            while (sx >= p.kw) {
                sx -= p.kw;
                if (++r == p.kh) {
                    r = 0;
                    ++k;
                }
            }
        }
    }

    // stage the weights (a thread takes a (tap, ci) row for all 16 channels:
    // consecutive threads read consecutive positions of a channel and write
    // consecutive rows) and the tap table
    const long long w_bytes = p.w_floats * (long long)sizeof(T);
    for (int kc = threadIdx.x; kc < K; kc += kW16Threads) {
        float v[16];
#pragma unroll
        for (int co = 0; co < 16; ++co) {
            v[co] = 0.f;
            const T* src = w + (long long)co * K + kc;
            if (co < p.Cout && in_bounds(p.status, src, sizeof(T), w, w_bytes))
                v[co] = to_f32<T>(__ldg(src));
        }
        float4* row = reinterpret_cast<float4*>(ws + kc * kW16Stride);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
    for (int tp = threadIdx.x; tp < ntaps; tp += kW16Threads) {
        const int k = tp / taps2d, rs = tp - k * taps2d, r = rs / p.kw, sx = rs - r * p.kw;
        tap_tab[tp] = make_int4(k, r * p.d_h, sx * p.d_w, 0);
    }
    __syncthreads();

    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    for (;;) {
#pragma unroll
        for (int u = 0; u < kZ; ++u) {
            const int tap = t + u * tpi;
            if (tap >= ntaps) break;  // a lane's taps increase with u
            const float4* wr = reinterpret_cast<const float4*>(ws + (tap * p.Cin + ci) * kW16Stride);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 wv = wr[q];
                acc[4 * q + 0] = fmaf(z[u], wv.x, acc[4 * q + 0]);
                acc[4 * q + 1] = fmaf(z[u], wv.y, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(z[u], wv.z, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(z[u], wv.w, acc[4 * q + 3]);
            }
        }
        t += kZ * tpi;
        if (t >= ntaps) break;
#pragma unroll
        for (int u = 0; u < kZ; ++u) {  // next batch: taps from the table
            const int tap = t + u * tpi;
            const int4 e = tap < ntaps ? tap_tab[tap] : make_int4(0, 0, 0, 0);
            load_step(u, tap, e.x, e.y, e.z);
        }
    }
    // recursive halving: after the step of offset 16 >> s a lane holds 8 >> s
    // channels, the upper or lower half of those it held, summed with its
    // partner's
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const int off = 16 >> s, h = 8 >> s;
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = up ? acc[i] : acc[i + h];
            const float keep = up ? acc[i + h] : acc[i];
            acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
    const int co = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                   ((lane >> 1) & 1);
    if (half == 1 && (lane & 1) == 0) red[pl * 16 + co] = acc[0];
    __syncthreads();
    if (!live || half == 1 || (lane & 1) != 0 || co >= p.Cout) return;
    const long long oi = ((((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo) * p.Cout + co;
    if (!index_ok(p.status, oi, p.out_elems)) return;
    float v = acc[0] + red[pl * 16 + co];
    const T* bias = static_cast<const T*>(p.bias);
    if (bias != nullptr) v += to_f32<T>(bias[co]);
    static_cast<T*>(p.out)[oi] = from_f32<T>(v);
}

// Small calls (a few thousand (pixel, 4-channel) units, e.g. the 16-channel
// fp32 contract call): one block per (output frame, band of band_h output
// rows).  The block first stages, as fp32 in shared memory and with 16-byte
// global loads where the layout allows, every weight of the call and, for
// each active tap of its frame, the input rows its band reads (zero rows and
// columns stand for the spatial padding, so the inner loop has no bounds
// checks).  Each thread then computes (pixel, 4 output channels) units from
// shared memory, four input channels per float4 read.  Global memory is read
// once per block and never in the reduction loop, which removes the load
// latency chains that bound these calls.
// Stage n values of T as fp32 into shared memory; with `vec` (n a multiple of
// 16 / sizeof(T), both ends 16-byte aligned) by 16-byte loads, four in flight
// per thread before their stores.
template <typename T>
__device__ __forceinline__ void stage_f32(float* dst, const T* src, long long n, bool vec,
                                          int tid, int nthreads) {
    constexpr int V = 16 / sizeof(T);
    if (vec) {
        const uint4* s = reinterpret_cast<const uint4*>(src);
        const int nv = (int)(n / V);
        constexpr int kU = 4;
        for (int i0 = tid; i0 < nv; i0 += kU * nthreads) {
            uint4 r[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u)
                if (i0 + u * nthreads < nv) r[u] = __ldg(s + i0 + u * nthreads);
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int i = i0 + u * nthreads;
                if (i >= nv) break;
                float f[V];
                unpack16<T>(r[u], f);
#pragma unroll
                for (int q = 0; q < V / 4; ++q)
                    reinterpret_cast<float4*>(dst + (long long)i * V)[q] =
                        make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
            }
        }
    } else {
        for (long long i = tid; i < n; i += nthreads) dst[i] = to_f32<T>(src[i]);
    }
}

// Shared-memory layout of the small-call kernel, in floats: the weights as
// [(k, r, s, ci)][Cout rounded up to 4] (one float4 holds the 4 output
// channels of a thread's unit), then the input rows as [tap][row][Wp][Cin + 4]
// (the 4 pad floats per pixel put the pixels a warp reads in different banks).
__host__ __device__ inline int simt_cout_pad(int Cout) { return (Cout + 3) / 4 * 4; }
__host__ __device__ inline long long simt_band_offset(int kt, int kh, int kw, int Cin, int Cout) {
    return (long long)kt * kh * kw * Cin * simt_cout_pad(Cout);
}
__host__ __device__ inline long long simt_smem_floats(int kt, int kh, int kw, int Cin, int Cout,
                                                      int rows_in, int Wp) {
    return simt_band_offset(kt, kh, kw, Cin, Cout) + (long long)kt * rows_in * Wp * (Cin + 4);
}

template <typename T>
__global__ void __launch_bounds__(256)
conv_simt_smem_kernel(const __grid_constant__ SimtParams p) {
    if ((int)blockIdx.x >= p.conv_blocks) {
        copy_new_cache(p.copy, blockIdx.x - p.conv_blocks, p.copy_blocks, threadIdx.x,
                       blockDim.x);
        return;
    }
    extern __shared__ __align__(16) float sm[];
    const int K = p.taps.kt * p.kh * p.kw * p.Cin;  // reduction length per output channel
    const int CoP = simt_cout_pad(p.Cout), CinP = p.Cin + 4;
    float* wsm = sm;                                 // [(k, r, s, ci)][CoP]
    float* band = sm + simt_band_offset(p.taps.kt, p.kh, p.kw, p.Cin, p.Cout);
                                                     // [kt][rows_in][Wp = W + 2 p_w][CinP]
    const int tid = threadIdx.x, nth = blockDim.x;
    const int frame = blockIdx.x / p.bands;
    const int bnd = blockIdx.x - frame * p.bands;
    const int o = frame % p.T_o, n = frame / p.T_o;
    const int y0 = bnd * p.band_h;
    const int V = sizeof(T) == 4 ? 4 : 8;  // elements per 16-byte load

    // ---- stage the weights, transposed to [(k, r, s, ci)][co] (four loads in
    // flight per thread), zeros for the padded output channels
    {
        const T* w = static_cast<const T*>(p.w);
        constexpr int kU = 4;
        for (int e0 = tid; e0 < K * CoP; e0 += kU * nth) {
            float r[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int e = e0 + u * nth;
                r[u] = 0.f;
                if (e >= K * CoP) continue;
                const int co = e / K;  // e = co * K + (k, r, s, ci): w[e] when co < Cout
                if (co < p.Cout && in_bounds(p.status, w + e, sizeof(T), w,
                                             p.w_floats * (long long)sizeof(T)))
                    r[u] = to_f32<T>(w[e]);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int e = e0 + u * nth;
                if (e >= K * CoP) break;
                const int co = e / K, ki = e - co * K;
                wsm[ki * CoP + co] = r[u];
            }
        }
    }
    const T* x = static_cast<const T*>(p.x);
    const T* cache = static_cast<const T*>(p.cache);
    const int row_elems = p.W * p.Cin;  // < 2^31: the rows fit in shared memory
    const int Wp_elems = p.Wp * CinP;
    int act[kMaxTaps], n_act = 0;
    for (int k = 0; k < p.taps.kt; ++k)
        if (o >= p.taps.o_l[k] && o < p.taps.o_h[k]) act[n_act++] = k;
    // zeros: padding columns, and rows outside the frame
    for (int e = tid; e < n_act * p.rows_in * Wp_elems; e += nth) {
        const int ai = e / Wp_elems, c = e - ai * Wp_elems;
        const int a = ai / p.rows_in, i = ai - a * p.rows_in;
        const int yi = y0 * p.s_h - p.p_h + i;
        if (yi < 0 || yi >= p.H || c < p.p_w * CinP || c >= (p.p_w + p.W) * CinP)
            band[((long long)act[a] * p.rows_in + i) * Wp_elems + c] = 0.f;
    }
    // rows inside the frame: one pass over (active tap, row, 16-byte vector),
    // four loads in flight per thread before their stores (a vector never
    // straddles two pixels: Cin is a multiple of its V channels)
    const bool row_vec = p.Cin % V == 0;
    const int rv = row_vec ? row_elems / V : row_elems;  // units per row
    const int total = n_act * p.rows_in * rv;
    constexpr int kU = 4;
    for (int e0 = tid; e0 < total; e0 += kU * nth) {
        uint4 r[kU];
        float* dst[kU];
        bool live[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int e = e0 + u * nth;
            live[u] = false;
            if (e >= total) continue;
            const int ai = e / rv, v = e - ai * rv;
            const int a = ai / p.rows_in, i = ai - a * p.rows_in;
            const int yi = y0 * p.s_h - p.p_h + i;
            if (yi < 0 || yi >= p.H) continue;
            const int t = o * p.taps.s_t + p.taps.delta[act[a]];
            const T* fr = t < p.cache_len
                              ? cache + (long long)ring_frame(n, t, p.cache_slots, p.cache_head) *
                                            p.H * row_elems
                              : x + ((long long)n * p.T_x + (t - p.cache_len)) * p.H * row_elems;
            const T* sp = fr + (long long)yi * row_elems + (long long)v * (row_vec ? V : 1);
            if (!in_bounds(p.status, sp, (row_vec ? 16 : (int)sizeof(T)),
                           t < p.cache_len ? (const void*)cache : (const void*)x,
                           t < p.cache_len ? p.copy.cache_bytes : p.copy.x_bytes))
                continue;
            const int el = v * (row_vec ? V : 1);    // element of the row
            const int px = el / p.Cin, c = el - px * p.Cin;
            dst[u] = band + ((long long)act[a] * p.rows_in + i) * Wp_elems +
                     (long long)(p.p_w + px) * CinP + c;
            live[u] = true;
            if (row_vec)
                r[u] = __ldg(reinterpret_cast<const uint4*>(sp));
            else
                r[u].x = __float_as_uint(to_f32<T>(*sp));
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (!live[u]) continue;
            if (row_vec) {
                float f[V];
                unpack16<T>(r[u], f);
#pragma unroll
                for (int q = 0; q < V / 4; ++q)
                    reinterpret_cast<float4*>(dst[u])[q] =
                        make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
            } else {
                *dst[u] = __uint_as_float(r[u].x);
            }
        }
    }
    __syncthreads();

    // ---- one (pixel, 4-channel group) unit per thread step
    const int units = p.band_h * p.W_o * p.co_groups;
    for (int u = tid; u < units; u += nth) {
        const int cog = u % p.co_groups;
        const int px = u / p.co_groups;
        const int xo = px % p.W_o, yl = px / p.W_o;
        const int yo = y0 + yl;
        if (yo >= p.H_o) continue;
        const int co0 = cog * kSimtCoT;
        float acc[kSimtCoT] = {0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < p.taps.kt; ++k) {
            if (!(o >= p.taps.o_l[k] && o < p.taps.o_h[k])) continue;
            for (int r = 0; r < p.kh; ++r) {
                const float* zrow = band + ((long long)k * p.rows_in + yl * p.s_h + r * p.d_h) *
                                               Wp_elems;
                for (int s = 0; s < p.kw; ++s) {
                    const float* z = zrow + (long long)(xo * p.s_w + s * p.d_w) * CinP;
                    // this tap's weights: float4 of output channels co0..co0+3 per ci
                    const float* wk = wsm + (long long)(((k * p.kh + r) * p.kw + s) * p.Cin) * CoP + co0;
                    if (p.Cin % 4 == 0) {
#pragma unroll 4
                        for (int ci = 0; ci < p.Cin; ci += 4) {
                            const float4 z4 = *reinterpret_cast<const float4*>(z + ci);
                            const float zz[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float4 w4 =
                                    *reinterpret_cast<const float4*>(wk + (long long)(ci + e) * CoP);
                                acc[0] = fmaf(zz[e], w4.x, acc[0]);
                                acc[1] = fmaf(zz[e], w4.y, acc[1]);
                                acc[2] = fmaf(zz[e], w4.z, acc[2]);
                                acc[3] = fmaf(zz[e], w4.w, acc[3]);
                            }
                        }
                    } else {
                        for (int ci = 0; ci < p.Cin; ++ci) {
                            const float4 w4 =
                                *reinterpret_cast<const float4*>(wk + (long long)ci * CoP);
                            acc[0] = fmaf(z[ci], w4.x, acc[0]);
                            acc[1] = fmaf(z[ci], w4.y, acc[1]);
                            acc[2] = fmaf(z[ci], w4.z, acc[2]);
                            acc[3] = fmaf(z[ci], w4.w, acc[3]);
                        }
                    }
                }
            }
        }
        const T* bias = static_cast<const T*>(p.bias);
        const long long out_i = (((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo;
        T* out = static_cast<T*>(p.out) + out_i * p.Cout;
#pragma unroll
        for (int j = 0; j < kSimtCoT; ++j) {
            if (co0 + j >= p.Cout) break;
            if (!index_ok(p.status, out_i * p.Cout + co0 + j, p.out_elems)) break;
            float v = acc[j];
            if (bias != nullptr) v += to_f32<T>(bias[co0 + j]);
            out[co0 + j] = from_f32<T>(v);
        }
    }
}

// Large calls with at most 4 output channels (the decoder's RGB output conv,
// 96 -> 3 channels at full resolution), unit spatial stride: every input
// value feeds only Cout FMAs, so the kernel is bound by how often an input
// value is read, not by the arithmetic.  A block of 256 threads owns 8 output
// rows x 128 output columns of one frame; a thread owns 4 adjacent pixels of
// one row and all (<= 4) output channels.
//   * The weights are staged once per block as fp32, [k][r][s][ci][4 channels],
//     so one broadcast float4 read gives all output channels of a tap.
//   * Per (active tap, block of 8 input channels) the block stages the input
//     patch the tile reads, (8 - 1 + (kh - 1) d_h + 1) rows x (128 + (kw - 1)
//     d_w) columns, as fp32 in [channel quad][row][column][4] order (a thread
//     loads 16 bytes of one pixel: 8 bf16 or 4 fp32 channels), zeros outside
//     the frame; lanes then read consecutive 16-byte words.
//   * A thread reads the 4 + KW - 1 patch columns of a kernel row once into
//     registers and uses each for all KW column taps (KW = kw in {1, 3}, unit
//     column dilation: compile-time window indices).
constexpr int kTileRows = 8, kTileCols = 128, kTilePx = 4, kTileCc = 8;
constexpr int kTilePf = 8;  // 16-byte loads of the next patch a thread holds (x 256 threads)

__host__ __device__ inline int simt_tile_rows_in(int kh, int d_h) {
    return kTileRows - 1 + (kh - 1) * d_h + 1;
}
__host__ __device__ inline int simt_tile_cols_in(int kw, int d_w) {
    return kTileCols + (kw - 1) * d_w;
}
// 16-byte loads of one patch (element size `esize`): must not exceed kTilePf x 256
__host__ __device__ inline int simt_tile_patch_loads(int kh, int kw, int d_h, int d_w, int esize) {
    return simt_tile_rows_in(kh, d_h) * simt_tile_cols_in(kw, d_w) * (kTileCc * esize / 16);
}
// Patch columns are stored permuted, column c at (c % 4) * C4 + c / 4 with
// C4 = ceil(cols / 4): a warp whose lane l reads column 4 l + j then touches
// 32 consecutive 16-byte words (no bank conflicts), and the permuted index of
// 4 l + j is (j % 4) * C4 + l + j / 4.
__host__ __device__ inline int simt_tile_c4(int kw, int d_w) {
    return (simt_tile_cols_in(kw, d_w) + 3) / 4;
}
// shared memory in floats: weights [kt*kh*kw*Cin][4] + one patch [2 quads][rows][4*C4][4]
__host__ __device__ inline long long simt_tile_smem_floats(int kt, int kh, int kw, int Cin,
                                                           int d_h, int d_w) {
    return (long long)kt * kh * kw * Cin * 4 +
           (long long)(kTileCc / 4) * simt_tile_rows_in(kh, d_h) * 4 * simt_tile_c4(kw, d_w) * 4;
}

template <typename T, int KW>
__global__ void __launch_bounds__(256, 2)
conv_simt_tile_kernel(const __grid_constant__ SimtParams p) {
    if ((int)blockIdx.x >= p.conv_blocks) {
        copy_new_cache(p.copy, blockIdx.x - p.conv_blocks, p.copy_blocks, threadIdx.x,
                       blockDim.x);
        return;
    }
    extern __shared__ __align__(16) float sm[];
    const int taps2d = p.kh * p.kw;
    float* wsm = sm;                                         // [kt*kh*kw*Cin][4]
    float* patch = sm + (long long)p.taps.kt * taps2d * p.Cin * 4;
    const int rows_in = simt_tile_rows_in(p.kh, p.d_h);
    const int cols_in = simt_tile_cols_in(p.kw, p.d_w);
    const int C4 = simt_tile_c4(p.kw, p.d_w);
    const int row_pos = 4 * C4;                              // permuted positions per row
    const int quad_stride = rows_in * row_pos * 4;           // floats per channel quad

    const int tid = threadIdx.x;
    const int tiles_x = (p.W_o + kTileCols - 1) / kTileCols;
    const int tiles_y = (p.H_o + kTileRows - 1) / kTileRows;
    const int tile = blockIdx.x % (tiles_x * tiles_y);
    const int frame = blockIdx.x / (tiles_x * tiles_y);
    const int o = frame % p.T_o, n = frame / p.T_o;
    const int oy0 = (tile / tiles_x) * kTileRows, ox0 = (tile % tiles_x) * kTileCols;
    const int iy0 = oy0 - p.p_h, ix0 = ox0 - p.p_w;          // patch origin in the frame (s = 1)

    // ---- weights, once: [co][k][r][s][ci] -> [(k, r, s, ci)][co], four
    // loads in flight per thread
    const T* w = static_cast<const T*>(p.w);
    const int wk = p.taps.kt * taps2d * p.Cin;
    for (int e0 = tid; e0 < wk * 4; e0 += 4 * (int)blockDim.x) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u * (int)blockDim.x;
            v[u] = 0.f;
            if (e >= wk * 4) continue;
            const int co = e / wk, rest = e - co * wk;
            if (co < p.Cout && in_bounds(p.status, w + (long long)co * wk + rest, sizeof(T), w,
                                         p.w_floats * (long long)sizeof(T)))
                v[u] = to_f32<T>(w[(long long)co * wk + rest]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u * (int)blockDim.x;
            if (e >= wk * 4) break;
            const int co = e / wk, rest = e - co * wk;
            wsm[rest * 4 + co] = v[u];
        }
    }

    const int ty = tid >> 5, lane = tid & 31;                // output row ty, pixels 4 lane ..
    float acc[kTilePx][4];
#pragma unroll
    for (int i = 0; i < kTilePx; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;

    // ---- steps (active tap, block of 8 channels); each thread holds its
    // share of the next step's patch (<= kTilePf 16-byte loads, checked by the
    // planner) in registers while the current step's FMAs run
    const T* x = static_cast<const T*>(p.x);
    const T* cache = static_cast<const T*>(p.cache);
    constexpr int V = 16 / (int)sizeof(T);                   // channels per 16-byte load
    constexpr int loads_px = kTileCc / V;                    // 1 (bf16) or 2 (fp32)
    const int nload = rows_in * cols_in * loads_px;
    int act[kMaxTaps], n_act = 0;
    for (int k = 0; k < p.taps.kt; ++k)
        if (o >= p.taps.o_l[k] && o < p.taps.o_h[k]) act[n_act++] = k;
    const int chunks = p.Cin / kTileCc;
    const int steps = n_act * chunks;
    uint4 pf[kTilePf];
    auto fetch = [&](int step) {
        const int k = act[step / chunks], c0 = (step % chunks) * kTileCc;
        const int t = o * p.taps.s_t + p.taps.delta[k];
        const T* fr = t < p.cache_len
                          ? cache + (long long)ring_frame(n, t, p.cache_slots, p.cache_head) *
                                        p.H * p.W * p.Cin
                          : x + ((long long)n * p.T_x + (t - p.cache_len)) * p.H * p.W * p.Cin;
        const void* fbase = t < p.cache_len ? (const void*)cache : (const void*)x;
        const long long fbytes = t < p.cache_len ? p.copy.cache_bytes : p.copy.x_bytes;
#pragma unroll
        for (int i = 0; i < kTilePf; ++i) {
            pf[i] = make_uint4(0u, 0u, 0u, 0u);  // zeros outside the frame
            const int e = tid + i * (int)blockDim.x;
            if (e >= nload) continue;
            const int h = e % loads_px, pix = e / loads_px;
            const int ry = pix / cols_in, rx = pix - ry * cols_in;
            const int yi = iy0 + ry, xi = ix0 + rx;
            if (yi < 0 || yi >= p.H || xi < 0 || xi >= p.W) continue;
            const T* sp = fr + ((long long)yi * p.W + xi) * p.Cin + c0 + h * V;
            if (in_bounds(p.status, sp, 16, fbase, fbytes))
                pf[i] = __ldg(reinterpret_cast<const uint4*>(sp));
        }
    };
    fetch(0);
    for (int step = 0; step < steps; ++step) {
        const int k = act[step / chunks], c0 = (step % chunks) * kTileCc;
        __syncthreads();  // the previous step's patch is no longer read
        // ---- the held loads into the patch, [channel quad][row][column][4]
#pragma unroll
        for (int i = 0; i < kTilePf; ++i) {
            const int e = tid + i * (int)blockDim.x;
            if (e >= nload) break;
            const int h = e % loads_px, pix = e / loads_px;
            const int ry = pix / cols_in, rx = pix - ry * cols_in;
            const int pos = ry * row_pos + (rx & 3) * C4 + (rx >> 2);
            float g[V];
            unpack16<T>(pf[i], g);
#pragma unroll
            for (int q = 0; q < V / 4; ++q)
                *reinterpret_cast<float4*>(patch + (h * (V / 4) + q) * quad_stride + pos * 4) =
                    make_float4(g[4 * q], g[4 * q + 1], g[4 * q + 2], g[4 * q + 3]);
        }
        __syncthreads();
        if (step + 1 < steps) fetch(step + 1);  // in flight during the FMAs below
        // ---- accumulate: kernel rows, channel quads, the register window
        for (int r = 0; r < p.kh; ++r) {
            const int prow = ty + r * p.d_h;
#pragma unroll
            for (int q = 0; q < kTileCc / 4; ++q) {
                float4 z[kTilePx + KW - 1];
                const float* zrow = patch + q * quad_stride + (prow * row_pos + lane) * 4;
#pragma unroll
                for (int j = 0; j < kTilePx + KW - 1; ++j)  // column 4 lane + j
                    z[j] = *reinterpret_cast<const float4*>(zrow + ((j & 3) * C4 + (j >> 2)) * 4);
#pragma unroll
                for (int sx = 0; sx < KW; ++sx) {
                    const float* wq =
                        wsm + ((((k * p.kh + r) * KW + sx) * p.Cin) + c0 + q * 4) * 4;
                    const float4 w0 = *reinterpret_cast<const float4*>(wq);
                    const float4 w1 = *reinterpret_cast<const float4*>(wq + 4);
                    const float4 w2 = *reinterpret_cast<const float4*>(wq + 8);
                    const float4 w3 = *reinterpret_cast<const float4*>(wq + 12);
#pragma unroll
                    for (int i = 0; i < kTilePx; ++i) {
                        const float4 zz = z[i + sx];
                        acc[i][0] = fmaf(zz.x, w0.x, fmaf(zz.y, w1.x, fmaf(zz.z, w2.x, fmaf(zz.w, w3.x, acc[i][0]))));
                        acc[i][1] = fmaf(zz.x, w0.y, fmaf(zz.y, w1.y, fmaf(zz.z, w2.y, fmaf(zz.w, w3.y, acc[i][1]))));
                        acc[i][2] = fmaf(zz.x, w0.z, fmaf(zz.y, w1.z, fmaf(zz.z, w2.z, fmaf(zz.w, w3.z, acc[i][2]))));
                        acc[i][3] = fmaf(zz.x, w0.w, fmaf(zz.y, w1.w, fmaf(zz.z, w2.w, fmaf(zz.w, w3.w, acc[i][3]))));
                    }
                }
            }
        }
    }

    // ---- bias once, round, store
    const T* bias = static_cast<const T*>(p.bias);
    const int yo = oy0 + ty;
    if (yo >= p.H_o) return;
#pragma unroll
    for (int i = 0; i < kTilePx; ++i) {
        const int xo = ox0 + lane * kTilePx + i;
        if (xo >= p.W_o) break;
        const long long out_i = (((long long)n * p.T_o + o) * p.H_o + yo) * p.W_o + xo;
        T* out = static_cast<T*>(p.out) + out_i * p.Cout;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (c >= p.Cout) break;
            if (!index_ok(p.status, out_i * p.Cout + c, p.out_elems)) break;
            float v = acc[i][c];
            if (bias != nullptr) v += to_f32<T>(bias[c]);
            out[c] = from_f32<T>(v);
        }
    }
}

}  // namespace ccv3d
