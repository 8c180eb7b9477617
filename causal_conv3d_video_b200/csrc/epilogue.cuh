// epilogue.cuh -- accumulator -> bias -> bf16 -> TMA tensor store.
//
// After a tile's last MMA the shared-memory ring is idle, so the epilogue
// stages its output there: each thread owns one accumulator row (one output
// pixel) and writes bf16 channels into blocks of `kCh` channels laid out with
// the same swizzle the TMA unit uses (so the 16-byte writes of a warp spread
// over all banks), then one thread stores each block with a tensor store.
// The output tensor map clips rows past H_o/W_o and channels past Cout, so
// ragged tiles need no per-element masking.
#pragma once
#include <cuda_bf16.h>

#include "checked.cuh"
#include "params.h"
#include "ptx.cuh"

namespace ccv3d {

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* m, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];"
        ::"l"(reinterpret_cast<uint64_t>(m)), "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_group_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_group0() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Named barrier over the four epilogue warps (barrier 1, 128 threads).
__device__ __forceinline__ void epi_bar() {
    asm volatile("bar.sync 1, 128;" ::: "memory");
}

// The same barrier, returning the AND of `v` over the 128 epilogue threads,
// so that decisions taken from bounded waits are uniform across them.
__device__ __forceinline__ bool epi_bar_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// 16-byte chunk c of row `row` inside a block of kRowB-byte rows, swizzled the
// way TMA's 128/64/32-byte modes place it (chunk bits XOR address bits 7+).
template <int kRowB>
__device__ __forceinline__ int swizzled_chunk(int c, int row) {
    if constexpr (kRowB == 128) return c ^ (row & 7);
    else if constexpr (kRowB == 64) return c ^ ((row >> 1) & 3);
    else return c ^ ((row >> 2) & 1);
}

// Channels per store block for a Cout tile of `bn` columns (a multiple of 16).
__host__ __device__ constexpr int out_block_channels(int bn) {
    return bn % 64 == 0 ? 64 : (bn % 32 == 0 ? 32 : 16);
}

// Store this CTA's 128 x bn accumulator slab (TMEM lanes 0-127, columns from
// `tmem_acc`) as bf16 of (acc + bias) to output channels [co0, co0 + bn) of
// the box whose first pixel is (x0, y0) in output frame `frame`.
// `stage` is 1024-byte aligned shared memory of at least 128 * bn * 2 bytes.
// Called by the 128 epilogue threads (etid = 0..127, TMEM lane quarter q).
template <int kCh>
__device__ __forceinline__ void epilogue_store(const TcParams& p, uint32_t tmem_acc,
                                               bool have_acc, const float* bias_s, int bn,
                                               uint8_t* stage, int co0, int x0, int y0,
                                               int frame, int etid, int q, int lane,
                                               bool do_store) {
    constexpr int kRowB = kCh * 2;
    const int row = q * 32 + lane;
    const int nblk = bn / kCh;
    for (int b = 0; b < nblk; ++b) {
        uint32_t v[kCh];
#pragma unroll
        for (int j = 0; j < kCh / 16; ++j)
            tmem_ld_32x32b_x16(tmem_acc + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kCh + j * 16),
                               *reinterpret_cast<uint32_t(*)[16]>(&v[j * 16]));
        tmem_ld_wait();
        uint8_t* blk = stage + (size_t)b * (kTileM * kRowB) + (size_t)row * kRowB;
#pragma unroll
        for (int c = 0; c < kCh / 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int ch = b * kCh + c * 8 + 2 * i;
                const float a0 = (have_acc ? __uint_as_float(v[c * 8 + 2 * i]) : 0.f) + bias_s[ch];
                const float a1 =
                    (have_acc ? __uint_as_float(v[c * 8 + 2 * i + 1]) : 0.f) + bias_s[ch + 1];
                const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
                w[i] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(blk + (swizzled_chunk<kRowB>(c, row) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    fence_proxy_async_smem();  // generic-proxy writes -> visible to the TMA unit
    epi_bar();
    if (etid == 0 && do_store && index_ok(p.status, frame, (long long)p.N * p.T_o)) {
        for (int b = 0; b < nblk; ++b)
            tma_store_4d(&p.tmap_out, smem_u32(stage + (size_t)b * (kTileM * kRowB)),
                         co0 + b * kCh, x0, y0, frame);
        bulk_commit_group();
        bulk_wait_group0();  // stores complete before the CTA reuses or releases the stage
    }
}

// The same store, each warp on its own: warp q converts its 32 accumulator
// rows (pixels 32q .. 32q+31 of the box, in row-major order) block by block
// and, as soon as a block is in shared memory, its lane 0 stores that 32-pixel
// slab with a tensor store (p.tmap_out_w).  No barrier between the warps, and
// the stores of one block overlap the conversion of the next.
template <int kCh>
__device__ __forceinline__ void epilogue_store_warp(const TcParams& p, uint32_t tmem_acc,
                                                    bool have_acc, const float* bias_s, int bn,
                                                    uint8_t* stage, int co0, int x0, int y0,
                                                    int frame, int q, int lane, bool do_store) {
    constexpr int kRowB = kCh * 2;
    const int row = q * 32 + lane;
    const int nblk = bn / kCh;
    const int bw = p.box_w;
    const int sx = bw >= 32 ? x0 + (32 * q) % bw : x0;
    const int sy = bw >= 32 ? y0 + (32 * q) / bw : y0 + q * (32 / bw);
    // a slab that starts past the frame's edge has nothing to store
    const bool slab = do_store && sx < p.W_o && sy < p.H_o &&
                      index_ok(p.status, frame, (long long)p.N * p.T_o);
    for (int b = 0; b < nblk; ++b) {
        uint32_t v[kCh];
#pragma unroll
        for (int j = 0; j < kCh / 16; ++j)
            tmem_ld_32x32b_x16(tmem_acc + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kCh + j * 16),
                               *reinterpret_cast<uint32_t(*)[16]>(&v[j * 16]));
        tmem_ld_wait();
        uint8_t* blk = stage + (size_t)b * (kTileM * kRowB) + (size_t)row * kRowB;
#pragma unroll
        for (int c = 0; c < kCh / 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int ch = b * kCh + c * 8 + 2 * i;
                const float a0 = (have_acc ? __uint_as_float(v[c * 8 + 2 * i]) : 0.f) + bias_s[ch];
                const float a1 =
                    (have_acc ? __uint_as_float(v[c * 8 + 2 * i + 1]) : 0.f) + bias_s[ch + 1];
                const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
                w[i] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(blk + (swizzled_chunk<kRowB>(c, row) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();  // this lane's writes -> visible to the TMA unit
        __syncwarp();
        if (lane == 0 && slab)
            tma_store_4d(&p.tmap_out_w,
                         smem_u32(stage + (size_t)b * (kTileM * kRowB) + (size_t)(q * 32) * kRowB),
                         co0 + b * kCh, sx, sy, frame);
    }
    if (lane == 0 && slab) {
        bulk_commit_group();
        bulk_wait_group0();  // stores complete before the CTA releases the stage
    }
    __syncwarp();
}

}  // namespace ccv3d
