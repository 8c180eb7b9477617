// conv_tc2h.cuh -- CTA-pair implicit-GEMM Conv3D with the input row halo
// loaded once per (temporal tap, channel block).
//
// When a tile is one output row of 128 pixels (box 1 x 128, unit W stride),
// the A operands of the kw spatial taps s of one kernel row r are the same
// strip of input pixels shifted by s*d_w: rows s*d_w .. s*d_w+127 of the
// 128 + (kw-1)*d_w pixel strip.  One pipeline stage therefore holds, for one
// active temporal tap k and one block of BK input channels, the kh strips
// (one per kernel row r, each loaded by one TMA box) and the kh*kw weight
// tiles; the MMA issuer walks (r, s) inside the stage by offsetting the A
// descriptor's start address by s*d_w rows.  Each input element crosses from
// L2 to the SM about (128 + (kw-1)*d_w)/128 times per (k, r) instead of kw
// times, which matters on the thin-channel, full-resolution decoder calls
// where the A operand dominates the operand traffic.
//
// Pair structure, barriers, epilogue and bounded waits are those of
// conv_tc2.cuh.
#pragma once
#include <cuda_bf16.h>

#include "cache_copy.cuh"
#include "conv_tc.cuh"
#include "epilogue.cuh"
#include "kwalk.cuh"
#include "params.h"
#include "ptx.cuh"

namespace ccv3d {

// Bytes of one halo strip of `halo_w` pixels x BK channels, 1024-aligned.
template <int BK>
__host__ __device__ constexpr size_t halo_strip_bytes(int halo_w) {
    return ((size_t)halo_w * TcSmem<BK>::kRowBytes + 1023) / 1024 * 1024;
}

// One stage: kh strips + kh*kw weight tiles of bn/2 rows (per CTA).
template <int BK>
__host__ __device__ constexpr size_t tc2h_stage_bytes(int bn, int kh, int kw, int halo_w) {
    return (size_t)kh * halo_strip_bytes<BK>(halo_w) +
           (size_t)kh * kw * (bn / 2) * TcSmem<BK>::kRowBytes;
}

template <int BK>
__host__ __device__ constexpr size_t tc2h_smem_bytes(int bn, int stages, int kh, int kw,
                                                     int halo_w) {
    return 1024 + ring_bytes((size_t)stages * tc2h_stage_bytes<BK>(bn, kh, kw, halo_w), bn) +
           (size_t)(2 * stages + 1) * 8 + 16 + (size_t)bn * 4;
}

template <int BK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
conv_tc2h_kernel(const __grid_constant__ TcParams p) {
    constexpr int kRow = TcSmem<BK>::kRowBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = p.stages;
    const int BN = p.BN;
    const int BNs = BN / p.n_sub;
    const int hB = BNs / 2;
    const int kBc = (BN / 2) * kRow;  // weight bytes per CTA per (r, s)
    const int kBh = hB * kRow;
    const int halo_w = p.halo_w;
    const int kStrip = (int)halo_strip_bytes<BK>(halo_w);
    const int kAst = p.kh * kStrip;                 // strips of one stage
    const int kStage = kAst + p.kh * p.kw * kBc;    // whole stage
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(
        smem + ring_bytes((size_t)stages * kStage, BN));
    uint64_t* empty_bar = full_bar + stages;
    uint64_t* acc_bar = empty_bar + stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);
    float* bias_s = reinterpret_cast<float*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    const int pair = blockIdx.x >> 1;
    const int n_tile = pair % p.tiles_n;
    const int m_pair = pair / p.tiles_n;
    // output frame fastest: the tiles that read one source frame through
    // different temporal taps run close together and share it in L2
    const int frames = p.N * p.T_o;
    const int frame = m_pair % frames;
    const int box = (m_pair / frames) * 2 + (int)rank;
    const int o = frame % p.T_o;
    const int n = frame / p.T_o;
    int tx = 0, ty = p.tiles_y;
    if (box < p.tiles_x * p.tiles_y) {
        tx = box % p.tiles_x;
        ty = box / p.tiles_x;
    }
    int act[kMaxTaps];
    const int n_act = active_tap_list(p, o, act);
    const int iters = n_act * p.n_cb;  // stages of this tile: (tap, channel block)

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        mbar_init(smem_u32(acc_bar), 1);
        fence_mbar_init();
        tma_prefetch_desc(&p.tmap_x);
        if (p.cache_len > 0) tma_prefetch_desc(&p.tmap_c);
        tma_prefetch_desc(&p.tmap_w);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
        tmem_relinquish_pair();
    }
    if (warp >= 2) {
        for (int i = threadIdx.x - 64; i < BN; i += 128) {
            const int co = n_tile * BN + i;
            float b = 0.f;
            if (p.bias != nullptr && co < p.Cout && index_ok(p.status, co, p.Cout))
                b = __bfloat162float(__ushort_as_bfloat16(p.bias[co]));
            bias_s[i] = b;
        }
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && iters > 0) {
            // ------------------------------- TMA producer (both CTAs)
            const int rot = (int)(((long long)pair * iters) / p.rot_div) % iters;
            const uint32_t pair_bytes = 2u * (uint32_t)(p.kh * halo_w * kRow + p.kh * p.kw * kBc);
            const int xs = tx * p.box_w - p.p_w;  // first pixel of the strip (s_w = 1)
            const int y_out = ty * p.box_h;
            int ti = rot / p.n_cb, cb = rot - ti * p.n_cb;
            TapSrc ts = tap_source(p, act[ti], n, o);
            Ring ring;
            for (int it = 0; it < iters; ++it) {
                if (it >= stages && !mbar_wait(smem_u32(&empty_bar[ring.st]), ring.ph ^ 1u,
                                               p.status, p.wait_limit_ns))
                    break;
                uint8_t* st_base = smem + (size_t)ring.st * kStage;
                const uint32_t fb_local = smem_u32(&full_bar[ring.st]);
                if (leader) mbar_arrive_expect_tx(fb_local, pair_bytes);
                const uint32_t fb = pair_leader_addr(fb_local);
                for (int r = 0; r < p.kh; ++r)
                    tma_load_4d_pair(smem_u32(st_base + r * kStrip), ts.map, fb, cb * BK, xs,
                                     y_out * p.s_h + r * p.d_h - p.p_h, ts.frame);
                uint8_t* b_base = st_base + kAst;
                for (int rs = 0; rs < p.kh * p.kw; ++rs)
                    for (int j = 0; j < p.n_sub; ++j)
                        tma_load_3d_pair(smem_u32(b_base + rs * kBc + j * kBh), &p.tmap_w, fb,
                                         cb * BK, ts.wtap + rs,
                                         n_tile * BN + j * BNs + (int)rank * hB);
                ring.next(stages);
                if (++cb == p.n_cb) {
                    cb = 0;
                    if (++ti == n_act) ti = 0;
                    ts = tap_source(p, act[ti], n, o);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------ MMA issuer (even CTA only)
            const uint32_t idesc = idesc_bf16_m256((uint32_t)BNs);
            const uint64_t d0 = smem_desc_kmajor(smem_u32(smem), kRow);
            Ring ring;
            for (int it = 0; it < iters; ++it) {
                if (!mbar_wait(smem_u32(&full_bar[ring.st]), ring.ph, p.status, p.wait_limit_ns))
                    break;
                tc_fence_after();
                const uint32_t st_off = (uint32_t)ring.st * (uint32_t)kStage;
                for (int r = 0; r < p.kh; ++r)
                    for (int s = 0; s < p.kw; ++s) {
                        // A: the strip of row r shifted by s*d_w pixels (rows)
                        const uint64_t a_desc =
                            d0 + (uint64_t)((st_off + r * kStrip + s * p.d_w * kRow) >> 4);
                        const uint64_t b_desc =
                            d0 + (uint64_t)((st_off + kAst + (r * p.kw + s) * kBc) >> 4);
                        const bool first = it == 0 && r == 0 && s == 0;
                        for (int j = 0; j < p.n_sub; ++j) {
                            const uint64_t bj = b_desc + (uint64_t)((j * kBh) >> 4);
#pragma unroll
                            for (int kk = 0; kk < BK / 16; ++kk)
                                umma_bf16_pair(tmem_base + (uint32_t)(j * BNs), a_desc + 2u * kk,
                                               bj + 2u * kk, idesc,
                                               (first && kk == 0) ? 0u : 1u);
                        }
                    }
                umma_commit_pair(smem_u32(&empty_bar[ring.st]), (uint16_t)0x3);
                ring.next(stages);
            }
            umma_commit_pair(smem_u32(acc_bar), (uint16_t)0x3);
        }
        __syncwarp();
    } else {
        // ------------------------- new_cache slice, then this CTA's epilogue
        const int etid = threadIdx.x - 64;
        copy_new_cache(p.copy, blockIdx.x, gridDim.x, etid, 128);
        const bool ok = mbar_wait(smem_u32(acc_bar), 0, p.status, p.wait_limit_ns);
        tc_fence_after();
        const int q = warp & 3;
        const int fo = n * p.T_o + o;
        const int x0 = tx * p.box_w, y0 = ty * p.box_h, co0 = n_tile * BN;
        const bool have_acc = iters > 0;
        const bool store = ok && ty < p.tiles_y;
        switch (out_block_channels(BN)) {
            case 64: epilogue_store<64>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, fo, etid, q, lane, store); break;
            case 32: epilogue_store<32>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, fo, etid, q, lane, store); break;
            default: epilogue_store<16>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, fo, etid, q, lane, store); break;
        }
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, (uint32_t)p.tmem_cols);
    }
}

}  // namespace ccv3d
