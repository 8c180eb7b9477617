// conv_tc2.cuh -- the implicit-GEMM Conv3D on CTA pairs (tcgen05 cta_group::2).
//
// Same GEMM view as conv_tc.cuh (rows = output pixels of one output frame,
// columns = Cout, reduction over active taps x kh x kw x Cin), but a cluster
// of two CTAs computes a 256 x BN tile with M=256 pair MMAs:
//   * each CTA loads its own 128-pixel A box (two neighbouring boxes of the
//     same output frame, so both CTAs walk the same active taps) and HALF of
//     the weight rows of every MMA; the even CTA issues the MMAs, which read
//     A and B from both CTAs' shared memory;
//   * both CTAs' TMA loads complete on the even CTA's "full" barrier (the
//     even producer posts the byte count for the pair), and the even CTA's
//     tcgen05.commit releases the stage on both CTAs' "empty" barriers;
//   * each CTA holds its 128 accumulator rows in its own TMEM and runs its own
//     epilogue (bias, bf16, TMA store staged in its idle ring) and its slice
//     of the new_cache copy.
// Per SM this halves the weight bytes pulled from L2 per FLOP, the operand
// that dominates on the wide-Cout decoder signatures.  No load is
// multicast.  All waits are bounded.
#pragma once
#include <cuda_bf16.h>

#include "cache_copy.cuh"
#include "conv_tc.cuh"
#include "epilogue.cuh"
#include "kwalk.cuh"
#include "params.h"
#include "ptx.cuh"

namespace ccv3d {

template <int BK>
__host__ __device__ constexpr size_t tc2_smem_bytes(int bn, int stages) {
    // per CTA: A box (128 rows) + half of the BN weight rows per stage
    return 1024 +
           ring_bytes((size_t)stages * (TcSmem<BK>::kABytes + (size_t)(bn / 2) * TcSmem<BK>::kRowBytes),
                      bn) +
           (size_t)(2 * stages + 1) * 8 + 16 + (size_t)bn * 4;
}

template <int BK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
conv_tc2_kernel(const __grid_constant__ TcParams p) {
    constexpr int kRow = TcSmem<BK>::kRowBytes;
    constexpr int kA = TcSmem<BK>::kABytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = p.stages;
    const int BN = p.BN;            // accumulator columns of the pair tile
    const int BNs = BN / p.n_sub;   // N of one pair MMA (<= 256)
    const int hB = BNs / 2;         // weight rows per CTA per MMA
    const int kBc = (BN / 2) * kRow;  // weight bytes per CTA per stage
    const int kBh = hB * kRow;
    uint8_t* sA = smem;
    uint8_t* sB = smem + (size_t)stages * kA;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(
        smem + ring_bytes((size_t)stages * (kA + kBc), BN));
    uint64_t* empty_bar = full_bar + stages;
    uint64_t* acc_bar = empty_bar + stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);
    float* bias_s = reinterpret_cast<float*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    // ---- pair tile: (pair of boxes, n, o) x n_tile
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
    int tx = 0, ty = p.tiles_y;  // a box past the frame's last one stores nothing
    if (box < p.tiles_x * p.tiles_y) {
        tx = box % p.tiles_x;
        ty = box / p.tiles_x;
    }

    int n_active = 0;
#pragma unroll
    for (int k = 0; k < kMaxTaps; ++k)
        if (k < p.taps.kt && o >= p.taps.o_l[k] && o < p.taps.o_h[k]) ++n_active;
    const int iters = n_active * p.kh * p.kw * p.n_cb;

    if (warp == 2) {
        // An epilogue warp (idle until the accumulator is complete) arrives
        // at the pair's rendezvous at once -- the set-up needs nothing from
        // it -- and its lane 0 then fetches the first stages' operand boxes
        // into L2 while thread 0 and warp 1 set up (barriers, TMEM), so that
        // the launch's first DRAM round trip overlaps the set-up; the
        // producer's loads of these stages then hit L2.
        cluster_arrive();
        if (lane == 0 && iters > 0) {
            int act[kMaxTaps];
            const int n_act = active_tap_list(p, o, act);
            const int rot = (int)(((long long)pair * iters) / p.rot_div) % iters;
            const int ybase = ty * p.box_h * p.s_h - p.p_h;
            const int xbase = tx * p.box_w * p.s_w - p.p_w;
            KWalk w;
            w.set(rot, p);
            TapSrc ts = tap_source(p, act[w.ti], n, o);
            const int first = stages < iters ? stages : iters;
            for (int it = 0; it < first; ++it) {
                // (start coordinates kept inside the frame: a prefetch only
                // warms L2, so a box shifted off the padding is as good)
                const int xp = min(max(xbase + w.s * p.d_w, 0), p.W - 1);
                const int yp = min(max(ybase + w.r * p.d_h, 0), p.H - 1);
                tma_prefetch_l2_4d(ts.map, w.cb * BK, xp, yp, ts.frame);
                const int wrow = ts.wtap + w.r * p.kw + w.s;
                for (int j = 0; j < p.n_sub; ++j)
                    tma_prefetch_l2_3d(&p.tmap_w, w.cb * BK, wrow,
                                       n_tile * BN + j * BNs + (int)rank * hB);
                if (w.next(p)) {
                    if (w.ti == n_act) w.ti = 0;
                    ts = tap_source(p, act[w.ti], n, o);
                }
            }
        }
        __syncwarp();
    }
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
    tc_fence_before();
    // barriers initialised in both CTAs before any remote use (warp 2 has
    // arrived already)
    if (warp != 2) cluster_arrive();
    cluster_wait();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && iters > 0) {
            // --------------------------------- TMA producer (both CTAs)
            // Each pair starts its reduction at a different k-block, so
            // pairs running at the same time read different weight rows.
            int act[kMaxTaps];
            const int n_act = active_tap_list(p, o, act);
            const int rot = (int)(((long long)pair * iters) / p.rot_div) % iters;
            const uint32_t pair_bytes = 2u * (uint32_t)(kA + kBc);
            const int ybase = ty * p.box_h * p.s_h - p.p_h;
            const int xbase = tx * p.box_w * p.s_w - p.p_w;
            KWalk w;
            w.set(rot, p);
            TapSrc ts = tap_source(p, act[w.ti], n, o);
            Ring ring;
            for (int it = 0; it < iters; ++it) {
                if (it >= stages && !mbar_wait(smem_u32(&empty_bar[ring.st]), ring.ph ^ 1u,
                                               p.status, p.wait_limit_ns))
                    break;
                const int y0 = ybase + w.r * p.d_h;
                const int x0 = xbase + w.s * p.d_w;
                const int wrow = ts.wtap + w.r * p.kw + w.s;
                const uint32_t fb_local = smem_u32(&full_bar[ring.st]);
                if (leader) mbar_arrive_expect_tx(fb_local, pair_bytes);
                const uint32_t fb = pair_leader_addr(fb_local);
                tma_load_4d_pair(smem_u32(sA + ring.st * kA), ts.map, fb, w.cb * BK, x0, y0,
                                 ts.frame);
                for (int j = 0; j < p.n_sub; ++j)
                    tma_load_3d_pair(smem_u32(sB + ring.st * kBc + j * kBh), &p.tmap_w, fb,
                                     w.cb * BK, wrow, n_tile * BN + j * BNs + (int)rank * hB);
                ring.next(stages);
                if (w.next(p)) {
                    if (w.ti == n_act) w.ti = 0;
                    ts = tap_source(p, act[w.ti], n, o);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------ MMA issuer (even CTA only)
            const uint32_t idesc = idesc_bf16_m256((uint32_t)BNs);
            const uint64_t a0 = smem_desc_kmajor(smem_u32(sA), kRow);
            const uint64_t b0 = smem_desc_kmajor(smem_u32(sB), kRow);
            Ring ring;
            for (int it = 0; it < iters; ++it) {
                if (!mbar_wait(smem_u32(&full_bar[ring.st]), ring.ph, p.status, p.wait_limit_ns))
                    break;
                tc_fence_after();
                const uint64_t a_desc = a0 + (uint64_t)((ring.st * kA) >> 4);
                const uint64_t b_desc = b0 + (uint64_t)((ring.st * kBc) >> 4);
                for (int j = 0; j < p.n_sub; ++j) {
                    const uint64_t bj = b_desc + (uint64_t)((j * kBh) >> 4);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_bf16_pair(tmem_base + (uint32_t)(j * BNs), a_desc + 2u * kk,
                                       bj + 2u * kk, idesc, (it | kk) != 0 ? 1u : 0u);
                }
                umma_commit_pair(smem_u32(&empty_bar[ring.st]), (uint16_t)0x3);
                ring.next(stages);
            }
            umma_commit_pair(smem_u32(acc_bar), (uint16_t)0x3);
        }
        __syncwarp();
    } else {
        // ------------------- bias, new_cache slice, then this CTA's epilogue
        // (the bias is read here, off the set-up path, and is in shared
        // memory long before the accumulator is complete)
        const int etid = threadIdx.x - 64;
        for (int i = etid; i < BN; i += 128) {
            const int co = n_tile * BN + i;
            float b = 0.f;
            if (p.bias != nullptr && co < p.Cout && index_ok(p.status, co, p.Cout))
                b = __bfloat162float(__ushort_as_bfloat16(p.bias[co]));
            bias_s[i] = b;
        }
        epi_bar();
        copy_new_cache(p.copy, blockIdx.x, gridDim.x, etid, 128);

        const bool ok = mbar_wait(smem_u32(acc_bar), 0, p.status, p.wait_limit_ns);
        tc_fence_after();
        // every pair MMA has completed: neither CTA's ring is read any more,
        // so this CTA stages its output rows there
        const int q = warp & 3;
        const int frame = n * p.T_o + o;
        const int x0 = tx * p.box_w, y0 = ty * p.box_h, co0 = n_tile * BN;
        const bool have_acc = iters > 0;
        const bool store = ok && ty < p.tiles_y;  // a box past the frame stores nothing
        switch (out_block_channels(BN)) {
            case 64: epilogue_store_warp<64>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, frame, q, lane, store); break;
            case 32: epilogue_store_warp<32>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, frame, q, lane, store); break;
            default: epilogue_store_warp<16>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, frame, q, lane, store); break;
        }
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync();  // the peer's shared memory and barriers stay alive until both are done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, (uint32_t)p.tmem_cols);
    }
}

}  // namespace ccv3d
