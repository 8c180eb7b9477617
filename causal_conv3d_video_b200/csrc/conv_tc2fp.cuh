// conv_tc2fp.cuh -- persistent form of the frame-pair kernel (conv_tc2f.cuh).
//
// The stage structure is conv_tc2f's: a tile is two consecutive output frames
// of one 128-pixel output row (pair of boxes), a stage is (source frame,
// channel block, kernel row) holding one input strip and, per kernel column,
// both temporal taps' weight rows stacked along N, so one N = 2 Cout MMA
// accumulates both frames (Sec. 4's per-tap sum regrouped by source frame).
//
// What changes is the life of a CTA pair: one pair per SM pair stays resident
// and walks the tiles g, g + G, g + 2G, ... (G pairs), so
//   * the operand ring runs continuously across tiles (no per-tile prologue,
//     pipeline fill or drain);
//   * the accumulators are double-buffered in TMEM (2 x 2 Cout columns) when
//     the kernel runs one CTA per SM: the epilogue warps drain tile u's
//     frames while the MMA issuer fills tile u + 1's buffer; sized for two
//     CTAs per SM (n_acc = 1) each CTA holds one buffer and the other CTA's
//     MMAs run while it drains;
//   * the epilogue stages output blocks in two dedicated buffers (the ring is
//     never idle) and stores them with TMA tensor stores;
//   * warps 6-9 copy new_cache: frames no tap reads in equal slices at the
//     start, each other kept frame box by box when the producer starts the
//     first tile of the frame pair that reads it, so the copy and the GEMM's
//     strip loads meet in L2.
// Every wait is bounded; decisions taken from bounded waits are made uniform
// over the epilogue threads.
#pragma once
#include <cuda_bf16.h>

#include "cache_copy.cuh"
#include "checked.cuh"
#include "conv_tc.cuh"
#include "conv_tc2f.cuh"
#include "conv_tc2h.cuh"
#include "conv_tcp.cuh"
#include "epilogue.cuh"
#include "params.h"
#include "ptx.cuh"

namespace ccv3d {

template <int BK>
__host__ __device__ constexpr size_t tc2fp_smem_bytes(int bn, int stages, int kh, int kw,
                                                      int halo_w) {
    // ring, output staging (two blocks), ring barriers, 2 x (acc full, acc
    // empty), producer progress, TMEM address slot, bias
    return 1024 + (size_t)stages * tc2f_stage_bytes<BK>(bn, kh, kw, halo_w) +
           tcp_staging_bytes(bn) + (size_t)(2 * stages + 4) * 8 + 8 + 16 + (size_t)bn * 4;
}

// Drain one frame's 128 x BN accumulator (TMEM columns from `tacc`) as bf16 of
// acc + bias into the output, one block of kCh channels at a time through the
// two staging buffers (`slot` alternates; a buffer is refilled only after the
// tensor store that last read it has read it).  128 epilogue threads.
template <int kCh>
__device__ __forceinline__ void tc2fp_frame_epilogue(const TcParams& p, uint32_t tacc, bool have,
                                                     const float* bias_s, int BN,
                                                     uint8_t* staging, int& slot, int x0, int y0,
                                                     int frame, bool store, int etid, int q,
                                                     int lane) {
    constexpr int kRowB = kCh * 2;
    constexpr int kBuf = kTileM * kRowB;
    const int row = q * 32 + lane;
    for (int b = 0; b < BN / kCh; ++b) {
        uint32_t v[kCh];
#pragma unroll
        for (int j = 0; j < kCh / 16; ++j)
            tmem_ld_32x32b_x16(tacc + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kCh + j * 16),
                               *reinterpret_cast<uint32_t(*)[16]>(&v[j * 16]));
        tmem_ld_wait();
        if (etid == 0) bulk_wait_group_read1();  // buffer `slot` was read by its last store
        epi_bar();
        uint8_t* blk = staging + slot * kBuf + (size_t)row * kRowB;
#pragma unroll
        for (int c = 0; c < kCh / 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int ch = b * kCh + c * 8 + 2 * i;
                const float a0 = (have ? __uint_as_float(v[c * 8 + 2 * i]) : 0.f) + bias_s[ch];
                const float a1 =
                    (have ? __uint_as_float(v[c * 8 + 2 * i + 1]) : 0.f) + bias_s[ch + 1];
                const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
                w[i] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(blk + (swizzled_chunk<kRowB>(c, row) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        epi_bar();
        if (etid == 0 && store && index_ok(p.status, frame, (long long)p.N * p.T_o)) {
            tma_store_4d(&p.tmap_out, smem_u32(staging + slot * kBuf), b * kCh, x0, y0, frame);
            bulk_commit_group();
        }
        slot ^= 1;
    }
}

template <int BK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcpThreads, 1)
conv_tc2fp_kernel(const __grid_constant__ TcParams p) {
    constexpr int kRow = TcSmem<BK>::kRowBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = p.stages;
    const int BN = p.BN;    // channels of one frame (one Cout tile, n_sub = 1)
    const int hB = BN / 2;  // weight rows per CTA of a one-frame stage
    const int kWt = BN * kRow;
    const int halo_w = p.halo_w;
    const int kStrip = (int)halo_strip_bytes<BK>(halo_w);
    const int kStage = kStrip + p.kw * kWt;
    uint8_t* staging = smem + (size_t)stages * kStage;  // 1024-aligned (stages are)
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(staging + tcp_staging_bytes(BN));
    uint64_t* empty_bar = full_bar + stages;
    uint64_t* acc_full = empty_bar + stages;  // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2], used in the even CTA
    // tiles the producer has started (paces the new_cache copy)
    volatile long long* progress = reinterpret_cast<volatile long long*>(acc_empty + 2);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<long long*>(progress) + 1);
    float* bias_s = reinterpret_cast<float*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int n_acc = p.sk.n_acc;  // TMEM accumulator buffers (1 or 2)
    const int G = (int)(gridDim.x >> 1);
    const int g = (int)(blockIdx.x >> 1);
    const int fpairs = (p.T_o + 1) / 2;
    const int frames = p.N * fpairs;  // (n, output-frame pair), fastest in the tile order
    const int n_tiles = frames * ((p.tiles_x * p.tiles_y + 1) / 2);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), 8);  // 4 epilogue warps x 2 CTAs
        }
        *progress = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.tmap_x);
        if (p.cache_len > 0) tma_prefetch_desc(&p.tmap_c);
        tma_prefetch_desc(&p.tmap_w);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
        tmem_relinquish_pair();
    }
    if (warp >= 2 && warp < 6) {
        for (int i = threadIdx.x - 64; i < BN; i += 128) {
            float b = 0.f;
            if (p.bias != nullptr && i < p.Cout && index_ok(p.status, i, p.Cout))
                b = __bfloat162float(__ushort_as_bfloat16(p.bias[i]));
            bias_s[i] = b;
        }
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------ TMA producer
            const uint32_t strip_bytes = 2u * (uint32_t)(halo_w * kRow);
            Ring ring;  // continues across tiles
            long long issued = 0;
            bool ok = true;
            long long u = 0;
            for (int tile = g; tile < n_tiles && ok; tile += G, ++u) {
                const int fp = tile % frames;
                const int box = (tile / frames) * 2 + (int)rank;
                const int o0 = (fp % fpairs) * 2, n = fp / fpairs;
                int tx = 0, ty = p.tiles_y;
                if (box < p.tiles_x * p.tiles_y) {
                    tx = box % p.tiles_x;
                    ty = box / p.tiles_x;
                }
                const FusedSrc src = fused_sources(p, o0);
                const int iters = src.n * p.n_cb * p.kh;
                const int xs = tx * p.box_w - p.p_w;  // first pixel of the strip (s_w = 1)
                const int y_out = ty * p.box_h;
                *progress = u + 1;
                int si = 0, cb = 0, r = 0;
                for (int it = 0; it < iters; ++it) {
                    if (issued >= stages &&
                        !mbar_wait(smem_u32(&empty_bar[ring.st]), ring.ph ^ 1u, p.status,
                                   p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    const int t = src.t[si];
                    const int ka = src.k0[si], kb = src.k1[si];
                    const bool both = ka >= 0 && kb >= 0;
                    const int my_tap = both ? (leader ? ka : kb) : (ka >= 0 ? ka : kb);
                    const int wbytes_cta = p.kw * (both ? BN : hB) * kRow;
                    uint8_t* st_base = smem + (size_t)ring.st * kStage;
                    const uint32_t fb_local = smem_u32(&full_bar[ring.st]);
                    if (leader)
                        mbar_arrive_expect_tx(fb_local, strip_bytes + 2u * (uint32_t)wbytes_cta);
                    const uint32_t fb = pair_leader_addr(fb_local);
                    const CUtensorMap* map = t < p.cache_len ? &p.tmap_c : &p.tmap_x;
                    int frame = t < p.cache_len ? ring_frame(n, t, p.cache_slots, p.cache_head)
                                                : n * p.T_x + (t - p.cache_len);
                    if (!index_ok(p.status, frame, t < p.cache_len ? p.c_frames : p.x_frames))
                        frame = 0;
                    tma_load_4d_pair(smem_u32(st_base), map, fb, cb * BK, xs,
                                     y_out * p.s_h + r * p.d_h - p.p_h, frame);
                    uint8_t* b_base = st_base + kStrip;
                    const int wrow = my_tap * p.kh * p.kw + r * p.kw;
                    for (int sx = 0; sx < p.kw; ++sx) {
                        if (both) {
                            tma_load_3d_pair(smem_u32(b_base + sx * kWt), &p.tmap_w, fb, cb * BK,
                                             wrow + sx, 0);
                            tma_load_3d_pair(smem_u32(b_base + sx * kWt + hB * kRow), &p.tmap_w,
                                             fb, cb * BK, wrow + sx, hB);
                        } else {
                            tma_load_3d_pair(smem_u32(b_base + sx * kWt), &p.tmap_w, fb, cb * BK,
                                             wrow + sx, (int)rank * hB);
                        }
                    }
                    ring.next(stages);
                    ++issued;
                    if (++r == p.kh) {
                        r = 0;
                        if (++cb == p.n_cb) {
                            cb = 0;
                            ++si;
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------- MMA issuer (even CTA only)
            const uint32_t idesc_one = idesc_bf16_m256((uint32_t)BN);
            const uint32_t idesc_two = idesc_bf16_m256((uint32_t)(2 * BN));
            const uint64_t d0 = smem_desc_kmajor(smem_u32(smem), kRow);
            Ring ring;
            bool ok = true;
            int u = 0;
            for (int tile = g; tile < n_tiles && ok; tile += G, ++u) {
                const int fp = tile % frames;
                const int o0 = (fp % fpairs) * 2;
                const FusedSrc src = fused_sources(p, o0);
                const int iters = src.n * p.n_cb * p.kh;
                const int b = n_acc == 2 ? (u & 1) : 0, round = n_acc == 2 ? (u >> 1) : u;
                if (round > 0 &&
                    !mbar_wait(smem_u32(&acc_empty[b]), (uint32_t)((round & 1) ^ 1), p.status,
                               p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem_base + (uint32_t)(b * 2 * BN);
                int si = 0, cb = 0, r = 0;
                for (int it = 0; it < iters; ++it) {
                    if (!mbar_wait(smem_u32(&full_bar[ring.st]), ring.ph, p.status,
                                   p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const bool both = src.k0[si] >= 0 && src.k1[si] >= 0;
                    const uint32_t idesc = both ? idesc_two : idesc_one;
                    const uint32_t d_tmem = acc + (src.k0[si] >= 0 ? 0u : (uint32_t)BN);
                    const bool zero = src.zero[si] && cb == 0 && r == 0;
                    const uint32_t st_off = (uint32_t)ring.st * (uint32_t)kStage;
                    for (int sx = 0; sx < p.kw; ++sx) {
                        const uint64_t a_desc = d0 + (uint64_t)((st_off + sx * p.d_w * kRow) >> 4);
                        const uint64_t b_desc = d0 + (uint64_t)((st_off + kStrip + sx * kWt) >> 4);
                        const bool first = zero && sx == 0;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            umma_bf16_pair(d_tmem, a_desc + 2u * kk, b_desc + 2u * kk, idesc,
                                           (first && kk == 0) ? 0u : 1u);
                    }
                    umma_commit_pair(smem_u32(&empty_bar[ring.st]), (uint16_t)0x3);
                    ring.next(stages);
                    if (++r == p.kh) {
                        r = 0;
                        if (++cb == p.n_cb) {
                            cb = 0;
                            ++si;
                        }
                    }
                }
                umma_commit_pair(smem_u32(&acc_full[b]), (uint16_t)0x3);
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ------------------------------------------------- new_cache
        const int ctid = threadIdx.x - 192;
        copy_new_cache(p.copy, blockIdx.x, gridDim.x, ctid, 128);
        if (p.copy.paced_mask != 0u) {
            const CopyJob& c = p.copy;
            bool pace = true;
            long long u = 0;
            for (int tile = g; tile < n_tiles; tile += G, ++u) {
                const int fp = tile % frames;
                const int op = fp % fpairs, n = fp / fpairs;
                const int box = (tile / frames) * 2 + (int)rank;
                if (box >= p.tiles_x * p.tiles_y) continue;
                bool any = false;
                for (int j = 0; j < c.keep && j < kMaxPaced; ++j)
                    any |= ((c.paced_mask >> j) & 1u) && p.paced.o[j] == op;
                if (!any) continue;
                if (pace && ctid == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    while (*progress < u + 1) {
                        if (globaltimer_ns() - t0 > p.wait_limit_ns) {
                            atomicCAS(p.status, 0, kStatusTimeout);
                            break;
                        }
                        __nanosleep(256);
                    }
                    if (*progress < u + 1) pace = false;
                }
                copy_bar();
                const int tx = box % p.tiles_x, ty = box / p.tiles_x;
                for (int j = 0; j < c.keep && j < kMaxPaced; ++j)
                    if (((c.paced_mask >> j) & 1u) && p.paced.o[j] == op)
                        copy_box_share(c, n, j, tx, ty, p.tiles_x, p.tiles_y, p.box_w, p.box_h,
                                       p.s_w, p.s_h, p.H, p.W, ctid, 128);
            }
        }
    } else {
        // ------------------------------------------------- the epilogues
        const int etid = threadIdx.x - 64;
        const int q = warp & 3;
        // launched without copy warps (192 threads, two CTAs per SM): the
        // epilogue warps take the sliced new_cache copy before the first tile
        if (blockDim.x <= 192) copy_new_cache(p.copy, blockIdx.x, gridDim.x, etid, 128);
        const uint32_t empty_leader = mapa_cluster(smem_u32(&acc_empty[0]), 0);
        int slot = 0;
        bool ok = true;
        int u = 0;
        for (int tile = g; tile < n_tiles; tile += G, ++u) {
            const int fp = tile % frames;
            const int box = (tile / frames) * 2 + (int)rank;
            const int o0 = (fp % fpairs) * 2, n = fp / fpairs;
            int tx = 0, ty = p.tiles_y;
            if (box < p.tiles_x * p.tiles_y) {
                tx = box % p.tiles_x;
                ty = box / p.tiles_x;
            }
            const FusedSrc src = fused_sources(p, o0);
            const int b = n_acc == 2 ? (u & 1) : 0, round = n_acc == 2 ? (u >> 1) : u;
            if (ok && !mbar_wait(smem_u32(&acc_full[b]), (uint32_t)(round & 1), p.status,
                                 p.wait_limit_ns))
                ok = false;
            tc_fence_after();
            ok = epi_bar_and(ok);
            const bool store = ok && ty < p.tiles_y;
            const int x0 = tx * p.box_w, y0 = ty * p.box_h;
            for (int f = 0; f < 2; ++f) {
                const int o = o0 + f;
                if (o >= p.T_o) break;
                const uint32_t tacc = tmem_base + (uint32_t)(b * 2 * BN + f * BN);
                const bool have = f == 0 ? src.has0 : src.has1;
                const int fo = n * p.T_o + o;
                switch (out_block_channels(BN)) {
                    case 64: tc2fp_frame_epilogue<64>(p, tacc, have, bias_s, BN, staging, slot, x0, y0, fo, store, etid, q, lane); break;
                    case 32: tc2fp_frame_epilogue<32>(p, tacc, have, bias_s, BN, staging, slot, x0, y0, fo, store, etid, q, lane); break;
                    default: tc2fp_frame_epilogue<16>(p, tacc, have, bias_s, BN, staging, slot, x0, y0, fo, store, etid, q, lane); break;
                }
            }
            // TMEM buffer b is drained: hand it back to the MMA issuer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(smem_u32(&acc_empty[b]));
                else
                    mbar_arrive_remote(empty_leader + (uint32_t)(b * 8));
            }
        }
        if (etid == 0) bulk_wait_group0();  // output stores complete before exit
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
