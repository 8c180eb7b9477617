// conv_tcn.cuh -- tensor-core kernel for thin outputs: the temporal and column
// taps of the kernel stacked along the MMA's N.
//
// A call with few output channels (the decoder's RGB output conv, 96 -> 3)
// cannot fill an MMA's N with Cout, and a tcgen05 MMA costs about the same
// below N = 192 whatever its N.  Here N holds (temporal tap k, column tap s,
// output channel co) instead: for kernel row r the weight tile is
//     row k*Cbk + s*Cout + co  =  W[co, k, r, s, :]      (Cbk = kw*Cout rounded
//                                                          up to 16; the rows
//                                                          between are zero)
// and M holds 128 consecutive input pixels of one row strip, so a stage
// (source frame t of Z, kernel row r, channel block) accumulates
//     D[i, (k, s, co)] += sum_ci Z[t, y*s_h + r*d_h - p_h, x0 - p_w + i, ci] W[co, k, r, s, ci].
// Output frame o reads source frame t through tap k = t - delta_0 - o (unit
// temporal stride and dilation, Sec. 4's per-tap sum regrouped by source
// frame).  Aiming the MMA of source t at TMEM column Cbk*(t_hi - t) therefore
// puts tap k's block of every source at column Cbk*(t_hi - delta_0 - o): one
// fixed region per output frame, whatever the source.  Blocks for frames
// outside the tile's group land in regions nobody reads.  Every source frame
// is loaded once per tile for all the output frames it feeds.
//
// The column taps are summed in the epilogue: output pixel x0 + j is
//     out[o, y, x0 + j, co] = bias[co] + sum_s D_o[j + s*d_w, (s, co)],
// formed from a shared-memory copy of the frame's region (the rows of a
// 128-pixel strip give 128 - (kw-1)*d_w outputs).  MMAs of different sources
// overlap in TMEM, so none starts a region with accumulate = 0: the epilogue
// warps zero the accumulator columns before the first MMA.
//
// Tile: (output row y, group of G output frames, batch entry n, x tile);
// warp roles as in conv_tc.cuh (warp 0 TMA, warp 1 MMA, warps 2-5 new_cache
// slice + epilogue); every wait is bounded.
#pragma once
#include <cuda_bf16.h>

#include "cache_copy.cuh"
#include "checked.cuh"
#include "conv_tc.cuh"
#include "epilogue.cuh"
#include "kwalk.cuh"
#include "params.h"
#include "ptx.cuh"

namespace ccv3d {

// Bytes of one stage: the 128-pixel strip and the n-row weight tile.
template <int BK>
__host__ __device__ constexpr size_t tcn_stage_bytes(int n) {
    return (size_t)(kTileM + n) * TcSmem<BK>::kRowBytes;
}

// fp32 epilogue copy of one frame's region: 128 strip pixels x (kw*Cout | 1).
__host__ __device__ constexpr size_t tcn_frame_stage_bytes(int kw, int cout) {
    return (size_t)kTileM * ((kw * cout) | 1) * 4;
}

template <int BK>
__host__ __device__ constexpr size_t tcn_smem_bytes(int n, int stages, int kw, int cout) {
    const size_t ring = (size_t)stages * tcn_stage_bytes<BK>(n);
    const size_t epi = tcn_frame_stage_bytes(kw, cout);
    const size_t r = ((ring > epi ? ring : epi) + 1023) / 1024 * 1024;
    return 1024 + r + (size_t)(2 * stages + 1) * 8 + 16 + (size_t)cout * 4;
}

// Named barrier between the MMA warp and the epilogue warps (barrier 3,
// 160 threads): the accumulator columns are zero.
__device__ __forceinline__ void tcn_zero_bar() {
    asm volatile("bar.sync 3, 160;" ::: "memory");
}

template <int BK>
__global__ void __launch_bounds__(kTcThreads, 1)
conv_tcn_kernel(const __grid_constant__ TcParams p) {
    constexpr int kRow = TcSmem<BK>::kRowBytes;
    constexpr int kA = TcSmem<BK>::kABytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = p.stages;
    const int NB = p.BN;              // MMA N = kt * Cbk
    const int cbk = p.tn_cbk;         // TMEM columns per output frame
    const int wrows = p.tn_rows;      // weight rows one tap's load writes (kw * Cout)
    const int kB = NB * kRow;
    const int kStage = kA + kB;
    const size_t ring = (size_t)stages * kStage;
    const size_t epi1 = tcn_frame_stage_bytes(p.kw, p.Cout);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(
        smem + ((ring > epi1 ? ring : epi1) + 1023) / 1024 * 1024);
    uint64_t* empty_bar = full_bar + stages;
    uint64_t* acc_bar = empty_bar + stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);
    float* bias_s = reinterpret_cast<float*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- tile: x tile fastest, then output row, frame group, batch entry
    int b = blockIdx.x;
    const int tx = b % p.tiles_x;
    b /= p.tiles_x;
    const int y = b % p.H_o;
    b /= p.H_o;
    const int grp = b % p.tn_groups;
    const int n = b / p.tn_groups;
    const int G = p.tn_G;
    const int o0 = grp * G;
    const int kt = p.taps.kt;
    const int z_len = p.cache_len + p.T_x;
    const int t_lo = max(0, o0 + p.taps.delta[0]);
    const int t_hi = o0 + G - 1 + p.taps.delta[0] + kt - 1;  // column origin
    const int t_end = min(z_len - 1, t_hi);
    const int x0 = tx * p.box_w;  // first output pixel (box_w outputs per tile)
    const int xs = x0 - p.p_w;    // first strip pixel (s_w = 1)

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
    // weight tiles: the rows between the taps' blocks stay zero (the loads
    // never write them)
    for (int s = 0; s < stages; ++s) {
        uint4* wt = reinterpret_cast<uint4*>(smem + (size_t)s * kStage + kA);
        for (int i = threadIdx.x; i < kB / 16; i += blockDim.x) wt[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
        tmem_relinquish();
    }
    if (warp >= 2) {
        for (int i = threadIdx.x - 64; i < p.Cout; i += 128) {
            float bv = 0.f;
            if (p.bias != nullptr && index_ok(p.status, i, p.Cout))
                bv = __bfloat162float(__ushort_as_bfloat16(p.bias[i]));
            bias_s[i] = bv;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            Ring rg;
            int it = 0;
            bool go = true;
            const uint32_t bytes = (uint32_t)(kA + kt * wrows * kRow);
            for (int t = t_lo; go && t <= t_end; ++t) {
                const CUtensorMap* map = t < p.cache_len ? &p.tmap_c : &p.tmap_x;
                int frame = t < p.cache_len ? ring_frame(n, t, p.cache_slots, p.cache_head)
                                            : n * p.T_x + (t - p.cache_len);
                if (!index_ok(p.status, frame, t < p.cache_len ? p.c_frames : p.x_frames)) frame = 0;
                for (int r = 0; go && r < p.kh; ++r) {
                    const int yi = y * p.s_h + r * p.d_h - p.p_h;
                    if (yi < 0 || yi >= p.H) continue;  // a zero row adds nothing
                    for (int cb = 0; cb < p.n_cb; ++cb, ++it) {
                        if (it >= stages && !mbar_wait(smem_u32(&empty_bar[rg.st]), rg.ph ^ 1u,
                                                       p.status, p.wait_limit_ns)) {
                            go = false;
                            break;
                        }
                        uint8_t* st = smem + (size_t)rg.st * kStage;
                        const uint32_t fb = smem_u32(&full_bar[rg.st]);
                        mbar_arrive_expect_tx(fb, bytes);
                        tma_load_4d(smem_u32(st), map, fb, cb * BK, xs, yi, frame);
                        for (int k = 0; k < kt; ++k)
                            tma_load_5d(smem_u32(st + kA + k * cbk * kRow), &p.tmap_w, fb,
                                        cb * BK, 0, 0, r, k);
                        rg.next(stages);
                    }
                }
            }
        }
    } else if (warp == 1) {
        tcn_zero_bar();  // the epilogue warps have zeroed the accumulator
        tc_fence_after();
        if (lane == 0) {
            // ------------------------------------------------- MMA issuer
            const uint32_t idesc = idesc_bf16_m128((uint32_t)NB);
            const uint64_t d0 = smem_desc_kmajor(smem_u32(smem), kRow);
            Ring rg;
            bool go = true;
            for (int t = t_lo; go && t <= t_end; ++t) {
                const uint32_t d_tmem = tmem_base + (uint32_t)(cbk * (t_hi - t));
                for (int r = 0; go && r < p.kh; ++r) {
                    const int yi = y * p.s_h + r * p.d_h - p.p_h;
                    if (yi < 0 || yi >= p.H) continue;
                    for (int cb = 0; cb < p.n_cb; ++cb) {
                        if (!mbar_wait(smem_u32(&full_bar[rg.st]), rg.ph, p.status,
                                       p.wait_limit_ns)) {
                            go = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t off = (uint32_t)rg.st * (uint32_t)kStage;
                        const uint64_t a_desc = d0 + (uint64_t)(off >> 4);
                        const uint64_t b_desc = d0 + (uint64_t)((off + kA) >> 4);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            umma_bf16(d_tmem, a_desc + 2u * kk, b_desc + 2u * kk, idesc, 1u);
                        umma_commit(smem_u32(&empty_bar[rg.st]));
                        rg.next(stages);
                    }
                }
            }
            umma_commit(smem_u32(acc_bar));
        }
        __syncwarp();
    } else {
        // ------------------- zero the accumulator, new_cache slice, epilogue
        const int etid = threadIdx.x - 64;
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t lane_base = tmem_base + ((uint32_t)(32 * q) << 16);
        const int zero_cols = cbk * (G + kt - 2) + NB;  // multiple of 16
        for (int c = 0; c < zero_cols; c += 16) tmem_st_32x32b_x16_fill(lane_base + c, 0u);
        tmem_st_wait();
        tc_fence_before();
        tcn_zero_bar();

        copy_new_cache(p.copy, blockIdx.x, gridDim.x, etid, 128);
        const bool ok = epi_bar_and(mbar_wait(smem_u32(acc_bar), 0, p.status, p.wait_limit_ns));
        tc_fence_after();
        if (ok) {
            // the ring is idle once the accumulator is complete: stage there
            float* stg = reinterpret_cast<float*>(smem);
            const int cb_used = p.kw * p.Cout;
            const int cbs = cb_used | 1;
            const int i = 32 * q + lane;  // strip pixel of this thread's TMEM lane
            const int nj = min(p.box_w, p.W_o - x0);
            const long long out_elems = (long long)p.N * p.T_o * p.H_o * p.W_o * p.Cout;
            for (int f = 0; f < G; ++f) {
                const int o = o0 + f;
                if (o >= p.T_o) break;
                const uint32_t col = (uint32_t)(cbk * (t_hi - p.taps.delta[0] - o));
                for (int c0 = 0; c0 < cb_used; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(lane_base + col + (uint32_t)c0, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (c0 + c < cb_used) stg[i * cbs + c0 + c] = __uint_as_float(v[c]);
                }
                epi_bar();
                const long long obase =
                    ((((long long)n * p.T_o + o) * p.H_o + y) * p.W_o + x0) * p.Cout;
                for (int e = etid; e < nj * p.Cout; e += 128) {
                    const int j = e / p.Cout;
                    const int co = e - j * p.Cout;
                    float acc = bias_s[co];
                    for (int s = 0; s < p.kw; ++s)
                        acc += stg[(j + s * p.d_w) * cbs + s * p.Cout + co];
                    if (index_ok(p.status, obase + e, out_elems))
                        p.out[obase + e] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
                }
                epi_bar();  // the staging area is reused by the next frame
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
    }
}

}  // namespace ccv3d
