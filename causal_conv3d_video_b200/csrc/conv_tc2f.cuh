// conv_tc2f.cuh -- CTA-pair halo kernel that computes two consecutive output
// frames per tile, sharing each source frame between them.
//
// With unit temporal stride and dilation, output frames o and o+1 read the
// same source frame t through adjacent temporal taps: k = t - o + p_l for
// frame o and k - 1 for frame o+1 (Sec. 4's per-tap decomposition, regrouped
// by source frame).  A pipeline stage is (source frame t, channel block,
// kernel row r): the input strip of row r of frame t and, per kernel column
// s, the weight rows of both temporal taps stacked along N:
//     N rows [0, BN)      tap k   (frame o,   TMEM columns [0, BN))
//     N rows [BN, 2 BN)   tap k-1 (frame o+1, TMEM columns [BN, 2 BN))
// and one MMA of N = 2 BN accumulates both frames.  In the CTA pair the N rows
// split by halves, so the even CTA holds tap k's rows and the odd CTA tap
// k-1's.  A source frame that only one of the two frames reads is a stage of
// N = BN aimed at that frame's columns (each CTA holding half its rows).
// Stages this small fit four per CTA at two CTAs per SM, so the loads of the
// next stages stay in flight while an MMA group runs.
//
// Thin channel counts (BN <= 128) are where this pays: a tcgen05 MMA has a
// floor of about 125 cycles whatever its N, so N = 96 instructions run at
// half the tensor rate; stacking two frames makes them N = 192, and each
// source strip is loaded once for both frames.
//
// Stage order: every TMEM region must first be written by an MMA with
// accumulate = 0.  When both single-frame kinds exist they come first (one
// zeroes each region), then the shared stages; otherwise the first stage
// (shared, or the only kind) zeroes what it writes.
//
// Halo strips (one per stage here), pair barriers, epilogue and bounded waits
// are those of conv_tc2h.cuh.
#pragma once
#include <cuda_bf16.h>

#include "cache_copy.cuh"
#include "checked.cuh"
#include "conv_tc.cuh"
#include "conv_tc2h.cuh"
#include "epilogue.cuh"
#include "kwalk.cuh"
#include "params.h"
#include "ptx.cuh"

namespace ccv3d {

// One stage (per CTA): one strip + kw weight areas of bn rows (two taps'
// rows, or one tap's half in the first bn/2 rows).
template <int BK>
__host__ __device__ constexpr size_t tc2f_stage_bytes(int bn, int kh, int kw, int halo_w) {
    return (void)kh, halo_strip_bytes<BK>(halo_w) + (size_t)kw * bn * TcSmem<BK>::kRowBytes;
}

template <int BK>
__host__ __device__ constexpr size_t tc2f_smem_bytes(int bn, int stages, int kh, int kw,
                                                     int halo_w) {
    return 1024 + ring_bytes((size_t)stages * tc2f_stage_bytes<BK>(bn, kh, kw, halo_w), bn) +
           (size_t)(2 * stages + 1) * 8 + 16 + (size_t)bn * 4;
}

// Source frames of one output-frame pair, in stage order.
struct FusedSrc {
    int n;                    // stages (<= kMaxTaps + 1)
    int t[kMaxTaps + 1];      // source frame of Z
    int k0[kMaxTaps + 1];     // tap for frame o0 (-1: none)
    int k1[kMaxTaps + 1];     // tap for frame o1 (-1: none)
    bool zero[kMaxTaps + 1];  // first MMA of this stage starts its region(s)
    bool has0, has1;          // frame o0 / o1 receives any MMA
};

__device__ __forceinline__ bool tap_active(const TcParams& p, int k, int o) {
    return k >= 0 && k < p.taps.kt && o >= p.taps.o_l[k] && o < p.taps.o_h[k];
}

// Schedule for output frames o0 and o1 = o0 + 1 (o1 >= T_o: frame o0 alone),
// unit temporal stride and dilation: frame o reads t = o + k + delta_0.
__device__ __forceinline__ FusedSrc fused_sources(const TcParams& p, int o0) {
    const int o1 = o0 + 1;
    const bool two = o1 < p.T_o;
    int ts[kMaxTaps + 1], a[kMaxTaps + 1], b[kMaxTaps + 1], m = 0;
    const int t_lo = o0 + p.taps.delta[0];
    for (int t = t_lo; t <= t_lo + p.taps.kt; ++t) {
        const int ka = t - p.taps.delta[0] - o0;
        const int kb = ka - 1;
        const bool va = tap_active(p, ka, o0);
        const bool vb = two && tap_active(p, kb, o1);
        if (!va && !vb) continue;
        ts[m] = t;
        a[m] = va ? ka : -1;
        b[m] = vb ? kb : -1;
        ++m;
    }
    FusedSrc f;
    f.n = 0;
    f.has0 = f.has1 = false;
    int n0 = 0, n1 = 0;
    for (int i = 0; i < m; ++i) {
        n0 += (a[i] >= 0 && b[i] < 0);
        n1 += (a[i] < 0 && b[i] >= 0);
    }
    // kinds in stage order: 0 = frame o0 only, 1 = frame o1 only, 2 = both
    const int order_split[3] = {0, 1, 2};
    const int order_both[3] = {2, 0, 1};
    const int* order = (n0 > 0 && n1 > 0) ? order_split : order_both;
    for (int oi = 0; oi < 3; ++oi)
        for (int i = 0; i < m; ++i) {
            const int kind = (a[i] >= 0 && b[i] >= 0) ? 2 : (a[i] >= 0 ? 0 : 1);
            if (kind != order[oi]) continue;
            const bool w0 = kind != 1, w1 = kind != 0;
            f.t[f.n] = ts[i];
            f.k0[f.n] = a[i];
            f.k1[f.n] = b[i];
            f.zero[f.n] = (w0 && !f.has0) || (w1 && !f.has1);
            f.has0 |= w0;
            f.has1 |= w1;
            ++f.n;
        }
    return f;
}

template <int BK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
conv_tc2f_kernel(const __grid_constant__ TcParams p) {
    constexpr int kRow = TcSmem<BK>::kRowBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = p.stages;
    const int BN = p.BN;              // channels of one frame (n_sub = 1, one Cout tile)
    const int hB = BN / 2;            // weight rows per CTA of a one-frame stage
    const int kWt = BN * kRow;        // weight area per (r, s), per CTA
    const int halo_w = p.halo_w;
    const int kStrip = (int)halo_strip_bytes<BK>(halo_w);
    const int kAst = kStrip;                 // the stage's strip
    const int kStage = kAst + p.kw * kWt;
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

    // ---- pair tile: (pair of boxes, n, output-frame pair); frame pair fastest
    const int pair = blockIdx.x >> 1;
    const int fpairs = (p.T_o + 1) / 2;
    const int frames = p.N * fpairs;
    const int fp = pair % frames;
    const int box = (pair / frames) * 2 + (int)rank;
    const int o0 = (fp % fpairs) * 2;
    const int n = fp / fpairs;
    int tx = 0, ty = p.tiles_y;
    if (box < p.tiles_x * p.tiles_y) {
        tx = box % p.tiles_x;
        ty = box / p.tiles_x;
    }
    const FusedSrc src = fused_sources(p, o0);
    const int per_slot = p.n_cb * p.kh;       // stages of one source frame
    const int iters = src.n * per_slot;       // stages: (source frame, channel block, row r)
    // Each pair starts every source frame's (channel block, row) walk at its
    // own offset, so pairs running at the same time read different weight
    // tiles (the first stage of a slot is always the offset one, and it is
    // the one that starts the slot's accumulator region when zero[] says so).
    const int rot = (int)(((long long)pair * per_slot) / p.rot_div % per_slot);

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
        if (lane == 0 && iters > 0) {
            // ------------------------------- TMA producer (both CTAs)
            const uint32_t strip_bytes = 2u * (uint32_t)(halo_w * kRow);
            const int xs = tx * p.box_w - p.p_w;  // first pixel of the strip (s_w = 1)
            const int y_out = ty * p.box_h;
            Ring ring;
            int si = 0, j = 0, cb = rot / p.kh, r = rot % p.kh;
            for (int it = 0; it < iters; ++it) {
                if (it >= stages && !mbar_wait(smem_u32(&empty_bar[ring.st]), ring.ph ^ 1u,
                                               p.status, p.wait_limit_ns))
                    break;
                const int t = src.t[si];
                const int ka = src.k0[si], kb = src.k1[si];
                const bool both = ka >= 0 && kb >= 0;
                // this CTA's rows: both -> all BN rows of its tap (even CTA tap ka, odd
                // CTA tap kb); one frame -> its half (hB rows) of the single tap
                const int my_tap = both ? (leader ? ka : kb) : (ka >= 0 ? ka : kb);
                const int wbytes_cta = p.kw * (both ? BN : hB) * kRow;
                uint8_t* st_base = smem + (size_t)ring.st * kStage;
                const uint32_t fb_local = smem_u32(&full_bar[ring.st]);
                if (leader) mbar_arrive_expect_tx(fb_local, strip_bytes + 2u * (uint32_t)wbytes_cta);
                const uint32_t fb = pair_leader_addr(fb_local);
                const CUtensorMap* map = t < p.cache_len ? &p.tmap_c : &p.tmap_x;
                int frame = t < p.cache_len ? ring_frame(n, t, p.cache_slots, p.cache_head)
                                            : n * p.T_x + (t - p.cache_len);
                // checked build: a frame outside the tensor map is recorded and
                // clamped (the load still completes its barrier)
                if (!index_ok(p.status, frame, t < p.cache_len ? p.c_frames : p.x_frames)) frame = 0;
                tma_load_4d_pair(smem_u32(st_base), map, fb, cb * BK, xs,
                                 y_out * p.s_h + r * p.d_h - p.p_h, frame);
                uint8_t* b_base = st_base + kAst;
                const int wrow = my_tap * p.kh * p.kw + r * p.kw;
                if (p.w_kw_boxes) {
                    // one load: kw column taps x (BN or BN/2) rows, [sx][rows][BK]
                    if (both)
                        tma_load_3d_pair(smem_u32(b_base), &p.tmap_wkw_full, fb, cb * BK, 0, wrow);
                    else
                        tma_load_3d_pair(smem_u32(b_base), &p.tmap_wkw_half, fb, cb * BK,
                                         (int)rank * hB, wrow);
                } else
                for (int sx = 0; sx < p.kw; ++sx) {
                    if (both) {
                        tma_load_3d_pair(smem_u32(b_base + sx * kWt), &p.tmap_w, fb, cb * BK,
                                         wrow + sx, 0);
                        tma_load_3d_pair(smem_u32(b_base + sx * kWt + hB * kRow), &p.tmap_w, fb,
                                         cb * BK, wrow + sx, hB);
                    } else {
                        tma_load_3d_pair(smem_u32(b_base + sx * kWt), &p.tmap_w, fb, cb * BK,
                                         wrow + sx, (int)rank * hB);
                    }
                }
                ring.next(stages);
                if (++r == p.kh) {
                    r = 0;
                    if (++cb == p.n_cb) cb = 0;
                }
                if (++j == per_slot) {  // next source frame, from the offset again
                    j = 0;
                    ++si;
                    cb = rot / p.kh;
                    r = rot % p.kh;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------ MMA issuer (even CTA only)
            const uint32_t idesc_one = idesc_bf16_m256((uint32_t)BN);
            const uint32_t idesc_two = idesc_bf16_m256((uint32_t)(2 * BN));
            const uint64_t d0 = smem_desc_kmajor(smem_u32(smem), kRow);
            Ring ring;
            int si = 0, j = 0;
            for (int it = 0; it < iters; ++it) {
                if (!mbar_wait(smem_u32(&full_bar[ring.st]), ring.ph, p.status, p.wait_limit_ns))
                    break;
                tc_fence_after();
                const bool both = src.k0[si] >= 0 && src.k1[si] >= 0;
                const uint32_t idesc = both ? idesc_two : idesc_one;
                const uint32_t d_tmem = tmem_base + (src.k0[si] >= 0 ? 0u : (uint32_t)BN);
                const bool zero = src.zero[si] && j == 0;
                const uint32_t st_off = (uint32_t)ring.st * (uint32_t)kStage;
                // weight tile of column tap sx: kWt apart, or, loaded as one
                // [kw][rows][BK] box, (rows x kRow) apart
                const int wstride = (p.w_kw_boxes && !both) ? hB * kRow : kWt;
                for (int sx = 0; sx < p.kw; ++sx) {
                    // A: the strip shifted by sx*d_w pixels (rows)
                    const uint64_t a_desc = d0 + (uint64_t)((st_off + sx * p.d_w * kRow) >> 4);
                    const uint64_t b_desc = d0 + (uint64_t)((st_off + kAst + sx * wstride) >> 4);
                    const bool first = zero && sx == 0;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        umma_bf16_pair(d_tmem, a_desc + 2u * kk, b_desc + 2u * kk, idesc,
                                       (first && kk == 0) ? 0u : 1u);
                }
                umma_commit_pair(smem_u32(&empty_bar[ring.st]), (uint16_t)0x3);
                ring.next(stages);
                if (++j == per_slot) {
                    j = 0;
                    ++si;
                }
            }
            umma_commit_pair(smem_u32(acc_bar), (uint16_t)0x3);
        }
        __syncwarp();
    } else {
        // ------------------- new_cache slice, then both frames' epilogues
        const int etid = threadIdx.x - 64;
        copy_new_cache(p.copy, blockIdx.x, gridDim.x, etid, 128);
        const bool ok = mbar_wait(smem_u32(acc_bar), 0, p.status, p.wait_limit_ns);
        tc_fence_after();
        const int q = warp & 3;
        const int x0 = tx * p.box_w, y0 = ty * p.box_h;
        const bool store = ok && ty < p.tiles_y;
        for (int f = 0; f < 2; ++f) {
            const int o = o0 + f;
            if (o >= p.T_o) break;
            const uint32_t tacc = tmem_base + (uint32_t)(f * BN);
            const bool have = f == 0 ? src.has0 : src.has1;
            const int fo = n * p.T_o + o;
            switch (out_block_channels(BN)) {
                case 64: epilogue_store<64>(p, tacc, have, bias_s, BN, smem, 0, x0, y0, fo, etid, q, lane, store); break;
                case 32: epilogue_store<32>(p, tacc, have, bias_s, BN, smem, 0, x0, y0, fo, etid, q, lane, store); break;
                default: epilogue_store<16>(p, tacc, have, bias_s, BN, smem, 0, x0, y0, fo, etid, q, lane, store); break;
            }
            epi_bar();  // the staging area is reused by the next frame's epilogue
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
