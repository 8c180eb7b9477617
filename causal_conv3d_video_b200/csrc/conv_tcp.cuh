// conv_tcp.cuh -- persistent, stream-K implicit-GEMM Conv3D on CTA pairs.
//
// The work of one call is the list of pair tiles (two 128-pixel boxes of one
// output frame x a Cout tile), each a reduction of iters(o) k-blocks, where
// iters(o) = (active taps of frame o) x kh x kw x ceil(Cin/BK) follows the
// paper's per-tap intervals (Sec. 4).  The k-blocks of all tiles, laid end to
// end, are cut into G equal ranges, one per resident CTA pair (stream-K), so
// every SM pair gets the same number of MMAs whatever the tile count.
//
// A tile cut by range boundaries is finished by the pair whose range holds
// its first k-block (the "owner"): that pair reaches the tile last, at the end
// of its range, while every other pair holding a piece of the tile meets it
// first, at the start of its range.  Those pairs store their fp32 partial
// accumulators in the scratch area (one slot per CTA: only a range's first
// piece can be partial) and publish a flag carrying the launch's epoch; the
// owner waits for the flags (bounded), adds the partials, then applies bias
// and rounding once.
//
// Per CTA: warp 0 streams TMA loads, warp 1 holds TMEM (the even CTA's lane 0
// issues the pair MMAs), warps 2-5 run the epilogues and warps 6-9 copy this
// CTA's slice of new_cache while the GEMM runs.  With Cout tiles of <= 256 columns the accumulator is double
// buffered in TMEM, so a tile's epilogue overlaps the next tile's main loop.
#pragma once
#include <cuda_bf16.h>

#include "cache_copy.cuh"
#include "conv_tc.cuh"
#include "conv_tc2.cuh"
#include "epilogue.cuh"
#include "kwalk.cuh"
#include "params.h"
#include "ptx.cuh"

namespace ccv3d {

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
                 ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ uint32_t mapa_cluster(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Order this thread's earlier generic-proxy observations of global memory
// before its later async-proxy (bulk copy) reads of it.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Plain (untiled) bulk copy of `bytes` bytes global -> this CTA's shared
// memory, completing on mbarrier `bar`.  Both addresses and `bytes` are
// multiples of 16.
__device__ __forceinline__ void bulk_load_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}


// One piece of a pair's range: pair tile `tile` (frame f, index in frame),
// k-blocks [kb0, kb1) of its reduction of `iters` k-blocks.
struct Seg {
    long long tile_start;  // global k-block index of the tile's first k-block
    int f, tile_in_frame, iters, kb0, kb1;
};

// Range of k-blocks of pair g: [start(g), start(g+1)).
__device__ __forceinline__ long long sk_start(const TcParams& p, int g) {
    return (long long)g * p.sk.total / p.sk.G;  // g <= G <= 128, total < 2^40
}

__device__ __forceinline__ int active_taps(const TcParams& p, int o) {
    int a = 0;
#pragma unroll
    for (int k = 0; k < kMaxTaps; ++k)
        if (k < p.taps.kt && o >= p.taps.o_l[k] && o < p.taps.o_h[k]) ++a;
    return a;
}

// The segment of pair tile work containing global k-block I, clipped to end.
__device__ __forceinline__ Seg sk_locate(const TcParams& p, long long I, long long end) {
    Seg s;
    int f = 0;
    while (f + 1 < p.sk.n_frames && p.sk.frame_start[f + 1] <= I) ++f;
    const int o = f % p.T_o;
    const int iters = active_taps(p, o) * p.kh * p.kw * p.n_cb;
    const long long local = I - p.sk.frame_start[f];
    s.f = f;
    s.iters = iters;
    s.tile_in_frame = (int)(local / iters);
    s.tile_start = p.sk.frame_start[f] + (long long)s.tile_in_frame * iters;
    s.kb0 = (int)(I - s.tile_start);
    const long long e = end - s.tile_start;
    s.kb1 = e < iters ? (int)e : iters;
    return s;
}

// Pair whose range holds global k-block J.
__device__ __forceinline__ int sk_owner_of(const TcParams& p, long long J) {
    int g = (int)(J * p.sk.G / p.sk.total);
    if (g >= p.sk.G) g = p.sk.G - 1;
    while (g + 1 < p.sk.G && sk_start(p, g + 1) <= J) ++g;
    while (g > 0 && sk_start(p, g) > J) --g;
    return g;
}

// Fp32 partial tile layout in a scratch slot, for one CTA's 128 x BN piece:
// blocks of kCh channels, each block [16-channel chunk][quad e][row][4
// floats], so that a warp's float4 stores (thread = row) cover 512 contiguous
// bytes and one block is one contiguous run the owner fetches in one copy.
template <int kCh>
__device__ __forceinline__ size_t tcp_partial_index(int b, int j, int e, int row) {
    return (size_t)b * (kTileM * kCh) + ((size_t)(j * 4 + e) * kTileM + row) * 4;
}

// Epilogue of one segment of the persistent kernel, for this CTA's 128 rows of
// TMEM accumulator buffer `tmem_acc`, in blocks of kCh channels:
//   * a piece of a tile owned by an earlier pair ("contributor") is published
//     as fp32 in this CTA's scratch slot (layout above);
//   * the owner adds the contributors' pieces, then bias, rounds to bf16 and
//     writes the block through one of two swizzled staging buffers with a TMA
//     tensor store (the previous store from that buffer is waited for first).
//     A tile with contributors is always the last segment of the owner's
//     range, so the operand ring is idle by then: the contributors' blocks are
//     fetched into it with bulk copies, up to `n_fbuf` in flight, one fetch
//     barrier per ring buffer; `fetch_uses` counts this CTA's fetches so far
//     (the parity of each buffer's next completion).
template <int kCh>
__device__ __forceinline__ void tcp_segment_epilogue(const TcParams& p, uint32_t tmem_acc,
                                                     int q, int lane, int etid, bool owner,
                                                     bool ok, int g, int g_last, int rank,
                                                     int BN, int co0, int x0, int y0,
                                                     int frame, bool store, uint8_t* staging,
                                                     int& slot, uint8_t* ring, int n_fbuf,
                                                     uint64_t* fetch_bar, uint32_t& fetch_uses,
                                                     const float* bias_s) {
    constexpr int kRowB = kCh * 2;
    constexpr int kBuf = kTileM * kRowB;
    constexpr uint32_t kUnit = kTileM * kCh * 4;  // bytes of one fp32 block
    const int row = q * 32 + lane;
    const size_t slot_floats = (size_t)kTileM * BN;
    const int nblk = BN / kCh;
    // checked build: extent of the partial tiles ([2G][128][BN] fp32)
    const long long partial_bytes = (long long)2 * p.sk.G * kTileM * BN * 4;
    if (!owner) {
        float* mine = p.sk.partial + (size_t)(2 * g + rank) * slot_floats;
        if (!in_bounds(p.status, mine, (long long)slot_floats * 4, p.sk.partial, partial_bytes))
            ok = false;
        for (int b = 0; b < nblk; ++b) {
            uint32_t v[kCh];
#pragma unroll
            for (int j = 0; j < kCh / 16; ++j)
                tmem_ld_32x32b_x16(tmem_acc + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kCh + j * 16),
                                   *reinterpret_cast<uint32_t(*)[16]>(&v[j * 16]));
            tmem_ld_wait();
            if (!ok) continue;
#pragma unroll
            for (int j = 0; j < kCh / 16; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    *reinterpret_cast<float4*>(mine + tcp_partial_index<kCh>(b, j, e, row)) =
                        make_float4(__uint_as_float(v[j * 16 + 4 * e]),
                                    __uint_as_float(v[j * 16 + 4 * e + 1]),
                                    __uint_as_float(v[j * 16 + 4 * e + 2]),
                                    __uint_as_float(v[j * 16 + 4 * e + 3]));
        }
        return;
    }
    // ---- owner: fetch units u = (block b, contributor c), block-major
    const int ncon = ok ? g_last - g : 0;
    const int units = nblk * ncon;
    const uint32_t use0 = fetch_uses;
    auto issue = [&](int u) {
        const int b = u / ncon, c = u - b * ncon;
        const int buf = (int)((use0 + (uint32_t)u) % (uint32_t)n_fbuf);
        const float* src = p.sk.partial + (size_t)(2 * (g + 1 + c) + rank) * slot_floats +
                           (size_t)b * (kTileM * kCh);
        const uint32_t bar = smem_u32(&fetch_bar[buf]);
        // checked build: an out-of-range piece is recorded and fetched from
        // the first slot instead (the fetch barrier still completes)
        if (!in_bounds(p.status, src, kUnit, p.sk.partial, partial_bytes)) src = p.sk.partial;
        mbar_arrive_expect_tx(bar, kUnit);
        bulk_load_g2s(smem_u32(ring + (size_t)buf * kUnit), src, kUnit, bar);
    };
    if (etid == 0 && units > 0) {
        fence_proxy_async_global();  // the flags were acquired through the generic proxy
        for (int u = 0; u < units && u < n_fbuf; ++u) issue(u);
    }
    bool fetched = true;
    int u = 0;
    for (int b = 0; b < nblk; ++b) {
        uint32_t v[kCh];
#pragma unroll
        for (int j = 0; j < kCh / 16; ++j)
            tmem_ld_32x32b_x16(tmem_acc + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kCh + j * 16),
                               *reinterpret_cast<uint32_t(*)[16]>(&v[j * 16]));
        tmem_ld_wait();
        float a[kCh];
#pragma unroll
        for (int i = 0; i < kCh; ++i) a[i] = __uint_as_float(v[i]);
        for (int c = 0; c < ncon; ++c, ++u) {
            const uint32_t use = use0 + (uint32_t)u;
            const int buf = (int)(use % (uint32_t)n_fbuf);
            if (fetched && !mbar_wait(smem_u32(&fetch_bar[buf]), (use / (uint32_t)n_fbuf) & 1u,
                                      p.status, p.wait_limit_ns))
                fetched = false;
            if (!fetched) continue;
            const float* src = reinterpret_cast<const float*>(ring + (size_t)buf * kUnit);
#pragma unroll
            for (int j = 0; j < kCh / 16; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 w4 =
                        *reinterpret_cast<const float4*>(src + tcp_partial_index<kCh>(0, j, e, row));
                    a[j * 16 + 4 * e] += w4.x;
                    a[j * 16 + 4 * e + 1] += w4.y;
                    a[j * 16 + 4 * e + 2] += w4.z;
                    a[j * 16 + 4 * e + 3] += w4.w;
                }
        }
        // staging buffer `slot`: its previous tensor store must have read it
        if (etid == 0) bulk_wait_group_read1();
        // also: every thread is done with this block's fetch buffers; a fetch
        // wait that ran out in any thread stops the refills in all of them
        fetched = epi_bar_and(fetched);
        if (etid == 0 && fetched) {
            fence_proxy_async_smem();
            for (int r = u - ncon; r < u; ++r)
                if (r + n_fbuf < units) issue(r + n_fbuf);
        }
        uint8_t* blk = staging + slot * kBuf + (size_t)row * kRowB;
#pragma unroll
        for (int c = 0; c < kCh / 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int ch = b * kCh + c * 8 + 2 * i;
                const __nv_bfloat162 h = __floats2bfloat162_rn(a[c * 8 + 2 * i] + bias_s[ch],
                                                               a[c * 8 + 2 * i + 1] + bias_s[ch + 1]);
                w[i] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(blk + (swizzled_chunk<kRowB>(c, row) << 4)) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        epi_bar();
        if (etid == 0 && store && ok && index_ok(p.status, frame, (long long)p.N * p.T_o)) {
            tma_store_4d(&p.tmap_out, smem_u32(staging + slot * kBuf), co0 + b * kCh, x0, y0, frame);
            bulk_commit_group();
        }
        slot ^= 1;
    }
    fetch_uses = use0 + (uint32_t)units;
}

// Named barrier over the four new_cache copy warps (barrier 2, 128 threads).
__device__ __forceinline__ void copy_bar() {
    asm volatile("bar.sync 2, 128;" ::: "memory");
}

// The paced share of the new_cache copy (frames of copy.paced_mask): walking
// the pair's range like the producer, for every tile of Cout tile 0 whose
// segment issues the first k-block of a tap that reads kept frame j, wait
// (bounded) until the producer has issued that k-block, then copy this CTA's
// box share of frame j.  The input lines the copy reads are then being
// fetched into L2 for the GEMM's loads at the same time, so the frame
// crosses from DRAM once instead of twice.  Called by the 128 copy threads.
__device__ __forceinline__ void tcp_paced_copy(const TcParams& p, int rank, long long range0,
                                               long long range1,
                                               volatile long long* progress, int ctid) {
    const CopyJob& c = p.copy;
    bool pace = true;  // stop waiting after a wait ran out (the producer stopped)
    for (long long I = range0; I < range1;) {
        const Seg sg = sk_locate(p, I, range1);
        I = sg.tile_start + sg.kb1;
        if (sg.tile_in_frame % p.tiles_n != 0) continue;  // one Cout tile copies
        const int o = sg.f % p.T_o, n = sg.f / p.T_o;
        const int box = (sg.tile_in_frame / p.tiles_n) * 2 + rank;
        if (box >= p.tiles_x * p.tiles_y) continue;
        const int tx = box % p.tiles_x, ty = box / p.tiles_x;
        for (int j = 0; j < c.keep && j < kMaxPaced; ++j) {
            if (!((c.paced_mask >> j) & 1u) || p.paced.o[j] != o) continue;
            const int kb = p.paced.kb[j];
            if (kb < sg.kb0 || kb >= sg.kb1) continue;
            if (pace && ctid == 0) {
                const long long want = sg.tile_start + kb + 1;
                const uint64_t t0 = globaltimer_ns();
                while (*progress < want) {
                    if (globaltimer_ns() - t0 > p.wait_limit_ns) {
                        atomicCAS(p.status, 0, kStatusTimeout);
                        break;
                    }
                    __nanosleep(256);
                }
                if (*progress < want) pace = false;
            }
            copy_bar();
            copy_box_share(c, n, j, tx, ty, p.tiles_x, p.tiles_y, p.box_w, p.box_h, p.s_w,
                           p.s_h, p.H, p.W, ctid, 128);
        }
    }
}

// Two staging buffers of one output block (kCh channels x 128 rows, bf16).
__host__ __device__ constexpr size_t tcp_staging_bytes(int bn) {
    return (size_t)2 * kTileM * out_block_channels(bn) * 2;
}

constexpr int kTcpFetchBufs = 8;  // most partial-block fetch buffers in flight

template <int BK>
__host__ __device__ constexpr size_t tcp_ring_bytes(int bn, int stages) {
    return (size_t)stages * (TcSmem<BK>::kABytes + (size_t)(bn / 2) * TcSmem<BK>::kRowBytes);
}

template <int BK>
__host__ __device__ constexpr size_t tcp_smem_bytes(int bn, int stages) {
    // A box + half the weight rows per stage, output staging, ring barriers,
    // 2 x (acc full, acc empty) barriers, fetch barriers, TMEM address slot,
    // the Cout tile's bias
    return 1024 + tcp_ring_bytes<BK>(bn, stages) + tcp_staging_bytes(bn) +
           (size_t)(2 * stages + 4 + kTcpFetchBufs) * 8 + 8 /* producer progress */ + 16 +
           (size_t)bn * 4;
}

constexpr int kTcpThreads = 320;  // + warps 6-9: the new_cache copy

template <int BK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcpThreads, 1)
conv_tcp_kernel(const __grid_constant__ TcParams p) {
    constexpr int kRow = TcSmem<BK>::kRowBytes;
    constexpr int kA = TcSmem<BK>::kABytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = p.stages;
    const int BN = p.BN;
    const int BNs = BN / p.n_sub;
    const int hB = BNs / 2;
    const int kBc = (BN / 2) * kRow;
    const int kBh = hB * kRow;
    const int n_acc = p.sk.n_acc;
    uint8_t* sA = smem;
    uint8_t* sB = smem + (size_t)stages * kA;
    // staging buffers: aligned to their swizzle atom (kA is a multiple of
    // 4 KB and kBc of 8 rows x kRow; the 64-channel case has kBc % 1024 == 0)
    uint8_t* staging = sB + (size_t)stages * kBc;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(staging + tcp_staging_bytes(BN));
    uint64_t* empty_bar = full_bar + stages;
    uint64_t* acc_full = empty_bar + stages;   // [2]
    uint64_t* acc_empty = acc_full + 2;        // [2], used in the even CTA
    uint64_t* fetch_bar = acc_empty + 2;       // [kTcpFetchBufs]
    // k-blocks of this pair's range the producer has issued (global index + 1)
    volatile long long* progress = reinterpret_cast<volatile long long*>(fetch_bar + kTcpFetchBufs);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(
        const_cast<long long*>(progress) + 1);
    float* bias_s = reinterpret_cast<float*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int g = blockIdx.x >> 1;  // this pair's range
    const long long range0 = sk_start(p, g), range1 = sk_start(p, g + 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), 8);  // 4 epilogue warps x 2 CTAs
        }
        for (int b = 0; b < kTcpFetchBufs; ++b) mbar_init(smem_u32(&fetch_bar[b]), 1);
        *progress = range0;
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
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------ TMA producer
            const uint32_t pair_bytes = 2u * (uint32_t)(kA + kBc);
            Ring ring;  // continues across segments
            long long issued = 0;
            bool ok = true;
            for (long long I = range0; I < range1 && ok;) {
                const Seg sg = sk_locate(p, I, range1);
                const int o = sg.f % p.T_o, n = sg.f / p.T_o;
                const int pp = sg.tile_in_frame / p.tiles_n;
                const int n_tile = sg.tile_in_frame % p.tiles_n;
                const int box = pp * 2 + (int)rank;
                int tx = 0, ty = p.tiles_y;
                if (box < p.tiles_x * p.tiles_y) {
                    tx = box % p.tiles_x;
                    ty = box / p.tiles_x;
                }
                int act[kMaxTaps];
                active_tap_list(p, o, act);
                const int ybase = ty * p.box_h * p.s_h - p.p_h;
                const int xbase = tx * p.box_w * p.s_w - p.p_w;
                const int nrow = n_tile * BN + (int)rank * hB;
                KWalk w;
                w.set(sg.kb0, p);
                TapSrc ts = tap_source(p, act[w.ti], n, o);
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (issued >= stages &&
                        !mbar_wait(smem_u32(&empty_bar[ring.st]), ring.ph ^ 1u, p.status,
                                   p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
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
                                         w.cb * BK, wrow, nrow + j * BNs);
                    ring.next(stages);
                    ++issued;
                    *progress = sg.tile_start + kb + 1;  // paces the new_cache copy
                    if (w.next(p) && kb + 1 < sg.kb1) ts = tap_source(p, act[w.ti], n, o);
                }
                I = sg.tile_start + sg.kb1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------- MMA issuer (even CTA only)
            const uint32_t idesc = idesc_bf16_m256((uint32_t)BNs);
            const uint64_t a0 = smem_desc_kmajor(smem_u32(sA), kRow);
            const uint64_t b0 = smem_desc_kmajor(smem_u32(sB), kRow);
            Ring ring;
            int seg = 0;
            bool ok = true;
            for (long long I = range0; I < range1 && ok; ++seg) {
                const Seg sg = sk_locate(p, I, range1);
                const int b = n_acc == 2 ? (seg & 1) : 0;
                const int round = n_acc == 2 ? (seg >> 1) : seg;
                if (round > 0 &&
                    !mbar_wait(smem_u32(&acc_empty[b]), (uint32_t)((round & 1) ^ 1), p.status,
                               p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!mbar_wait(smem_u32(&full_bar[ring.st]), ring.ph, p.status,
                                   p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = a0 + (uint64_t)((ring.st * kA) >> 4);
                    const uint64_t b_desc = b0 + (uint64_t)((ring.st * kBc) >> 4);
                    const uint32_t first = kb == sg.kb0 ? 1u : 0u;
                    for (int j = 0; j < p.n_sub; ++j) {
                        const uint64_t bj = b_desc + (uint64_t)((j * kBh) >> 4);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            umma_bf16_pair(d_tmem + (uint32_t)(j * BNs), a_desc + 2u * kk,
                                           bj + 2u * kk, idesc, (first && kk == 0) ? 0u : 1u);
                    }
                    umma_commit_pair(smem_u32(&empty_bar[ring.st]), (uint16_t)0x3);
                    ring.next(stages);
                }
                umma_commit_pair(smem_u32(&acc_full[b]), (uint16_t)0x3);
                I = sg.tile_start + sg.kb1;
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ----------------- new_cache, beside the GEMM of this CTA: frames no
        // tap reads in equal slices, the others tile by tile with the loads
        const int ctid = threadIdx.x - 192;
        copy_new_cache(p.copy, blockIdx.x, gridDim.x, ctid, 128);
        if (p.copy.paced_mask != 0u) tcp_paced_copy(p, (int)rank, range0, range1, progress, ctid);
    } else {
        // ------------------------------------------------- the epilogues
        const int etid = threadIdx.x - 64;
        const int q = warp & 3;
        const uint32_t empty_leader = mapa_cluster(smem_u32(&acc_empty[0]), 0);
        int seg = 0, slot = 0;
        bool ok = true;
        uint32_t fetch_uses = 0;
        int bias_tile = -1;  // Cout tile whose bias bias_s holds
        // fp32 partial blocks the idle ring holds at once (the planner keeps
        // the ring at least one block large)
        int n_fbuf = (int)(tcp_ring_bytes<BK>(BN, stages) /
                           ((size_t)kTileM * out_block_channels(BN) * 4));
        if (n_fbuf > kTcpFetchBufs) n_fbuf = kTcpFetchBufs;
        for (long long I = range0; I < range1; ++seg) {
            const Seg sg = sk_locate(p, I, range1);
            const int b = n_acc == 2 ? (seg & 1) : 0;
            const int round = n_acc == 2 ? (seg >> 1) : seg;
            const int o = sg.f % p.T_o, n = sg.f / p.T_o;
            const int pp = sg.tile_in_frame / p.tiles_n;
            const int n_tile = sg.tile_in_frame % p.tiles_n;
            const int box = pp * 2 + (int)rank;
            int tx = 0, ty = p.tiles_y;
            if (box < p.tiles_x * p.tiles_y) {
                tx = box % p.tiles_x;
                ty = box / p.tiles_x;
            }
            if (ok && !mbar_wait(smem_u32(&acc_full[b]), (uint32_t)(round & 1), p.status,
                                 p.wait_limit_ns))
                ok = false;
            tc_fence_after();
            // from here on `ok` decides counts and barrier phases (fetch units,
            // fetch-buffer parities): make it uniform over the epilogue threads
            ok = epi_bar_and(ok);
            const bool owner = sg.kb0 == 0;
            const bool whole = owner && sg.kb1 == sg.iters;
            if (owner && n_tile != bias_tile) {
                epi_bar();  // the previous tile's epilogue is done with bias_s
                for (int i = etid; i < BN; i += 128) {
                    const int co = n_tile * BN + i;
                    bias_s[i] = (p.bias != nullptr && co < p.Cout && index_ok(p.status, co, p.Cout))
                                    ? __bfloat162float(__ushort_as_bfloat16(__ldg(p.bias + co)))
                                    : 0.f;
                }
                epi_bar();
                bias_tile = n_tile;
            }
            // pairs holding the other pieces of this tile (owner only)
            int g_last = g;
            if (owner && !whole) g_last = sk_owner_of(p, sg.tile_start + sg.iters - 1);
            if (owner && !whole && ok) {
                // one thread waits until every contributor of this CTA's rank
                // has published (its acquire orders the fetches it then
                // issues); the outcome is shared by the barrier below
                bool got = true;
                if (etid == 0) {
                    for (int gc = g + 1; gc <= g_last && got; ++gc) {
                        if (!index_ok(p.status, 2 * gc + rank, 2LL * p.sk.G)) {
                            got = false;
                            break;
                        }
                        const unsigned* flag = p.sk.flags + 2 * gc + rank;
                        const uint64_t t0 = globaltimer_ns();
                        while (ld_acquire_gpu(flag) != p.sk.epoch) {
                            if (globaltimer_ns() - t0 > p.wait_limit_ns) {
                                atomicCAS(p.status, 0, kStatusTimeout);
                                got = false;
                                break;
                            }
                        }
                    }
                }
                ok = epi_bar_and(got);
            }
            const int fo = n * p.T_o + o;
            const int x0 = tx * p.box_w, y0 = ty * p.box_h, co0 = n_tile * BN;
            const bool store = ty < p.tiles_y;  // a box past the frame stores nothing
            const uint32_t tacc = tmem_base + (uint32_t)(b * BN);
            switch (out_block_channels(BN)) {
                case 64: tcp_segment_epilogue<64>(p, tacc, q, lane, etid, owner, ok, g, g_last, (int)rank, BN, co0, x0, y0, fo, store, staging, slot, smem, n_fbuf, fetch_bar, fetch_uses, bias_s); break;
                case 32: tcp_segment_epilogue<32>(p, tacc, q, lane, etid, owner, ok, g, g_last, (int)rank, BN, co0, x0, y0, fo, store, staging, slot, smem, n_fbuf, fetch_bar, fetch_uses, bias_s); break;
                default: tcp_segment_epilogue<16>(p, tacc, q, lane, etid, owner, ok, g, g_last, (int)rank, BN, co0, x0, y0, fo, store, staging, slot, smem, n_fbuf, fetch_bar, fetch_uses, bias_s); break;
            }
            // Contributors' flags consumed (every epilogue thread has passed
            // its flag wait: the fix-up has block barriers): clear them, so a
            // replay of the same launch parameters (a captured graph, whose
            // epoch is fixed) waits for fresh pieces again.
            if (owner && !whole && ok && etid == 0)
                for (int gc = g + 1; gc <= g_last; ++gc)
                    if (index_ok(p.status, 2 * gc + rank, 2LL * p.sk.G)) p.sk.flags[2 * gc + rank] = 0u;
            // TMEM buffer b is drained: hand it back to the MMA issuer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader)
                    mbar_arrive(smem_u32(&acc_empty[b]));
                else
                    mbar_arrive_remote(empty_leader + (uint32_t)(b * 8));
            }
            if (!owner) {
                // publish this CTA's piece: stores visible before the flag
                __threadfence();
                epi_bar();  // all 128 epilogue threads (owner is uniform)
                if (etid == 0 && ok && index_ok(p.status, 2 * g + rank, 2LL * p.sk.G))
                    st_release_gpu(p.sk.flags + 2 * g + rank, p.sk.epoch);
            }
            I = sg.tile_start + sg.kb1;
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
