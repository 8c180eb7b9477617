// conv_tc.cuh -- bf16 cached causal Conv3D as one implicit GEMM on the
// sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// GEMM view of the paper's per-tap sum (Sec. 4): rows = output pixels
// (n, o, y, x) of one output frame, columns = Cout, reduction over
// (active tap k, r, s, ci).  A tile of 128 output pixels is a box_h x box_w
// spatial box of frame o.  For every active tap k the source frame
// t = o*s_t + delta_k is picked from the cache or the input tensor map (no
// concatenation), and for every spatial tap (r, s) one TMA box load brings the
// shifted, strided box of BK input channels, zero-filled outside the image.
// Weights W[co, k, r, s, ci] are read in place (K-major rows).
//
// Warp roles (192 threads, one CTA per output tile):
//   warp 0     TMA producer (one lane): A box + B box per pipeline stage
//   warp 1     TMEM owner; one lane issues tcgen05.mma (M=128, N=BN, K=16)
//   warps 2-5  copy a slice of new_cache while the GEMM runs, then the
//              epilogue: tcgen05.ld -> + bias (fp32) -> bf16 (RNE) -> swizzled
//              shared-memory stage (the idle ring) -> TMA tensor store
// Every mbarrier wait is bounded (mbar_wait); a timeout is recorded in the
// status block and the roles drain and exit instead of hanging.
#pragma once
#include <cuda_bf16.h>

#include "cache_copy.cuh"
#include "epilogue.cuh"
#include "kwalk.cuh"
#include "params.h"
#include "ptx.cuh"

namespace ccv3d {

template <int BK>
struct TcSmem {
    static constexpr int kRowBytes = BK * 2;            // one swizzle span
    static constexpr int kABytes = kTileM * kRowBytes;  // one A stage
};

// Bytes of the operand ring, which the epilogue reuses to stage its
// 128 x bn bf16 output tile (1024-byte multiple).
__host__ __device__ constexpr size_t ring_bytes(size_t ring, int bn) {
    const size_t stage_out = (size_t)kTileM * bn * 2;
    const size_t r = ring > stage_out ? ring : stage_out;
    return (r + 1023) / 1024 * 1024;
}

// Dynamic shared memory needed for `stages` stages of an N=BN tile.
template <int BK>
__host__ __device__ constexpr size_t tc_smem_bytes(int bn, int stages) {
    return 1024 /* alignment slack */ +
           ring_bytes((size_t)stages * (TcSmem<BK>::kABytes + (size_t)bn * TcSmem<BK>::kRowBytes), bn) +
           (size_t)(2 * stages + 1) * 8 /* mbarriers */ + 16 /* tmem slot */ +
           (size_t)bn * 4 /* bias */;
}

template <int BK>
__global__ void __launch_bounds__(kTcThreads, 1)
conv_tc_kernel(const __grid_constant__ TcParams p) {
    constexpr int kRow = TcSmem<BK>::kRowBytes;
    constexpr int kA = TcSmem<BK>::kABytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stages = p.stages;
    const int BN = p.BN;              // Cout columns of this CTA's tile
    const int BNs = BN / p.n_sub;     // columns per MMA (<= 256)
    const int kB = BN * kRow;
    const int kBs = BNs * kRow;
    uint8_t* sA = smem;
    uint8_t* sB = smem + (size_t)stages * kA;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(
        smem + ring_bytes((size_t)stages * (kA + kB), BN));
    uint64_t* empty_bar = full_bar + stages;
    uint64_t* acc_bar = empty_bar + stages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_bar + 1);
    float* bias_s = reinterpret_cast<float*>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- tile coordinates: (ty, tx, n, o) x n_tile, n_tile fastest so that
    // neighbouring CTAs share the A operand in L2, then the output frame so
    // that the tiles reading one source frame through different temporal
    // taps run close together.
    const int n_tile = blockIdx.x % p.tiles_n;
    int m_tile = blockIdx.x / p.tiles_n;
    const int o = m_tile % p.T_o;
    m_tile /= p.T_o;
    const int n = m_tile % p.N;
    m_tile /= p.N;
    const int tx = m_tile % p.tiles_x;
    const int ty = m_tile / p.tiles_x;

    int n_active = 0;
#pragma unroll
    for (int k = 0; k < kMaxTaps; ++k)
        if (k < p.taps.kt && o >= p.taps.o_l[k] && o < p.taps.o_h[k]) ++n_active;
    const int iters = n_active * p.kh * p.kw * p.n_cb;

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
        tmem_alloc(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
        tmem_relinquish();
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
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0 && iters > 0) {
            // ------------------------------------------------ TMA producer
            // The reduction is walked from a per-tile starting k-block spread
            // over [0, iters), so CTAs running at the same time read
            // different weight rows.
            int act[kMaxTaps];
            const int n_act = active_tap_list(p, o, act);
            const int rot = (int)(((long long)blockIdx.x * iters) / p.rot_div) % iters;
            const uint32_t stage_bytes = (uint32_t)(kA + kB);
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
                const uint32_t fb = smem_u32(&full_bar[ring.st]);
                mbar_arrive_expect_tx(fb, stage_bytes);
                tma_load_4d(smem_u32(sA + ring.st * kA), ts.map, fb, w.cb * BK, x0, y0, ts.frame);
                for (int j = 0; j < p.n_sub; ++j)
                    tma_load_3d(smem_u32(sB + ring.st * kB + j * kBs), &p.tmap_w, fb, w.cb * BK,
                                wrow, n_tile * BN + j * BNs);
                ring.next(stages);
                if (w.next(p)) {
                    if (w.ti == n_act) w.ti = 0;  // wrap past the last tap (rotated start)
                    ts = tap_source(p, act[w.ti], n, o);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------- MMA issuer
            const uint32_t idesc = idesc_bf16_m128((uint32_t)BNs);
            const uint64_t a0 = smem_desc_kmajor(smem_u32(sA), kRow);
            const uint64_t b0 = smem_desc_kmajor(smem_u32(sB), kRow);
            Ring ring;
            for (int it = 0; it < iters; ++it) {
                if (!mbar_wait(smem_u32(&full_bar[ring.st]), ring.ph, p.status, p.wait_limit_ns))
                    break;
                tc_fence_after();
                const uint64_t a_desc = a0 + (uint64_t)((ring.st * kA) >> 4);
                const uint64_t b_desc = b0 + (uint64_t)((ring.st * kB) >> 4);
                for (int j = 0; j < p.n_sub; ++j) {
                    const uint64_t bj = b_desc + (uint64_t)((j * kBs) >> 4);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        // +32 bytes of K per step inside the swizzle span
                        umma_bf16(tmem_base + (uint32_t)(j * BNs), a_desc + 2u * kk,
                                  bj + 2u * kk, idesc, (it | kk) != 0 ? 1u : 0u);
                }
                umma_commit(smem_u32(&empty_bar[ring.st]));
                ring.next(stages);
            }
            umma_commit(smem_u32(acc_bar));
        }
        __syncwarp();
    } else {
        // ------------------------------- new_cache slice, then epilogue
        const int etid = threadIdx.x - 64;
        copy_new_cache(p.copy, blockIdx.x, gridDim.x, etid, 128);

        const bool ok = mbar_wait(smem_u32(acc_bar), 0, p.status, p.wait_limit_ns);
        tc_fence_after();
        // the ring is idle once the accumulator is complete: stage the output there
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int frame = n * p.T_o + o;
        const int x0 = tx * p.box_w, y0 = ty * p.box_h, co0 = n_tile * BN;
        const bool have_acc = iters > 0;
        switch (out_block_channels(BN)) {
            case 64: epilogue_store<64>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, frame, etid, q, lane, ok); break;
            case 32: epilogue_store<32>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, frame, etid, q, lane, ok); break;
            default: epilogue_store<16>(p, tmem_base, have_acc, bias_s, BN, smem, co0, x0, y0, frame, etid, q, lane, ok); break;
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
