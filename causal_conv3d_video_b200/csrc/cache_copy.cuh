// cache_copy.cuh -- the new_cache write: the last `keep` frames of
// Z = [cache; x] are copied to new_cache without ever forming Z.  Frame t of
// Z is cache[t] when t < |C|, else x[t - |C|] (the paper's cache-augmented
// input, Sec. 4; the cache carries Z's trailing frames to the next call).
#pragma once
#include "checked.cuh"
#include "params.h"

namespace ccv3d {

__device__ __forceinline__ const uint8_t* z_frame(const CopyJob& c, int n, int t) {
    return t < c.cache_len
               ? c.cache + (long long)ring_frame(n, t, c.cache_slots, c.cache_head) * c.frame_bytes
               : c.x + ((long long)n * c.T_x + (t - c.cache_len)) * c.frame_bytes;
}

// Copy part `part` of `parts` equal slices of the job with `nthreads`
// threads (thread index `tid`).  Uses 16-byte vectors when every frame is a
// multiple of 16 bytes (all pointers are 16-byte aligned by contract), else
// 4-byte, else 2-byte words.
__device__ __forceinline__ void copy_new_cache(const CopyJob& c, long long part,
                                               long long parts, int tid,
                                               int nthreads) {
    if (c.keep <= 0) return;
    const int vb = (c.frame_bytes % 16 == 0) ? 16 : ((c.frame_bytes % 4 == 0) ? 4 : 2);
    const long long per_frame = c.frame_bytes / vb;
    const long long frames = (long long)c.N * c.keep;
    const long long total = per_frame * frames;
    const long long slice = (total + parts - 1) / parts;
    const long long begin = part * slice;
    const long long end = begin + slice < total ? begin + slice : total;
    if (begin >= end) return;
    for (long long f = begin / per_frame; f < frames && f * per_frame < end; ++f) {
        const long long lo = begin > f * per_frame ? begin - f * per_frame : 0;
        const long long hi = end < (f + 1) * per_frame ? end - f * per_frame : per_frame;
        const int n = (int)(f / c.keep), j = (int)(f % c.keep);
        if ((c.paced_mask >> j) & 1u) continue;  // copied tile by tile with the GEMM
        const int t = c.z_len - c.keep + j;
        const uint8_t* src = z_frame(c, n, t);
        uint8_t* dst = c.dst + (long long)ring_frame(n, j, c.dst_slots, c.dst_head) * c.frame_bytes;
        // checked build: this slice's loop reads and writes exactly these ranges
        if (!in_bounds(c.status, src + lo * vb, (hi - lo) * vb,
                       t < c.cache_len ? c.cache : c.x,
                       t < c.cache_len ? c.cache_bytes : c.x_bytes) ||
            !in_bounds(c.status, dst + lo * vb, (hi - lo) * vb, c.dst, c.dst_bytes))
            continue;
        if (vb == 16) {
            // kU independent 16-byte loads in flight per thread before their
            // stores (source and destination never overlap: checked on host)
            constexpr int kU = 8;
            const int4* __restrict__ s = reinterpret_cast<const int4*>(src);
            int4* __restrict__ d = reinterpret_cast<int4*>(dst);
            long long v = lo + tid;
            for (; v + (long long)(kU - 1) * nthreads < hi; v += (long long)kU * nthreads) {
                int4 r[kU];
#pragma unroll
                for (int u = 0; u < kU; ++u) r[u] = __ldg(s + v + (long long)u * nthreads);
#pragma unroll
                for (int u = 0; u < kU; ++u) __stcs(d + v + (long long)u * nthreads, r[u]);
            }
            for (; v < hi; v += nthreads) __stcs(d + v, __ldg(s + v));
        } else if (vb == 4) {
            const int* s = reinterpret_cast<const int*>(src);
            int* d = reinterpret_cast<int*>(dst);
            for (long long v = lo + tid; v < hi; v += nthreads) d[v] = __ldg(s + v);
        } else {
            const unsigned short* s = reinterpret_cast<const unsigned short*>(src);
            unsigned short* d = reinterpret_cast<unsigned short*>(dst);
            for (long long v = lo + tid; v < hi; v += nthreads) d[v] = __ldg(s + v);
        }
    }
}

// Copy the share of kept frame j of batch entry n that belongs to the output
// box (tx, ty): input rows [ty*box_h*s_h, (ty+1)*box_h*s_h) and columns
// [tx*box_w*s_w, (tx+1)*box_w*s_w), the last box row and column extended to
// the frame's edge, so the boxes' shares partition the frame.  `nthreads`
// threads, 16-byte vectors (frames of tensor-core calls have Cin % 16 == 0).
__device__ __forceinline__ void copy_box_share(const CopyJob& c, int n, int j, int tx, int ty,
                                               int tiles_x, int tiles_y, int box_w, int box_h,
                                               int s_w, int s_h, int H, int W, int tid,
                                               int nthreads) {
    const int r0 = ty * box_h * s_h, c0 = tx * box_w * s_w;
    const int r1 = ty + 1 == tiles_y ? H : min(H, (ty + 1) * box_h * s_h);
    const int c1 = tx + 1 == tiles_x ? W : min(W, (tx + 1) * box_w * s_w);
    if (r0 >= r1 || c0 >= c1) return;
    const long long px_bytes = c.frame_bytes / ((long long)H * W);
    const long long row_vecs = (long long)(c1 - c0) * px_bytes / 16;
    const int t = c.z_len - c.keep + j;
    const uint8_t* src = z_frame(c, n, t);
    uint8_t* dst = c.dst + (long long)ring_frame(n, j, c.dst_slots, c.dst_head) * c.frame_bytes;
    const long long first = ((long long)r0 * W + c0) * px_bytes;
    const long long span = ((long long)(r1 - 1) * W + c1) * px_bytes - first;
    if (!in_bounds(c.status, src + first, span, t < c.cache_len ? c.cache : c.x,
                   t < c.cache_len ? c.cache_bytes : c.x_bytes) ||
        !in_bounds(c.status, dst + first, span, c.dst, c.dst_bytes))
        return;
    // warps take rows, lanes take 16-byte vectors of a row (no division)
    const int warp = tid >> 5, lane = tid & 31, nwarps = nthreads >> 5;
    constexpr int kU = 4;
    for (int row = r0 + warp; row < r1; row += nwarps) {
        const int4* s = reinterpret_cast<const int4*>(src + ((long long)row * W + c0) * px_bytes);
        int4* d = reinterpret_cast<int4*>(dst + ((long long)row * W + c0) * px_bytes);
        long long v = lane;
        for (; v + (kU - 1) * 32 < row_vecs; v += kU * 32) {
            int4 r[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) r[u] = __ldg(s + v + u * 32);
#pragma unroll
            for (int u = 0; u < kU; ++u) __stcs(d + v + u * 32, r[u]);
        }
        for (; v < row_vecs; v += 32) __stcs(d + v, __ldg(s + v));
    }
}

}  // namespace ccv3d
