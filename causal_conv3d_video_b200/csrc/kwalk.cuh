// kwalk.cuh -- division-free bookkeeping for the single-thread issue loops.
//
// The TMA producer and the MMA issuer are single threads on the critical
// path of every k-block; an integer division there costs tens of cycles (a
// 64-bit one ~100), against 48-96 tensor-core cycles of work per k-block on
// the thin signatures.  These helpers step the ring slot/phase and the
// (tap, r, s, channel block) coordinates of the reduction incrementally.
#pragma once
#include "checked.cuh"
#include "params.h"

namespace ccv3d {

// Slot and phase bit of a `stages`-deep ring.
struct Ring {
    int st = 0;
    uint32_t ph = 0;
    __device__ __forceinline__ void next(int stages) {
        if (++st == stages) {
            st = 0;
            ph ^= 1u;
        }
    }
};

// Position in the reduction of one output tile: active tap index `ti` (into
// the tile's list of active taps), spatial tap (r, s), channel block cb;
// channel block fastest, then s, then r, then tap.
struct KWalk {
    int ti, r, s, cb;

    __device__ __forceinline__ void set(int kb, const TcParams& p) {
        const int per_tap = p.kh * p.kw * p.n_cb;
        ti = kb / per_tap;
        const int rem = kb - ti * per_tap;
        const int rs = rem / p.n_cb;
        cb = rem - rs * p.n_cb;
        r = rs / p.kw;
        s = rs - r * p.kw;
    }

    // Advance by one k-block; true when the tap index changed.
    __device__ __forceinline__ bool next(const TcParams& p) {
        if (++cb < p.n_cb) return false;
        cb = 0;
        if (++s < p.kw) return false;
        s = 0;
        if (++r < p.kh) return false;
        r = 0;
        ++ti;
        return true;
    }
};

// Source of one temporal tap of output frame o (paper, Sec. 4): frame
// t = o*s_t + delta_k of Z, taken from the cache when t < |C|, else from x.
struct TapSrc {
    const CUtensorMap* map;
    int frame;  // frame coordinate in that tensor map (n * T + t)
    int wtap;   // k * kh * kw: first weight row of the tap
};

__device__ __forceinline__ TapSrc tap_source(const TcParams& p, int k, int n, int o) {
    TapSrc ts;
    const int t = o * p.taps.s_t + p.taps.delta[k];
    if (t < p.cache_len) {
        ts.map = &p.tmap_c;
        ts.frame = ring_frame(n, t, p.cache_slots, p.cache_head);
    } else {
        ts.map = &p.tmap_x;
        ts.frame = n * p.T_x + (t - p.cache_len);
    }
    // checked build: a frame outside the tensor map is recorded and clamped
    // (the load still completes its barrier, so the call ends promptly)
    if (!index_ok(p.status, ts.frame, t < p.cache_len ? p.c_frames : p.x_frames)) ts.frame = 0;
    ts.wtap = k * p.kh * p.kw;
    return ts;
}

// Active taps of output frame o, in order; returns their count.
__device__ __forceinline__ int active_tap_list(const TcParams& p, int o, int (&act)[kMaxTaps]) {
    int n_act = 0;
    for (int k = 0; k < p.taps.kt; ++k)
        if (o >= p.taps.o_l[k] && o < p.taps.o_h[k]) act[n_act++] = k;
    return n_act;
}

}  // namespace ccv3d
