// checked.cuh -- range checks of the bounds-checked build (-DCCV3D_CHECKED).
//
// The checked build (libccv3d_checked.so) tests, before every global access a
// kernel computes (generic loads and stores, the fp32 partial tiles and flags
// of the persistent kernel, bulk copies, the frame coordinate of every TMA
// load), that the address range falls inside the buffer it is meant to fall
// in.  A violation records kStatusBounds in the call's status word and the
// access is skipped, so an indexing defect shows up as CCV3D_ERR_BOUNDS from
// the status query instead of as a memory fault.  In the normal build every
// check is the constant `true` and compiles away.
#pragma once
#include <cstdint>

namespace ccv3d {

constexpr int kStatusBounds = 9;  // mirrors CCV3D_ERR_BOUNDS

#ifdef CCV3D_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

// Record a violation (first error wins, as for timeouts).
__device__ __forceinline__ void record_bounds(int* status) {
    if (status != nullptr) atomicCAS(status, 0, kStatusBounds);
}

// [p, p + nbytes) inside [base, base + extent)?
__device__ __forceinline__ bool in_bounds(int* status, const void* p, long long nbytes,
                                          const void* base, long long extent) {
    if constexpr (!kChecked) {
        return true;
    } else {
        const uintptr_t a = reinterpret_cast<uintptr_t>(p);
        const uintptr_t b = reinterpret_cast<uintptr_t>(base);
        const bool ok = base != nullptr && nbytes >= 0 && extent >= 0 && a >= b &&
                        a - b <= (uintptr_t)extent && (uintptr_t)nbytes <= (uintptr_t)extent - (a - b);
        if (!ok) record_bounds(status);
        return ok;
    }
}

// 0 <= i < n?
__device__ __forceinline__ bool index_ok(int* status, long long i, long long n) {
    if constexpr (!kChecked) {
        return true;
    } else {
        const bool ok = i >= 0 && i < n;
        if (!ok) record_bounds(status);
        return ok;
    }
}

}  // namespace ccv3d
