/*
 * ccv3d.h -- cache-aware causal Conv3D for NVIDIA B200 (sm_100a), C ABI.
 *
 * The operator ("Cache-Aware Conv3D Lowering Across Embedded World-Model
 * Decoders", Sec. 4): a temporal cache C and the current frames X form the
 * cache-augmented input Z = [C; X]_T.  With one group, temporal kernel k_t = 3
 * and effective left pad p_l = p_l^base - |C|_T, output frame o of tap k reads
 * frame o*s_t + delta_k of Z, delta_k = k*d_t - p_l; frames outside Z
 * contribute zero.  The paper's lowering has unit temporal stride (s_t = 1);
 * s_t > 1 (the encoders' temporal downsampling, which the paper leaves on
 * native Conv3D) is the same sum with output frames s_t apart, and
 * T_o = floor((|Z| + p_l - d_t*(k_t-1) - 1) / s_t) + 1.  The output is the sum
 * over taps of a spatial cross-correlation with W_k = W[:, :, k, :, :]
 * (PyTorch convention, spatial stride s, padding p, dilation d), plus the bias
 * exactly once.  Tap k is active on the output interval [o_l, o_h) where
 *   o_l = max(0, ceil(-delta_k / s_t)),  o_h = min(T_o, ceil((|Z|_T - delta_k) / s_t)),
 * and reads the source frames o_l*s_t + delta_k, ..., (o_h-1)*s_t + delta_k
 * (for s_t = 1 the equally long interval [o_l + delta_k, o_h + delta_k)).
 * Each call also writes new_cache = the last min(cache_keep, |Z|_T) frames of
 * Z, ready to be passed as the next call's cache.  (With s_t > 1, threading
 * the cache this way reproduces one whole-sequence call when every chunk
 * boundary falls on a multiple of s_t frames.)
 *
 * Memory layout (every tensor dense, row-major, channels innermost -- the
 * physical order of PyTorch's channels_last_3d):
 *   x          [N, T_x,  H,   W,   Cin ]
 *   cache      [N, |C|,  H,   W,   Cin ]   NULL allowed iff cache_len == 0
 *   w          [Cout, k_t, k_h, k_w, Cin]   a channels_last_3d Conv3d weight
 *   bias       [Cout]                       NULL iff has_bias == 0
 *   out        [N, T_o,  H_o, W_o, Cout]
 *   new_cache  [N, K',   H,   W,   Cin ]   K' = min(cache_keep, |C| + T_x);
 *                                           NULL allowed iff K' == 0
 * Element type: CCV3D_BF16 (bf16 in, fp32 accumulate, fp32 bias add, one
 * round-to-nearest-even to bf16 out) or CCV3D_FP32 (IEEE fp32 FMA, no TF32).
 * bias has the element type of the activations.
 *
 * Ownership: the caller owns every device buffer.  A plan owns host state and
 * one small device status block; ccv3d_forward allocates nothing, never
 * synchronises the host, and runs asynchronously on the given stream.
 * new_cache must not overlap x or cache (ping-pong two buffers across calls).
 *
 * Errors: functions return a ccv3d_status; nothing throws, exits or traps.
 * Device-side waits are bounded: a wait that runs out records
 * CCV3D_ERR_TIMEOUT in the plan's status block, which ccv3d_get_status reads.
 */
#ifndef CCV3D_H
#define CCV3D_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define CCV3D_API __attribute__((visibility("default")))
#else
#define CCV3D_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define CCV3D_ABI_VERSION 2 /* 2: ccv3d_stats.plans_unsupported, stream-scoped status
                               reads, ring-buffer caches */
#define CCV3D_MAX_KT 3 /* the contract's temporal kernel size */

typedef enum { CCV3D_BF16 = 0, CCV3D_FP32 = 1 } ccv3d_dtype;

typedef enum {
    CCV3D_OK = 0,
    CCV3D_ERR_INVALID = 1,      /* bad or inconsistent argument (NULL plan or
                                   pointer, negative size, forward's
                                   stride/pad/dilation differ from the plan) */
    CCV3D_ERR_UNSUPPORTED = 2,  /* outside the contract: groups != 1,
                                   k_t != 3, unknown dtype */
    CCV3D_ERR_EMPTY_OUTPUT = 3, /* T_o, H_o or W_o would be <= 0, or N == 0 */
    CCV3D_ERR_ALIGNMENT = 4,    /* a pointer is not 16-byte aligned */
    CCV3D_ERR_ALIAS = 5,        /* new_cache overlaps x or cache, or out
                                   overlaps an input */
    CCV3D_ERR_CUDA = 6,         /* a CUDA runtime/driver call failed */
    CCV3D_ERR_TIMEOUT = 7,      /* a bounded device-side wait ran out */
    CCV3D_ERR_SCRATCH_LIMIT = 8, /* ccv3d_forward_noalloc: the call needs more
                                    device scratch than its fixed array holds */
    CCV3D_ERR_BOUNDS = 9         /* bounds-checked build (libccv3d_checked.so)
                                    only: a kernel computed an address outside
                                    the buffer it indexes; the access was
                                    skipped and the output is not valid */
} ccv3d_status;

/* Conv3D call signature.  Sizes are in elements/frames. */
typedef struct {
    int N, Cin, Cout;
    int kt, kh, kw;       /* kernel extent (k_t must be 3) */
    int H, W;             /* spatial size of x and cache */
    int T_x;              /* frames in x, >= 1 */
    int cache_len;        /* |C|_T, frames in cache, >= 0 */
    int pad_t_base;       /* p_l^base, causal left pad with an empty cache */
    int cache_keep;       /* frames of Z kept in new_cache (usually p_l^base) */
    int stride_t;         /* temporal stride s_t >= 1 (1: the paper's decoder calls) */
    int stride_h, stride_w;
    int pad_h, pad_w;     /* symmetric zero padding */
    int dil_t, dil_h, dil_w;
    int groups;           /* must be 1 */
    ccv3d_dtype dtype;
    int has_bias;
} ccv3d_desc;

typedef struct {
    uint64_t calls;       /* successful ccv3d_forward calls */
    uint64_t tc_path;     /* of which ran the tcgen05 implicit-GEMM kernel */
    uint64_t simt_path;   /* of which ran the FP32 / thin-channel kernel */
    uint64_t unsupported; /* forward calls of this plan refused with
                             CCV3D_ERR_UNSUPPORTED (strict mode: no fallback) */
    uint64_t errors;      /* forward calls refused for any other reason */
    uint64_t workspace_bytes; /* device scratch the plan holds (0 unless the
                                 persistent stream-K kernel runs it) */
    uint64_t plans_unsupported; /* process-wide: ccv3d_plan calls refused with
                                   CCV3D_ERR_UNSUPPORTED (no plan exists to
                                   count them on) */
} ccv3d_stats;

typedef struct ccv3d_plan_s* ccv3d_plan_t;

/* Validate the signature, compute the output shape and the per-tap intervals
 * (integer arithmetic), choose the kernel and its tiling, and allocate the
 * plan's 256-byte device status block on the current device.  On a host with
 * no CUDA device the plan is still made, for inspection only (intervals,
 * sizes, path); ccv3d_forward then returns CCV3D_ERR_CUDA.  *out is set to
 * NULL on failure.  Errors: INVALID, UNSUPPORTED (also counted in
 * ccv3d_stats.plans_unsupported), EMPTY_OUTPUT, CUDA.
 *
 * The kernel and tiling are the planner's own choice.  Environment variables
 * CCV3D_PERSIST, CCV3D_HALO, CCV3D_FUSE, CCV3D_PAIR, CCV3D_TILE_N,
 * CCV3D_STAGES, CCV3D_BOX_W, CCV3D_HALO_BK, CCV3D_SK_PAIRS, CCV3D_NO_ROT, CCV3D_ROT,
 * CCV3D_SIMT_SMEM, CCV3D_SIMT_TILE, CCV3D_SIMT_W16, CCV3D_THIN, CCV3D_W_KW,
 * CCV3D_PACED, CCV3D_FUSED_PERSIST and CCV3D_FORCE_PATH=simt
 * override it for tests and tuning
 * sweeps, and are read only when CCV3D_TEST_OVERRIDES=1 is also set.
 *
 * The persistent stream-K kernel ("tc_persistent") launches one CTA pair per
 * resident pair slot (the occupancy of an otherwise idle GPU, queried at plan
 * time) and finishes split tiles from pieces other pairs publish, so it needs
 * all of its pairs resident at once.  If other work on the GPU keeps some off
 * the SMs for longer than the 2 s device wait limit, the waiting pairs give
 * up: the call's output is incomplete and CCV3D_ERR_TIMEOUT is recorded in
 * the status block (read it with ccv3d_get_status or
 * ccv3d_get_status_stream).  The kernel never hangs. */
CCV3D_API ccv3d_status ccv3d_plan(ccv3d_plan_t* out, const ccv3d_desc* desc);

/* The planner's temporal bookkeeping, for inspection and testing.
 * T_o/H_o/W_o: output extents.  For k < k_t: delta[k] = k*d_t - p_l,
 * [o_l[k], o_h[k]) the output frames on which tap k is active; an inactive
 * tap reports o_l = o_h = 0.  Any output pointer may be NULL. */
CCV3D_API ccv3d_status ccv3d_plan_intervals(ccv3d_plan_t plan, int* T_o, int* H_o,
                                  int* W_o, int delta[CCV3D_MAX_KT],
                                  int o_l[CCV3D_MAX_KT],
                                  int o_h[CCV3D_MAX_KT]);

/* 1 when the plan runs the tcgen05 tensor-core kernel, 0 for the SIMT kernel;
 * tile_m/tile_n receive the GEMM tile of one CTA or CTA pair: tile_m is 256
 * when a CTA pair shares each MMA (cta_group::2), else 128 (may be NULL). */
CCV3D_API int ccv3d_plan_path(ccv3d_plan_t plan, int* tile_m, int* tile_n);

/* Name of the kernel the plan launches (static string; "" for NULL):
 *   "tc_pair"        CTA-pair implicit GEMM (cta_group::2)
 *   "tc_pair_halo"   CTA pair, one input row strip per (tap, channel block)
 *   "tc_pair_fused"  CTA pair with row strips, two output frames per tile
 *   "tc_pair_fused_persistent"  the same stages, one resident CTA pair per SM
 *                    pair walking the tiles, double-buffered accumulators
 *   "tc_persistent"  persistent stream-K over all SM pairs
 *   "tc_single"      one CTA per tile
 *   "tc_thin"        one CTA per (output row, group of output frames) for
 *                    outputs too narrow for an MMA's N (Cout not a multiple of
 *                    16): the temporal and column taps stacked along N, the
 *                    column taps summed in the epilogue
 *   "simt"           FFMA, one thread per pixel and 4 output channels
 *   "simt_warp"      FFMA, one warp per pixel and 4 output channels (small calls)
 *   "simt_warp16"    FFMA, one warp per pixel and all (<= 16) output channels,
 *                    weights staged in shared memory (small calls, Cin | 32)
 *   "simt_smem"      FFMA, one block per band of output rows with the weights
 *                    and input rows staged in shared memory (small calls that fit)
 *   "simt_tile"      FFMA, large calls with <= 4 output channels: 8 x 128-pixel
 *                    tiles, input patches staged per 8 channels in shared memory */
CCV3D_API const char* ccv3d_plan_kernel(ccv3d_plan_t plan);

/* Reduction tiling of a tensor-core plan (inspection; no counterpart in the
 * paper): k_block = input channels per pipeline stage (64, 32 or 16), stages
 * = depth of the shared-memory ring, workspace_pairs = CTA pairs of the
 * persistent stream-K kernel (0 for the other kernels).  Any output pointer
 * may be NULL.  Errors: INVALID for a NULL plan, UNSUPPORTED for a SIMT plan
 * (outputs are then 0). */
CCV3D_API ccv3d_status ccv3d_plan_tiling(ccv3d_plan_t plan, int* k_block, int* stages,
                                         int* workspace_pairs);

/* Run one cached causal Conv3D call on `stream` (device pointers, layouts as
 * above).  stride = {s_h, s_w}, pad = {p_h, p_w}, dilation = {d_t, d_h, d_w}
 * must equal the plan's (the call signature of the paper's patched module).
 * Pointers must be 16-byte aligned.  out and new_cache are written in the
 * same launch.  Errors: INVALID, ALIGNMENT, ALIAS, CUDA. */
CCV3D_API ccv3d_status ccv3d_forward(ccv3d_plan_t plan, const void* x, const void* cache,
                           const void* w, const void* bias, void* out,
                           void* new_cache, const int stride[2],
                           const int pad[2], const int dilation[3],
                           cudaStream_t stream);

/* The same call with the cache kept in a ring buffer (the cache-augmented
 * input Z = [C; X] of Sec. 4, with the cache state carried from chunk to
 * chunk in place).  Instead of rewriting all K' = min(cache_keep, |Z|) frames
 * of new_cache, a call writes only the frames of the new cache that arrive
 * with it -- n_w = min(K', T_x) frames of x -- so a streaming decoder
 * (T_x = 1, K' = 2) writes one frame per call instead of two.
 *
 *   ring  [N, ring_slots, H, W, Cin], device memory owned by the caller.
 *         Cache frame t (0 <= t < |C|, |C| = the plan's cache_len) of batch
 *         entry n is slot (head + t) mod ring_slots of entry n.  The call
 *         writes the last n_w frames of x to slots (head + |C| + i) mod
 *         ring_slots, i < n_w; no other slot changes.
 *   next_head  (may be NULL) receives (head + |C| + n_w - K') mod ring_slots:
 *         the head of the new cache, whose K' frames then sit at slots
 *         (next_head + t) mod ring_slots -- pass it, with cache_len = K', to
 *         the next call.
 * Requirements: 0 <= head < ring_slots and ring_slots >= |C| + n_w (so no
 * slot the call writes holds a frame it reads; ring_slots = cache_keep + T_x
 * always suffices), ring 16-byte aligned and overlapping neither x, w nor
 * out.  The first call of a stream uses a plan with cache_len = 0 and any
 * head.  Outputs, kernels and numerics are those of ccv3d_forward (the same
 * plan gives bit-identical out).  Errors: INVALID (as ccv3d_forward, or
 * ring_slots / head out of range), ALIGNMENT, ALIAS, CUDA. */
CCV3D_API ccv3d_status ccv3d_forward_ring(ccv3d_plan_t plan, const void* x, void* ring,
                                          int ring_slots, int head, const void* w,
                                          const void* bias, void* out, const int stride[2],
                                          const int pad[2], const int dilation[3],
                                          cudaStream_t stream, int* next_head);

/* Counters since the plan was made (route counters of the paper's acceptance
 * criteria: fast-path hits, refusals). */
CCV3D_API ccv3d_status ccv3d_get_stats(ccv3d_plan_t plan, ccv3d_stats* stats);

/* Synchronise the device, then return and clear the status recorded by the
 * plan's kernels: CCV3D_OK, or CCV3D_ERR_TIMEOUT after a bounded wait ran out.
 * CCV3D_ERR_CUDA when the device reports an error. */
CCV3D_API ccv3d_status ccv3d_get_status(ccv3d_plan_t plan);

/* As ccv3d_get_status, but ordered on `stream` only: waits for the work
 * already queued on that stream (not the whole device), then returns and
 * clears the status the plan's kernels recorded.  Calls of the plan on other
 * streams are covered only once they have completed.  Allocates nothing.
 * Errors: INVALID (NULL plan), CUDA. */
CCV3D_API ccv3d_status ccv3d_get_status_stream(ccv3d_plan_t plan, cudaStream_t stream);

/* Free the plan and its device status block.  NULL is ignored. */
CCV3D_API void ccv3d_destroy(ccv3d_plan_t plan);

/* Static description of a status code. */
CCV3D_API const char* ccv3d_strerror(ccv3d_status status);

/* Bytes of output and new_cache for a plan (sizes for the caller's
 * allocation).  Any pointer may be NULL. */
CCV3D_API ccv3d_status ccv3d_plan_sizes(ccv3d_plan_t plan, size_t* out_bytes,
                              size_t* new_cache_bytes, int* new_cache_frames);

/* Self-test of the bounded device wait: launches one block that waits on an
 * mbarrier nothing will complete, with a limit of `limit_ns` nanoseconds.
 * Returns CCV3D_ERR_TIMEOUT (the expected outcome: the wait gave up and
 * reported it, and the context stays usable), CCV3D_OK if the wait completed
 * (a defect), or CCV3D_ERR_CUDA. */
CCV3D_API ccv3d_status ccv3d_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

/* Self-test of the range checks: launches one thread that hands the device
 * check one byte range ending past its buffer and one index past its count
 * (neither is dereferenced).  Returns CCV3D_ERR_BOUNDS in the bounds-checked
 * build (libccv3d_checked.so, compiled with -DCCV3D_CHECKED: every computed
 * global address is checked before use and a violation is recorded, the
 * access skipped), CCV3D_OK in the normal build, where the checks compile
 * away; CCV3D_ERR_CUDA on a CUDA failure.  Allocates a 4-byte status word. */
CCV3D_API ccv3d_status ccv3d_selftest_bounds(cudaStream_t stream);

/* Post-decode uint8 quantisation of decoded frames, the step after the
 * decoder (FastVideo pull request "Quantize frames to uint8 on-device before
 * the post-decode D->H copy", Summary and Correctness):
 *   out[i] = trunc(clamp(fp32(in[i]) * 255, 0, 255)),  NaN -> 0,
 * the multiply in fp32 for both input types, the cast truncating toward zero
 * (PyTorch's float -> uint8).  Elementwise over n values in any layout; the
 * caller copies `out` to the host (n bytes instead of 4n or 2n).
 *   in     n values of `dtype` (CCV3D_FP32 or CCV3D_BF16), device memory
 *   out    n bytes, device memory; must not overlap `in`
 * Both pointers 16-byte aligned.  Asynchronous on `stream`; no allocation.
 * Errors: INVALID (n < 0, unknown dtype, NULL pointer with n > 0), ALIGNMENT,
 * ALIAS (the buffers overlap), CUDA (launch failure).  n == 0 does nothing. */
CCV3D_API ccv3d_status ccv3d_quantize_u8(const void* in, ccv3d_dtype dtype, void* out,
                                         long long n, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Forward call that allocates nothing.
 *
 * The paper has no counterpart to this entry point: it serves callers that
 * must not allocate device memory, directly or through this library -- code
 * that runs inside a caching allocator's own hooks, or under a serving
 * runtime that owns the whole device-memory budget and forbids cudaMalloc /
 * cudaFree (and the device-wide synchronisation cudaFree implies) outside its
 * pool.  Such a caller cannot create a plan (ccv3d_plan allocates the plan's
 * status block and, for split tiles, its scratch), so this call takes the
 * signature itself and plans on the host stack each time.
 *
 * It runs the persistent stream-K CTA-pair kernel.  That kernel's device
 * scratch -- a status word, the split-tile flags and the fp32 partial tiles --
 * lives in one static array of CCV3D_NOALLOC_SCRATCH_BYTES bytes compiled into
 * this library: a GPU holds the array, from the moment the CUDA driver loads
 * this library's device code on it, until the process exits.  Under the
 * driver's lazy module loading (the default) that load can happen inside the
 * first call of this function on a device -- the first call also looks up
 * the array's device address (cudaGetSymbolAddress) with that device current
 * -- so make one call (or one ccv3d_plan / ccv3d_forward) on each device
 * before entering the context that may not allocate, and before any stream
 * capture.
 *
 * All calls share the array and it keeps what the last call left there, so
 * calls that overlap on the GPU (other streams, other host threads) race:
 * the caller must order them.  The split-tile flags carry a per-device call
 * number, so stale flags from earlier calls are never mistaken for this
 * call's.  A device-side wait that runs out (see the persistent kernel's
 * co-residency note at ccv3d_plan) leaves that call's output incomplete and
 * records CCV3D_ERR_TIMEOUT in the array's status word, which keeps the first
 * such record until ccv3d_noalloc_get_status reads and clears it.
 *
 * Arguments and layouts are those of ccv3d_forward, with the signature in
 * `desc` instead of a plan.  Covered: bf16 signatures that run on the
 * CTA-pair tensor-core path with at most 64 (n, o) output frames, each with
 * an active tap; others return CCV3D_ERR_UNSUPPORTED.  A call whose scratch
 * (2 x pairs x 128 x Cout-tile x 4 bytes, plus flags) would not fit returns
 * CCV3D_ERR_SCRATCH_LIMIT before any device work.  Other errors as
 * ccv3d_forward.  This call never synchronises the host; no device memory is
 * allocated or freed. */
#define CCV3D_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
CCV3D_API ccv3d_status ccv3d_forward_noalloc(const ccv3d_desc* desc, const void* x,
                                             const void* cache, const void* w,
                                             const void* bias, void* out, void* new_cache,
                                             const int stride[2], const int pad[2],
                                             const int dilation[3], cudaStream_t stream);

/* Status of the ccv3d_forward_noalloc calls on the current device: waits for
 * the work queued on `stream`, then returns and clears the status word of the
 * static array -- CCV3D_OK, or CCV3D_ERR_TIMEOUT when a call's bounded wait
 * ran out since the last read.  Allocates nothing (the word is copied to
 * pageable host memory).  Errors: CUDA. */
CCV3D_API ccv3d_status ccv3d_noalloc_get_status(cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CCV3D_H */
