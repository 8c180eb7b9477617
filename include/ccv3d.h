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

#define CCV3D_ABI_VERSION 1
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
    CCV3D_ERR_SCRATCH_LIMIT = 8 /* ccv3d_forward_noalloc: the call needs more
                                   device scratch than its fixed array holds */
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
    uint64_t unsupported; /* forward calls refused as outside the contract */
    uint64_t errors;      /* forward calls refused for any other reason */
    uint64_t workspace_bytes; /* device scratch used per call (0) */
} ccv3d_stats;

typedef struct ccv3d_plan_s* ccv3d_plan_t;

/* Validate the signature, compute the output shape and the per-tap intervals
 * (integer arithmetic), choose the kernel and its tiling, and allocate the
 * plan's 256-byte device status block on the current device.  On a host with
 * no CUDA device the plan is still made, for inspection only (intervals,
 * sizes, path); ccv3d_forward then returns CCV3D_ERR_CUDA.  *out is set to
 * NULL on failure.  Errors: INVALID, UNSUPPORTED, EMPTY_OUTPUT, CUDA. */
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
 *   "tc_persistent"  persistent stream-K over all SM pairs
 *   "tc_single"      one CTA per tile
 *   "simt"           FFMA, one thread per pixel and 4 output channels
 *   "simt_warp"      FFMA, one warp per pixel and 4 output channels (small calls) */
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

/* Counters since the plan was made (route counters of the paper's acceptance
 * criteria: fast-path hits, refusals). */
CCV3D_API ccv3d_status ccv3d_get_stats(ccv3d_plan_t plan, ccv3d_stats* stats);

/* Synchronise the device, then return and clear the status recorded by the
 * plan's kernels: CCV3D_OK, or CCV3D_ERR_TIMEOUT after a bounded wait ran out.
 * CCV3D_ERR_CUDA when the device reports an error. */
CCV3D_API ccv3d_status ccv3d_get_status(ccv3d_plan_t plan);

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
 * this library: every GPU that loads the library holds the array until the
 * process exits, whether or not it calls this function.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.
 *
 * All calls share the array and it keeps what the last call left there, so
 * calls that overlap on the GPU (other streams, other host threads) race:
 * the caller must order them.  Each call clears the status word before its
 * launch; the split-tile flags carry a per-device call number, so stale flags
 * from earlier calls are never mistaken for this call's.
 *
 * Arguments and layouts are those of ccv3d_forward, with the signature in
 * `desc` instead of a plan.  Covered: bf16 signatures that run on the
 * CTA-pair tensor-core path with at most 64 (n, o) output frames, each with
 * an active tap; others return CCV3D_ERR_UNSUPPORTED.  A call whose scratch
 * (2 x pairs x 128 x Cout-tile x 4 bytes, plus flags) would not fit returns
 * CCV3D_ERR_SCRATCH_LIMIT before any device work.  Other errors as
 * ccv3d_forward; a device-side wait that runs out is recorded in the shared
 * status word, which this entry point does not read back (it never
 * synchronises the host).  No device memory is allocated or freed. */
#define CCV3D_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
CCV3D_API ccv3d_status ccv3d_forward_noalloc(const ccv3d_desc* desc, const void* x,
                                             const void* cache, const void* w,
                                             const void* bias, void* out, void* new_cache,
                                             const int stride[2], const int pad[2],
                                             const int dilation[3], cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CCV3D_H */
