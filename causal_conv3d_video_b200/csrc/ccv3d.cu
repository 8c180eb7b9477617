// ccv3d.cu -- C ABI of libccv3d: planner, tensor-map builder and launches.
//
// The planner computes the temporal bookkeeping of "Cache-Aware Conv3D
// Lowering Across Embedded World-Model Decoders" (Sec. 4) in integer
// arithmetic: |Z| = |C| + T_x, p_l = p_l^base - |C|,
// T_o = floor((|Z| + p_l - d_t (k_t - 1) - 1) / s_t) + 1, delta_k = k d_t - p_l
// and the valid output interval of every tap, [o_l, o_h) =
// [max(0, ceil(-delta_k / s_t)), min(T_o, ceil((|Z| - delta_k) / s_t))) (the
// intersection of 0 <= o < T_o and 0 <= o s_t + delta_k < |Z|; s_t = 1 in the
// paper, s_t > 1 for the encoders' temporal downsampling).  Nothing
// concatenates C and X: the kernels pick each source frame from one or the
// other.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "ccv3d.h"
#include "checked.cuh"
#include "conv_simt.cuh"
#include "conv_tc.cuh"
#include "conv_tc2.cuh"
#include "conv_tc2f.cuh"
#include "conv_tc2fp.cuh"
#include "conv_tc2h.cuh"
#include "conv_tcp.cuh"
#include "conv_tcn.cuh"
#include "params.h"
#include "quantize.cuh"

using namespace ccv3d;

struct ccv3d_plan_s {
    ccv3d_desc d;
    int T_o, H_o, W_o, z_len, p_l, keep;
    int delta[kMaxTaps], o_l[kMaxTaps], o_h[kMaxTaps];
    int path_tc;  // 1: tcgen05 implicit GEMM, 0: SIMT
    int path_tc_candidate;  // the tensor-core tiling below is filled in
    int BK, BN, n_sub, box_h, box_w, tiles_x, tiles_y, tiles_n, stages, tmem_cols;
    int pair;  // 1: CTA-pair kernel (M = 256 per pair), 0: one CTA per 128-row tile
    int persist;  // 1: persistent stream-K pair kernel
    int halo;     // 1: pair kernel loading each input row strip once per (tap, channel block)
    int halo_w;   // halo: pixels per strip
    int fused;    // 1: halo pair kernel computing two output frames per tile
    int fused_persist;  // 1: the persistent form of the two-frame kernel (conv_tc2fp.cuh)
    int thin;     // 1: thin-output kernel, taps stacked along N (conv_tcn.cuh)
    int tn_G, tn_groups, tn_cbk;  // thin: frames per tile, frame groups, TMEM columns per frame
    int simt_kind;  // SIMT plans: 0 thread per unit, 1 warp per unit, 2 shared-memory blocks,
                    // 3 tiles of thin outputs, 4 warp per pixel for all (<= 16) channels
    int simt_band_h, simt_rows_in, simt_threads;
    size_t simt_smem;
    int G, n_acc;  // persistent: CTA pairs launched, TMEM accumulator buffers
    long long frame_start[kMaxFrames + 1], sk_total;
    size_t smem_bytes;
    int device;
    int* d_status;
    void* scratch;  // persistent: flags [2G] then fp32 partial tiles [2G][128][BN]
    size_t scratch_bytes;
    std::atomic<unsigned> epoch{0};
    std::atomic<uint64_t> calls{0}, tc{0}, simt{0}, unsupported{0}, errors{0};
};

namespace {

// ccv3d_plan calls refused as outside the contract, over the whole process
// (a refused signature never gets a plan whose counters could hold it).
std::atomic<uint64_t> g_plans_unsupported{0};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// ceil(a / b) for b > 0 and any sign of a.
int ceil_div_floor0(long long a, long long b) {
    return a >= 0 ? (int)((a + b - 1) / b) : -(int)((-a) / b);
}

// Planner: the paper's closed forms.  Returns CCV3D_OK or the refusal code.
ccv3d_status compute_intervals(const ccv3d_desc& d, ccv3d_plan_s* p) {
    if (d.N < 0 || d.Cin <= 0 || d.Cout <= 0 || d.kt <= 0 || d.kh <= 0 || d.kw <= 0 ||
        d.H <= 0 || d.W <= 0 || d.T_x < 1 || d.cache_len < 0 || d.pad_t_base < 0 ||
        d.cache_keep < 0 || d.stride_t <= 0 || d.stride_h <= 0 || d.stride_w <= 0 ||
        d.pad_h < 0 || d.pad_w < 0 || d.dil_t <= 0 || d.dil_h <= 0 || d.dil_w <= 0 ||
        d.groups <= 0)
        return CCV3D_ERR_INVALID;
    if (d.groups != 1 || d.kt != 3 || (d.dtype != CCV3D_BF16 && d.dtype != CCV3D_FP32))
        return CCV3D_ERR_UNSUPPORTED;
    const int s_t = d.stride_t;
    p->z_len = d.cache_len + d.T_x;
    p->p_l = d.pad_t_base - d.cache_len;
    // output o's tap k reads frame o*s_t + delta_k of Z; no right pad
    const long long tn = (long long)p->z_len + p->p_l - (long long)d.dil_t * (d.kt - 1) - 1;
    const long long hn = (long long)d.H + 2LL * d.pad_h - (long long)d.dil_h * (d.kh - 1) - 1;
    const long long wn = (long long)d.W + 2LL * d.pad_w - (long long)d.dil_w * (d.kw - 1) - 1;
    const long long T_o = tn < 0 ? 0 : tn / s_t + 1;
    const long long H_o = hn < 0 ? 0 : hn / d.stride_h + 1;
    const long long W_o = wn < 0 ? 0 : wn / d.stride_w + 1;
    // extents the kernels index with 32-bit integers (tiles, frames, pixels of a frame)
    constexpr long long kMax = 0x7fffffffLL;
    if ((long long)p->z_len > kMax || T_o > kMax || H_o * W_o > kMax ||
        (long long)d.H * d.W > kMax || (long long)d.N * (T_o > p->z_len ? T_o : p->z_len) > kMax)
        return CCV3D_ERR_UNSUPPORTED;
    p->T_o = (int)T_o;
    p->H_o = (int)H_o;
    p->W_o = (int)W_o;
    p->keep = std::min(d.cache_keep, p->z_len);
    for (int k = 0; k < kMaxTaps; ++k) {
        p->delta[k] = p->o_l[k] = p->o_h[k] = 0;
        if (k >= d.kt) continue;
        const int delta = k * d.dil_t - p->p_l;
        // o*s_t + delta in [0, |Z|)  <=>  ceil(-delta/s_t) <= o < ceil((|Z|-delta)/s_t)
        const int lo = std::max(0, ceil_div_floor0(-delta, s_t));
        const int hi = std::min(p->T_o, ceil_div_floor0(p->z_len - delta, s_t));
        p->delta[k] = delta;
        if (hi > lo) {
            p->o_l[k] = lo;
            p->o_h[k] = hi;
        }
    }
    if (d.N == 0 || p->T_o <= 0 || p->H_o <= 0 || p->W_o <= 0) return CCV3D_ERR_EMPTY_OUTPUT;
    return CCV3D_OK;
}

constexpr size_t kSmemBudget = 225 * 1024;

// kind: 0 one CTA per tile, 1 CTA pair, 2 persistent CTA pair (3: halo pair,
// sized by halo_smem_for)
template <int BK>
size_t smem_for(int kind, int bn, int stages) {
    return kind == 2 ? tcp_smem_bytes<BK>(bn, stages)
                     : (kind == 1 ? tc2_smem_bytes<BK>(bn, stages) : tc_smem_bytes<BK>(bn, stages));
}

size_t fused_smem_for(int bk, int bn, int stages, int kh, int kw, int halo_w) {
    switch (bk) {
        case 64: return tc2f_smem_bytes<64>(bn, stages, kh, kw, halo_w);
        case 32: return tc2f_smem_bytes<32>(bn, stages, kh, kw, halo_w);
        default: return tc2f_smem_bytes<16>(bn, stages, kh, kw, halo_w);
    }
}

size_t halo_smem_for(int bk, int bn, int stages, int kh, int kw, int halo_w) {
    switch (bk) {
        case 64: return tc2h_smem_bytes<64>(bn, stages, kh, kw, halo_w);
        case 32: return tc2h_smem_bytes<32>(bn, stages, kh, kw, halo_w);
        default: return tc2h_smem_bytes<16>(bn, stages, kh, kw, halo_w);
    }
}

template <int BK>
int pick_stages(int kind, int bn, int want) {
    int s = want > 0 ? std::min(want, 12) : 8;
    int lo = 2;
    if (kind == 2) {
        // the persistent kernel's owner fetches whole fp32 output blocks of
        // the contributors into its idle ring: keep room for one
        while (tcp_ring_bytes<BK>(bn, lo) < (size_t)kTileM * out_block_channels(bn) * 4) ++lo;
        s = std::max(s, lo);
    }
    while (s > lo && smem_for<BK>(kind, bn, s) > kSmemBudget) --s;
    return s;
}

// Function attributes belong to each device's context: set them once per
// device (the current one).
constexpr int kMaxDevices = 64;

template <int BK>
void set_smem_attrs() {
    static std::atomic<bool> done[kMaxDevices];
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    if (dev < 0 || dev >= kMaxDevices || done[dev].load(std::memory_order_acquire)) return;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev].load(std::memory_order_relaxed)) return;
    {
        cudaFuncSetAttribute(conv_tc_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(227 * 1024));
        cudaFuncSetAttribute(conv_tc2_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(227 * 1024));
        cudaFuncSetAttribute(conv_tcp_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(227 * 1024));
        cudaFuncSetAttribute(conv_tc2h_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(227 * 1024));
        cudaFuncSetAttribute(conv_tc2f_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(227 * 1024));
        cudaFuncSetAttribute(conv_tc2fp_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(227 * 1024));
        cudaFuncSetAttribute(conv_tcn_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(227 * 1024));
        cudaGetLastError();
    }
    done[dev].store(true, std::memory_order_release);
}

// CTA pairs of the persistent kernel that can be resident at once.  The
// occupancy query costs milliseconds of host time, so its answer is kept per
// (device, channel block, shared memory) for the life of the process.
struct ResidentEntry {
    int dev, bk, pairs;
    size_t smem;
    int threads;
};
constexpr int kResidentEntries = 64;
std::mutex g_resident_mu;
ResidentEntry g_resident[kResidentEntries];
int g_resident_n = 0;

template <int BK>
int resident_pairs(size_t smem, bool fused = false, int threads = kTcpThreads) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    {
        std::lock_guard<std::mutex> lock(g_resident_mu);
        for (int i = 0; i < g_resident_n; ++i)
            if (g_resident[i].dev == dev && g_resident[i].bk == (fused ? -BK : BK) &&
                g_resident[i].smem == smem && g_resident[i].threads == threads)
                return g_resident[i].pairs;
    }
    set_smem_attrs<BK>();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    const cudaError_t e = fused ? cudaOccupancyMaxActiveClusters(&n, conv_tc2fp_kernel<BK>, &cfg)
                                : cudaOccupancyMaxActiveClusters(&n, conv_tcp_kernel<BK>, &cfg);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> lock(g_resident_mu);
    if (g_resident_n < kResidentEntries)
        g_resident[g_resident_n++] = {dev, fused ? -BK : BK, n, smem, threads};
    return n;
}

// Planner overrides (kernel form, tiling, ring depth) for tests and tuning
// sweeps.  They are read only when CCV3D_TEST_OVERRIDES=1 is also set, so a
// deployment's environment cannot change the kernel, the reduction order or
// the performance behind the ABI; without the gate every plan is the
// planner's own choice.
const char* override_env(const char* name) {
    const char* gate = std::getenv("CCV3D_TEST_OVERRIDES");
    if (gate == nullptr || std::strcmp(gate, "1") != 0) return nullptr;
    return std::getenv(name);
}

bool force_simt() {
    const char* e = override_env("CCV3D_FORCE_PATH");
    return e != nullptr && std::strcmp(e, "simt") == 0;
}

// Integer override (0 = the planner's choice).
int env_int(const char* name) {
    const char* e = override_env(name);
    return e != nullptr ? std::atoi(e) : 0;
}

// Widest channel block (k-block depth) that divides Cin.
int widest_bk(int Cin) { return Cin % 64 == 0 ? 64 : (Cin % 32 == 0 ? 32 : 16); }

// Schedule of the persistent stream-K pair kernel: usable when the plan runs
// CTA pairs, every output frame has an active tap and the (n, o) frames fit
// the schedule table.  On success the plan switches to it (persist = 1, no
// halo strips, the widest channel block: a halo sizing may have narrowed it)
// and true is returned; otherwise the plan is left as it was.
bool setup_persistent(const ccv3d_desc& d, ccv3d_plan_s* p) {
    if (!p->path_tc_candidate || !p->pair) return false;
    const int frames = d.N * p->T_o;
    if (frames > kMaxFrames) return false;
    const int bk = widest_bk(d.Cin);
    const int per_tap = d.kh * d.kw * ceil_div(d.Cin, bk);
    long long start[kMaxFrames + 1];
    long long acc = 0;
    const long long tiles_per_frame = (long long)((p->tiles_x * p->tiles_y + 1) / 2) * p->tiles_n;
    for (int f = 0; f < frames; ++f) {
        const int o = f % p->T_o;
        int a = 0;
        for (int k = 0; k < d.kt; ++k) a += (o >= p->o_l[k] && o < p->o_h[k]) ? 1 : 0;
        if (a == 0) return false;
        start[f] = acc;
        acc += tiles_per_frame * a * per_tap;
    }
    start[frames] = acc;
    for (int f = 0; f <= frames; ++f) p->frame_start[f] = start[f];
    p->sk_total = acc;
    p->BK = bk;
    p->halo = 0;
    p->fused = 0;
    p->fused_persist = 0;
    p->persist = 1;
    return true;
}

// Ring depth, shared memory and TMEM columns of the chosen tensor-core kernel.
void size_tc(const ccv3d_desc& d, ccv3d_plan_s* p) {
    const int per_tap = d.kh * d.kw * ceil_div(d.Cin, p->BK);
    const int kind = p->persist ? 2 : p->pair;
    // Short reductions (few k-blocks per tile) are dominated by each tile's
    // fill and epilogue: without the persistent kernel, keep the ring small
    // enough for 3 CTAs per SM so one CTA's epilogue overlaps the others.
    int want_s = env_int("CCV3D_STAGES");
    if (want_s == 0 && !p->persist && 3 * per_tap <= 96) want_s = 4;
    switch (p->BK) {
        case 64: p->stages = pick_stages<64>(kind, p->BN, want_s); p->smem_bytes = smem_for<64>(kind, p->BN, p->stages); break;
        case 32: p->stages = pick_stages<32>(kind, p->BN, want_s); p->smem_bytes = smem_for<32>(kind, p->BN, p->stages); break;
        default: p->stages = pick_stages<16>(kind, p->BN, want_s); p->smem_bytes = smem_for<16>(kind, p->BN, p->stages); break;
    }
    p->n_acc = (p->persist && 2 * p->BN <= 512) ? 2 : 1;
    p->tmem_cols = 32;
    while (p->tmem_cols < p->n_acc * p->BN) p->tmem_cols *= 2;
}

// Halo variant of the pair kernel for tiles of one 128-pixel output row at
// unit W stride.  Its stages are large (kh strips + kh*kw weight tiles), so
// it is sized for two CTAs per SM: the widest channel block whose stages fit
// at least 2 deep in half of the shared memory.  Measured on the 96-channel
// 720x1280 call it beats the plain pair kernel (which needs 3-4 CTAs per SM
// of small stages) by a third.  CCV3D_HALO=0 disables it; CCV3D_HALO_BK and
// CCV3D_STAGES override its channel block and depth.
void setup_halo(const ccv3d_desc& d, ccv3d_plan_s* p) {
    p->halo = 0;
    const char* he = override_env("CCV3D_HALO");
    if (he != nullptr && std::atoi(he) == 0) return;
    if (!p->pair || p->persist) return;
    if (p->box_w != 128 || p->box_h != 1 || d.stride_w != 1) return;
    const int halo_w = 128 + (d.kw - 1) * d.dil_w;
    if (halo_w > 256) return;
    const size_t budget = kSmemBudget / 2;  // two CTAs per SM
    const int want_bk = env_int("CCV3D_HALO_BK"), want_s = env_int("CCV3D_STAGES");
    for (int bk : {64, 32, 16}) {
        if (d.Cin % bk != 0 || (want_bk > 0 && bk != want_bk)) continue;
        int s = want_s >= 2 ? want_s : 8;
        const size_t cap = want_s >= 2 ? kSmemBudget : budget;
        while (s >= 2 && halo_smem_for(bk, p->BN, s, d.kh, d.kw, halo_w) > cap) --s;
        if (s < 2) continue;
        p->halo = 1;
        p->halo_w = halo_w;
        p->BK = bk;
        p->stages = s;
        p->smem_bytes = halo_smem_for(bk, p->BN, s, d.kh, d.kw, halo_w);
        return;
    }
}

// Two output frames per tile on the halo kernel (conv_tc2f.cuh): with unit
// temporal stride and dilation, frames o and o+1 share their source frames,
// so one MMA of N = 2 Cout covers both, with 1.5x fewer MMAs and strip loads
// per output frame for thin Cout (<= 128).  Stages of one kernel row keep 4
// in flight per CTA at two CTAs per SM.  Measured on the 720x1280 four-frame
// calls: 2068 vs 2405 us (96 channels) and 3631 vs 4315 us (192 -> 96)
// against the halo kernel.  CCV3D_FUSE=0 disables it.
void setup_fused(const ccv3d_desc& d, ccv3d_plan_s* p) {
    p->fused = 0;
    const char* fe = override_env("CCV3D_FUSE");
    if (fe != nullptr && std::atoi(fe) == 0) return;
    if (!p->halo || d.stride_t != 1 || d.dil_t != 1 || p->T_o < 2) return;
    if (p->tiles_n != 1 || p->n_sub != 1 || 2 * p->BN > 256) return;
    const size_t budget = kSmemBudget / 2;  // two CTAs per SM
    const int want_s = env_int("CCV3D_STAGES"), want_bk = env_int("CCV3D_HALO_BK");
    // the widest channel block that keeps 4 stages per CTA, else 2
    for (int min_s : {4, 2})
    for (int bk : {64, 32, 16}) {
        if (d.Cin % bk != 0 || (want_bk > 0 && bk != want_bk)) continue;
        int s = want_s >= 2 ? want_s : 8;
        const size_t cap = want_s >= 2 ? kSmemBudget : budget;
        while (s >= 2 && fused_smem_for(bk, p->BN, s, d.kh, d.kw, p->halo_w) > cap) --s;
        if (s < (want_s >= 2 ? 2 : min_s)) continue;
        p->fused = 1;
        p->BK = bk;
        p->stages = s;
        p->smem_bytes = fused_smem_for(bk, p->BN, s, d.kh, d.kw, p->halo_w);
        p->tmem_cols = 32;
        while (p->tmem_cols < 2 * p->BN) p->tmem_cols *= 2;
        return;
    }
}

size_t fused_persist_smem_for(int bk, int bn, int stages, int kh, int kw, int halo_w) {
    switch (bk) {
        case 64: return tc2fp_smem_bytes<64>(bn, stages, kh, kw, halo_w);
        case 32: return tc2fp_smem_bytes<32>(bn, stages, kh, kw, halo_w);
        default: return tc2fp_smem_bytes<16>(bn, stages, kh, kw, halo_w);
    }
}

// The persistent form of the two-frame kernel (conv_tc2fp.cuh): one CTA pair
// per SM pair walks the tiles with a continuous ring and double-buffered TMEM
// accumulators.  Sized for one CTA per SM: the widest channel block that
// keeps at least four stages.  Opt-in (CCV3D_FUSED_PERSIST=1) until measured.
void setup_fused_persistent(const ccv3d_desc& d, ccv3d_plan_s* p) {
    p->fused_persist = 0;
    const int mode = env_int("CCV3D_FUSED_PERSIST");  // 1: one CTA per SM, 2: two
    if (!p->fused || p->persist || mode <= 0) return;
    const int want_s = env_int("CCV3D_STAGES");
    const size_t budget = mode == 2 ? kSmemBudget / 2 : kSmemBudget;
    for (int min_s : {4, 3, 2})
        for (int bk : {64, 32, 16}) {
            if (d.Cin % bk != 0) continue;
            int s = want_s >= 2 ? want_s : 12;
            while (s >= 2 && fused_persist_smem_for(bk, p->BN, s, d.kh, d.kw, p->halo_w) > budget)
                --s;
            if (s < min_s) continue;
            p->fused_persist = 1;
            p->BK = bk;
            p->stages = s;
            p->smem_bytes = fused_persist_smem_for(bk, p->BN, s, d.kh, d.kw, p->halo_w);
            p->n_acc = mode == 2 ? 1 : 2;
            p->tmem_cols = 32;
            while (p->tmem_cols < 2 * p->n_acc * p->BN) p->tmem_cols *= 2;  // buffers of two frames
            return;
        }
}

// Whether the persistent stream-K kernel should replace one launch of pair
// tiles (the plan as sized for that launch).  Measured over the decoder
// signatures on B200, stream-K is 5-30% faster where
//   * the launch runs at least two waves of pair tiles (one per SM pair) and
//     its last wave is ragged (waves / ceil(waves) < 0.9), e.g. 180x320
//     outputs, stride-2 and 3x1x1 calls; or
//   * the halo kernel would run a call of Cout >= 192 (360x640 calls);
// and slower where the tiles make less than two waves (the fix-up of split
// tiles is not amortised), where the waves are nearly even, and on the thin
// 720x1280 calls the halo kernel suits.  CCV3D_PERSIST=0/1 overrides.
bool prefer_persistent(const ccv3d_desc& d, const ccv3d_plan_s& p) {
    if (!p.pair) return false;
    if (p.halo) return d.Cout >= 192;
    const long long tiles =
        (long long)d.N * p.T_o * ((p.tiles_x * p.tiles_y + 1) / 2) * p.tiles_n;
    const double waves = (double)tiles / (kSmCount / 2);
    return waves >= 2.0 && waves / std::ceil(waves) < 0.9;
}

size_t thin_smem_for(int bk, int n, int stages, int kw, int cout) {
    switch (bk) {
        case 64: return tcn_smem_bytes<64>(n, stages, kw, cout);
        case 32: return tcn_smem_bytes<32>(n, stages, kw, cout);
        default: return tcn_smem_bytes<16>(n, stages, kw, cout);
    }
}

// Thin outputs (conv_tcn.cuh): Cout too narrow for an MMA's N (not a multiple
// of 16, e.g. the RGB output conv 96 -> 3).  The kernel stacks the temporal
// and column taps along N (kt blocks of kw*Cout rounded up to 16 columns) and
// needs unit temporal stride and dilation and unit W stride.  A tile covers
// one output row, 128 - (kw-1)*d_w output pixels and a group of G output
// frames whose accumulators take (G + kt - 2) blocks + N TMEM columns; G is
// as large as 256 columns allow (two CTAs per SM), in equal groups.  Stages
// aim at three CTAs per SM so that one CTA's epilogue overlaps the others'
// MMAs.  CCV3D_THIN=0 disables the kernel; CCV3D_THIN=1 also takes it for
// Cout that are multiples of 16 (tests).
bool setup_thin(const ccv3d_desc& d, ccv3d_plan_s* p) {
    p->thin = 0;
    const char* te = override_env("CCV3D_THIN");
    if (te != nullptr && std::atoi(te) == 0) return false;
    if (d.dtype != CCV3D_BF16 || d.Cin % 16 != 0 || force_simt()) return false;
    if (d.stride_t != 1 || d.dil_t != 1 || d.stride_w != 1) return false;
    const int cbk = ((d.kw * d.Cout + 15) / 16) * 16;
    const int nb = d.kt * cbk;
    if (nb > 256) return false;
    const int mo = kTileM - (d.kw - 1) * d.dil_w;
    if (mo < 64) return false;
    const int gmax = (256 - nb) / cbk - d.kt + 2;
    if (gmax < 1) return false;
    const int groups = ceil_div(p->T_o, gmax);
    const int G = ceil_div(p->T_o, groups);
    const int bk = widest_bk(d.Cin);
    const int want_s = env_int("CCV3D_STAGES");
    int s = want_s >= 2 ? want_s : 8;
    const size_t cap = want_s >= 2 ? kSmemBudget : kSmemBudget / 3;
    while (s >= 2 && thin_smem_for(bk, nb, s, d.kw, d.Cout) > cap) --s;
    if (s < 2) return false;
    p->thin = 1;
    p->path_tc = 1;
    p->pair = p->persist = p->halo = p->fused = p->fused_persist = 0;
    p->BK = bk;
    p->BN = nb;
    p->n_sub = 1;
    p->stages = s;
    p->smem_bytes = thin_smem_for(bk, nb, s, d.kw, d.Cout);
    p->box_w = mo;
    p->box_h = 1;
    p->halo_w = kTileM;
    p->tiles_x = ceil_div(p->W_o, mo);
    p->tiles_y = p->H_o;
    p->tiles_n = 1;
    p->tn_G = G;
    p->tn_groups = groups;
    p->tn_cbk = cbk;
    const int cols = cbk * (G + d.kt - 2) + nb;
    p->tmem_cols = 32;
    while (p->tmem_cols < cols) p->tmem_cols *= 2;
    // no more CTAs per SM than their TMEM columns fit (a further CTA's
    // allocation would wait for one of them to finish): request enough
    // shared memory to keep the (512 / tmem_cols + 1)-th CTA off the SM
    const size_t per_sm = 228 * 1024;
    const size_t floor_bytes = per_sm / (size_t)(512 / p->tmem_cols + 1) + 1024;
    if (p->smem_bytes < floor_bytes) p->smem_bytes = floor_bytes;
    return true;
}

// Kernel choice and tiling.
void choose_path(const ccv3d_desc& d, ccv3d_plan_s* p) {
    p->path_tc = 0;
    p->thin = 0;
    const bool tc_ok = d.dtype == CCV3D_BF16 && d.Cin % 16 == 0 && d.Cout % 16 == 0 &&
                       d.stride_h <= 2 && d.stride_w <= 2 && !force_simt();
    if (!tc_ok || env_int("CCV3D_THIN") > 0) {
        setup_thin(d, p);
        return;
    }
    // spatial box of 128 output pixels: fewest tiles, then widest rows
    int best_w = 0, best_tiles = 0;
    const int want_w = env_int("CCV3D_BOX_W");
    for (int bw = 128; bw >= 8; bw /= 2) {
        const int bh = kTileM / bw;
        if (bw * d.stride_w > 256 || bh * d.stride_h > 256) continue;
        if (want_w > 0 && bw != want_w) continue;
        const int tiles = ceil_div(p->H_o, bh) * ceil_div(p->W_o, bw);
        if (best_w == 0 || tiles < best_tiles) {
            best_w = bw;
            best_tiles = tiles;
        }
    }
    if (best_w == 0) return;
    p->box_w = best_w;
    p->box_h = kTileM / best_w;
    p->tiles_x = ceil_div(p->W_o, p->box_w);
    p->tiles_y = ceil_div(p->H_o, p->box_h);
    // Cout tile: up to 256 columns per MMA, up to 2 MMAs (512 TMEM columns).
    // One CTA covers up to 384 output channels so that each A box is loaded
    // once for all of them (measured best on the 384-channel decoder calls).
    // Wider outputs that split into 256-column tiles (768 = 3 x 256) take
    // those instead, on the persistent kernel (below): one N = 256 MMA per
    // k-step and double-buffered accumulators, 136 against 148 us on the
    // 3x1x1 384 -> 768 call at 180x320.
    const int want_n = env_int("CCV3D_TILE_N");
    const bool wide256 = want_n == 0 && d.Cout > 384 && d.Cout % 256 == 0;
    const int max_n = (want_n >= 16 && want_n <= 512) ? want_n : (wide256 ? 256 : 384);
    p->tiles_n = ceil_div(d.Cout, max_n);
    p->BN = ((ceil_div(d.Cout, p->tiles_n) + 15) / 16) * 16;
    p->n_sub = p->BN > 256 ? 2 : 1;
    if (p->n_sub == 2 && p->BN % 32 != 0) p->BN = ((p->BN + 31) / 32) * 32;
    p->BK = widest_bk(d.Cin);
    // CTA pairs whenever every pair MMA has N >= 32 (16 weight rows per CTA)
    const char* pe = override_env("CCV3D_PAIR");
    p->pair = (p->BN / p->n_sub) >= 32 ? 1 : 0;
    if (pe != nullptr) p->pair = std::atoi(pe) != 0 && (p->BN / p->n_sub) >= 32;
    p->path_tc_candidate = 1;
    p->persist = 0;
    size_tc(d, p);
    setup_halo(d, p);
    setup_fused(d, p);
    const char* ps = override_env("CCV3D_PERSIST");
    const bool persist = ps != nullptr ? std::atoi(ps) > 0 : (wide256 || prefer_persistent(d, *p));
    if (persist && setup_persistent(d, p)) size_tc(d, p);
    setup_fused_persistent(d, p);
    p->path_tc = 1;
}

// Persistent grid size: one CTA pair per resident pair slot, but at least 32
// k-blocks per pair.  CCV3D_SK_PAIRS forces a size (tests of split tiles).
// Threads of the persistent two-frame kernel: with two CTAs per SM (one
// accumulator buffer each) it runs without the copy warps, so that two CTAs'
// registers fit on an SM.
int fused_persist_threads(const ccv3d_plan_s* p) { return p->n_acc == 1 ? 192 : kTcpThreads; }

void size_persistent(ccv3d_plan_s* p, bool have_device) {
    if (p->fused_persist) {
        // one CTA pair per resident pair slot, at most one per tile; no scratch
        int pairs = 74;
        if (have_device) {
            int n = 0;
            const int th = fused_persist_threads(p);
            switch (p->BK) {
                case 64: n = resident_pairs<64>(p->smem_bytes, true, th); break;
                case 32: n = resident_pairs<32>(p->smem_bytes, true, th); break;
                default: n = resident_pairs<16>(p->smem_bytes, true, th); break;
            }
            if (n > 0) pairs = n;
        }
        const long long tiles =
            (long long)p->d.N * ((p->T_o + 1) / 2) * ((p->tiles_x * p->tiles_y + 1) / 2);
        p->G = (int)std::max<long long>(1, std::min<long long>(pairs, tiles));
        return;
    }
    if (!p->persist) return;
    int pairs = 74;
    if (have_device) {
        int n = 0;
        switch (p->BK) {
            case 64: n = resident_pairs<64>(p->smem_bytes); break;
            case 32: n = resident_pairs<32>(p->smem_bytes); break;
            default: n = resident_pairs<16>(p->smem_bytes); break;
        }
        if (n > 0) pairs = n;
    }
    long long G = std::min<long long>(pairs, std::max<long long>(1, p->sk_total / 32));
    const int want = env_int("CCV3D_SK_PAIRS");
    if (want > 0) G = std::min<long long>(want, pairs);
    p->G = (int)std::max<long long>(1, std::min<long long>(G, p->sk_total));
    const size_t flags = ((size_t)2 * p->G * sizeof(unsigned) + 255) / 256 * 256;
    p->scratch_bytes = flags + (size_t)2 * p->G * kTileM * p->BN * sizeof(float);
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
    if (a == nullptr || b == nullptr || an == 0 || bn == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bn && b0 < a0 + an;
}

size_t elt(const ccv3d_desc& d) { return d.dtype == CCV3D_BF16 ? 2 : 4; }

ccv3d_status encode_act(CUtensorMap* m, const void* base, int frames, const ccv3d_desc& d,
                        const ccv3d_plan_s* p) {
    const cuuint64_t dims[4] = {(cuuint64_t)d.Cin, (cuuint64_t)d.W, (cuuint64_t)d.H,
                                (cuuint64_t)frames};
    const cuuint64_t strides[3] = {(cuuint64_t)d.Cin * 2, (cuuint64_t)d.W * d.Cin * 2,
                                   (cuuint64_t)d.H * d.W * d.Cin * 2};
    // halo and thin kernels: one input row strip of halo_w pixels; otherwise the
    // shifted, strided box of box_h x box_w output pixels
    const bool strip = p->halo || p->thin;
    const cuuint32_t box[4] = {(cuuint32_t)p->BK,
                               (cuuint32_t)(strip ? p->halo_w : p->box_w * d.stride_w),
                               (cuuint32_t)(strip ? 1 : p->box_h * d.stride_h), 1};
    const cuuint32_t estr[4] = {1, strip ? 1u : (cuuint32_t)d.stride_w,
                                strip ? 1u : (cuuint32_t)d.stride_h, 1};
    const CUtensorMapSwizzle sw = p->BK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : p->BK == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base),
                             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CCV3D_OK : CCV3D_ERR_CUDA;
}

ccv3d_status encode_w(CUtensorMap* m, const void* base, const ccv3d_desc& d,
                      const ccv3d_plan_s* p) {
    const int taps = d.kt * d.kh * d.kw;
    const cuuint64_t dims[3] = {(cuuint64_t)d.Cin, (cuuint64_t)taps, (cuuint64_t)d.Cout};
    const cuuint64_t strides[2] = {(cuuint64_t)d.Cin * 2, (cuuint64_t)taps * d.Cin * 2};
    // rows per load: one MMA's N, or half of it when a CTA pair splits the MMA
    const int rows = (p->BN / p->n_sub) / (p->pair ? 2 : 1);
    const cuuint32_t box[3] = {(cuuint32_t)p->BK, 1, (cuuint32_t)rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = p->BK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : p->BK == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CCV3D_OK : CCV3D_ERR_CUDA;
}

// Weights as [taps, Cout, Cin] (a view of the [Cout, taps, Cin] tensor with
// the two outer strides swapped), box [BK, rows, kw]: one load brings a kernel
// row's kw column taps of `rows` output channels, as kw K-major tiles.
ccv3d_status encode_w_kw(CUtensorMap* m, const void* base, const ccv3d_desc& d,
                         const ccv3d_plan_s* p, int rows) {
    const int taps = d.kt * d.kh * d.kw;
    const cuuint64_t dims[3] = {(cuuint64_t)d.Cin, (cuuint64_t)d.Cout, (cuuint64_t)taps};
    const cuuint64_t strides[2] = {(cuuint64_t)taps * d.Cin * 2, (cuuint64_t)d.Cin * 2};
    const cuuint32_t box[3] = {(cuuint32_t)p->BK, (cuuint32_t)rows, (cuuint32_t)d.kw};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = p->BK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : p->BK == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CCV3D_OK : CCV3D_ERR_CUDA;
}

// Thin-output kernel: weights as the 5-D tensor [kt, kh, kw, Cout, Cin]
// (dims Cin, Cout, kw, kh, kt; a view of [Cout, kt, kh, kw, Cin]), box
// [BK, Cout, kw, 1, 1]: one load brings temporal tap k's kw x Cout rows of
// kernel row r, row s*Cout + co, as one K-major tile.
ccv3d_status encode_w_thin(CUtensorMap* m, const void* base, const ccv3d_desc& d,
                           const ccv3d_plan_s* p) {
    const cuuint64_t e = 2;
    const cuuint64_t dims[5] = {(cuuint64_t)d.Cin, (cuuint64_t)d.Cout, (cuuint64_t)d.kw,
                                (cuuint64_t)d.kh, (cuuint64_t)d.kt};
    const cuuint64_t strides[4] = {(cuuint64_t)d.kt * d.kh * d.kw * d.Cin * e,
                                   (cuuint64_t)d.Cin * e, (cuuint64_t)d.kw * d.Cin * e,
                                   (cuuint64_t)d.kh * d.kw * d.Cin * e};
    const cuuint32_t box[5] = {(cuuint32_t)p->BK, (cuuint32_t)d.Cout, (cuuint32_t)d.kw, 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUtensorMapSwizzle sw = p->BK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : p->BK == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base),
                             dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CCV3D_OK : CCV3D_ERR_CUDA;
}

// Output as a 4-D tensor [N*T_o, H_o, W_o, Cout] for the epilogue's tensor
// stores: boxes of (16/32/64 channels) x box_w x box_h pixels of one frame,
// swizzled like the staging buffer; rows and channels past the tensor are
// clipped by the hardware.
// per_warp: the box of one warp's 32 pixels of a box (the pair kernel's
// per-warp epilogue), [kCh, min(32, box_w), max(1, 32 / box_w), 1].
ccv3d_status encode_out(CUtensorMap* m, void* base, const ccv3d_desc& d, const ccv3d_plan_s* p,
                        bool per_warp = false) {
    const int kch = out_block_channels(p->BN);
    const cuuint64_t dims[4] = {(cuuint64_t)d.Cout, (cuuint64_t)p->W_o, (cuuint64_t)p->H_o,
                                (cuuint64_t)d.N * p->T_o};
    const cuuint64_t strides[3] = {(cuuint64_t)d.Cout * 2, (cuuint64_t)p->W_o * d.Cout * 2,
                                   (cuuint64_t)p->H_o * p->W_o * d.Cout * 2};
    const int bw = per_warp ? std::min(32, p->box_w) : p->box_w;
    const int bh = per_warp ? std::max(1, 32 / p->box_w) : p->box_h;
    const cuuint32_t box[4] = {(cuuint32_t)kch, (cuuint32_t)bw, (cuuint32_t)bh, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw = kch == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : kch == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box,
                             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? CCV3D_OK : CCV3D_ERR_CUDA;
}

// Where one call reads its cached frames and writes the frames it keeps.
struct CacheIO {
    const void* cache;            // [N, cache_slots, H, W, Cin]
    int cache_slots, cache_head;  // cache frame t at slot (cache_head + t) mod cache_slots
    void* dst;                    // [N, dst_slots, H, W, Cin]
    int dst_slots, dst_head;      // kept frame j at slot (dst_head + j) mod dst_slots
    int copy_frames;              // frames written per batch entry: the last ones of Z
};

// ccv3d_forward: a dense cache in, a dense new_cache of K' frames out.
CacheIO dense_io(const ccv3d_plan_s* p, const void* cache, void* nc) {
    CacheIO io;
    io.cache = cache;
    io.cache_slots = p->d.cache_len;
    io.cache_head = 0;
    io.dst = nc;
    io.dst_slots = p->keep;
    io.dst_head = 0;
    io.copy_frames = nc != nullptr ? p->keep : 0;
    return io;
}

// Frames of x a ring-buffer call writes: those of the new cache that arrive
// with this call (the others are already in the ring).
int ring_writes(const ccv3d_plan_s* p) { return std::min(p->keep, p->d.T_x); }

CopyJob make_copy(const ccv3d_plan_s* p, const void* x, const CacheIO& io) {
    CopyJob c;
    c.x = static_cast<const uint8_t*>(x);
    c.cache = static_cast<const uint8_t*>(io.cache);
    c.dst = static_cast<uint8_t*>(io.dst);
    c.frame_bytes = (long long)p->d.H * p->d.W * p->d.Cin * (long long)elt(p->d);
    c.keep = io.dst != nullptr ? io.copy_frames : 0;
    c.cache_len = p->d.cache_len;
    c.T_x = p->d.T_x;
    c.z_len = p->z_len;
    c.N = p->d.N;
    c.cache_slots = io.cache_slots;
    c.cache_head = io.cache_head;
    c.dst_slots = io.dst_slots;
    c.dst_head = io.dst_head;
    c.x_bytes = (long long)p->d.N * p->d.T_x * c.frame_bytes;
    c.cache_bytes = io.cache != nullptr ? (long long)p->d.N * io.cache_slots * c.frame_bytes : 0;
    c.dst_bytes = io.dst != nullptr ? (long long)p->d.N * io.dst_slots * c.frame_bytes : 0;
    c.status = p->d_status;
    return c;
}

Taps make_taps(const ccv3d_plan_s* p) {
    Taps t;
    t.kt = p->d.kt;
    t.s_t = p->d.stride_t;
    for (int k = 0; k < kMaxTaps; ++k) {
        t.delta[k] = p->delta[k];
        t.o_l[k] = p->o_l[k];
        t.o_h[k] = p->o_h[k];
    }
    return t;
}

// Paced new_cache copy of the persistent kernel: for each frame the call
// keeps, the output frame and tap that read it (the last such tap) and that
// tap's first k-block in the frame's tiles.  Frames no tap reads stay with
// the sliced copy.  On by default for one output frame with a cache
// (measured on B200: the stride-2 360x640 call 160.6 -> 156.9 us, with
// |C| = 1 126.1 -> 119.6 us, with a ring cache 152.5 -> 146.6 us, the 3x1x1
// 384 -> 768 call 133.9 -> 131.9 us), off otherwise: with no cache
// (67.9 -> 71.9 us) and on the two-frame encoder calls (3x1x1 s_t = 2:
// 146.5 -> 180.6 us) the paced copy of the last tiles lengthens the kernel's
// tail, while the sliced copy starts at once and overlaps the whole GEMM.
// CCV3D_PACED=0/1 overrides.
bool paced_copy_on(const ccv3d_plan_s* p) {
    if (override_env("CCV3D_PACED") != nullptr) return env_int("CCV3D_PACED") > 0;
    return p->d.N * p->T_o == 1 && p->d.cache_len >= 1;
}

void plan_paced_copy(const ccv3d_plan_s* p, TcParams& prm) {
    prm.copy.paced_mask = 0u;
    const int keep = prm.copy.keep;
    if (!p->persist || keep <= 0 || keep > kMaxPaced || !paced_copy_on(p)) return;
    const ccv3d_desc& d = p->d;
    const int per_tap = d.kh * d.kw * ceil_div(d.Cin, p->BK);
    for (int j = 0; j < keep; ++j) {
        const int t = p->z_len - keep + j;
        for (int k = d.kt - 1; k >= 0; --k) {
            const int rel = t - p->delta[k];
            if (rel < 0 || rel % d.stride_t != 0) continue;
            const int o = rel / d.stride_t;
            if (o < p->o_l[k] || o >= p->o_h[k]) continue;
            int ti = 0;  // position of tap k among frame o's active taps
            for (int k2 = 0; k2 < k; ++k2) ti += (o >= p->o_l[k2] && o < p->o_h[k2]) ? 1 : 0;
            prm.paced.o[j] = o;
            prm.paced.kb[j] = ti * per_tap;
            prm.copy.paced_mask |= 1u << j;
            break;
        }
    }
}

// Paced new_cache copy of the persistent two-frame kernel: kept frame j is
// copied box by box when the producer starts the tile of the output-frame
// pair that reads it (all of a tile's stages run within one tile's time).
void plan_paced_copy_fused(const ccv3d_plan_s* p, TcParams& prm) {
    prm.copy.paced_mask = 0u;
    const int keep = prm.copy.keep;
    // (the two-CTA-per-SM form has no copy warps: it takes the sliced copy)
    if (keep <= 0 || keep > kMaxPaced || !paced_copy_on(p) || p->n_acc == 1) return;
    const ccv3d_desc& d = p->d;
    for (int j = 0; j < keep; ++j) {
        const int t = p->z_len - keep + j;
        for (int k = d.kt - 1; k >= 0; --k) {
            const int o = t - p->delta[k];  // unit temporal stride and dilation here
            if (o < p->o_l[k] || o >= p->o_h[k]) continue;
            prm.paced.o[j] = o / 2;  // the output-frame pair holding o
            prm.paced.kb[j] = 0;
            prm.copy.paced_mask |= 1u << j;
            break;
        }
    }
}

template <int BK>
cudaError_t launch_tc(const TcParams& prm, int kind, int grid, size_t smem, cudaStream_t s,
                      int threads) {
    set_smem_attrs<BK>();
    if (kind == 6)
        conv_tcn_kernel<BK><<<grid, kTcThreads, smem, s>>>(prm);
    else if (kind == 5)
        conv_tc2fp_kernel<BK><<<grid, threads, smem, s>>>(prm);
    else if (kind == 4)
        conv_tc2f_kernel<BK><<<grid, kTcThreads, smem, s>>>(prm);
    else if (kind == 3)
        conv_tc2h_kernel<BK><<<grid, kTcThreads, smem, s>>>(prm);
    else if (kind == 2)
        conv_tcp_kernel<BK><<<grid, kTcpThreads, smem, s>>>(prm);
    else if (kind == 1)
        conv_tc2_kernel<BK><<<grid, kTcThreads, smem, s>>>(prm);
    else
        conv_tc_kernel<BK><<<grid, kTcThreads, smem, s>>>(prm);
    return cudaGetLastError();
}

ccv3d_status run_tc(ccv3d_plan_s* p, const void* x, const CacheIO& io, const void* w,
                    const void* bias, void* out, cudaStream_t stream) {
    if (encode_fn() == nullptr) return CCV3D_ERR_CUDA;
    const ccv3d_desc& d = p->d;
    TcParams prm;
    std::memset(&prm, 0, sizeof(prm));
    ccv3d_status st = encode_act(&prm.tmap_x, x, d.N * d.T_x, d, p);
    if (st == CCV3D_OK && d.cache_len > 0)
        st = encode_act(&prm.tmap_c, io.cache, d.N * io.cache_slots, d, p);
    if (st == CCV3D_OK) st = p->thin ? encode_w_thin(&prm.tmap_w, w, d, p) : encode_w(&prm.tmap_w, w, d, p);
    // two-frame kernel: all kw column taps of a stage in one load (test-gated
    // A/B switch CCV3D_W_KW=0 keeps one load per column tap)
    if (st == CCV3D_OK && p->fused && !p->fused_persist && d.kw <= 8 &&
        !(override_env("CCV3D_W_KW") != nullptr && env_int("CCV3D_W_KW") == 0)) {
        st = encode_w_kw(&prm.tmap_wkw_full, w, d, p, p->BN);
        if (st == CCV3D_OK) st = encode_w_kw(&prm.tmap_wkw_half, w, d, p, p->BN / 2);
        if (st == CCV3D_OK) prm.w_kw_boxes = 1;
    }
    // (the thin kernel stores with plain stores: a row of Cout < 8 channels
    // is no tensor-map stride)
    if (st == CCV3D_OK && !p->thin) st = encode_out(&prm.tmap_out, out, d, p);
    if (st == CCV3D_OK && !p->thin) st = encode_out(&prm.tmap_out_w, out, d, p, true);
    if (st != CCV3D_OK) return st;
    prm.bias = d.has_bias ? static_cast<const uint16_t*>(bias) : nullptr;
    prm.out = static_cast<uint16_t*>(out);
    prm.status = p->d_status;
    prm.copy = make_copy(p, x, io);
    prm.taps = make_taps(p);
    prm.N = d.N; prm.T_o = p->T_o; prm.H_o = p->H_o; prm.W_o = p->W_o;
    prm.Cin = d.Cin; prm.Cout = d.Cout; prm.kh = d.kh; prm.kw = d.kw;
    prm.s_h = d.stride_h; prm.s_w = d.stride_w; prm.p_h = d.pad_h; prm.p_w = d.pad_w;
    prm.d_h = d.dil_h; prm.d_w = d.dil_w;
    prm.cache_len = d.cache_len; prm.T_x = d.T_x;
    prm.cache_slots = io.cache_slots; prm.cache_head = io.cache_head;
    prm.x_frames = d.N * d.T_x;
    prm.c_frames = d.N * io.cache_slots;
    prm.H = d.H;
    prm.W = d.W;
    prm.box_h = p->box_h; prm.box_w = p->box_w;
    prm.tiles_x = p->tiles_x; prm.tiles_y = p->tiles_y; prm.tiles_n = p->tiles_n;
    prm.BN = p->BN; prm.n_sub = p->n_sub; prm.n_cb = ceil_div(d.Cin, p->BK);
    prm.stages = p->stages;
    prm.tmem_cols = p->tmem_cols;
    prm.wait_limit_ns = kWaitLimitNs;
    prm.pairs_per_frame = (p->tiles_x * p->tiles_y + 1) / 2;
    long long grid =
        p->pair ? 2LL * d.N * p->T_o * prm.pairs_per_frame * p->tiles_n
                : (long long)d.N * p->T_o * p->tiles_y * p->tiles_x * p->tiles_n;
    if (p->fused) grid = 2LL * d.N * ((p->T_o + 1) / 2) * prm.pairs_per_frame;  // frame pairs
    if (p->thin) {
        grid = (long long)d.N * p->tn_groups * p->H_o * p->tiles_x;
        prm.tn_G = p->tn_G;
        prm.tn_groups = p->tn_groups;
        prm.tn_cbk = p->tn_cbk;
        prm.tn_rows = d.kw * d.Cout;
    }
    if (p->fused_persist) {
        grid = 2LL * p->G;
        prm.sk.n_acc = p->n_acc;
        plan_paced_copy_fused(p, prm);
    }
    if (p->persist) {
        if (p->scratch == nullptr) return CCV3D_ERR_CUDA;
        grid = 2LL * p->G;
        const int frames = d.N * p->T_o;
        for (int f = 0; f <= frames; ++f) prm.sk.frame_start[f] = p->frame_start[f];
        prm.sk.total = p->sk_total;
        prm.sk.n_frames = frames;
        prm.sk.G = p->G;
        prm.sk.n_acc = p->n_acc;
        const size_t flags = ((size_t)2 * p->G * sizeof(unsigned) + 255) / 256 * 256;
        prm.sk.flags = static_cast<unsigned*>(p->scratch);
        prm.sk.partial = reinterpret_cast<float*>(static_cast<char*>(p->scratch) + flags);
        unsigned e = p->epoch.fetch_add(1) + 1;
        if (e == 0) e = p->epoch.fetch_add(1) + 1;  // 0 marks "never published"
        prm.sk.epoch = e;
        plan_paced_copy(p, prm);
    }
    if (grid > 0x7fffffffLL) return CCV3D_ERR_UNSUPPORTED;
    const int kind = p->thin ? 6 : p->fused_persist ? 5 : (p->fused ? 4 : (p->halo ? 3 : (p->persist ? 2 : p->pair)));
    // spread the K-start offsets over one wave of concurrently running tiles,
    // so that tiles running together read different weight rows -- except on
    // the plain pair kernel, whose tiles all start at k-block 0: measured on
    // B200 2-3 % faster there (the 384-channel 90x160 calls: 104.6 -> 102.7
    // us with |C| = 2, 73.8 -> 71.9 us with |C| = 1), with the first stages'
    // boxes prefetched into L2 during set-up.  CCV3D_NO_ROT=1 / CCV3D_ROT=1
    // override.
    const long long units = p->pair ? grid / 2 : grid;
    const long long wave = p->pair ? kSmCount / 2 : kSmCount;
    const bool rot_off = env_int("CCV3D_NO_ROT") > 0 || (kind == 1 && env_int("CCV3D_ROT") <= 0);
    prm.rot_div = rot_off ? 0x7fffffff : (int)std::max(1LL, std::min(units, wave));
    prm.halo_w = p->halo_w;
    cudaError_t e;
    const int threads = p->fused_persist ? fused_persist_threads(p) : kTcpThreads;
    switch (p->BK) {
        case 64: e = launch_tc<64>(prm, kind, (int)grid, p->smem_bytes, stream, threads); break;
        case 32: e = launch_tc<32>(prm, kind, (int)grid, p->smem_bytes, stream, threads); break;
        default: e = launch_tc<16>(prm, kind, (int)grid, p->smem_bytes, stream, threads); break;
    }
    return e == cudaSuccess ? CCV3D_OK : CCV3D_ERR_CUDA;
}

// SIMT variant: one warp per (pixel, 4-channel group) when one thread per
// unit would leave the SMs under 128 threads each (the calls are latency
// bound, so parallelism over the reduction wins); otherwise one thread.
bool simt_uses_warps(const ccv3d_plan_s& p) {
    const long long units =
        (long long)p.d.N * p.T_o * p.H_o * p.W_o * ceil_div(p.d.Cout, kSimtCoT);
    return units < (long long)kSmCount * kSimtThreads;
}

constexpr size_t kSimtSmemMax = 96 * 1024;

// Small calls whose weights and a band of input rows fit in shared memory run
// the shared-memory kernel; its band height aims at ~256 units per block.
void choose_simt(ccv3d_plan_s* p) {
    const ccv3d_desc& d = p->d;
    p->simt_kind = simt_uses_warps(*p) ? 1 : 0;
    // large calls with <= 4 output channels: the tiled kernel (two blocks per SM)
    const bool tile_off = override_env("CCV3D_SIMT_TILE") != nullptr && env_int("CCV3D_SIMT_TILE") == 0;
    if (p->simt_kind == 0 && !tile_off && d.Cout <= 4 && d.Cin % kTileCc == 0 &&
        d.stride_h == 1 && d.stride_w == 1 && d.dil_w == 1 && (d.kw == 1 || d.kw == 3) &&
        simt_tile_patch_loads(d.kh, d.kw, d.dil_h, d.dil_w, (int)elt(d)) <= kTilePf * 256) {
        const size_t bytes =
            4 * (size_t)simt_tile_smem_floats(d.kt, d.kh, d.kw, d.Cin, d.dil_h, d.dil_w);
        if (bytes <= 113 * 1024) {
            p->simt_kind = 3;
            p->simt_smem = bytes;
            p->simt_threads = 256;
            return;
        }
    }
    // the shared-memory block kernel is opt-in (CCV3D_SIMT_SMEM=1): on the
    // 16-channel fp32 contract call it measured 28.7 us against 18.5 us for
    // one warp per unit (12 blocks cannot hide their staging latency)
    const bool smem_on = env_int("CCV3D_SIMT_SMEM") > 0;
    // one warp per pixel for all (<= 16) output channels when Cin divides 32
    // and the weights fit in shared memory (CCV3D_SIMT_W16=0 disables)
    const bool w16_off = override_env("CCV3D_SIMT_W16") != nullptr && env_int("CCV3D_SIMT_W16") == 0;
    if (p->simt_kind == 1 && !smem_on && !w16_off && 32 % d.Cin == 0 && d.Cout <= 16) {
        const size_t bytes = simt_warp16_smem_bytes(d.kt * d.kh * d.kw, d.Cin);
        if (bytes <= kSimtSmemMax) {
            p->simt_kind = 4;
            p->simt_smem = bytes;
            p->simt_threads = kW16Threads;
            return;
        }
    }
    if (p->simt_kind != 1 || !smem_on) return;
    const int Wp = d.W + 2 * d.pad_w;
    const long long row_units = (long long)p->W_o * ceil_div(d.Cout, kSimtCoT);
    int bh = (int)std::max<long long>(1, std::min<long long>(p->H_o, 256 / std::max(1LL, row_units)));
    if (env_int("CCV3D_SIMT_BAND") > 0) bh = std::min(p->H_o, env_int("CCV3D_SIMT_BAND"));
    for (; bh >= 1; --bh) {
        const int rows_in = (bh - 1) * d.stride_h + (d.kh - 1) * d.dil_h + 1;
        const size_t bytes =
            4 * (size_t)simt_smem_floats(d.kt, d.kh, d.kw, d.Cin, d.Cout, rows_in, Wp);
        if (bytes <= kSimtSmemMax) {
            p->simt_kind = 2;
            p->simt_band_h = bh;
            p->simt_rows_in = rows_in;
            p->simt_smem = bytes;
            const long long u = bh * row_units;
            p->simt_threads = (int)std::min<long long>(256, std::max<long long>(32, (u + 31) / 32 * 32));
            return;
        }
    }
}

template <typename T>
void set_simt_smem_attr() {
    static std::atomic<bool> done[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    if (dev < 0 || dev >= kMaxDevices || done[dev].load(std::memory_order_acquire)) return;
    cudaFuncSetAttribute(conv_simt_smem_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kSimtSmemMax);
    cudaFuncSetAttribute(conv_simt_warp16_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kSimtSmemMax);
    cudaFuncSetAttribute(conv_simt_tile_kernel<T, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         113 * 1024);
    cudaFuncSetAttribute(conv_simt_tile_kernel<T, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         113 * 1024);
    cudaGetLastError();
    done[dev].store(true, std::memory_order_release);
}

template <typename T>
void launch_simt_tile(const SimtParams& prm, int kw, int grid, size_t smem, cudaStream_t s) {
    set_simt_smem_attr<T>();
    if (kw == 3)
        conv_simt_tile_kernel<T, 3><<<grid, 256, smem, s>>>(prm);
    else
        conv_simt_tile_kernel<T, 1><<<grid, 256, smem, s>>>(prm);
}

ccv3d_status run_simt(ccv3d_plan_s* p, const void* x, const CacheIO& io, const void* w,
                      const void* bias, void* out, cudaStream_t stream) {
    const ccv3d_desc& d = p->d;
    SimtParams prm;
    std::memset(&prm, 0, sizeof(prm));
    prm.x = x; prm.cache = io.cache; prm.w = w;
    prm.bias = d.has_bias ? bias : nullptr;
    prm.out = out;
    prm.copy = make_copy(p, x, io);
    prm.cache_slots = io.cache_slots; prm.cache_head = io.cache_head;
    prm.status = p->d_status;
    prm.w_floats = (long long)d.Cout * d.kt * d.kh * d.kw * d.Cin;
    prm.out_elems = (long long)d.N * p->T_o * p->H_o * p->W_o * d.Cout;
    prm.taps = make_taps(p);
    prm.N = d.N; prm.T_o = p->T_o; prm.H_o = p->H_o; prm.W_o = p->W_o;
    prm.Cin = d.Cin; prm.Cout = d.Cout; prm.H = d.H; prm.W = d.W; prm.kh = d.kh; prm.kw = d.kw;
    prm.s_h = d.stride_h; prm.s_w = d.stride_w; prm.p_h = d.pad_h; prm.p_w = d.pad_w;
    prm.d_h = d.dil_h; prm.d_w = d.dil_w;
    prm.cache_len = d.cache_len; prm.T_x = d.T_x;
    prm.co_groups = ceil_div(d.Cout, kSimtCoT);
    prm.conv_threads = (long long)d.N * p->T_o * p->H_o * p->W_o * prm.co_groups;
    if (p->simt_kind == 3) {
        const long long cb = (long long)d.N * p->T_o * ceil_div(p->H_o, kTileRows) *
                             ceil_div(p->W_o, kTileCols);
        const long long copy_bytes = (long long)prm.copy.keep * d.N * prm.copy.frame_bytes;
        const long long kb =
            copy_bytes > 0 ? std::min<long long>(1184, (copy_bytes + 65535) / 65536) : 0;
        if (cb + kb > 0x7fffffffLL) return CCV3D_ERR_UNSUPPORTED;
        prm.conv_blocks = (int)cb;
        prm.copy_blocks = (int)kb;
        if (d.dtype == CCV3D_FP32)
            launch_simt_tile<float>(prm, d.kw, (int)(cb + kb), p->simt_smem, stream);
        else
            launch_simt_tile<__nv_bfloat16>(prm, d.kw, (int)(cb + kb), p->simt_smem, stream);
        return cudaGetLastError() == cudaSuccess ? CCV3D_OK : CCV3D_ERR_CUDA;
    }
    if (p->simt_kind == 4) {
        prm.co_groups = 1;
        prm.conv_threads = (long long)d.N * p->T_o * p->H_o * p->W_o;  // pixels
        const long long cb = (prm.conv_threads + kW16Pixels - 1) / kW16Pixels;
        const long long copy_bytes = (long long)prm.copy.keep * d.N * prm.copy.frame_bytes;
        // 16 KB per copy block: two 16-byte vectors per thread, one round of loads
        const long long kb =
            copy_bytes > 0 ? std::min<long long>(1184, (copy_bytes + 16383) / 16384) : 0;
        if (cb + kb > 0x7fffffffLL) return CCV3D_ERR_UNSUPPORTED;
        prm.conv_blocks = (int)cb;
        prm.copy_blocks = (int)kb;
        const int grid = (int)(cb + kb);
        if (d.dtype == CCV3D_FP32) {
            set_simt_smem_attr<float>();
            conv_simt_warp16_kernel<float><<<grid, kW16Threads, p->simt_smem, stream>>>(prm);
        } else {
            set_simt_smem_attr<__nv_bfloat16>();
            conv_simt_warp16_kernel<__nv_bfloat16><<<grid, kW16Threads, p->simt_smem, stream>>>(prm);
        }
        return cudaGetLastError() == cudaSuccess ? CCV3D_OK : CCV3D_ERR_CUDA;
    }
    if (p->simt_kind == 2) {
        prm.band_h = p->simt_band_h;
        prm.bands = ceil_div(p->H_o, p->simt_band_h);
        prm.rows_in = p->simt_rows_in;
        prm.Wp = d.W + 2 * d.pad_w;
        const long long cb = (long long)d.N * p->T_o * prm.bands;
        const long long copy_bytes = (long long)prm.copy.keep * d.N * prm.copy.frame_bytes;
        const long long kb =
            copy_bytes > 0 ? std::min<long long>(1184, (copy_bytes + 16383) / 16384) : 0;
        if (cb + kb > 0x7fffffffLL) return CCV3D_ERR_UNSUPPORTED;
        prm.conv_blocks = (int)cb;
        prm.copy_blocks = (int)kb;
        const int grid = (int)(cb + kb);
        if (d.dtype == CCV3D_FP32) {
            set_simt_smem_attr<float>();
            conv_simt_smem_kernel<float><<<grid, p->simt_threads, p->simt_smem, stream>>>(prm);
        } else {
            set_simt_smem_attr<__nv_bfloat16>();
            conv_simt_smem_kernel<__nv_bfloat16><<<grid, p->simt_threads, p->simt_smem, stream>>>(prm);
        }
        return cudaGetLastError() == cudaSuccess ? CCV3D_OK : CCV3D_ERR_CUDA;
    }
    const bool warp = p->simt_kind == 1;
    const long long cb = (prm.conv_threads * (warp ? 32 : 1) + kSimtThreads - 1) / kSimtThreads;
    const long long copy_bytes = (long long)prm.copy.keep * d.N * prm.copy.frame_bytes;
    const long long kb = copy_bytes > 0 ? std::min<long long>(1184, (copy_bytes + 32767) / 32768) : 0;
    if (cb + kb > 0x7fffffffLL) return CCV3D_ERR_UNSUPPORTED;
    prm.conv_blocks = (int)cb;
    prm.copy_blocks = (int)kb;
    const int grid = (int)(cb + kb);
    if (warp && d.dtype == CCV3D_FP32)
        conv_simt_warp_kernel<float><<<grid, kSimtThreads, 0, stream>>>(prm);
    else if (warp)
        conv_simt_warp_kernel<__nv_bfloat16><<<grid, kSimtThreads, 0, stream>>>(prm);
    else if (d.dtype == CCV3D_FP32)
        conv_simt_kernel<float><<<grid, kSimtThreads, 0, stream>>>(prm);
    else
        conv_simt_kernel<__nv_bfloat16><<<grid, kSimtThreads, 0, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? CCV3D_OK : CCV3D_ERR_CUDA;
}

// Argument checks of a forward call against its plan (no device work).
ccv3d_status check_call(const ccv3d_plan_s* p, const void* x, const void* cache, const void* w,
                        const void* bias, const void* out, const void* nc, const int stride[2],
                        const int pad[2], const int dilation[3]) {
    const ccv3d_desc& d = p->d;
    if (stride == nullptr || pad == nullptr || dilation == nullptr) return CCV3D_ERR_INVALID;
    if (stride[0] != d.stride_h || stride[1] != d.stride_w || pad[0] != d.pad_h ||
        pad[1] != d.pad_w || dilation[0] != d.dil_t || dilation[1] != d.dil_h ||
        dilation[2] != d.dil_w)
        return CCV3D_ERR_INVALID;
    if (x == nullptr || w == nullptr || out == nullptr || (d.cache_len > 0 && cache == nullptr) ||
        (d.has_bias && bias == nullptr) || (p->keep > 0 && nc == nullptr))
        return CCV3D_ERR_INVALID;
    if (!aligned16(x) || !aligned16(w) || !aligned16(out) ||
        (d.cache_len > 0 && !aligned16(cache)) || (nc != nullptr && !aligned16(nc)) ||
        (d.has_bias && (reinterpret_cast<uintptr_t>(bias) % elt(d)) != 0))
        return CCV3D_ERR_ALIGNMENT;
    const size_t e = elt(d);
    const size_t frame = (size_t)d.H * d.W * d.Cin * e;
    const size_t x_bytes = (size_t)d.N * d.T_x * frame;
    const size_t c_bytes = d.cache_len > 0 ? (size_t)d.N * d.cache_len * frame : 0;
    const size_t nc_bytes = nc != nullptr ? (size_t)d.N * p->keep * frame : 0;
    const size_t o_bytes = (size_t)d.N * p->T_o * p->H_o * p->W_o * d.Cout * e;
    const size_t w_bytes = (size_t)d.Cout * d.kt * d.kh * d.kw * d.Cin * e;
    if (overlaps(nc, nc_bytes, x, x_bytes) || overlaps(nc, nc_bytes, cache, c_bytes) ||
        overlaps(out, o_bytes, x, x_bytes) || overlaps(out, o_bytes, cache, c_bytes) ||
        overlaps(out, o_bytes, w, w_bytes) || overlaps(out, o_bytes, nc, nc_bytes))
        return CCV3D_ERR_ALIAS;
    return CCV3D_OK;
}

// Read a status word after the work already queued on `stream`, and clear
// it when it holds an error.  Synchronises that stream only; the copy goes to
// pageable host memory, so nothing is allocated.
ccv3d_status read_and_clear_status(int* d_status, cudaStream_t stream) {
    int v = 0;
    if (cudaMemcpyAsync(&v, d_status, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return CCV3D_ERR_CUDA;
    }
    if (v != 0 && (cudaMemsetAsync(d_status, 0, sizeof(int), stream) != cudaSuccess ||
                   cudaStreamSynchronize(stream) != cudaSuccess)) {
        cudaGetLastError();
        return CCV3D_ERR_CUDA;
    }
    return v == 0 ? CCV3D_OK : (ccv3d_status)v;
}

// Argument checks of a ring-buffer call against its plan (no device work).
ccv3d_status check_ring_call(const ccv3d_plan_s* p, const void* x, const void* ring,
                             int ring_slots, int head, const void* w, const void* bias,
                             const void* out, const int stride[2], const int pad[2],
                             const int dilation[3]) {
    const ccv3d_desc& d = p->d;
    if (stride == nullptr || pad == nullptr || dilation == nullptr) return CCV3D_ERR_INVALID;
    if (stride[0] != d.stride_h || stride[1] != d.stride_w || pad[0] != d.pad_h ||
        pad[1] != d.pad_w || dilation[0] != d.dil_t || dilation[1] != d.dil_h ||
        dilation[2] != d.dil_w)
        return CCV3D_ERR_INVALID;
    const int writes = ring_writes(p);
    const bool uses_ring = d.cache_len > 0 || writes > 0;
    // the slots this call writes must not hold a frame it reads
    if (ring_slots < 1 || head < 0 || head >= ring_slots || d.cache_len + writes > ring_slots)
        return CCV3D_ERR_INVALID;
    if (x == nullptr || w == nullptr || out == nullptr || (uses_ring && ring == nullptr) ||
        (d.has_bias && bias == nullptr))
        return CCV3D_ERR_INVALID;
    if (!aligned16(x) || !aligned16(w) || !aligned16(out) || (uses_ring && !aligned16(ring)) ||
        (d.has_bias && (reinterpret_cast<uintptr_t>(bias) % elt(d)) != 0))
        return CCV3D_ERR_ALIGNMENT;
    const size_t e = elt(d);
    const size_t frame = (size_t)d.H * d.W * d.Cin * e;
    const size_t x_bytes = (size_t)d.N * d.T_x * frame;
    const size_t r_bytes = uses_ring ? (size_t)d.N * ring_slots * frame : 0;
    const size_t o_bytes = (size_t)d.N * p->T_o * p->H_o * p->W_o * d.Cout * e;
    const size_t w_bytes = (size_t)d.Cout * d.kt * d.kh * d.kw * d.Cin * e;
    if (overlaps(ring, r_bytes, x, x_bytes) || overlaps(out, o_bytes, ring, r_bytes) ||
        overlaps(out, o_bytes, x, x_bytes) || overlaps(out, o_bytes, w, w_bytes) ||
        overlaps(ring, r_bytes, w, w_bytes))
        return CCV3D_ERR_ALIAS;
    return CCV3D_OK;
}

// One thread hands the range checks a byte range that ends one byte past its
// buffer and an index one past its count; nothing is dereferenced.
__global__ void bounds_selftest_kernel(int* status) {
    const char* base = reinterpret_cast<const char*>(status);
    if (in_bounds(status, base, sizeof(int) + 1, base, sizeof(int))) return;
    index_ok(status, 1, 1);
}

__global__ void wait_selftest_kernel(int* status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
        // Nothing ever arrives on `bar`: the bounded wait must give up.
        if (mbar_wait(smem_u32(&bar), 0, status, limit_ns)) atomicExch(status, -1);
    }
}

}  // namespace

extern "C" {

ccv3d_status ccv3d_plan(ccv3d_plan_t* out, const ccv3d_desc* desc) {
    if (out == nullptr) return CCV3D_ERR_INVALID;
    *out = nullptr;
    if (desc == nullptr) return CCV3D_ERR_INVALID;
    ccv3d_plan_s* p = new (std::nothrow) ccv3d_plan_s();
    if (p == nullptr) return CCV3D_ERR_INVALID;
    p->d = *desc;
    ccv3d_status st = compute_intervals(*desc, p);
    if (st != CCV3D_OK) {
        if (st == CCV3D_ERR_UNSUPPORTED) g_plans_unsupported.fetch_add(1, std::memory_order_relaxed);
        delete p;
        return st;
    }
    choose_path(*desc, p);
    if (!p->path_tc) choose_simt(p);
    // The status block lives on the current device.  Without any CUDA device
    // the plan still serves inspection (intervals, sizes, path) and
    // ccv3d_forward refuses with CCV3D_ERR_CUDA.
    p->device = -1;
    p->d_status = nullptr;
    p->scratch = nullptr;
    p->scratch_bytes = 0;
    int ndev = 0;
    const bool have_device = cudaGetDeviceCount(&ndev) == cudaSuccess && ndev > 0;
    if (!have_device) cudaGetLastError();
    size_persistent(p, have_device);
    if (have_device) {
        bool ok = cudaGetDevice(&p->device) == cudaSuccess &&
                  cudaMalloc(&p->d_status, 256) == cudaSuccess &&
                  cudaMemset(p->d_status, 0, 256) == cudaSuccess;
        if (ok && p->scratch_bytes > 0) {
            // split-tile flags start at 0 ("never published"); launches tag
            // theirs with a per-plan epoch, so no clearing between calls
            ok = cudaMalloc(&p->scratch, p->scratch_bytes) == cudaSuccess &&
                 cudaMemset(p->scratch, 0, p->scratch_bytes) == cudaSuccess;
        }
        if (!ok) {
            cudaGetLastError();
            if (p->d_status) cudaFree(p->d_status);
            if (p->scratch) cudaFree(p->scratch);
            delete p;
            return CCV3D_ERR_CUDA;
        }
    }
    *out = p;
    return CCV3D_OK;
}

ccv3d_status ccv3d_plan_intervals(ccv3d_plan_t p, int* T_o, int* H_o, int* W_o,
                                  int delta[CCV3D_MAX_KT], int o_l[CCV3D_MAX_KT],
                                  int o_h[CCV3D_MAX_KT]) {
    if (p == nullptr) return CCV3D_ERR_INVALID;
    if (T_o) *T_o = p->T_o;
    if (H_o) *H_o = p->H_o;
    if (W_o) *W_o = p->W_o;
    for (int k = 0; k < CCV3D_MAX_KT; ++k) {
        if (delta) delta[k] = p->delta[k];
        if (o_l) o_l[k] = p->o_l[k];
        if (o_h) o_h[k] = p->o_h[k];
    }
    return CCV3D_OK;
}

int ccv3d_plan_path(ccv3d_plan_t p, int* tile_m, int* tile_n) {
    if (p == nullptr) return -1;
    if (tile_m) *tile_m = p->path_tc ? kTileM * (p->pair ? 2 : 1) : 0;
    if (tile_n) *tile_n = p->path_tc ? p->BN : 0;
    return p->path_tc;
}

const char* ccv3d_plan_kernel(ccv3d_plan_t p) {
    if (p == nullptr) return "";
    if (!p->path_tc)
        return p->simt_kind == 4 ? "simt_warp16"
               : p->simt_kind == 3 ? "simt_tile"
                                 : (p->simt_kind == 2 ? "simt_smem"
                                                      : (p->simt_kind == 1 ? "simt_warp" : "simt"));
    if (p->thin) return "tc_thin";
    if (p->fused_persist) return "tc_pair_fused_persistent";
    if (p->fused) return "tc_pair_fused";
    if (p->halo) return "tc_pair_halo";
    if (p->persist) return "tc_persistent";
    return p->pair ? "tc_pair" : "tc_single";
}

ccv3d_status ccv3d_plan_tiling(ccv3d_plan_t p, int* k_block, int* stages, int* workspace_pairs) {
    if (k_block) *k_block = 0;
    if (stages) *stages = 0;
    if (workspace_pairs) *workspace_pairs = 0;
    if (p == nullptr) return CCV3D_ERR_INVALID;
    if (!p->path_tc) return CCV3D_ERR_UNSUPPORTED;
    if (k_block) *k_block = p->BK;
    if (stages) *stages = p->stages;
    if (workspace_pairs) *workspace_pairs = p->persist ? p->G : 0;
    return CCV3D_OK;
}

ccv3d_status ccv3d_plan_sizes(ccv3d_plan_t p, size_t* out_bytes, size_t* nc_bytes,
                              int* nc_frames) {
    if (p == nullptr) return CCV3D_ERR_INVALID;
    const ccv3d_desc& d = p->d;
    if (out_bytes) *out_bytes = (size_t)d.N * p->T_o * p->H_o * p->W_o * d.Cout * elt(d);
    if (nc_bytes) *nc_bytes = (size_t)d.N * p->keep * d.H * d.W * d.Cin * elt(d);
    if (nc_frames) *nc_frames = p->keep;
    return CCV3D_OK;
}

ccv3d_status ccv3d_forward(ccv3d_plan_t p, const void* x, const void* cache, const void* w,
                           const void* bias, void* out, void* nc, const int stride[2],
                           const int pad[2], const int dilation[3], cudaStream_t stream) {
    if (p == nullptr) return CCV3D_ERR_INVALID;
    auto refuse = [&](ccv3d_status s) {
        (s == CCV3D_ERR_UNSUPPORTED ? p->unsupported : p->errors)
            .fetch_add(1, std::memory_order_relaxed);
        return s;
    };
    const ccv3d_status chk = check_call(p, x, cache, w, bias, out, nc, stride, pad, dilation);
    if (chk != CCV3D_OK) return refuse(chk);
    if (p->d_status == nullptr) return refuse(CCV3D_ERR_CUDA);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) return refuse(CCV3D_ERR_INVALID);
    const CacheIO io = dense_io(p, cache, nc);
    ccv3d_status st = p->path_tc ? run_tc(p, x, io, w, bias, out, stream)
                                 : run_simt(p, x, io, w, bias, out, stream);
    if (st != CCV3D_OK) return refuse(st);
    p->calls.fetch_add(1, std::memory_order_relaxed);
    (p->path_tc ? p->tc : p->simt).fetch_add(1, std::memory_order_relaxed);
    return CCV3D_OK;
}

ccv3d_status ccv3d_forward_ring(ccv3d_plan_t p, const void* x, void* ring, int ring_slots,
                                int head, const void* w, const void* bias, void* out,
                                const int stride[2], const int pad[2], const int dilation[3],
                                cudaStream_t stream, int* next_head) {
    if (p == nullptr) return CCV3D_ERR_INVALID;
    auto refuse = [&](ccv3d_status s) {
        (s == CCV3D_ERR_UNSUPPORTED ? p->unsupported : p->errors)
            .fetch_add(1, std::memory_order_relaxed);
        return s;
    };
    const ccv3d_status chk =
        check_ring_call(p, x, ring, ring_slots, head, w, bias, out, stride, pad, dilation);
    if (chk != CCV3D_OK) return refuse(chk);
    if (p->d_status == nullptr) return refuse(CCV3D_ERR_CUDA);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) return refuse(CCV3D_ERR_INVALID);
    const ccv3d_desc& d = p->d;
    const int writes = ring_writes(p);
    CacheIO io;
    io.cache = ring;
    io.cache_slots = ring_slots;
    io.cache_head = head;
    io.dst = ring;
    io.dst_slots = ring_slots;
    io.dst_head = (head + d.cache_len) % ring_slots;
    io.copy_frames = writes;
    ccv3d_status st = p->path_tc ? run_tc(p, x, io, w, bias, out, stream)
                                 : run_simt(p, x, io, w, bias, out, stream);
    if (st != CCV3D_OK) return refuse(st);
    if (next_head != nullptr)
        *next_head = (int)(((long long)head + d.cache_len + writes - p->keep) % ring_slots +
                           ring_slots) % ring_slots;
    p->calls.fetch_add(1, std::memory_order_relaxed);
    (p->path_tc ? p->tc : p->simt).fetch_add(1, std::memory_order_relaxed);
    return CCV3D_OK;
}

ccv3d_status ccv3d_get_stats(ccv3d_plan_t p, ccv3d_stats* s) {
    if (p == nullptr || s == nullptr) return CCV3D_ERR_INVALID;
    s->calls = p->calls.load();
    s->tc_path = p->tc.load();
    s->simt_path = p->simt.load();
    s->unsupported = p->unsupported.load();
    s->errors = p->errors.load();
    s->workspace_bytes = p->scratch_bytes;
    s->plans_unsupported = g_plans_unsupported.load();
    return CCV3D_OK;
}

ccv3d_status ccv3d_get_status(ccv3d_plan_t p) {
    if (p == nullptr) return CCV3D_ERR_INVALID;
    if (p->d_status == nullptr) return CCV3D_ERR_CUDA;
    int v = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return CCV3D_ERR_CUDA;
    if (cudaMemcpy(&v, p->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return CCV3D_ERR_CUDA;
    if (v != 0 && cudaMemset(p->d_status, 0, sizeof(int)) != cudaSuccess) return CCV3D_ERR_CUDA;
    return v == 0 ? CCV3D_OK : (ccv3d_status)v;
}

ccv3d_status ccv3d_get_status_stream(ccv3d_plan_t p, cudaStream_t stream) {
    if (p == nullptr) return CCV3D_ERR_INVALID;
    if (p->d_status == nullptr) return CCV3D_ERR_CUDA;
    return read_and_clear_status(p->d_status, stream);
}

void ccv3d_destroy(ccv3d_plan_t p) {
    if (p == nullptr) return;
    if (p->d_status) cudaFree(p->d_status);
    if (p->scratch) cudaFree(p->scratch);
    delete p;
}

const char* ccv3d_strerror(ccv3d_status s) {
    switch (s) {
        case CCV3D_OK: return "ok";
        case CCV3D_ERR_INVALID: return "invalid argument";
        case CCV3D_ERR_UNSUPPORTED: return "unsupported call (outside the cached causal Conv3D contract)";
        case CCV3D_ERR_EMPTY_OUTPUT: return "empty output";
        case CCV3D_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case CCV3D_ERR_ALIAS: return "output buffer overlaps an input";
        case CCV3D_ERR_CUDA: return "CUDA error";
        case CCV3D_ERR_TIMEOUT: return "bounded device wait timed out";
        case CCV3D_ERR_SCRATCH_LIMIT:
            return "call needs more device scratch than the no-allocation entry point holds";
        case CCV3D_ERR_BOUNDS:
            return "bounds-checked build: a kernel computed an address outside its buffer";
    }
    return "unknown status";
}

ccv3d_status ccv3d_quantize_u8(const void* in, ccv3d_dtype dtype, void* out, long long n,
                               cudaStream_t stream) {
    if (n < 0 || (dtype != CCV3D_FP32 && dtype != CCV3D_BF16)) return CCV3D_ERR_INVALID;
    if (n == 0) return CCV3D_OK;
    if (in == nullptr || out == nullptr) return CCV3D_ERR_INVALID;
    const uintptr_t a = reinterpret_cast<uintptr_t>(in), b = reinterpret_cast<uintptr_t>(out);
    if ((a | b) & 15u) return CCV3D_ERR_ALIGNMENT;
    const uintptr_t a_end = a + (uintptr_t)n * (dtype == CCV3D_FP32 ? 4u : 2u);
    if (a < b + (uintptr_t)n && b < a_end) return CCV3D_ERR_ALIAS;
    const long long units = n / 16;  // 16 values per thread step
    const int blocks = (int)std::min<long long>(std::max<long long>(1, (units + 255) / 256),
                                                (long long)kSmCount * 8);
    if (dtype == CCV3D_FP32)
        quantize_u8_f32_kernel<<<blocks, 256, 0, stream>>>(static_cast<const float*>(in),
                                                            static_cast<uint8_t*>(out), n);
    else
        quantize_u8_bf16_kernel<<<blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(in),
                                                             static_cast<uint8_t*>(out), n);
    return cudaGetLastError() == cudaSuccess ? CCV3D_OK : CCV3D_ERR_CUDA;
}

ccv3d_status ccv3d_selftest_bounds(cudaStream_t stream) {
    int* d = nullptr;
    if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) return CCV3D_ERR_CUDA;
    int v = -1;
    cudaError_t e = cudaMemsetAsync(d, 0, sizeof(int), stream);
    if (e == cudaSuccess) {
        bounds_selftest_kernel<<<1, 1, 0, stream>>>(d);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(&v, d, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    cudaFree(d);
    if (e != cudaSuccess) return CCV3D_ERR_CUDA;
    return v == kStatusBounds ? CCV3D_ERR_BOUNDS : (v == 0 ? CCV3D_OK : CCV3D_ERR_CUDA);
}

ccv3d_status ccv3d_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream) {
    int* d = nullptr;
    if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) return CCV3D_ERR_CUDA;
    int v = 0;
    cudaError_t e = cudaMemsetAsync(d, 0, sizeof(int), stream);
    if (e == cudaSuccess) {
        wait_selftest_kernel<<<1, 32, 0, stream>>>(d, limit_ns);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpyAsync(&v, d, sizeof(int), cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    cudaFree(d);
    if (e != cudaSuccess) return CCV3D_ERR_CUDA;
    if (v == kStatusTimeout) return CCV3D_ERR_TIMEOUT;
    return v == 0 ? CCV3D_ERR_CUDA : CCV3D_OK;
}


}  // extern "C"

// ---------------------------------------------------------------------------
// ccv3d_forward_noalloc: the persistent stream-K kernel with its scratch in a
// static device array instead of plan-owned memory.  The array's name is a
// host-side stand-in in host code; its device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[CCV3D_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoallocDevices = 64;
constexpr size_t kNoallocStatusBytes = 256;  // status word, padded; then the flags
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoallocDevices];
std::atomic<unsigned> g_noalloc_calls[kNoallocDevices];

ccv3d_status noalloc_scratch(int dev, void** out) {
    if (dev < 0 || dev >= kNoallocDevices) return CCV3D_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
            cudaGetLastError();
            return CCV3D_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
    return CCV3D_OK;
}

}  // namespace

extern "C" ccv3d_status ccv3d_forward_noalloc(const ccv3d_desc* desc, const void* x,
                                              const void* cache, const void* w,
                                              const void* bias, void* out, void* nc,
                                              const int stride[2], const int pad[2],
                                              const int dilation[3], cudaStream_t stream) {
    if (desc == nullptr) return CCV3D_ERR_INVALID;
    ccv3d_plan_s p{};  // host stack only
    p.d = *desc;
    ccv3d_status st = compute_intervals(*desc, &p);
    if (st != CCV3D_OK) return st;
    choose_path(*desc, &p);
    if (!p.path_tc || !setup_persistent(*desc, &p)) return CCV3D_ERR_UNSUPPORTED;
    size_tc(*desc, &p);
    st = check_call(&p, x, cache, w, bias, out, nc, stride, pad, dilation);
    if (st != CCV3D_OK) return st;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return CCV3D_ERR_CUDA;
    }
    size_persistent(&p, true);
    if (kNoallocStatusBytes + p.scratch_bytes > (size_t)CCV3D_NOALLOC_SCRATCH_BYTES)
        return CCV3D_ERR_SCRATCH_LIMIT;
    void* base = nullptr;
    st = noalloc_scratch(dev, &base);
    if (st != CCV3D_OK) return st;
    p.device = dev;
    p.d_status = static_cast<int*>(base);
    p.scratch = static_cast<unsigned char*>(base) + kNoallocStatusBytes;
    // This call's split-tile epoch: the next value of the device's call
    // counter, skipping 0 ("never published"), so no two calls within 2^32
    // share one.  run_tc adds 1 to the plan's counter, hence the e - 1.
    unsigned e;
    do {
        e = g_noalloc_calls[dev].fetch_add(1) + 1u;
    } while (e == 0u);
    p.epoch.store(e - 1u);
    // The status word is not cleared here: it keeps the first timeout any
    // call recorded until ccv3d_noalloc_get_status reads it.
    return run_tc(&p, x, dense_io(&p, cache, nc), w, bias, out, stream);
}

extern "C" ccv3d_status ccv3d_noalloc_get_status(cudaStream_t stream) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return CCV3D_ERR_CUDA;
    }
    void* base = nullptr;
    const ccv3d_status st = noalloc_scratch(dev, &base);
    if (st != CCV3D_OK) return st;
    return read_and_clear_status(static_cast<int*>(base), stream);
}
