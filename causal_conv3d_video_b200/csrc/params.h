// params.h -- kernel parameter blocks shared by the host launcher and the
// kernels of libccv3d.  Passed by value as __grid_constant__ parameters.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace ccv3d {

constexpr int kMaxTaps = 3;
constexpr int kTileM = 128;          // output pixels per GEMM tile (UMMA M)
constexpr int kSmCount = 148;        // B200 SMs (scheduling heuristics only)
constexpr int kTcThreads = 192;      // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded device waits: 2 s

// Frame index, in a cache tensor of `slots` frames per batch entry, of cache
// frame t (0 <= t < slots) of batch entry n, when frame 0 sits at slot `head`
// (0 <= head < slots).  A dense cache has slots = |C| and head = 0; a ring
// buffer wraps around its slots.
__host__ __device__ __forceinline__ int ring_frame(int n, int t, int slots, int head) {
    int s = head + t;
    if (s >= slots) s -= slots;
    return n * slots + s;
}

// The cache write of one call: the last `keep` frames of Z = [cache; x],
// copied frame by frame, Z's frame z_len - keep + j to slot
// (dst_head + j) mod dst_slots of dst.  Dense new_cache: dst_slots = keep,
// dst_head = 0.  Ring buffer: only the arriving frames, into the slots that
// follow the cached ones.
struct CopyJob {
    const uint8_t* x;       // [N, T_x, frame_bytes]
    const uint8_t* cache;   // [N, cache_slots, frame_bytes], frame t at ring_frame(n, t, ...)
    uint8_t* dst;           // [N, dst_slots, frame_bytes]
    long long frame_bytes;
    int keep, cache_len, T_x, z_len, N;
    int cache_slots, cache_head;
    int dst_slots, dst_head;
    long long x_bytes, cache_bytes, dst_bytes;  // buffer extents (checked build)
    int* status;                                // status word (checked build)
    unsigned paced_mask;  // bit j: frame j is copied tile by tile with the GEMM's loads
};

constexpr int kMaxPaced = 8;  // kept frames the paced copy can handle

// Paced new_cache copy of the persistent kernel: kept frame j (Z's frame
// z_len - keep + j) is read by output frame o[j] through the tap whose first
// k-block in that frame's tiles is kb[j]; the CTA that issues that k-block
// copies its box's share of the frame right after issuing it, while the same
// input lines are being fetched into L2 for the GEMM.
struct PacedCopy {
    int o[kMaxPaced];
    int kb[kMaxPaced];
};

// Temporal bookkeeping of one call (paper, Sec. 4): tap k of output frame o
// reads frame o + delta[k] of Z, and is active iff o_l[k] <= o < o_h[k].
struct Taps {
    int kt;
    int s_t;                // temporal stride: output o's tap k reads frame o*s_t + delta[k]
    int delta[kMaxTaps];
    int o_l[kMaxTaps];
    int o_h[kMaxTaps];
};

constexpr int kMaxFrames = 64;  // (n, o) frames a persistent stream-K launch can hold

// Stream-K schedule of the persistent pair kernel.
struct StreamK {
    long long frame_start[kMaxFrames + 1];  // first k-block of each frame's tiles
    long long total;                        // k-blocks of all tiles
    int n_frames;                           // N * T_o
    int G;                                  // CTA pairs in the persistent grid
    int n_acc;                              // TMEM accumulator buffers (1 or 2)
    float* partial;                         // [2G][128][BN] fp32 pieces of split tiles
    unsigned* flags;                        // [2G] epoch of the last published piece
    unsigned epoch;                         // this launch's tag (never 0)
};

struct __align__(64) TcParams {
    CUtensorMap tmap_x;      // x      as [N*T_x, H, W, Cin], box [BK, bw*s_w, bh*s_h, 1]
    CUtensorMap tmap_c;      // cache  as [N*|C|, H, W, Cin] (unused when |C| = 0)
    CUtensorMap tmap_w;      // weight as [Cout, kt*kh*kw, Cin], box [BK, 1, BN]
    // two-frame kernel, one load per stage for all kw column taps: weight as
    // [taps, Cout, Cin] (dims Cin, Cout, taps), box [BK, rows, kw] -> smem
    // [kw][rows][BK], the per-tap K-major tiles the MMAs read; rows = BN
    // (both frames' stages) or BN/2 (one frame's)
    CUtensorMap tmap_wkw_full, tmap_wkw_half;
    int w_kw_boxes;          // 1: the two-frame kernel loads weights with the maps above
    CUtensorMap tmap_out;    // out as [N*T_o, H_o, W_o, Cout], box [kCh, box_w, box_h, 1]
    // the same tensor, box of one warp's 32 pixels of a box:
    // [kCh, min(32, box_w), max(1, 32 / box_w), 1] (pair kernel's epilogue)
    CUtensorMap tmap_out_w;
    const uint16_t* bias;    // bf16 [Cout] or null
    uint16_t* out;           // bf16 [N, T_o, H_o, W_o, Cout]
    int* status;
    CopyJob copy;
    Taps taps;
    int N, T_o, H_o, W_o, Cin, Cout, kh, kw;
    int s_h, s_w, p_h, p_w, d_h, d_w;
    int cache_len, T_x;
    int cache_slots, cache_head;  // cache frame t of entry n: ring_frame(n, t, cache_slots, cache_head)
    int box_h, box_w, tiles_x, tiles_y, tiles_n;
    int BN, n_sub, n_cb, stages, tmem_cols;
    int pairs_per_frame;     // CTA-pair kernel: ceil(tiles_x * tiles_y / 2)
    int rot_div;             // tiles (or pairs) over which K-start offsets are spread
    int halo_w;              // halo kernel: pixels per input strip (128 + (kw-1)*d_w)
    StreamK sk;
    uint64_t wait_limit_ns;
    int x_frames, c_frames;  // frames of the x and cache tensor maps (checked build)
    PacedCopy paced;         // persistent kernel: frames of copy.paced_mask
    int H, W;                // input frame extent (the paced copy's regions)
    // thin-output kernel (conv_tcn.cuh): G output frames per tile in tn_groups
    // groups, tn_cbk TMEM columns per frame, tn_rows = kw*Cout weight rows per tap
    int tn_G, tn_groups, tn_cbk, tn_rows;
};

struct SimtParams {
    const void* x;
    const void* cache;
    const void* w;
    const void* bias;
    void* out;
    CopyJob copy;
    Taps taps;
    int N, T_o, H_o, W_o, Cin, Cout, H, W, kh, kw;
    int s_h, s_w, p_h, p_w, d_h, d_w;
    int cache_len, T_x;
    int cache_slots, cache_head;
    int co_groups;
    long long conv_threads;  // N*T_o*H_o*W_o*co_groups
    int conv_blocks, copy_blocks;
    // shared-memory kernel (small calls): bands of band_h output rows per
    // frame, rows_in staged input rows per tap, staged rows padded to Wp
    // pixels; w_floats = Cout*kt*kh*kw*Cin staged weights
    int band_h, bands, rows_in, Wp;
    long long w_floats;
    long long out_elems;  // buffer extent (checked build; w's is w_floats)
    int* status;          // status word: bounds violations of the checked build
};

}  // namespace ccv3d
