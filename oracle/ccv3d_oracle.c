/*
 * ccv3d_oracle.c -- plain FP64 CPU oracle for the cached causal Conv3D.
 *
 * TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the CPU
 * baseline leg of the benchmark are the only callers.  The CUDA library never
 * links, loads or calls this file, and this file uses nothing from it.
 *
 * What it computes ("Cache-Aware Conv3D Lowering Across Embedded World-Model
 * Decoders", Sec. 4, the temporal-tap lowering and its cache semantics):
 *
 *   Z  = [C ; X]_T            the temporal cache followed by the current frames
 *   p_l = p_l^base - |C|_T    the effective causal left pad
 *   Zp = p_l zero frames followed by Z        (p_l >= 0)
 *      = Z with its first -p_l frames dropped (p_l <  0)
 *   out[n,o,y,x,co] = bias[co] + sum_{k,r,s,ci}
 *        Zp[n, o*s_t + k*d_t, y*s_h + r*d_h - p_h, x*s_w + s*d_w - p_w, ci]
 *        * W[co, k, r, s, ci]
 *
 * which is PyTorch's cross-correlation convention with one group; spatial
 * positions outside [0,H)x[0,W) read zero.  The paper's lowering covers unit
 * temporal stride (s_t = 1); s_t > 1 (the encoders' temporal downsampling,
 * which the paper leaves on native Conv3D) is the same definition with the
 * output frames s_t apart on Zp.  Sums are
 * accumulated in double starting from 0 and the bias is added last, once.
 * new_cache holds the last min(cache_keep, |Z|) frames of Z (the plain reading
 * of "the cache carries the trailing frames of the cache-augmented input").
 *
 * This is the DEFINITION, not the paper's lowering: Z is materialised, the
 * causal pad is materialised as zero frames, every (k, r, s) term is visited
 * and no interval arithmetic is used.  Output sizes come from the usual
 * convolution length formula (stride s_t, no right pad) applied to the padded
 * sequence.
 *
 * Layouts (all row-major, channels innermost, "NTHWC"):
 *   x         [N, T_x, H, W, Cin]
 *   cache     [N, |C|, H, W, Cin]      (may be NULL when |C| == 0)
 *   w         [Cout, kt, kh, kw, Cin]
 *   bias      [Cout]                   (may be NULL: no bias)
 *   out       [N, T_o, H_o, W_o, Cout]
 *   new_cache [N, K', H, W, Cin]       K' = min(cache_keep, |Z|)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int N, Cin, Cout;
    int kt, kh, kw;
    int H, W;
    int T_x;        /* frames in X */
    int cache_len;  /* |C|_T */
    int pad_t_base; /* p_l^base */
    int cache_keep; /* frames kept for the next call */
    int s_h, s_w;
    int p_h, p_w;
    int d_t, d_h, d_w;
    int s_t;        /* temporal stride (1 in the paper's supported contract) */
} oracle_params;

/* Output extents of the convolution over the padded sequence Zp.
 * Returns 0 on success, -1 when a parameter is out of range. */
int oracle_shape(const oracle_params* p, int* T_o, int* H_o, int* W_o,
                 int* keep) {
    if (p->N < 0 || p->Cin <= 0 || p->Cout <= 0 || p->kt <= 0 || p->kh <= 0 ||
        p->kw <= 0 || p->H <= 0 || p->W <= 0 || p->T_x < 0 ||
        p->cache_len < 0 || p->pad_t_base < 0 || p->cache_keep < 0 ||
        p->s_h <= 0 || p->s_w <= 0 || p->p_h < 0 || p->p_w < 0 ||
        p->d_t <= 0 || p->d_h <= 0 || p->d_w <= 0 || p->s_t <= 0)
        return -1;
    int z_len = p->cache_len + p->T_x;
    int p_l = p->pad_t_base - p->cache_len;
    int zp_len = z_len + p_l; /* pad in front, or crop when p_l < 0 */
    if (zp_len < 0) zp_len = 0;
    /* standard length formula, stride s_t, no right pad */
    int tn = zp_len - p->d_t * (p->kt - 1) - 1;
    *T_o = tn < 0 ? 0 : tn / p->s_t + 1;
    *H_o = (p->H + 2 * p->p_h - p->d_h * (p->kh - 1) - 1) / p->s_h + 1;
    *W_o = (p->W + 2 * p->p_w - p->d_w * (p->kw - 1) - 1) / p->s_w + 1;
    if (p->H + 2 * p->p_h - p->d_h * (p->kh - 1) - 1 < 0) *H_o = 0;
    if (p->W + 2 * p->p_w - p->d_w * (p->kw - 1) - 1 < 0) *W_o = 0;
    if (*T_o < 0) *T_o = 0;
    *keep = p->cache_keep < z_len ? p->cache_keep : z_len;
    return 0;
}

/* Materialise Z = [C; X] along T. Returns a malloc'd [N, |Z|, H, W, Cin]. */
static double* concat_cache_input(const oracle_params* p, const double* x,
                                  const double* cache) {
    size_t frame = (size_t)p->H * p->W * p->Cin;
    int z_len = p->cache_len + p->T_x;
    double* z = (double*)malloc(sizeof(double) * (size_t)p->N * z_len * frame + 1);
    if (!z) return NULL;
    for (int n = 0; n < p->N; ++n) {
        for (int t = 0; t < p->cache_len; ++t)
            memcpy(z + ((size_t)n * z_len + t) * frame,
                   cache + ((size_t)n * p->cache_len + t) * frame,
                   sizeof(double) * frame);
        for (int t = 0; t < p->T_x; ++t)
            memcpy(z + ((size_t)n * z_len + p->cache_len + t) * frame,
                   x + ((size_t)n * p->T_x + t) * frame, sizeof(double) * frame);
    }
    return z;
}

/* Zp = causal zero pad of p_l frames in front of Z (or Z cropped by -p_l). */
static double* causal_pad(const oracle_params* p, const double* z, int* zp_len_out) {
    size_t frame = (size_t)p->H * p->W * p->Cin;
    int z_len = p->cache_len + p->T_x;
    int p_l = p->pad_t_base - p->cache_len;
    int zp_len = z_len + p_l;
    if (zp_len < 0) zp_len = 0;
    double* zp = (double*)calloc((size_t)p->N * zp_len * frame + 1, sizeof(double));
    if (!zp) return NULL;
    for (int n = 0; n < p->N; ++n)
        for (int i = 0; i < zp_len; ++i) {
            int src = i - p_l; /* frame of Z that lands at position i of Zp */
            if (src < 0) continue; /* zero frame */
            memcpy(zp + ((size_t)n * zp_len + i) * frame,
                   z + ((size_t)n * z_len + src) * frame, sizeof(double) * frame);
        }
    *zp_len_out = zp_len;
    return zp;
}

/* Full forward: out and new_cache as defined in the header comment.
 * Returns 0 on success, -1 on bad parameters, -2 on allocation failure. */
int oracle_forward(const oracle_params* p, const double* x, const double* cache,
                   const double* w, const double* bias, double* out,
                   double* new_cache) {
    int T_o, H_o, W_o, keep;
    if (oracle_shape(p, &T_o, &H_o, &W_o, &keep) != 0) return -1;
    double* z = concat_cache_input(p, x, cache);
    if (!z) return -2;
    int zp_len = 0;
    double* zp = causal_pad(p, z, &zp_len);
    if (!zp) { free(z); return -2; }

    const int H = p->H, Wd = p->W, Cin = p->Cin, Cout = p->Cout;
    const int kt = p->kt, kh = p->kh, kw = p->kw;
    long long rows = (long long)p->N * T_o * H_o;
#pragma omp parallel for schedule(dynamic, 1)
    for (long long row = 0; row < rows; ++row) {
        int n = (int)(row / ((long long)T_o * H_o));
        int o = (int)((row / H_o) % T_o);
        int y = (int)(row % H_o);
        for (int xo = 0; xo < W_o; ++xo)
            for (int co = 0; co < Cout; ++co) {
                double acc = 0.0;
                for (int k = 0; k < kt; ++k)
                    for (int r = 0; r < kh; ++r)
                        for (int s = 0; s < kw; ++s) {
                            int t = o * p->s_t + k * p->d_t;
                            int yi = y * p->s_h + r * p->d_h - p->p_h;
                            int xi = xo * p->s_w + s * p->d_w - p->p_w;
                            if (yi < 0 || yi >= H || xi < 0 || xi >= Wd) continue;
                            const double* zrow =
                                zp + ((((size_t)n * zp_len + t) * H + yi) * Wd + xi) * Cin;
                            const double* wrow =
                                w + ((((size_t)co * kt + k) * kh + r) * kw + s) * Cin;
                            for (int ci = 0; ci < Cin; ++ci) acc += zrow[ci] * wrow[ci];
                        }
                if (bias) acc += bias[co];
                out[((((size_t)n * T_o + o) * H_o + y) * W_o + xo) * Cout + co] = acc;
            }
    }

    if (new_cache && keep > 0) {
        size_t frame = (size_t)H * Wd * Cin;
        int z_len = p->cache_len + p->T_x;
        for (int n = 0; n < p->N; ++n)
            memcpy(new_cache + (size_t)n * keep * frame,
                   z + ((size_t)n * z_len + (z_len - keep)) * frame,
                   sizeof(double) * keep * frame);
    }
    free(zp);
    free(z);
    return 0;
}

/* Element of Zp read without materialising it: position i of Zp is frame
 * i - p_l of Z, and frame t of Z is cache[t] when t < |C|, else x[t - |C|]. */
static double zp_at(const oracle_params* p, const double* x, const double* cache,
                    int n, int i, int yi, int xi, int ci) {
    int p_l = p->pad_t_base - p->cache_len;
    int t = i - p_l;
    if (t < 0 || t >= p->cache_len + p->T_x) return 0.0;
    if (yi < 0 || yi >= p->H || xi < 0 || xi >= p->W) return 0.0;
    if (t < p->cache_len)
        return cache[((((size_t)n * p->cache_len + t) * p->H + yi) * p->W + xi) * p->Cin + ci];
    t -= p->cache_len;
    return x[((((size_t)n * p->T_x + t) * p->H + yi) * p->W + xi) * p->Cin + ci];
}

/* The same definition evaluated at chosen outputs, for inputs too large to
 * materialise.  idx holds P rows of (n, o, y, x, co).  Returns 0, or -1 when
 * an index is outside the output. */
int oracle_points(const oracle_params* p, const double* x, const double* cache,
                  const double* w, const double* bias, const long long* idx,
                  long long P, double* vals) {
    int T_o, H_o, W_o, keep;
    if (oracle_shape(p, &T_o, &H_o, &W_o, &keep) != 0) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(| : bad)
    for (long long q = 0; q < P; ++q) {
        int n = (int)idx[5 * q + 0], o = (int)idx[5 * q + 1], y = (int)idx[5 * q + 2];
        int xo = (int)idx[5 * q + 3], co = (int)idx[5 * q + 4];
        if (n < 0 || n >= p->N || o < 0 || o >= T_o || y < 0 || y >= H_o ||
            xo < 0 || xo >= W_o || co < 0 || co >= p->Cout) {
            bad = 1;
            vals[q] = 0.0;
            continue;
        }
        double acc = 0.0;
        for (int k = 0; k < p->kt; ++k)
            for (int r = 0; r < p->kh; ++r)
                for (int s = 0; s < p->kw; ++s) {
                    int i = o * p->s_t + k * p->d_t;
                    int yi = y * p->s_h + r * p->d_h - p->p_h;
                    int xi = xo * p->s_w + s * p->d_w - p->p_w;
                    const double* wrow =
                        w + ((((size_t)co * p->kt + k) * p->kh + r) * p->kw + s) * p->Cin;
                    for (int ci = 0; ci < p->Cin; ++ci)
                        acc += zp_at(p, x, cache, n, i, yi, xi, ci) * wrow[ci];
                }
        if (bias) acc += bias[co];
        vals[q] = acc;
    }
    return bad ? -1 : 0;
}

/* Brute-force temporal tap scan.  For each tap k and each output frame o,
 * position o*s_t + k*d_t of Zp is a real frame of Z exactly when it is not one of
 * the p_l pad frames and not past the end of Z.  The scan records, per tap,
 * the frame of Z read at output 0 (delta[k]), the smallest and one past the
 * largest output frame whose tap is real (o_l, o_h), and whether any is
 * (active).  Inactive taps report o_l = o_h = 0.  Returns 0, or -1 when the
 * real frames of a tap do not form one contiguous run (never expected). */
int oracle_tap_scan(const oracle_params* p, int* T_o_out, int* delta, int* o_l,
                    int* o_h, int* active) {
    int T_o, H_o, W_o, keep;
    if (oracle_shape(p, &T_o, &H_o, &W_o, &keep) != 0) return -1;
    int z_len = p->cache_len + p->T_x;
    int p_l = p->pad_t_base - p->cache_len;
    *T_o_out = T_o;
    for (int k = 0; k < p->kt; ++k) {
        int first = -1, last = -1, count = 0;
        for (int o = 0; o < T_o; ++o) {
            int zframe = (o * p->s_t + k * p->d_t) - p_l; /* Zp position -> Z frame */
            if (zframe >= 0 && zframe < z_len) {
                if (first < 0) first = o;
                last = o;
                ++count;
            }
        }
        delta[k] = (0 + k * p->d_t) - p_l;
        if (count == 0) {
            active[k] = 0;
            o_l[k] = 0;
            o_h[k] = 0;
        } else {
            if (count != last - first + 1) return -1;
            active[k] = 1;
            o_l[k] = first;
            o_h[k] = last + 1;
        }
    }
    return 0;
}

/* Post-decode uint8 quantisation of decoded frames (FastVideo pull request
 * "Quantize frames to uint8 on-device before the post-decode D->H copy",
 * Summary and Correctness): each value is multiplied by 255, clamped to
 * [0, 255] and cast to uint8, the cast truncating toward zero as PyTorch's
 * float -> uint8 conversion does.  The product is taken in fp32, the decoded
 * video's precision on that page, for fp32 and bf16 inputs alike (a bf16
 * input is widened to fp32 first, exactly).  A NaN clamps to 0 (C's fmaxf
 * returns the non-NaN operand).  `in` holds the input values widened to
 * double (exact for fp32/bf16 values).  Returns 0. */
int oracle_quantize_u8(const double* in, long long n, uint8_t* out) {
    for (long long i = 0; i < n; ++i) {
        float v = (float)in[i];          /* the fp32 value, exactly */
        float y = v * 255.0f;            /* one fp32 multiply */
        y = fmaxf(y, 0.0f);              /* NaN -> 0 */
        y = fminf(y, 255.0f);
        out[i] = (uint8_t)(int)y;        /* truncation toward zero */
    }
    return 0;
}

/* Threads an OpenMP region of this library uses (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
#endif
int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
