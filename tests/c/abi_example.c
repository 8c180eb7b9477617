/*
 * abi_example.c -- the C ABI used from plain C (no Python, no torch).
 *
 * Plans the decoder-bottleneck call (bf16 384->384, 3x3x3, 90x160, a 2-frame
 * cache, 1 new frame), prints the planner's intervals and kernel, and, when a
 * CUDA device is present, runs one forward on zero inputs with a known bias
 * and checks that every output equals the bias and that new_cache is zero.
 * Exit status 0 on success.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "ccv3d.h"

static uint16_t bf16_of(float f) {  /* exact for the small integers used here */
    union { float f; uint32_t u; } v;
    v.f = f;
    return (uint16_t)(v.u >> 16);
}

int main(void) {
    ccv3d_desc d = {0};
    d.N = 1; d.Cin = 384; d.Cout = 384; d.kt = 3; d.kh = 3; d.kw = 3;
    d.H = 90; d.W = 160; d.T_x = 1; d.cache_len = 2; d.pad_t_base = 2; d.cache_keep = 2;
    d.stride_t = 1; d.stride_h = 1; d.stride_w = 1; d.pad_h = 1; d.pad_w = 1;
    d.dil_t = 1; d.dil_h = 1; d.dil_w = 1; d.groups = 1; d.dtype = CCV3D_BF16; d.has_bias = 1;

    ccv3d_plan_t plan = NULL;
    ccv3d_status st = ccv3d_plan(&plan, &d);
    if (st != CCV3D_OK) {
        printf("ccv3d_plan: %s\n", ccv3d_strerror(st));
        return 1;
    }
    int T_o, H_o, W_o, delta[CCV3D_MAX_KT], o_l[CCV3D_MAX_KT], o_h[CCV3D_MAX_KT];
    ccv3d_plan_intervals(plan, &T_o, &H_o, &W_o, delta, o_l, o_h);
    size_t out_bytes = 0, nc_bytes = 0;
    int nc_frames = 0;
    ccv3d_plan_sizes(plan, &out_bytes, &nc_bytes, &nc_frames);
    printf("kernel=%s T_o=%d H_o=%d W_o=%d delta=(%d,%d,%d) new_cache_frames=%d\n",
           ccv3d_plan_kernel(plan), T_o, H_o, W_o, delta[0], delta[1], delta[2], nc_frames);
    if (T_o != 1 || H_o != 90 || W_o != 160 || nc_frames != 2) return 2;

    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        printf("no CUDA device: host-only checks passed\n");
        ccv3d_destroy(plan);
        return 0;
    }
    const size_t frame = (size_t)d.H * d.W * d.Cin * 2;
    void *x, *cache, *w, *bias, *out, *nc;
    if (cudaMalloc(&x, frame) || cudaMalloc(&cache, 2 * frame) ||
        cudaMalloc(&w, (size_t)d.Cout * 27 * d.Cin * 2) || cudaMalloc(&bias, d.Cout * 2) ||
        cudaMalloc(&out, out_bytes) || cudaMalloc(&nc, nc_bytes))
        return 3;
    cudaMemset(x, 0, frame);
    cudaMemset(cache, 0, 2 * frame);
    cudaMemset(w, 0, (size_t)d.Cout * 27 * d.Cin * 2);
    cudaMemset(nc, 0xFF, nc_bytes);
    uint16_t* hb = (uint16_t*)malloc(d.Cout * 2);
    for (int c = 0; c < d.Cout; ++c) hb[c] = bf16_of((float)(c % 7 - 3));
    cudaMemcpy(bias, hb, d.Cout * 2, cudaMemcpyHostToDevice);

    const int stride[2] = {1, 1}, pad[2] = {1, 1}, dil[3] = {1, 1, 1};
    st = ccv3d_forward(plan, x, cache, w, bias, out, nc, stride, pad, dil, (cudaStream_t)0);
    if (st != CCV3D_OK) {
        printf("ccv3d_forward: %s\n", ccv3d_strerror(st));
        return 4;
    }
    if (cudaDeviceSynchronize() != cudaSuccess || ccv3d_get_status(plan) != CCV3D_OK) return 5;
    uint16_t* ho = (uint16_t*)malloc(out_bytes);
    uint16_t* hn = (uint16_t*)malloc(nc_bytes);
    cudaMemcpy(ho, out, out_bytes, cudaMemcpyDeviceToHost);
    cudaMemcpy(hn, nc, nc_bytes, cudaMemcpyDeviceToHost);
    long long bad = 0;
    for (size_t i = 0; i < out_bytes / 2; ++i) bad += ho[i] != hb[i % d.Cout];
    for (size_t i = 0; i < nc_bytes / 2; ++i) bad += hn[i] != 0;
    ccv3d_stats s;
    ccv3d_get_stats(plan, &s);
    printf("forward ok: mismatches=%lld calls=%llu tc=%llu\n", bad, (unsigned long long)s.calls,
           (unsigned long long)s.tc_path);
    ccv3d_destroy(plan);
    return bad == 0 ? 0 : 6;
}
