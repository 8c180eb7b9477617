"""GPU parity: the C-ABI call against the FP64 oracle on the same seeded inputs.

Small signatures are compared element by element over the whole output (they
span several 128-pixel tiles, several Cout tiles and ragged tails); the
decoder-sized workloads are compared at sampled outputs the oracle evaluates
one by one, with new_cache compared in full and the whole output checked for
NaN/Inf.  Tolerance: max|gpu - oracle| <= 2e-2 rms(oracle) for bf16 and
1e-4 rms(oracle) for fp32.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_conv3d_video_b200 import ccv3d, workloads
from causal_conv3d_video_b200.workloads import Conv
from parity_util import (GpuCall, assert_close, expected_new_cache, inputs_for,
                         oracle_params, sample_indices)

pytestmark = pytest.mark.gpu

SMALL = [
    # multi-tile, ragged 20x37 map, every cache length
    Conv("s64_c0", 64, 64, 20, 37, T_x=1, cache_len=0),
    Conv("s64_c1", 64, 64, 20, 37, T_x=1, cache_len=1),
    Conv("s64_c2", 64, 64, 20, 37, T_x=1, cache_len=2),
    Conv("s64_c2_t3", 64, 64, 20, 37, T_x=3, cache_len=2),
    Conv("s64_c0_t3", 64, 64, 20, 37, T_x=3, cache_len=0),
    # Cout tiles: 384 -> 2 x 192, 768 -> 3 x 256, 400 -> 2 x 208 (ragged N)
    Conv("s128to384", 128, 384, 12, 20, T_x=1, cache_len=2),
    Conv("s64to400", 64, 400, 9, 15, T_x=1, cache_len=1),
    Conv("s3x1x1_384to768", 384, 768, 10, 16, T_x=1, cache_len=2, kh=1, kw=1, pad=(0, 0)),
    # K blocks: Cin 96 (BK 32), 48 and 16 (BK 16), Cout 96 / 48
    Conv("s96", 96, 96, 24, 40, T_x=4, cache_len=2, sigma_b=0.1),
    Conv("s192to96", 192, 96, 16, 24, T_x=2, cache_len=1, sigma_b=0.1),
    Conv("s48to48", 48, 48, 11, 13, T_x=2, cache_len=2),
    Conv("s16to384", 16, 384, 18, 32, T_x=1, cache_len=0),
    # stride 2, dilations, odd sizes, batch 2
    Conv("s_stride2", 64, 64, 36, 64, T_x=1, cache_len=2, stride=(2, 2)),
    Conv("s_stride2_odd", 32, 32, 17, 23, T_x=2, cache_len=1, stride=(2, 2)),
    Conv("s_dt2_c4", 64, 64, 18, 32, T_x=1, cache_len=4, dilation=(2, 1, 1)),
    Conv("s_dt2_c1_t3", 64, 64, 18, 32, T_x=3, cache_len=1, dilation=(2, 1, 1)),
    Conv("s_dil_hw2", 32, 32, 19, 27, T_x=1, cache_len=2, pad=(2, 2), dilation=(1, 2, 2)),
    Conv("s_odd", 64, 64, 23, 41, T_x=1, cache_len=2),
    Conv("s_batch2", 32, 48, 10, 12, T_x=2, cache_len=2, N=2),
    # |C| > p_l^base (negative p_l: oldest cached frame dropped)
    Conv("s_crop", 32, 32, 10, 12, T_x=1, cache_len=3),
    # p_l^base = 4 > d_t(kt-1): leading output frames have no active tap (bias only)
    Conv("s_biasonly", 32, 32, 10, 12, T_x=2, cache_len=0, pad_t_base=4, cache_keep=2),
    # 3 boxes per frame: the last CTA pair has a box past the frame
    Conv("s_odd_boxes", 64, 64, 12, 32, T_x=2, cache_len=1),
    # no bias, asymmetric pad/kernel
    Conv("s_nobias", 64, 32, 14, 30, T_x=2, cache_len=2, has_bias=False),
    Conv("s_k3x1x3", 32, 32, 14, 30, T_x=1, cache_len=2, kh=1, kw=3, pad=(0, 1)),
]


def _run_small(c, force_simt=False, env=None):
    inp = inputs_for(c)
    call = GpuCall(c, inp, force_simt=force_simt, env=env).run()
    torch.cuda.synchronize()
    ref, ref_nc = oracle.forward(oracle_params(c), inp["x"], inp["cache"], inp["w"],
                                 inp["bias"])
    got = call.out_f64()
    assert got.shape == ref.shape
    m = assert_close(got, ref, c.dtype, c.name)
    nc = call.nc_f64()
    if ref_nc.size:
        assert np.array_equal(nc, ref_nc), c.name
    assert call.guards_intact(), c.name
    assert call.plan.status() == ccv3d.CCV3D_OK
    return call, m


@pytest.mark.parametrize("smem,w16,kernel", [(1, 1, "simt_smem"), (0, 0, "simt_warp"),
                                              (0, 1, "simt_warp16")])
def test_config1_fp32_exact_workload(smem, w16, kernel):
    call, m = _run_small(workloads.C1, env={"CCV3D_SIMT_SMEM": smem, "CCV3D_SIMT_W16": w16})
    assert call.plan.path["tc"] is False
    assert call.plan.kernel == kernel
    assert call.plan.stats()["simt_path"] == 1


KERNELS = {"persistent": {"CCV3D_PERSIST": 1}, "pair": {"CCV3D_PERSIST": 0},
           "single": {"CCV3D_PAIR": 0, "CCV3D_PERSIST": 0}}


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("c", SMALL, ids=lambda c: c.name)
def test_small_tensor_core(c, kernel):
    call, _ = _run_small(c, env=KERNELS[kernel])
    assert call.plan.path["tc"] is True
    st = call.plan.stats()
    assert st["calls"] == 1 and st["tc_path"] == 1 and st["errors"] == 0


@pytest.mark.parametrize("pairs", [2, 3, 5, 11])
@pytest.mark.parametrize("c", [SMALL[3], SMALL[5], SMALL[8], SMALL[12], SMALL[15], SMALL[18]],
                         ids=lambda c: c.name)
def test_small_stream_k_split_tiles(c, pairs):
    """Few persistent pairs: tiles are cut across pairs and finished by their
    owner from published fp32 pieces; repeated calls reuse the scratch flags."""
    call, _ = _run_small(c, env={"CCV3D_PERSIST": 1, "CCV3D_SK_PAIRS": pairs})
    first = call.out.clone()
    call.run()
    call.run()
    torch.cuda.synchronize()
    assert torch.equal(first, call.out)
    assert call.plan.status() == ccv3d.CCV3D_OK


@pytest.mark.parametrize("env", [{"CCV3D_TILE_N": 384}, {"CCV3D_TILE_N": 384, "CCV3D_PAIR": 0},
                                 {"CCV3D_TILE_N": 128}, {"CCV3D_STAGES": 2}],
                         ids=["n384_pair", "n384_single", "n128", "stages2"])
@pytest.mark.parametrize("c", [SMALL[5], SMALL[6], SMALL[13]], ids=lambda c: c.name)
def test_small_tile_variants(c, env):
    _run_small(c, env=env)


@pytest.mark.parametrize("box_w", [128, 64, 32, 16, 8])
@pytest.mark.parametrize("c", [SMALL[3], SMALL[12], SMALL[16], SMALL[18]], ids=lambda c: c.name)
def test_small_pair_box_shapes(c, box_w):
    """The pair kernel on every box shape (128 output pixels as box_w x
    128/box_w): its epilogue warps each store their own 32 pixels of the box
    -- a row segment, or 32/box_w whole rows -- clipped at the frame edges."""
    call, _ = _run_small(c, env={"CCV3D_BOX_W": box_w, "CCV3D_PERSIST": 0, "CCV3D_HALO": 0})
    assert call.plan.kernel == "tc_pair", call.plan.kernel


HALO = [
    # one 128-pixel output row per tile: the input strip is loaded once per (tap, channel block)
    Conv("h96_3x256", 96, 96, 3, 384, T_x=2, cache_len=1, sigma_b=0.1),    # 9 boxes: odd
    Conv("h64_6x256", 64, 64, 6, 256, T_x=1, cache_len=2),
    Conv("h32to48_3x200", 32, 48, 3, 200, T_x=3, cache_len=0),              # ragged row
    Conv("h192to96_2x256", 192, 96, 2, 256, T_x=4, cache_len=2, sigma_b=0.1),
    Conv("h64_dilw2", 64, 64, 4, 256, T_x=1, cache_len=2, pad=(2, 2), dilation=(1, 2, 2)),
    Conv("h64_k3x1x1", 64, 128, 4, 256, T_x=1, cache_len=2, kh=1, kw=1, pad=(0, 0)),
    Conv("h64_s2h", 64, 64, 9, 256, T_x=1, cache_len=2, stride=(2, 1)),
]


@pytest.mark.parametrize("halo", [1, 0], ids=["halo", "no_halo"])
@pytest.mark.parametrize("c", HALO, ids=lambda c: c.name)
def test_small_halo_strips(c, halo):
    call, _ = _run_small(c, env={"CCV3D_HALO": halo, "CCV3D_PERSIST": 0, "CCV3D_FUSE": 0})
    assert (call.plan.kernel == "tc_pair_halo") == bool(halo), call.plan.kernel


FUSED = [
    # two output frames per tile, sharing source frames (unit temporal stride)
    Conv("f96_t4_c2", 96, 96, 3, 256, T_x=4, cache_len=2, sigma_b=0.1),
    Conv("f64_t3_c0", 64, 64, 4, 256, T_x=3, cache_len=0),            # odd T_o, warm-up taps
    Conv("f32to48_t5_c1", 32, 48, 3, 200, T_x=5, cache_len=1),        # ragged row, odd T_o
    Conv("f64_biasonly", 64, 64, 2, 256, T_x=3, cache_len=0, pad_t_base=4, cache_keep=2),
    Conv("f64_crop", 64, 64, 2, 256, T_x=2, cache_len=3),              # |C| > p_l^base
    Conv("f128_k311", 128, 128, 2, 256, T_x=4, cache_len=2, kh=1, kw=1, pad=(0, 0)),
    Conv("f64_n2", 64, 64, 2, 256, T_x=2, cache_len=2, N=2),
    Conv("f96_dilw2", 96, 96, 2, 256, T_x=2, cache_len=2, pad=(2, 2), dilation=(1, 2, 2)),
    Conv("f128_s2h", 128, 128, 9, 256, T_x=2, cache_len=1, stride=(2, 1)),
    Conv("f192to96_t4", 192, 96, 2, 384, T_x=4, cache_len=2, sigma_b=0.1),
]


@pytest.mark.parametrize("wkw", [1, 0], ids=["w_one_load", "w_load_per_tap"])
@pytest.mark.parametrize("c", FUSED, ids=lambda c: c.name)
def test_small_fused_frame_pairs(c, wkw):
    """The two-frame kernel, its weights loaded as one [kw][rows][BK] box per
    stage (default) or one box per column tap."""
    call, _ = _run_small(c, env={"CCV3D_PERSIST": 0, "CCV3D_FUSE": 1, "CCV3D_W_KW": wkw})
    assert call.plan.kernel == "tc_pair_fused", call.plan.kernel


@pytest.mark.parametrize("c", FUSED[:3], ids=lambda c: c.name)
def test_small_fused_off_is_halo(c):
    call, _ = _run_small(c, env={"CCV3D_PERSIST": 0, "CCV3D_FUSE": 0})
    assert call.plan.kernel == "tc_pair_halo", call.plan.kernel


def test_full_size_fused_sampled():
    """The 96-channel 720x1280 four-frame call on the frame-pair kernel."""
    c = workloads.C3
    inp = inputs_for(c)
    call = GpuCall(c, inp, env={"CCV3D_FUSE": 1}).run()
    torch.cuda.synchronize()
    assert call.plan.kernel == "tc_pair_fused"
    idx = sample_indices(tuple(call.out.shape), call.plan, n_random=2000)
    ref = oracle.points(oracle_params(c), inp["x"], inp["cache"], inp["w"], inp["bias"], idx)
    got = call.out[tuple(torch.from_numpy(idx.T).cuda())].double().cpu().numpy()
    assert_close(got, ref, c.dtype, c.name)
    assert np.array_equal(call.nc_f64(), expected_new_cache(c, inp))
    assert call.guards_intact() and call.plan.status() == ccv3d.CCV3D_OK


SMALL_ST = [
    # temporal stride (the encoders' downsampling): output frames s_t apart on Zp
    Conv("st2_c2_t4", 64, 64, 20, 37, T_x=4, cache_len=2, stride_t=2),
    Conv("st2_c0_t5", 64, 96, 12, 20, T_x=5, cache_len=0, stride_t=2),      # odd |Zp|
    Conv("st2_3x1x1", 128, 384, 10, 16, T_x=4, cache_len=2, kh=1, kw=1, pad=(0, 0),
         stride_t=2),
    Conv("st2_dt2_c4", 64, 64, 18, 32, T_x=2, cache_len=4, dilation=(2, 1, 1), stride_t=2),
    Conv("st3_c1_t6", 32, 48, 10, 12, T_x=6, cache_len=1, stride_t=3),
    Conv("st2_s2", 64, 64, 36, 64, T_x=2, cache_len=2, stride=(2, 2), stride_t=2),
    Conv("st2_batch2", 32, 48, 10, 12, T_x=4, cache_len=2, N=2, stride_t=2),
]


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("c", SMALL_ST, ids=lambda c: c.name)
def test_small_temporal_stride(c, kernel):
    call, _ = _run_small(c, env=KERNELS[kernel])
    assert call.plan.path["tc"] is True


@pytest.mark.parametrize("pairs", [2, 3])
def test_small_temporal_stride_split_tiles(pairs):
    _run_small(SMALL_ST[0], env={"CCV3D_PERSIST": 1, "CCV3D_SK_PAIRS": pairs})


def test_small_temporal_stride_halo():
    c = Conv("st2_halo", 96, 96, 3, 384, T_x=4, cache_len=2, stride_t=2)
    call, _ = _run_small(c, env={"CCV3D_HALO": 1, "CCV3D_PERSIST": 0})
    assert call.plan.kernel == "tc_pair_halo"


@pytest.mark.parametrize("c", [SMALL_ST[0], SMALL_ST[4],
                               Conv("st2_f32", 8, 12, 13, 17, T_x=3, cache_len=1, stride_t=2,
                                    dtype="fp32")], ids=lambda c: c.name)
def test_small_temporal_stride_simt(c):
    call, _ = _run_small(c, force_simt=c.dtype == "bf16")
    assert call.plan.path["tc"] is False


@pytest.mark.parametrize("smem", [1, 0], ids=["smem", "no_smem"])
@pytest.mark.parametrize("c", SMALL[:4] + SMALL[8:9] + SMALL[12:15] + SMALL[19:21],
                         ids=lambda c: c.name)
def test_small_simt_bf16(c, smem):
    call, _ = _run_small(c, force_simt=True, env={"CCV3D_SIMT_SMEM": smem})
    assert call.plan.path["tc"] is False
    # below 148 x 128 (pixel, 4 channels) units: the shared-memory block kernel
    # when its staged weights and rows fit, else one warp per unit; above: one
    # thread per unit
    iv = call.plan.intervals
    units = c.N * iv["T_o"] * iv["H_o"] * iv["W_o"] * -(-c.Cout // 4)
    if units >= 148 * 128:
        assert call.plan.kernel == "simt"
    else:
        assert call.plan.kernel in (("simt_smem", "simt_warp") if smem
                                    else ("simt_warp", "simt_warp16"))


@pytest.mark.parametrize("c", [
    Conv("f32_s2", 8, 12, 13, 17, T_x=2, cache_len=1, stride=(2, 2), dtype="fp32"),
    Conv("f32_dt2", 5, 7, 9, 11, T_x=1, cache_len=4, dilation=(2, 1, 1), dtype="fp32"),
    Conv("f32_3x1x1", 24, 40, 6, 10, T_x=3, cache_len=0, kh=1, kw=1, pad=(0, 0), dtype="fp32"),
    Conv("bf16_thin_cin3", 3, 16, 12, 12, T_x=2, cache_len=2),
], ids=lambda c: c.name)
def test_small_simt_other(c):
    call, _ = _run_small(c)
    assert call.plan.path["tc"] is False
    call, _ = _run_small(c, env={"CCV3D_SIMT_SMEM": 1})
    assert call.plan.path["tc"] is False


FULL = [n for n, c in workloads.WORKLOADS.items() if c.dtype == "bf16"]
# the oracle evaluates these whole in seconds on the host cores; the two
# 720x1280 four-frame calls (1.8 and 3.7 TFLOP) are compared at sampled outputs
SAMPLED_ONLY = {workloads.C3.name, workloads.C3B.name, workloads.C_RGB.name}


@pytest.mark.parametrize("name", FULL)
def test_full_size(name):
    """Every decoder-sized workload in the launch configuration the bench
    times: element by element against the oracle (sampled for the 720x1280
    calls), new_cache in full, guard bands intact."""
    c = workloads.WORKLOADS[name]
    inp = inputs_for(c)
    call = GpuCall(c, inp).run()
    torch.cuda.synchronize()
    assert call.plan.path["tc"] is (c.Cin % 16 == 0)
    if c.Cout % 16 != 0:
        assert call.plan.kernel == "tc_thin"
    out = call.out
    if name in SAMPLED_ONLY:
        assert bool(torch.isfinite(out.float()).all())
        idx = sample_indices(tuple(out.shape), call.plan, n_random=2000)
        ref = oracle.points(oracle_params(c), inp["x"], inp["cache"], inp["w"], inp["bias"], idx)
        got = out[tuple(torch.from_numpy(idx.T).cuda())].double().cpu().numpy()
        assert_close(got, ref, c.dtype, name)
        want_nc = expected_new_cache(c, inp)
    else:
        ref, want_nc = oracle.forward(oracle_params(c), inp["x"], inp["cache"], inp["w"],
                                      inp["bias"])
        got = call.out_f64()
        assert got.shape == ref.shape
        assert_close(got, ref, c.dtype, name)
    assert np.array_equal(call.nc_f64(), want_nc)
    assert call.guards_intact()
    assert call.plan.status() == ccv3d.CCV3D_OK
    assert call.plan.status_stream() == ccv3d.CCV3D_OK


def test_repeat_calls_identical_and_counters():
    c = SMALL[3]
    inp = inputs_for(c)
    call = GpuCall(c, inp).run()
    first = call.out.clone()
    for _ in range(4):
        call.run()
    torch.cuda.synchronize()
    assert torch.equal(first, call.out)  # fixed reduction order: deterministic
    st = call.plan.stats()
    assert st["calls"] == 5 and st["tc_path"] == 5


def test_other_stream():
    c = SMALL[5]
    inp = inputs_for(c)
    ref_call = GpuCall(c, inp).run()
    s = torch.cuda.Stream()
    call = GpuCall(c, inp)
    with torch.cuda.stream(s):
        call.run(stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(ref_call.out, call.out)


def test_bounded_wait_reports_timeout_and_context_survives():
    st = ccv3d.ccv3d_selftest_wait_timeout(50_000_000)  # 50 ms, nothing arrives
    assert st == ccv3d.CCV3D_ERR_TIMEOUT
    _run_small(SMALL[0])  # the context is still usable


def test_forward_refusals_on_device():
    c = SMALL[2]
    inp = inputs_for(c)
    call = GpuCall(c, inp)
    p = call.plan
    # new_cache aliasing x (ping-pong misuse)
    rc = ccv3d.ccv3d_forward(p.handle, call.x, call.cache, call.w, call.bias, call.out,
                             call.x, p.stride, p.pad, p.dilation, check=False)
    assert rc == ccv3d.CCV3D_ERR_ALIAS
    # misaligned x
    rc = ccv3d.ccv3d_forward(p.handle, call.x.data_ptr() + 2, call.cache, call.w, call.bias,
                             call.out, call.nc, p.stride, p.pad, p.dilation, check=False)
    assert rc == ccv3d.CCV3D_ERR_ALIGNMENT
    assert p.stats()["errors"] == 2 and p.stats()["calls"] == 0


PACED = [
    # kept frames read by a tap are copied tile by tile with the GEMM's loads
    Conv("p64_c2", 64, 64, 20, 37, T_x=1, cache_len=2),
    Conv("p64_c2_t3", 64, 64, 20, 37, T_x=3, cache_len=2),             # kept frames of o > 0
    Conv("p64_dt2_c4", 64, 64, 18, 32, T_x=1, cache_len=4, dilation=(2, 1, 1)),  # 2 of 4 unread
    Conv("p64_s2", 64, 64, 36, 64, T_x=1, cache_len=2, stride=(2, 2)),
    Conv("p64_s2_odd", 32, 32, 17, 23, T_x=2, cache_len=1, stride=(2, 2)),  # edges extend
    Conv("p64_st2", 64, 96, 12, 20, T_x=4, cache_len=2, stride_t=2),
    Conv("p3x1x1", 384, 768, 10, 16, T_x=1, cache_len=2, kh=1, kw=1, pad=(0, 0)),  # 2 Cout tiles
    Conv("p_batch2", 32, 48, 10, 12, T_x=2, cache_len=2, N=2),
]


@pytest.mark.parametrize("pairs", [0, 3])
@pytest.mark.parametrize("paced", [1, 0], ids=["paced", "sliced"])
@pytest.mark.parametrize("c", PACED, ids=lambda c: c.name)
def test_persistent_new_cache_paced_or_sliced(c, paced, pairs):
    """The persistent kernel's new_cache copy, paced with the producer (box
    shares of the frames a tap reads) or in equal slices: out against the
    oracle and new_cache exact either way, with whole or split tiles."""
    env = {"CCV3D_PERSIST": 1, "CCV3D_PACED": paced}
    if pairs:
        env["CCV3D_SK_PAIRS"] = pairs
    call, _ = _run_small(c, env=env)
    assert call.plan.kernel == "tc_persistent"


@pytest.mark.parametrize("mode,paced", [(1, 1), (1, 0), (2, 0)],
                         ids=["one_cta_paced", "one_cta_sliced", "two_ctas"])
@pytest.mark.parametrize("c", FUSED, ids=lambda c: c.name)
def test_small_fused_persistent(c, mode, paced):
    """The persistent form of the two-frame kernel: the same stages, CTA pairs
    walking the tiles, with double-buffered accumulators at one CTA per SM or
    one buffer each at two CTAs per SM (no copy warps); every pair runs many
    tiles, so the accumulator and staging buffers cycle."""
    call, _ = _run_small(c, env={"CCV3D_PERSIST": 0, "CCV3D_FUSE": 1, "CCV3D_FUSED_PERSIST": mode,
                                 "CCV3D_PACED": paced})
    assert call.plan.kernel == "tc_pair_fused_persistent", call.plan.kernel
    first = call.out.clone()
    call.run()
    torch.cuda.synchronize()
    assert torch.equal(first, call.out)
    assert call.plan.status() == ccv3d.CCV3D_OK


def test_full_size_fused_persistent_sampled():
    """The 96-channel 720x1280 four-frame call on the persistent two-frame kernel."""
    c = workloads.C3
    inp = inputs_for(c)
    call = GpuCall(c, inp, env={"CCV3D_FUSED_PERSIST": 1}).run()
    torch.cuda.synchronize()
    assert call.plan.kernel == "tc_pair_fused_persistent"
    idx = sample_indices(tuple(call.out.shape), call.plan, n_random=2000)
    ref = oracle.points(oracle_params(c), inp["x"], inp["cache"], inp["w"], inp["bias"], idx)
    got = call.out[tuple(torch.from_numpy(idx.T).cuda())].double().cpu().numpy()
    assert_close(got, ref, c.dtype, c.name)
    assert np.array_equal(call.nc_f64(), expected_new_cache(c, inp))
    assert call.guards_intact() and call.plan.status() == ccv3d.CCV3D_OK


SIMT_TILE = [
    # large calls with <= 4 output channels: 8 x 128 output tiles, patches per
    # 8 input channels (>= 148 x 128 (pixel, 4-channel) units each)
    Conv("t16to3_45x150_t3", 16, 3, 45, 150, T_x=3, cache_len=2, sigma_b=0.1),     # ragged rows, cols
    Conv("t32to4_40x160_c0", 32, 4, 40, 160, T_x=3, cache_len=0),
    Conv("t8to1_48x130_c1", 8, 1, 48, 130, T_x=4, cache_len=1),
    Conv("t16to2_3x1x1", 16, 2, 40, 200, T_x=3, cache_len=2, kh=1, kw=1, pad=(0, 0)),
    Conv("t16to3_dilh2", 16, 3, 48, 140, T_x=3, cache_len=2, pad=(2, 1), dilation=(1, 2, 1)),
    Conv("t16to3_st2", 16, 3, 40, 160, T_x=6, cache_len=2, stride_t=2),
    Conv("t16to3_fp32", 16, 3, 49, 139, T_x=3, cache_len=2, dtype="fp32", sigma_b=0.1),
    Conv("t8to4_fp32_3x1x1", 8, 4, 48, 150, T_x=3, cache_len=1, kh=1, kw=1, pad=(0, 0),
         dtype="fp32"),
]


@pytest.mark.parametrize("tile", [1, 0], ids=["tile", "thread"])
@pytest.mark.parametrize("c", SIMT_TILE, ids=lambda c: c.name)
def test_simt_tile_thin_cout(c, tile):
    call, _ = _run_small(c, env={"CCV3D_SIMT_TILE": tile, "CCV3D_THIN": 0})
    assert call.plan.path["tc"] is False
    # an fp32 3x3 patch takes more 16-byte loads than a thread holds ahead
    # (10 x 130 pixels x 2): those calls keep the thread kernel
    fits = c.dtype == "bf16" or c.kh * c.kw == 1
    assert call.plan.kernel == ("simt_tile" if tile and fits else "simt"), call.plan.kernel


THIN = [
    # RGB-like 96 -> 3 (channel block 32), ragged last x tile (300 = 2 x 126 + 48)
    Conv("n96to3_c2_t4", 96, 3, 24, 300, T_x=4, cache_len=2, sigma_b=0.1),
    # first chunk (no cache), channel block 64
    Conv("n64to3_c0_t3", 64, 3, 17, 130, T_x=3, cache_len=0),
    # one output channel, channel block 16
    Conv("n16to1_c1", 16, 1, 20, 140, T_x=2, cache_len=1),
    # |C| = 4 > p_l^base: the oldest cached frame is dropped
    Conv("n32to5_c4_crop", 32, 5, 12, 200, T_x=1, cache_len=4),
    # 32 TMEM columns per frame: 4 frames per tile, 9 output frames in 3 groups
    Conv("n48to8_groups", 48, 8, 10, 150, T_x=9, cache_len=2),
    # spatial dilation 2 (124 outputs per strip) and stride 2 along H
    Conv("n32to3_dil2", 32, 3, 19, 160, T_x=2, cache_len=2, pad=(2, 2), dilation=(1, 2, 2)),
    Conv("n32to3_sh2", 32, 3, 21, 150, T_x=2, cache_len=2, stride=(2, 1)),
    # 3x1x1 and 3x1x3 kernels
    Conv("n32to3_3x1x1", 32, 3, 16, 140, T_x=3, cache_len=2, kh=1, kw=1, pad=(0, 0)),
    Conv("n32to6_k3x1x3", 32, 6, 14, 150, T_x=2, cache_len=2, kh=1, kw=3, pad=(0, 1)),
    # batch 2 without bias; leading bias-only frames; rows with no input row at all
    Conv("n32to3_batch2_nobias", 32, 3, 10, 140, T_x=2, cache_len=2, N=2, has_bias=False),
    Conv("n32to3_biasonly", 32, 3, 10, 140, T_x=2, cache_len=0, pad_t_base=4, cache_keep=2),
    Conv("n32to3_pad3", 32, 3, 9, 140, T_x=2, cache_len=2, pad=(3, 3)),
    # six channel blocks of 32, Cout = 8 (32 TMEM columns per frame)
    Conv("n192to8", 192, 8, 7, 140, T_x=2, cache_len=2),
]


@pytest.mark.parametrize("c", THIN, ids=lambda c: c.name)
def test_small_thin_output(c):
    """The thin-output kernel (temporal and column taps stacked along N)
    against the oracle over the whole output."""
    call, _ = _run_small(c)
    assert call.plan.kernel == "tc_thin", call.plan.kernel


def test_small_thin_output_forced_cout16():
    """Cout = 16 on the thin-output kernel (48 TMEM columns per frame, one
    frame per tile) when forced."""
    c = Conv("n32to16_thin", 32, 16, 12, 140, T_x=3, cache_len=2)
    call, _ = _run_small(c, env={"CCV3D_THIN": 1})
    assert call.plan.kernel == "tc_thin", call.plan.kernel


WARP16 = [
    # one warp per pixel for all output channels (Cin divides 32, Cout <= 16)
    Conv("w16_f32_c2_t3", 16, 16, 16, 16, T_x=3, cache_len=2, dtype="fp32", sigma_b=0.1),
    Conv("w16_f32_8to5_c0", 8, 5, 13, 19, T_x=2, cache_len=0, dtype="fp32"),
    Conv("w16_f32_32to12_c4_crop", 32, 12, 9, 11, T_x=1, cache_len=4, dtype="fp32"),
    Conv("w16_f32_4to16_dil", 4, 16, 12, 14, T_x=2, cache_len=2, pad=(2, 2),
         dilation=(2, 2, 2), dtype="fp32"),
    Conv("w16_f32_16to3_s2", 16, 3, 17, 15, T_x=2, cache_len=1, stride=(2, 2), dtype="fp32",
         has_bias=False),
    Conv("w16_f32_2to7_3x1x1_b2", 2, 7, 10, 12, T_x=3, cache_len=2, kh=1, kw=1, pad=(0, 0),
         N=2, dtype="fp32"),
    Conv("w16_bf16_16to8", 16, 8, 14, 18, T_x=2, cache_len=2, sigma_b=0.1, dtype="bf16"),
    Conv("w16_f32_biasonly", 8, 8, 10, 12, T_x=2, cache_len=0, pad_t_base=4, cache_keep=2,
         dtype="fp32"),
]


@pytest.mark.parametrize("c", WARP16, ids=lambda c: c.name)
def test_small_simt_warp16(c):
    call, _ = _run_small(c, force_simt=True)
    assert call.plan.kernel == "simt_warp16", call.plan.kernel
