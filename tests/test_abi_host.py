"""Host-side checks of libccv3d (no GPU needed): exported symbols, the
planner against the oracle's brute-force tap scan, validation and error codes."""
import itertools
import os
import re
import subprocess

import pytest

import oracle
from causal_conv3d_video_b200 import ccv3d, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "ccv3d.h")).read()
    return set(re.findall(r"CCV3D_API\s+[\w\s\*]*?\b(ccv3d_\w+)\s*\(", hdr))


def test_library_exports_every_declared_symbol():
    declared = _declared_symbols()
    assert declared == set(ccv3d.EXPORTED)
    out = subprocess.check_output(["nm", "-D", "--defined-only", ccv3d.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (ccv3d_\w+)", out))
    assert declared <= exported, declared - exported
    for name in declared:
        assert hasattr(ccv3d.lib, name)


def test_no_oracle_in_product():
    # the product library must not link or name the oracle
    out = subprocess.check_output(["nm", "-D", ccv3d.LIB_PATH]).decode()
    assert "oracle" not in out
    deps = subprocess.check_output(["ldd", ccv3d.LIB_PATH]).decode()
    assert "oracle" not in deps


def _plan(**kw):
    return ccv3d.ccv3d_plan(ccv3d.make_desc(**kw))


@pytest.mark.parametrize("s_t", [1, 2, 3])
@pytest.mark.parametrize("d_t", [1, 2, 3])
def test_planner_matches_oracle_scan_exhaustive(d_t, s_t):
    """Intervals of the closed forms == brute-force scan, bit for bit."""
    for cl, T_x, pb in itertools.product(range(0, 7), range(1, 7), range(0, 7)):
        kw = dict(N=1, Cin=16, Cout=16, H=4, W=4, T_x=T_x, cache_len=cl,
                  dilation=(d_t, 1, 1), pad_t_base=pb, stride_t=s_t)
        op = oracle.params(1, 16, 16, 4, 4, T_x, cl, dilation=(d_t, 1, 1), pad_t_base=pb,
                           stride_t=s_t)
        T_o, H_o, W_o, keep = oracle.shape(op)
        if T_o <= 0:
            with pytest.raises(ccv3d.CCV3DError) as e:
                _plan(**kw)
            assert e.value.status == ccv3d.CCV3D_ERR_EMPTY_OUTPUT
            continue
        h = _plan(**kw)
        try:
            iv = ccv3d.ccv3d_plan_intervals(h)
            T_s, delta, o_l, o_h, active = oracle.tap_scan(op)
            assert (iv["T_o"], iv["H_o"], iv["W_o"]) == (T_o, H_o, W_o)
            assert iv["delta"] == delta
            assert iv["o_l"] == o_l and iv["o_h"] == o_h, (cl, T_x, pb, iv, o_l, o_h)
            assert ccv3d.ccv3d_plan_sizes(h)["new_cache_frames"] == keep
        finally:
            ccv3d.ccv3d_destroy(h)


@pytest.mark.parametrize("name", sorted(workloads.WORKLOADS))
def test_planner_shapes_match_oracle_on_workloads(name):
    c = workloads.WORKLOADS[name]
    op = oracle.params(c.N, c.Cin, c.Cout, c.H, c.W, c.T_x, c.cache_len, kt=c.kt,
                       kh=c.kh, kw=c.kw, pad_t_base=c.pad_t_base, cache_keep=c.cache_keep,
                       stride=c.stride, pad=c.pad, dilation=c.dilation, stride_t=c.stride_t)
    plan = ccv3d.Plan(ccv3d.desc_for(c))
    T_o, H_o, W_o, keep = oracle.shape(op)
    _, delta, o_l, o_h, _ = oracle.tap_scan(op)
    iv = plan.intervals
    assert (iv["T_o"], iv["H_o"], iv["W_o"]) == (T_o, H_o, W_o)
    assert (iv["delta"], iv["o_l"], iv["o_h"]) == (delta, o_l, o_h)
    assert plan.sizes["new_cache_frames"] == keep
    # bf16 workloads with 16-multiple input channels take the tensor cores (the
    # 3-channel RGB output conv the thin-output kernel); fp32 the SIMT path
    assert plan.path["tc"] == (c.dtype == "bf16" and c.Cin % 16 == 0)
    if plan.path["tc"] and c.Cout % 16 != 0:
        assert plan.kernel == "tc_thin"


@pytest.mark.parametrize("kw,status", [
    (dict(kt=2), ccv3d.CCV3D_ERR_UNSUPPORTED),
    (dict(stride_t=0), ccv3d.CCV3D_ERR_INVALID),
    (dict(stride_t=2, T_x=2, cache_len=0, pad_t_base=0), ccv3d.CCV3D_ERR_EMPTY_OUTPUT),  # |Zp| = 2 < 3
    (dict(groups=2), ccv3d.CCV3D_ERR_UNSUPPORTED),
    (dict(Cin=0), ccv3d.CCV3D_ERR_INVALID),
    (dict(T_x=0), ccv3d.CCV3D_ERR_INVALID),
    (dict(cache_len=-1), ccv3d.CCV3D_ERR_INVALID),
    (dict(stride=(0, 1)), ccv3d.CCV3D_ERR_INVALID),
    (dict(N=0), ccv3d.CCV3D_ERR_EMPTY_OUTPUT),
    (dict(H=1, pad=(0, 1)), ccv3d.CCV3D_ERR_EMPTY_OUTPUT),
    (dict(pad_t_base=0, cache_len=0, T_x=1), ccv3d.CCV3D_ERR_EMPTY_OUTPUT),
])
def test_plan_refusals(kw, status):
    base = dict(N=1, Cin=16, Cout=16, H=8, W=8, T_x=1, cache_len=2)
    base.update(kw)
    with pytest.raises(ccv3d.CCV3DError) as e:
        _plan(**base)
    assert e.value.status == status


def test_bad_dtype_refused():
    d = ccv3d.make_desc(N=1, Cin=16, Cout=16, H=8, W=8, T_x=1, cache_len=2)
    d.dtype = 7
    with pytest.raises(ccv3d.CCV3DError) as e:
        ccv3d.ccv3d_plan(d)
    assert e.value.status == ccv3d.CCV3D_ERR_UNSUPPORTED


def test_null_arguments():
    assert ccv3d.lib.ccv3d_plan(None, None) == ccv3d.CCV3D_ERR_INVALID
    assert ccv3d.lib.ccv3d_plan_intervals(None, None, None, None, None, None, None) == \
        ccv3d.CCV3D_ERR_INVALID
    assert ccv3d.ccv3d_plan_path(None)["tc"] is False
    ccv3d.ccv3d_destroy(None)  # ignored
    for s in range(9):
        assert ccv3d.ccv3d_strerror(s)


def test_forward_validation_order_without_gpu():
    """Argument checks run before any device work; with no GPU a well-formed
    call is refused with CCV3D_ERR_CUDA, never executed on the host."""
    plan = ccv3d.Plan(ccv3d.make_desc(N=1, Cin=16, Cout=16, H=8, W=8, T_x=1, cache_len=2))
    A = 1 << 20
    args = dict(x=A, cache=2 * A, w=3 * A, bias=4 * A, out=5 * A, new_cache=6 * A)

    def call(**over):
        a = dict(args)
        a.update(over)
        st = dict(stride=plan.stride, pad=plan.pad, dilation=plan.dilation)
        st.update({k: over.pop(k) for k in list(over) if k in st})
        a = {k: v for k, v in a.items() if k not in st}
        return ccv3d.ccv3d_forward(plan.handle, a["x"], a["cache"], a["w"], a["bias"],
                                   a["out"], a["new_cache"], st["stride"], st["pad"],
                                   st["dilation"], stream=0, check=False)

    assert call(stride=(2, 1)) == ccv3d.CCV3D_ERR_INVALID
    assert call(dilation=(2, 1, 1)) == ccv3d.CCV3D_ERR_INVALID
    assert call(x=None) == ccv3d.CCV3D_ERR_INVALID
    assert call(cache=None) == ccv3d.CCV3D_ERR_INVALID
    assert call(bias=None) == ccv3d.CCV3D_ERR_INVALID
    assert call(new_cache=None) == ccv3d.CCV3D_ERR_INVALID
    assert call(x=A + 8) == ccv3d.CCV3D_ERR_ALIGNMENT
    assert call(new_cache=A + 64) == ccv3d.CCV3D_ERR_ALIAS      # inside x
    assert call(out=2 * A + 16) == ccv3d.CCV3D_ERR_ALIAS        # inside cache
    st = call()
    import torch
    if not torch.cuda.is_available():
        assert st == ccv3d.CCV3D_ERR_CUDA
    stats = plan.stats()
    assert stats["calls"] == 0 and stats["errors"] >= 9
    assert stats["workspace_bytes"] == 0


def test_tile_choice_on_bottleneck():
    plan = ccv3d.Plan(ccv3d.desc_for(workloads.C2))
    assert plan.path == {"tc": True, "tile_m": 256, "tile_n": 384}
    assert ccv3d.Plan(ccv3d.desc_for(workloads.C3)).path["tile_n"] == 96
    assert ccv3d.Plan(ccv3d.desc_for(workloads.C4_TIME)).path["tile_n"] == 256  # 768 = 3 x 256
    thin = ccv3d.Plan(ccv3d.make_desc(N=1, Cin=3, Cout=16, H=8, W=8, T_x=1, cache_len=0))
    assert thin.path["tc"] is False


@pytest.mark.parametrize("conv,kernel", [
    (workloads.C2, "tc_pair"),                      # 0.8 wave of pair tiles
    (workloads.C3, "tc_pair_fused"),                # thin 720x1280, 4 frames: frame pairs
    (workloads.C4_TIME, "tc_persistent"),           # 6.1 waves, ragged last wave
    (workloads.C4_STRIDE, "tc_persistent"),         # 3.04 waves
    (workloads.C4_DIL, "tc_persistent"),
    (workloads.C4_ODD, "tc_pair"),
    (workloads.Conv("g8", 192, 192, 360, 640, T_x=2, cache_len=2), "tc_persistent"),  # halo, Cout 192
    (workloads.Conv("g5", 384, 384, 360, 640, T_x=2, cache_len=2), "tc_pair"),        # 24.3 even waves
], ids=lambda v: getattr(v, "name", v))
def test_kernel_choice(conv, kernel, monkeypatch):
    """Persistent stream-K where one launch of pair tiles leaves a ragged
    last wave over >= 2 waves, or where the halo kernel would run Cout >= 192;
    CCV3D_PERSIST=0/1 overrides."""
    monkeypatch.delenv("CCV3D_PERSIST", raising=False)
    assert ccv3d.Plan(ccv3d.desc_for(conv)).kernel == kernel
    monkeypatch.setenv("CCV3D_TEST_OVERRIDES", "1")
    monkeypatch.setenv("CCV3D_PERSIST", "0")
    assert ccv3d.Plan(ccv3d.desc_for(conv)).kernel != "tc_persistent"
    monkeypatch.setenv("CCV3D_PERSIST", "1")
    plan = ccv3d.Plan(ccv3d.desc_for(conv))
    assert plan.kernel == "tc_persistent"
    # the persistent kernel streams the widest channel block, whatever a halo
    # sizing (two CTAs per SM) would have chosen
    want_bk = 64 if conv.Cin % 64 == 0 else (32 if conv.Cin % 32 == 0 else 16)
    assert plan.tiling["k_block"] == want_bk


def test_plan_tiling_reports():
    halo = ccv3d.Plan(ccv3d.desc_for(workloads.C3.replace(T_x=1)))
    assert halo.kernel == "tc_pair_halo"
    assert halo.tiling["k_block"] in (16, 32) and halo.tiling["stages"] >= 2
    assert halo.tiling["workspace_pairs"] == 0
    simt = ccv3d.Plan(ccv3d.desc_for(workloads.C1))
    assert simt.tiling == {"k_block": 0, "stages": 0, "workspace_pairs": 0}
    assert ccv3d.lib.ccv3d_plan_tiling(None, None, None, None) == ccv3d.CCV3D_ERR_INVALID


def test_quantize_validation_without_gpu():
    """Argument checks of ccv3d_quantize_u8 run before any device work."""
    lib = ccv3d.lib
    A = 1 << 20
    assert lib.ccv3d_quantize_u8(A, ccv3d.CCV3D_FP32, 2 * A, -1, None) == ccv3d.CCV3D_ERR_INVALID
    assert lib.ccv3d_quantize_u8(A, 9, 2 * A, 16, None) == ccv3d.CCV3D_ERR_INVALID
    assert lib.ccv3d_quantize_u8(None, ccv3d.CCV3D_FP32, 2 * A, 16, None) == ccv3d.CCV3D_ERR_INVALID
    assert lib.ccv3d_quantize_u8(A + 4, ccv3d.CCV3D_FP32, 2 * A, 16, None) == ccv3d.CCV3D_ERR_ALIGNMENT
    assert lib.ccv3d_quantize_u8(A, ccv3d.CCV3D_FP32, A + 48, 16, None) == ccv3d.CCV3D_ERR_ALIAS
    assert lib.ccv3d_quantize_u8(A, ccv3d.CCV3D_BF16, A + 16, 16, None) == ccv3d.CCV3D_ERR_ALIAS
    assert lib.ccv3d_quantize_u8(A, ccv3d.CCV3D_FP32, 2 * A, 0, None) == ccv3d.CCV3D_OK


def test_simt_variant_choice():
    """Calls too small for one thread per (pixel, 4 channels) to fill the SMs
    run one warp per unit (the lanes split the reduction)."""
    # Cin = 16 divides 32 and Cout = 16: one warp per pixel for all channels
    assert ccv3d.Plan(ccv3d.desc_for(workloads.C1)).kernel == "simt_warp16"
    from parity_util import plan_env
    with plan_env({"CCV3D_SIMT_W16": 0}):
        assert ccv3d.Plan(ccv3d.desc_for(workloads.C1)).kernel == "simt_warp"
    with plan_env({"CCV3D_SIMT_SMEM": 1}):  # the shared-memory kernel is opt-in
        assert ccv3d.Plan(ccv3d.desc_for(workloads.C1)).kernel == "simt_smem"
    # 17 output channels, or Cin = 12 (does not divide 32): 4 channels per warp
    c17 = workloads.Conv("f32_17", 16, 17, 16, 16, T_x=3, cache_len=2, dtype="fp32")
    assert ccv3d.Plan(ccv3d.desc_for(c17)).kernel == "simt_warp"
    c12 = workloads.Conv("f32_12", 12, 16, 16, 16, T_x=3, cache_len=2, dtype="fp32")
    assert ccv3d.Plan(ccv3d.desc_for(c12)).kernel == "simt_warp"
    # weights of 384 -> 384 x 27 fp32 (15.9 MB) do not fit in shared memory
    wide = workloads.Conv("f32_wide", 384, 384, 4, 4, T_x=1, cache_len=2, dtype="fp32")
    assert ccv3d.Plan(ccv3d.desc_for(wide)).kernel == "simt_warp"
    big = workloads.Conv("f32_big", 32, 32, 64, 64, T_x=4, cache_len=2, dtype="fp32")
    assert ccv3d.Plan(ccv3d.desc_for(big)).kernel == "simt"


def test_thin_output_kernel_choice():
    """Outputs too narrow for an MMA's N take the kernel that stacks the
    temporal and column taps along N, where its conditions hold (unit temporal
    stride and dilation, unit W stride, kt * (kw * Cout rounded up to 16) <= 256
    columns); otherwise the SIMT kernels."""
    from parity_util import plan_env
    rgb = workloads.C_RGB
    plan = ccv3d.Plan(ccv3d.desc_for(rgb))
    assert plan.kernel == "tc_thin"
    assert plan.path["tile_m"] == 128 and plan.path["tile_n"] == 48  # 3 taps x 16 columns
    assert plan.tiling["k_block"] == 32  # widest channel block dividing 96
    with plan_env({"CCV3D_THIN": 0}):
        assert ccv3d.Plan(ccv3d.desc_for(rgb)).kernel == "simt_tile"
    with plan_env({"CCV3D_THIN": 1}):  # also for Cout = 16 (tests)
        c = workloads.Conv("bf16_thin16", 32, 16, 24, 40, T_x=3, cache_len=2)
        assert ccv3d.Plan(ccv3d.desc_for(c)).kernel == "tc_thin"
    base = dict(T_x=4, cache_len=2, sigma_b=0.1)
    # temporal stride 2: output frames do not share the taps' column layout
    s2 = workloads.Conv("s2", 96, 3, 32, 64, stride_t=2, **base)
    assert ccv3d.Plan(ccv3d.desc_for(s2)).kernel.startswith("simt")
    # 3 x (3 x 40 -> 128) columns > 256
    wide = workloads.Conv("wide", 96, 40, 32, 64, **base)
    assert ccv3d.Plan(ccv3d.desc_for(wide)).kernel.startswith("simt")
    # stride 2 along W: the strip is not the output row
    sw = workloads.Conv("sw2", 96, 3, 32, 64, stride=(1, 2), **base)
    assert ccv3d.Plan(ccv3d.desc_for(sw)).kernel.startswith("simt")
    # fp32 and Cin not a multiple of 16 stay on FFMA
    assert ccv3d.Plan(ccv3d.desc_for(workloads.Conv("f", 96, 3, 32, 64, dtype="fp32", **base))).kernel.startswith("simt")
    assert ccv3d.Plan(ccv3d.desc_for(workloads.Conv("c8", 8, 3, 32, 64, **base))).kernel.startswith("simt")


@pytest.mark.parametrize("kw", [
    dict(H=1 << 30, pad=(1 << 30, 1)),            # H_o past 2^31
    dict(H=1 << 16, W=1 << 16),                   # one frame of 2^32 pixels
    dict(N=1 << 20, T_x=1 << 12),                 # N * frames past 2^31
])
def test_plan_refuses_extents_past_32_bit_indexing(kw):
    base = dict(N=1, Cin=16, Cout=16, H=8, W=8, T_x=1, cache_len=2)
    base.update(kw)
    with pytest.raises(ccv3d.CCV3DError) as e:
        ccv3d.Plan(ccv3d.make_desc(**base))
    assert e.value.status == ccv3d.CCV3D_ERR_UNSUPPORTED


def test_overrides_need_the_test_gate(monkeypatch):
    """Without CCV3D_TEST_OVERRIDES=1 the planner ignores every CCV3D_* override:
    a deployment's environment cannot change the kernel or its tiling."""
    monkeypatch.delenv("CCV3D_TEST_OVERRIDES", raising=False)
    want = ccv3d.Plan(ccv3d.desc_for(workloads.C2))
    assert want.kernel == "tc_pair"
    for k, v in (("CCV3D_PERSIST", "1"), ("CCV3D_TILE_N", "128"), ("CCV3D_PAIR", "0"),
                 ("CCV3D_STAGES", "2"), ("CCV3D_FORCE_PATH", "simt")):
        monkeypatch.setenv(k, v)
    plan = ccv3d.Plan(ccv3d.desc_for(workloads.C2))
    assert plan.kernel == want.kernel and plan.path == want.path
    assert plan.tiling == want.tiling
    monkeypatch.setenv("CCV3D_TEST_OVERRIDES", "0")
    assert ccv3d.Plan(ccv3d.desc_for(workloads.C2)).kernel == want.kernel
    monkeypatch.setenv("CCV3D_TEST_OVERRIDES", "1")
    assert ccv3d.Plan(ccv3d.desc_for(workloads.C2)).kernel == "simt"


def test_unsupported_counted_apart_from_errors():
    """Refused plans count in the process-wide plans_unsupported counter (there
    is no plan to hold them); a plan's own counters keep errors apart."""
    plan = ccv3d.Plan(ccv3d.make_desc(N=1, Cin=16, Cout=16, H=8, W=8, T_x=1, cache_len=2))
    before = plan.stats()["plans_unsupported"]
    for kw in (dict(kt=2), dict(groups=2), dict(kt=5)):
        base = dict(N=1, Cin=16, Cout=16, H=8, W=8, T_x=1, cache_len=2)
        base.update(kw)
        with pytest.raises(ccv3d.CCV3DError) as e:
            _plan(**base)
        assert e.value.status == ccv3d.CCV3D_ERR_UNSUPPORTED
    with pytest.raises(ccv3d.CCV3DError):
        _plan(N=1, Cin=0, Cout=16, H=8, W=8, T_x=1, cache_len=2)   # INVALID: not counted
    st = plan.stats()
    assert st["plans_unsupported"] == before + 3
    assert st["unsupported"] == 0 and st["errors"] == 0


def test_ring_call_validation_without_gpu():
    """ccv3d_forward_ring checks its ring arguments before any device work."""
    plan = ccv3d.Plan(ccv3d.make_desc(N=1, Cin=16, Cout=16, H=8, W=8, T_x=1, cache_len=2))
    A = 1 << 20
    frame = 8 * 8 * 16 * 2

    def call(ring=8 * A, slots=3, head=0, x=A, out=5 * A, w=3 * A, bias=4 * A):
        return ccv3d.ccv3d_forward_ring(plan.handle, x, ring, slots, head, w, bias, out,
                                        plan.stride, plan.pad, plan.dilation, stream=0,
                                        check=False)[0]

    assert call(slots=2) == ccv3d.CCV3D_ERR_INVALID       # |C| + 1 written > 2 slots
    assert call(head=3) == ccv3d.CCV3D_ERR_INVALID        # head outside the ring
    assert call(head=-1) == ccv3d.CCV3D_ERR_INVALID
    assert call(ring=None) == ccv3d.CCV3D_ERR_INVALID
    assert call(ring=8 * A + 8) == ccv3d.CCV3D_ERR_ALIGNMENT
    assert call(ring=A + frame // 2) == ccv3d.CCV3D_ERR_ALIAS    # ring overlaps x
    assert call(out=8 * A + frame) == ccv3d.CCV3D_ERR_ALIAS      # out inside the ring
    import torch
    if not torch.cuda.is_available():
        assert call() == ccv3d.CCV3D_ERR_CUDA
    assert plan.stats()["calls"] == 0 and plan.stats()["errors"] >= 7


def test_checked_build_exports_the_same_abi():
    """libccv3d_checked.so (-DCCV3D_CHECKED) is the same ABI with every kernel
    address range-checked; it exports every declared symbol too."""
    from causal_conv3d_video_b200 import build
    path = build.CHECKED_LIB_PATH
    if not os.path.exists(path):
        build.build(checked=True)
    out = subprocess.check_output(["nm", "-D", "--defined-only", path]).decode()
    exported = set(re.findall(r"\bT (ccv3d_\w+)", out))
    assert _declared_symbols() <= exported
    assert "oracle" not in subprocess.check_output(["nm", "-D", path]).decode()
