"""Pins for the FP64 oracle: each checks it against something other than itself.

* hand-worked fixtures (tests/golden/hand_worked.json), derived on paper from
  the definition in "Cache-Aware Conv3D Lowering Across Embedded World-Model
  Decoders", Sec. 4;
* library special cases: torch.nn.functional.conv3d / conv2d in float64 on
  the explicitly padded [C;X], and numpy.correlate for the 1-D temporal case;
* the paper's own identities: the per-tap decomposition equals the Conv3D,
  out-of-range taps contribute nothing, bias counted once, chunked decoding
  with the carried cache equals whole-sequence causal convolution, and the
  source and output intervals have equal length;
* planted mistakes: mutated copies of the oracle source must fail a pin.
"""
import itertools
import json
import os
import re
import subprocess

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from causal_conv3d_video_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "hand_worked.json")


def _params_from(d):
    return oracle.OracleParams(
        d["N"], d["Cin"], d["Cout"], d["kt"], d["kh"], d["kw"], d["H"], d["W"],
        d["T_x"], d["cache_len"], d["pad_t_base"], d["cache_keep"],
        d["stride"][0], d["stride"][1], d["pad"][0], d["pad"][1],
        d["dilation"][0], d["dilation"][1], d["dilation"][2], d.get("stride_t", 1))


def _rand(shape, seed, stream):
    return synth.normal(shape, 1.0, seed, stream).astype(np.float64)


def _ints(shape, rng, lo=-3, hi=4):
    return rng.integers(lo, hi, size=shape).astype(np.float64)


def _torch_reference(p, x, cache, w, bias):
    """F.conv3d (float64, CPU) on F.pad([C;X]) in NCDHW layout."""
    xt = torch.from_numpy(x).permute(0, 4, 1, 2, 3)
    if p.cache_len > 0:
        z = torch.cat([torch.from_numpy(cache).permute(0, 4, 1, 2, 3), xt], dim=2)
    else:
        z = xt
    p_l = p.pad_t_base - p.cache_len
    if p_l >= 0:
        z = F.pad(z, (p.p_w, p.p_w, p.p_h, p.p_h, p_l, 0))
    else:
        z = F.pad(z[:, :, -p_l:], (p.p_w, p.p_w, p.p_h, p.p_h, 0, 0))
    wt = torch.from_numpy(w).permute(0, 4, 1, 2, 3)
    b = torch.from_numpy(bias) if bias is not None else None
    y = F.conv3d(z, wt, b, stride=(p.s_t, p.s_h, p.s_w), padding=0,
                 dilation=(p.d_t, p.d_h, p.d_w))
    return y.permute(0, 2, 3, 4, 1).contiguous().numpy()


def _run_pins_hand(lib):
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        p = _params_from(c["params"])
        T_o, H_o, W_o, keep = oracle.shape(p)
        x = np.array(c["x"], np.float64).reshape(p.N, p.T_x, p.H, p.W, p.Cin)
        cache = (np.array(c["cache"], np.float64).reshape(p.N, p.cache_len, p.H, p.W, p.Cin)
                 if p.cache_len else None)
        w = np.array(c["w"], np.float64).reshape(p.Cout, p.kt, p.kh, p.kw, p.Cin)
        bias = np.array(c["bias"], np.float64)
        out, nc = oracle.forward(p, x, cache, w, bias, lib=lib)
        assert out.ravel().tolist() == c["out"], c["name"]
        assert nc.ravel().tolist() == c["new_cache"], c["name"]


TORCH_CASES = [
    # (N, Cin, Cout, H, W, T_x, |C|, kt, kh, kw, stride, pad, dilation, p_base)
    (1, 3, 4, 5, 6, 3, 2, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), None),
    (2, 4, 3, 6, 5, 1, 2, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), None),
    (1, 5, 2, 7, 9, 2, 0, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), None),
    (1, 2, 3, 4, 4, 4, 1, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), None),
    (1, 3, 2, 9, 8, 1, 2, 3, 3, 3, (2, 2), (1, 1), (1, 1, 1), None),
    (1, 3, 3, 10, 11, 2, 2, 3, 3, 3, (2, 1), (0, 2), (1, 2, 1), None),
    (1, 2, 5, 6, 7, 1, 4, 3, 3, 3, (1, 1), (1, 1), (2, 1, 1), None),
    (1, 2, 2, 6, 7, 3, 3, 3, 3, 3, (1, 1), (1, 1), (2, 1, 1), None),
    (1, 4, 6, 5, 5, 1, 2, 3, 1, 1, (1, 1), (0, 0), (1, 1, 1), None),
    (1, 3, 3, 5, 6, 2, 3, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), None),  # |C| > p_base
    (1, 2, 3, 7, 5, 2, 1, 3, 3, 2, (1, 2), (2, 0), (1, 1, 2), None),
    (1, 3, 2, 5, 5, 2, 0, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), 1),   # p_base < d_t(kt-1)
]
# temporal stride (the encoders' downsampling): same columns + s_t
TORCH_CASES_ST = [
    (1, 3, 4, 5, 6, 4, 2, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), None, 2),
    (1, 2, 3, 4, 5, 5, 0, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), None, 2),   # odd |Z|
    (2, 3, 2, 6, 5, 3, 1, 3, 3, 3, (2, 2), (1, 1), (1, 1, 1), None, 2),
    (1, 2, 3, 5, 4, 6, 4, 3, 3, 3, (1, 1), (1, 1), (2, 1, 1), None, 2),   # d_t = 2
    (1, 4, 4, 3, 3, 7, 2, 3, 1, 1, (1, 1), (0, 0), (1, 1, 1), None, 3),   # s_t = 3, 3x1x1
    (1, 2, 2, 4, 4, 3, 0, 3, 3, 3, (1, 1), (1, 1), (1, 1, 1), 0, 2),      # p_base 0
]


def _case(ci):
    row = (TORCH_CASES + TORCH_CASES_ST)[ci]
    N, Cin, Cout, H, W, T_x, cl, kt, kh, kw, st, pd, dl, pb = row[:14]
    s_t = row[14] if len(row) > 14 else 1
    p = oracle.params(N, Cin, Cout, H, W, T_x, cl, kt=kt, kh=kh, kw=kw,
                      stride=st, pad=pd, dilation=dl, pad_t_base=pb, stride_t=s_t)
    x = _rand((N, T_x, H, W, Cin), ci, 1)
    cache = _rand((N, cl, H, W, Cin), ci, 2) if cl else None
    w = _rand((Cout, kt, kh, kw, Cin), ci, 3)
    b = _rand((Cout,), ci, 4)
    return p, x, cache, w, b


def _run_pins_torch(lib):
    for ci in range(len(TORCH_CASES) + len(TORCH_CASES_ST)):
        p, x, cache, w, b = _case(ci)
        out, nc = oracle.forward(p, x, cache, w, b, lib=lib)
        ref = _torch_reference(p, x, cache, w, b)
        assert out.shape == ref.shape, (ci, out.shape, ref.shape)
        err = np.max(np.abs(out - ref)) / max(1e-300, np.max(np.abs(ref)))
        assert err <= 1e-12, (ci, err)
        z = np.concatenate([cache, x], axis=1) if cache is not None else x
        keep = min(p.cache_keep, z.shape[1])
        assert np.array_equal(nc, z[:, z.shape[1] - keep:]), ci


def test_hand_worked_fixtures(oracle_lib):
    _run_pins_hand(oracle_lib)


def test_matches_torch_conv3d_float64(oracle_lib):
    _run_pins_torch(oracle_lib)


def test_points_match_torch(oracle_lib):
    rng = np.random.default_rng(5)
    for ci in (0, 1, 4, 5, 6, 9, len(TORCH_CASES), len(TORCH_CASES) + 2,
               len(TORCH_CASES) + 4):
        p, x, cache, w, b = _case(ci)
        ref = _torch_reference(p, x, cache, w, b)
        idx = np.stack([rng.integers(0, s, 64) for s in ref.shape], axis=1)
        vals = oracle.points(p, x, cache, w, b, idx, lib=oracle_lib)
        want = ref[tuple(idx.T)]
        assert np.max(np.abs(vals - want)) <= 1e-12 * np.max(np.abs(ref))


def test_points_reject_out_of_range(oracle_lib):
    p, x, cache, w, b = _case(0)
    with pytest.raises(ValueError):
        oracle.points(p, x, cache, w, b, np.array([[0, 99, 0, 0, 0]]))


def test_temporal_only_is_numpy_correlate(oracle_lib):
    # 3x1x1 kernel on a 1x1 image, one channel: a 1-D causal correlation.
    for d_t, cl, T_x in [(1, 2, 5), (1, 0, 4), (2, 4, 3), (2, 1, 6), (3, 6, 2)]:
        p = oracle.params(1, 1, 1, 1, 1, T_x, cl, kh=1, kw=1, pad=(0, 0),
                          dilation=(d_t, 1, 1))
        x = _rand((1, T_x, 1, 1, 1), d_t, 1)
        cache = _rand((1, cl, 1, 1, 1), d_t, 2) if cl else None
        w = _rand((1, 3, 1, 1, 1), d_t, 3)
        out, _ = oracle.forward(p, x, cache, w, None, lib=oracle_lib)
        z = np.concatenate([cache.ravel(), x.ravel()]) if cl else x.ravel()
        p_l = p.pad_t_base - cl
        zp = np.concatenate([np.zeros(max(p_l, 0)), z[max(-p_l, 0):]])
        wd = np.zeros(2 * d_t + 1)
        wd[::d_t] = w.ravel()
        ref = np.correlate(zp, wd, mode="valid")
        assert out.ravel().shape == ref.shape
        assert np.allclose(out.ravel(), ref, rtol=1e-13, atol=1e-13)


def test_single_active_tap_is_conv2d(oracle_lib):
    # |C| = 0, one frame: only the newest tap (k = kt-1) reads a real frame.
    p = oracle.params(1, 4, 5, 8, 9, 1, 0)
    x = _rand((1, 1, 8, 9, 4), 11, 1)
    w = _rand((5, 3, 3, 3, 4), 11, 3)
    b = _rand((5,), 11, 4)
    out, _ = oracle.forward(p, x, None, w, b, lib=oracle_lib)
    ref = F.conv2d(torch.from_numpy(x[:, 0]).permute(0, 3, 1, 2),
                   torch.from_numpy(w[:, 2]).permute(0, 3, 1, 2),
                   torch.from_numpy(b), padding=1)
    ref = ref.permute(0, 2, 3, 1).numpy()
    assert np.allclose(out[:, 0], ref, rtol=1e-13, atol=1e-12)


def _frame_of_z(x, cache, t):
    cl = 0 if cache is None else cache.shape[1]
    return cache[:, t] if t < cl else x[:, t - cl]


def test_per_tap_decomposition_bit_identical(oracle_lib):
    """Y = b + sum over taps k, over output frames o whose source frame
    o + k*d_t - p_l lies in Z, of conv2d(Z[source], W_k): the paper's
    decomposition, built here from torch conv2d on integer data (exact)."""
    rng = np.random.default_rng(1)
    for (cl, T_x, d_t, pb) in [(2, 1, 1, 2), (0, 3, 1, 2), (1, 2, 1, 2),
                               (4, 1, 2, 4), (2, 3, 2, 4), (3, 2, 1, 2)]:
        p = oracle.params(1, 3, 2, 6, 7, T_x, cl, dilation=(d_t, 1, 1),
                          pad_t_base=pb)
        x = _ints((1, T_x, 6, 7, 3), rng)
        cache = _ints((1, cl, 6, 7, 3), rng) if cl else None
        w = _ints((2, 3, 3, 3, 3), rng)
        b = _ints((2,), rng, -50, 50)
        out, _ = oracle.forward(p, x, cache, w, b, lib=oracle_lib)
        T_o = out.shape[1]
        p_l = pb - cl
        acc = np.zeros_like(out)
        for k in range(3):
            wk = torch.from_numpy(w[:, k]).permute(0, 3, 1, 2)
            for o in range(T_o):
                t = o + k * d_t - p_l
                if not (0 <= t < cl + T_x):
                    continue
                src = torch.from_numpy(_frame_of_z(x, cache, t)).permute(0, 3, 1, 2)
                acc[:, o] += F.conv2d(src, wk, padding=1).permute(0, 2, 3, 1).numpy()
        acc += b
        assert np.array_equal(out, acc)


def test_tap_scan_matches_conv_support(oracle_lib):
    """The scan's [o_l, o_h) per tap is exactly the set of output frames on
    which that tap's weights change the output (perturbation on the conv)."""
    for cl, T_x, d_t, pb in itertools.product(range(0, 5), range(1, 4), (1, 2), (2, 4)):
        p = oracle.params(1, 1, 1, 1, 1, T_x, cl, kh=1, kw=1, pad=(0, 0),
                          dilation=(d_t, 1, 1), pad_t_base=pb)
        T_o, _, _, _ = oracle.shape(p)
        if T_o <= 0:
            continue
        T_s, delta, o_l, o_h, active = oracle.tap_scan(p, lib=oracle_lib)
        assert T_s == T_o
        x = np.ones((1, T_x, 1, 1, 1))
        cache = np.ones((1, cl, 1, 1, 1)) if cl else None
        for k in range(3):
            w = np.zeros((1, 3, 1, 1, 1))
            w[0, k] = 1.0
            out, _ = oracle.forward(p, x, cache, w, None, lib=oracle_lib)
            support = [o for o in range(T_o) if out[0, o, 0, 0, 0] != 0]
            if active[k]:
                assert support == list(range(o_l[k], o_h[k]))
                # source interval [o_l+delta, o_h+delta) lies inside Z, same length
                assert 0 <= o_l[k] + delta[k] and o_h[k] + delta[k] <= cl + T_x
            else:
                assert support == [] and o_l[k] == o_h[k] == 0


def test_tap_scan_causal_invariant(oracle_lib):
    # With |C| <= p_l^base = d_t*(kt-1), every call returns T_x frames and
    # the newest tap is always active over all of them.
    for cl, T_x, d_t in itertools.product(range(0, 7), range(1, 7), (1, 2, 3)):
        pb = d_t * 2
        if cl > pb:
            continue
        p = oracle.params(1, 1, 1, 1, 1, T_x, cl, kh=1, kw=1, pad=(0, 0),
                          dilation=(d_t, 1, 1))
        T_o, delta, o_l, o_h, active = oracle.tap_scan(p, lib=oracle_lib)
        assert T_o == T_x
        assert active[2] and (o_l[2], o_h[2]) == (0, T_x)


def test_bias_counted_once(oracle_lib):
    rng = np.random.default_rng(2)
    for cl in (0, 1, 2):
        p = oracle.params(1, 3, 4, 5, 5, 2, cl)
        x = _ints((1, 2, 5, 5, 3), rng)
        cache = _ints((1, cl, 5, 5, 3), rng) if cl else None
        w = _ints((4, 3, 3, 3, 3), rng)
        b = _ints((4,), rng, -100, 100)
        with_b, _ = oracle.forward(p, x, cache, w, b, lib=oracle_lib)
        without, _ = oracle.forward(p, x, cache, w, None, lib=oracle_lib)
        assert np.array_equal(with_b - without, np.broadcast_to(b, with_b.shape))


@pytest.mark.parametrize("d_t,chunks", [(1, (1, 1, 1, 1, 1)), (1, (1, 4, 4, 4)),
                                         (1, (2, 1, 3)), (2, (1, 1, 1, 1, 1, 1)),
                                         (2, (3, 2, 4))])
def test_chunked_equals_whole(oracle_lib, d_t, chunks):
    """Threading new_cache between chunks reproduces whole-sequence causal
    convolution (|C| = 0 over all frames), bit-identically on integer data."""
    rng = np.random.default_rng(3)
    T = sum(chunks)
    frames = _ints((1, T, 5, 6, 2), rng)
    w = _ints((3, 3, 3, 3, 2), rng)
    b = _ints((3,), rng, -9, 9)
    p_whole = oracle.params(1, 2, 3, 5, 6, T, 0, dilation=(d_t, 1, 1))
    whole, _ = oracle.forward(p_whole, frames, None, w, b, lib=oracle_lib)
    outs, cache, t0 = [], None, 0
    for n in chunks:
        cl = 0 if cache is None else cache.shape[1]
        p = oracle.params(1, 2, 3, 5, 6, n, cl, dilation=(d_t, 1, 1))
        out, cache = oracle.forward(p, frames[:, t0:t0 + n], cache, w, b, lib=oracle_lib)
        outs.append(out)
        t0 += n
    assert np.array_equal(np.concatenate(outs, axis=1), whole)


@pytest.mark.parametrize("s_t,d_t,chunks", [(2, 1, (2, 2, 2, 2)), (2, 1, (4, 2, 6)),
                                             (2, 2, (2, 4, 2, 4)), (3, 1, (3, 6, 3))])
def test_chunked_equals_whole_temporal_stride(oracle_lib, s_t, d_t, chunks):
    """With a temporal stride, threading the cache (the last p_l^base frames)
    reproduces the whole-sequence call when every chunk boundary falls on a
    multiple of s_t frames: the next chunk's first window then starts on the
    stride grid of the whole sequence.  Bit-identical on integer data."""
    rng = np.random.default_rng(8)
    T = sum(chunks)
    frames = _ints((1, T, 4, 5, 2), rng)
    w = _ints((3, 3, 3, 3, 2), rng)
    b = _ints((3,), rng, -9, 9)
    mk = lambda n, cl: oracle.params(1, 2, 3, 4, 5, n, cl, dilation=(d_t, 1, 1), stride_t=s_t)
    whole, _ = oracle.forward(mk(T, 0), frames, None, w, b, lib=oracle_lib)
    outs, cache, t0 = [], None, 0
    for n in chunks:
        cl = 0 if cache is None else cache.shape[1]
        out, cache = oracle.forward(mk(n, cl), frames[:, t0:t0 + n], cache, w, b, lib=oracle_lib)
        outs.append(out)
        t0 += n
    assert np.array_equal(np.concatenate(outs, axis=1), whole)


def test_temporal_stride_scan_matches_conv_support(oracle_lib):
    """With s_t > 1 the scan's [o_l, o_h) per tap is still exactly the set of
    output frames a tap's weight reaches (perturbation on the conv)."""
    for cl, T_x, d_t, pb, s_t in itertools.product(range(0, 5), range(1, 7), (1, 2), (0, 2, 4),
                                                   (2, 3)):
        p = oracle.params(1, 1, 1, 1, 1, T_x, cl, kh=1, kw=1, pad=(0, 0),
                          dilation=(d_t, 1, 1), pad_t_base=pb, stride_t=s_t)
        T_o, _, _, _ = oracle.shape(p)
        if T_o <= 0:
            continue
        T_s, delta, o_l, o_h, active = oracle.tap_scan(p, lib=oracle_lib)
        assert T_s == T_o
        x = np.ones((1, T_x, 1, 1, 1))
        cache = np.ones((1, cl, 1, 1, 1)) if cl else None
        for k in range(3):
            w = np.zeros((1, 3, 1, 1, 1))
            w[0, k] = 1.0
            out, _ = oracle.forward(p, x, cache, w, None, lib=oracle_lib)
            support = [o for o in range(T_o) if out[0, o, 0, 0, 0] != 0]
            if active[k]:
                assert support == list(range(o_l[k], o_h[k]))
                assert 0 <= o_l[k] * s_t + delta[k] and (o_h[k] - 1) * s_t + delta[k] < cl + T_x
            else:
                assert support == [] and o_l[k] == o_h[k] == 0


def test_intervals_equal_length_exhaustive(oracle_lib):
    for cl, T_x, d_t, pb in itertools.product(range(0, 7), range(1, 7), (1, 2, 3), range(0, 7)):
        p = oracle.params(1, 1, 1, 1, 1, T_x, cl, kh=1, kw=1, pad=(0, 0),
                          dilation=(d_t, 1, 1), pad_t_base=pb)
        T_o, _, _, _ = oracle.shape(p)
        if T_o <= 0:
            continue
        _, delta, o_l, o_h, active = oracle.tap_scan(p, lib=oracle_lib)
        for k in range(3):
            if active[k]:
                src_l, src_h = o_l[k] + delta[k], o_h[k] + delta[k]
                assert src_h - src_l == o_h[k] - o_l[k]
                assert 0 <= src_l < src_h <= cl + T_x


# ---- post-decode uint8 quantisation ---------------------------------------
def _run_pins_quantize(lib):
    """trunc(clamp(fp32(v) * 255, 0, 255)) -- the page's expression
    (x * 255).clamp_(0, 255).to(uint8) -- pinned by closed forms, by torch's
    CPU evaluation of that expression, and exhaustively over bf16."""
    # closed forms: truncation (0.5 -> 127, not 128), clamping (no wraparound)
    special = np.array([0.0, 1.0, 0.5, 0.25, -0.1, 1.2, -3.0, 7.5, np.inf, -np.inf, np.nan,
                        254.5 / 255, 1e-30, -0.0], np.float32)
    want = np.array([0, 255, 127, 63, 0, 255, 0, 255, 255, 0, 0, 254, 0, 0], np.uint8)
    got = oracle.quantize_u8(special.astype(np.float64), lib=lib)
    assert np.array_equal(got, want), (got, want)
    # torch on random fp32 values around [0, 1], and on exact k/255 grid points
    rng = np.random.default_rng(17)
    v = np.concatenate([rng.uniform(-0.1, 1.1, 20000), np.arange(256) / 255.0,
                        (np.arange(256) + 0.5) / 255.0]).astype(np.float32)
    ref = (torch.from_numpy(v) * 255).clamp_(0, 255).to(torch.uint8).numpy()
    assert np.array_equal(oracle.quantize_u8(v.astype(np.float64), lib=lib), ref)
    # every finite bf16 value, widened exactly to fp32, multiplied in fp32
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    f = bits.float()
    f = f[torch.isfinite(f)]
    ref = (f * 255).clamp_(0, 255).to(torch.uint8).numpy()
    assert np.array_equal(oracle.quantize_u8(f.double().numpy(), lib=lib), ref)


def test_quantize_u8_pins(oracle_lib):
    _run_pins_quantize(oracle_lib)


# ---- planted mistakes: each mutant of the oracle must fail a pin ----------
MUTANTS = {
    "channel_reversed": ("acc += zrow[ci] * wrow[ci];",
                         "acc += zrow[ci] * wrow[Cin - 1 - ci];"),
    "taps_flipped": ("int t = o * p->s_t + k * p->d_t;",
                     "int t = o * p->s_t + (kt - 1 - k) * p->d_t;"),
    "temporal_stride_dropped": ("int t = o * p->s_t + k * p->d_t;",
                                "int t = o + k * p->d_t;"),
    # (a mutant that over-counts outputs would read past Zp; this one loses
    # the last output whenever tn is a multiple of s_t, e.g. |Zp| = 7, s_t = 2)
    "temporal_stride_length": ("*T_o = tn < 0 ? 0 : tn / p->s_t + 1;",
                               "*T_o = tn < 0 ? 0 : (tn + 1) / p->s_t;"),
    "pad_sign": ("int yi = y * p->s_h + r * p->d_h - p->p_h;",
                 "int yi = y * p->s_h + r * p->d_h + p->p_h;"),
    "bias_twice": ("if (bias) acc += bias[co];\n                out[",
                   "if (bias) acc += 2.0 * bias[co];\n                out["),
    "cache_ignored_in_pad": ("int p_l = p->pad_t_base - p->cache_len;\n    int zp_len = z_len + p_l;\n    if (zp_len < 0) zp_len = 0;\n    double* zp",
                             "int p_l = p->pad_t_base;\n    int zp_len = z_len + p_l - p->cache_len;\n    if (zp_len < 0) zp_len = 0;\n    double* zp"),
    "dilation_dropped": ("int xi = xo * p->s_w + s * p->d_w - p->p_w;\n                            if",
                         "int xi = xo * p->s_w + s - p->p_w;\n                            if"),
    "oldest_frames_kept": ("(z_len - keep)) * frame", "0) * frame"),
    "quantize_rounds": ("out[i] = (uint8_t)(int)y;", "out[i] = (uint8_t)(int)(y + 0.5f);"),
    "quantize_unclamped": ("y = fminf(y, 255.0f);", "y = y;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, name):
    src = open(oracle._SRC).read()
    before, after = MUTANTS[name]
    assert src.count(before) >= 1, name
    mut = tmp_path / f"mut_{name}.c"
    mut.write_text(src.replace(before, after, 1))  # first site: oracle_forward
    so = str(tmp_path / f"libmut_{name}.so")
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-fopenmp", "-std=c99",
                           str(mut), "-o", so, "-lm"])
    lib = oracle.load(so)
    caught = False
    for pin in (_run_pins_hand, _run_pins_torch, _run_pins_quantize):
        try:
            pin(lib)
        except AssertionError:
            caught = True
    assert caught, f"mutant {name} passed every pin"
