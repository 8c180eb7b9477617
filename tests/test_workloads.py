"""Host checks of the synthetic workloads and the seeded generator."""
import collections

import numpy as np
import pytest

from causal_conv3d_video_b200 import synth, workloads


def test_decode17_schedule_counts():
    calls = workloads.decode17_schedule()
    assert len(calls) == 164
    sigs = {workloads.signature(c.conv) for c in calls}
    assert len(sigs) == 28
    chans = {c.conv.Cin for c in calls} | {c.conv.Cout for c in calls}
    assert {16, 96, 192, 384} <= chans
    sizes = {(c.conv.H, c.conv.W) for c in calls}
    assert (90, 160) in sizes and (720, 1280) in sizes


def test_decode17_caches_thread():
    """The cache length of every call equals the frames the previous call of
    the same module keeps (min(p_l^base, |Z|)); 3x1x1 modules start with
    the frame of the chunk they skip."""
    by_mod = collections.defaultdict(list)
    for c in workloads.decode17_schedule():
        by_mod[c.module].append(c)
    for m, cs in by_mod.items():
        prev = None
        for c in cs:
            if prev is None:
                expect = 1 if c.chunk == 1 else 0
            else:
                z = prev.conv.cache_len + prev.conv.T_x
                expect = min(prev.conv.cache_keep, z)
            assert c.conv.cache_len == expect, (m, c.chunk)
            prev = c


def test_generator_deterministic_and_distributed():
    a = synth.normal((1 << 20,), 1.0, 0, 1)
    b = synth.normal((1 << 20,), 1.0, 0, 1)
    c = synth.normal((1 << 20,), 1.0, 0, 2)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert abs(a.mean()) < 5e-3 and abs(a.std() - 1) < 5e-3
    # prefix-stable: element i does not depend on the array size
    assert np.array_equal(synth.normal((1000,), 1.0, 0, 1), a[:1000])


def test_bf16_rounding_is_rne():
    import torch
    a = synth.normal((1 << 16,), 3.0, 4, 1)
    ref = torch.from_numpy(a).to(torch.bfloat16).float().numpy()
    assert np.array_equal(synth.round_to_bf16(a), ref)
    assert np.array_equal(synth.normal((1 << 16,), 3.0, 4, 1, bf16=True), ref)


def test_decode17_json_matches_schedule():
    """configs/decode17.json is the committed form of decode17_schedule()."""
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "configs", "decode17.json")
    doc = json.load(open(path))
    assert doc["calls"] == workloads.decode17_records()
    assert len(doc["calls"]) == 164
    sigs = {json.dumps({k: v for k, v in r.items() if k not in ("call", "module", "group",
                                                                 "chunk")}, sort_keys=True)
            for r in doc["calls"]}
    assert len(sigs) == 28


# per-call effective GFLOP and algorithmic MB of the decoder workloads, as the
# measurement plan tabulates them from the formulas (active taps only; Z and W
# read once, out and new_cache written once)
_TABLE = {"bf16_384ch_90x160_c2_t1": (114.7, 74.3), "bf16_384ch_90x160_c0_t1": (38.2, 41.1),
          "bf16_96ch_720x1280_c2_t4": (1834.6, 2124), "bf16_192to96_720x1280_c2_t4": (3669.2, 3540),
          "bf16_3x1x1_384to768_180x320_c2_t1": (101.9, 311),
          "bf16_192ch_dt2_180x320_c4_t1": (114.7, 223), "bf16_192ch_s2_360x640_c2_t1": (114.7, 466),
          "bf16_384ch_90x160_c1_t1": (76.4, 63.3), "bf16_192ch_89x157_c2_t1": (27.8, 34.2)}


@pytest.mark.parametrize("name", sorted(_TABLE))
def test_bench_algorithmic_flops_and_bytes(name):
    """bench.algorithmic() against the tabulated figures, and its FLOP count
    against a brute-force count of the (output frame, tap) pairs whose source
    frame lies in Z (the oracle's scan)."""
    import bench
    import oracle
    c = workloads.WORKLOADS[name]
    op = oracle.params(c.N, c.Cin, c.Cout, c.H, c.W, c.T_x, c.cache_len, kt=c.kt, kh=c.kh,
                       kw=c.kw, pad_t_base=c.pad_t_base, cache_keep=c.cache_keep,
                       stride=c.stride, pad=c.pad, dilation=c.dilation, stride_t=c.stride_t)
    T_o, H_o, W_o, _ = oracle.shape(op)
    _, delta, o_l, o_h, _ = oracle.tap_scan(op)
    iv = {"T_o": T_o, "H_o": H_o, "W_o": W_o, "o_l": o_l, "o_h": o_h}
    flops, nbytes = bench.algorithmic(c, iv)
    z = c.cache_len + c.T_x
    pairs = sum(1 for o in range(T_o) for k in range(c.kt)
                if 0 <= o * c.stride_t + k * c.dilation[0] - (c.pad_t_base - c.cache_len) < z)
    assert flops == 2.0 * c.N * c.Cout * H_o * W_o * c.Cin * c.kh * c.kw * pairs
    gf, mb = _TABLE[name]
    assert abs(flops / 1e9 - gf) <= 0.051 * max(1.0, gf / 100), (flops / 1e9, gf)
    assert abs(nbytes / 1e6 - mb) <= 0.6 + 0.001 * mb, (nbytes / 1e6, mb)


def test_bench_ring_bytes_and_legs():
    """A ring-buffer call writes only the arriving frames of the new cache:
    on the stride-2 call (|C| = 2, T_x = 1, K' = 2) one 88.5 MB frame less
    than the dense call.  The bench reports a leg for every configuration."""
    import bench
    c = workloads.C4_STRIDE
    iv = {"T_o": 1, "H_o": 180, "W_o": 320, "o_l": [0, 0, 0], "o_h": [1, 1, 1]}
    _, dense = bench.algorithmic(c, iv)
    ring = bench.ring_algorithmic_bytes(c, iv, dense)
    assert dense - ring == 2 * 360 * 640 * 192
    c3 = workloads.C3  # T_x = 4 >= K' = 2: both kept frames arrive with the call
    iv3 = {"T_o": 4, "H_o": 720, "W_o": 1280, "o_l": [0] * 3, "o_h": [4] * 3}
    _, d3 = bench.algorithmic(c3, iv3)
    assert bench.ring_algorithmic_bytes(c3, iv3, d3) == d3
    names = {n for n, _, _ in bench.bench_legs()}
    for w in (workloads.C1, workloads.C2, workloads.C2_EMPTY, workloads.C3, workloads.C3B,
              workloads.C4_TIME, workloads.C4_DIL, workloads.C4_STRIDE, workloads.C4_C1,
              workloads.C4_ODD, workloads.C6_ST2, workloads.C6_ST2_TIME, workloads.C_RGB):
        assert w.name in names
    assert workloads.C4_STRIDE.name + "+ring" in names
