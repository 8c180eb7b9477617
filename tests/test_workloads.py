"""Host checks of the synthetic workloads and the seeded generator."""
import collections

import numpy as np

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
