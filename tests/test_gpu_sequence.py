"""The synthetic 17-frame decode: 164 cached causal Conv3D calls over 28
signatures, with each module's cache threaded from one chunk to the next
(new_cache of chunk i is the cache of chunk i+1).

Checks, through the C ABI on the GPU:
  * every module's concatenated chunk outputs equal one whole-sequence call
    with an empty cache (the causal alignment the temporal-tap lowering keeps,
    Sec. 4 of "Cache-Aware Conv3D Lowering Across Embedded World-Model
    Decoders"), at a reduced 16x32 spatial size;
  * the first call of every signature against the FP64 oracle;
  * the threaded cache equals the last frames of [cache; x] at every step;
  * at full size, one steady-state call per module group at sampled outputs.
"""
import collections

import numpy as np
import pytest
import torch

import oracle
from causal_conv3d_video_b200 import ccv3d, synth, workloads
from parity_util import (TOL, assert_close, expected_new_cache, oracle_params, sample_indices,
                         to_device)

pytestmark = pytest.mark.gpu


def _module_weights(conv, module):
    seed = 7000 + module
    w = synth.tensor((conv.Cout, conv.kt, conv.kh, conv.kw, conv.Cin),
                     1.0 / np.sqrt(conv.Cin * conv.kt * conv.kh * conv.kw), seed,
                     synth.STREAM_W, conv.dtype)
    b = synth.tensor((conv.Cout,), conv.sigma_b, seed, synth.STREAM_BIAS, conv.dtype)
    return w, b


def _frames(conv, module, chunk, T):
    return synth.tensor((1, T, conv.H, conv.W, conv.Cin), 1.0, 8000 + 10 * module + chunk,
                        synth.STREAM_X, conv.dtype)


def _run(conv, x, cache, w, b):
    plan = ccv3d.Plan(ccv3d.desc_for(conv))
    out, nc = plan.alloc_outputs("cuda")
    plan.forward(x, cache, w, b, out, nc)
    return out, nc


def test_decode17_chunked_equals_whole_and_oracle():
    calls = workloads.decode17_schedule(scale_hw=(16, 32))
    assert len(calls) == 164
    by_module = collections.defaultdict(list)
    for c in calls:
        by_module[c.module].append(c)
    checked_sigs = set()
    for m, mcalls in by_module.items():
        conv0 = mcalls[0].conv
        w_np, b_np = _module_weights(conv0, m)
        w, b = to_device(w_np, conv0.dtype), to_device(b_np, conv0.dtype)
        temporal_only = conv0.kh == 1 and conv0.kw == 1
        xs, outs = [], []
        cache_dev = cache_np = None
        if temporal_only:  # chunk 0 only seeds the cache of a time-upsampling module
            x0 = _frames(conv0, m, 0, 1)
            xs.append(x0)
            cache_np = x0
            cache_dev = to_device(x0, conv0.dtype)
        for call in mcalls:
            c = call.conv
            x_np = _frames(c, m, call.chunk, c.T_x)
            xs.append(x_np)
            assert (0 if cache_np is None else cache_np.shape[1]) == c.cache_len
            out, nc = _run(c, to_device(x_np, c.dtype), cache_dev, w, b)
            torch.cuda.synchronize()
            sig = workloads.signature(c)
            if sig not in checked_sigs:
                checked_sigs.add(sig)
                ref, _ = oracle.forward(oracle_params(c), x_np, cache_np, w_np, b_np)
                assert_close(out.double().cpu().numpy(), ref, c.dtype, c.name)
            nc_np = nc.double().cpu().numpy()
            want_nc = expected_new_cache(c, {"x": x_np, "cache": cache_np})
            assert np.array_equal(nc_np, want_nc), c.name
            outs.append(out)
            cache_np, cache_dev = nc_np.astype(np.float32), nc
        # whole sequence, empty cache
        whole_x = np.concatenate(xs, axis=1)
        cw = conv0.replace(name=f"m{m}_whole", T_x=whole_x.shape[1], cache_len=0)
        whole, _ = _run(cw, to_device(whole_x, cw.dtype), None, w, b)
        torch.cuda.synchronize()
        chunked = torch.cat(outs, dim=1)
        want = whole[:, 1:] if temporal_only else whole
        assert chunked.shape == want.shape, m
        g = chunked.double().cpu().numpy()
        r = want.double().cpu().numpy()
        rms = float(np.sqrt(np.mean(r * r)))
        assert float(np.max(np.abs(g - r))) <= TOL[cw.dtype] * rms, m
    # at 16x32, groups that differ only in spatial size share a signature
    assert checked_sigs == {workloads.signature(c.conv) for c in calls}


def _steady_state_calls():
    seen, picked = set(), []
    for c in workloads.decode17_schedule():
        if c.group not in seen and c.chunk == 2:
            seen.add(c.group)
            picked.append(c)
    return picked


@pytest.mark.parametrize("call", _steady_state_calls(), ids=lambda c: f"group{c.group}")
def test_decode17_full_size_sampled(call):
    c = call.conv
    inp = synth.conv_inputs(**c.synth_kwargs())
    plan = ccv3d.Plan(ccv3d.desc_for(c))
    out, nc = plan.alloc_outputs("cuda")
    dev = {k: to_device(v, c.dtype) for k, v in inp.items()}
    plan.forward(dev["x"], dev["cache"], dev["w"], dev["bias"], out, nc)
    torch.cuda.synchronize()
    assert plan.path["tc"] is True
    assert bool(torch.isfinite(out.float()).all())
    idx = sample_indices(tuple(out.shape), plan, n_random=1500)
    ref = oracle.points(oracle_params(c), inp["x"], inp["cache"], inp["w"], inp["bias"], idx)
    got = out[tuple(torch.from_numpy(idx.T).cuda())].double().cpu().numpy()
    assert_close(got, ref, c.dtype, c.name)


@pytest.mark.parametrize("s_t,chunks", [(2, (2, 4, 2, 4)), (2, (4, 2, 2)), (3, (3, 6, 3))])
def test_temporal_stride_chunked_equals_whole(s_t, chunks):
    """Encoder-style temporal downsampling: with chunk boundaries on multiples
    of s_t, threading new_cache reproduces one whole-sequence call."""
    base = workloads.Conv("st", 64, 64, 16, 32, T_x=1, cache_len=0, stride_t=s_t)
    w_np, b_np = _module_weights(base, 90 + s_t)
    w, b = to_device(w_np, base.dtype), to_device(b_np, base.dtype)
    T = sum(chunks)
    frames = synth.tensor((1, T, base.H, base.W, base.Cin), 1.0, 9100 + s_t, synth.STREAM_X,
                          base.dtype)
    outs, cache_np, cache_dev, t0 = [], None, None, 0
    for i, n in enumerate(chunks):
        cl = 0 if cache_np is None else cache_np.shape[1]
        c = base.replace(name=f"st{s_t}_k{i}", T_x=n, cache_len=cl)
        x_np = frames[:, t0:t0 + n]
        out, nc = _run(c, to_device(x_np, c.dtype), cache_dev, w, b)
        torch.cuda.synchronize()
        if i < 2:
            ref, _ = oracle.forward(oracle_params(c), x_np, cache_np, w_np, b_np)
            assert_close(out.double().cpu().numpy(), ref, c.dtype, c.name)
        outs.append(out)
        cache_np, cache_dev = nc.double().cpu().numpy().astype(np.float32), nc
        t0 += n
    whole, _ = _run(base.replace(name="whole", T_x=T), to_device(frames, base.dtype), None, w, b)
    torch.cuda.synchronize()
    chunked = torch.cat(outs, dim=1)
    assert chunked.shape == whole.shape
    g, r = chunked.double().cpu().numpy(), whole.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(r * r)))
    assert float(np.max(np.abs(g - r))) <= TOL[base.dtype] * rms
