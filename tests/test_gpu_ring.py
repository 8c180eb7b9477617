"""Ring-buffer caches (ccv3d_forward_ring): the cache of the cache-augmented
input Z = [C; X] (Sec. 4 of "Cache-Aware Conv3D Lowering Across Embedded
World-Model Decoders") carried from chunk to chunk in place, each call writing
only the frames of the new cache that arrive with it.

Checked through the C ABI on the GPU, call by call, against
  * the dense path (ccv3d_forward with ping-pong new_cache buffers) on the same
    plan: outputs bit-identical, the ring's live slots equal to new_cache;
  * the FP64 oracle on the same inputs.
Cases: the 164-call synthetic decode at 16x32; ring sizes from the minimum
|C| + n_w upwards with the head wrapping; every kernel form (pair, persistent
with split tiles, halo, frame-pair, single CTA, thin output, SIMT fp32 and
bf16); the
full-size stride-2 call.
"""
import collections

import numpy as np
import pytest
import torch

import oracle
from causal_conv3d_video_b200 import ccv3d, synth, workloads
from causal_conv3d_video_b200.workloads import Conv
from parity_util import (assert_close, oracle_params, plan_env, sample_indices, to_device,
                         torch_dtype)

pytestmark = pytest.mark.gpu


class RingStream:
    """One module's cache threaded two ways: a ring of `slots` frames and dense
    ping-pong new_cache buffers (the reference path)."""

    def __init__(self, conv, slots, head, w, b):
        self.c0, self.slots, self.head = conv, slots, head
        self.w, self.b = w, b
        self.ring = torch.full((conv.N, slots, conv.H, conv.W, conv.Cin), -7.0,
                               dtype=torch_dtype(conv.dtype), device="cuda")
        self.dense = None     # device new_cache of the previous call
        self.cache_np = None  # the same, on the host (oracle input)

    def seed(self, x_np):
        """A frame that only seeds the cache (time-upsampling modules' chunk 0)."""
        x = to_device(x_np, self.c0.dtype)
        for t in range(x.shape[1]):
            self.ring[:, (self.head + t) % self.slots] = x[:, t]
        self.dense, self.cache_np = x, x_np

    def step(self, c, x_np, env=None, check_oracle=True):
        with plan_env(env or {}):
            plan = ccv3d.Plan(ccv3d.desc_for(c))
        assert c.cache_len == (0 if self.cache_np is None else self.cache_np.shape[1])
        x = to_device(x_np, c.dtype)
        out_d, nc_d = plan.alloc_outputs("cuda")
        plan.forward(x, self.dense, self.w, self.b, out_d, nc_d)
        out_r, _ = plan.alloc_outputs("cuda")
        out_r.fill_(float("nan"))
        before = self.ring.clone()
        new_head = plan.forward_ring(x, self.ring, self.slots, self.head, self.w, self.b, out_r)
        torch.cuda.synchronize()
        assert plan.status() == ccv3d.CCV3D_OK
        assert torch.equal(out_r, out_d), c.name          # same kernel, same order
        keep = plan.sizes["new_cache_frames"]
        writes = plan.ring_writes()
        assert new_head == (self.head + c.cache_len + writes - keep) % self.slots
        for t in range(keep):                               # live slots == new_cache
            assert torch.equal(self.ring[:, (new_head + t) % self.slots], nc_d[:, t]), (c.name, t)
        written = {(self.head + c.cache_len + i) % self.slots for i in range(writes)}
        for s in range(self.slots):                         # nothing else was touched
            if s not in written:
                assert torch.equal(self.ring[:, s], before[:, s]), (c.name, s)
        if check_oracle:
            ref, _ = oracle.forward(oracle_params(c), x_np, self.cache_np,
                                    self.w.double().cpu().numpy(), None if self.b is None
                                    else self.b.double().cpu().numpy())
            assert_close(out_r.double().cpu().numpy(), ref, c.dtype, c.name)
        self.head = new_head
        self.dense = nc_d
        self.cache_np = nc_d.double().cpu().numpy().astype(np.float32)
        return plan, out_r


def _weights(conv, seed):
    w = synth.tensor((conv.Cout, conv.kt, conv.kh, conv.kw, conv.Cin),
                     1.0 / np.sqrt(conv.Cin * conv.kt * conv.kh * conv.kw), seed,
                     synth.STREAM_W, conv.dtype)
    b = synth.tensor((conv.Cout,), conv.sigma_b, seed, synth.STREAM_BIAS, conv.dtype)
    return to_device(w, conv.dtype), to_device(b, conv.dtype)


def _frames(conv, seed, T):
    return synth.tensor((conv.N, T, conv.H, conv.W, conv.Cin), 1.0, seed, synth.STREAM_X,
                        conv.dtype)


def test_decode17_ring_equals_ping_pong_and_oracle():
    """Every module of the 164-call decode threads its cache through a ring of
    cache_keep + (largest chunk) slots, starting at a wrapping head."""
    calls = workloads.decode17_schedule(scale_hw=(16, 32))
    by_module = collections.defaultdict(list)
    for c in calls:
        by_module[c.module].append(c)
    n = 0
    for m, mcalls in by_module.items():
        c0 = mcalls[0].conv
        w, b = _weights(c0, 7000 + m)
        slots = c0.cache_keep + max(c.conv.T_x for c in mcalls)
        rs = RingStream(c0, slots, slots - 1, w, b)
        if c0.kh == 1 and c0.kw == 1:
            rs.seed(_frames(c0, 8000 + 10 * m, 1))
        for call in mcalls:
            rs.step(call.conv, _frames(call.conv, 8000 + 10 * m + call.chunk, call.conv.T_x))
            n += 1
    assert n == 164


RING_SIGS = [
    # (signature, planner overrides): every kernel form the planner can pick
    (Conv("r64_pair", 64, 64, 20, 37, T_x=1, cache_len=0), {"CCV3D_PERSIST": 0}),
    (Conv("r64_persist_split", 64, 64, 20, 37, T_x=1, cache_len=0),
     {"CCV3D_PERSIST": 1, "CCV3D_SK_PAIRS": 3}),
    (Conv("r64_single", 64, 64, 20, 37, T_x=1, cache_len=0), {"CCV3D_PAIR": 0, "CCV3D_PERSIST": 0}),
    (Conv("r96_halo", 96, 96, 3, 384, T_x=1, cache_len=0, sigma_b=0.1),
     {"CCV3D_HALO": 1, "CCV3D_PERSIST": 0, "CCV3D_FUSE": 0}),
    (Conv("r96_fused_t3", 96, 96, 3, 256, T_x=3, cache_len=0, sigma_b=0.1),
     {"CCV3D_PERSIST": 0, "CCV3D_FUSE": 1}),
    (Conv("r96_fused_persist_t3", 96, 96, 3, 256, T_x=3, cache_len=0, sigma_b=0.1),
     {"CCV3D_PERSIST": 0, "CCV3D_FUSE": 1, "CCV3D_FUSED_PERSIST": 1}),
    (Conv("r96_fused_persist2_t3", 96, 96, 3, 256, T_x=3, cache_len=0, sigma_b=0.1),
     {"CCV3D_PERSIST": 0, "CCV3D_FUSE": 1, "CCV3D_FUSED_PERSIST": 2}),
    (Conv("r64_dt2", 64, 64, 18, 32, T_x=1, cache_len=0, dilation=(2, 1, 1)), {}),
    (Conv("r32_batch2_t2", 32, 48, 10, 12, T_x=2, cache_len=0, N=2), {}),
    (Conv("r16_fp32", 16, 16, 16, 16, T_x=3, cache_len=0, dtype="fp32", sigma_b=0.1), {}),
    (Conv("r8_fp32_t1", 8, 12, 13, 17, T_x=1, cache_len=0, dtype="fp32"), {}),
    (Conv("r_thin_bf16", 3, 16, 12, 12, T_x=2, cache_len=0), {}),
    (Conv("r_thin_out_t2", 32, 3, 10, 140, T_x=2, cache_len=0, sigma_b=0.1), {"CCV3D_THIN": 1}),
]


@pytest.mark.parametrize("extra", [0, 1, 3], ids=lambda e: f"slots+{e}")
@pytest.mark.parametrize("sig,env", RING_SIGS, ids=lambda v: getattr(v, "name", None) or "env")
def test_ring_chunks_every_kernel(sig, env, extra):
    """Six chunks, from the empty cache to the steady state, on a ring of the
    minimum size (|C| + n_w) plus `extra` slots, with the head wrapping."""
    K = sig.cache_keep
    slots = K + min(K, sig.T_x) + extra
    w, b = _weights(sig, 500 + slots)
    rs = RingStream(sig, slots, slots - 1, w, b)
    seen = 0
    kernels = set()
    for chunk in range(6):
        c = sig.replace(name=f"{sig.name}_k{chunk}", cache_len=min(seen, K))
        plan, _ = rs.step(c, _frames(c, 600 + 10 * slots + chunk, c.T_x), env=env,
                          check_oracle=chunk < 4)
        kernels.add(plan.kernel)
        seen += c.T_x
    # the override that forces a kernel form (key, value) -> the form
    forced = {("CCV3D_PAIR", 0): "tc_single", ("CCV3D_HALO", 1): "tc_pair_halo",
              ("CCV3D_PERSIST", 1): "tc_persistent", ("CCV3D_THIN", 1): "tc_thin"}
    if env.get("CCV3D_FUSE") == 1:
        forced[("CCV3D_FUSE", 1)] = ("tc_pair_fused_persistent" if env.get("CCV3D_FUSED_PERSIST")
                                     else "tc_pair_fused")
    for (k, v), name in forced.items():
        if env.get(k) == v:
            assert kernels == {name}, (sig.name, kernels)


def test_ring_full_size_stride2():
    """The full-size stride-2 call (192 ch, 360x640 -> 180x320, |C| = 2) on a
    3-slot ring whose cache wraps: out equal to the dense call and, at sampled
    outputs, to the oracle; the one frame written is x."""
    c = workloads.C4_STRIDE
    inp = synth.conv_inputs(**c.synth_kwargs())
    dev = {k: to_device(v, c.dtype) for k, v in inp.items()}
    plan = ccv3d.Plan(ccv3d.desc_for(c))
    slots, head = 3, 2
    ring = torch.zeros((1, slots, c.H, c.W, c.Cin), dtype=torch.bfloat16, device="cuda")
    ring[:, 2] = dev["cache"][:, 0]
    ring[:, 0] = dev["cache"][:, 1]
    out_d, nc_d = plan.alloc_outputs("cuda")
    plan.forward(dev["x"], dev["cache"], dev["w"], dev["bias"], out_d, nc_d)
    out_r, _ = plan.alloc_outputs("cuda")
    new_head = plan.forward_ring(dev["x"], ring, slots, head, dev["w"], dev["bias"], out_r)
    torch.cuda.synchronize()
    assert plan.status() == ccv3d.CCV3D_OK
    assert new_head == 0
    assert torch.equal(out_r, out_d)
    assert torch.equal(ring[:, 1], dev["x"][:, 0])          # the arriving frame
    assert torch.equal(ring[:, 0], nc_d[:, 0]) and torch.equal(ring[:, 1], nc_d[:, 1])
    idx = sample_indices(tuple(out_r.shape), plan, n_random=1500)
    ref = oracle.points(oracle_params(c), inp["x"], inp["cache"], inp["w"], inp["bias"], idx)
    got = out_r[tuple(torch.from_numpy(idx.T).cuda())].double().cpu().numpy()
    assert_close(got, ref, c.dtype, c.name)
    st = plan.stats()
    assert st["calls"] == 2 and st["errors"] == 0


def test_ring_refusals_on_device():
    c = Conv("r_ref", 32, 32, 10, 12, T_x=1, cache_len=2)
    plan = ccv3d.Plan(ccv3d.desc_for(c))
    w, b = _weights(c, 1)
    x = to_device(_frames(c, 2, 1), c.dtype)
    ring = torch.zeros((1, 3, c.H, c.W, c.Cin), dtype=torch.bfloat16, device="cuda")
    out, _ = plan.alloc_outputs("cuda")
    f = lambda **kw: ccv3d.ccv3d_forward_ring(
        plan.handle, kw.get("x", x), kw.get("ring", ring), kw.get("slots", 3), kw.get("head", 0),
        w, b, kw.get("out", out), plan.stride, plan.pad, plan.dilation, check=False)[0]
    assert f(slots=2) == ccv3d.CCV3D_ERR_INVALID
    assert f(head=3) == ccv3d.CCV3D_ERR_INVALID
    assert f(x=ring[:, 1]) == ccv3d.CCV3D_ERR_ALIAS
    assert f() == ccv3d.CCV3D_OK
    torch.cuda.synchronize()
    st = plan.stats()
    assert st["calls"] == 1 and st["errors"] == 3
    assert plan.status_stream() == ccv3d.CCV3D_OK
