"""Shared helpers for the GPU parity tests: run one call through the C ABI and
compare it with the FP64 oracle on the same seeded inputs."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from causal_conv3d_video_b200 import ccv3d, synth

# Tolerances of the contract: max|gpu - oracle| <= TOL * rms(oracle).
TOL = {"bf16": 2e-2, "fp32": 1e-4}


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def oracle_params(c):
    return oracle.params(c.N, c.Cin, c.Cout, c.H, c.W, c.T_x, c.cache_len, kt=c.kt,
                         kh=c.kh, kw=c.kw, pad_t_base=c.pad_t_base,
                         cache_keep=c.cache_keep, stride=c.stride, pad=c.pad,
                         dilation=c.dilation, stride_t=c.stride_t)


def inputs_for(c, stream_base=0):
    return synth.conv_inputs(**c.synth_kwargs(), stream_base=stream_base)


def to_device(a, dtype):
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch_dtype(dtype)).cuda()


class plan_env:
    """Temporarily set CCV3D_* planner overrides (read at plan time only, and
    only with CCV3D_TEST_OVERRIDES=1, which this sets too)."""

    def __init__(self, env):
        self.env = dict(env)
        if self.env:
            self.env["CCV3D_TEST_OVERRIDES"] = 1

    def __enter__(self):
        self.old = {k: os.environ.get(k) for k in self.env}
        os.environ.update({k: str(v) for k, v in self.env.items()})

    def __exit__(self, *exc):
        for k, v in self.old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


class GpuCall:
    """One plan + device buffers (with guard bands around the outputs)."""

    GUARD = 256  # elements of sentinel before and after each output

    def __init__(self, c, inp, force_simt=False, env=None):
        self.c = c
        env = dict(env or {})
        if force_simt:
            env["CCV3D_FORCE_PATH"] = "simt"
        with plan_env(env):
            self.plan = ccv3d.Plan(ccv3d.desc_for(c))
        dt = c.dtype
        self.x = to_device(inp["x"], dt)
        self.cache = to_device(inp["cache"], dt)
        self.w = to_device(inp["w"], dt)
        self.bias = to_device(inp["bias"], dt)
        g = self.GUARD
        n_out = int(np.prod(self.plan.out_shape()))
        n_nc = int(np.prod(self.plan.new_cache_shape()))
        self.sentinel = -12345.0 if dt == "fp32" else -12288.0  # exact in bf16
        self.out_buf = torch.full((n_out + 2 * g,), self.sentinel, dtype=torch_dtype(dt),
                                  device="cuda")
        self.nc_buf = torch.full((n_nc + 2 * g,), self.sentinel, dtype=torch_dtype(dt),
                                 device="cuda")
        self.out = self.out_buf[g:g + n_out].view(self.plan.out_shape())
        self.nc = self.nc_buf[g:g + n_nc].view(self.plan.new_cache_shape()) if n_nc else None

    def run(self, stream=None):
        self.plan.forward(self.x, self.cache, self.w, self.bias, self.out, self.nc, stream)
        return self

    def guards_intact(self) -> bool:
        g = self.GUARD
        ok = True
        for buf in (self.out_buf, self.nc_buf):
            ok &= bool((buf[:g] == self.sentinel).all()) and bool((buf[-g:] == self.sentinel).all())
        return ok

    def out_f64(self):
        return self.out.double().cpu().numpy()

    def nc_f64(self):
        return None if self.nc is None else self.nc.double().cpu().numpy()


def assert_close(got, ref, dtype, what=""):
    m = oracle.metrics(got, ref)
    tol = TOL[dtype] * m["rms_ref"]
    assert m["nonfinite"] == 0, (what, m)
    assert m["max_abs"] <= tol, (what, m, tol)
    return m


def expected_new_cache(c, inp):
    """The last min(cache_keep, |Z|) frames of Z = [cache; x], from the inputs."""
    z = inp["x"] if inp["cache"] is None else np.concatenate([inp["cache"], inp["x"]], axis=1)
    keep = min(c.cache_keep, z.shape[1])
    return z[:, z.shape[1] - keep:].astype(np.float64)


def sample_indices(out_shape, plan, n_random=3000, seed=0):
    """Random output positions plus the edges of the image and of the tiles."""
    N, T_o, H_o, W_o, Cout = out_shape
    rng = np.random.default_rng(seed)
    idx = [rng.integers(0, s, n_random) for s in out_shape]
    pts = [np.stack(idx, axis=1)]
    tn = plan.path["tile_n"] or Cout
    ys = sorted({0, 1, H_o // 2, H_o - 2, H_o - 1} & set(range(H_o)))
    xs = sorted({0, 1, 31, 32, 63, 64, W_o // 2, W_o - 2, W_o - 1} & set(range(W_o)))
    cos = sorted({0, 1, 15, 16, tn - 1, tn, Cout // 2, Cout - 1} & set(range(Cout)))
    grid = np.array([(n, o, y, x, co) for n in range(N) for o in range(T_o) for y in ys
                     for x in xs for co in cos], dtype=np.int64)
    pts.append(grid)
    return np.concatenate(pts, axis=0)
