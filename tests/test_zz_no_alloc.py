"""ccv3d_forward_noalloc: the forward call for callers that may not allocate
device memory (code inside an allocator's hooks, or under a serving runtime
that owns the device-memory budget).  It must agree with ccv3d_forward on the
same inputs, call after call, while the library allocates nothing: its scratch
is a fixed array inside the shared library, reused by every such call.

This file is collected last so that a failure here does not hide any other
test; it also passes when run on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from causal_conv3d_video_b200 import ccv3d
from causal_conv3d_video_b200.workloads import Conv
import oracle
from parity_util import (TOL, assert_close, inputs_for, oracle_params, plan_env,
                         sample_indices, to_device)

pytestmark = pytest.mark.gpu


def _buffers(plan, c, seed_base):
    inp = inputs_for(c, stream_base=seed_base)
    dev = {k: to_device(v, c.dtype) for k, v in inp.items()}
    return dev


def _close(a, b, dtype):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(b * b)))
    return float(np.max(np.abs(a - b))) <= TOL[dtype] * rms


@pytest.mark.parametrize("env", [{}, {"CCV3D_HALO": 1}], ids=["default", "halo_planner"])
@pytest.mark.parametrize("c", [
    Conv("na_384ch_18x40_c2", 384, 384, 18, 40, T_x=1, cache_len=2),
    Conv("na_96ch_24x128_c1_t3", 96, 96, 24, 128, T_x=3, cache_len=1, sigma_b=0.1),
], ids=lambda c: c.name)
def test_noalloc_matches_forward_twice(c, env):
    """Two calls in a row agree with ccv3d_forward; also when the planner's
    options would pick another kernel for ccv3d_forward."""
    torch.cuda.set_device(0)
    desc = ccv3d.desc_for(c)
    with plan_env(env):
        plan = ccv3d.Plan(desc)
    for call in range(2):  # the second call reuses the scratch the first left
        with plan_env(env):
            _noalloc_vs_forward(c, desc, plan, call)


def _noalloc_vs_forward(c, desc, plan, call):
    b = _buffers(plan, c, seed_base=100 * call)
    out_ref, nc_ref = plan.alloc_outputs("cuda")
    plan.forward(b["x"], b["cache"], b["w"], b["bias"], out_ref, nc_ref)
    out, nc = plan.alloc_outputs("cuda")
    out.fill_(float("nan"))
    torch.cuda.synchronize()
    reserved = torch.cuda.memory_reserved()
    free_before = torch.cuda.mem_get_info()[0]
    rc = ccv3d.ccv3d_forward_noalloc(desc, b["x"], b["cache"], b["w"], b["bias"], out, nc,
                                     c.stride, c.pad, c.dilation)
    torch.cuda.synchronize()
    assert rc == ccv3d.CCV3D_OK
    assert torch.cuda.memory_reserved() == reserved
    if call == 1:  # the first call may load the kernel's code; later ones take nothing
        assert torch.cuda.mem_get_info()[0] == free_before
    assert bool(torch.isfinite(out.float()).all())
    assert _close(out, out_ref, c.dtype), (c.name, call)
    if nc is not None:
        assert torch.equal(nc, nc_ref)
    # and against the FP64 oracle, at sampled outputs plus the tile edges
    inp = inputs_for(c, stream_base=100 * call)
    idx = sample_indices(tuple(out.shape), plan, n_random=1500)
    ref = oracle.points(oracle_params(c), inp["x"], inp["cache"], inp["w"], inp["bias"], idx)
    got = out[tuple(torch.from_numpy(idx.T).cuda())].double().cpu().numpy()
    assert_close(got, ref, c.dtype, c.name)
    # the status word of the static array: no bounded wait ran out
    assert ccv3d.ccv3d_noalloc_get_status() == ccv3d.CCV3D_OK


def test_noalloc_refuses_what_it_cannot_hold():
    torch.cuda.set_device(0)
    # 512 output channels in one tile on every SM pair: 74 pairs x 2 x 128 x
    # 512 fp32 partial tiles (38.8 MB) exceed the fixed 32 MiB scratch array
    big = Conv("na_512ch_96x160", 384, 512, 96, 160, T_x=1, cache_len=2)
    b = _buffers(None, big, 0)
    plan = ccv3d.Plan(ccv3d.desc_for(big))
    out, nc = plan.alloc_outputs("cuda")
    with plan_env({"CCV3D_TILE_N": 512}):
        rc = ccv3d.ccv3d_forward_noalloc(ccv3d.desc_for(big), b["x"], b["cache"], b["w"],
                                         b["bias"], out, nc, big.stride, big.pad, big.dilation,
                                         check=False)
    assert rc == ccv3d.CCV3D_ERR_SCRATCH_LIMIT
    assert "scratch" in ccv3d.ccv3d_strerror(rc)
    # fp32 signatures do not run the tensor-core kernel this call wraps
    f32 = Conv("na_fp32", 16, 16, 8, 8, T_x=1, cache_len=2, dtype="fp32")
    b = _buffers(None, f32, 0)
    plan = ccv3d.Plan(ccv3d.desc_for(f32))
    out, nc = plan.alloc_outputs("cuda")
    rc = ccv3d.ccv3d_forward_noalloc(ccv3d.desc_for(f32), b["x"], b["cache"], b["w"], b["bias"],
                                     out, nc, f32.stride, f32.pad, f32.dilation, check=False)
    assert rc == ccv3d.CCV3D_ERR_UNSUPPORTED
