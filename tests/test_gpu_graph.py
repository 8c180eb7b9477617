"""CUDA-graph capture of ccv3d_forward.

A captured launch keeps the parameters it was captured with, including the
stream-K epoch of the persistent kernel; the kernel clears the flags it
consumed, so back-to-back replays must still wait for fresh split-tile
pieces.  Each replay here runs on new input contents and must equal an eager
call on the same contents bit for bit (the fix-up order is fixed).
"""
import numpy as np
import pytest
import torch

import oracle
from causal_conv3d_video_b200 import ccv3d, synth, workloads
from parity_util import GpuCall, assert_close, oracle_params

pytestmark = pytest.mark.gpu

Conv = workloads.Conv

CASES = [
    (Conv("g64_c2_t3", 64, 64, 20, 37, T_x=3, cache_len=2), {"CCV3D_PERSIST": 1, "CCV3D_SK_PAIRS": 3}),
    (Conv("g128to384", 128, 384, 12, 20, T_x=1, cache_len=2), {"CCV3D_PERSIST": 1, "CCV3D_SK_PAIRS": 5}),
    (Conv("g96_halo", 96, 96, 3, 384, T_x=2, cache_len=1), {"CCV3D_PERSIST": 0}),
    (Conv("g64_pair", 64, 64, 20, 37, T_x=1, cache_len=2), {"CCV3D_PERSIST": 0}),
]


@pytest.mark.parametrize("c,env", CASES, ids=lambda v: getattr(v, "name", None) or str(v))
def test_graph_replays_match_eager(c, env):
    inp = synth.conv_inputs(**c.synth_kwargs())
    call = GpuCall(c, inp, env=env)
    # first: an eager call against the oracle
    call.run()
    torch.cuda.synchronize()
    ref, _ = oracle.forward(oracle_params(c), inp["x"], inp["cache"], inp["w"], inp["bias"])
    assert_close(call.out_f64(), ref, c.dtype, c.name)

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call.run()
    torch.cuda.synchronize()

    replayed = []
    for seed in (11, 12, 13):  # replays back to back, new contents each time
        x = synth.tensor(call.x.shape, 1.0, seed, synth.STREAM_X, c.dtype)
        call.x.copy_(torch.from_numpy(x).to(call.x.dtype))
        graph.replay()
        torch.cuda.synchronize()
        replayed.append((x, call.out.clone(), None if call.nc is None else call.nc.clone()))
    for x, out_g, nc_g in replayed:
        call.x.copy_(torch.from_numpy(x).to(call.x.dtype))
        call.run()
        torch.cuda.synchronize()
        assert torch.equal(call.out, out_g), c.name
        if nc_g is not None:
            assert torch.equal(call.nc, nc_g), c.name
    assert not torch.equal(replayed[0][1], replayed[1][1])
    assert call.plan.status() == ccv3d.CCV3D_OK
    assert call.guards_intact()
    del graph
