"""Post-decode uint8 quantisation on the device (FastVideo pull request
"Quantize frames to uint8 on-device before the post-decode D->H copy"),
bit-exact against the oracle: trunc(clamp(fp32(v) * 255, 0, 255)), NaN -> 0."""
import numpy as np
import pytest
import torch

import oracle
from causal_conv3d_video_b200 import ccv3d, synth

pytestmark = pytest.mark.gpu


def _values(n, seed):
    rng = np.random.default_rng(seed)
    v = rng.uniform(-0.2, 1.2, n).astype(np.float32)
    special = np.array([0.0, 1.0, 0.5, -0.0, np.nan, np.inf, -np.inf, 254.5 / 255, 1e-30,
                        -1e-30, 3.0, -3.0], np.float32)
    grid = (np.arange(512) / 510.0).astype(np.float32)   # k/255 and midpoints
    pool = np.concatenate([special, grid])
    k = min(n, pool.size)
    v[rng.choice(n, k, replace=False)] = pool[:k] if n else v[:0]
    return v


@pytest.mark.parametrize("n", [1, 15, 16, 17, 255, 4097, 1_000_003])
def test_fp32_bit_exact(n):
    v = _values(n, n)
    x = torch.from_numpy(v).cuda()
    out = torch.full((n,), 0xA5, dtype=torch.uint8, device="cuda")
    ccv3d.ccv3d_quantize_u8(x, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), oracle.quantize_u8(v.astype(np.float64)))


def test_bf16_every_value():
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    x = torch.cat([bits, bits.flip(0)[:4099]]).cuda()       # ragged tail, NaNs included
    out = torch.empty(x.numel(), dtype=torch.uint8, device="cuda")
    ccv3d.ccv3d_quantize_u8(x, out)
    torch.cuda.synchronize()
    want = oracle.quantize_u8(x.cpu().double().numpy())
    assert np.array_equal(out.cpu().numpy(), want)


def test_decoded_video_full_size():
    """17 decoded 720x1280 RGB frames, fp32 (the page's fp32 video), values
    around [0, 1] as a decoder's output: compared in full."""
    shape = (1, 17, 720, 1280, 3)
    v = synth.normal(shape, 0.3, 41, 1).astype(np.float32) + np.float32(0.5)
    x = torch.from_numpy(v).cuda()
    out = torch.empty(shape, dtype=torch.uint8, device="cuda")
    ccv3d.ccv3d_quantize_u8(x, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), oracle.quantize_u8(v.astype(np.float64)))


def test_refusals_on_device():
    x = torch.rand(1024, device="cuda")
    out = torch.empty(1024 + 16, dtype=torch.uint8, device="cuda")
    lib = ccv3d.lib
    # misaligned output (1 byte in), overlapping buffers, bad dtype, n < 0
    assert lib.ccv3d_quantize_u8(x.data_ptr(), ccv3d.CCV3D_FP32, out.data_ptr() + 1, 1024,
                                 None) == ccv3d.CCV3D_ERR_ALIGNMENT
    assert lib.ccv3d_quantize_u8(x.data_ptr(), ccv3d.CCV3D_FP32, x.data_ptr() + 1024, 1024,
                                 None) == ccv3d.CCV3D_ERR_ALIAS
    assert lib.ccv3d_quantize_u8(x.data_ptr(), 7, out.data_ptr(), 1024,
                                 None) == ccv3d.CCV3D_ERR_INVALID
    assert lib.ccv3d_quantize_u8(x.data_ptr(), ccv3d.CCV3D_FP32, out.data_ptr(), -1,
                                 None) == ccv3d.CCV3D_ERR_INVALID
    assert lib.ccv3d_quantize_u8(x.data_ptr(), ccv3d.CCV3D_FP32, out.data_ptr(), 0,
                                 None) == ccv3d.CCV3D_OK
    torch.cuda.synchronize()
