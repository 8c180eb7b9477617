"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle runs.

This module only draws random numbers: it holds none of the convolution's
arithmetic and imports neither the CUDA binding nor the oracle.

Generator (one counter-based stream per tensor):
  * splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014) as a mixing function over a counter,
  * Box-Muller (Box & Muller, 1958) on two 53-bit uniforms, in double,
  * scaled by sigma, rounded to float32, and -- for bf16 workloads -- rounded
    to the nearest bfloat16 (ties to even) so that the same values feed the
    GPU (as bf16) and the oracle (widened to double) exactly.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_STREAM_MUL = 0xD1B54A32D192ED03
_CHUNK = 1 << 22

# Per-tensor substreams.
STREAM_X, STREAM_CACHE, STREAM_W, STREAM_BIAS = 1, 2, 3, 4


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        k = np.uint64((seed ^ (stream * _STREAM_MUL)) & 0xFFFFFFFFFFFFFFFF)
        return _mix(np.array([k], np.uint64))[0]


def _fill(out, lo, hi, key, sigma, bf16=False):
    with np.errstate(over="ignore"):
        i = np.arange(lo, hi, dtype=np.uint64)
        c1 = key + (np.uint64(2) * i + np.uint64(1)) * _GAMMA
        c2 = key + (np.uint64(2) * i + np.uint64(2)) * _GAMMA
        u1 = ((_mix(c1) >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0**-53
        u2 = (_mix(c2) >> np.uint64(11)).astype(np.float64) * 2.0**-53
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
        out[lo:hi] = (z * sigma).astype(np.float32)
        if bf16:
            out[lo:hi] = round_to_bf16(out[lo:hi])


def normal(shape, sigma: float, seed: int, stream: int, bf16: bool = False) -> np.ndarray:
    """N(0, sigma^2) samples as float32, element i of the C-order array drawn
    from counters 2i+1 and 2i+2 of the (seed, stream) key.  Large arrays are
    filled chunk by chunk on a thread pool (the values do not depend on it)."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, np.float32)
    key = stream_key(seed, stream)
    chunks = [(lo, min(n, lo + _CHUNK)) for lo in range(0, n, _CHUNK)]
    if len(chunks) <= 1:
        for lo, hi in chunks:
            _fill(out, lo, hi, key, sigma, bf16)
    else:
        workers = min(len(chunks), max(1, (os.cpu_count() or 1)))
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(lambda c: _fill(out, c[0], c[1], key, sigma, bf16), chunks))
    return out.reshape(shape)


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returned
    as float32 holding bf16-representable values.  Inputs are finite (their
    bit patterns plus the rounding increment stay below 2**32)."""
    a = np.ascontiguousarray(a, np.float32)
    u = a.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32).reshape(a.shape)


def tensor(shape, sigma, seed, stream, dtype: str) -> np.ndarray:
    return normal(shape, sigma, seed, stream, bf16=(dtype == "bf16"))


def conv_inputs(*, N, Cin, Cout, H, W, T_x, cache_len, kt=3, kh=3, kw=3,
                dtype="bf16", seed=0, sigma_x=1.0, sigma_w=None,
                sigma_b=0.02, has_bias=True, stream_base=0):
    """Inputs of one cached causal Conv3D call, NTHWC, as float32 arrays.

    sigma_w defaults to 1/sqrt(Cin*kt*kh*kw): the "N(0, 1/(Cin*27))" weight
    recipe read as a variance.  The cache is drawn from its own stream with
    the activations' sigma.
    """
    if sigma_w is None:
        sigma_w = 1.0 / np.sqrt(Cin * kt * kh * kw)
    b = stream_base
    x = tensor((N, T_x, H, W, Cin), sigma_x, seed, b + STREAM_X, dtype)
    cache = (tensor((N, cache_len, H, W, Cin), sigma_x, seed, b + STREAM_CACHE, dtype)
             if cache_len > 0 else None)
    w = tensor((Cout, kt, kh, kw, Cin), sigma_w, seed, b + STREAM_W, dtype)
    bias = tensor((Cout,), sigma_b, seed, b + STREAM_BIAS, dtype) if has_bias else None
    return {"x": x, "cache": cache, "w": w, "bias": bias}
