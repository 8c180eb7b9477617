"""FP64 CPU oracle for the cached causal Conv3D -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python binding
never import it; the two share no code.

The arithmetic lives in ``ccv3d_oracle.c`` (plain C, double accumulation,
OpenMP over output rows).  This module compiles it with gcc into
``oracle/_build/libccv3d_oracle.so`` and marshals numpy arrays to it.

Definition followed ("Cache-Aware Conv3D Lowering Across Embedded World-Model
Decoders", Sec. 4): Z = [C; X] along time, effective left pad
p_l = p_l^base - |C|, PyTorch cross-correlation with unit temporal stride,
out-of-range frames and pixels contribute zero, bias added exactly once.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ccv3d_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libccv3d_oracle.so")
_lock = threading.Lock()
_lib = None


class OracleParams(ctypes.Structure):
    """Mirror of ``oracle_params`` in ccv3d_oracle.c (oracle-private)."""

    _fields_ = [(n, ctypes.c_int) for n in (
        "N", "Cin", "Cout", "kt", "kh", "kw", "H", "W", "T_x", "cache_len",
        "pad_t_base", "cache_keep", "s_h", "s_w", "p_h", "p_w", "d_t", "d_h",
        "d_w", "s_t")]


def build(src: str = _SRC, out: str = _LIB_PATH, force: bool = False) -> str:
    """Compile the oracle C file into a shared library (gcc, -O2, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp",
                           "-std=c99", src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building first if needed) and return the ctypes library."""
    global _lib
    with _lock:
        if path is not None:
            return _bind(ctypes.CDLL(path))
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _bind(lib):
    P = ctypes.POINTER(OracleParams)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    lib.oracle_shape.argtypes = [P, ip, ip, ip, ip]
    lib.oracle_forward.argtypes = [P, dp, dp, dp, dp, dp, dp]
    lib.oracle_points.argtypes = [P, dp, dp, dp, dp,
                                  ctypes.POINTER(ctypes.c_longlong),
                                  ctypes.c_longlong, dp]
    lib.oracle_tap_scan.argtypes = [P, ip, ip, ip, ip, ip]
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = ctypes.c_int
    lib.oracle_quantize_u8.argtypes = [dp, ctypes.c_longlong, ctypes.POINTER(ctypes.c_uint8)]
    lib.oracle_quantize_u8.restype = ctypes.c_int
    for f in (lib.oracle_shape, lib.oracle_forward, lib.oracle_points,
              lib.oracle_tap_scan):
        f.restype = ctypes.c_int
    return lib


def params(N, Cin, Cout, H, W, T_x, cache_len, *, kt=3, kh=3, kw=3,
           pad_t_base=None, cache_keep=None, stride=(1, 1), pad=(1, 1),
           dilation=(1, 1, 1), stride_t=1) -> OracleParams:
    """Build an OracleParams.  pad_t_base defaults to d_t*(kt-1) and
    cache_keep to pad_t_base; stride is (s_h, s_w), stride_t the temporal
    stride."""
    d_t, d_h, d_w = dilation
    if pad_t_base is None:
        pad_t_base = d_t * (kt - 1)
    if cache_keep is None:
        cache_keep = pad_t_base
    return OracleParams(N, Cin, Cout, kt, kh, kw, H, W, T_x, cache_len,
                        pad_t_base, cache_keep, stride[0], stride[1], pad[0],
                        pad[1], d_t, d_h, d_w, stride_t)


def _dptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=np.float64)


def shape(p: OracleParams):
    """(T_o, H_o, W_o, K') from the convolution length formula on Zp."""
    lib = load()
    v = [ctypes.c_int() for _ in range(4)]
    rc = lib.oracle_shape(ctypes.byref(p), *[ctypes.byref(t) for t in v])
    if rc != 0:
        raise ValueError("oracle_shape: invalid parameters")
    return tuple(t.value for t in v)


def forward(p: OracleParams, x, cache, w, bias, lib=None):
    """Direct FP64 cached causal Conv3D.

    x [N,T_x,H,W,Cin], cache [N,|C|,H,W,Cin] or None, w [Cout,kt,kh,kw,Cin],
    bias [Cout] or None.  Returns (out [N,T_o,H_o,W_o,Cout], new_cache
    [N,K',H,W,Cin]) as float64 arrays.
    """
    lib = lib or load()
    T_o, H_o, W_o, keep = shape(p)
    x, cache, w, bias = _f64(x), _f64(cache), _f64(w), _f64(bias)
    _check(p, x, cache, w, bias)
    out = np.zeros((p.N, T_o, H_o, W_o, p.Cout), np.float64)
    nc = np.zeros((p.N, keep, p.H, p.W, p.Cin), np.float64)
    rc = lib.oracle_forward(ctypes.byref(p), _dptr(x),
                            _dptr(cache) if p.cache_len > 0 else None,
                            _dptr(w), _dptr(bias), _dptr(out), _dptr(nc))
    if rc != 0:
        raise RuntimeError(f"oracle_forward failed ({rc})")
    return out, nc


def points(p: OracleParams, x, cache, w, bias, idx, lib=None):
    """Evaluate the definition at the (n, o, y, x, co) rows of ``idx``."""
    lib = lib or load()
    x, cache, w, bias = _f64(x), _f64(cache), _f64(w), _f64(bias)
    _check(p, x, cache, w, bias)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 5)
    vals = np.zeros(idx.shape[0], np.float64)
    rc = lib.oracle_points(ctypes.byref(p), _dptr(x),
                           _dptr(cache) if p.cache_len > 0 else None,
                           _dptr(w), _dptr(bias),
                           idx.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)),
                           idx.shape[0], _dptr(vals))
    if rc != 0:
        raise ValueError("oracle_points: index outside the output")
    return vals


def tap_scan(p: OracleParams, lib=None):
    """Brute-force per-tap scan: (T_o, delta, o_l, o_h, active) lists."""
    lib = lib or load()
    kt = p.kt
    T_o = ctypes.c_int()
    arrs = [(ctypes.c_int * kt)() for _ in range(4)]
    rc = lib.oracle_tap_scan(ctypes.byref(p), ctypes.byref(T_o), *arrs)
    if rc != 0:
        raise RuntimeError("oracle_tap_scan: invalid parameters or gap")
    return (T_o.value,) + tuple(list(a) for a in arrs)


def _check(p, x, cache, w, bias):
    if x.shape != (p.N, p.T_x, p.H, p.W, p.Cin):
        raise ValueError(f"x shape {x.shape}")
    if p.cache_len > 0 and (cache is None or cache.shape != (
            p.N, p.cache_len, p.H, p.W, p.Cin)):
        raise ValueError("cache shape")
    if w.shape != (p.Cout, p.kt, p.kh, p.kw, p.Cin):
        raise ValueError(f"w shape {w.shape}")
    if bias is not None and bias.shape != (p.Cout,):
        raise ValueError("bias shape")


def quantize_u8(values, lib=None) -> np.ndarray:
    """uint8 frames from decoded values (fp32 or bf16 numbers given as any
    float array): trunc(clamp(fp32(v) * 255, 0, 255)), NaN -> 0."""
    v = np.ascontiguousarray(np.asarray(values, np.float64))
    out = np.zeros(v.shape, np.uint8)
    (lib or load()).oracle_quantize_u8(
        v.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), v.size,
        out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    return out


def threads(lib=None) -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int((lib or load()).oracle_threads())


def metrics(got, ref):
    """Agreement metrics with FP64 accumulation: max/mean |diff|, RMSE,
    rms(ref), cosine, NaN/Inf count of ``got``."""
    g = np.asarray(got, np.float64).ravel()
    r = np.asarray(ref, np.float64).ravel()
    d = g - r
    nonfinite = int(np.count_nonzero(~np.isfinite(g)))
    denom = float(np.linalg.norm(g) * np.linalg.norm(r))
    return {
        "max_abs": float(np.max(np.abs(d))) if d.size else 0.0,
        "mean_abs": float(np.mean(np.abs(d))) if d.size else 0.0,
        "rmse": float(np.sqrt(np.mean(d * d))) if d.size else 0.0,
        "rms_ref": float(np.sqrt(np.mean(r * r))) if r.size else 0.0,
        "cosine": float(np.dot(g, r) / denom) if denom > 0 else 1.0,
        "nonfinite": nonfinite,
    }
