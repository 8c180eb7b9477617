"""ctypes binding of libccv3d (include/ccv3d.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  Device
buffers are passed as torch tensors (their data pointers) or as raw integer
addresses; nothing is computed in Python.  If the shared library is missing
the import of this module fails loudly: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# CCV3D_LIBRARY=checked loads the bounds-checked build (libccv3d_checked.so:
# the same ABI, every computed device address range-checked); the tests use it
LIB_PATH = os.path.join(_HERE, "_lib", "libccv3d_checked.so"
                        if os.environ.get("CCV3D_LIBRARY") == "checked" else "libccv3d.so")

CCV3D_BF16, CCV3D_FP32 = 0, 1
STATUS = {0: "CCV3D_OK", 1: "CCV3D_ERR_INVALID", 2: "CCV3D_ERR_UNSUPPORTED",
          3: "CCV3D_ERR_EMPTY_OUTPUT", 4: "CCV3D_ERR_ALIGNMENT", 5: "CCV3D_ERR_ALIAS",
          6: "CCV3D_ERR_CUDA", 7: "CCV3D_ERR_TIMEOUT", 8: "CCV3D_ERR_SCRATCH_LIMIT",
          9: "CCV3D_ERR_BOUNDS"}
for _code, _name in STATUS.items():
    globals()[_name] = _code
CCV3D_MAX_KT = 3

# every symbol include/ccv3d.h declares
EXPORTED = ("ccv3d_plan", "ccv3d_plan_intervals", "ccv3d_plan_path", "ccv3d_forward",
            "ccv3d_get_stats", "ccv3d_get_status", "ccv3d_destroy", "ccv3d_strerror",
            "ccv3d_plan_sizes", "ccv3d_selftest_wait_timeout", "ccv3d_forward_noalloc",
            "ccv3d_plan_kernel", "ccv3d_plan_tiling", "ccv3d_quantize_u8",
            "ccv3d_get_status_stream", "ccv3d_noalloc_get_status", "ccv3d_forward_ring",
            "ccv3d_selftest_bounds")
CCV3D_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class ccv3d_desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "N", "Cin", "Cout", "kt", "kh", "kw", "H", "W", "T_x", "cache_len",
        "pad_t_base", "cache_keep", "stride_t", "stride_h", "stride_w", "pad_h",
        "pad_w", "dil_t", "dil_h", "dil_w", "groups", "dtype", "has_bias")]


class ccv3d_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "calls", "tc_path", "simt_path", "unsupported", "errors", "workspace_bytes",
        "plans_unsupported")]


class CCV3DError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({ccv3d_strerror(status)})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libccv3d.so not built ({LIB_PATH}); run "
            "`python -m causal_conv3d_video_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, ip, i3 = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int), ctypes.c_int * 3
    lib.ccv3d_plan.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(ccv3d_desc)]
    lib.ccv3d_plan_intervals.argtypes = [vp, ip, ip, ip, ip, ip, ip]
    lib.ccv3d_plan_path.argtypes = [vp, ip, ip]
    lib.ccv3d_plan_path.restype = ctypes.c_int
    lib.ccv3d_forward.argtypes = [vp, vp, vp, vp, vp, vp, vp, ip, ip, ip, vp]
    lib.ccv3d_get_stats.argtypes = [vp, ctypes.POINTER(ccv3d_stats)]
    lib.ccv3d_get_status.argtypes = [vp]
    lib.ccv3d_destroy.argtypes = [vp]
    lib.ccv3d_destroy.restype = None
    lib.ccv3d_strerror.argtypes = [ctypes.c_int]
    lib.ccv3d_strerror.restype = ctypes.c_char_p
    lib.ccv3d_plan_kernel.argtypes = [vp]
    lib.ccv3d_plan_kernel.restype = ctypes.c_char_p
    lib.ccv3d_plan_tiling.argtypes = [vp, ip, ip, ip]
    lib.ccv3d_plan_tiling.restype = ctypes.c_int
    lib.ccv3d_plan_sizes.argtypes = [vp, ctypes.POINTER(ctypes.c_size_t),
                                     ctypes.POINTER(ctypes.c_size_t), ip]
    lib.ccv3d_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.ccv3d_quantize_u8.argtypes = [vp, ctypes.c_int, vp, ctypes.c_longlong, vp]
    lib.ccv3d_quantize_u8.restype = ctypes.c_int
    lib.ccv3d_forward_noalloc.argtypes = [ctypes.POINTER(ccv3d_desc), vp, vp, vp, vp, vp, vp,
                                          ip, ip, ip, vp]
    lib.ccv3d_get_status_stream.argtypes = [vp, vp]
    lib.ccv3d_selftest_bounds.argtypes = [vp]
    lib.ccv3d_selftest_bounds.restype = ctypes.c_int
    lib.ccv3d_noalloc_get_status.argtypes = [vp]
    lib.ccv3d_forward_ring.argtypes = [vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, vp, vp,
                                       ip, ip, ip, vp, ip]
    for f in ("ccv3d_plan", "ccv3d_plan_intervals", "ccv3d_forward", "ccv3d_get_stats",
              "ccv3d_get_status", "ccv3d_plan_sizes", "ccv3d_selftest_wait_timeout",
              "ccv3d_forward_noalloc", "ccv3d_get_status_stream", "ccv3d_noalloc_get_status",
              "ccv3d_forward_ring"):
        getattr(lib, f).restype = ctypes.c_int
    del i3
    return lib


lib = _load()


def _ptr(t) -> int | None:
    """Device address of a tensor (or an int address); None for NULL."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def ccv3d_strerror(status: int) -> str:
    return lib.ccv3d_strerror(int(status)).decode()


def ccv3d_plan(desc: ccv3d_desc) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    rc = lib.ccv3d_plan(ctypes.byref(h), ctypes.byref(desc))
    if rc != 0:
        raise CCV3DError(rc, "ccv3d_plan")
    return h


def ccv3d_plan_intervals(plan) -> dict:
    T_o, H_o, W_o = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    d, lo, hi = (ctypes.c_int * 3)(), (ctypes.c_int * 3)(), (ctypes.c_int * 3)()
    rc = lib.ccv3d_plan_intervals(plan, ctypes.byref(T_o), ctypes.byref(H_o),
                                  ctypes.byref(W_o), d, lo, hi)
    if rc != 0:
        raise CCV3DError(rc, "ccv3d_plan_intervals")
    return {"T_o": T_o.value, "H_o": H_o.value, "W_o": W_o.value,
            "delta": list(d), "o_l": list(lo), "o_h": list(hi)}


def ccv3d_plan_path(plan):
    tm, tn = ctypes.c_int(), ctypes.c_int()
    tc = lib.ccv3d_plan_path(plan, ctypes.byref(tm), ctypes.byref(tn))
    return {"tc": bool(tc == 1), "tile_m": tm.value, "tile_n": tn.value}


def ccv3d_plan_kernel(plan) -> str:
    return lib.ccv3d_plan_kernel(plan).decode()


def ccv3d_plan_tiling(plan) -> dict:
    kb, st, g = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    rc = lib.ccv3d_plan_tiling(plan, ctypes.byref(kb), ctypes.byref(st), ctypes.byref(g))
    if rc not in (0, 2):
        raise CCV3DError(rc, "ccv3d_plan_tiling")
    return {"k_block": kb.value, "stages": st.value, "workspace_pairs": g.value}


def ccv3d_plan_sizes(plan):
    ob, nb, nf = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_int()
    rc = lib.ccv3d_plan_sizes(plan, ctypes.byref(ob), ctypes.byref(nb), ctypes.byref(nf))
    if rc != 0:
        raise CCV3DError(rc, "ccv3d_plan_sizes")
    return {"out_bytes": ob.value, "new_cache_bytes": nb.value, "new_cache_frames": nf.value}


def ccv3d_forward(plan, x, cache, w, bias, out, new_cache, stride, pad, dilation,
                  stream=None, check: bool = True) -> int:
    """One cached causal Conv3D call.  Tensors are device tensors in NTHWC
    physical order (contiguous, or channels_last_3d views) or int addresses.
    Raises CCV3DError on a refused call unless check=False (then returns the
    status code)."""
    s = (ctypes.c_int * 2)(*stride)
    p = (ctypes.c_int * 2)(*pad)
    d = (ctypes.c_int * 3)(*dilation)
    rc = lib.ccv3d_forward(plan, _ptr(x), _ptr(cache), _ptr(w), _ptr(bias), _ptr(out),
                           _ptr(new_cache), s, p, d, _stream(stream))
    if rc != 0 and check:
        raise CCV3DError(rc, "ccv3d_forward")
    return rc


def ccv3d_forward_ring(plan, x, ring, ring_slots: int, head: int, w, bias, out, stride, pad,
                       dilation, stream=None, check: bool = True):
    """The call with its cache in a ring buffer of ring_slots frames per batch
    entry (cache frame t at slot (head + t) % ring_slots).  Writes only the
    arriving frames of the new cache into the ring.  Returns (status,
    next_head); raises CCV3DError on a refused call unless check=False."""
    s = (ctypes.c_int * 2)(*stride)
    p = (ctypes.c_int * 2)(*pad)
    d = (ctypes.c_int * 3)(*dilation)
    nh = ctypes.c_int(-1)
    rc = lib.ccv3d_forward_ring(plan, _ptr(x), _ptr(ring), int(ring_slots), int(head), _ptr(w),
                                _ptr(bias), _ptr(out), s, p, d, _stream(stream),
                                ctypes.byref(nh))
    if rc != 0 and check:
        raise CCV3DError(rc, "ccv3d_forward_ring")
    return rc, nh.value


def ccv3d_forward_noalloc(desc: ccv3d_desc, x, cache, w, bias, out, new_cache, stride, pad,
                          dilation, stream=None, check: bool = True) -> int:
    """The no-allocation variant of ccv3d_forward: no plan, no device memory
    allocated by the library (its scratch is a fixed array inside the shared
    library, shared by all such calls on a device -- they must not overlap on
    the GPU).  For callers that may not allocate device memory."""
    s = (ctypes.c_int * 2)(*stride)
    p = (ctypes.c_int * 2)(*pad)
    d = (ctypes.c_int * 3)(*dilation)
    rc = lib.ccv3d_forward_noalloc(ctypes.byref(desc), _ptr(x), _ptr(cache), _ptr(w), _ptr(bias),
                                   _ptr(out), _ptr(new_cache), s, p, d, _stream(stream))
    if rc != 0 and check:
        raise CCV3DError(rc, "ccv3d_forward_noalloc")
    return rc


def ccv3d_get_stats(plan) -> dict:
    st = ccv3d_stats()
    rc = lib.ccv3d_get_stats(plan, ctypes.byref(st))
    if rc != 0:
        raise CCV3DError(rc, "ccv3d_get_stats")
    return {n: getattr(st, n) for n, _ in ccv3d_stats._fields_}


def ccv3d_get_status(plan) -> int:
    return lib.ccv3d_get_status(plan)


def ccv3d_get_status_stream(plan, stream=None) -> int:
    return lib.ccv3d_get_status_stream(plan, _stream(stream))


def ccv3d_noalloc_get_status(stream=None) -> int:
    return lib.ccv3d_noalloc_get_status(_stream(stream))


def ccv3d_destroy(plan) -> None:
    lib.ccv3d_destroy(plan)


def ccv3d_quantize_u8(x, out, stream=None, check: bool = True) -> int:
    """uint8 frames from decoded values on the device: out = trunc(clamp(
    fp32(x) * 255, 0, 255)), NaN -> 0.  x: a float32 or bfloat16 device
    tensor (any shape, contiguous); out: a uint8 device tensor of as many
    elements.  Raises CCV3DError on a refused call unless check=False."""
    import torch
    dt = {torch.float32: CCV3D_FP32, torch.bfloat16: CCV3D_BF16}.get(x.dtype)
    if dt is None or out.dtype != torch.uint8 or out.numel() != x.numel():
        raise ValueError("ccv3d_quantize_u8: x float32/bfloat16, out uint8 of x.numel()")
    if not (x.is_contiguous() and out.is_contiguous()):
        raise ValueError("ccv3d_quantize_u8: contiguous tensors only")
    rc = lib.ccv3d_quantize_u8(_ptr(x), dt, _ptr(out), x.numel(), _stream(stream))
    if rc != 0 and check:
        raise CCV3DError(rc, "ccv3d_quantize_u8")
    return rc


def ccv3d_selftest_wait_timeout(limit_ns: int, stream=None) -> int:
    return lib.ccv3d_selftest_wait_timeout(int(limit_ns), _stream(stream))


def ccv3d_selftest_bounds(stream=None) -> int:
    return lib.ccv3d_selftest_bounds(_stream(stream))


# ---------------------------------------------------------------- helpers
def make_desc(*, N, Cin, Cout, H, W, T_x, cache_len, kt=3, kh=3, kw=3,
              pad_t_base=None, cache_keep=None, stride=(1, 1), pad=(1, 1),
              dilation=(1, 1, 1), dtype="bf16", has_bias=True, stride_t=1,
              groups=1) -> ccv3d_desc:
    if pad_t_base is None:
        pad_t_base = dilation[0] * (kt - 1)
    if cache_keep is None:
        cache_keep = pad_t_base
    return ccv3d_desc(N, Cin, Cout, kt, kh, kw, H, W, T_x, cache_len, pad_t_base,
                      cache_keep, stride_t, stride[0], stride[1], pad[0], pad[1],
                      dilation[0], dilation[1], dilation[2], groups,
                      CCV3D_BF16 if dtype == "bf16" else CCV3D_FP32, int(bool(has_bias)))


def desc_for(conv) -> ccv3d_desc:
    """Descriptor for a workloads.Conv signature."""
    return make_desc(N=conv.N, Cin=conv.Cin, Cout=conv.Cout, H=conv.H, W=conv.W,
                     T_x=conv.T_x, cache_len=conv.cache_len, kt=conv.kt, kh=conv.kh,
                     kw=conv.kw, pad_t_base=conv.pad_t_base, cache_keep=conv.cache_keep,
                     stride=conv.stride, pad=conv.pad, dilation=conv.dilation,
                     dtype=conv.dtype, has_bias=conv.has_bias, stride_t=conv.stride_t)


class Plan:
    """Owning wrapper of a ccv3d plan handle (destroyed with the object)."""

    def __init__(self, desc: ccv3d_desc):
        self.desc = desc
        self.handle = ccv3d_plan(desc)
        self.intervals = ccv3d_plan_intervals(self.handle)
        self.sizes = ccv3d_plan_sizes(self.handle)
        self.path = ccv3d_plan_path(self.handle)
        self.kernel = ccv3d_plan_kernel(self.handle)
        self.tiling = ccv3d_plan_tiling(self.handle)

    @property
    def stride(self):
        return (self.desc.stride_h, self.desc.stride_w)

    @property
    def pad(self):
        return (self.desc.pad_h, self.desc.pad_w)

    @property
    def dilation(self):
        return (self.desc.dil_t, self.desc.dil_h, self.desc.dil_w)

    def out_shape(self):
        d, iv = self.desc, self.intervals
        return (d.N, iv["T_o"], iv["H_o"], iv["W_o"], d.Cout)

    def new_cache_shape(self):
        d = self.desc
        return (d.N, self.sizes["new_cache_frames"], d.H, d.W, d.Cin)

    def forward(self, x, cache, w, bias, out, new_cache, stream=None):
        return ccv3d_forward(self.handle, x, cache, w, bias, out, new_cache, self.stride,
                             self.pad, self.dilation, stream)

    def forward_ring(self, x, ring, ring_slots, head, w, bias, out, stream=None):
        """Ring-buffer cache call; returns the head of the new cache."""
        return ccv3d_forward_ring(self.handle, x, ring, ring_slots, head, w, bias, out,
                                  self.stride, self.pad, self.dilation, stream)[1]

    def ring_writes(self):
        """Frames of x a ring-buffer call writes into the ring."""
        return min(self.sizes["new_cache_frames"], self.desc.T_x)

    def alloc_outputs(self, device="cuda"):
        import torch
        dt = torch.bfloat16 if self.desc.dtype == CCV3D_BF16 else torch.float32
        out = torch.empty(self.out_shape(), dtype=dt, device=device)
        nc = (torch.empty(self.new_cache_shape(), dtype=dt, device=device)
              if self.sizes["new_cache_frames"] > 0 else None)
        return out, nc

    def stats(self):
        return ccv3d_get_stats(self.handle)

    def status(self):
        return ccv3d_get_status(self.handle)

    def status_stream(self, stream=None):
        return ccv3d_get_status_stream(self.handle, stream)

    def close(self):
        if getattr(self, "handle", None) is not None:
            ccv3d_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
