"""causal_conv3d_video_b200 -- cache-aware causal Conv3D on NVIDIA B200.

The operator and its CUDA kernels live in the shared library built from
``csrc/`` (C ABI: ``include/ccv3d.h``); ``ccv3d`` is its ctypes binding.
Binding names are re-exported lazily so that ``synth`` and ``workloads`` can
be imported on machines where the library has not been built.
"""
import importlib

__all__ = ["ccv3d", "synth", "workloads"]


def __getattr__(name):
    if name in ("ccv3d", "synth", "workloads", "build"):
        return importlib.import_module(f"{__name__}.{name}")
    mod = importlib.import_module(f"{__name__}.ccv3d")
    try:
        return getattr(mod, name)
    except AttributeError:
        raise AttributeError(name) from None
